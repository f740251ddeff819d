"""GPU parity: the CUDA path through the C ABI against the float64 oracle.

Tolerances (normwise relative, max|x - ref| / max|ref|): O and LSE 1e-5 for
fp32 and 2e-2 for bf16; gradients 5e-2; block index lists bit-exact.
Full-size workloads are checked on sampled rows / kv-groups / sequences that
the oracle computes one by one, in the launch configuration the bench times.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from gated_block_sparse_gate_b200 import binding as gb
from gated_block_sparse_gate_b200.build import build
from gated_block_sparse_gate_b200.inputs import WORKLOADS, make_decode_inputs, make_prefill_inputs
from tests.oracle_refs import rel_err

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-5
TOL_BF16 = 2e-2
TOL_GRAD = 5e-2
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    gb.load_library()


def np64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def _small(seed, B, Hq, Hkv, N, d, dtype, scaled, with_grad=True):
    g = torch.Generator().manual_seed(seed)
    scl = d ** -0.5 if scaled else 1.0
    Q = (torch.randn(B, Hq, N, d, generator=g) * scl).to(dtype)
    K = (torch.randn(B, Hkv, N, d, generator=g) * scl).to(dtype)
    V = (torch.randn(B, Hkv, N, d, generator=g) * scl).to(dtype)
    S = torch.randn(B, Hq, N // 64, N // 64, generator=g) * math.sqrt(2)
    dO = torch.randn(B, Hq, N, d, generator=g).to(dtype)
    return dict(Q=Q, K=K, V=V, S=S, dO=dO)


def _dev(x):
    return {k: v.to(DEV) for k, v in x.items()}


# ------------------------------------------------------------------- selection

def test_select_tiny_workload_bit_exact():
    w = WORKLOADS["tiny_f32_n1024"]
    S = make_prefill_inputs(w)["S"]
    for k in (0, 1, 4, 15, 16, 40):
        idx, cnt, logg, slse = gb.select(S.to(DEV), topk=k, mode="sparse")
        ri, rc, rl, rs = oracle.select_blocks(S.numpy(), 16, k)
        assert np.array_equal(idx.cpu().numpy(), ri)
        assert np.array_equal(cnt.cpu().numpy(), rc)
        assert np.max(np.abs(logg.cpu().numpy() - rl), initial=0.0) < 1e-5
    _, _, _, slse = gb.select(S.to(DEV), mode="train")
    _, _, _, rs = oracle.select_blocks(S.numpy(), 16, None, mode=oracle.TRAIN)
    fin = np.isfinite(rs)
    assert np.array_equal(np.isfinite(slse.cpu().numpy()), fin)
    assert np.max(np.abs(slse.cpu().numpy()[fin] - rs[fin])) < 1e-5


def test_select_ties_and_signed_zero_bit_exact():
    g = torch.Generator().manual_seed(123)
    S = torch.randint(-2, 3, (2, 3, 70, 70), generator=g).float()
    S[torch.rand(S.shape, generator=g) < 0.2] = -0.0
    for k in (1, 3, 7, 33, 69, 200):
        idx, cnt, _, _ = gb.select(S.to(DEV), topk=k, mode="sparse")
        ri, rc, _, _ = oracle.select_blocks(S.numpy(), 70, k)
        assert np.array_equal(idx.cpu().numpy(), ri), k
        assert np.array_equal(cnt.cpu().numpy(), rc), k


@pytest.mark.parametrize("k", [8, 16, 32, 64])
def test_select_sparse_prefill_full_size_sampled(k):
    """Planted-score workload (N=65536, 1024 blocks per row), sampled rows."""
    w = WORKLOADS["sparse_prefill_bf16_n65536"]
    S = make_prefill_inputs(w, with_grad=False)["S"]
    idx, cnt, logg, _ = gb.select(S.to(DEV), topk=k, mode="sparse")
    idx, cnt, logg = idx.cpu().numpy(), cnt.cpu().numpy(), logg.cpu().numpy()
    rng = np.random.default_rng(k)
    Sn = S.numpy()
    for h in (0, 13, 31):
        for r in list(rng.integers(0, 1024, 40)) + [0, 1, k - 1, k, k + 1, 1023]:
            A = oracle.attended_blocks(Sn[0, h, r], r, oracle.SPARSE, k)
            assert cnt[0, h, r] == len(A)
            assert np.array_equal(idx[0, h, r, :len(A)], A)
            assert np.all(idx[0, h, r, len(A):] == -1)
            lg = oracle.log_gates(Sn[0, h, r], A, r)
            assert np.max(np.abs(logg[0, h, r, :len(A)] - lg), initial=0) < 1e-5


# ------------------------------------------------------------ threshold select
# The kernel decides S[r,c] - lse_r >= ln(tau) in fp32, the oracle in float64;
# they can only disagree for a gate within rounding of tau. Rows with a gate
# within THR_BAND (in log units) of ln(tau) are "boundary" rows: there the
# kernel's count must lie between the two oracle counts of the band's edges and
# its list must be the oracle's Top-k for that count; elsewhere bit-exact.
# A row with one historical block has gate exactly 1 on both sides (its
# log-sum-exp is the score itself), so it is never a boundary row.
THR_BAND = 1e-4


def _is_boundary(s, r, tau):
    return r > 1 and (oracle.threshold_count(s, r, tau * math.exp(THR_BAND))
                      != oracle.threshold_count(s, r, tau * math.exp(-THR_BAND)))


def _threshold_rows_agree(Sn, idx, cnt, logg, k, tau, rows):
    n_boundary = 0
    for b, h, r in rows:
        s = Sn[b, h, r]
        lo = min(k, oracle.threshold_count(s, r, tau * math.exp(THR_BAND)))
        hi = min(k, oracle.threshold_count(s, r, tau * math.exp(-THR_BAND)))
        want = min(k, oracle.threshold_count(s, r, tau))
        got = int(cnt[b, h, r])
        if _is_boundary(s, r, tau) and lo != hi:
            n_boundary += 1
            assert lo <= got <= hi, (b, h, r, lo, got, hi)
        else:
            assert got == want, (b, h, r, got, want)
        A = oracle.attended_blocks(s, r, oracle.SPARSE, got)
        assert np.array_equal(idx[b, h, r, :got], A), (b, h, r)
        assert np.all(idx[b, h, r, got:] == -1)
        lg = oracle.log_gates(s, A, r)
        assert np.max(np.abs(logg[b, h, r, :got] - lg), initial=0) < 1e-5
    return n_boundary


@pytest.mark.parametrize("tau", [1e-3, 0.02, 0.1, 0.5, 1.0])
def test_select_threshold_tiny_workload(tau):
    w = WORKLOADS["tiny_f32_n1024"]
    S = make_prefill_inputs(w)["S"]
    Sn = S.numpy()
    rows = [(b, h, r) for b in range(S.shape[0]) for h in range(S.shape[1]) for r in range(16)]
    for k in (0, 1, 3, 16):
        idx, cnt, logg, _ = gb.select(S.to(DEV), topk=k, mode="threshold", tau=tau)
        nb = _threshold_rows_agree(Sn, idx.cpu().numpy(), cnt.cpu().numpy(), logg.cpu().numpy(),
                                   k, tau, rows)
        assert nb == 0, nb  # this seed has no gate within the band of these taus


@pytest.mark.parametrize("tau,k", [(0.01, 64), (0.002, 32), (0.05, 8)])
def test_select_threshold_full_size_sampled(tau, k):
    """Planted-score prefill workload (N=65536): sampled rows, threshold mode."""
    w = WORKLOADS["sparse_prefill_bf16_n65536"]
    S = make_prefill_inputs(w, with_grad=False)["S"]
    idx, cnt, logg, _ = gb.select(S.to(DEV), topk=k, mode="threshold", tau=tau)
    rng = np.random.default_rng(int(tau * 1e4) + k)
    rows = [(0, h, int(r)) for h in (0, 13, 31)
            for r in list(rng.integers(0, 1024, 40)) + [0, 1, 2, 50, 1023]]
    nb = _threshold_rows_agree(S.numpy(), idx.cpu().numpy(), cnt.cpu().numpy(),
                               logg.cpu().numpy(), k, tau, rows)
    assert nb <= 2, nb
    kept = cnt.cpu().numpy()[0, :, 64:]
    assert kept.min() < min(k, 64) or tau <= 0.002  # the threshold does prune


# ---------------------------------------------------------------------- forward

def _check_fwd(x, mode, k, tol, rows=None, tau=None):
    Qd, Kd, Vd, Sd = (x[n].to(DEV) for n in "QKVS")
    O, LSE = gb.forward(Qd, Kd, Vd, Sd, mode=mode, topk=k, tau=0.0 if tau is None else tau)
    torch.cuda.synchronize()
    Or, Lr = oracle.gated_attention_forward(np64(x["Q"]), np64(x["K"]), np64(x["V"]), x["S"].numpy(),
                                            64, mode=mode, topk=k, rows=rows, tau=tau)
    eo, el = rel_err(np64(O), Or), rel_err(LSE.cpu().numpy(), Lr)
    assert eo < tol and el < tol, (eo, el)
    return eo, el


def test_fwd_tiny_f32_train_and_sparse():
    x = make_prefill_inputs(WORKLOADS["tiny_f32_n1024"])
    _check_fwd(x, "train", 0, TOL_F32)
    _check_fwd(x, "sparse", 4, TOL_F32)


@pytest.mark.parametrize("mode,k", [("train", 0), ("sparse", 0), ("sparse", 3), ("sparse", 100)])
@pytest.mark.parametrize("scaled", [True, False])
def test_fwd_bf16_small(mode, k, scaled):
    x = _small(7, 1, 8, 2, 1024, 128, torch.bfloat16, scaled)
    _check_fwd(x, mode, k, TOL_BF16)


@pytest.mark.parametrize("shape", [
    (1, 2, 2, 64, 128),    # one block: no history
    (2, 4, 4, 320, 64),    # odd block count, MHA, d=64
    (1, 4, 1, 448, 128),   # GQA 4:1, 7 blocks
])
@pytest.mark.parametrize("mode,k", [("train", 0), ("sparse", 2)])
def test_fwd_edge_shapes(shape, mode, k):
    B, Hq, Hkv, N, d = shape
    for dtype, tol in ((torch.bfloat16, TOL_BF16), (torch.float32, TOL_F32)):
        x = _small(11, B, Hq, Hkv, N, d, dtype, scaled=False)
        _check_fwd(x, mode, k, tol)


@pytest.mark.parametrize("shape,k", [
    ((1, 4, 2, 320, 128), 2),    # odd block count, two q-heads per kv-head pair
    ((2, 8, 2, 448, 64), 3),     # d = 64, G = 4
    ((1, 4, 2, 512, 128), 0),    # current block only
    ((1, 4, 2, 512, 128), 100),  # full budget: equals training mode
    ((1, 8, 4, 1024, 128), 5),
])
@pytest.mark.parametrize("scaled", [True, False])
def test_fwd_sparse_two_tile_kernel(shape, k, scaled):
    """Sparse mode with an even q-heads-per-kv-head ratio (two tiles per CTA)."""
    B, Hq, Hkv, N, d = shape
    x = _small(23 + k, B, Hq, Hkv, N, d, torch.bfloat16, scaled)
    _check_fwd(x, "sparse", k, TOL_BF16)


def test_fwd_sparse_full_budget_matches_training():
    x = _small(29, 1, 4, 2, 512, 128, torch.bfloat16, False)
    Qd, Kd, Vd, Sd = (x[n].to(DEV) for n in "QKVS")
    Ot, Lt = gb.forward(Qd, Kd, Vd, Sd, mode="train")
    Os, Ls = gb.forward(Qd, Kd, Vd, Sd, mode="sparse", topk=8)
    torch.cuda.synchronize()
    assert rel_err(np64(Os), np64(Ot)) < 1e-2 and rel_err(Ls.cpu().numpy(), Lt.cpu().numpy()) < 1e-5


def _no_boundary_gates(S, tau):
    """True when no gate of S lies within THR_BAND of tau (log units)."""
    Sn = S.numpy()
    B, H, Nb, _ = Sn.shape
    return not any(_is_boundary(Sn[b, h, r], r, tau)
                   for b in range(B) for h in range(H) for r in range(Nb))


@pytest.mark.parametrize("shape,k,tau", [
    ((1, 8, 2, 1024, 128), 6, 0.05),   # two tiles per CTA (G even)
    ((2, 4, 4, 320, 64), 3, 0.2),      # G = 1: one tile per CTA
    ((1, 4, 1, 448, 128), 100, 0.1),   # budget above every count: threshold alone
    ((1, 4, 2, 512, 128), 4, 1.0),     # only a sole historical block passes
])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_fwd_threshold(shape, k, tau, dtype):
    B, Hq, Hkv, N, d = shape
    x = _small(41 + k, B, Hq, Hkv, N, d, dtype, scaled=True)
    assert _no_boundary_gates(x["S"], tau)
    _check_fwd(x, "threshold", k, TOL_F32 if dtype == torch.float32 else TOL_BF16, tau=tau)


def test_fwd_threshold_tiny_tau_equals_training():
    x = _small(43, 1, 4, 2, 512, 128, torch.bfloat16, False)
    Qd, Kd, Vd, Sd = (x[n].to(DEV) for n in "QKVS")
    Ot, Lt = gb.forward(Qd, Kd, Vd, Sd, mode="train")
    Os, Ls = gb.forward(Qd, Kd, Vd, Sd, mode="threshold", topk=8, tau=1e-30)
    torch.cuda.synchronize()
    assert rel_err(np64(Os), np64(Ot)) < 1e-2 and rel_err(Ls.cpu().numpy(), Lt.cpu().numpy()) < 1e-5


def test_fwd_train_full_size_sampled():
    """Training workload N=8192, 32/8 heads, bf16: sampled query blocks."""
    w = WORKLOADS["train_bf16_n8192"]
    x = make_prefill_inputs(w, with_grad=False)
    rng = np.random.default_rng(8192)
    rows = [(0, h, int(r)) for h in (0, 5, 13, 22, 31)
            for r in [0, 1, 2, 63, 64, 100, 126, 127] + list(rng.integers(0, 128, 4))]
    _check_fwd(x, "train", 0, TOL_BF16, rows=rows)


def test_fwd_train_long_context_sampled():
    """Long-context training workload N=32768 (512 blocks), 32/8 heads, bf16,
    in the bench's launch configuration: sampled query blocks of several heads
    (first blocks, the middle, the heaviest last ones)."""
    w = WORKLOADS["train_bf16_n32768"]
    x = make_prefill_inputs(w, with_grad=False)
    rng = np.random.default_rng(32768)
    rows = [(0, h, int(r)) for h in (0, 3, 12, 21, 31)
            for r in [0, 1, 255, 256, 510, 511] + list(rng.integers(0, 512, 3))]
    _check_fwd(x, "train", 0, TOL_BF16, rows=rows)


@pytest.mark.parametrize("k", [8, 16, 32, 64])
def test_fwd_sparse_prefill_full_size_sampled(k):
    """Planted prefill workload N=65536, Top-K: sampled query blocks of four heads."""
    w = WORKLOADS["sparse_prefill_bf16_n65536"]
    x = make_prefill_inputs(w, with_grad=False)
    rng = np.random.default_rng(65536 + k)
    rows = [(0, h, int(r)) for h in (0, 9, 17, 30)
            for r in [0, 1, 5, k - 1, k, k + 1, 300, 511, 512, 1022, 1023]
            + list(rng.integers(0, 1024, 4))]
    _check_fwd(x, "sparse", k, TOL_BF16, rows=rows)


def test_fwd_threshold_prefill_full_size_sampled():
    """Planted prefill workload N=65536, threshold tau = 0.01 with at most 64
    blocks (the bench's threshold case): sampled rows away from the tau band."""
    w = WORKLOADS["sparse_prefill_bf16_n65536"]
    x = make_prefill_inputs(w, with_grad=False)
    Sn = x["S"].numpy()
    rng = np.random.default_rng(7)
    rows = [(0, h, int(r)) for h in (2, 19)
            for r in [0, 1, 2, 64, 700, 1023] + list(rng.integers(0, 1024, 6))]
    rows = [t for t in rows if not _is_boundary(Sn[t[0], t[1], t[2]], t[2], 0.01)]
    _check_fwd(x, "threshold", 64, TOL_BF16, rows=rows, tau=0.01)


@pytest.mark.parametrize("k", [1, 2, 8, 16, 31])
def test_fwd_sparse_budgets(k):
    """Top-K budgets with odd and even list lengths (the kernel attends two
    blocks per stage and pads an odd count), 32 blocks per head."""
    x = _small(71 + k, 2, 4, 2, 2048, 128, torch.bfloat16, scaled=False)
    _check_fwd(x, "sparse", k, TOL_BF16)


@pytest.mark.parametrize("mode,k", [("sparse", 5), ("sparse", 12), ("train", 0)])
def test_fwd_large_logits(mode, k):
    """Logits with a spread of tens (queries scaled by 6, scores by 4): row
    maxima move by more than 2^8 between stages, so the online-softmax rescale
    of O and of the row sums runs many times per row."""
    x = _small(83 + k, 1, 4, 2, 1536, 128, torch.bfloat16, scaled=False)
    x["Q"] = (x["Q"].float() * 6).to(torch.bfloat16)
    x["S"] = x["S"] * 4
    _check_fwd(x, mode, k, TOL_BF16)


# --------------------------------------------------------------------- backward

def _check_bwd(x, tol, heads=None, mode="train", k=0, tau=None):
    d = _dev(x)
    tv = 0.0 if tau is None else tau
    O, LSE = gb.forward(d["Q"], d["K"], d["V"], d["S"], mode=mode, topk=k, tau=tv)
    dQ, dK, dV, dS = gb.backward(d["Q"], d["K"], d["V"], d["S"], O, LSE, d["dO"], mode=mode,
                                 topk=k, tau=tv)
    torch.cuda.synchronize()
    ref = oracle.gated_attention_backward(np64(x["Q"]), np64(x["K"]), np64(x["V"]), x["S"].numpy(),
                                          np64(x["dO"]), 64, heads=heads, mode=mode, topk=k, tau=tau)
    errs = {n: rel_err(np64(t) if t.dtype != torch.float32 else t.cpu().numpy().astype(np.float64), r)
            for n, t, r in zip(("dQ", "dK", "dV", "dS"), (dQ, dK, dV, dS), ref[:4])}
    for n, e in errs.items():
        assert e < tol, (n, errs)
    return errs


def test_bwd_tiny_f32():
    errs = _check_bwd(make_prefill_inputs(WORKLOADS["tiny_f32_n1024"]), TOL_GRAD)
    assert max(errs.values()) < 1e-4, errs  # the fp32 path is far inside the bound


@pytest.mark.parametrize("scaled", [True, False])
def test_bwd_bf16_small(scaled):
    _check_bwd(_small(5, 1, 8, 2, 1024, 128, torch.bfloat16, scaled), TOL_GRAD)


@pytest.mark.parametrize("shape", [(1, 2, 2, 64, 128), (2, 4, 4, 320, 64), (1, 4, 1, 448, 128)])
def test_bwd_edge_shapes(shape):
    B, Hq, Hkv, N, d = shape
    for dtype in (torch.bfloat16, torch.float32):
        _check_bwd(_small(3, B, Hq, Hkv, N, d, dtype, scaled=False), TOL_GRAD)


# Sparse and threshold backward: gradients through the gates renormalised over
# the kept blocks; blocks outside A_r get dS = 0.

def test_bwd_sparse_tiny_f32():
    errs = _check_bwd(make_prefill_inputs(WORKLOADS["tiny_f32_n1024"]), TOL_GRAD, mode="sparse", k=4)
    assert max(errs.values()) < 1e-4, errs


@pytest.mark.parametrize("k", [0, 3, 100])
@pytest.mark.parametrize("scaled", [True, False])
def test_bwd_sparse_bf16_small(k, scaled):
    _check_bwd(_small(13 + k, 1, 8, 2, 1024, 128, torch.bfloat16, scaled), TOL_GRAD,
               mode="sparse", k=k)


@pytest.mark.parametrize("shape", [(1, 2, 2, 64, 128), (2, 4, 4, 320, 64), (1, 4, 1, 448, 128),
                                   (1, 8, 2, 1344, 64)])
def test_bwd_sparse_edge_shapes(shape):
    B, Hq, Hkv, N, d = shape
    for dtype in (torch.bfloat16, torch.float32):
        _check_bwd(_small(17, B, Hq, Hkv, N, d, dtype, scaled=False), TOL_GRAD, mode="sparse", k=2)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_bwd_threshold_small(dtype):
    x = _small(47, 1, 8, 2, 1024, 128, dtype, scaled=True)
    assert _no_boundary_gates(x["S"], 0.05)
    _check_bwd(x, TOL_GRAD, mode="threshold", k=6, tau=0.05)


def test_bwd_sparse_full_budget_matches_training():
    x = _dev(_small(53, 1, 4, 2, 512, 128, torch.bfloat16, False))
    O, LSE = gb.forward(x["Q"], x["K"], x["V"], x["S"], mode="train")
    gt = gb.backward(x["Q"], x["K"], x["V"], x["S"], O, LSE, x["dO"])
    gs = gb.backward(x["Q"], x["K"], x["V"], x["S"], O, LSE, x["dO"], mode="sparse", topk=8)
    torch.cuda.synchronize()
    for a, b in zip(gt, gs):  # the two normalisers may differ in the last fp32 bit
        assert rel_err(np64(b), np64(a)) < 1e-2


@pytest.mark.parametrize("k", [8, 16, 32, 64])
def test_bwd_sparse_prefill_full_size_one_group(k):
    """Planted prefill workload N=65536, 32/8 heads, sparse K, computed in full
    on the GPU; every gradient of kv-group 0 against the oracle."""
    w = WORKLOADS["sparse_prefill_bf16_n65536"]
    x = make_prefill_inputs(w)
    d = _dev(x)
    O, LSE = gb.forward(d["Q"], d["K"], d["V"], d["S"], mode="sparse", topk=k)
    dQ, dK, dV, dS = gb.backward(d["Q"], d["K"], d["V"], d["S"], O, LSE, d["dO"], mode="sparse",
                                 topk=k)
    torch.cuda.synchronize()
    G = w.Hq // w.Hkv
    ref = oracle.gated_attention_backward(np64(x["Q"][:, :G]), np64(x["K"][:, :1]),
                                          np64(x["V"][:, :1]), x["S"][:, :G].numpy(),
                                          np64(x["dO"][:, :G]), 64, mode="sparse", topk=k)
    got = (dQ[:, :G], dK[:, :1], dV[:, :1], dS[:, :G])
    for n, t, r in zip(("dQ", "dK", "dV", "dS"), got, ref[:4]):
        e = rel_err(t.float().cpu().numpy().astype(np.float64), r)
        assert e < TOL_GRAD, (n, e)


def test_bwd_train_full_size_one_group():
    """Training workload N=8192, 32/8 heads: all gradients of kv-group 0."""
    w = WORKLOADS["train_bf16_n8192"]
    _check_bwd(make_prefill_inputs(w), TOL_GRAD, heads=[(0, 0)])


def test_bwd_train_long_context_one_group():
    """Long-context training workload N=32768 (512 blocks), 32/8 heads, bf16,
    computed in full on the GPU in the bench's launch configuration: every
    gradient of kv group 0 (q-heads 0-3; dS over 512 x 512 blocks) against the
    oracle."""
    w = WORKLOADS["train_bf16_n32768"]
    x = make_prefill_inputs(w)
    d = _dev(x)
    O, LSE = gb.forward(d["Q"], d["K"], d["V"], d["S"], mode="train")
    dQ, dK, dV, dS = gb.backward(d["Q"], d["K"], d["V"], d["S"], O, LSE, d["dO"])
    torch.cuda.synchronize()
    G = w.Hq // w.Hkv
    got = [t.float().cpu().numpy().astype(np.float64)
           for t in (dQ[:, :G], dK[:, :1], dV[:, :1], dS[:, :G])]
    del d, O, LSE, dQ, dK, dV, dS
    torch.cuda.empty_cache()
    ref = oracle.gated_attention_backward(np64(x["Q"][:, :G]), np64(x["K"][:, :1]),
                                          np64(x["V"][:, :1]), x["S"][:, :G].numpy(),
                                          np64(x["dO"][:, :G]), 64)
    for n, t, r in zip(("dQ", "dK", "dV", "dS"), got, ref[:4]):
        e = rel_err(t, r)
        assert e < TOL_GRAD, (n, e)


# ----------------------------------------------------------------------- decode

def _check_decode(x, L, k, tol, seqs, num_splits=0, tau=None):
    O, LSE = gb.decode(x["q"].to(DEV), x["Kc"].to(DEV), x["Vc"].to(DEV), x["S"].to(DEV), L=L,
                       topk=k, num_splits=num_splits, tau=tau)
    torch.cuda.synchronize()
    Kc = x["Kc"][seqs].cpu() if x["Kc"].is_cuda else x["Kc"][seqs]
    Vc = x["Vc"][seqs].cpu() if x["Vc"].is_cuda else x["Vc"][seqs]
    mode = oracle.SPARSE if tau is None else oracle.THRESHOLD
    Or, Lr = oracle.gated_decode(np64(x["q"][seqs]), np64(Kc), np64(Vc), x["S"][seqs].cpu().numpy(),
                                 L, 64, k, mode=mode, tau=tau)
    eo = rel_err(np64(O[seqs]), Or)
    el = rel_err(LSE[seqs].cpu().numpy(), Lr)
    assert eo < tol and el < tol, (eo, el)


@pytest.mark.parametrize("L", [64, 4096, 4133])
@pytest.mark.parametrize("splits", [0, 1, 3])
def test_decode_small(L, splits):
    from dataclasses import replace
    w = replace(WORKLOADS["sparse_decode_bf16_b64_l131072"], B=4, N=L)
    x = make_decode_inputs(w, B=4, L=L)
    _check_decode(x, L, 8, TOL_BF16, seqs=[0, 1, 2, 3], num_splits=splits)


def test_decode_f32_small():
    from dataclasses import replace
    w = replace(WORKLOADS["sparse_decode_bf16_b64_l131072"], B=2, N=2000, dtype="f32")
    x = make_decode_inputs(w, B=2, L=2000)
    _check_decode(x, 2000, 5, TOL_F32, seqs=[0, 1])


@pytest.mark.parametrize("tau,k", [(0.01, 64), (0.05, 8), (1e-30, 256)])
def test_decode_threshold_small(tau, k):
    from dataclasses import replace
    L = 8133
    w = replace(WORKLOADS["sparse_decode_bf16_b64_l131072"], B=4, N=L)
    x = make_decode_inputs(w, B=4, L=L)
    cur = (L - 1) // 64
    Sn = x["S"].numpy()
    assert not any(_is_boundary(Sn[b, h], cur, tau) for b in range(4) for h in range(Sn.shape[1]))
    _check_decode(x, L, k, TOL_BF16, seqs=[0, 1, 2, 3], tau=tau)


def test_decode_full_size_sampled():
    """64 sequences x 131072 cache, K=32: sampled sequences against the oracle."""
    w = WORKLOADS["sparse_decode_bf16_b64_l131072"]
    x = make_decode_inputs(w, device=DEV)
    _check_decode(x, w.N, 32, TOL_BF16, seqs=[0, 37, 63])
    del x
    torch.cuda.empty_cache()


# ------------------------------------------------------------------ determinism

def test_run_to_run_determinism():
    """Forward and decode have no atomics: their outputs repeat bit for bit.
    In the backward dK and dV accumulate inside one CTA (bitwise too); dQ and the
    tile sums behind dS are summed across CTAs in hardware order, so they repeat
    to within fp32 rounding: dS (fp32) to 1e-5, and dQ, that fp32 sum rounded
    once to bf16, to within one bf16 ulp of each element plus the fp32 rounding
    of the sum itself, which an element that cancels can expose (2^-16 of the
    largest |dQ| here: 16 key tiles, each change of order worth a few fp32 ulps
    of the partial sums)."""
    x = _dev(_small(61, 1, 8, 2, 1024, 128, torch.bfloat16, scaled=False))
    for mode, k in (("train", 0), ("sparse", 3)):
        O1, L1 = gb.forward(x["Q"], x["K"], x["V"], x["S"], mode=mode, topk=k)
        O2, L2 = gb.forward(x["Q"], x["K"], x["V"], x["S"], mode=mode, topk=k)
        assert torch.equal(O1, O2) and torch.equal(L1, L2), mode
        g1 = gb.backward(x["Q"], x["K"], x["V"], x["S"], O1, L1, x["dO"], mode=mode, topk=k)
        g2 = gb.backward(x["Q"], x["K"], x["V"], x["S"], O1, L1, x["dO"], mode=mode, topk=k)
        assert torch.equal(g1[1], g2[1]) and torch.equal(g1[2], g2[2]), mode
        a, b = np64(g1[0]), np64(g2[0])
        floor = 2.0 ** -16 * max(np.abs(a).max(), np.abs(b).max())
        assert np.all(np.abs(a - b) <= 2.0 ** -8 * np.maximum(np.abs(a), np.abs(b)) + floor), mode
        assert rel_err(np64(g1[3]), np64(g2[3])) < 1e-5, mode
    from dataclasses import replace
    w = replace(WORKLOADS["sparse_decode_bf16_b64_l131072"], B=4, N=5000)
    d = {n: t.to(DEV) for n, t in make_decode_inputs(w, B=4, L=5000).items()}
    r1 = gb.decode(d["q"], d["Kc"], d["Vc"], d["S"], topk=16)
    r2 = gb.decode(d["q"], d["Kc"], d["Vc"], d["S"], topk=16)
    assert torch.equal(r1[0], r2[0]) and torch.equal(r1[1], r2[1])
