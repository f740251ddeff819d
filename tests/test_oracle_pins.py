"""Pins for the float64 oracle: results fixed by mathematics or by library routines.

Each test ties the oracle to something other than itself: torch SDPA and
autograd, central finite differences, closed forms derived by hand, brute-force
rank counting, and invariants of the softmax. The mutation tests at the end
plant plausible mistakes in copies of the oracle and check that a pin fails.
"""
import inspect
import math
import types

import numpy as np
import pytest

import oracle
from oracle import gated_attention as ga
from tests.oracle_refs import rel_err, sdpa_dense_causal, sdpa_gated

TOL = 1e-10


def _rand(seed, B, Hq, Hkv, N, d, block, s_std=math.sqrt(2.0), qkv_std=1.0):
    rng = np.random.default_rng(seed)
    Nb = -(-N // block)
    Q = rng.standard_normal((B, Hq, N, d)) * qkv_std
    K = rng.standard_normal((B, Hkv, N, d)) * qkv_std
    V = rng.standard_normal((B, Hkv, N, d))
    S = rng.standard_normal((B, Hq, Nb, Nb)) * s_std
    dO = rng.standard_normal((B, Hq, N, d))
    return Q, K, V, S, dO


# ---------------------------------------------------------------- textbook cases

@pytest.mark.parametrize("shape", [(1, 2, 2, 64, 16, 16), (2, 4, 2, 48, 8, 8), (1, 2, 1, 40, 8, 16)])
def test_gates_one_is_dense_causal(shape):
    """Gates forced to 1 with every block kept reduces to dense causal attention."""
    B, Hq, Hkv, N, d, bs = shape
    Q, K, V, S, _ = _rand(1, B, Hq, Hkv, N, d, bs)
    O, LSE = oracle.gated_attention_forward(Q, K, V, S, bs, gate="ones")
    O_ref, LSE_ref = sdpa_dense_causal(Q, K, V)
    assert rel_err(O, O_ref) < TOL
    assert rel_err(LSE, LSE_ref) < TOL


def test_single_block_is_dense_causal():
    """block = N: there is no history, so the method is plain causal attention."""
    Q, K, V, _, dO = _rand(2, 1, 2, 2, 32, 8, 32)
    S = np.random.default_rng(3).standard_normal((1, 2, 1, 1))
    O, LSE = oracle.gated_attention_forward(Q, K, V, S, 32)
    O_ref, LSE_ref = sdpa_dense_causal(Q, K, V)
    assert rel_err(O, O_ref) < TOL and rel_err(LSE, LSE_ref) < TOL
    *_, dS, _ = oracle.gated_attention_backward(Q, K, V, S, dO, 32)
    assert np.all(dS == 0.0)


def test_constant_scores_give_uniform_gates():
    """A constant score row gives g = 1/|A|, i.e. log-gate -ln r (train) or -ln K."""
    S = np.full((1, 1, 9, 9), 0.7)
    idx, cnt, logg, _ = oracle.select_blocks(S, 9, None, mode=oracle.TRAIN)
    for r in range(1, 9):
        assert np.allclose(logg[0, 0, r, :r], -math.log(r), atol=1e-15)
    idx, cnt, logg, _ = oracle.select_blocks(S, 9, 3, mode=oracle.SPARSE)
    for r in range(4, 9):
        assert cnt[0, 0, r] == 3
        assert list(idx[0, 0, r, :3]) == [0, 1, 2]  # ties resolve to the lowest indices
        assert np.allclose(logg[0, 0, r, :3], -math.log(3), atol=1e-15)


# ------------------------------------------------------------ library cross-check

CASES = [
    # B, Hq, Hkv, N, d, block
    (1, 2, 2, 64, 16, 16),
    (1, 4, 2, 96, 8, 16),
    (2, 2, 1, 40, 8, 16),    # ragged last block
    (1, 2, 2, 24, 4, 1),     # per-token context units
]


@pytest.mark.parametrize("case", CASES)
def test_train_matches_sdpa_autograd(case):
    B, Hq, Hkv, N, d, bs = case
    Q, K, V, S, dO = _rand(10 + N, B, Hq, Hkv, N, d, bs)
    O, LSE = oracle.gated_attention_forward(Q, K, V, S, bs)
    dQ, dK, dV, dS, _ = oracle.gated_attention_backward(Q, K, V, S, dO, bs)
    ref = sdpa_gated(Q, K, V, S, bs, dO=dO)
    for name, x in dict(O=O, LSE=LSE, dQ=dQ, dK=dK, dV=dV, dS=dS).items():
        assert rel_err(x, ref[name]) < 1e-9, name


@pytest.mark.parametrize("renormalise", [True, False])
@pytest.mark.parametrize("topk", [0, 1, 3])
def test_sparse_matches_sdpa_autograd(topk, renormalise):
    B, Hq, Hkv, N, d, bs = 1, 4, 2, 128, 8, 16
    Q, K, V, S, dO = _rand(20 + topk, B, Hq, Hkv, N, d, bs)
    kw = dict(mode=oracle.SPARSE, topk=topk, renormalise=renormalise)
    O, LSE = oracle.gated_attention_forward(Q, K, V, S, bs, **kw)
    dQ, dK, dV, dS, _ = oracle.gated_attention_backward(Q, K, V, S, dO, bs, **kw)
    ref = sdpa_gated(Q, K, V, S, bs, mode="sparse", topk=topk, renormalise=renormalise, dO=dO)
    for name, x in dict(O=O, LSE=LSE, dQ=dQ, dK=dK, dV=dV, dS=dS).items():
        assert rel_err(x, ref[name]) < 1e-9, name


@pytest.mark.parametrize("tau,topk", [(0.05, 3), (0.15, 8), (0.3, 5)])
def test_threshold_matches_sdpa_autograd(tau, topk):
    """Threshold selection (gate over the whole history >= tau, at most topk
    blocks) with gates renormalised over the kept set: forward and all four
    gradients against SDPA + autograd with the mask built by torch."""
    B, Hq, Hkv, N, d, bs = 1, 4, 2, 160, 8, 16
    Q, K, V, S, dO = _rand(40 + topk, B, Hq, Hkv, N, d, bs)
    kw = dict(mode=oracle.THRESHOLD, topk=topk, tau=tau)
    O, LSE = oracle.gated_attention_forward(Q, K, V, S, bs, **kw)
    dQ, dK, dV, dS, _ = oracle.gated_attention_backward(Q, K, V, S, dO, bs, **kw)
    ref = sdpa_gated(Q, K, V, S, bs, mode="threshold", topk=topk, tau=tau, dO=dO)
    for name, x in dict(O=O, LSE=LSE, dQ=dQ, dK=dK, dV=dV, dS=dS).items():
        assert rel_err(x, ref[name]) < 1e-9, name
    # the threshold must bind on some rows and the budget on others
    _, cnt, _, _ = oracle.select_blocks(S, N // bs, topk, mode=oracle.THRESHOLD, tau=tau)
    r = np.arange(N // bs)
    assert (cnt < np.minimum(topk, r)).any()


# ---------------------------------------------------------- finite differences

def _fd_check(Q, K, V, S, bs, W, n_pick=24, seed=0, eps=1e-6, bwd=None):
    bwd = bwd or oracle.gated_attention_backward
    rng = np.random.default_rng(seed)

    def loss(Q_, K_, V_, S_):
        O, _ = oracle.gated_attention_forward(Q_, K_, V_, S_, bs)
        return float(np.sum(W * O))

    dQ, dK, dV, dS, _ = bwd(Q, K, V, S, W, bs)
    worst = 0.0
    for name, X, dX in (("Q", Q, dQ), ("K", K, dK), ("V", V, dV), ("S", S, dS)):
        flat = np.flatnonzero(np.ones(X.shape, dtype=bool))
        if name == "S":  # only historical entries (c < r) feed the method
            r = np.arange(X.shape[2])[:, None]
            c = np.arange(X.shape[3])[None, :]
            flat = np.flatnonzero(np.broadcast_to(c < r, X.shape))
        pick = rng.choice(flat, size=min(n_pick, flat.size), replace=False)
        for f in pick:
            ix = np.unravel_index(f, X.shape)
            args = {"Q": Q, "K": K, "V": V, "S": S}
            Xp = X.copy(); Xp[ix] += eps
            Xm = X.copy(); Xm[ix] -= eps
            args[name] = Xp; lp = loss(**{k + "_": v for k, v in args.items()})
            args[name] = Xm; lm = loss(**{k + "_": v for k, v in args.items()})
            num = (lp - lm) / (2 * eps)
            worst = max(worst, abs(num - dX[ix]) / max(1.0, abs(num)))
    return worst


def test_finite_differences_tiny():
    """dQ, dK, dV and dS agree with central differences (N=32, d=8, block=4)."""
    Q, K, V, S, W = _rand(5, 1, 2, 1, 32, 8, 4)
    assert _fd_check(Q, K, V, S, 4, W) < 1e-6


# -------------------------------------------------------------------- invariants

def test_gate_rows_sum_to_one():
    S = np.random.default_rng(7).standard_normal((2, 3, 12, 12)) * math.sqrt(2)
    for mode, k in ((oracle.TRAIN, None), (oracle.SPARSE, 4)):
        idx, cnt, logg, _ = oracle.select_blocks(S, 12, k, mode=mode)
        for b in range(2):
            for h in range(3):
                for r in range(1, 12):
                    n = cnt[b, h, r]
                    assert abs(np.exp(logg[b, h, r, :n]).sum() - 1.0) < 1e-14


def _slse_pin_error(select):
    """Largest deviation of select_blocks' slse from the log-normaliser of the
    training gates as torch.log_softmax computes it over each row's history
    c < r (HF page Abstract: gates normalised over the historical blocks), plus
    the closed form of a constant row (slse = a + ln r) and -inf at r = 0."""
    import torch

    S = np.random.default_rng(3).standard_normal((2, 3, 11, 11)) * math.sqrt(2)
    slse = select(S, 11, None, mode=oracle.TRAIN)[3]
    err = 0.0
    hist = torch.arange(11)[None, :] < torch.arange(11)[:, None]
    ls = torch.log_softmax(torch.as_tensor(S).masked_fill(~hist, -math.inf), dim=-1).numpy()
    for b in range(2):
        for h in range(3):
            if slse[b, h, 0] != -np.inf:
                return math.inf
            for r in range(1, 11):
                err = max(err, float(np.max(np.abs((S[b, h, r, :r] - slse[b, h, r]) - ls[b, h, r, :r]))))
    a = 0.7
    const = select(np.full((1, 1, 9, 9), a), 9, None, mode=oracle.TRAIN)[3]
    for r in range(1, 9):
        err = max(err, abs(const[0, 0, r] - (a + math.log(r))))
    return err


def test_select_slse_is_history_normaliser():
    assert _slse_pin_error(oracle.select_blocks) < 1e-12


def test_dS_rows_sum_to_zero_and_G_rows_cancel():
    Q, K, V, S, dO = _rand(8, 1, 2, 2, 80, 8, 16)
    for kw in ({}, dict(mode=oracle.SPARSE, topk=2)):
        *_, dS, Gs = oracle.gated_attention_backward(Q, K, V, S, dO, 16, **kw)
        assert np.max(np.abs(dS.sum(-1))) < 1e-12
        # rows of dZ sum to zero, so block sums over a query block cancel
        assert np.max(np.abs(np.nansum(Gs, -1))) < 1e-12


def test_score_row_shift_invariance():
    Q, K, V, S, dO = _rand(9, 1, 2, 2, 64, 8, 16)
    shift = np.random.default_rng(1).standard_normal((1, 2, 4, 1)) * 5
    for kw in ({}, dict(mode=oracle.SPARSE, topk=2)):
        O1, L1 = oracle.gated_attention_forward(Q, K, V, S, 16, **kw)
        O2, L2 = oracle.gated_attention_forward(Q, K, V, S + shift, 16, **kw)
        assert rel_err(O2, O1) < 1e-12 and rel_err(L2, L1) < 1e-12
        dS1 = oracle.gated_attention_backward(Q, K, V, S, dO, 16, **kw)[3]
        dS2 = oracle.gated_attention_backward(Q, K, V, S + shift, dO, 16, **kw)[3]
        assert rel_err(dS2, dS1) < 1e-9


def test_full_budget_topk_equals_training():
    Q, K, V, S, dO = _rand(11, 1, 2, 1, 96, 8, 16)
    O1, L1 = oracle.gated_attention_forward(Q, K, V, S, 16)
    for k in (5, 6, 100):
        O2, L2 = oracle.gated_attention_forward(Q, K, V, S, 16, mode=oracle.SPARSE, topk=k)
        assert np.array_equal(O1, O2) and np.array_equal(L1, L2)


def test_gqa_equals_repeated_kv_heads():
    Q, K, V, S, dO = _rand(12, 1, 4, 2, 48, 8, 16)
    Kr, Vr = np.repeat(K, 2, axis=1), np.repeat(V, 2, axis=1)
    O1, L1 = oracle.gated_attention_forward(Q, K, V, S, 16)
    O2, L2 = oracle.gated_attention_forward(Q, Kr, Vr, S, 16)
    assert rel_err(O1, O2) < 1e-14 and rel_err(L1, L2) < 1e-14
    g1 = oracle.gated_attention_backward(Q, K, V, S, dO, 16)
    g2 = oracle.gated_attention_backward(Q, Kr, Vr, S, dO, 16)
    assert rel_err(g1[0], g2[0]) < 1e-13
    assert rel_err(g1[1], g2[1].reshape(1, 2, 2, 48, 8).sum(2)) < 1e-13
    assert rel_err(g1[2], g2[2].reshape(1, 2, 2, 48, 8).sum(2)) < 1e-13
    assert rel_err(g1[3], g2[3]) < 1e-13


def test_naive_equals_blockwise():
    Q, K, V, S, _ = _rand(13, 1, 2, 1, 48, 8, 8)
    for kw in ({}, dict(mode=oracle.SPARSE, topk=2), dict(mode=oracle.SPARSE, topk=2, renormalise=False)):
        O1, L1 = oracle.gated_attention_forward(Q, K, V, S, 8, **kw)
        O2, L2, _ = oracle.gated_attention_naive(Q, K, V, S, 8, **kw)
        assert rel_err(O1, O2) < 1e-13 and rel_err(L1, L2) < 1e-13


# ------------------------------------------------------------------------ Top-K

def _brute_topk(s, r, k):
    """Selected set by rank counting: c is kept iff fewer than k blocks beat it."""
    keep = []
    for c in range(r):
        beats = sum(1 for c2 in range(r) if s[c2] > s[c] or (s[c2] == s[c] and c2 < c))
        if beats < k:
            keep.append(c)
    return keep


def test_topk_against_brute_force_with_ties():
    rng = np.random.default_rng(14)
    for trial in range(40):
        r = int(rng.integers(0, 40))
        s = rng.integers(-2, 3, size=r).astype(np.float64)
        s[rng.random(r) < 0.2] = -0.0
        for k in (0, 1, 3, 8, 50):
            got = list(oracle.attended_blocks(s, r, oracle.SPARSE, k))
            assert got == _brute_topk(s, r, k), (trial, k)


def test_negative_zero_equals_positive_zero():
    s = np.array([0.0, -0.0, 0.0, -0.0, -1.0])
    assert list(oracle.attended_blocks(s, 5, oracle.SPARSE, 2)) == [0, 1]
    s2 = np.array([-0.0, 0.0, -0.0])
    assert list(oracle.attended_blocks(s2, 3, oracle.SPARSE, 1)) == [0]


# ------------------------------------------------------------ dynamic threshold

def _brute_threshold(s, r, k, tau):
    """Blocks whose gate exp(s_c - logsumexp(s)) reaches tau, keeping the k best."""
    if r == 0:
        return []
    g = np.exp(s[:r] - np.log(np.sum(np.exp(s[:r]))))
    passing = [c for c in range(r) if g[c] >= tau]
    passing.sort(key=lambda c: (-s[c], c))
    return sorted(passing[:k])


def test_threshold_selection_against_definition():
    rng = np.random.default_rng(31)
    for trial in range(60):
        r = int(rng.integers(0, 30))
        s = rng.standard_normal(r) * math.sqrt(2)
        for tau in (1e-4, 0.02, 0.1, 0.3, 1.0):
            for k in (0, 2, 5, 40):
                got = list(oracle.attended_blocks(s, r, oracle.THRESHOLD, k, tau))
                assert got == _brute_threshold(s, r, k, tau), (trial, tau, k)


def test_threshold_limits():
    """tau below every gate with an unlimited budget is training mode; tau = 1
    keeps a block only when it is the sole historical block."""
    Q, K, V, S, _ = _rand(32, 1, 2, 1, 96, 8, 16)
    O1, L1 = oracle.gated_attention_forward(Q, K, V, S, 16)
    O2, L2 = oracle.gated_attention_forward(Q, K, V, S, 16, mode=oracle.THRESHOLD, topk=100, tau=1e-30)
    assert np.array_equal(O1, O2) and np.array_equal(L1, L2)
    idx, cnt, _, _ = oracle.select_blocks(S, 6, 100, mode=oracle.THRESHOLD, tau=1.0)
    assert list(cnt[0, 0]) == [0, 1, 0, 0, 0, 0]


def test_threshold_is_topk_with_passing_count():
    S = np.random.default_rng(33).standard_normal((1, 2, 20, 20)) * math.sqrt(2)
    for tau in (0.05, 0.15):
        for k in (3, 8):
            it, ct, lt, _ = oracle.select_blocks(S, 20, k, mode=oracle.THRESHOLD, tau=tau)
            for h in range(2):
                for r in range(20):
                    kk = min(k, oracle.threshold_count(S[0, h, r], r, tau))
                    ref = oracle.attended_blocks(S[0, h, r], r, oracle.SPARSE, kk)
                    assert ct[0, h, r] == len(ref) and list(it[0, h, r, :len(ref)]) == list(ref)
                    if len(ref):
                        assert abs(np.exp(lt[0, h, r, :len(ref)]).sum() - 1) < 1e-14


# ----------------------------------------------------------------------- decode

@pytest.mark.parametrize("L", [64, 80, 127])
def test_decode_equals_last_prefill_row(L):
    """Decode at position L-1 equals row L-1 of sparse prefill with the same score row."""
    rng = np.random.default_rng(L)
    B, Hq, Hkv, d, bs, k = 2, 4, 2, 8, 8, 3
    Nb = -(-L // bs)
    Q = rng.standard_normal((B, Hq, L, d))
    K = rng.standard_normal((B, Hkv, L, d))
    V = rng.standard_normal((B, Hkv, L, d))
    S_dec = rng.standard_normal((B, Hq, Nb)) * math.sqrt(2)
    S = rng.standard_normal((B, Hq, Nb, Nb))
    S[:, :, Nb - 1, :] = S_dec
    O, LSE = oracle.gated_attention_forward(Q, K, V, S, bs, mode=oracle.SPARSE, topk=k)
    Od, Ld = oracle.gated_decode(Q[:, :, L - 1], K, V, S_dec, L, bs, k)
    assert rel_err(Od, O[:, :, L - 1]) < 1e-13 and rel_err(Ld, LSE[:, :, L - 1]) < 1e-13


def _paged_case(seed, B=3, Hq=4, Hkv=2, d=8, bs=8, Lmax=61):
    """Contiguous caches, their blocks scattered over a shuffled page pool."""
    rng = np.random.default_rng(seed)
    nbmax = -(-Lmax // bs)
    Kc = rng.standard_normal((B, Hkv, nbmax * bs, d))
    Vc = rng.standard_normal((B, Hkv, nbmax * bs, d))
    n_pages = B * nbmax + 5
    perm = rng.permutation(n_pages)
    table = perm[:B * nbmax].reshape(B, nbmax)
    Kpool = rng.standard_normal((n_pages, Hkv, bs, d))  # unused pages hold noise
    Vpool = rng.standard_normal((n_pages, Hkv, bs, d))
    for b in range(B):
        for c in range(nbmax):
            Kpool[table[b, c]] = Kc[b, :, c * bs:(c + 1) * bs]
            Vpool[table[b, c]] = Vc[b, :, c * bs:(c + 1) * bs]
    lens = np.array([Lmax, 17, 40][:B])
    q = rng.standard_normal((B, Hq, d))
    return rng, q, Kc, Vc, Kpool, Vpool, table, lens


@pytest.mark.parametrize("group_shared", [False, True])
def test_paged_decode_equals_prefill_row_at_each_length(group_shared):
    """Each sequence of a paged, variable-length batch equals row L_b - 1 of the
    naive token-level forward over its own unpaged cache."""
    rng, q, Kc, Vc, Kpool, Vpool, table, lens = _paged_case(41)
    B, Hq, d = q.shape
    Hkv, bs, k = Kc.shape[1], 8, 2
    nbmax = table.shape[1]
    S_dec = rng.standard_normal((B, Hkv if group_shared else Hq, nbmax)) * math.sqrt(2)
    O, LSE = oracle.gated_decode_paged(q, Kpool, Vpool, table, lens, S_dec, bs, k,
                                       group_shared=group_shared)
    G = Hq // Hkv
    for b in range(B):
        L = int(lens[b])
        Nb = -(-L // bs)
        Q = rng.standard_normal((1, Hq, L, d))
        Q[0, :, L - 1] = q[b]
        S = rng.standard_normal((1, Hq, Nb, Nb))
        rows = np.repeat(S_dec[b], G, axis=0) if group_shared else S_dec[b]
        S[0, :, Nb - 1, :] = rows[:, :Nb]
        On, Ln, _ = oracle.gated_attention_naive(Q, Kc[b:b + 1, :, :L], Vc[b:b + 1, :, :L], S, bs,
                                                 mode=oracle.SPARSE, topk=k)
        assert rel_err(O[b], On[0, :, L - 1]) < 1e-12 and rel_err(LSE[b], Ln[0, :, L - 1]) < 1e-12


def test_group_shared_heads_differ_only_by_query():
    """With one selection per group, heads whose queries are equal get equal outputs."""
    rng, q, Kc, Vc, Kpool, Vpool, table, lens = _paged_case(43)
    q[:, 1] = q[:, 0]  # heads 0 and 1 form kv group 0
    S_dec = rng.standard_normal((3, 2, table.shape[1]))
    O, LSE = oracle.gated_decode_paged(q, Kpool, Vpool, table, lens, S_dec, 8, 2, group_shared=True)
    assert np.array_equal(O[:, 0], O[:, 1]) and np.array_equal(LSE[:, 0], LSE[:, 1])


def test_attended_pairs_counts():
    S = np.zeros((1, 1, 4, 4))
    # train: history 0+1+2+3 blocks of 4x4 plus 4 triangles of 10
    assert oracle.attended_pairs(S, 16, 4)[0, 0] == 6 * 16 + 4 * 10
    assert oracle.attended_pairs(S, 16, 4, mode=oracle.SPARSE, topk=1)[0, 0] == 3 * 16 + 4 * 10


# ------------------------------------------------------------- planted mistakes

def _mutant(old, new):
    """A fresh copy of the oracle module with one source substitution applied."""
    src = inspect.getsource(ga)
    assert src.count(old) == 1, old
    ns = {"__name__": "oracle_mutant"}
    exec(compile(src.replace(old, new), "<oracle mutant>", "exec"), ns)
    return types.SimpleNamespace(**ns)


def test_pins_catch_wrong_page_lookup():
    bad = _mutant("pages = [int(block_table[b, c]) for c in range(nb)]",
                  "pages = [c for c in range(nb)]")
    rng, q, Kc, Vc, Kpool, Vpool, table, lens = _paged_case(47)
    S_dec = rng.standard_normal((3, 4, table.shape[1]))
    good = oracle.gated_decode_paged(q, Kpool, Vpool, table, lens, S_dec, 8, 2)[0]
    assert rel_err(bad.gated_decode_paged(q, Kpool, Vpool, table, lens, S_dec, 8, 2)[0], good) > 1e-3


def test_pins_catch_dropped_gate_term():
    m = _mutant("gs - g_att * gs.sum()", "gs")
    Q, K, V, S, W = _rand(5, 1, 2, 1, 32, 8, 4)
    assert _fd_check(Q, K, V, S, 4, W, bwd=m.gated_attention_backward) > 1e-3


def test_pins_catch_sign_error_in_softmax_jacobian():
    m = _mutant("dz = p * (dp - np.sum(p * dp, axis=1, keepdims=True))",
                "dz = p * (dp + np.sum(p * dp, axis=1, keepdims=True))")
    Q, K, V, S, W = _rand(5, 1, 2, 1, 32, 8, 4)
    assert _fd_check(Q, K, V, S, 4, W, bwd=m.gated_attention_backward) > 1e-3


def test_pins_catch_unnormalised_gate():
    m = _mutant("return s[A] - _logsumexp(s[norm_set])", "return s[A]")
    Q = np.zeros((1, 1, 3, 1)); K = np.zeros((1, 1, 3, 1))
    V = np.array([1.0, 2.0, 3.0]).reshape(1, 1, 3, 1)
    S = np.zeros((1, 1, 3, 3)); S[0, 0, 2, 0] = math.log(3.0)
    O, _ = m.gated_attention_forward(Q, K, V, S, 1)
    assert abs(O[0, 0, 2, 0] - 17.0 / 8.0) > 1e-3


def test_pins_catch_current_block_in_history():
    m = _mutant("return np.arange(r, dtype=np.int64)", "return np.arange(r + 1, dtype=np.int64)")
    Q, K, V, S, _ = _rand(1, 1, 2, 2, 64, 16, 16)
    O, _ = m.gated_attention_forward(Q, K, V, S, 16, gate="ones")
    O_ref, _ = sdpa_dense_causal(Q, K, V)
    assert rel_err(O, O_ref) > 1e-3


def test_pins_catch_slse_over_current_block():
    m = _mutant("slse[b, h, r] = _logsumexp(_as_f64(S[b, h, r, :r]))",
                "slse[b, h, r] = _logsumexp(_as_f64(S[b, h, r, :r + 1]))")
    assert _slse_pin_error(m.select_blocks) > 1e-3
