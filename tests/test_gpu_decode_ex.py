"""GPU parity of gbs_decode_ex: paged and variable-length KV caches and
group-shared selection, against the float64 oracle (gated_decode_paged).

Tolerances as for the decode: O and LSE normwise 2e-2 (bf16) and 1e-5 (fp32).
At full size (64 sequences x 131072 tokens) a paged cache whose blocks sit on
shuffled pages must give exactly the contiguous decode's bits: the kernel does
the same arithmetic in the same order wherever a block lives.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from gated_block_sparse_gate_b200 import binding as gb
from gated_block_sparse_gate_b200.build import build
from gated_block_sparse_gate_b200.inputs import WORKLOADS, make_decode_inputs
from tests.oracle_refs import rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    gb.load_library()


def np64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def _paged(seed, B, Hq, Hkv, d, Lmax, lens, dtype, group_shared, extra_pages=7):
    g = torch.Generator().manual_seed(seed)
    scl = d ** -0.5
    nb = -(-Lmax // 64)
    Kc = (torch.randn(B, Hkv, nb * 64, d, generator=g) * scl).to(dtype)
    Vc = (torch.randn(B, Hkv, nb * 64, d, generator=g) * scl).to(dtype)
    n_pages = B * nb + extra_pages
    perm = torch.randperm(n_pages, generator=g)
    table = perm[:B * nb].view(B, nb).to(torch.int32)
    Kpool = (torch.randn(n_pages, Hkv, 64, d, generator=g) * scl).to(dtype)
    Vpool = (torch.randn(n_pages, Hkv, 64, d, generator=g) * scl).to(dtype)
    for b in range(B):
        for c in range(nb):
            Kpool[table[b, c]] = Kc[b, :, c * 64:(c + 1) * 64]
            Vpool[table[b, c]] = Vc[b, :, c * 64:(c + 1) * 64]
    q = (torch.randn(B, Hq, d, generator=g) * scl).to(dtype)
    S = torch.randn(B, Hkv if group_shared else Hq, nb, generator=g) * math.sqrt(2)
    return dict(q=q, Kc=Kc, Vc=Vc, Kpool=Kpool, Vpool=Vpool, table=table, S=S,
                lens=torch.tensor(lens, dtype=torch.int32))


def _run_and_check(x, Lmax, k, tol, group_shared, paged=True, splits=0, tau=None):
    dev = {n: t.to(DEV) for n, t in x.items()}
    # a contiguous cache is [B, Hkv, Lmax, d]
    Kc, Vc = ((dev["Kpool"], dev["Vpool"]) if paged else
              (dev["Kc"][:, :, :Lmax].contiguous(), dev["Vc"][:, :, :Lmax].contiguous()))
    O, LSE = gb.decode_ex(dev["q"], Kc, Vc, dev["S"], Lmax, topk=k, num_splits=splits,
                          block_table=dev["table"] if paged else None, seq_lens=dev["lens"],
                          group_shared=group_shared, tau=tau)
    torch.cuda.synchronize()
    Or, Lr = oracle.gated_decode_paged(np64(x["q"]), np64(x["Kpool"]), np64(x["Vpool"]),
                                       x["table"].numpy(), x["lens"].numpy(), x["S"].numpy(), 64, k,
                                       group_shared=group_shared,
                                       mode=oracle.SPARSE if tau is None else oracle.THRESHOLD,
                                       tau=tau)
    eo, el = rel_err(np64(O), Or), rel_err(LSE.cpu().numpy(), Lr)
    assert eo < tol and el < tol, (eo, el)


@pytest.mark.parametrize("group_shared", [False, True])
@pytest.mark.parametrize("splits", [0, 1, 3])
def test_paged_varlen_bf16(group_shared, splits):
    x = _paged(3, 4, 8, 2, 128, 4133, [4133, 64, 1000, 2049], torch.bfloat16, group_shared)
    _run_and_check(x, 4133, 8, 2e-2, group_shared, splits=splits)


@pytest.mark.parametrize("group_shared", [False, True])
def test_varlen_contiguous_bf16(group_shared):
    x = _paged(5, 3, 8, 2, 128, 3000, [3000, 65, 1], torch.bfloat16, group_shared)
    _run_and_check(x, 3000, 5, 2e-2, group_shared, paged=False)


@pytest.mark.parametrize("group_shared", [False, True])
def test_paged_f32_d64(group_shared):
    x = _paged(7, 2, 4, 2, 64, 2000, [2000, 700], torch.float32, group_shared)
    _run_and_check(x, 2000, 6, 1e-5, group_shared)


@pytest.mark.parametrize("Hq,Hkv", [(16, 2), (6, 2), (4, 2), (4, 4)])
def test_group_shared_group_sizes(Hq, Hkv):
    """G = 8, 3, 2, 1: two, one, two and one q-heads per CTA."""
    x = _paged(11 + Hq, 2, Hq, Hkv, 128, 1500, [1500, 900], torch.bfloat16, True)
    _run_and_check(x, 1500, 4, 2e-2, True)


def test_paged_threshold_group_shared():
    x = _paged(13, 3, 8, 2, 128, 5000, [5000, 3000, 640], torch.bfloat16, True)
    Sn = x["S"].numpy()
    tau = 0.02
    for b, L in enumerate(x["lens"].tolist()):
        cur = (L - 1) // 64
        for h in range(Sn.shape[1]):
            band = [oracle.threshold_count(Sn[b, h], cur, tau * math.exp(s)) for s in (1e-4, -1e-4)]
            assert cur <= 1 or band[0] == band[1]
    _run_and_check(x, 5000, 16, 2e-2, True, tau=tau)


def test_out_of_range_page_and_length_are_reported():
    """The kernel's own bounds checks skip a bad page and clamp a bad length,
    and the workspace error word reports GBS_ERR_INVALID_ARG."""
    x = _paged(17, 2, 4, 2, 128, 1000, [1000, 1000], torch.bfloat16, False)
    dev = {n: t.to(DEV) for n, t in x.items()}
    p = gb.make_params(2, 4, 2, 1000, 128, 64, 4, "sparse", torch.bfloat16)
    for table, lens in ((dev["table"].clone(), dev["lens"]), (dev["table"], dev["lens"].clone())):
        if table is not dev["table"]:
            table[1, 999 // 64] = dev["Kpool"].shape[0]  # current block: one past the last page
        else:
            lens[0] = 0
        ws = gb.alloc_workspace(p, gb.OP_DECODE, DEV)
        gb.decode_ex(dev["q"], dev["Kpool"], dev["Vpool"], dev["S"], 1000, topk=4,
                     block_table=table, seq_lens=lens, ws=ws)
        with pytest.raises(gb.GbsError) as e:
            gb.check(ws)
        assert e.value.status == 1


def test_full_size_paged_equals_contiguous_bitwise():
    """64 sequences x 131072 cache, K=32, blocks on shuffled pages: same bits."""
    w = WORKLOADS["sparse_decode_bf16_b64_l131072"]
    x = make_decode_inputs(w, device=DEV)
    Kc, Vc = x["Kc"], x["Vc"]
    B, Hkv, L, d = Kc.shape
    nb = L // 64
    g = torch.Generator(device="cpu").manual_seed(99)
    perm = torch.randperm(B * nb, generator=g).to(DEV)
    table = perm.view(B, nb).to(torch.int32)
    O_ref, L_ref = gb.decode(x["q"], Kc, Vc, x["S"], topk=32)
    for name, src in (("K", Kc), ("V", Vc)):
        pool = torch.empty(B * nb, Hkv, 64, d, dtype=src.dtype, device=DEV)
        pool[perm] = src.view(B, Hkv, nb, 64, d).permute(0, 2, 1, 3, 4).reshape(B * nb, Hkv, 64, d)
        if name == "K":
            Kpool = pool
        else:
            Vpool = pool
        del src
    del Kc, Vc, x["Kc"], x["Vc"]
    torch.cuda.empty_cache()
    O, LSE = gb.decode_ex(x["q"], Kpool, Vpool, x["S"], L, topk=32, block_table=table)
    torch.cuda.synchronize()
    assert torch.equal(O, O_ref) and torch.equal(LSE, L_ref)
    del Kpool, Vpool
    torch.cuda.empty_cache()


def test_full_size_group_shared_sampled():
    """Decode workload with one score row per kv group: sampled sequences."""
    w = WORKLOADS["sparse_decode_bf16_b64_l131072"]
    x = make_decode_inputs(w, device=DEV)
    g = torch.Generator().manual_seed(101)
    Sg = torch.randn(w.B, w.Hkv, w.N // 64, generator=g) * math.sqrt(2)
    O, LSE = gb.decode_ex(x["q"], x["Kc"], x["Vc"], Sg.to(DEV), w.N, topk=32, group_shared=True)
    torch.cuda.synchronize()
    seqs = [0, 41, 63]
    G = w.Hq // w.Hkv
    for b in seqs:
        rows = np.repeat(Sg[b].numpy(), G, axis=0)[None]
        o, l = oracle.gated_decode(np64(x["q"][b:b + 1]), np64(x["Kc"][b:b + 1]),
                                   np64(x["Vc"][b:b + 1]), rows, w.N, 64, 32)
        assert rel_err(np64(O[b:b + 1]), o) < 2e-2 and rel_err(LSE[b:b + 1].cpu().numpy(), l) < 2e-2
    del x
    torch.cuda.empty_cache()
