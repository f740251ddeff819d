"""The debug build of the library (libgbs_debug.so, compiled with -DGBS_DEBUG).

Its kernels check every index they take from a list (K1's Top-K lists and
counts, the backward's per-CTA plans, the decode's lists) and report one
outside its range as GBS_ERR_DEVICE_CHECK, with the access clamped. No device
memory checker runs where these tests run, so this build stands in for one:
the same cases through the release and the debug library must give the same
bits (the checks change no arithmetic), and every debug workspace must come
back without a recorded error.
"""
import dataclasses

import pytest
import torch

from gated_block_sparse_gate_b200 import binding as gb
from gated_block_sparse_gate_b200.build import build
from gated_block_sparse_gate_b200.inputs import WORKLOADS, make_decode_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module")
def libs():
    saved = gb._lib
    out = {}
    for name, debug in (("release", False), ("debug", True)):
        path = build(debug=debug)
        gb._lib = None
        out[name] = gb.load_library(path)
    gb._lib = saved
    yield out
    gb._lib = saved


def _on(lib, fn):
    saved = gb._lib
    gb._lib = lib
    try:
        return fn()
    finally:
        gb._lib = saved


def _prefill(seed, B, Hq, Hkv, N, d):
    g = torch.Generator().manual_seed(seed)
    x = {n: torch.randn(B, Hq if n in "QdO" else Hkv, N, d, generator=g).to(torch.bfloat16)
         for n in ("Q", "K", "V")}
    x["S"] = torch.randn(B, Hq, N // 64, N // 64, generator=g) * 2 ** 0.5
    x["dO"] = torch.randn(B, Hq, N, d, generator=g).to(torch.bfloat16)
    return {n: t.to(DEV) for n, t in x.items()}


def _prefill_run(x, mode, k, tau):
    Q, K, V, S, dO = (x[n] for n in ("Q", "K", "V", "S", "dO"))
    pf = gb.make_params(Q.shape[0], Q.shape[1], K.shape[1], Q.shape[2], Q.shape[3], 64, k, mode,
                        Q.dtype, tau=tau)
    ws_f = gb.alloc_workspace(pf, gb.OP_FWD, DEV)
    ws_b = gb.alloc_workspace(pf, gb.OP_BWD, DEV)
    O, LSE = gb.forward(Q, K, V, S, mode=mode, topk=k, tau=tau, ws=ws_f)
    grads = gb.backward(Q, K, V, S, O, LSE, dO, mode=mode, topk=k, tau=tau, ws=ws_b)
    gb.check(ws_f)
    gb.check(ws_b)
    return (O, LSE) + tuple(grads)


@pytest.mark.parametrize("shape,mode,k,tau", [
    ((2, 8, 2, 1024, 128), "sparse", 3, 0.0),      # slot plans and key-tile step lists
    ((1, 8, 2, 1024, 128), "threshold", 6, 0.05),
    ((1, 4, 2, 448, 64), "sparse", 2, 0.0),         # d = 64, odd block count
    ((1, 8, 2, 1024, 128), "train", 0, 0.0),
])
def test_debug_build_matches_release_and_reports_nothing(libs, shape, mode, k, tau):
    x = _prefill(97 + k, *shape)
    rel = _on(libs["release"], lambda: _prefill_run(x, mode, k, tau))
    dbg = _on(libs["debug"], lambda: _prefill_run(x, mode, k, tau))
    torch.cuda.synchronize()
    names = ("O", "LSE", "dQ", "dK", "dV", "dS")
    for n, a, b in zip(names, rel, dbg):
        if n in ("dQ", "dS"):  # sums across CTAs in hardware order
            assert torch.allclose(a.float(), b.float(), rtol=2 ** -7, atol=1e-6), n
        else:
            assert torch.equal(a, b), n


def test_debug_build_decode(libs):
    w = dataclasses.replace(WORKLOADS["sparse_decode_bf16_b64_l131072"], B=4, N=5000)
    x = make_decode_inputs(w, B=4, L=5000, device=DEV)
    g = torch.Generator().manual_seed(5)
    Sg = (torch.randn(4, w.Hkv, w.Nb, generator=g) * 2 ** 0.5).to(DEV)
    lens = torch.tensor([5000, 1, 64, 3333], dtype=torch.int32, device=DEV)

    def run():
        p = gb.make_params(4, w.Hq, w.Hkv, 5000, w.d, 64, 16, "sparse", x["q"].dtype)
        ws = gb.alloc_workspace(p, gb.OP_DECODE, DEV)
        a = gb.decode(x["q"], x["Kc"], x["Vc"], x["S"], topk=16, ws=ws)
        b = gb.decode_ex(x["q"], x["Kc"], x["Vc"], Sg, 5000, topk=16, group_shared=True,
                         seq_lens=lens, ws=ws)
        gb.check(ws)
        return a + b

    rel = _on(libs["release"], run)
    dbg = _on(libs["debug"], run)
    for a, b in zip(rel, dbg):
        assert torch.equal(a, b)
