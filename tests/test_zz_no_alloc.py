"""gbs_decode_noalloc: the decode for callers that cannot allocate device memory.

Some callers cannot give the library a workspace when they decode, for
instance a serving loop whose device memory is reserved up front by another
allocator, or one that must not call cudaMalloc on its hot path because the
call can synchronise the device. gbs_decode_noalloc keeps its scratch in a
static device array inside the library instead. These tests call it through
the C ABI and check it against gbs_decode (which uses a caller workspace) on
two calls in a row, within the bf16 tolerance the other decode tests use, and
check that sizes beyond the static scratch are refused before any launch.
This file is collected last so a stop at the first failure has already run
every other test; it needs nothing from them and passes on its own too.
"""
import ctypes
import dataclasses

import pytest
import torch

from gated_block_sparse_gate_b200 import binding as gb
from gated_block_sparse_gate_b200.build import build
from gated_block_sparse_gate_b200.inputs import WORKLOADS, make_decode_inputs
from tests.oracle_refs import rel_err

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-2
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    gb.load_library()


def _inputs(B, L, d=128):
    w = dataclasses.replace(WORKLOADS["sparse_decode_bf16_b64_l131072"], B=B, N=L, d=d)
    return make_decode_inputs(w, B=B, L=L, device=DEV)


@pytest.mark.parametrize("B,L,k,splits,tau,d", [
    (8, 4133, 8, 0, None, 128),     # ragged current block, automatic split count
    (4, 8192, 32, 3, None, 128),
    (2, 64, 4, 1, None, 128),       # no history at all
    (3, 700, 32, 0, None, 128),     # budget above the 10 historical blocks
    (4, 5000, 8, 0, 0.05, 128),     # threshold mode
    (4, 3000, 6, 2, None, 64),      # head dim 64
])
def test_noalloc_matches_workspace_decode_twice(B, L, k, splits, tau, d):
    x = _inputs(B, L, d)
    O_ref, L_ref = gb.decode(x["q"], x["Kc"], x["Vc"], x["S"], topk=k, num_splits=splits, tau=tau)
    for _ in range(2):  # the second call reuses the scratch the first one left behind
        O, LSE = gb.decode_noalloc(x["q"], x["Kc"], x["Vc"], x["S"], topk=k, num_splits=splits,
                                   tau=tau)
        torch.cuda.synchronize()
        assert rel_err(O.float().cpu().numpy(), O_ref.float().cpu().numpy()) < TOL_BF16
        assert rel_err(LSE.cpu().numpy(), L_ref.cpu().numpy()) < TOL_BF16
        # the same split count and kernels as gbs_decode: the same bits
        assert torch.equal(O, O_ref) and torch.equal(LSE, L_ref)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    lib = gb.load_library()
    lib.gbs_decode_noalloc.restype = ctypes.c_int
    # 256 x 64 rows with topk 256: a valid decode (B * Hq * N < 2^31) whose Top-K
    # lists alone (16 MiB) exceed the static array
    p = gb.make_params(256, 64, 8, 16384, 128, 64, 256, "sparse", torch.bfloat16)
    fake = ctypes.c_void_p(4096)
    st = lib.gbs_decode_noalloc(ctypes.byref(p), fake, fake, fake, fake, fake, fake, 0, None)
    assert st == 1
    assert b"static scratch" in lib.gbs_last_error()
