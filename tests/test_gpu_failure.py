"""Failure detection on the GPU without a fault.

The tensor-core kernels bound every pipeline wait: a wait that outlives its
limit records GBS_ERR_TIMEOUT in the workspace's error word and the kernel
drains and returns. Here a self-test kernel makes that branch run (a wait on a
barrier nothing arrives at, limited to a few milliseconds); the host reads the
status through gbs_check, and the same context then decodes as before.
"""
import dataclasses

import pytest
import torch

from gated_block_sparse_gate_b200 import binding as gb
from gated_block_sparse_gate_b200.build import build
from gated_block_sparse_gate_b200.inputs import WORKLOADS, make_decode_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    gb.load_library()


def test_bounded_wait_expiry_reports_timeout_and_context_survives():
    w = dataclasses.replace(WORKLOADS["sparse_decode_bf16_b64_l131072"], B=2, N=3000)
    x = make_decode_inputs(w, B=2, L=3000, device=DEV)
    O1, L1 = gb.decode(x["q"], x["Kc"], x["Vc"], x["S"], topk=8)
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    gb.check(ws)  # starts clean
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    gb.selftest_wait_timeout(ws, 2000)  # 2 ms
    b.record()
    with pytest.raises(gb.GbsError) as info:
        gb.check(ws)
    assert info.value.status == 4  # GBS_ERR_TIMEOUT
    ms = a.elapsed_time(b)
    assert 2.0 <= ms < 1000.0, ms  # gave up after its limit, not never
    gb.clear_error(ws)
    gb.check(ws)
    O2, L2 = gb.decode(x["q"], x["Kc"], x["Vc"], x["S"], topk=8)
    torch.cuda.synchronize()
    assert torch.equal(O1, O2) and torch.equal(L1, L2)


def test_selftest_rejects_bad_arguments():
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    for limit in (0, 2_000_000):
        with pytest.raises(gb.GbsError) as info:
            gb.selftest_wait_timeout(ws, limit)
        assert info.value.status == 1
