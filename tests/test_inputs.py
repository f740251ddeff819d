"""The seeded input recipe (shared by the oracle and the CUDA path): the
planted column structure of the sparse prefill workload, determinism, and the
per-sequence seeding of decode caches."""
import dataclasses

import numpy as np
import torch

from gated_block_sparse_gate_b200.inputs import WORKLOADS, make_decode_inputs, make_prefill_inputs


def test_planted_columns():
    """Per (b, h) a random 10% of key-block columns get +3.0 on every row; the
    rest of S is the same N(0, 2) draw as without the plant."""
    w = WORKLOADS["sparse_prefill_bf16_n65536"]
    base = dataclasses.replace(w, plant_frac=0.0, plant_boost=0.0)
    kw = dict(N=2048, Hq=4, Hkv=2, with_grad=False)
    diff = (make_prefill_inputs(w, **kw)["S"] - make_prefill_inputs(base, **kw)["S"]).numpy()
    Nb = 2048 // 64
    n_plant = round(0.10 * Nb)
    for h in range(4):
        cols = np.flatnonzero(np.any(diff[0, h] != 0, axis=0))
        assert len(cols) == n_plant
        assert np.allclose(diff[0, h][:, cols], 3.0, atol=1e-6)
    assert not np.array_equal(np.flatnonzero(diff[0, 0].any(0)), np.flatnonzero(diff[0, 1].any(0)))


def test_scores_have_variance_two():
    S = make_prefill_inputs(WORKLOADS["train_bf16_n8192"], N=4096, Hq=8, Hkv=2, with_grad=False)["S"]
    assert abs(float(S.var()) - 2.0) < 0.05 and abs(float(S.mean())) < 0.02


def test_prefill_inputs_are_deterministic_and_scaled():
    w = WORKLOADS["train_bf16_n8192"]
    a = make_prefill_inputs(w, N=256, Hq=2, Hkv=1)
    b = make_prefill_inputs(w, N=256, Hq=2, Hkv=1)
    assert all(torch.equal(a[k], b[k]) for k in a)
    assert a["Q"].dtype == torch.bfloat16 and a["S"].dtype == torch.float32
    # Q, K, V are N(0, 1) scaled by d^-1/2 (std about 0.088 at d = 128)
    assert abs(float(a["Q"].float().std()) - 128 ** -0.5) < 0.01


def test_decode_sequences_are_seeded_one_by_one():
    """Sequence b's cache depends only on (seed, b): a batch of 3 repeats the
    first two sequences of a batch of 2."""
    w = dataclasses.replace(WORKLOADS["sparse_decode_bf16_b64_l131072"], N=300)
    two = make_decode_inputs(w, B=2, L=300)
    three = make_decode_inputs(w, B=3, L=300)
    assert torch.equal(two["Kc"], three["Kc"][:2]) and torch.equal(two["Vc"], three["Vc"][:2])
    assert not torch.equal(three["Kc"][0], three["Kc"][1])
