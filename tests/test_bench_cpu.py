"""Host-side pieces of bench.py: the work model (attended pairs behind every
TFLOP/s figure) against the oracle's own count, and the rule that a DRAM-traffic
figure is reported only for the kernel source it was measured on."""
import hashlib
import json
import math

import numpy as np
import pytest

import bench
import oracle


@pytest.mark.parametrize("Nb,k", [(1, 4), (7, 3), (16, 4), (16, 100), (33, 8)])
def test_pair_counts_match_the_oracle(Nb, k):
    bs = 4
    S = np.random.default_rng(Nb + k).standard_normal((1, 2, Nb, Nb)) * math.sqrt(2)
    train = oracle.attended_pairs(S, Nb * bs, bs, mode=oracle.TRAIN)
    sparse = oracle.attended_pairs(S, Nb * bs, bs, mode=oracle.SPARSE, topk=k)
    assert np.all(train == bench.train_pairs_per_head(Nb, bs))
    assert np.all(sparse == bench.sparse_pairs_per_head(Nb, bs, k))


def test_headline_pair_count():
    """train_bf16_n8192: 1.0739e9 attended pairs over the 32 heads (FLOP basis);
    train_bf16_n32768 (the headline): 1.7180e10."""
    assert bench.train_pairs_per_head(128, 64) * 32 == 1073872896  # 64*64*(128*127/2) + 128*(64*65/2), x 32
    assert bench.train_pairs_per_head(512, 64) * 32 == 17180393472  # 64*64*(512*511/2) + 512*(64*65/2), x 32


def test_decode_union_blocks_against_sets():
    """Decode bytes count each distinct block of a (sequence, kv group) once:
    the count equals the size of the union of the group's per-head Top-K sets
    (oracle selection) plus one current block per group."""
    import torch
    rng = np.random.default_rng(5)
    for B, Hq, G, Nb, k in ((3, 8, 4, 40, 6), (2, 4, 1, 17, 5), (1, 6, 3, 9, 20), (2, 4, 2, 12, 0)):
        S = rng.standard_normal((B, Hq, Nb)) * math.sqrt(2)
        cur = Nb - 1
        want = 0
        for b in range(B):
            for g in range(Hq // G):
                u = set()
                for h in range(g * G, (g + 1) * G):
                    u |= set(oracle.attended_blocks(S[b, h], cur, oracle.SPARSE, k).tolist())
                want += len(u) + 1
        assert bench.decode_union_blocks(torch.as_tensor(S), cur, k, G) == want


def test_prefix_inputs_are_the_workload_prefix():
    """The CPU samples read the first tokens of the workload's own inputs."""
    from gated_block_sparse_gate_b200.inputs import WORKLOADS, make_prefill_inputs
    import dataclasses
    w = dataclasses.replace(WORKLOADS["train_bf16_n8192"], N=1024)
    full = make_prefill_inputs(w)
    x, wp = bench.prefix_inputs(w, 256)
    assert wp.N == 256 and wp.Nb == 4
    for k in ("Q", "K", "V", "dO"):
        assert np.array_equal(x[k].float().numpy(), full[k][:, :, :256].float().numpy())
    assert np.array_equal(x["S"].numpy(), full["S"][:, :, :4, :4].numpy())


def test_traffic_is_tied_to_the_measured_source(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("// kernel v1\n")
    digest = hashlib.sha256(src.read_bytes()).hexdigest()
    (tmp_path / "profiles").mkdir()
    table = {"k/w1": {"source": "k.cu", "sha256": digest, "bytes_per_launch": 12345}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(table))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_for("k", "w1") == 12345.0
    assert bench.traffic_for("k", "w2") is None  # measured on another workload
    assert bench.traffic_for("missing", "w1") is None
    src.write_text("// kernel v2\n")  # the kernel changed since the counters were taken
    assert bench.traffic_for("k", "w1") is None


def _union_tiling_fraction(S, k):
    """Attended pairs / pairs the sparse forward's stages compute, for the
    tiling that pairs query blocks 2t and 2t+1 over the union of their kept
    blocks plus both current blocks, padded to an even count of 64-key slots,
    two slots per 128 x 128 stage."""
    Hq, Nb = S.shape[1], S.shape[2]
    attended = computed = 0.0
    for h in range(Hq):
        kept = [set(oracle.attended_blocks(S[0, h, r], r, oracle.SPARSE, k).tolist()) for r in range(Nb)]
        for t in range(Nb // 2):
            r0, r1 = 2 * t, 2 * t + 1
            slots = len(kept[r0] | kept[r1] | {r0, r1})
            computed += (slots + (slots & 1)) * 64 * 128
            attended += (len(kept[r0]) + len(kept[r1])) * 64 * 64 + 2 * (64 * 65 // 2)
    return attended / computed


def test_sparse_prefill_tiling_ceiling():
    """On the planted N = 65536 recipe (two heads drawn), the two-query-block
    tiles compute about twice the attended pairs: the tiling's ceiling is about
    half the tensor peak at K = 8 and about 60% at K = 32."""
    from gated_block_sparse_gate_b200.inputs import WORKLOADS, make_prefill_inputs
    w = WORKLOADS["sparse_prefill_bf16_n65536"]
    S = make_prefill_inputs(w, Hq=2, Hkv=1, with_grad=False)["S"].numpy().astype(np.float64)
    f8, f32 = _union_tiling_fraction(S, 8), _union_tiling_fraction(S, 32)
    assert 0.45 < f8 < 0.56 and 0.55 < f32 < 0.65, (f8, f32)


def _backward_tiling_fraction(S, k, G):
    """Attended pairs / pairs the sparse backward's steps compute: per 128-key
    tile (blocks 2u, 2u+1) of a kv group, every (q-head, query block) that keeps
    either block (or is one of them) is an entry, two entries per 128 x 128 step."""
    Nb = S.shape[2]
    kept = [[set(oracle.attended_blocks(S[0, h, r], r, oracle.SPARSE, k).tolist()) | {r}
             for r in range(Nb)] for h in range(G)]
    attended = computed = 0.0
    for u in range(Nb // 2):
        tile = {2 * u, 2 * u + 1}
        entries = 0
        for h in range(G):
            for r in range(2 * u, Nb):
                n = len(kept[h][r] & tile)
                if n:
                    entries += 1
                    diag = r in tile
                    attended += (n - diag) * 64 * 64 + diag * (64 * 65 // 2)
        computed += ((entries + 1) // 2) * 128 * 128
    return attended / computed


def test_sparse_backward_tiling_ceiling():
    """On one kv group of the planted N = 65536 recipe the backward's steps
    compute about twice the attended pairs: its ceiling is about half the
    tensor peak."""
    from gated_block_sparse_gate_b200.inputs import WORKLOADS, make_prefill_inputs
    w = WORKLOADS["sparse_prefill_bf16_n65536"]
    S = make_prefill_inputs(w, Hq=4, Hkv=1, with_grad=False)["S"].numpy().astype(np.float64)
    f8, f32 = _backward_tiling_fraction(S, 8, 4), _backward_tiling_fraction(S, 32, 4)
    assert 0.43 < f8 < 0.52 and 0.48 < f32 < 0.57, (f8, f32)


def test_reference_arm_prints_the_contract_line(capsys):
    """bench.py --impl reference: the oracle on the host cores, one JSON line."""
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "1"]) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["steps"] == 1
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["unit"] == line["unit"]
    assert line["config"]["workload"] == "train_bf16_n32768"
