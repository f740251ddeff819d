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
    """train_bf16_n8192: 1.0739e9 attended pairs over the 32 heads (FLOP basis)."""
    assert bench.train_pairs_per_head(128, 64) * 32 == 1073872896  # 64*64*(128*127/2) + 128*(64*65/2), x 32


def test_traffic_is_tied_to_the_measured_source(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("// kernel v1\n")
    digest = hashlib.sha256(src.read_bytes()).hexdigest()
    (tmp_path / "profiles").mkdir()
    table = {"k": {"source": "k.cu", "sha256": digest, "bytes_per_launch": 12345}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(table))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_for("k") == 12345.0
    assert bench.traffic_for("missing") is None
    src.write_text("// kernel v2\n")  # the kernel changed since the counters were taken
    assert bench.traffic_for("k") is None
