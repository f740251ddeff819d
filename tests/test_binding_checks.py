"""The binding's argument checks (CPU): the layouts the C ABI reads are
enforced before any pointer reaches the library, so a host tensor, a strided
view or a mismatched dtype or shape raises instead of being read as device
memory. Shapes and dtypes are exercised on ``meta`` tensors (no storage)."""
import pytest
import torch

from gated_block_sparse_gate_b200 import binding as gb

BF, F32 = torch.bfloat16, torch.float32


def meta(*shape, dtype=BF):
    return torch.empty(*shape, dtype=dtype, device="meta")


@pytest.fixture
def on_meta(monkeypatch):
    monkeypatch.setattr(gb, "_DEVICE_TYPES", ("meta",))


def prefill(B=1, Hq=4, Hkv=2, N=256, d=64, dtype=BF):
    return (meta(B, Hq, N, d, dtype=dtype), meta(B, Hkv, N, d, dtype=dtype),
            meta(B, Hkv, N, d, dtype=dtype), meta(B, Hq, N // 64, N // 64, dtype=F32))


def rejected(fn, *args, **kw):
    with pytest.raises(gb.GbsError) as e:
        fn(*args, **kw)
    assert e.value.status == 1
    return str(e.value)


def test_prefill_layouts_accepted(on_meta):
    for dtype in (BF, F32):
        Q, K, V, S = prefill(dtype=dtype)
        gb._check_prefill("t", Q, K, V, S, 64)
        gb._check_prefill("t", Q, K, V, S, 64, outs=(
            ("O", meta(*Q.shape, dtype=dtype), Q.shape, (dtype,)),
            ("LSE", meta(1, 4, 256, dtype=F32), Q.shape[:3], gb._F32),
            ("ws", meta(4096, dtype=torch.uint8), None, gb._U8)))


def test_prefill_mismatches_rejected(on_meta):
    Q, K, V, S = prefill()
    assert "dtype" in rejected(gb._check_prefill, "t", Q, K.float(), V, S, 64)
    assert "S has shape" in rejected(gb._check_prefill, "t", Q, K, V, meta(1, 4, 4, 3, dtype=F32), 64)
    assert "S has dtype" in rejected(gb._check_prefill, "t", Q, K, V, S.to(BF), 64)
    assert "V has shape" in rejected(gb._check_prefill, "t", Q, K, meta(1, 2, 128, 64), S, 64)
    Qt = meta(1, 4, 64, 256).transpose(2, 3)  # right shape, wrong strides
    assert "contiguous" in rejected(gb._check_prefill, "t", Qt, K, V, S, 64)
    assert "float16" in rejected(gb._check_prefill, "t", Q.half(), K.half(), V.half(), S, 64)
    Kcpu = torch.empty(1, 2, 256, 64, dtype=BF)
    assert "expected meta" in rejected(gb._check_prefill, "t", Q, Kcpu, V, S, 64)
    dS_bad = ("dS", meta(1, 4, 4, 4, dtype=BF), S.shape, gb._F32)
    assert "dS has dtype" in rejected(gb._check_prefill, "t", Q, K, V, S, 64, outs=(dS_bad,))


def test_decode_layouts_accepted(on_meta):
    B, Hq, Hkv, d, L = 4, 8, 2, 128, 4133
    nb = -(-L // 64)
    q = meta(B, Hq, d)
    gb._check_decode("t", q, meta(B, Hkv, L, d), meta(B, Hkv, L, d), meta(B, Hq, nb, dtype=F32), L, 64)
    pools = meta(B * nb + 7, Hkv, 64, d)
    gb._check_decode("t", q, pools, pools, meta(B, Hkv, nb, dtype=F32), L, 64,
                     block_table=meta(B, nb, dtype=torch.int32),
                     seq_lens=meta(B, dtype=torch.int32), group_shared=True)


def test_decode_mismatches_rejected(on_meta):
    B, Hq, Hkv, d, L = 4, 8, 2, 128, 4133
    nb = -(-L // 64)
    q, S = meta(B, Hq, d), meta(B, Hq, nb, dtype=F32)
    longer = meta(B, Hkv, nb * 64, d)  # rows past L would be read at the wrong stride
    assert "Kc has shape" in rejected(gb._check_decode, "t", q, longer, longer, S, L, 64)
    Kc = meta(B, Hkv, L, d)
    assert "S has shape" in rejected(gb._check_decode, "t", q, Kc, Kc, S, L, 64, group_shared=True)
    pools = meta(B * nb, Hkv, 64, d)
    assert "block_table has dtype" in rejected(gb._check_decode, "t", q, pools, pools, S, L, 64,
                                               block_table=meta(B, nb, dtype=torch.int64))
    assert "block_table must be" in rejected(gb._check_decode, "t", q, pools, pools, S, L, 64,
                                             block_table=meta(B + 1, nb, dtype=torch.int32))
    assert "seq_lens has shape" in rejected(gb._check_decode, "t", q, Kc, Kc, S, L, 64,
                                            seq_lens=meta(B + 1, dtype=torch.int32))
    assert "Vc has dtype" in rejected(gb._check_decode, "t", q, Kc, Kc.float(), S, L, 64)


def test_host_tensors_never_reach_the_library():
    """Without a CUDA device the binding refuses host memory up front."""
    gb.load_library()
    Q, K, V = (torch.zeros(1, 2, 128, 64, dtype=BF) for _ in range(3))
    S = torch.zeros(1, 2, 2, 2)
    assert "CUDA" in rejected(gb.forward, Q, K, V, S)
    assert "CUDA" in rejected(gb.select, S, topk=1)
    q = torch.zeros(1, 2, 64, dtype=BF)
    assert "CUDA" in rejected(gb.decode, q, K, V, torch.zeros(1, 2, 2), topk=1)
