"""C ABI checks that need no GPU: the library loads, exports every symbol the
header declares, sizes workspaces, and rejects bad arguments before any launch."""
import ctypes
import os
import re

import pytest

from gated_block_sparse_gate_b200 import binding as gb
from gated_block_sparse_gate_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build()
    return gb.load_library()


def _declared():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"GBS_API\s+[\w\s\*]+?\b(gbs_\w+)\s*\(", src)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    declared = _declared()
    assert len(declared) >= 10
    for name in declared:
        assert hasattr(lib, name), name
    assert set(gb.EXPORTED) <= set(declared)


def test_version_and_status_strings(lib):
    assert lib.gbs_version() == (0 << 16) | 1
    for s in range(7):
        assert lib.gbs_status_string(s) != b"unknown status"


def test_workspace_sizes(lib):
    p = gb.make_params(1, 32, 8, 8192, 128, 64, 0, "train")
    fwd = gb.workspace_bytes(p, gb.OP_FWD)
    bwd = gb.workspace_bytes(p, gb.OP_BWD)
    assert fwd >= 256 + 32 * 128 * 4
    # D vector [B,Hq,N] and the tile sums [B,Hq,Nb,Nb]
    assert bwd >= 256 + 32 * 8192 * 4 + 32 * 128 * 128 * 4
    ps = gb.make_params(1, 32, 8, 65536, 128, 64, 64, "sparse")
    assert gb.workspace_bytes(ps, gb.OP_FWD) > 32 * 1024 * 64 * 8
    pd = gb.make_params(64, 32, 8, 131072, 128, 64, 32, "sparse")
    assert gb.workspace_bytes(pd, gb.OP_DECODE) > 64 * 32 * 32 * 8


@pytest.mark.parametrize("kw,status", [
    (dict(Hq=6, Hkv=4), 1),          # Hq not a multiple of Hkv
    (dict(N=100), 1),                 # N not a multiple of the block
    (dict(block=32, N=128), 2),       # block size not built
    (dict(d=96), 2),                  # head dim not built
    (dict(mode="sparse", topk=-1), 1),
    (dict(mode="sparse", topk=10_000), 1),
    (dict(B=0), 1),
    (dict(B=1024, Hq=64, Hkv=8, N=32768), 1),   # 2^31 token rows: beyond 32-bit coordinates
])
def test_invalid_params_rejected_before_launch(lib, kw, status):
    args = dict(B=1, Hq=4, Hkv=2, N=256, d=64, block=64, topk=0, mode="train")
    args.update(kw)
    p = gb.make_params(**args)
    assert gb.workspace_bytes(p, gb.OP_FWD) == 0
    fake = ctypes.c_void_p(4096)
    st = lib.gbs_fwd(ctypes.byref(p), fake, fake, fake, fake, fake, fake, fake, 1 << 30, None)
    assert st == status, lib.gbs_last_error()


@pytest.mark.parametrize("tau", [0.0, -0.5, 1.5, float("nan")])
def test_threshold_mode_needs_tau_in_unit_interval(lib, tau):
    p = gb.make_params(1, 4, 2, 256, 64, 64, 4, "threshold", tau=tau)
    assert gb.workspace_bytes(p, gb.OP_FWD) == 0
    assert gb.workspace_bytes(p, gb.OP_DECODE) == 0
    fake = ctypes.c_void_p(4096)
    st = lib.gbs_fwd(ctypes.byref(p), fake, fake, fake, fake, fake, fake, fake, 1 << 30, None)
    assert st == 1 and b"tau" in lib.gbs_last_error()


def test_threshold_mode_workspace_matches_sparse(lib):
    for op in (gb.OP_FWD, gb.OP_DECODE):
        ps = gb.make_params(2, 8, 2, 4096, 128, 64, 16, "sparse")
        pt = gb.make_params(2, 8, 2, 4096, 128, 64, 16, "threshold", tau=0.05)
        assert gb.workspace_bytes(pt, op) == gb.workspace_bytes(ps, op) > 0


def test_null_and_misaligned_pointers_rejected(lib):
    p = gb.make_params(1, 4, 2, 256, 64, 64, 0, "train")
    ok = ctypes.c_void_p(4096)
    bad = ctypes.c_void_p(4100)
    st = lib.gbs_fwd(ctypes.byref(p), None, ok, ok, ok, ok, ok, ok, 1 << 30, None)
    assert st == 1 and b"Q is NULL" in lib.gbs_last_error()
    st = lib.gbs_fwd(ctypes.byref(p), ok, bad, ok, ok, ok, ok, ok, 1 << 30, None)
    assert st == 1 and b"K is not 16-byte aligned" in lib.gbs_last_error()


def test_workspace_checks(lib):
    p = gb.make_params(1, 4, 2, 256, 64, 64, 0, "train")
    ok = ctypes.c_void_p(4096)
    need = gb.workspace_bytes(p, gb.OP_FWD)
    assert lib.gbs_fwd(ctypes.byref(p), ok, ok, ok, ok, ok, ok, None, need, None) == 5
    assert lib.gbs_fwd(ctypes.byref(p), ok, ok, ok, ok, ok, ok, ok, need - 1, None) == 5
    assert lib.gbs_fwd(ctypes.byref(p), ok, ok, ok, ok, ok, ok, ctypes.c_void_p(4096 + 16), need,
                       None) == 5


def test_sparse_backward_workspace(lib):
    """Outside training mode the backward also holds K1's lists, the kept-block
    bitmap and the per-key-tile step lists of the tensor-core path."""
    pt = gb.make_params(1, 32, 8, 65536, 128, 64, 0, "train")
    ps = gb.make_params(1, 32, 8, 65536, 128, 64, 64, "sparse")
    rows, nt = 32 * 1024, 512
    extra = rows * 64 * 8 + rows * 4 + rows * 32 * 4 + 8 * nt * (1 + 4 * nt) * 4
    assert gb.workspace_bytes(ps, gb.OP_BWD) >= gb.workspace_bytes(pt, gb.OP_BWD) + extra
    bad = gb.make_params(1, 4, 2, 256, 64, 64, 4, "threshold", tau=2.0)
    assert gb.workspace_bytes(bad, gb.OP_BWD) == 0


def test_decode_split_bounds(lib):
    p = gb.make_params(2, 4, 2, 1000, 64, 64, 4, "sparse")
    ok = ctypes.c_void_p(4096)
    st = lib.gbs_decode(ctypes.byref(p), ok, ok, ok, ok, ok, ok, 999, ok, 1 << 30, None)
    assert st == 1


@pytest.mark.parametrize("kw", [
    dict(mode=7),                                   # unknown mode
    dict(B=1024, Hq=64, Hkv=8, N=32768),            # 2^31 token rows: 32-bit cache row index
    dict(d=96),                                     # head dim not built
    dict(topk=10_000),                              # budget beyond the limit
    dict(mode="threshold", tau=1.5),                # tau outside (0, 1]
    dict(Hq=6, Hkv=4),                              # Hq not a multiple of Hkv
])
def test_noalloc_decode_rejects_what_decode_rejects(lib, kw):
    """gbs_decode_noalloc validates exactly as gbs_decode does, before any
    device call: same status for every invalid parameter block."""
    args = dict(B=2, Hq=4, Hkv=2, N=1000, d=64, block=64, topk=4, mode="sparse", tau=0.0)
    mode = kw.pop("mode", "sparse")
    args.update(kw)
    p = gb.make_params(**{**args, "mode": "sparse"})
    p.mode = mode if isinstance(mode, int) else gb.MODES[mode]
    ok = ctypes.c_void_p(4096)
    lib.gbs_decode_noalloc.restype = ctypes.c_int
    st_ws = lib.gbs_decode(ctypes.byref(p), ok, ok, ok, ok, ok, ok, 1, ok, 1 << 30, None)
    st_na = lib.gbs_decode_noalloc(ctypes.byref(p), ok, ok, ok, ok, ok, ok, 1, None)
    assert st_ws == st_na != 0, (st_ws, st_na, lib.gbs_last_error())


def test_noalloc_decode_split_bounds(lib):
    p = gb.make_params(2, 4, 2, 1000, 64, 64, 4, "sparse")
    ok = ctypes.c_void_p(4096)
    lib.gbs_decode_noalloc.restype = ctypes.c_int
    for splits in (-1, 33):
        assert lib.gbs_decode_noalloc(ctypes.byref(p), ok, ok, ok, ok, ok, ok, splits, None) == 1


def test_binding_fails_loudly_without_library(tmp_path):
    saved = gb._lib
    gb._lib = None
    try:
        with pytest.raises(RuntimeError):
            gb.load_library(str(tmp_path / "missing.so"))
    finally:
        gb._lib = saved


@pytest.mark.parametrize("field,value", [("max_blocks", 3), ("num_pages", 0), ("group_shared", 2),
                                         ("num_pages", 1 << 25)])  # 2^25 pages x 2 heads x 64 rows
def test_decode_ex_layout_checks(lib, field, value):
    """Paged-layout fields are checked before any launch."""
    p = gb.make_params(2, 8, 2, 1000, 64, 64, 4, "sparse")  # Nb = 16
    ok = ctypes.c_void_p(4096)
    kv = gb.KvLayout(4096, 16, 40, None, 0)
    setattr(kv, field, value)
    st = lib.gbs_decode_ex(ctypes.byref(p), ctypes.byref(kv), ok, ok, ok, ok, ok, ok, 0, ok,
                           1 << 30, None)
    assert st == 1, lib.gbs_last_error()


def test_decode_ex_misaligned_tables(lib):
    p = gb.make_params(2, 8, 2, 1000, 64, 64, 4, "sparse")
    ok = ctypes.c_void_p(4096)
    for kv in (gb.KvLayout(4098, 16, 40, None, 0), gb.KvLayout(None, 0, 0, 4098, 0)):
        st = lib.gbs_decode_ex(ctypes.byref(p), ctypes.byref(kv), ok, ok, ok, ok, ok, ok, 0, ok,
                               1 << 30, None)
        assert st == 1 and b"aligned" in lib.gbs_last_error()
