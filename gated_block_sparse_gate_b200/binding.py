"""Thin ctypes binding over libgbs.so (the C ABI in include/gbs.h).

Argument marshalling only: torch tensors supply device memory and the current
stream; every step of the computation runs in the library's CUDA kernels.
There is no fallback: if the library or a CUDA device is missing, calls raise.
"""
from __future__ import annotations

import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libgbs.so")

GBS_OK = 0
STATUS_NAMES = {0: "GBS_OK", 1: "GBS_ERR_INVALID_ARG", 2: "GBS_ERR_UNSUPPORTED", 3: "GBS_ERR_CUDA",
                4: "GBS_ERR_TIMEOUT", 5: "GBS_ERR_WORKSPACE", 6: "GBS_ERR_DEVICE_CHECK"}
MODES = {"train": 0, "sparse": 1, "threshold": 2}
DTYPES = {torch.bfloat16: 0, torch.float32: 1}
OP_FWD, OP_BWD, OP_DECODE = 0, 1, 2

EXPORTED = ("gbs_version", "gbs_status_string", "gbs_last_error", "gbs_workspace_bytes",
            "gbs_clear_error", "gbs_check", "gbs_select", "gbs_fwd", "gbs_bwd", "gbs_decode",
            "gbs_set_timer", "gbs_launch_count", "gbs_selftest_wait_timeout")


class GbsError(RuntimeError):
    def __init__(self, status, where, detail=""):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} {detail}".strip())


class Params(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
                ("N", ctypes.c_int), ("d", ctypes.c_int), ("block", ctypes.c_int),
                ("topk", ctypes.c_int), ("mode", ctypes.c_int), ("dtype", ctypes.c_int),
                ("scale", ctypes.c_float), ("tau", ctypes.c_float)]


class KvLayout(ctypes.Structure):
    """gbs_kv_layout: paged / variable-length cache and group-shared selection."""
    _fields_ = [("block_table", ctypes.c_void_p), ("max_blocks", ctypes.c_int),
                ("num_pages", ctypes.c_int), ("seq_lens", ctypes.c_void_p),
                ("group_shared", ctypes.c_int)]


_lib = None


def load_library(path: str = LIB_PATH):
    """Loads libgbs.so and declares the argument types of every entry point."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing; build it with gated_block_sparse_gate_b200.build")
    lib = ctypes.CDLL(path)
    P = ctypes.POINTER(Params)
    vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    sigs = {
        "gbs_version": (i32, []),
        "gbs_status_string": (ctypes.c_char_p, [i32]),
        "gbs_last_error": (ctypes.c_char_p, []),
        "gbs_workspace_bytes": (sz, [P, i32]),
        "gbs_clear_error": (i32, [vp, vp]),
        "gbs_check": (i32, [vp, vp]),
        "gbs_select": (i32, [P, vp, vp, vp, vp, vp, vp]),
        "gbs_fwd": (i32, [P, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "gbs_bwd": (i32, [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "gbs_decode": (i32, [P, vp, vp, vp, vp, vp, vp, i32, vp, sz, vp]),
        "gbs_decode_ex": (i32, [P, ctypes.POINTER(KvLayout), vp, vp, vp, vp, vp, vp, i32, vp, sz,
                                vp]),
        "gbs_set_timer": (i32, [i32, vp, vp]),
        "gbs_launch_count": (ctypes.c_uint64, []),
    }
    for name, (res, args) in sigs.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def _check(status, where):
    if status != GBS_OK:
        detail = load_library().gbs_last_error().decode()
        raise GbsError(status, where, detail)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


# Device types whose memory the kernels may be given; only the unit tests of
# the checks below widen it (to "meta", which has shapes but no storage).
_DEVICE_TYPES = ("cuda",)
_F32 = (torch.float32,)
_I32 = (torch.int32,)
_U8 = (torch.uint8,)


def _invalid(where, detail):
    return GbsError(1, where, detail)


def _device(where, name, t):
    """The device of the call's anchor tensor, which must be a CUDA tensor."""
    if not isinstance(t, torch.Tensor):
        raise _invalid(where, f"{name} must be a torch.Tensor")
    if t.device.type not in _DEVICE_TYPES:
        raise _invalid(where, f"{name} is on {t.device}; the kernels need CUDA memory")
    return t.device


def _need(where, name, t, shape, dtypes, device):
    """t is a contiguous tensor on ``device`` with one of ``dtypes`` and, unless
    ``shape`` is None, exactly that shape: the layout the C ABI reads."""
    if not isinstance(t, torch.Tensor):
        raise _invalid(where, f"{name} must be a torch.Tensor")
    if t.device != device:
        raise _invalid(where, f"{name} is on {t.device}; expected {device}")
    if t.dtype not in dtypes:
        raise _invalid(where, f"{name} has dtype {t.dtype}; expected {' or '.join(map(str, dtypes))}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise _invalid(where, f"{name} has shape {tuple(t.shape)}; expected {tuple(shape)}")
    if not t.is_contiguous():
        raise _invalid(where, f"{name} must be contiguous")


def _act_dtype(where, name, t):
    if t.dtype not in DTYPES:
        raise _invalid(where, f"{name} has dtype {t.dtype}; expected torch.bfloat16 or torch.float32")
    return (t.dtype,)


def _check_prefill(where, Q, K, V, S, block, outs=()):
    """Q [B,Hq,N,d], K and V [B,Hkv,N,d] of Q's dtype, S [B,Hq,Nb,Nb] fp32, and
    each (name, tensor, shape, dtypes) of ``outs``; returns (device, shape dict)."""
    dev = _device(where, "Q", Q)
    if Q.dim() != 4 or not isinstance(K, torch.Tensor) or K.dim() != 4:
        raise _invalid(where, "Q and K must be 4-D: [B, H, N, d]")
    B, Hq, N, d = Q.shape
    Hkv = K.shape[1]
    Nb = -(-N // block)
    act = _act_dtype(where, "Q", Q)
    _need(where, "Q", Q, (B, Hq, N, d), act, dev)
    _need(where, "K", K, (B, Hkv, N, d), act, dev)
    _need(where, "V", V, (B, Hkv, N, d), act, dev)
    _need(where, "S", S, (B, Hq, Nb, Nb), _F32, dev)
    for name, t, shape, dtypes in outs:
        _need(where, name, t, shape, dtypes, dev)
    return dev


def _check_decode(where, q, Kc, Vc, S, L, block, block_table=None, seq_lens=None,
                  group_shared=False, outs=()):
    """q [B,Hq,d]; a cache [B,Hkv,L,d] or, with a block table, page pools
    [pages,Hkv,block,d]; S [B,Hq,Nb] (group-shared: [B,Hkv,Nb]) fp32; an int32
    block table [B, max_blocks] and int32 lengths [B]."""
    dev = _device(where, "q", q)
    if q.dim() != 3 or not isinstance(Kc, torch.Tensor) or Kc.dim() != 4:
        raise _invalid(where, "q must be [B, Hq, d] and the cache 4-D")
    B, Hq, d = q.shape
    Hkv = Kc.shape[1]
    Nb = -(-L // block)
    act = _act_dtype(where, "q", q)
    _need(where, "q", q, (B, Hq, d), act, dev)
    cache = (Kc.shape[0], Hkv, block, d) if block_table is not None else (B, Hkv, L, d)
    _need(where, "Kc", Kc, cache, act, dev)
    _need(where, "Vc", Vc, cache, act, dev)
    _need(where, "S", S, (B, Hkv if group_shared else Hq, Nb), _F32, dev)
    if block_table is not None:
        _need(where, "block_table", block_table, None, _I32, dev)
        if block_table.dim() != 2 or block_table.shape[0] != B:
            raise _invalid(where, f"block_table must be [B={B}, max_blocks]")
    if seq_lens is not None:
        _need(where, "seq_lens", seq_lens, (B,), _I32, dev)
    for name, t, shape, dtypes in outs:
        _need(where, name, t, shape, dtypes, dev)
    return dev


def make_params(B, Hq, Hkv, N, d, block=64, topk=0, mode="train", dtype=torch.bfloat16, scale=0.0,
                tau=0.0):
    return Params(B, Hq, Hkv, N, d, block, topk, MODES[mode], DTYPES[dtype], float(scale),
                  float(tau))


def workspace_bytes(params: Params, op: int) -> int:
    return int(load_library().gbs_workspace_bytes(ctypes.byref(params), op))


def alloc_workspace(params: Params, op: int, device) -> torch.Tensor:
    n = workspace_bytes(params, op)
    if n == 0:
        raise GbsError(1, "workspace_bytes", load_library().gbs_last_error().decode())
    ws = torch.zeros(n, dtype=torch.uint8, device=device)
    assert ws.data_ptr() % 256 == 0
    return ws


def _prefill_params(Q, K, S, block, topk, mode, scale, tau=0.0):
    B, Hq, N, d = Q.shape
    return make_params(B, Hq, K.shape[1], N, d, block, topk, mode, Q.dtype, scale, tau)


def select(S, block=64, topk=0, mode="sparse", N=None, tau=0.0, stream=None):
    """K1: (idx, cnt, logg, slse) for S [B, Hq, Nb, Nb]."""
    lib = load_library()
    dev = _device("gbs_select", "S", S)
    if S.dim() != 4:
        raise _invalid("gbs_select", "S must be [B, Hq, Nb, Nb]")
    B, Hq, Nb, _ = S.shape
    _need("gbs_select", "S", S, (B, Hq, Nb, Nb), _F32, dev)
    N = N if N is not None else Nb * block
    p = make_params(B, Hq, Hq, N, 64, block, topk, mode, torch.float32, tau=tau)
    idx = cnt = logg = None
    if mode != "train":
        idx = torch.empty(B, Hq, Nb, topk, dtype=torch.int32, device=dev)
        cnt = torch.empty(B, Hq, Nb, dtype=torch.int32, device=dev)
        logg = torch.empty(B, Hq, Nb, topk, dtype=torch.float32, device=dev)
    slse = torch.empty(B, Hq, Nb, dtype=torch.float32, device=dev)
    _check(lib.gbs_select(ctypes.byref(p), _ptr(S), _ptr(idx), _ptr(cnt), _ptr(logg), _ptr(slse),
                          _stream(stream)), "gbs_select")
    return idx, cnt, logg, slse


def forward(Q, K, V, S, block=64, mode="train", topk=0, scale=0.0, out=None, lse=None, ws=None,
            tau=0.0, stream=None):
    """Gated attention forward: returns (O, LSE)."""
    lib = load_library()
    _check_prefill("gbs_fwd", Q, K, V, S, block)
    p = _prefill_params(Q, K, S, block, topk, mode, scale, tau)
    O = out if out is not None else torch.empty_like(Q)
    LSE = lse if lse is not None else torch.empty(Q.shape[:3], dtype=torch.float32, device=Q.device)
    if ws is None:
        ws = alloc_workspace(p, OP_FWD, Q.device)
    _check_prefill("gbs_fwd", Q, K, V, S, block,
                   outs=(("O", O, Q.shape, (Q.dtype,)), ("LSE", LSE, Q.shape[:3], _F32),
                         ("ws", ws, None, _U8)))
    _check(lib.gbs_fwd(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(S), _ptr(O), _ptr(LSE),
                       _ptr(ws), ws.numel(), _stream(stream)), "gbs_fwd")
    return O, LSE


def backward(Q, K, V, S, O, LSE, dO, block=64, scale=0.0, grads=None, ws=None, mode="train",
             topk=0, tau=0.0, stream=None):
    """Backward of ``forward`` with the same mode/topk/tau: returns (dQ, dK, dV, dS)."""
    lib = load_library()
    _check_prefill("gbs_bwd", Q, K, V, S, block)
    p = _prefill_params(Q, K, S, block, topk, mode, scale, tau)
    if grads is None:
        grads = (torch.empty_like(Q), torch.empty_like(K), torch.empty_like(V), torch.empty_like(S))
    dQ, dK, dV, dS = grads
    if ws is None:
        ws = alloc_workspace(p, OP_BWD, Q.device)
    act = (Q.dtype,)
    _check_prefill("gbs_bwd", Q, K, V, S, block,
                   outs=(("O", O, Q.shape, act), ("LSE", LSE, Q.shape[:3], _F32),
                         ("dO", dO, Q.shape, act), ("dQ", dQ, Q.shape, act),
                         ("dK", dK, K.shape, act), ("dV", dV, V.shape, act),
                         ("dS", dS, S.shape, _F32), ("ws", ws, None, _U8)))
    _check(lib.gbs_bwd(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(S), _ptr(O), _ptr(LSE),
                       _ptr(dO), _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(dS), _ptr(ws), ws.numel(),
                       _stream(stream)), "gbs_bwd")
    return dQ, dK, dV, dS


def decode(q, Kc, Vc, S, L=None, block=64, topk=32, scale=0.0, num_splits=0, out=None, lse=None,
           ws=None, tau=None, stream=None):
    """Sparse one-token decode: returns (O [B,Hq,d], LSE [B,Hq]).

    ``tau`` set selects threshold mode (blocks whose gate reaches tau, at most topk).
    """
    lib = load_library()
    L = Kc.shape[2] if L is None else L
    _check_decode("gbs_decode", q, Kc, Vc, S, L, block)
    B, Hq, d = q.shape
    mode = "sparse" if tau is None else "threshold"
    p = make_params(B, Hq, Kc.shape[1], L, d, block, topk, mode, q.dtype, scale,
                    0.0 if tau is None else tau)
    O = out if out is not None else torch.empty_like(q)
    LSE = lse if lse is not None else torch.empty(B, Hq, dtype=torch.float32, device=q.device)
    if ws is None:
        ws = alloc_workspace(p, OP_DECODE, q.device)
    _check_decode("gbs_decode", q, Kc, Vc, S, L, block,
                  outs=(("O", O, q.shape, (q.dtype,)), ("LSE", LSE, (B, Hq), _F32),
                        ("ws", ws, None, _U8)))
    _check(lib.gbs_decode(ctypes.byref(p), _ptr(q), _ptr(Kc), _ptr(Vc), _ptr(S), _ptr(O), _ptr(LSE),
                          num_splits, _ptr(ws), ws.numel(), _stream(stream)), "gbs_decode")
    return O, LSE


def decode_ex(q, Kc, Vc, S, L, block=64, topk=32, scale=0.0, num_splits=0, block_table=None,
              seq_lens=None, group_shared=False, out=None, lse=None, ws=None, tau=None,
              stream=None):
    """gbs_decode_ex: decode over a paged and/or variable-length cache, with one
    selection per q-head or per kv group. ``L`` is the maximum length; with
    ``block_table`` (int32 [B, max_blocks]) Kc/Vc are page pools
    [num_pages, Hkv, block, d]; ``seq_lens`` (int32 [B]) gives each length;
    with ``group_shared`` S is [B, Hkv, Nb]. Returns (O, LSE)."""
    lib = load_library()
    _check_decode("gbs_decode_ex", q, Kc, Vc, S, L, block, block_table, seq_lens, group_shared)
    B, Hq, d = q.shape
    mode = "sparse" if tau is None else "threshold"
    p = make_params(B, Hq, Kc.shape[1], L, d, block, topk, mode, q.dtype, scale,
                    0.0 if tau is None else tau)
    kv = KvLayout(None if block_table is None else block_table.data_ptr(),
                  0 if block_table is None else block_table.shape[1],
                  0 if block_table is None else Kc.shape[0],
                  None if seq_lens is None else seq_lens.data_ptr(), 1 if group_shared else 0)
    O = out if out is not None else torch.empty_like(q)
    LSE = lse if lse is not None else torch.empty(B, Hq, dtype=torch.float32, device=q.device)
    if ws is None:
        ws = alloc_workspace(p, OP_DECODE, q.device)
    _check_decode("gbs_decode_ex", q, Kc, Vc, S, L, block, block_table, seq_lens, group_shared,
                  outs=(("O", O, q.shape, (q.dtype,)), ("LSE", LSE, (B, Hq), _F32),
                        ("ws", ws, None, _U8)))
    _check(lib.gbs_decode_ex(ctypes.byref(p), ctypes.byref(kv), _ptr(q), _ptr(Kc), _ptr(Vc), _ptr(S),
                             _ptr(O), _ptr(LSE), num_splits, _ptr(ws), ws.numel(), _stream(stream)),
           "gbs_decode_ex")
    return O, LSE


def set_timer(op: int, start=None, stop=None):
    """Brackets the main kernel of ``op`` with two recorded torch.cuda.Events.

    The events must already exist on the device (record them once first).
    Pass None to clear.
    """
    h0 = None if start is None else ctypes.c_void_p(start.cuda_event)
    h1 = None if stop is None else ctypes.c_void_p(stop.cuda_event)
    _check(load_library().gbs_set_timer(op, h0, h1), "gbs_set_timer")


def launch_count() -> int:
    """Kernels launched by the library so far in this process."""
    return int(load_library().gbs_launch_count())


def check(ws, stream=None):
    """Raises GbsError if a kernel recorded a device-side error in ``ws``."""
    _device("gbs_check", "ws", ws)
    _check(load_library().gbs_check(_ptr(ws), _stream(stream)), "gbs_check")


def clear_error(ws, stream=None):
    """Clears the device error word of ``ws`` (asynchronous)."""
    _device("gbs_clear_error", "ws", ws)
    _check(load_library().gbs_clear_error(_ptr(ws), _stream(stream)), "gbs_clear_error")


def selftest_wait_timeout(ws, limit_us, stream=None):
    """gbs_selftest_wait_timeout: one bounded device wait that nothing releases;
    after ``limit_us`` it records GBS_ERR_TIMEOUT in the error word of ``ws``."""
    lib = load_library()
    f = lib.gbs_selftest_wait_timeout
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_uint, ctypes.c_void_p]
    _device("gbs_selftest_wait_timeout", "ws", ws)
    _check(f(_ptr(ws), int(limit_us), _stream(stream)), "gbs_selftest_wait_timeout")


def decode_noalloc(q, Kc, Vc, S, L=None, block=64, topk=32, scale=0.0, num_splits=0, out=None,
                   lse=None, tau=None, stream=None):
    """gbs_decode_noalloc: the decode with the library's own static scratch.

    For callers that cannot allocate device memory while decoding; see
    include/gbs.h for the limits and the sharing rules.
    """
    lib = load_library()
    f = lib.gbs_decode_noalloc
    vp = ctypes.c_void_p
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.POINTER(Params), vp, vp, vp, vp, vp, vp, ctypes.c_int, vp]
    L = Kc.shape[2] if L is None else L
    _check_decode("gbs_decode_noalloc", q, Kc, Vc, S, L, block)
    B, Hq, d = q.shape
    mode = "sparse" if tau is None else "threshold"
    p = make_params(B, Hq, Kc.shape[1], L, d, block, topk, mode, q.dtype, scale,
                    0.0 if tau is None else tau)
    O = out if out is not None else torch.empty_like(q)
    LSE = lse if lse is not None else torch.empty(B, Hq, dtype=torch.float32, device=q.device)
    _check_decode("gbs_decode_noalloc", q, Kc, Vc, S, L, block,
                  outs=(("O", O, q.shape, (q.dtype,)), ("LSE", LSE, (B, Hq), _F32)))
    _check(f(ctypes.byref(p), _ptr(q), _ptr(Kc), _ptr(Vc), _ptr(S), _ptr(O), _ptr(LSE), num_splits,
             _stream(stream)), "gbs_decode_noalloc")
    return O, LSE
