"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

This module holds input recipes only, none of the method's arithmetic. Each
workload draws, from one ``torch.Generator`` seeded with the workload's seed,
in this order: Q, K, V (standard normal, optionally multiplied by d^-1/2),
the selector scores S (normal with variance 2), the optional planted column
boost, and the upstream gradient dO (standard normal). Values are drawn in
fp32 and then cast to the compute dtype, so the oracle reads exactly the values
the kernels read.

The pages publish no datasets or trained selectors for this path, so every
tensor is synthetic with the shapes of the workloads below.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

SCORE_STD = math.sqrt(2.0)  # "N(0,2)" read as variance 2


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    block: int
    dtype: str            # "bf16" or "f32"
    seed: int
    scale_inputs: bool    # Q, K, V multiplied by d^-1/2 before the logit scale
    topk: tuple = ()      # sparse budgets (empty: training mode only)
    plant_frac: float = 0.0
    plant_boost: float = 0.0
    decode: bool = False
    notes: str = field(default="", compare=False)

    @property
    def Nb(self) -> int:
        return -(-self.N // self.block)

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32


WORKLOADS = {
    "tiny_f32_n1024": Workload(
        "tiny_f32_n1024", B=1, Hq=2, Hkv=2, N=1024, d=64, block=64, dtype="f32", seed=0,
        scale_inputs=False, topk=(4,),
        notes="fp32 correctness case: train fwd+bwd and sparse fwd with K=4"),
    "train_bf16_n8192": Workload(
        "train_bf16_n8192", B=1, Hq=32, Hkv=8, N=8192, d=128, block=64, dtype="bf16", seed=1,
        scale_inputs=True, notes="training mode, Llama-8B-like GQA shape"),
    "train_bf16_n32768": Workload(
        "train_bf16_n32768", B=1, Hq=32, Hkv=8, N=32768, d=128, block=64, dtype="bf16", seed=2,
        scale_inputs=True, notes="long-context training mode, 512 blocks"),
    "sparse_prefill_bf16_n65536": Workload(
        "sparse_prefill_bf16_n65536", B=1, Hq=32, Hkv=8, N=65536, d=128, block=64, dtype="bf16",
        seed=3, scale_inputs=True, topk=(8, 16, 32, 64), plant_frac=0.10, plant_boost=3.0,
        notes="sparse prefill, Top-K sweep, heavy-tailed planted columns"),
    "sparse_decode_bf16_b64_l131072": Workload(
        "sparse_decode_bf16_b64_l131072", B=64, Hq=32, Hkv=8, N=131072, d=128, block=64,
        dtype="bf16", seed=4, scale_inputs=True, topk=(32,), decode=True,
        notes="sparse decode, one query per sequence, K=32"),
}


def _qkv_scale(w: Workload) -> float:
    return w.d ** -0.5 if w.scale_inputs else 1.0


def make_prefill_inputs(w: Workload, N: int | None = None, Hq: int | None = None,
                        Hkv: int | None = None, B: int | None = None, with_grad: bool = True,
                        scale_inputs: bool | None = None, device="cpu"):
    """Q, K, V [B,H,N,d], S [B,Hq,Nb,Nb] fp32 and dO, drawn in the fixed order.

    Overrides of N / heads / batch give smaller cases of the same recipe.
    Returns a dict of CPU (or ``device``) tensors; Q/K/V/dO in the workload's
    dtype, S in fp32.
    """
    B = w.B if B is None else B
    Hq = w.Hq if Hq is None else Hq
    Hkv = w.Hkv if Hkv is None else Hkv
    N = w.N if N is None else N
    scl = _qkv_scale(w) if scale_inputs is None else (w.d ** -0.5 if scale_inputs else 1.0)
    Nb = -(-N // w.block)
    g = torch.Generator(device="cpu").manual_seed(w.seed)
    Q = torch.randn(B, Hq, N, w.d, generator=g) * scl
    K = torch.randn(B, Hkv, N, w.d, generator=g) * scl
    V = torch.randn(B, Hkv, N, w.d, generator=g) * scl
    S = torch.randn(B, Hq, Nb, Nb, generator=g) * SCORE_STD
    if w.plant_frac > 0:
        n_plant = max(1, round(w.plant_frac * Nb))
        for b in range(B):
            for h in range(Hq):
                cols = torch.randperm(Nb, generator=g)[:n_plant]
                S[b, h, :, cols] += w.plant_boost
    out = {"Q": Q, "K": K, "V": V, "S": S}
    if with_grad:
        out["dO"] = torch.randn(B, Hq, N, w.d, generator=g)
    dt = w.torch_dtype
    for k in ("Q", "K", "V", "dO"):
        if k in out:
            out[k] = out[k].to(dt).contiguous()
    out["S"] = out["S"].contiguous()
    if device != "cpu":
        out = {k: v.to(device) for k, v in out.items()}
    return out


def make_decode_inputs(w: Workload, B: int | None = None, L: int | None = None,
                       device="cpu"):
    """q [B,Hq,d], Kc/Vc [B,Hkv,L,d], S_dec [B,Hq,Nb] for one-token decode.

    Each sequence b draws from its own generator seeded (seed, b), on
    ``device``, in the order Kc[b], Vc[b]; q and S come from a generator seeded
    with the workload seed. Large caches are therefore made on the GPU, and a
    checked subset of sequences is copied back for the oracle.
    """
    B = w.B if B is None else B
    L = w.N if L is None else L
    Nb = -(-L // w.block)
    scl = _qkv_scale(w)
    dt = w.torch_dtype
    g = torch.Generator(device="cpu").manual_seed(w.seed)
    q = (torch.randn(B, w.Hq, w.d, generator=g) * scl).to(dt)
    S = torch.randn(B, w.Hq, Nb, generator=g) * SCORE_STD
    Kc = torch.empty(B, w.Hkv, L, w.d, dtype=dt, device=device)
    Vc = torch.empty(B, w.Hkv, L, w.d, dtype=dt, device=device)
    for b in range(B):
        gb = torch.Generator(device=device).manual_seed(w.seed * 1_000_003 + b)
        for t in (Kc, Vc):
            for h in range(w.Hkv):
                x = torch.randn(L, w.d, generator=gb, device=device) * scl
                t[b, h].copy_(x.to(dt))
    return {"q": q.to(device).contiguous(), "Kc": Kc, "Vc": Vc, "S": S.to(device).contiguous()}
