"""Runs one operation of the path a few times, for profilers (ncu) to capture.

    python -m gated_block_sparse_gate_b200.profile_cases --case train_fwd --reps 3
    python -m gated_block_sparse_gate_b200.profile_cases --case train_bwd --reps 3
    python -m gated_block_sparse_gate_b200.profile_cases --case train_bwd --workload train_bf16_n32768
    python -m gated_block_sparse_gate_b200.profile_cases --case sparse_fwd --topk 16 --reps 3
    python -m gated_block_sparse_gate_b200.profile_cases --case sparse_bwd --topk 16 --seq 16384
    python -m gated_block_sparse_gate_b200.profile_cases --case decode --batch 8 --reps 3
    python -m gated_block_sparse_gate_b200.profile_cases --case decode_grouped --batch 8

Inputs are the seeded workloads of ``inputs.py`` (optionally cut down with
--seq / --batch so a capture stays small); every launch goes through the C ABI.
"""
from __future__ import annotations

import argparse
import dataclasses

import torch

from . import binding as gb
from .build import build
from .inputs import WORKLOADS, make_decode_inputs, make_prefill_inputs


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--case", required=True, choices=("train_fwd", "train_bwd", "sparse_fwd",
                                                      "sparse_bwd", "decode", "decode_grouped"))
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--seq", type=int, default=None, help="override N (prefill) or L (decode)")
    ap.add_argument("--batch", type=int, default=None, help="override B (decode)")
    ap.add_argument("--topk", type=int, default=None)
    ap.add_argument("--workload", default=None, help="training workload (default train_bf16_n8192)")
    args = ap.parse_args(argv)
    build()
    gb.load_library()
    dev = torch.device("cuda", 0)
    if args.case in ("decode", "decode_grouped"):
        w = WORKLOADS["sparse_decode_bf16_b64_l131072"]
        B = args.batch or w.B
        L = args.seq or w.N
        w = dataclasses.replace(w, B=B, N=L)
        x = make_decode_inputs(w, device=dev)
        k = args.topk or w.topk[0]
        S = x["S"]
        if args.case == "decode_grouped":  # one score row per kv group
            g = torch.Generator().manual_seed(w.seed + 1)
            S = (torch.randn(B, w.Hkv, w.Nb, generator=g) * 2 ** 0.5).to(dev)
        for _ in range(args.reps):
            gb.decode_ex(x["q"], x["Kc"], x["Vc"], S, L, topk=k,
                         group_shared=args.case == "decode_grouped")
    else:
        sparse = args.case in ("sparse_fwd", "sparse_bwd")
        w = WORKLOADS["sparse_prefill_bf16_n65536" if sparse else
                      (args.workload or "train_bf16_n8192")]
        if args.seq:
            w = dataclasses.replace(w, N=args.seq)
        bwd = args.case in ("train_bwd", "sparse_bwd")
        x = make_prefill_inputs(w, with_grad=bwd)
        d = {k: v.to(dev) for k, v in x.items()}
        mode = "sparse" if sparse else "train"
        k = (args.topk or w.topk[0]) if mode == "sparse" else 0
        O, LSE = gb.forward(d["Q"], d["K"], d["V"], d["S"], mode=mode, topk=k)
        for _ in range(args.reps):
            if bwd:
                gb.backward(d["Q"], d["K"], d["V"], d["S"], O, LSE, d["dO"], mode=mode, topk=k)
            else:
                gb.forward(d["Q"], d["K"], d["V"], d["S"], mode=mode, topk=k, out=O, lse=LSE)
    torch.cuda.synchronize()
    print("ok", args.case)


if __name__ == "__main__":
    main()
