"""Runs one operation of the path a few times, for profilers (ncu) to capture.

    python -m gated_block_sparse_gate_b200.profile_cases --case train_fwd --reps 3
    python -m gated_block_sparse_gate_b200.profile_cases --case train_bwd --reps 3
    python -m gated_block_sparse_gate_b200.profile_cases --case sparse_fwd --topk 16 --reps 3
    python -m gated_block_sparse_gate_b200.profile_cases --case decode --batch 8 --reps 3

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
    ap.add_argument("--case", required=True, choices=("train_fwd", "train_bwd", "sparse_fwd", "decode"))
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--seq", type=int, default=None, help="override N (prefill) or L (decode)")
    ap.add_argument("--batch", type=int, default=None, help="override B (decode)")
    ap.add_argument("--topk", type=int, default=None)
    args = ap.parse_args(argv)
    build()
    gb.load_library()
    dev = torch.device("cuda", 0)
    if args.case == "decode":
        w = WORKLOADS["sparse_decode_bf16_b64_l131072"]
        B = args.batch or w.B
        L = args.seq or w.N
        w = dataclasses.replace(w, B=B, N=L)
        x = make_decode_inputs(w, device=dev)
        k = args.topk or w.topk[0]
        for _ in range(args.reps):
            gb.decode(x["q"], x["Kc"], x["Vc"], x["S"], topk=k)
    else:
        name = "sparse_prefill_bf16_n65536" if args.case == "sparse_fwd" else "train_bf16_n8192"
        w = WORKLOADS[name]
        if args.seq:
            w = dataclasses.replace(w, N=args.seq)
        x = make_prefill_inputs(w, with_grad=args.case == "train_bwd")
        d = {k: v.to(dev) for k, v in x.items()}
        mode = "sparse" if args.case == "sparse_fwd" else "train"
        k = (args.topk or w.topk[0]) if mode == "sparse" else 0
        O, LSE = gb.forward(d["Q"], d["K"], d["V"], d["S"], mode=mode, topk=k)
        for _ in range(args.reps):
            if args.case == "train_bwd":
                gb.backward(d["Q"], d["K"], d["V"], d["S"], O, LSE, d["dO"])
            else:
                gb.forward(d["Q"], d["K"], d["V"], d["S"], mode=mode, topk=k, out=O, lse=LSE)
    torch.cuda.synchronize()
    print("ok", args.case)


if __name__ == "__main__":
    main()
