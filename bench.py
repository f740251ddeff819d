#!/usr/bin/env python3
"""Benchmark of the gated block-sparse attention hot path on B200.

Headline: one training step of the hot path (gate normalisation, gated
forward, gated backward with dS) on the long-context training workload
B=1, Hq=32, Hkv=8, d=128, N=32768 (512 blocks), block 64, bf16, inputs
resident in HBM, L2 flushed between steps, device-timed with CUDA events. The
metric is algorithmic TFLOP/s (attended pairs only: fwd 4*d*P, fwd+bwd
14*d*P). The N=8192 training step, the sparse prefill and the decode are
reported under "extra".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (torchrun): every rank runs its own shard of independent
(batch, kv-head) problems (no data-path collective); the step time is the max
over ranks and `value` counts the work of all ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from gated_block_sparse_gate_b200 import dist as gdist  # noqa: E402
from gated_block_sparse_gate_b200.inputs import WORKLOADS, make_decode_inputs, make_prefill_inputs  # noqa: E402

METRIC = "gated sparse attention TFLOP/s (fwd+bwd and fwd) and % of bf16 tensor peak"
UNIT = "TFLOP/s"
HEADLINE = "train_bf16_n32768"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20


# ------------------------------------------------------------------ work model

def train_pairs_per_head(Nb: int, bs: int) -> int:
    """Attended (i, j) pairs of one head in training mode."""
    return bs * bs * Nb * (Nb - 1) // 2 + Nb * bs * (bs + 1) // 2


def sparse_pairs_per_head(Nb: int, bs: int, k: int) -> int:
    """Attended pairs of one head with a Top-K budget of k historical blocks."""
    hist = sum(min(k, r) for r in range(Nb))
    return bs * bs * hist + Nb * bs * (bs + 1) // 2


def decode_union_blocks(S, cur: int, k: int, G: int) -> int:
    """Distinct K/V blocks one decode step must read: per (sequence, kv group),
    the union of its q-heads' Top-K historical blocks, plus the current block.

    S is the per-q-head score tensor [B, Hq, Nb] (on any device); selection
    follows the decode's rule (the k largest scores among blocks 0 .. cur-1).
    Byte accounting only: which rows tie is irrelevant to the count for these
    continuous scores."""
    B, Hq = S.shape[:2]
    kk = min(k, cur)
    n_groups = B * (Hq // G)
    if kk == 0:
        return n_groups
    top = torch.topk(S[..., :cur], kk, dim=-1).indices
    mark = torch.zeros(B, Hq // G, cur, dtype=torch.bool, device=S.device)
    mark.scatter_(2, top.reshape(B, Hq // G, G * kk), True)
    return int(mark.sum().item()) + n_groups


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return {k: float(pk[k]) for k in FALLBACK_PEAKS}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def traffic_for(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if still current.

    profiles/traffic.json maps "kernel/workload" to the bytes ncu measured for
    one launch on that workload and the SHA-256 of the source file it was
    measured from; a changed source voids it.
    """
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            entry = json.load(f)[f"{kernel}/{workload}"]
        src = os.path.join(ROOT, entry["source"])
        with open(src, "rb") as f:
            if hashlib.sha256(f.read()).hexdigest() != entry["sha256"]:
                return None
        return float(entry["bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


# --------------------------------------------------------------------- clocks

class ClockSampler:
    """Samples nvidia-smi SM clocks and throttle reasons during a region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.device = device
        self.proc = None
        self.path = None

    def start(self):
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(self.device).uuid)
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", uuid],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, RuntimeError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------- our arm

def _events(n):
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    for e in ev:
        e.record()  # creates the underlying cudaEvent_t
    return ev


def bench_training(w, steps, warmup, rank, dev, peaks):
    from gated_block_sparse_gate_b200 import binding as gb

    seed = gdist.shard_seed(w.seed, rank)
    x = make_prefill_inputs(w.__class__(**{**w.__dict__, "seed": seed}))
    d = {k: v.to(dev) for k, v in x.items()}
    Q, K, V, S, dO = d["Q"], d["K"], d["V"], d["S"], d["dO"]
    pf = gb.make_params(w.B, w.Hq, w.Hkv, w.N, w.d, w.block, 0, "train", Q.dtype)
    ws_f = gb.alloc_workspace(pf, gb.OP_FWD, dev)
    ws_b = gb.alloc_workspace(pf, gb.OP_BWD, dev)
    O = torch.empty_like(Q)
    LSE = torch.empty(Q.shape[:3], dtype=torch.float32, device=dev)
    grads = (torch.empty_like(Q), torch.empty_like(K), torch.empty_like(V), torch.empty_like(S))
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def step():
        gb.forward(Q, K, V, S, mode="train", out=O, lse=LSE, ws=ws_f)
        gb.backward(Q, K, V, S, O, LSE, dO, grads=grads, ws=ws_b)

    for _ in range(warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()

    ev0, ev1 = _events(steps), _events(steps)
    f0, f1, b0, b1 = _events(steps), _events(steps), _events(steps), _events(steps)
    torch.cuda.synchronize()
    clocks = ClockSampler(dev.index)
    clocks.start()
    gdist.barrier()
    torch.cuda.synchronize()
    n0 = gb.launch_count()
    for k in range(steps):
        flush.zero_()
        gb.set_timer(gb.OP_FWD, f0[k], f1[k])
        gb.set_timer(gb.OP_BWD, b0[k], b1[k])
        ev0[k].record()
        step()
        ev1[k].record()
    torch.cuda.synchronize()
    gdist.barrier()
    launches = gb.launch_count() - n0
    gb.set_timer(gb.OP_FWD)
    gb.set_timer(gb.OP_BWD)
    clk = clocks.stop()
    gb.check(ws_f)
    gb.check(ws_b)

    step_ms = [a.elapsed_time(b) for a, b in zip(ev0, ev1)]
    fwd_ms = [a.elapsed_time(b) for a, b in zip(f0, f1)]
    bwd_ms = [a.elapsed_time(b) for a, b in zip(b0, b1)]
    P = train_pairs_per_head(w.Nb, w.block) * w.B * w.Hq
    fl_fwd, fl_fb = 4.0 * w.d * P, 14.0 * w.d * P
    ms = statistics.mean(step_ms)
    kern = {
        "fwd_tc2_kernel": {"ms": statistics.mean(fwd_ms), "flops": fl_fwd},
        "bwd_tc_kernel": {"ms": statistics.mean(bwd_ms), "flops": fl_fb - fl_fwd},
    }
    dom = max(kern, key=lambda n: kern[n]["ms"])
    ach = kern[dom]["flops"] / (kern[dom]["ms"] * 1e-3) / 1e12
    tr = traffic_for(dom, w.name)
    roof = {"bound": "tensor", "kernel": dom, "achieved": ach, "peak": peaks["bf16_tflops"],
            "unit": "TFLOP/s", "frac": ach / peaks["bf16_tflops"],
            "peak_sustained": peaks["bf16_tflops_sustained"],
            "frac_of_sustained": ach / peaks["bf16_tflops_sustained"],
            "traffic": tr, "traffic_unit": "bytes per launch",
            "flops_per_launch": kern[dom]["flops"], "launch_ms": kern[dom]["ms"]}
    res = dict(ms=ms, flops=fl_fb, fl_fwd=fl_fwd, launches=launches, clocks=clk, roofline=roof,
               fwd_ms=statistics.mean(fwd_ms), bwd_ms=statistics.mean(bwd_ms),
               per_step_launches=launches / steps)

    # End to end through the public API: every step copies its inputs in from
    # pinned host memory and all of its results (O, LSE, dQ, dK, dV, dS) back
    # out. Steps are pipelined over two device buffer sets on three streams
    # (host-to-device, compute, device-to-host), so step k's compute overlaps
    # the input copy of step k+1 and the result copy of step k-1; the time is
    # the whole run's, from the first input copy to the last result copy.
    names = ("Q", "K", "V", "S", "dO")
    host_in = {k: x[k].pin_memory() for k in names}
    bufs = [dict(d, O=O, LSE=LSE, grads=grads)]
    bufs.append({**{k: torch.empty_like(d[k]) for k in names}, "O": torch.empty_like(O),
                 "LSE": torch.empty_like(LSE), "grads": tuple(torch.empty_like(t) for t in grads)})
    host_out = [[torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in (O, LSE, *grads)]
                for _ in range(2)]
    s_in, s_cmp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    e_steps = max(3, min(steps, 20))
    in_done, cmp_done, out_done = _events(e_steps), _events(e_steps), _events(e_steps)
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t_start.record(s_in)
    for k in range(e_steps):
        bf = bufs[k % 2]
        with torch.cuda.stream(s_in):
            if k >= 2:
                s_in.wait_event(cmp_done[k - 2])  # step k-2 has finished reading this set
            for n in names:
                bf[n].copy_(host_in[n], non_blocking=True)
            in_done[k].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(in_done[k])
            if k >= 2:
                s_cmp.wait_event(out_done[k - 2])  # step k-2's results are out of this set
            flush.zero_()
            gb.forward(bf["Q"], bf["K"], bf["V"], bf["S"], mode="train", out=bf["O"],
                       lse=bf["LSE"], ws=ws_f, stream=s_cmp)
            gb.backward(bf["Q"], bf["K"], bf["V"], bf["S"], bf["O"], bf["LSE"], bf["dO"],
                        grads=bf["grads"], ws=ws_b, stream=s_cmp)
            cmp_done[k].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(cmp_done[k])
            for h, t in zip(host_out[k % 2], (bf["O"], bf["LSE"], *bf["grads"])):
                h.copy_(t, non_blocking=True)
            out_done[k].record(s_out)
    s_out.wait_event(in_done[e_steps - 1])
    t_end.record(s_out)
    torch.cuda.synchronize()
    e_ms = t_start.elapsed_time(t_end) / e_steps
    # One call on its own: copy in, compute, copy out, on one stream, nothing
    # overlapped (the latency a single step through the API costs).
    bf = bufs[0]
    serial = []
    for k in range(max(3, min(steps, 10))):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record()
        for n in names:
            bf[n].copy_(host_in[n], non_blocking=True)
        gb.forward(bf["Q"], bf["K"], bf["V"], bf["S"], mode="train", out=bf["O"], lse=bf["LSE"],
                   ws=ws_f)
        gb.backward(bf["Q"], bf["K"], bf["V"], bf["S"], bf["O"], bf["LSE"], bf["dO"],
                    grads=bf["grads"], ws=ws_b)
        for h, t in zip(host_out[0], (bf["O"], bf["LSE"], *bf["grads"])):
            h.copy_(t, non_blocking=True)
        b.record()
        torch.cuda.synchronize()
        if k > 0:  # the first call warms the copy paths
            serial.append(a.elapsed_time(b))
    res["e2e"] = {"ms": e_ms, "h2d": sum(t.numel() * t.element_size() for t in host_in.values()),
                  "d2h": sum(t.numel() * t.element_size() for t in host_out[0]),
                  "pipelined": "two buffer sets; the copies of steps k+1 and k-1 overlap step k",
                  "serial_ms": statistics.mean(serial)}
    return res


def bench_training_extra(name, dev, peaks, reps=5):
    """Another training workload's step: forward + backward kernel times."""
    from gated_block_sparse_gate_b200 import binding as gb

    w = WORKLOADS[name]
    x = make_prefill_inputs(w)
    d = {k: v.to(dev) for k, v in x.items()}
    del x
    Q, K, V, S, dO = d["Q"], d["K"], d["V"], d["S"], d["dO"]
    pf = gb.make_params(w.B, w.Hq, w.Hkv, w.N, w.d, w.block, 0, "train", Q.dtype)
    ws_f = gb.alloc_workspace(pf, gb.OP_FWD, dev)
    ws_b = gb.alloc_workspace(pf, gb.OP_BWD, dev)
    O = torch.empty_like(Q)
    LSE = torch.empty(Q.shape[:3], dtype=torch.float32, device=dev)
    grads = (torch.empty_like(Q), torch.empty_like(K), torch.empty_like(V), torch.empty_like(S))
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def step():
        gb.forward(Q, K, V, S, mode="train", out=O, lse=LSE, ws=ws_f)
        gb.backward(Q, K, V, S, O, LSE, dO, grads=grads, ws=ws_b)

    for _ in range(3):
        flush.zero_()
        step()
    a0, a1 = _events(reps), _events(reps)
    f0, f1, b0, b1 = _events(reps), _events(reps), _events(reps), _events(reps)
    torch.cuda.synchronize()
    for i in range(reps):
        flush.zero_()
        gb.set_timer(gb.OP_FWD, f0[i], f1[i])
        gb.set_timer(gb.OP_BWD, b0[i], b1[i])
        a0[i].record()
        step()
        a1[i].record()
    torch.cuda.synchronize()
    gb.set_timer(gb.OP_FWD)
    gb.set_timer(gb.OP_BWD)
    gb.check(ws_f)
    gb.check(ws_b)
    ms = statistics.mean(a.elapsed_time(b) for a, b in zip(a0, a1))
    fms = statistics.mean(a.elapsed_time(b) for a, b in zip(f0, f1))
    bms = statistics.mean(a.elapsed_time(b) for a, b in zip(b0, b1))
    P = train_pairs_per_head(w.Nb, w.block) * w.B * w.Hq
    fl_f, fl_fb = 4.0 * w.d * P, 14.0 * w.d * P
    del d, grads, O
    torch.cuda.empty_cache()
    return {"ms_per_step": ms, "tflops": fl_fb / ms / 1e9,
            "pct_of_bf16_peak": 100.0 * fl_fb / ms / 1e9 / peaks["bf16_tflops"],
            "fwd_kernel_ms": fms, "fwd_kernel_tflops": fl_f / fms / 1e9,
            "bwd_main_ms": bms, "bwd_main_tflops": (fl_fb - fl_f) / bms / 1e9}


def _time_backward(gb, Q, K, V, S, O, LSE, dO, mode, k, tau, dev, flush, reps):
    """Mean whole-call and main-kernel times (ms) of the backward."""
    pb = gb.make_params(1, Q.shape[1], K.shape[1], Q.shape[2], Q.shape[3], 64, k, mode, Q.dtype,
                        tau=tau)
    ws = gb.alloc_workspace(pb, gb.OP_BWD, dev)
    grads = (torch.empty_like(Q), torch.empty_like(K), torch.empty_like(V), torch.empty_like(S))
    kw = dict(mode=mode, topk=k, tau=tau, grads=grads, ws=ws)
    for _ in range(2):
        gb.backward(Q, K, V, S, O, LSE, dO, **kw)
    a0, a1, k0, k1 = _events(reps), _events(reps), _events(reps), _events(reps)
    torch.cuda.synchronize()
    for i in range(reps):
        flush.zero_()
        gb.set_timer(gb.OP_BWD, k0[i], k1[i])
        a0[i].record()
        gb.backward(Q, K, V, S, O, LSE, dO, **kw)
        a1[i].record()
    torch.cuda.synchronize()
    gb.set_timer(gb.OP_BWD)
    gb.check(ws)
    del ws, grads
    return (statistics.mean(a.elapsed_time(b) for a, b in zip(a0, a1)),
            statistics.mean(a.elapsed_time(b) for a, b in zip(k0, k1)))


def bench_sparse_prefill(dev, peaks, reps=5):
    """Sparse prefill N=65536: Top-K sweep (forward, and the sparse backward as
    an extension), and one dynamic-threshold forward (tau=0.01, at most 64)."""
    from gated_block_sparse_gate_b200 import binding as gb

    w = WORKLOADS["sparse_prefill_bf16_n65536"]
    x = make_prefill_inputs(w)
    Q, K, V, S, dO = (x[n].to(dev) for n in ("Q", "K", "V", "S", "dO"))
    del x
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    out = {}
    cases = [(k, "sparse", 0.0) for k in w.topk] + [(64, "threshold", 0.01)]
    for k, mode, tau in cases:
        pf = gb.make_params(w.B, w.Hq, w.Hkv, w.N, w.d, w.block, k, mode, Q.dtype, tau=tau)
        ws = gb.alloc_workspace(pf, gb.OP_FWD, dev)
        O = torch.empty_like(Q)
        LSE = torch.empty(Q.shape[:3], dtype=torch.float32, device=dev)
        fkw = dict(mode=mode, topk=k, tau=tau, out=O, lse=LSE, ws=ws)
        for _ in range(2):
            gb.forward(Q, K, V, S, **fkw)
        a0, a1, k0, k1 = _events(reps), _events(reps), _events(reps), _events(reps)
        torch.cuda.synchronize()
        for i in range(reps):
            flush.zero_()
            gb.set_timer(gb.OP_FWD, k0[i], k1[i])
            a0[i].record()
            gb.forward(Q, K, V, S, **fkw)
            a1[i].record()
        torch.cuda.synchronize()
        gb.set_timer(gb.OP_FWD)
        gb.check(ws)
        ms = statistics.mean(a.elapsed_time(b) for a, b in zip(a0, a1))
        kms = statistics.mean(a.elapsed_time(b) for a, b in zip(k0, k1))
        if mode == "sparse":
            P = sparse_pairs_per_head(w.Nb, w.block, k) * w.B * w.Hq
        else:  # the kept counts of this S, from K1
            _, cnt, _, _ = gb.select(S, topk=k, mode=mode, tau=tau)
            P = int(cnt.sum().item()) * w.block * w.block + w.Nb * w.B * w.Hq * w.block * (w.block + 1) // 2
        fl = 4.0 * w.d * P
        comp_bytes = (Q.numel() * 2 * 2 + K.numel() * 2 * 2 + S.numel() * 4)
        t_roof = max(fl / (peaks["bf16_tflops"] * 1e12), comp_bytes / (peaks["hbm_gbs"] * 1e9))
        name = f"K{k}" if mode == "sparse" else f"tau{tau:g}_K{k}"
        out[name] = {"ms": ms, "tflops": fl / ms / 1e9, "kernel_ms": kms,
                     "kernel_tflops": fl / kms / 1e9, "frac_of_roofline": t_roof / (kms * 1e-3),
                     "attended_pairs": P}
        del ws
        if mode == "sparse":
            bms, bkms = _time_backward(gb, Q, K, V, S, O, LSE, dO, mode, k, tau, dev, flush, reps)
            flb = 10.0 * w.d * P
            out[name].update({"bwd_ms": bms, "bwd_tflops": flb / bms / 1e9, "bwd_kernel_ms": bkms,
                              "bwd_kernel_tflops": flb / bkms / 1e9})
    del Q, K, V, S, dO
    torch.cuda.empty_cache()
    return out


def bench_decode(dev, peaks, reps=10):
    """Sparse decode: 64 sequences x 131072 cache, K=32."""
    from gated_block_sparse_gate_b200 import binding as gb

    w = WORKLOADS["sparse_decode_bf16_b64_l131072"]
    x = make_decode_inputs(w, device=dev)
    k = w.topk[0]
    p = gb.make_params(w.B, w.Hq, w.Hkv, w.N, w.d, w.block, k, "sparse", x["q"].dtype)
    ws = gb.alloc_workspace(p, gb.OP_DECODE, dev)
    O = torch.empty_like(x["q"])
    LSE = torch.empty(w.B, w.Hq, dtype=torch.float32, device=dev)
    for _ in range(3):
        gb.decode(x["q"], x["Kc"], x["Vc"], x["S"], topk=k, out=O, lse=LSE, ws=ws)
    a0, a1, k0, k1 = _events(reps), _events(reps), _events(reps), _events(reps)
    torch.cuda.synchronize()
    for i in range(reps):
        gb.set_timer(gb.OP_DECODE, k0[i], k1[i])
        a0[i].record()
        gb.decode(x["q"], x["Kc"], x["Vc"], x["S"], topk=k, out=O, lse=LSE, ws=ws)
        a1[i].record()
    torch.cuda.synchronize()
    gb.set_timer(gb.OP_DECODE)
    gb.check(ws)
    ms = statistics.mean(a.elapsed_time(b) for a, b in zip(a0, a1))
    kms = statistics.mean(a.elapsed_time(b) for a, b in zip(k0, k1))
    cur = (w.N - 1) // w.block
    blocks = min(k, cur) + 1
    G = w.Hq // w.Hkv
    blk_bytes = w.block * w.d * 2 * 2  # K and V rows of one 64-token block
    # algorithmic bytes: each distinct block of a (sequence, kv group) once
    union = decode_union_blocks(x["S"], cur, k, G)
    kv_bytes = union * blk_bytes
    # logical bytes: every q-head's own selection (blocks shared by the heads of
    # a group are requested once per head; the repeats mostly hit L2)
    kv_logical = w.B * w.Hq * blocks * blk_bytes
    other = x["q"].numel() * 2 * 2 + x["S"].numel() * 4
    tot = kv_bytes + other
    out = {"ms": ms, "kernel_ms": kms, "tokens_per_s": w.B / (ms * 1e-3),
           "hbm_gbs": tot / (ms * 1e-3) / 1e9, "kernel_hbm_gbs": kv_bytes / (kms * 1e-3) / 1e9,
           "frac_of_hbm_roofline": (tot / (peaks["hbm_gbs"] * 1e9)) / (ms * 1e-3),
           "bytes_per_step": tot, "kv_union_blocks": union,
           "bytes_note": "union of the selected blocks per (sequence, kv group) + q, O, S",
           "logical_bytes_per_q_head": kv_logical + other,
           "kernel_logical_gbs_per_q_head": kv_logical / (kms * 1e-3) / 1e9}

    def timed(call):
        for _ in range(3):
            call()
        b0, b1, c0, c1 = _events(reps), _events(reps), _events(reps), _events(reps)
        torch.cuda.synchronize()
        for i in range(reps):
            gb.set_timer(gb.OP_DECODE, c0[i], c1[i])
            b0[i].record()
            call()
            b1[i].record()
        torch.cuda.synchronize()
        gb.set_timer(gb.OP_DECODE)
        gb.check(ws)
        return (statistics.mean(a.elapsed_time(b) for a, b in zip(b0, b1)),
                statistics.mean(a.elapsed_time(b) for a, b in zip(c0, c1)))

    # one selection per kv group: each selected block is read once per group
    g = torch.Generator().manual_seed(w.seed + 1)
    Sg = (torch.randn(w.B, w.Hkv, w.Nb, generator=g) * 2 ** 0.5).to(dev)
    gms, gkms = timed(lambda: gb.decode_ex(x["q"], x["Kc"], x["Vc"], Sg, w.N, topk=k,
                                            group_shared=True, out=O, lse=LSE, ws=ws))
    g_kv = w.B * w.Hkv * blocks * w.block * w.d * 2 * 2
    g_tot = g_kv + x["q"].numel() * 2 * 2 + Sg.numel() * 4
    out["group_shared"] = {
        "ms": gms, "kernel_ms": gkms, "tokens_per_s": w.B / (gms * 1e-3),
        "hbm_gbs": g_tot / (gms * 1e-3) / 1e9,
        "frac_of_hbm_roofline": (g_tot / (peaks["hbm_gbs"] * 1e9)) / (gms * 1e-3),
        "bytes_per_step": g_tot}
    # the same cache on shuffled 64-token pages through a block table
    nb = w.N // w.block
    perm = torch.randperm(w.B * nb, generator=g).to(dev)
    table = perm.view(w.B, nb).to(torch.int32)
    pools = []
    for src in (x["Kc"], x["Vc"]):
        pool = torch.empty(w.B * nb, w.Hkv, w.block, w.d, dtype=src.dtype, device=dev)
        pool[perm] = src.view(w.B, w.Hkv, nb, w.block, w.d).permute(0, 2, 1, 3, 4).reshape(
            w.B * nb, w.Hkv, w.block, w.d)
        pools.append(pool)
    del x["Kc"], x["Vc"]
    torch.cuda.empty_cache()
    pms, pkms = timed(lambda: gb.decode_ex(x["q"], pools[0], pools[1], x["S"], w.N, topk=k,
                                            block_table=table, out=O, lse=LSE, ws=ws))
    p_tot = tot + table.numel() * 4
    out["paged"] = {"ms": pms, "kernel_ms": pkms, "tokens_per_s": w.B / (pms * 1e-3),
                    "hbm_gbs": p_tot / (pms * 1e-3) / 1e9,
                    "frac_of_hbm_roofline": (p_tot / (peaks["hbm_gbs"] * 1e9)) / (pms * 1e-3),
                    "bytes_per_step": p_tot}
    del x, pools
    torch.cuda.empty_cache()
    return out


def prefix_inputs(w, max_tokens):
    """The workload's seeded inputs cut to their first ``max_tokens`` tokens
    (query blocks 0 .. max_tokens/64 - 1 and the keys they attend: a causal
    prefix computes exactly what those rows compute in the full problem).
    Returns (inputs, workload with N = the prefix length)."""
    import dataclasses

    x = make_prefill_inputs(w)
    if w.N <= max_tokens:
        return x, w
    nb = max_tokens // w.block
    x = {k: (v[:, :, :max_tokens] if k != "S" else v[:, :, :nb, :nb]).contiguous()
         for k, v in x.items()}
    return x, dataclasses.replace(w, N=max_tokens)


def cpu_baseline_sample(w, min_s=10.0, max_tokens=8192):
    """The float64 oracle on whole kv groups (G q-heads each) of the training
    workload, group after group until at least ``min_s`` seconds are timed.

    Workloads longer than ``max_tokens`` are sampled on their first
    ``max_tokens`` tokens (query blocks 0 .. max_tokens/64 - 1 with the keys
    they attend, a causal prefix of the same seeded inputs), so the sample
    stays within tens of seconds of CPU work."""
    import numpy as np

    import oracle

    n_full = w.N
    x, w = prefix_inputs(w, max_tokens)
    G = w.Hq // w.Hkv
    f64 = lambda t: t.float().numpy().astype(np.float64)  # noqa: E731
    dt, groups = 0.0, 0
    while groups < w.Hkv and dt < min_s:
        hs = slice(groups * G, (groups + 1) * G)
        kv = slice(groups, groups + 1)
        Q, K, V, dO = f64(x["Q"][:, hs]), f64(x["K"][:, kv]), f64(x["V"][:, kv]), f64(x["dO"][:, hs])
        S = x["S"][:, hs].numpy()
        t0 = time.perf_counter()
        oracle.gated_attention_forward(Q, K, V, S, w.block)
        oracle.gated_attention_backward(Q, K, V, S, dO, w.block)
        dt += time.perf_counter() - t0
        groups += 1
    fl = 14.0 * w.d * train_pairs_per_head(w.Nb, w.block) * G * groups
    threads = os.cpu_count()
    try:
        from threadpoolctl import threadpool_info
        threads = max(int(i.get("num_threads", 1)) for i in threadpool_info()) or threads
    except Exception:  # noqa: BLE001
        pass
    return {"value": fl / dt / 1e12, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"float64 NumPy oracle, forward+backward of "
                      f"{'kv group 0' if groups == 1 else f'kv groups 0-{groups - 1}'} "
                      f"({groups * G} of {w.Hq} q-heads) of {w.name}"
                      + (f", first {w.N} of {n_full} tokens" if n_full != w.N else "")
                      + f"; {dt:.1f} s; host cores {os.cpu_count()}"}


# -------------------------------------------------------------- reference arm

def run_reference(args, w):
    """The oracle timed on the host cores, each step a bounded sample."""
    import numpy as np

    import oracle

    rank, _, ws = gdist.world()
    if rank != 0:
        return 0
    n_sub = 2048  # kv group 0 (q-heads 0-3) over the first 2048 tokens of the workload
    x, _ = prefix_inputs(w, n_sub)
    G = w.Hq // w.Hkv
    f64 = lambda t: t.float().numpy().astype(np.float64)  # noqa: E731
    Q, dO, S = f64(x["Q"][:, :G]), f64(x["dO"][:, :G]), x["S"][:, :G].numpy()
    K, V = f64(x["K"][:, :1]), f64(x["V"][:, :1])

    def step():
        oracle.gated_attention_forward(Q, K, V, S, w.block)
        oracle.gated_attention_backward(Q, K, V, S, dO, w.block)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    fl = 14.0 * w.d * train_pairs_per_head(n_sub // w.block, w.block) * G
    val = fl / dt / 1e12
    sample = (f"float64 NumPy oracle, forward+backward of kv group 0 ({G} q-heads) over the "
              f"first {n_sub} of {w.N} tokens of {w.name} per step")
    line = {"metric": METRIC, "value": val, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": _config(w, ws), "impl": "reference",
            "cpu_baseline": {"value": val, "unit": UNIT, "cores": os.cpu_count(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def _config(w, n):
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d,
            "block": w.block, "mode": "train", "step": "select + gated fwd + gated bwd (dQ,dK,dV,dS)",
            "parallelism": f"{n} independent shard(s), no collective",
            "l2": "flushed between steps (256 MB write, untimed)"}


# ----------------------------------------------------------------------- main

def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(WORKLOADS))
    ap.add_argument("--no-extra", action="store_true", help="skip sparse prefill / decode extras")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args(argv)
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)

    from gated_block_sparse_gate_b200 import binding as gb
    from gated_block_sparse_gate_b200.build import build

    rank, local, ws = gdist.world()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs CUDA devices")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if rank == 0:
        build()
    gdist.init("nccl")
    gdist.barrier()
    gb.load_library()
    peaks, peak_src = load_peaks()

    r = bench_training(w, args.steps, args.warmup, rank, dev, peaks)
    ms = gdist.max_over_ranks(r["ms"], dev)
    e2e_ms = gdist.max_over_ranks(r["e2e"]["ms"], dev)
    extra = {}
    if ws == 1 and not args.no_extra:
        extra["train_bf16_n8192"] = bench_training_extra("train_bf16_n8192", dev, peaks)
        extra["sparse_prefill_bf16_n65536"] = bench_sparse_prefill(dev, peaks)
        extra["sparse_decode_bf16_b64_l131072"] = bench_decode(dev, peaks)
    if rank == 0:
        total = r["flops"] * ws
        line = {
            "metric": METRIC, "value": total / (ms * 1e-3) / 1e12, "unit": UNIT, "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": _config(w, ws),
            "fwd_tflops": r["fl_fwd"] * ws / (r["fwd_ms"] * 1e-3) / 1e12,
            "fwd_ms": r["fwd_ms"], "bwd_main_ms": r["bwd_ms"],
            "pct_of_bf16_peak": 100.0 * total / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
            "peak_source": peak_src,
            "roofline": r["roofline"],
            "e2e": {"value": total / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
                    "h2d_bytes_per_step": r["e2e"]["h2d"], "d2h_bytes_per_step": r["e2e"]["d2h"],
                    "ms_per_step": e2e_ms, "pipelined": r["e2e"]["pipelined"],
                    "serial_ms_per_call": r["e2e"]["serial_ms"],
                    "serial_value": total / (r["e2e"]["serial_ms"] * 1e-3) / 1e12},
            "gpu_launches": r["launches"], "gpu_launches_per_step": r["per_step_launches"],
            "clocks": r["clocks"],
        }
        if extra:
            line["extra"] = extra
        if ws == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline_sample(w)
        print(json.dumps(line), flush=True)
    gdist.barrier()
    gdist.finalize()
    return 0


if __name__ == "__main__":
    sys.exit(main())
