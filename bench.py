#!/usr/bin/env python3
"""Benchmark: triangle attention forward + backward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one forward (o, resid, lse) and one backward (dq, dk, dv, dbias) of
the crop-768 training shape (B=1, N=768, H=4, d=32, BF16; q,k,v,dout ~ N(0,1),
bias ~ 2 N(0,1), all-valid zero mask), synthetic inputs resident in HBM.  The
metric counts 14*B*H*N^3*d flops per step (forward 4, backward 10 -- five
GEMM-shaped products including the one recompute).  The inputs (604 MB) are
larger than the 126 MB L2, so nothing is flushed between steps.

Multi-GPU: one process per GPU (torchrun); every rank runs its own replica of
the workload (the path has no exchange step), so scaling is weak and the value
is the flops of all ranks divided by the slowest rank's time.

--impl reference times the FP64 CPU oracle (the only other implementation;
test infrastructure) on the host cores: each step is a bounded sample of the
same workload (a few pair rows), rank 0 only.

Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "tri-attn fwd+bwd TFLOP/s at N=768,H=4,d=32 BF16; % of B200 BF16 TC peak"
WORKLOAD = "crop768 triangle attention fwd+bwd (starting node): B=1, N=768, H=4, d=32, BF16"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's time of the timed region: every rank passes its own and all
    get the maximum (a collective; every rank must call it)."""
    if world == 1:
        return ms
    import torch
    import torch.distributed as dist
    tt = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    return float(tt.item())


def whole_job_rate(world: int, work_per_step: float, steps: int, ms: float, scale: float = 1e12) -> float:
    """Whole-job throughput: every rank did `steps` steps of `work_per_step` each (weak
    scaling: replicas of the same workload) within the slowest rank's `ms`."""
    return world * work_per_step * steps / (ms * 1e-3) / scale


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def flops(B, N, H, d):
    cube = B * H * N ** 3 * d
    return {"fwd": 4.0 * cube, "bwd": 10.0 * cube, "step": 14.0 * cube,
            "bwd_main": 10.0 * cube, "bwd_dbias": 4.0 * cube}


# ---------------------------------------------------------------------------
# clock sampling during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", str(self.dev)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in out.strip().splitlines():
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# DRAM traffic of the dominant kernel, from the committed ncu capture
# ---------------------------------------------------------------------------
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic_crop768.md")


def kernel_source_digest() -> str:
    """sha256 over the sources the attention kernels are compiled from (their device
    code and shared helpers), in name order."""
    import hashlib
    csrc = os.path.join(ROOT, "triangle_attention_biomolecular_b200", "csrc")
    files = [os.path.join(csrc, n) for n in ("bwd.cuh", "dbias.cuh", "fwd.cuh", "sm100.cuh")]
    h = hashlib.sha256()
    for fn in files:
        h.update(os.path.basename(fn).encode())
        with open(fn, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def l2_note(input_bytes: int) -> str:
    """How the step's inputs relate to the 126 MB L2 (nothing is flushed between steps)."""
    mb = input_bytes / 1e6
    if input_bytes > 126e6:
        return f"inputs ({mb:.0f} MB) larger than the 126 MB L2; no flush"
    return f"inputs ({mb:.0f} MB) fit in the 126 MB L2; no flush (a profiling workload, not a bench line)"


def attn_launches_per_step(B: int, N: int, H: int) -> int:
    """Kernels of one fwd+bwd step: forward, prep, bias rearrangement, main backward,
    dBias pass, plus the ordered reduce of dBias row chunks when there are fewer
    128x128 tiles than SMs (the same rule as the library's workspace layout)."""
    nt = (N + 127) // 128
    tiles = B * H * nt * nt
    chunks = 1
    if tiles < 148:
        chunks = max(1, min(148 // tiles, (N + 7) // 8))
    return 5 + (1 if chunks > 1 else 0)


def committed_traffic(kernel: str):
    """dram__bytes_read.sum + dram__bytes_write.sum per launch of `kernel` from the
    committed capture, or None if there is none or the kernels changed since."""
    import re
    try:
        text = open(TRAFFIC_FILE).read()
    except OSError:
        return None
    m = re.search(r"source-sha256:\s*([0-9a-f]{64})", text)
    if not m or m.group(1) != kernel_source_digest():
        return None
    m = re.search(rf"\|\s*{kernel}\s*\|\s*([0-9]+)\s*\|\s*([0-9]+)\s*\|", text)
    return int(m.group(1)) + int(m.group(2)) if m else None


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from triangle_attention_biomolecular_b200 import _binding as Bd
    from triangle_attention_biomolecular_b200 import synthetic as S

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = {"crop768": S.CROP768, "crop640": S.CROP640, "crop384": S.CROP384, "b2n256": S.sweep(256, 32)}[args.workload]
    Bn, N, H, d = wl.B, wl.N, wl.H, wl.d
    x = S.make_inputs(wl, S.seed_for(3, rank))
    q, k, v, do, bias = (x[n].to(dev) for n in ("q", "k", "v", "dout", "bias"))
    mask = x["mask"].to(dev)
    o, r = torch.empty_like(q), torch.empty_like(q)
    lse = torch.empty((Bn, H, N, N), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    db = torch.empty((Bn, H, N, N), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(Bd.tri_attn_bwd_workspace_bytes(Bn, N, H, d), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        Bd.tri_attn_fwd(q, k, v, bias, mask, o, r, lse, 0.0, stream)
        if ev is None:
            Bd.tri_attn_bwd(q, k, v, bias, mask, o, r, lse, do, dq, dk, dv, db, ws, 0.0, 0, stream)
        else:
            Bd.tri_attn_bwd_marked(q, k, v, bias, mask, o, r, lse, do, dq, dk, dv, db, ws, ev[1:5], 0.0, 0,
                                   stream)

    torch.cuda.reset_peak_memory_stats(dev)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st, word = Bd.tri_attn_device_error(True)
    if st != 0:
        raise RuntimeError(f"device error word {word:#x} during warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    for e in evs:  # torch creates an event on its first record; the library re-records these handles
        for ev in e:
            ev.record(stream)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local_rank if "CUDA_VISIBLE_DEVICES" not in os.environ else
                           int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local_rank]))
    sampler.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0.record(stream)
    for s in range(args.steps):
        step(evs[s])
    t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    st, word = Bd.tri_attn_device_error(True)
    if st != 0:
        raise RuntimeError(f"device error word {word:#x} during timing")

    # per-kernel average durations, measured live on the launching stream
    kern = {"fwd": [], "bwd_prep": [], "bwd_main": [], "bwd_dbias": []}
    for e in evs:
        kern["fwd"].append(e[0].elapsed_time(e[1]))
        kern["bwd_prep"].append(e[1].elapsed_time(e[2]))
        kern["bwd_main"].append(e[2].elapsed_time(e[3]))
        kern["bwd_dbias"].append(e[3].elapsed_time(e[4]))
    kern_ms = {n: statistics.mean(v) for n, v in kern.items()}
    steps_ms = sorted(e[0].elapsed_time(e[4]) for e in evs)
    step_stats = {"median": statistics.median(steps_ms), "p90": steps_ms[min(len(steps_ms) - 1, int(0.9 * len(steps_ms)))],
                  "min": steps_ms[0]}
    lengths = [int(v) for v in x["lengths"]]

    # End to end through the same C ABI: every step copies its inputs from pinned host
    # memory to the device and its results back.  Steps are pipelined over two buffer sets
    # and three streams (host->device copies, compute, device->host copies), so step n's
    # compute overlaps step n+1's input copy and step n-1's result copy.
    e2e = None
    if not args.no_e2e:
        host_in = [t.cpu().pin_memory() for t in (q, k, v, do, bias, mask)]
        host_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in (o, dq, dk, dv, db)]
        h2d = sum(t.numel() * t.element_size() for t in host_in)
        d2h = sum(t.numel() * t.element_size() for t in host_out)
        n_e2e = max(2, min(args.steps, 12))

        def buffers():
            ins = [torch.empty_like(t) for t in (q, k, v, do, bias, mask)]
            outs = {"o": torch.empty_like(q), "r": torch.empty_like(q), "lse": torch.empty_like(lse),
                    "dq": torch.empty_like(q), "dk": torch.empty_like(q), "dv": torch.empty_like(q),
                    "db": torch.empty_like(db)}
            return ins, outs
        slots = [buffers(), buffers()]
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        ev = lambda: torch.cuda.Event(enable_timing=False)
        in_done, comp_done, out_done = ([ev() for _ in range(n_e2e + 1)] for _ in range(3))

        def e2e_step(n):
            ins, outs = slots[n % 2]
            with torch.cuda.stream(s_in):
                if n >= 2:
                    s_in.wait_event(comp_done[n - 2])  # step n-2 has finished reading these inputs
                for h, dt in zip(host_in, ins):
                    dt.copy_(h, non_blocking=True)
                in_done[n].record(s_in)
            stream.wait_event(in_done[n])
            if n >= 2:
                stream.wait_event(out_done[n - 2])  # step n-2's results have left these buffers
            qq, kk, vv, dd, bb, mm = ins
            Bd.tri_attn_fwd(qq, kk, vv, bb, mm, outs["o"], outs["r"], outs["lse"], 0.0, stream)
            Bd.tri_attn_bwd(qq, kk, vv, bb, mm, outs["o"], outs["r"], outs["lse"], dd, outs["dq"], outs["dk"],
                            outs["dv"], outs["db"], ws, 0.0, 0, stream)
            comp_done[n].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(comp_done[n])
                for h, name in zip(host_out, ("o", "dq", "dk", "dv", "db")):
                    h.copy_(outs[name], non_blocking=True)
                out_done[n].record(s_out)

        e2e_step(0)  # warm-up of the copy path
        torch.cuda.synchronize()
        in_done, comp_done, out_done = ([ev() for _ in range(n_e2e + 1)] for _ in range(3))
        if world > 1:
            dist.barrier()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a0.record(s_in)
        for n in range(n_e2e):
            e2e_step(n)
        a1.record(s_out)
        torch.cuda.synchronize()
        ems = max_over_ranks(a0.elapsed_time(a1), world, dev)
        st, word = Bd.tri_attn_device_error(True)
        if st != 0:
            raise RuntimeError(f"device error word {word:#x} during the end-to-end leg")
        fl = flops(Bn, N, H, d)["step"]
        e2e = {"value": round(whole_job_rate(world, fl, n_e2e, ems), 3), "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n_e2e,
               "ms_per_step": round(ems / n_e2e, 4),
               "pipelining": "two buffer sets; H2D, compute and D2H on three streams"}
    mem = {"peak_allocated_bytes": int(torch.cuda.max_memory_allocated(dev)),
           "bwd_workspace_bytes": int(ws.numel()),
           "saved_state_bytes": int(2 * o.numel() * o.element_size() + lse.numel() * lse.element_size())}
    return {"ms": ms, "kern_ms": kern_ms, "clocks": clocks, "e2e": e2e, "shape": (Bn, N, H, d),
            "step_stats": step_stats, "lengths": lengths, "memory": mem, "mask": wl.mask,
            "bias_std": wl.bias_std}


# ---------------------------------------------------------------------------
# all configurations (--sweep): one JSON line per workload
# ---------------------------------------------------------------------------
def run_sweep(args):
    """Forward-only and forward+backward times of every workload family: the three
    crops and the batched ragged sweep (B=2, N in 128..1024, d in 32/64, lengths
    L_b ~ U{N/2..N}).  TFLOP/s by the formula and effective (4*H*d*sum_b N^2*L_b per
    forward pass, 14*... per step), % of the BF16 peak, and for N <= 512 the
    algorithmic bytes per second against the HBM peak."""
    import torch
    from triangle_attention_biomolecular_b200 import _binding as Bd
    from triangle_attention_biomolecular_b200 import synthetic as S
    dev = torch.device("cuda", 0)
    pk, src = peaks()
    peak, hbm = float(pk["bf16_tflops"]), float(pk["hbm_gbs"])
    wls = [S.CROP384, S.CROP640, S.CROP768] + [S.sweep(N, d) for d in S.SWEEP_DS for N in S.SWEEP_NS]
    for wl in wls:
        x = S.make_inputs(wl, S.seed_for(9, wl.N + wl.d))
        q, k, v, do, bias = (x[n].to(dev) for n in ("q", "k", "v", "dout", "bias"))
        mask = x["mask"].to(dev) if x["mask"] is not None else None
        Bn, N, H, d = wl.B, wl.N, wl.H, wl.d
        o, r = torch.empty_like(q), torch.empty_like(q)
        lse = torch.empty((Bn, H, N, N), dtype=torch.float32, device=dev)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
        Np = (N + 7) // 8 * 8
        db = torch.empty((Bn, H, N, Np), dtype=torch.bfloat16, device=dev)[..., :N]
        ws = torch.empty(Bd.tri_attn_bwd_workspace_bytes(Bn, N, H, d), dtype=torch.uint8, device=dev)
        fwd = lambda: Bd.tri_attn_fwd(q, k, v, bias, mask, o, r, lse)
        bwd = lambda: Bd.tri_attn_bwd(q, k, v, bias, mask, o, r, lse, do, dq, dk, dv, db, ws)

        def timed(fn, n):
            for _ in range(3):
                fn()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            e0.record()
            for _ in range(n):
                fn()
            e1.record()
            torch.cuda.synchronize()
            return e0.elapsed_time(e1) / n
        def timed_graph(fn, n):
            # the same calls captured once into a CUDA graph and replayed: device time
            # without the per-call host marshalling of the Python binding (tens of
            # microseconds, which bounds the eager rate at small N)
            side = torch.cuda.Stream()
            side.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(side):
                for _ in range(3):
                    fn()
            torch.cuda.current_stream().wait_stream(side)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for _ in range(n):
                    fn()
            g.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            g.replay()
            e1.record()
            torch.cuda.synchronize()
            del g
            return e0.elapsed_time(e1) / n

        n_iter = max(5, min(200, int(2e12 / (14.0 * Bn * H * N ** 3 * d))))
        sampler = ClockSampler(0)
        sampler.start()
        time.sleep(0.3)
        t_f_eager = timed(fwd, n_iter)
        t_fb_eager = timed(lambda: (fwd(), bwd()), n_iter)
        t_f = timed_graph(fwd, n_iter)
        t_fb = timed_graph(lambda: (fwd(), bwd()), n_iter)
        clocks = sampler.stop()
        st, word = Bd.tri_attn_device_error(True)
        if st != 0:
            raise RuntimeError(f"device error word {word:#x} in {wl.name}")
        L = [int(v_) for v_ in x["lengths"]]
        cube = H * N ** 3 * d * Bn
        eff = H * d * sum(N * N * l_ for l_ in L)
        pair = Bn * N * N * H * d * 2
        fwd_bytes = 5 * pair + Bn * H * N * N * (2 + 4) + Bn * N * N * 4
        line = {"metric": "tri-attn TFLOP/s per workload", "workload": wl.name, "B": Bn, "N": N, "H": H, "d": d,
                "mask": wl.mask, "orientation": wl.orientation, "iters": n_iter,
                "timing": "CUDA graph of the calls, replayed (device time); *_eager: back-to-back Python calls",
                "fwd_ms_eager": round(t_f_eager, 4), "fwd_bwd_ms_eager": round(t_fb_eager, 4),
                "fwd_ms": round(t_f, 4), "fwd_tflops": round(4.0 * cube / (t_f * 1e-3) / 1e12, 2),
                "fwd_tflops_effective": round(4.0 * eff / (t_f * 1e-3) / 1e12, 2),
                "fwd_bwd_ms": round(t_fb, 4), "fwd_bwd_tflops": round(14.0 * cube / (t_fb * 1e-3) / 1e12, 2),
                "fwd_bwd_tflops_effective": round(14.0 * eff / (t_fb * 1e-3) / 1e12, 2),
                "pct_of_bf16_peak": round(100.0 * 14.0 * cube / (t_fb * 1e-3) / 1e12 / peak, 2),
                "peak_source": f"{src} bf16_tflops {peak}", "clocks": clocks}
        if N <= 512:
            gbs = fwd_bytes / (t_f * 1e-3) / 1e9
            line["fwd_algorithmic_gbs"] = round(gbs, 1)
            line["fwd_pct_of_hbm"] = round(100.0 * gbs / hbm, 2)
        print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# second operation: the triangle multiplicative contraction (--op tri_mul)
# ---------------------------------------------------------------------------
TRI_MUL_METRIC = "tri-mul contraction fwd+bwd TFLOP/s at N=768, C=128 pair channels, BF16"


def run_tri_mul(args, rank, world, local_rank):
    """One step = forward x = a (x) b over k (outgoing edges) and the backward da, db:
    three batched N x N x N products per channel, 6*B*C*N^3 flops."""
    import torch
    import torch.distributed as dist
    from triangle_attention_biomolecular_b200 import _binding as Bd
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    Bn, C, N = 1, 128, 768
    g = torch.Generator().manual_seed(1000 + rank)
    a, b, dx = (torch.randn((Bn, C, N, N), generator=g).to(torch.bfloat16).to(dev) for _ in range(3))
    x, da, db = torch.empty_like(a), torch.empty_like(a), torch.empty_like(a)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        Bd.tri_mul_fwd(a, b, x, False, stream)
        if ev is not None:
            ev[1].record(stream)
        Bd.tri_mul_bwd(a, b, dx, da, db, False, stream)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0.record(stream)
    for s_ in range(args.steps):
        step(evs[s_])
    t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    st, word = Bd.tri_attn_device_error(True)
    if st != 0:
        raise RuntimeError(f"device error word {word:#x}")
    fwd_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    bwd_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    return {"ms": ms, "fwd_ms": fwd_ms, "bwd_ms": bwd_ms, "clocks": clocks, "shape": (Bn, C, N)}


GATE_METRIC = ("gated output projection fwd+bwd GB/s at N=768 (589,824 pair positions, 128 channels), BF16")


def run_gate(args):
    """One step = forward y = (sigmoid(z Wg) * o) Wo and backward (dz, do, dWg, dWo for an
    upstream dy) over every pair position of the crop768 pair tensor.  HBM-bound: the
    forward reads z, o and writes y, the backward reads z, o, dy and writes dz, do:
    8 x R x 128 x 2 bytes (plus the weights)."""
    import torch
    from triangle_attention_biomolecular_b200 import _binding as Bd
    dev = torch.device("cuda", 0)
    R = args.gate_rows
    g = torch.Generator().manual_seed(5)
    z, o, dy = (torch.randn((R, 128), generator=g).to(torch.bfloat16).to(dev) for _ in range(3))
    wg, wo = ((torch.randn((128, 128), generator=g) / 128 ** 0.5).to(torch.bfloat16).to(dev) for _ in range(2))
    y, dz, d_o = (torch.empty_like(z) for _ in range(3))
    dwg, dwo = (torch.empty((128, 128), device=dev) for _ in range(2))
    ws = torch.empty(Bd.tri_gate_bwd_workspace_bytes(R), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    fwd = lambda: Bd.tri_gate_fwd(z, o, wg, wo, y, stream)
    bwd = lambda: Bd.tri_gate_bwd(z, o, wg, wo, dy, dz, d_o, dwg, dwo, ws, stream)
    for _ in range(args.warmup):
        fwd()
        bwd()
    torch.cuda.synchronize()
    sampler = ClockSampler(0)
    sampler.start()
    time.sleep(0.3)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * args.steps + 1)]
    torch.cuda.synchronize()
    ev[0].record(stream)
    for i in range(args.steps):
        fwd()
        ev[2 * i + 1].record(stream)
        bwd()
        ev[2 * i + 2].record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    st, word = Bd.tri_attn_device_error(True)
    if st != 0:
        raise RuntimeError(f"device error word {word:#x}")
    f_ms = sum(ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(args.steps)) / args.steps
    b_ms = sum(ev[2 * i + 1].elapsed_time(ev[2 * i + 2]) for i in range(args.steps)) / args.steps
    ms = f_ms + b_ms
    pk, src = peaks()
    hbm = float(pk["hbm_gbs"])
    row = R * 128 * 2
    f_bytes, b_bytes = 3 * row + 2 * 128 * 128 * 2, 5 * row + 2 * 128 * 128 * 2
    gbs = (f_bytes + b_bytes) / (ms * 1e-3) / 1e9
    b_gbs = b_bytes / (b_ms * 1e-3) / 1e9
    line = {"metric": GATE_METRIC, "value": round(gbs, 1), "unit": "GB/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "gated output projection y = (sigmoid(z Wg) * o) Wo and its backward, "
                                   f"R = {R} pair positions, cz = H*d = 128",
                       "bytes_per_step": f_bytes + b_bytes, "fwd_ms": round(f_ms, 4), "bwd_ms": round(b_ms, 4),
                       "fwd_gbs": round(f_bytes / (f_ms * 1e-3) / 1e9, 1), "bwd_gbs": round(b_gbs, 1),
                       "l2": "inputs (151 MB per tensor) larger than the 126 MB L2; no flush"},
            "tflops": round(7 * 2 * R * 128 * 128 / (ms * 1e-3) / 1e12, 2),  # 2 + 5 contractions
            "roofline": {"kernel": "tri_gate_bwd", "bound": "hbm", "achieved": round(b_gbs, 1), "peak": hbm,
                         "unit": "GB/s", "frac": round(b_gbs / hbm, 4), "traffic": None,
                         "peak_source": f"{src} hbm_gbs"},
            "gpu_launches": 3 * args.steps, "clocks": clocks, "e2e": None}
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = gate_cpu_baseline()
    print(json.dumps(line), flush=True)


def gate_cpu_baseline(target_s: float = 10.0):
    """The FP64 oracle of the gated projection (forward + backward) on the host cores
    over a bounded block of pair positions, in the bench's GB/s (8 x 128 x 2 bytes of
    BF16 traffic per position)."""
    import numpy as np
    from oracle import tri_gate_oracle as G
    rows = 16384
    rng = np.random.default_rng(0)
    z, o, dy = (rng.standard_normal((rows, 128)) for _ in range(3))
    wg, wo = (rng.standard_normal((128, 128)) / np.sqrt(128) for _ in range(2))

    def one():
        t = time.perf_counter()
        G.fwd(z, o, wg, wo)
        G.bwd(z, o, wg, wo, dy)
        return time.perf_counter() - t
    one()
    t1 = one()
    n = int(max(1, min(36, round(target_s / max(t1, 1e-4)))))
    t = sum(one() for _ in range(n))
    return {"value": round(8 * 128 * 2 * rows * n / t / 1e9, 3), "unit": "GB/s", "cores": os.cpu_count(),
            "kind": "oracle", "seconds": round(t, 3),
            "sample": f"{n} blocks of {rows} of the 589,824 pair positions: FP64 oracle forward + backward "
                      "(numpy matmul)"}


def tri_mul_cpu_baseline(target_s: float = 10.0):
    """The FP64 oracle on the host cores over a bounded number of channels."""
    import numpy as np
    from oracle import tri_mul_oracle as T
    N = 768
    rng = np.random.default_rng(0)
    a, b, dx = (rng.standard_normal((1, 1, N, N)) for _ in range(3))

    def one():
        t = time.perf_counter()
        T.fwd(a, b, "outgoing")
        T.bwd(a, b, dx, "outgoing")
        return time.perf_counter() - t
    one()
    t1 = one()
    n = int(max(1, min(128, round(target_s / max(t1, 1e-4)))))
    t = sum(one() for _ in range(n))
    return {"value": round(6.0 * N ** 3 * n / t / 1e12, 6), "unit": "TFLOP/s", "cores": os.cpu_count(),
            "kind": "oracle", "seconds": round(t, 3),
            "sample": f"{n} of the 128 channels at N=768: FP64 oracle forward + backward (numpy matmul)"}


# ---------------------------------------------------------------------------
# the oracle on host cores (CPU baseline and the reference arm)
# ---------------------------------------------------------------------------
def oracle_sample(rows_n: int):
    import numpy as np
    from oracle import oracle as O
    from triangle_attention_biomolecular_b200 import synthetic as S
    wl = S.CROP768
    x = S.make_inputs(wl, S.seed_for(3, 0))
    f64 = lambda t: t.double().numpy()
    q, k, v, do, bias = (f64(x[n]) for n in ("q", "k", "v", "dout", "bias"))
    mask = x["mask"].numpy().astype(np.float64)
    rows = [(0, (37 * r) % wl.N) for r in range(rows_n)]
    acc = np.zeros((wl.H, wl.N, wl.N))

    def run(rs):
        # the whole step restricted to the sampled pair rows: forward, dq/dk/dv, and the
        # rows' share of the dBias sum over i
        t = time.perf_counter()
        O.fwd(q, k, v, bias, mask, rows=rs)
        O.bwd_rows(q, k, v, bias, mask, do, rows=rs)
        for b, i in rs:
            O.dbias_add_row(acc, q[b, i], k[b, i], v[b, i], bias[b], mask[b, i], do[b, i])
        return time.perf_counter() - t
    return wl, rows, run


def cpu_rate(wl, nrows, seconds):
    per_row = 14.0 * wl.H * wl.N ** 2 * wl.d  # the step's flops restricted to one pair row
    return per_row * nrows / seconds / 1e12


def run_cpu_baseline(target_s: float = 15.0):
    # the oracle spreads rows over the host cores: calibrate on one row per core,
    # then time whole batches of rows adding up to about target_s seconds
    cores = os.cpu_count() or 1
    wl, rows, run = oracle_sample(768)
    run(rows[:cores])  # first touch of the FP64 inputs
    tc = run(rows[cores:2 * cores])
    n = int(max(cores, min(len(rows), cores * round(target_s / max(tc, 1e-3)))))
    t = run(rows[:n])
    return {"value": round(cpu_rate(wl, n, t), 6), "unit": "TFLOP/s", "cores": os.cpu_count(),
            "kind": "oracle", "seconds": round(t, 3),
            "sample": f"{n} pair rows (all 4 heads) of the crop768 workload: FP64 oracle forward, dq/dk/dv "
                      f"and the rows' share of dbias; rate counts 14*H*N^2*d flops per row"}


def run_reference(args, rank, world):
    if rank != 0:
        return
    cores = os.cpu_count() or 1
    per_step_rows = cores  # one pair row per host core and step, so every core has work
    wl, rows, run = oracle_sample(max(64, 4 * per_step_rows))
    for s in range(args.warmup):
        run(rows[:1])
    times = []
    for s in range(args.steps):
        rr = [rows[(s * per_step_rows + e) % len(rows)] for e in range(per_step_rows)]
        times.append(run(rr))
    tot = sum(times)
    val = cpu_rate(wl, per_step_rows * args.steps, tot)
    line = {
        "impl": "reference", "metric": METRIC, "value": round(val, 6), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * tot / max(1, args.steps), 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD + f" -- each step a bounded sample of {per_step_rows} pair rows"},
        "cpu_baseline": {"value": round(val, 6), "unit": "TFLOP/s", "cores": os.cpu_count(), "kind": "oracle",
                         "sample": f"{per_step_rows} pair rows per step (all 4 heads), FP64 oracle forward, "
                                   "dq/dk/dv and the rows' share of dbias"},
        "e2e": {"value": round(val, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", choices=("crop768", "crop640", "crop384", "b2n256"), default="crop768",
                    help="crop768 is the headline; the smaller crops and the batched B=2, N=256, d=32 ragged "
                         "sweep case serve profiler captures")
    ap.add_argument("--gate-rows", type=int, default=768 * 768,
                    help="pair positions R of the --op gate workload (default 768^2; smaller only for profiling)")
    ap.add_argument("--op", choices=("attention", "tri_mul", "gate"), default="attention",
                    help="attention (the headline), the triangle multiplicative contraction, or the gated "
                         "output projection")
    ap.add_argument("--sweep", action="store_true",
                    help="time every workload (crops and the ragged N/d sweep), one JSON line each")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip timing the oracle on host cores")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.sweep:
        run_sweep(args)
        return
    if args.op == "gate":
        run_gate(args)
        return

    import datetime

    import torch
    import torch.distributed as dist
    if world > 1:
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.op == "tri_mul":
            res = run_tri_mul(args, rank, world, local_rank)
        else:
            res = run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            dist.destroy_process_group()
    if rank != 0:
        return
    if args.op == "tri_mul":
        Bn, C, N = res["shape"]
        pk, src = peaks()
        peak = float(pk["bf16_tflops"])
        step_flops = 6.0 * Bn * C * N ** 3
        value = whole_job_rate(world, step_flops, args.steps, res["ms"])
        fwd_t = 2.0 * Bn * C * N ** 3 / (res["fwd_ms"] * 1e-3) / 1e12
        bwd_t = 4.0 * Bn * C * N ** 3 / (res["bwd_ms"] * 1e-3) / 1e12
        line = {
            "metric": TRI_MUL_METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(res["ms"] / args.steps, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "triangle multiplicative contraction, outgoing edges: B=1, C=128, N=768, BF16 "
                                   "(forward + backward, three batched N^3 products per channel)",
                       "flops_per_step": step_flops, "l2": "inputs (453 MB) larger than the 126 MB L2; no flush"},
            "kernels_ms": {"fwd": round(res["fwd_ms"], 4), "bwd": round(res["bwd_ms"], 4)},
            "roofline": {"kernel": "tri_mul_gemm (fwd)", "bound": "tensor", "achieved": round(fwd_t, 2), "peak": peak,
                         "unit": "TFLOP/s", "frac": round(fwd_t / peak, 4), "traffic": None,
                         "peak_source": f"{src} bf16_tflops (burst)"},
            "bwd_tflops": round(bwd_t, 2),
            "gpu_launches": 3 * args.steps,
            "clocks": res["clocks"],
            "e2e": None,
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = tri_mul_cpu_baseline()
        print(json.dumps(line), flush=True)
        return
    Bn, N, H, d = res["shape"]
    fl = flops(Bn, N, H, d)
    pk, src = peaks()
    peak = float(pk["bf16_tflops"])
    ms = res["ms"]
    per_step_ms = ms / args.steps
    value = whole_job_rate(world, fl["step"], args.steps, ms)
    km = res["kern_ms"]
    algo = {"fwd": fl["fwd"], "bwd_main": fl["bwd_main"], "bwd_dbias": fl["bwd_dbias"]}
    dom = max(algo, key=lambda n: km[n])
    achieved = algo[dom] / (km[dom] * 1e-3) / 1e12
    # the step's three roofs: tensor cores (flops), HBM (algorithmic bytes: fwd reads
    # q,k,v + bias + mask, writes o, resid, lse; bwd reads q,k,v,o,resid,dout + lse,
    # bias, mask, writes dq,dk,dv + dbias) and the exponential unit (one exp2 per
    # score in each of the three passes, 16 per clock per SM, at the sampled clock)
    pair = Bn * N * N * H * d * 2
    algo_bytes = (3 * pair + Bn * H * N * N * 2 + Bn * N * N * 4 + 2 * pair + Bn * H * N * N * 4
                  + 6 * pair + Bn * H * N * N * 4 + Bn * H * N * N * 2 + Bn * N * N * 4 + 3 * pair + Bn * H * N * N * 2)
    sm_mhz = float((res["clocks"] or {}).get("sm_mhz") or 1965.0)
    roofs_ms = {"tensor": fl["step"] / (peak * 1e12) * 1e3,
                "hbm": algo_bytes / (float(pk["hbm_gbs"]) * 1e9) * 1e3,
                "exp_unit_mufu_only": 3.0 * Bn * H * N ** 3 / (148 * 16 * sm_mhz * 1e6) * 1e3}
    lengths = res["lengths"]
    eff_flops = 14.0 * H * d * sum(N * N * L for L in lengths)
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(per_step_ms, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD if args.workload == "crop768" else args.workload, "B": Bn, "N": N, "H": H, "d": d,
                   "bias": f"{res['bias_std']:g}*N(0,1)", "mask": res["mask"],
                   "flops_per_step": fl["step"], "l2": l2_note(4 * Bn * N * N * H * d * 2)},
        "pct_of_bf16_peak": round(100.0 * value / world / peak, 2),
        "pct_of_bf16_peak_sustained": round(100.0 * value / world / float(pk["bf16_tflops_sustained"]), 2),
        "kernels_ms": {n: round(v, 4) for n, v in km.items()},
        "fwd_tflops": round(fl["fwd"] / (km["fwd"] * 1e-3) / 1e12, 2),
        "bwd_tflops": round(fl["bwd"] / ((km["bwd_prep"] + km["bwd_main"] + km["bwd_dbias"]) * 1e-3) / 1e12, 2),
        "roofline": {"kernel": dom, "bound": "tensor", "achieved": round(achieved, 2), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "traffic": committed_traffic(dom) if args.workload == "crop768" else None,
                     "peak_source": f"{src} bf16_tflops (burst)"},
        "step_ms": {k: round(v, 4) for k, v in res["step_stats"].items()},
        "roofs_ms": {k: round(v, 4) for k, v in roofs_ms.items()},
        "effective_tflops": round(whole_job_rate(world, eff_flops, args.steps, ms), 3),
        "gpu_launches": attn_launches_per_step(Bn, N, H) * args.steps,
        "clocks": res["clocks"],
        "memory": res["memory"],
        "e2e": res["e2e"],
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = run_cpu_baseline()
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
