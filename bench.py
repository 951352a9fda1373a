#!/usr/bin/env python3
"""Benchmark: causal CP-attention forward TFLOP/s on B200 (one JSON line on rank 0).

Default workload: Llama-3-8B-shaped GQA ring attention at L = 212992 (208K), 32 query heads,
8 KV heads, d = 128, N_cp = 16 virtual ranks on one GPU, bf16 inputs i.i.d. N(0,1) from a
fixed seed.  One step = one cp_attn_fwd call (the whole hot path: every ring step of every
virtual rank, the online-softmax merges and the bf16 output cast) on inputs already resident
in HBM.  Inputs (Q 1.6 GiB, K/V 0.4 GiB each) are larger than the 126 MB L2, so no flush is
needed between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload c3]

Multi-GPU: every virtual rank of a problem runs on one GPU (the path has no exchange between
GPUs), so N > 1 runs N independent replicas (one per GPU, weak scaling); value = total FLOPs /
max-over-ranks time.
--impl reference times the fp64 CPU oracle on a bounded row sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "causal CP-attention fwd TFLOP/s (1 B200) and % of dense BF16 peak, L=208K"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="c3")
    ap.add_argument("--e2e-steps", type=int, default=None, help="end-to-end steps (default: --steps)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="target CPU work of the oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-rows", action="store_true", help="skip the per-row measurements of the other hot-path steps")
    ap.add_argument("--rows-only", action="store_true", help="measure only the other hot-path steps (one JSON line)")
    ap.add_argument("--rows-l-div", type=int, default=1, help="divide each row's sequence length (small ncu cases)")
    ap.add_argument("--row", action="append", default=[], help="with --rows-only: measure only this row (repeatable)")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "sequence_long_context_ring_b200", "csrc")
    for fn in ("fwd_kernel.cuh", "sm100.cuh"):
        with open(os.path.join(csrc, fn), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_from_profile(workload_name: str):
    """DRAM bytes per launch of the forward kernel from the committed ncu summary, or None
    when there is none or the kernel source changed since it was captured."""
    p = os.path.join(ROOT, "profiles", "ring_fwd_kernel_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    if d.get("kernel_source_hash") != kernel_source_hash():
        return None
    per = d.get("per_launch_bytes", {}).get(workload_name)
    return float(per) if per is not None else None


class ClockSampler:
    """nvidia-smi SM clock / throttle sampling during the timed region."""
    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        return self.summarize(self.lines)

    @staticmethod
    def summarize(lines):
        """Median SM clock, max clock and the throttle reasons seen active, from the sampled
        CSV lines (sm, max, power, active mask, hw_slowdown, hw_thermal, sw_thermal, sw_power_cap)."""
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                clk, clk_max = float(parts[0]), float(parts[1])
            except ValueError:
                continue
            sm.append(clk)
            mx = clk_max
            for nm, val in zip(names, parts[4:8]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------------------------
class OracleSample:
    """The fp64 oracle on a bounded sample of the workload: whole query rows (each exact by the
    definition) of the query heads that share KV head 0.  Inputs are drawn once."""

    def __init__(self, w):
        import oracle
        from sequence_long_context_ring_b200 import synth
        self.oracle = oracle
        self.w = w
        self.G = w.Hq // w.Hkv
        self.cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
        k = synth.normal_bf16(w.cfg_id, synth.TENSOR_ID["k"], w.kv_shape(), w.input_scale)
        v = synth.normal_bf16(w.cfg_id, synth.TENSOR_ID["v"], w.kv_shape(), w.input_scale)
        q = synth.normal_bf16(w.cfg_id, synth.TENSOR_ID["q"], w.q_shape(), w.input_scale)
        if w.seq_major:
            self.kh, self.vh = synth.bf16_bits_to_f64(k[0, :, 0]), synth.bf16_bits_to_f64(v[0, :, 0])
            self.q = [q[0, :, h].copy() for h in range(self.G)]
        else:
            self.kh, self.vh = synth.bf16_bits_to_f64(k[0, 0]), synth.bf16_bits_to_f64(v[0, 0])
            self.q = [q[0, h].copy() for h in range(self.G)]
        self.to64 = synth.bf16_bits_to_f64
        self.rng = np.random.default_rng(12345)

    def run(self, target_seconds: float):
        """Grow the row count until ~target_seconds of oracle work; returns (TFLOP/s, s, rows)."""
        w = self.w
        n_rows, flops, elapsed, total_rows = 8, 0.0, 0.0, 0
        while elapsed < target_seconds:
            rows = np.sort(self.rng.integers(0, w.L, n_rows))
            t0 = time.perf_counter()
            for h in range(self.G):
                self.oracle.attention_rows(self.to64(self.q[h][rows]), self.kh, self.vh, rows, causal=True)
            dt = time.perf_counter() - t0
            elapsed += dt
            flops += self.G * float(np.sum(4.0 * w.d * (rows + 1)))
            total_rows += self.G * n_rows
            if dt < target_seconds / 4:
                n_rows *= 2
        return flops / elapsed / 1e12, elapsed, total_rows

    def describe(self, rows: int) -> str:
        return (f"{rows} sampled query rows (random positions, full causal key prefix each) of the "
                f"{self.G} query heads sharing KV head 0 of {self.w.name}; fp64 numpy oracle")


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    sampler = OracleSample(w)
    per_step = max(2.0, min(args.cpu_seconds, 60.0) / 4)
    t_steps, vals, rows_total = [], [], 0
    for i in range(args.warmup + args.steps):
        tflops, sec, rows = sampler.run(per_step)
        if i >= args.warmup:
            t_steps.append(sec)
            vals.append(tflops)
            rows_total += rows
    value = statistics.mean(vals)
    cores, desc = sampler.cores, sampler.describe(rows_total)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(t_steps),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded bf16 N(0,1), rows sampled)",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "L": w.L, "d": w.d,
                   "n_cp": w.n_cp, "mode": w.mode, "causal": w.causal},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------------------------------
def max_over_ranks(ms: float, world: int, device) -> float:
    """The largest of every rank's device time (the job is as slow as its slowest replica)."""
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_step: float, steps: int, world: int, max_ms: float) -> float:
    """Throughput of the whole job: every replica's FLOPs over the slowest replica's time."""
    return world * flops_per_step * steps / (max_ms / 1e3) / 1e12


def _time_ms(fn, stream, warmup=3, reps=10):
    """Median device time of fn() (CUDA events on `stream`, synchronised on both sides)."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
    ev[0].record(stream)
    for i in range(reps):
        fn()
        ev[i + 1].record(stream)
    torch.cuda.synchronize()
    return statistics.median(ev[i].elapsed_time(ev[i + 1]) for i in range(reps))


def measure_rows(dev, peaks, l_div: int = 1, only=None):
    """Device time of every other step of the hot path at its workload's shape (random bf16
    device inputs; no host data): the Ulysses permutes and the Ulysses forward (c4 shape), the
    2D forward and backward (c5 shape), the ring backward (c2 shape), one step-wise ring
    step plus its LSE merge (c2 shape), the point-to-point FIR convolution with a short and a
    medium filter (c3's sequence and chunking, 4096 channels), and the distributed FFT
    convolution with a sequence-long filter (c4's sequence, 4096 channels).  Each entry carries its
    roofline: HBM-bound steps against the measured copy bandwidth, contractions against the
    measured bf16 peak.  `only`: a set of row names to measure (None: all)."""
    import torch
    from sequence_long_context_ring_b200 import binding
    from sequence_long_context_ring_b200.binding import ConvPlan, FftConvPlan, Plan
    from sequence_long_context_ring_b200.configs import CONV_WORKLOADS, FFT_WORKLOADS, WORKLOADS

    hbm = float(peaks["hbm_gbs"])
    tc = float(peaks.get("bf16_tflops", peaks.get("bf16_tflops_sustained")))
    stream = torch.cuda.current_stream(dev)
    g = torch.Generator(device=dev)
    g.manual_seed(2024)
    rows = {}

    def rnd(*shape):
        return torch.randn(shape, device=dev, generator=g, dtype=torch.float32).to(torch.bfloat16)

    def hbm_row(name, workload, ms, nbytes):
        gbs = nbytes / (ms / 1e3) / 1e9
        rows[name] = {"workload": workload, "ms": ms, "value": gbs, "unit": "GB/s",
                      "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                                   "bytes": nbytes}}

    def tc_row(name, workload, ms, flops):
        tf = flops / (ms / 1e3) / 1e12
        rows[name] = {"workload": workload, "ms": ms, "value": tf, "unit": "TFLOP/s",
                      "roofline": {"bound": "tensor", "achieved": tf, "peak": tc, "unit": "TFLOP/s", "frac": tf / tc,
                                   "flops": flops}}

    groups = {"ulysses": ("seq2head", "head2seq", "seq2head_zigzag", "ulysses_fwd"), "2d": ("2d_fwd", "2d_bwd"),
              "ring": ("ring_bwd", "ring_step", "ring_step_zigzag", "lse_merge"), "fir": ("fir_short", "fir_medium"),
              "fft": ("fft_long",)}
    want = lambda grp: only is None or any(n in only for n in groups[grp])

    if want("ulysses"):
        # a4 / a5: Ulysses re-layout at the c4 shape (one 1 GiB tensor each way)
        w = WORKLOADS["c4"]
        L = w.L // l_div
        x = rnd(w.B, L, w.Hq, w.d)
        y = torch.empty((w.B, w.Hq, L, w.d), dtype=torch.bfloat16, device=dev)
        nbytes = 2 * x.numel() * 2
        hbm_row("seq2head", f"c4 shape [1,{L},32,128] bf16", _time_ms(lambda: binding.seq2head(w.n_cp, x, y), stream), nbytes)
        hbm_row("head2seq", f"c4 shape [1,32,{L},128] bf16", _time_ms(lambda: binding.head2seq(w.n_cp, y, x), stream), nbytes)
        # the same all-to-all with zig-zag rank-major rows (row remap between rank and position order)
        hbm_row("seq2head_zigzag", f"c4 shape [1,{L},32,128] bf16, zig-zag split",
                _time_ms(lambda: binding.seq2head(w.n_cp, x, y, split="zigzag"), stream), nbytes)
        del y
        # a6: Ulysses forward, c4 (seq->head, attention per head group, head->seq)
        k, v = rnd(w.B, L, w.Hkv, w.d), rnd(w.B, L, w.Hkv, w.d)
        plan = Plan(w.B, w.Hq, w.Hkv, L, w.d, n_cp=w.n_cp, mode="ulysses")
        o = torch.empty_like(x)
        lse = torch.empty((w.B, w.Hq, L), dtype=torch.float32, device=dev)
        ws = plan.workspace(False, dev)
        tc_row("ulysses_fwd", f"c4 L={L} degree 8", _time_ms(lambda: plan.fwd(x, k, v, o, lse, ws, stream), stream, reps=5),
               plan.flops(False))
        del x, k, v, o, lse, ws, plan

    if want("2d"):
        # 2D forward and backward, c5
        w = WORKLOADS["c5"]
        L = w.L // l_div
        q, k, v, do = rnd(w.B, L, w.Hq, w.d), rnd(w.B, L, w.Hkv, w.d), rnd(w.B, L, w.Hkv, w.d), rnd(w.B, L, w.Hq, w.d)
        plan = Plan(w.B, w.Hq, w.Hkv, L, w.d, n_cp=w.n_cp, n_hp=w.n_hp, mode="2d")
        o = torch.empty_like(q)
        lse = torch.empty((w.B, w.Hq, L), dtype=torch.float32, device=dev)
        ws = plan.workspace(False, dev)
        tc_row("2d_fwd", f"c5 L={L} grid 4x4", _time_ms(lambda: plan.fwd(q, k, v, o, lse, ws, stream), stream, reps=5),
               plan.flops(False))
        wsb = plan.workspace(True, dev)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        tc_row("2d_bwd", f"c5 L={L} grid 4x4 (D preprocess, a2a of q/k/v/dO, kernel, dQ cast, a2a back)",
               _time_ms(lambda: plan.bwd(q, k, v, o, lse, do, dq, dk, dv, wsb, stream), stream, reps=5), plan.flops(True))
        del q, k, v, do, o, lse, ws, wsb, dq, dk, dv, plan

    if want("ring"):
        # ring backward and the step-wise path at the c2 shape
        w = WORKLOADS["c2"]
        L = w.L // l_div
        q, k, v, do = rnd(w.B, w.Hq, L, w.d), rnd(w.B, w.Hkv, L, w.d), rnd(w.B, w.Hkv, L, w.d), rnd(w.B, w.Hq, L, w.d)
        plan = Plan(w.B, w.Hq, w.Hkv, L, w.d, n_cp=w.n_cp)
        o, lse = plan.fwd(q, k, v)
        wsb = plan.workspace(True, dev)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        tc_row("ring_bwd", f"c2 L={L} N=8 (D preprocess, kernel, dQ cast)",
               _time_ms(lambda: plan.bwd(q, k, v, o, lse, do, dq, dk, dv, wsb, stream), stream, reps=5), plan.flops(True))
        ch = L // w.n_cp
        po = torch.empty((w.B, w.Hq, ch, w.d), dtype=torch.float32, device=dev)
        pl = torch.empty((w.B, w.Hq, ch), dtype=torch.float32, device=dev)
        r = w.n_cp - 1
        tc_row("ring_step", f"c2 rank {r} step 1 (full chunk {r - 1} of {ch} keys)",
               _time_ms(lambda: plan.ring_step(r, 1, q, k, v, po, pl, stream), stream),
               4.0 * w.B * w.Hq * w.d * ch * ch)
        zplan = Plan(w.B, w.Hq, w.Hkv, L, w.d, n_cp=w.n_cp, split="zigzag")
        tc_row("ring_step_zigzag", f"c2 zig-zag rank {r} step 1 (two query shards x two KV shards)",
               _time_ms(lambda: zplan.ring_step(r, 1, q, k, v, po, pl, stream), stream),
               4.0 * w.B * w.Hq * w.d * (2 * (ch // 2) * (ch // 2)))
        acc_o = torch.zeros_like(po)
        acc_l = torch.full_like(pl, -float("inf"))
        hbm_row("lse_merge", f"c2 chunk [1,32,{ch},128] fp32",
                _time_ms(lambda: binding.lse_merge(acc_o, acc_l, po, pl, stream), stream),
                (3 * po.numel() + 3 * pl.numel()) * 4)
        torch.cuda.synchronize()
        st, word = plan.device_status(stream)
        if st != 0:
            raise RuntimeError(f"device status {st} ({word:#x}) in the row measurements")

    if want("fir"):
        # point-to-point FIR convolution over all 16 virtual ranks (halos read in place): x read
        # once, y written once (1.7 GB each at full size, well above L2)
        for key in [k for k in ("fir_short", "fir_medium") if only is None or k in only]:
            w = CONV_WORKLOADS[key]
            L = w.L // l_div
            x = rnd(w.B, w.D, L)
            h = (rnd(w.D, w.lh).float() * w.h_scale).to(torch.bfloat16)
            y = torch.empty_like(x)
            cplan = ConvPlan(w.B, w.D, L, w.lh, w.n_cp)
            hbm_row(key, f"[1,{w.D},{L}] bf16, l_h={w.lh}, N_cp={w.n_cp}",
                    _time_ms(lambda: cplan.fwd(x, h, y, stream), stream), cplan.cost()[0])
            torch.cuda.synchronize()
            st, word = cplan.device_status(stream)
            if st != 0:
                raise RuntimeError(f"device status {st} ({word:#x}) in the {key} row")
            del x, h, y, cplan

    if want("fft"):
        # distributed FFT convolution with a filter as long as the sequence (all 16 virtual
        # ranks): filter spectra, signal slices, cross-rank inverse; bytes of its three passes
        w = FFT_WORKLOADS["fft_long"]
        L = w.L // l_div
        x = rnd(w.B, w.D, L)
        h = (rnd(w.D, L).float() * L ** -0.5).to(torch.bfloat16)
        y = torch.empty_like(x)
        fplan = FftConvPlan(w.B, w.D, L, w.n_cp)
        fws = fplan.workspace(dev)
        hbm_row("fft_long", f"[1,{w.D},{L}] bf16, filter length {L}, N_cp={w.n_cp}",
                _time_ms(lambda: fplan.fwd(x, h, y, fws, stream), stream, reps=5), fplan.cost()[0])
        del x, h, y, fws, fplan
    return rows


def run_rows_only(args):
    import torch
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    peaks, src = load_peaks()
    rows = measure_rows(dev, peaks, args.rows_l_div, set(args.row) if args.row else None)
    print(json.dumps({"rows": rows, "peaks": src, "rows_l_div": args.rows_l_div}), flush=True)
    return 0


def run_ours(args, w):
    import torch
    import torch.distributed as dist

    from sequence_long_context_ring_b200 import synth
    from sequence_long_context_ring_b200.binding import Plan

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=120))

    def barrier():
        if world > 1:
            dist.barrier()

    # inputs: identical seeded data on every replica
    def up(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(torch.bfloat16)

    qb = synth.normal_bf16(w.cfg_id, synth.TENSOR_ID["q"], w.q_shape(), w.input_scale)
    kb = synth.normal_bf16(w.cfg_id, synth.TENSOR_ID["k"], w.kv_shape(), w.input_scale)
    vb = synth.normal_bf16(w.cfg_id, synth.TENSOR_ID["v"], w.kv_shape(), w.input_scale)
    q, k, v = up(qb), up(kb), up(vb)
    plan = Plan(w.B, w.Hq, w.Hkv, w.L, w.d, n_cp=w.n_cp, n_hp=w.n_hp, mode=w.mode, causal=w.causal)
    o = torch.empty(w.q_shape(), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.B, w.Hq, w.L), dtype=torch.float32, device=dev)
    ws = plan.workspace(False, dev)
    stream = torch.cuda.current_stream(dev)
    flops = plan.flops(False)

    for _ in range(args.warmup):
        plan.fwd(q, k, v, o, lse, ws, stream)
    torch.cuda.synchronize(dev)
    st, word = plan.device_status(stream)
    if st != 0:
        raise RuntimeError(f"device status {st} (word {word:#x}) after warm-up")

    # ---- device-timed region: K steps, inputs resident in HBM ----
    clocks = ClockSampler(torch.cuda.current_device() if world == 1 else local)
    barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    time.sleep(0.3)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    ev[0].record(stream)
    for i in range(args.steps):
        plan.fwd(q, k, v, o, lse, ws, stream)
        ev[i + 1].record(stream)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    barrier()
    per_step = [ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps)]
    total_ms = ev[0].elapsed_time(ev[-1])
    st, word = plan.device_status(stream)
    if st != 0:
        raise RuntimeError(f"device status {st} (word {word:#x}) in the timed region")
    max_ms = max_over_ranks(total_ms, world, dev)
    value = whole_job_tflops(flops, args.steps, world, max_ms)

    # ---- end-to-end through the public API with host buffers ----
    qh, kh, vh = (torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16).pin_memory()
                  for b in (qb, kb, vb))
    oh = torch.empty(w.q_shape(), dtype=torch.bfloat16).pin_memory()
    lh = torch.empty((w.B, w.Hq, w.L), dtype=torch.float32).pin_memory()
    staging = []                                 # device buffers of the e2e path, freed below
    if w.mode == "ring":
        # the library's host-buffer entry point: copies in and out overlap the kernels
        hws = torch.empty(plan.host_workspace_size(), dtype=torch.uint8, device=dev)
        staging.append(hws)

        def e2e_step():
            plan.fwd_host(qh, kh, vh, oh, lh, hws, stream)
    else:
        qd, kd, vd = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        staging += [qd, kd, vd]

        def e2e_step():
            qd.copy_(qh, non_blocking=True)
            kd.copy_(kh, non_blocking=True)
            vd.copy_(vh, non_blocking=True)
            plan.fwd(qd, kd, vd, o, lse, ws, stream)
            oh.copy_(o, non_blocking=True)
            lh.copy_(lse, non_blocking=True)
    e2e_step()                                   # warm-up (staging buffers touched once)
    barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_steps = args.e2e_steps or args.steps     # the same step count as the device figure
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1)
    e2e_value = whole_job_tflops(flops, e2e_steps, world, max_over_ranks(e2e_ms, world, dev))
    h2d = sum(x.numel() * x.element_size() for x in (qh, kh, vh))
    d2h = oh.numel() * oh.element_size() + lh.numel() * lh.element_size()

    # ---- roofline of the dominant kernel (ring mode: one fused launch per step) ----
    peaks, peak_src = load_peaks()
    peak = float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops")))
    launch_ms = statistics.mean(per_step) if w.mode == "ring" else None
    roof = None
    if launch_ms:
        achieved = flops / (launch_ms / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "traffic": traffic_from_profile(w.name),
                "kernel": "ring_fwd_kernel<128>",
                "peak_source": f"{peak_src} bf16_tflops_sustained (seconds-long back-to-back launches)"}
    launches = args.steps * (1 if w.mode == "ring" else 5)

    row_meas = None
    if world == 1 and not args.no_rows:
        del qh, kh, vh, oh, lh, e2e_step
        staging.clear()
        row_meas = measure_rows(dev, peaks)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        try:
            sampler = OracleSample(w)
            tf, sec, rows = sampler.run(args.cpu_seconds)
            cpu = {"value": tf, "unit": "TFLOP/s", "cores": sampler.cores, "kind": "oracle",
                   "sample": sampler.describe(rows), "seconds": sec}
        except Exception as exc:  # the GPU numbers above stay valid; report why this leg is missing
            cpu = {"value": None, "unit": "TFLOP/s", "kind": "oracle", "error": repr(exc)}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded bf16 N(0,1), Llama-3-8B-shaped)",
            "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "L": w.L, "d": w.d,
                       "n_cp": w.n_cp, "n_hp": w.n_hp, "mode": w.mode, "causal": w.causal,
                       "parallelism": f"{world} independent replica(s), all virtual ranks on each GPU",
                       "l2": "inputs larger than L2 (Q 1.6 GiB), no flush"},
            "pct_of_peak": 100.0 * (flops / (max_ms / args.steps / 1e3) / 1e12) / peak,
            "per_step_ms": per_step,
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "steps": e2e_steps},
            "gpu_launches": launches,
            "clocks": clk,
            "rows": row_meas,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    from sequence_long_context_ring_b200.configs import WORKLOADS
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    if args.rows_only:
        return run_rows_only(args)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
