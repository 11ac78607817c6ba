#!/usr/bin/env python
"""Benchmark of the hybrid-attention forward (one layer call = one step).

Default workload: the Wan-2.1-1.3B-shaped bidirectional layer (B=1, H=12,
d=128, 21 frames x 1560 tokens, 3-frame chunks +/- 1 frame, bf16). Prints one
JSON line: effective TFLOP/s (kept-window pairs x 4d plus linear-state FLOPs)
over all ranks, tokens/s, the dominant kernel's roofline, the oracle's CPU
throughput on a bounded sample, an end-to-end figure through the public API
with host buffers, and the SM clocks seen during the timed region.

  python bench.py [--gpus N --steps K --warmup W] [--impl reference] [--workload NAME]

Multi-GPU: one process per GPU (torchrun). Batch elements are independent, so
each rank runs its own layer call on its own inputs (weak scaling, no
data-path collective); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from linear_attention_video_hyat_b200 import workloads as wl  # noqa: E402

METRIC = "hybrid-attn effective TFLOP/s & tokens/s per layer; % of B200 BF16 TC peak"
L2_BYTES = 126 * 2 ** 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# the attention call of the default schedule: the wide-softmax kernel and its redo pass
KERNEL_SOURCES = ["linear_attention_video_hyat_b200/csrc/attn_tc_wide.cu", "linear_attention_video_hyat_b200/csrc/attn_tc.cu"]
# the streaming bench's --rope step: a temporal band of 44 of the 128 head dimensions, the
# index capped at 21 frames (the pages' example of a pretrained model's range), base 10000
ROPE = {"t_dims": 44, "cap": 21, "base": 10000.0}



# Idle time before the per-launch timing pass: the 1000 W power limit lowers the SM clock after
# the timed pass's load; a second of idle lets the kernel pass run at the timed pass's clocks.
KERNEL_PASS_IDLE_S = 1.0



def kernel_source_digest() -> str:
    """sha256 of the attention kernels' sources with comments and runs of blank space removed:
    the DRAM traffic record stays valid across edits of comments only, and lapses with any
    change to the code."""
    def code(path):
        t = open(os.path.join(ROOT, path), encoding="utf-8").read()
        t = re.sub(r"/\*.*?\*/", " ", t, flags=re.S)
        t = re.sub(r"//[^\n]*", " ", t)
        return re.sub(r"\s+", " ", t).strip().encode()
    return hashlib.sha256(b"".join(code(f) for f in KERNEL_SOURCES)).hexdigest()

def l2_note(io_bytes):
    """How the timed region stands to the 126 MB L2: the full-size layers' inputs exceed it."""
    mb = io_bytes / 1e6
    if mb > 126:
        return "inputs larger than L2 (Q,K,V,O %.0f MB > 126 MB); no flush" % mb
    return "inputs fit in L2 (Q,K,V,O %.1f MB); no flush, so repeated steps run from L2" % mb


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default=wl.WAN13B_BIDIR.name, choices=sorted(wl.WORKLOADS))
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--schedule", choices=["pair", "one-warp", "single"], default="pair",
                   help="tensor-core attention schedule: a pair of query tiles per CTA with two softmax "
                        "warps per row (default), the pair schedule with one softmax warp per row "
                        "(HYAT_FLAG_PAIR_ONE_WARP), or one query tile per CTA (HYAT_FLAG_SINGLE_TILE; "
                        "bidirectional modes)")
    p.add_argument("--rope", action="store_true",
                   help="streaming workload: the capped temporal RoPE of the chunk's Q and K fused "
                        "into each step (hyat_config.rope_t_dims)")
    p.add_argument("--rope-standalone", action="store_true",
                   help="streaming workload: the same RoPE as --rope, as two hyat_rope_temporal calls "
                        "(Q, K) before each plain step (the unfused baseline of --rope)")
    p.add_argument("--graph", action="store_true",
                   help="streaming workload: device step masks, steady steps replayed from the "
                        "library's CUDA graphs (hyat_fwd_stream_step_graph)")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------- work counts
def workload_mask(w):
    """The tile mask a block-mask workload runs with (None for the other modes)."""
    from linear_attention_video_hyat_b200 import hyat
    if w.mode == "lvsa":
        return hyat.lvsa_mask(w.n_frames, w.tokens_per_frame, w.window_frames, w.anchor_stride, w.rotation)[None]
    return None


def work_counts(w):
    """Effective FLOPs of one call and the attention kernel's share, from the library layout."""
    from linear_attention_video_hyat_b200 import hyat
    cfg = hyat.config_from_workload(w)
    work, ent = hyat.plan_layout(cfg, workload_mask(w))
    per_bh = work[work[:, 0] == 0]
    klen = np.concatenate([[0], np.cumsum(ent[:, 1].astype(np.int64))])
    pairs = int(sum(int(it[2]) * int(klen[it[5]] - klen[it[4]]) for it in per_bh))
    BH, d, N = w.B * w.H, w.d, w.N
    soft = 4 * d * pairs * BH
    fold = BH * N * (2 * d * d + d)
    apply = BH * N * (2 * d * d + 2 * d)
    return {"pairs_per_head": pairs, "softmax_flops": soft, "state_flops": fold + apply,
            "total_flops": soft + fold + apply, "attn_kernel_flops": soft + apply,
            "state_kernel_bytes": 2 * BH * N * d * 2 + BH * (N // w.tokens_per_frame) * (d * d + d) * 4}


# ----------------------------------------------------------------- multi-rank
def max_over_ranks(ms, device):
    """The slowest rank's time (every rank calls this; identity on one process)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return ms
    t = torch.tensor([ms], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(flops_per_rank, tokens_per_rank, ms_max, world):
    """Whole-job effective TFLOP/s and tokens/s: every rank's units over the slowest rank's time."""
    return flops_per_rank * world / (ms_max / 1e3) / 1e12, tokens_per_rank * world / (ms_max / 1e3)


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the GPU runs."""

    def __init__(self, index):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:
            pass
        self.names = {}
        if self._ok:
            for name in ("HwSlowdown", "HwThermalSlowdown", "SwThermalSlowdown", "SwPowerCap", "HwPowerBrakeSlowdown"):
                for prefix in ("nvmlClocksEventReason", "nvmlClocksThrottleReason"):
                    v = getattr(self.nv, prefix + name, None)
                    if v is not None:
                        self.names[name] = v
                        break

    def _run(self):
        get_reasons = getattr(self.nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            self.nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = get_reasons(self.h)
                for n, bit in self.names.items():
                    if r & bit:
                        self.reasons.add(n)
            except Exception:
                pass
            time.sleep(0.005)

    def __enter__(self):
        if self._ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._ok:
            self.t.join()

    def summary(self):
        snake = {"HwSlowdown": "hw_slowdown", "HwThermalSlowdown": "hw_thermal_slowdown",
                 "SwThermalSlowdown": "sw_thermal_slowdown", "SwPowerCap": "sw_power_cap",
                 "HwPowerBrakeSlowdown": "hw_power_brake_slowdown"}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "samples": len(self.samples),
                "reasons": sorted(snake[r] for r in self.reasons)}


# ----------------------------------------------------------------- oracle (CPU) leg
def oracle_sample(w, n_blocks, rows_per_block=256, seed=0, qkv=None):
    """Time the fp64 oracle on `n_blocks` blocks of query rows; returns (seconds, rows)."""
    import oracle
    q, k, v = wl.gen_qkv(w) if qkv is None else qkv
    rng = np.random.default_rng(seed)
    t = 0.0
    rows_done = 0
    for b in range(n_blocks):
        h = int(rng.integers(0, w.H))
        r0 = int(rng.integers(0, w.N - rows_per_block + 1))
        rows = np.arange(r0, r0 + rows_per_block)
        qs = q[:, h:h + 1].float().numpy()
        ks = k[:, h:h + 1].float().numpy()
        vs = v[:, h:h + 1].float().numpy()
        t0 = time.perf_counter()
        if w.mode == "window":
            oracle.bidir_window_attention(qs, ks, vs, w.tokens_per_frame, w.n_frames, w.chunk_frames,
                                          w.halo_frames, rows=rows)
        elif w.mode == "radial":
            oracle.radial_attention(qs, ks, vs, w.n_frames, w.tokens_per_frame, rows=rows)
        elif w.mode == "lvsa":
            mask = oracle.lvsa_tile_mask(w.n_frames, w.tokens_per_frame, w.window_frames, w.anchor_stride,
                                         w.rotation)[None]
            oracle.blockmask_attention(qs, ks, vs, mask, rows=rows)
        else:
            raise ValueError("oracle timing covers the bidirectional workloads")
        t += time.perf_counter() - t0
        rows_done += rows_per_block
    return t, rows_done


def cpu_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max((i.get("num_threads", 1) for i in info), default=os.cpu_count())
    except Exception:
        return os.cpu_count()


def cpu_info():
    """The host the oracle runs on: CPU model, logical cores, and the BLAS library with its
    thread count (the oracle's matrix products run in it)."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    blas = None
    try:
        import threadpoolctl
        for i in threadpoolctl.threadpool_info():
            if i.get("user_api") == "blas":
                blas = {"library": i.get("internal_api"), "threads": i.get("num_threads")}
                break
    except Exception:
        pass
    return {"cpu_model": model, "logical_cores": os.cpu_count(), "blas": blas}


def oracle_work_counts(w):
    """Effective FLOPs of one call from the oracle's own window and mask rules (the reference
    arm never loads the library)."""
    import oracle
    if w.mode == "window":
        pairs = int(oracle.effective_pairs_bidir(w.tokens_per_frame, w.n_frames, w.chunk_frames, w.halo_frames))
    else:
        if w.mode == "radial":
            tm = oracle.radial_tile_mask(w.n_frames, w.tokens_per_frame)[None]
        else:
            tm = oracle.lvsa_tile_mask(w.n_frames, w.tokens_per_frame, w.window_frames, w.anchor_stride,
                                       w.rotation)[None]
        pairs = int(oracle.effective_pairs_tile_mask(tm, w.N, w.N)[0])
    BH, d, N = w.B * w.H, w.d, w.N
    soft = 4 * d * pairs * BH
    state = BH * N * (2 * d * d + d) + BH * N * (2 * d * d + 2 * d)
    return {"pairs_per_head": pairs, "total_flops": soft + state}


def cpu_rate(w, counts, n_blocks, qkv=None):
    secs, rows = oracle_sample(w, n_blocks, qkv=qkv)
    total_rows = w.B * w.H * w.N
    frac = rows / total_rows
    tflops = counts["total_flops"] * frac / secs / 1e12
    return tflops, rows / secs, secs, rows


# ----------------------------------------------------------------- end to end
def e2e_pipelined(call, host_in, host_out, dev_in, dev_out, stream, steps, dev):
    """Milliseconds per step of: H2D of the step's inputs from pinned host memory, the layer
    call, D2H of its output. Device tensors are double-buffered and each copy direction has
    its own stream, so step i+1's inputs and step i-1's output cross PCIe while step i
    computes. Events on the compute stream bracket the whole loop (the copy streams join it
    at both ends)."""
    h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    in_free = [ev(), ev()]       # compute of the step that last read the buffer finished
    in_ready = [ev(), ev()]
    out_ready = [ev(), ev()]
    out_free = [ev(), ev()]      # D2H of the step that last wrote the buffer finished
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    h2d.wait_event(t0)
    d2h.wait_event(t0)
    for i in range(steps):
        b = i % 2
        with torch.cuda.stream(h2d):
            if i >= 2:
                h2d.wait_event(in_free[b])
            for dst, src in zip(dev_in[b], host_in):
                dst.copy_(src, non_blocking=True)
            in_ready[b].record(h2d)
        stream.wait_event(in_ready[b])
        if i >= 2:
            stream.wait_event(out_free[b])
        call(dev_in[b], dev_out[b], stream)
        in_free[b].record(stream)
        out_ready[b].record(stream)
        with torch.cuda.stream(d2h):
            d2h.wait_event(out_ready[b])
            host_out[b].copy_(dev_out[b], non_blocking=True)
            out_free[b].record(d2h)
    for b in range(2):
        stream.wait_event(out_free[b])
    t1.record(stream)
    torch.cuda.synchronize(dev)
    return t0.elapsed_time(t1) / steps


# ----------------------------------------------------------------- streaming workload
def stream_step_flops(w, mask, fold):
    """Effective FLOPs of one streaming step: 4d per (query, key) pair inside kept tiles, the
    fold of one evicted chunk (if any) and the linear term applied to every query."""
    L, d, BH = w.chunk_tokens, w.d, w.B * w.H
    nqt = wl.stream_tiles_per_chunk(w)
    qlen = np.minimum(wl.TILE, L - wl.TILE * np.arange(nqt)).astype(np.int64)
    klen = np.tile(qlen, mask.shape[2] // nqt)
    per_head = np.einsum("hij,i,j->h", mask.astype(np.int64), qlen, klen)
    pairs = int(per_head.sum()) * (w.B * w.H // mask.shape[0])
    soft = 4 * d * pairs
    apply = BH * L * (2 * d * d + 2 * d)
    folded = BH * L * (2 * d * d + d) if fold else 0
    return soft + apply + folded, soft + apply


def bench_stream(a, w, rank, world, local):
    """Streaming steps of chunk `w.chunk_tokens` tokens: K steady steps after W warm-up steps."""
    from linear_attention_video_hyat_b200 import hyat
    nwc = w.window_frames // w.chunk_frames
    warm = max(a.warmup, nwc, 3)
    config = {"workload": w.name, "B": w.B, "H": w.H, "d": w.d, "chunk_tokens": w.chunk_tokens,
              "tokens_per_frame": w.tokens_per_frame, "chunk_frames": w.chunk_frames,
              "window_frames": w.window_frames, "mode": w.mode, "mask": "Bernoulli(0.5) + diagonal tiles",
              "parallelism": f"replicas{world}" if world > 1 else "single",
              "l2": "per step: fresh Q, K, V (86 MB) and the ring (86 MB); no flush"}
    if a.rope:
        config["rope"] = dict(ROPE, ref="first frame of the oldest window chunk")
    n_dist = 4           # distinct steady-state inputs, cycled
    inputs = [wl.gen_stream_step(w, nwc + i, seed=w.seed + rank) for i in range(n_dist)]
    flops = [stream_step_flops(w, m, True) for _, _, _, m in inputs]
    mean_flops = float(np.mean([f[0] for f in flops]))
    mean_attn = float(np.mean([f[1] for f in flops]))
    if a.impl == "reference":
        if rank != 0:
            return 0
        import oracle
        L = w.chunk_tokens
        hist = [wl.gen_stream_step(w, s, seed=w.seed) for s in range(nwc + 1)]
        kh = np.concatenate([x[1].float().numpy() for x in hist], axis=2)
        vh = np.concatenate([x[2].float().numpy() for x in hist], axis=2)
        q, mask = hist[-1][0].float().numpy(), hist[-1][3]
        rng = np.random.default_rng(0)
        secs, rows_done = 0.0, 0
        for i in range(a.warmup + a.steps):
            hh = int(rng.integers(0, w.H))
            r0 = int(rng.integers(0, L - 256 + 1))
            t0 = time.perf_counter()
            oracle.stream_step_attention(q[:, hh:hh + 1], kh[:, hh:hh + 1], vh[:, hh:hh + 1], nwc, L, nwc,
                                         mask[hh:hh + 1], rows=np.arange(r0, r0 + 256))
            if i >= a.warmup:
                secs += time.perf_counter() - t0
                rows_done += 256
        frac = rows_done / (w.B * w.H * L)
        value = mean_flops * frac / secs / 1e12
        line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": a.gpus, "steps": a.steps,
                "warmup": a.warmup, "ms_per_step": 1e3 * secs / a.steps, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
                "impl": "reference", "tokens_per_s": rows_done / secs,
                "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
                                 "sample": f"{a.steps} blocks of 256 query rows (one head each) of a steady step",
                                 **cpu_info()},
                "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    cfg = hyat.config_from_workload(w, mask_heads=w.H, rope=ROPE if a.rope else None,
                                    flags=hyat.FLAG_PAIR_ONE_WARP if a.schedule == "one-warp" else 0)
    config["schedule"] = a.schedule
    if a.graph:
        config["graph"] = "device masks; steady steps replayed from the library's CUDA graphs"
    if a.rope or a.rope_standalone:
        config["rope"] = dict(ROPE, ref="first frame of the oldest rolling-window chunk",
                              path="fused into the step" if a.rope else "hyat_rope_temporal on Q and K, then the step")
    nsink = w.sink_frames // w.chunk_frames
    rope_events = []

    def rope_standalone(q, k, s_, timed):
        """The unfused RoPE of step s_: Q and K turned by their capped offsets from the first
        frame of the oldest rolling-window chunk (the chunk's own while the window has none)."""
        first_window = max(nsink, s_ - nwc + 1)
        f0 = s_ * w.chunk_frames
        ref = first_window * w.chunk_frames if s_ >= first_window else f0
        if timed:
            ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            ev[0].record(stream)
        for x, y in ((q, qr), (k, kr)):
            hyat.rope_temporal(x, w.tokens_per_frame, f0, ref, ROPE["cap"], ROPE["t_dims"], ROPE["base"], out=y)
        if timed:
            ev[1].record(stream)
            rope_events.append(ev)
        return qr, kr
    dev_in = [(q.to(dev), k.to(dev), v.to(dev), m, torch.from_numpy(np.ascontiguousarray(m)).to(dev))
              for q, k, v, m in inputs]
    od = torch.empty_like(dev_in[0][0])
    qr, kr = torch.empty_like(od), torch.empty_like(od)      # the unfused RoPE's outputs
    stream = torch.cuda.current_stream(dev)

    def step(h, x, m_host, s_, out, timed=False):
        q, k, v, m, md = x
        if a.rope_standalone:
            q, k = rope_standalone(q, k, s_, timed)
        if s_ < nwc:          # the window is still filling: masks of the growing shape
            m = wl.gen_stream_step(w, s_, seed=w.seed + rank)[3]
            md = torch.from_numpy(np.ascontiguousarray(m)).to(dev)
        if a.graph:
            h.stream_step_dev(q, k, v, mask=md, out=out, graph=True)
        else:
            h.stream_step(q, k, v, mask=m if m_host is None else m_host, out=out)

    def run(h, steps, first, timed=False):
        for i in range(steps):
            s_ = first + i
            step(h, dev_in[s_ % n_dist], None, s_, od, timed)

    h = hyat.Hyat(cfg, device=dev)
    run(h, warm + n_dist * nwc, 0)        # warm-up (and, with --graph, one capture per phase and input set)
    h.sync()
    first = warm + n_dist * nwc
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clk = ClockSampler(local)
    host0 = time.perf_counter()
    with clk:
        t0.record(stream)
        run(h, a.steps, first)
        t1.record(stream)
        host_s = time.perf_counter() - host0
        torch.cuda.synchronize(dev)
    h.sync()
    ms = max_over_ranks(t0.elapsed_time(t1) / a.steps, dev)
    first += a.steps
    time.sleep(KERNEL_PASS_IDLE_S)
    h.set_profiling(True)        # per-launch events (graph replay is off while profiling)
    h.kernel_times()
    with ClockSampler(local) as clk2:
        run(h, a.steps, first, timed=True)
        torch.cuda.synchronize(dev)
    first += a.steps
    kt = h.kernel_times()
    h.set_profiling(False)
    launches = sum(n for _, n in kt.values()) + 2 * len(rope_events)
    if a.schedule == "pair":
        launches += kt["attention"][1]          # the attention kernel and its redo pass
    value, tokens_per_s = job_throughput(mean_flops, w.B * w.chunk_tokens, ms, world)
    pk, pk_src = peaks()
    attn_ms = kt["attention"][0] / max(kt["attention"][1], 1)
    achieved = mean_attn / (attn_ms / 1e3) / 1e12
    roofline = {"bound": "tensor", "kernel": "attention", "achieved": achieved,
                "timing": "per-launch CUDA events over a second pass of K steps",
                "clocks_kernel_pass": clk2.summary(), "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / pk["bf16_tflops"], "peak_kind": f"{pk_src} bf16 burst",
                "peak_sustained": pk["bf16_tflops_sustained"],
                "frac_sustained": achieved / pk["bf16_tflops_sustained"], "traffic": None,
                "launch_ms": attn_ms, "algorithmic_flops_per_launch": mean_attn}
    kernels = {k_: {"ms_per_launch": t_ / max(n_, 1), "launches": n_} for k_, (t_, n_) in kt.items() if n_}
    if "prep" in kernels:
        # the prep kernel moves the chunk's K and V into the ring (read + write) and, with the
        # fused RoPE, Q into its turned copy; plus the fold's partial states it sums
        E = w.d * w.d + w.d
        kv = w.B * w.H * w.chunk_tokens * w.d * 2
        pbytes = 4 * kv + (2 * kv if a.rope else 0)
        kernels["prep"]["algorithmic_bytes"] = pbytes
        kernels["prep"]["hbm_gbs"] = pbytes / (kernels["prep"]["ms_per_launch"] / 1e3) / 1e9
    if rope_events:
        r_ms = sum(e0.elapsed_time(e1) for e0, e1 in rope_events) / (2 * len(rope_events))
        r_bytes = 2 * od.numel() * od.element_size()        # out of place: one read, one write
        kernels["rope"] = {"ms_per_launch": r_ms, "launches": 2 * len(rope_events),
                           "hbm_gbs": r_bytes / (r_ms / 1e3) / 1e9,
                           "timing": "CUDA events around the Q and K calls of each step, pass 2"}
    config["host_ms_per_step"] = 1e3 * host_s / a.steps

    e2e = None
    if not a.no_e2e:
        # H2D of the step's Q, K, V (pinned) and its mask, the step, D2H of its output; steps
        # run in order on the compute stream (each needs the ring the previous one wrote), while
        # step i+1's inputs and step i-1's output cross PCIe (double-buffered device tensors,
        # one copy stream per direction)
        pinned = [tuple(t.pin_memory() for t in x[:3]) for x in inputs]
        host_masks = [torch.from_numpy(np.ascontiguousarray(x[3])).pin_memory() for x in inputs]
        host_out = [torch.empty_like(pinned[0][0]).pin_memory() for _ in range(2)]
        dbuf = [tuple(torch.empty_like(t) for t in dev_in[0][:3]) for _ in range(2)]
        dmask = [torch.empty_like(dev_in[0][4]) for _ in range(2)]
        dout = [od, torch.empty_like(od)]
        e_steps = max(4, min(a.steps, 20))
        counter = [first]

        def e2e_run(steps):
            h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
            ev = lambda: torch.cuda.Event()
            in_free, in_ready, out_ready, out_free = ([ev(), ev()] for _ in range(4))
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            h2d.wait_event(e0)
            d2h.wait_event(e0)
            for i in range(steps):
                b, j = i % 2, counter[0] % n_dist
                with torch.cuda.stream(h2d):
                    if i >= 2:
                        h2d.wait_event(in_free[b])
                    for dst, src in zip(dbuf[b], pinned[j]):
                        dst.copy_(src, non_blocking=True)
                    dmask[b].copy_(host_masks[j], non_blocking=True)
                    in_ready[b].record(h2d)
                stream.wait_event(in_ready[b])
                if i >= 2:
                    stream.wait_event(out_free[b])
                q, k, v = dbuf[b]
                if a.rope_standalone:
                    q, k = rope_standalone(q, k, counter[0], False)
                if a.graph:
                    h.stream_step_dev(q, k, v, mask=dmask[b], out=dout[b], graph=True)
                else:
                    h.stream_step_dev(q, k, v, mask=dmask[b], out=dout[b])
                counter[0] += 1
                in_free[b].record(stream)
                out_ready[b].record(stream)
                with torch.cuda.stream(d2h):
                    d2h.wait_event(out_ready[b])
                    host_out[b].copy_(dout[b], non_blocking=True)
                    out_free[b].record(d2h)
            for b in range(2):
                stream.wait_event(out_free[b])
            e1.record(stream)
            torch.cuda.synchronize(dev)
            return e0.elapsed_time(e1) / steps
        e2e_run(2 * nwc * 2)                        # warm-up (captures for the double buffers)
        if world > 1:
            torch.distributed.barrier()
        ems = max_over_ranks(e2e_run(e_steps), dev)
        e_value, e_tokens = job_throughput(mean_flops, w.B * w.chunk_tokens, ems, world)
        q0 = inputs[0][0]
        e2e = {"value": e_value, "unit": "TFLOP/s", "ms_per_step": ems, "tokens_per_s": e_tokens,
               "h2d_bytes_per_step": 3 * q0.numel() * q0.element_size() + int(inputs[0][3].nbytes),
               "d2h_bytes_per_step": q0.numel() * q0.element_size(),
               "overlap": "steps in order; the next step's H2D and the previous step's D2H overlap "
                          "the step (double-buffered device tensors, one copy stream per direction)"}
    if world > 1:
        torch.distributed.barrier()
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": a.steps,
                "warmup": warm, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config,
                "tokens_per_s": tokens_per_s, "frac_of_peak": value / world / pk["bf16_tflops"],
                "effective_flops_per_step": mean_flops * world, "roofline": roofline, "kernels": kernels,
                "gpu_launches": launches, "clocks": clk.summary(), "e2e": e2e, "cpu_baseline": None}
        print(json.dumps(line), flush=True)
    h.close()
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


# ----------------------------------------------------------------- main
def main():
    a = parse()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))
    w = wl.WORKLOADS[a.workload]
    if w.mode == "stream":
        return bench_stream(a, w, rank, world, local)
    assert w.mode in ("window", "radial", "lvsa"), "the bench times a bidirectional layer call or streaming steps"
    config = {"workload": w.name, "B": w.B, "H": w.H, "d": w.d, "tokens": w.N,
              "tokens_per_frame": w.tokens_per_frame, "frames": w.n_frames, "mode": w.mode,
              "chunk_frames": w.chunk_frames, "halo_frames": w.halo_frames,
              **({"window_frames": w.window_frames, "anchor_stride": w.anchor_stride, "rotation": w.rotation}
                 if w.mode == "lvsa" else {}),
              "parallelism": f"replicas{world}" if world > 1 else "single",
              "schedule": a.schedule,
              "l2": l2_note(4 * w.B * w.H * w.N * w.d * (4 if w.dtype == "f32" else 2))}

    if a.impl == "reference":
        if rank != 0:
            return 0
        counts = oracle_work_counts(w)
        qkv = wl.gen_qkv(w)
        for _ in range(a.warmup):
            oracle_sample(w, 1, seed=99, qkv=qkv)
        secs, rows = 0.0, 0
        for i in range(a.steps):
            s, r = oracle_sample(w, 1, seed=i, qkv=qkv)
            secs += s
            rows += r
        frac = rows / (w.B * w.H * w.N)
        value = counts["total_flops"] * frac / secs / 1e12
        line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": a.gpus, "steps": a.steps,
                "warmup": a.warmup, "ms_per_step": 1e3 * secs / a.steps, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
                "impl": "reference", "tokens_per_s": rows / secs,
                "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
                                 "sample": f"{a.steps} blocks of 256 query rows (one head each) per run",
                                 **cpu_info()},
                "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0

    from linear_attention_video_hyat_b200 import hyat
    counts = work_counts(w)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    q, k, v = wl.gen_qkv(w, seed=w.seed + rank)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    od = torch.empty_like(qd)
    single = a.schedule == "single"
    flags = {"single": hyat.FLAG_SINGLE_TILE, "one-warp": hyat.FLAG_PAIR_ONE_WARP}.get(a.schedule, 0)
    h = hyat.Hyat(hyat.config_from_workload(w, flags=flags), workload_mask(w), device=dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(max(a.warmup, 3)):
        h.forward(qd, kd, vd, out=od)
    h.sync()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)

    # Pass 1 (the headline): K steps, no per-launch events, so the kernels of a step overlap
    # their launches (programmatic dependent launch) exactly as in production.
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        t0.record(stream)
        for _ in range(a.steps):
            h.forward(qd, kd, vd, out=od)
        t1.record(stream)
        torch.cuda.synchronize(dev)
    h.sync()
    ms = t0.elapsed_time(t1) / a.steps
    # Pass 2: K more steps with CUDA events around every launch (library-side), for the
    # per-kernel durations of the roofline. It starts after an idle second, so that it runs at
    # the clocks of pass 1 instead of those the power limit sets after pass 1's load (both
    # passes' clocks are in the line).
    time.sleep(KERNEL_PASS_IDLE_S)
    h.set_profiling(True)
    h.kernel_times()
    with ClockSampler(local) as clk2:
        for _ in range(a.steps):
            h.forward(qd, kd, vd, out=od)
        torch.cuda.synchronize(dev)
    kt = h.kernel_times()
    h.set_profiling(False)
    ms = max_over_ranks(ms, dev)
    launches = sum(n for _, n in kt.values())   # per-step launches x K (pass 2 mirrors pass 1)
    if a.schedule != "one-warp":
        launches += kt["attention"][1]          # each attention call is two kernels (+ redo pass)

    value, tokens_per_s = job_throughput(counts["total_flops"], w.B * w.N, ms, world)
    pk, pk_src = peaks()
    attn_ms = kt["attention"][0] / max(kt["attention"][1], 1)
    achieved = counts["attn_kernel_flops"] / (attn_ms / 1e3) / 1e12
    traffic = None
    tpath = os.path.join(ROOT, "profiles", "attn_traffic.json")
    if os.path.exists(tpath):
        t = json.load(open(tpath))
        sha = kernel_source_digest()
        if t.get("source_sha256") == sha and t.get("workload") == w.name and t.get("schedule", "pair") == a.schedule:
            traffic = t.get("dram_bytes_per_launch")
    roofline = {"bound": "tensor", "kernel": "attention", "achieved": achieved,
                "timing": "per-launch CUDA events over a second pass of the same K steps",
                "clocks_kernel_pass": clk2.summary(),
                "peak": pk["bf16_tflops"], "unit": "TFLOP/s", "frac": achieved / pk["bf16_tflops"],
                "peak_kind": f"{pk_src} bf16 burst", "peak_sustained": pk["bf16_tflops_sustained"],
                "frac_sustained": achieved / pk["bf16_tflops_sustained"], "traffic": traffic,
                "launch_ms": attn_ms, "algorithmic_flops_per_launch": counts["attn_kernel_flops"]}
    kernels = {k_: {"ms_per_launch": t_ / max(n_, 1), "launches": n_} for k_, (t_, n_) in kt.items() if n_}
    state_ms = kernels.get("state", {}).get("ms_per_launch")
    if state_ms:
        kernels["state"]["hbm_gbs"] = counts["state_kernel_bytes"] / (state_ms / 1e3) / 1e9

    e2e = None
    if not a.no_e2e:
        host_in = (q.pin_memory(), k.pin_memory(), v.pin_memory())
        host_out = [torch.empty_like(host_in[0]).pin_memory() for _ in range(2)]
        dev_in = [(qd, kd, vd), tuple(torch.empty_like(t) for t in (qd, kd, vd))]
        dev_out = [od, torch.empty_like(od)]
        call = lambda xin, xout, st: h.forward(*xin, out=xout, stream=st)
        e_steps = max(4, min(a.steps, 20))
        e2e_pipelined(call, host_in, host_out, dev_in, dev_out, stream, 2, dev)   # warm-up
        if world > 1:
            torch.distributed.barrier()
        ems = max_over_ranks(e2e_pipelined(call, host_in, host_out, dev_in, dev_out, stream, e_steps, dev), dev)
        e_value, e_tokens = job_throughput(counts["total_flops"], w.B * w.N, ems, world)
        e2e = {"value": e_value, "unit": "TFLOP/s", "ms_per_step": ems, "tokens_per_s": e_tokens,
               "h2d_bytes_per_step": 3 * q.numel() * q.element_size(),
               "d2h_bytes_per_step": q.numel() * q.element_size(),
               "overlap": "each step's H2D, layer call and D2H; consecutive steps overlap "
                          "(double-buffered device tensors, one copy stream per direction)"}

    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        tf, rps, secs, rows = cpu_rate(w, counts, n_blocks=24, qkv=(q, k, v))
        cpu = {"value": tf, "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
               "tokens_per_s": rps, "seconds": secs, **cpu_info(),
               "sample": f"{rows} query rows (24 blocks of 256 rows, one head each) of the same layer; "
                         f"FLOPs scaled by the sampled fraction of rows"}

    if world > 1:
        torch.distributed.barrier()
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": a.steps,
                "warmup": a.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config,
                "tokens_per_s": tokens_per_s, "frac_of_peak": value / world / pk["bf16_tflops"],
                "effective_flops_per_step": counts["total_flops"] * world,
                "roofline": roofline, "kernels": kernels, "gpu_launches": launches,
                "clocks": clk.summary(), "e2e": e2e, "cpu_baseline": cpu}
        print(json.dumps(line), flush=True)
    h.close()
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
