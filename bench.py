"""Benchmark of the Forcing-KV chunk step (fkv_step) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 480p]
                    [--impl ours|reference]

Prints ONE JSON line.  Metric: chunk-steps per second per layer (a chunk step
of one layer = score + select + compact + attend over all heads of that
layer).  ``value`` is whole-job throughput with the inputs resident in HBM;
``e2e`` the same metric through the same C-ABI call with the inputs copied
from pinned host memory and the output read back inside the timed region.

Timing: W untimed warm-up steps, then K steps each bracketed by CUDA events
on the launching stream; between timed steps the L2 is flushed outside the
events by writing a 256 MiB buffer and reading it back (the read evicts the
written lines, so the timed kernels start on a cold L2 with no dirty lines of
the flush left to write back).  The per-kernel breakdown (roofline) comes
from a second timed pass over the four entry points, each a C-ABI call whose
arguments were checked and converted once (``fkv.marshal``), with events
between them (so that a short kernel's time is not inflated by the Python
binding's host work in front of it).  N > 1: one process per GPU (torchrun), each rank runs
its own independent chunk step (replicas: the step has no exchange), and the
time is the max over ranks.

At N = 1 the workloads named by ``--extra`` (default: 1080P, the 30-layer
480P batch and the 14B token variant) are timed the same way after the
headline one and reported under ``workloads``.

``--impl reference`` times the fp64 CPU oracle (the only reference of this
method) on the host cores: each step a bounded sample of whole heads of the
same workload, ``ms_per_step`` its measured wall time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import fkv_workloads as wl  # noqa: E402

METRIC = "fkv_step chunk-steps/s per layer"
UNIT = "chunk-steps/s per layer"
SPEC_BF16_TFLOPS = 2250.0
# MUFU exp2 rate derived from unit counts and clocks: 16 per SM per cycle,
# 148 SMs, 1965 MHz maximum SM clock.
SFU_EXP2_PER_S = 16 * 148 * 1965e6
SPEC_HBM_GBS = 7700.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------------------- work model

def algorithmic(w, kept_cnt, head_role):
    """Algorithmic FLOPs / bytes of each kernel for one step (all layers).

    attention: 4 * Lq * keys * D per head (QK^T and PV), keys = kept rows + Lq;
    scoring (frame): 2 * n_s * N * D per dynamic head (QK^T), K read once;
    scoring (token): K candidates read once (GEMV) + q_score read once;
    compaction: kept rows of K and V read once and written once."""
    seg_len = w.T if (w.granularity == "frame" and not w.static_token_mask) else 1
    rows = kept_cnt.to(torch.int64) * seg_len
    keys = rows + w.Lq
    elem = 2 if w.dtype == "bf16" else 4
    attn_flops = float((4 * w.Lq * keys * w.D).sum())
    gather_bytes = float((rows * w.D * elem * 4).sum())
    if w.granularity == "frame":
        n_dyn = int(head_role.sum())
        n_s = -(-w.Lq // w.score_stride)
        score_flops = 2.0 * n_s * w.N * w.D * n_dyn
        score_bytes = float(n_dyn * (w.N + n_s) * w.D * elem)
    else:
        n_c = w.N - w.sink_tokens - w.recent_tokens
        score_flops = 2.0 * n_c * w.D * w.L * w.H
        score_bytes = float(w.L * w.H * (n_c + w.n_score_q) * w.D * elem)
    # exponentials the scoring must evaluate: every logit of every scoring row
    # (frame mode; the chunk's own keys too when they join the normaliser)
    if w.granularity == "frame":
        keys_scored = w.N + (w.Lq if w.score_with_chunk else 0)
        score_exps = float(n_dyn * n_s * keys_scored)
    else:
        score_exps = 0.0
    return {"attn_flops": attn_flops, "gather_bytes": gather_bytes,
            "score_flops": score_flops, "score_bytes": score_bytes, "score_exps": score_exps}


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during a region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": ["unavailable"], "samples": 0}
        busy = [s for s in sm if mx is None or s > 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------- our arm

def kernel_source_hash(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "kv_cache_compression_fkv_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def committed_traffic(kernel_key, workload, src_hash):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(f"{kernel_key}/{workload}")
    if not e or e.get("source_hash") != src_hash:
        return None
    return e.get("dram_bytes_per_launch")


def replica_workload(w, rank, world):
    """Weak scaling with replicas: rank r runs the same workload shape on its
    own independent inputs (seeds offset by rank); there is no exchange."""
    if world <= 1:
        return w
    return wl.scaled(w, seed=w.seed + 7919 * rank, layer_seeds=None if w.layer_seeds is None else
                     tuple(s + 7919 * rank for s in w.layer_seeds))


def max_over_ranks(value, dist=None, device=None):
    """Max of a per-rank float over the process group (the job's time is its
    slowest rank's)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(units_per_rank, world, max_ms):
    """Whole-job throughput: units processed by all ranks / slowest rank's time."""
    return units_per_rank * world / (max_ms / 1e3)


class L2Flush:
    """Empties the L2 between timed steps: a 256 MiB write (twice the L2),
    then a read of the same buffer, on the current stream, outside the
    events.  After the read the L2 holds clean lines of the flush buffer, so a
    timed kernel's misses do not also write back the flush's dirty lines."""

    def __init__(self, dev):
        self.buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        self.sink = torch.empty(1, dtype=torch.int64, device=dev)

    def __call__(self, i):
        self.buf.fill_(i & 0xFF)
        self.sink.copy_(self.buf.view(torch.int64).sum().view(1))


def time_calls(calls, flush, steps, stream):
    """Mean device time of each call of `calls` (pairs (c_function, c_args)
    from ``fkv.marshal``, issued in order), with the L2 flushed before each
    round.  The calls carry no Python-side work, so the GPU never waits on the
    host in front of a short kernel."""
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(calls) + 1)]
          for _ in range(steps)]
    for i in range(steps):
        flush(i)
        ev[i][0].record(stream)
        for k, (fn, args) in enumerate(calls):
            st = fn(*args)
            if st != 0:
                raise RuntimeError(f"{fn.__name__}: status {st}")
            ev[i][k + 1].record(stream)
    torch.cuda.synchronize()
    return [statistics.mean(ev[i][k].elapsed_time(ev[i][k + 1]) for i in range(steps))
            for k in range(len(calls))]


def hw_rates(dev):
    """The library's hardware-rate diagnostics (SM cycles, CTA 0 of one CTA
    per SM): tcgen05.mma of the attention's shapes issued back to back by one
    thread (Q.K^T and P.V through the attention's own grouped issue), and ex2
    per warp with 1, 2 and 4 warps per sub-partition."""
    from kv_cache_compression_fkv_b200 import _lib
    lib = _lib.load()
    cyc = torch.zeros(4, dtype=torch.int64, device=dev)
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    s = torch.cuda.current_stream(dev).cuda_stream
    n = 256
    mma = {}
    for name, shape, busy in (("qk_ss_m128n128k16", 6, 0), ("pv_ts_m128n128k16", 7, 0),
                              ("ss_m128n256k16", 2, 0), ("ss_m128n64k16", 3, 0),
                              ("qk_with_two_busy_warps", 6, 1),
                              ("e4m3_qk_ss_m128n128k32", 8, 0), ("e4m3_pv_ts_m128n128k32", 9, 0)):
        for _ in range(2):
            if lib.fkv_diag_mma_rate(shape, n, busy, cyc.data_ptr(), ws.data_ptr(), s) != 0:
                return None
        torch.cuda.synchronize(dev)
        mma[name] = round(int(cyc[1]) / n, 1)
    ex2 = {}
    for warps in (1, 2, 4):
        for _ in range(2):
            if lib.fkv_diag_ex2_rate(4096, warps, cyc.data_ptr(), s) != 0:
                return None
        torch.cuda.synchronize(dev)
        ex2[f"{warps}_warps_per_subpartition"] = round(int(cyc[0]) / 4096, 2)
    return {"mma_cycles_per_instruction": mma, "ex2_cycles_per_warp_instruction": ex2}


def entry_point_calls(fkv, p, x, outs):
    """The four entry points of the step as separate C-ABI calls, in step order."""
    return [
        fkv.marshal(fkv.score_segments, p, x["q_cur"], x.get("q_score"), x["k_hist"],
                    x.get("head_role"), outs["seg_score"], outs["ws"], k_cur=x["k_cur"]),
        fkv.marshal(fkv.select_topk, p, outs["seg_score"], x.get("head_role"),
                    x.get("static_mask"), x["k_per_head"], outs["kept_idx"], outs["kept_cnt"],
                    outs["ws"]),
        fkv.marshal(fkv.compact_gather, p, x["k_hist"], x["v_hist"], outs["kept_idx"],
                    outs["kept_cnt"], outs["k_comp"], outs["v_comp"], outs["ws"]),
        fkv.marshal(fkv.attend_compressed, p, x["q_cur"], x["k_cur"], x["v_cur"],
                    outs["k_comp"], outs["v_comp"], outs["kept_cnt"], outs["out"], outs["ws"]),
    ]


def kept_per_head(w):
    """Segments every head keeps in the workload's step: the static mask size
    (= the dynamic budget k) in frame mode, S + C + R tokens in token mode."""
    if w.granularity == "token":
        return int(w.sink_tokens + w.keep_tokens + w.recent_tokens)
    return int(w.k_dynamic)


def bench_config(base, w, world=1, split="replicas", extra=None):
    """The ``config`` object of the JSON line; both arms print the same one."""
    cfg = {"workload": base.name, "L": base.L, "H": base.H, "D": w.D, "T": w.T, "F": w.F,
           "Fc": w.Fc, "granularity": w.granularity, "kept_per_head": kept_per_head(base),
           "l2": "flushed between timed steps (256 MiB written, then read, outside the events)",
           "parallelism": (f"heads split over {world} GPUs" if split == "heads" and world > 1
                           else f"replicas x{world}" if world > 1 else "single GPU")}
    cfg.update(extra or {})
    return cfg


def cpu_model():
    """Host CPU model name (from /proc/cpuinfo), or None."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def measure_workload(fkv, w, x_cpu, dev, steps, warmup, flush):
    """One more workload on this GPU, timed like the headline one: the fused
    fkv_step (CUDA events around each step, L2 flushed between steps), then the
    entry points one by one for the per-kernel split and the roofline figures."""
    p = fkv.params_for(w)
    stream = torch.cuda.current_stream(dev)
    x = {k: v.to(dev) for k, v in x_cpu.items()}
    outs = fkv.allocate(p, dev)
    io = fkv.make_step_io(p, x, outs)
    for _ in range(warmup):
        fkv.step(p, x, outs, io=io)
    torch.cuda.synchronize(dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for i in range(steps):
        flush(i)
        evs[i][0].record(stream)
        fkv.step(p, x, outs, io=io)
        evs[i][1].record(stream)
    torch.cuda.synchronize(dev)
    step_ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
    part = dict(zip(["score", "select", "gather", "attend"],
                    time_calls(entry_point_calls(fkv, p, x, outs), flush, steps, stream)))
    st, det = fkv.read_status(outs["ws"])
    if st != 0:
        raise RuntimeError(f"device status {st} on head {det} ({w.name})")
    alg = algorithmic(w, outs["kept_cnt"].cpu(), x_cpu["head_role"] if w.granularity == "frame"
                      else torch.ones(w.L, w.H))
    peaks, _ = load_peaks()
    attn_tfs = alg["attn_flops"] / (part["attend"] * 1e-3) / 1e12
    gather_gbs = alg["gather_bytes"] / (part["gather"] * 1e-3) / 1e9
    score = {"ms": round(part["score"], 4)}
    if alg["score_exps"]:
        score["frac_sfu"] = round(alg["score_exps"] / (part["score"] * 1e-3) / SFU_EXP2_PER_S, 4)
    else:
        score["frac_hbm"] = round(alg["score_bytes"] / (part["score"] * 1e-3) / 1e9
                                  / peaks["hbm_gbs"], 4)
    res = {"value": round(aggregate_throughput(w.L * steps, 1, step_ms * steps), 3), "unit": UNIT,
           "ms_per_step": round(step_ms, 4), "steps": steps, "warmup": warmup,
           "config": bench_config(w, w),
           "kernels": {"score_segments": score, "select_topk": {"ms": round(part["select"], 4)},
                       "compact_gather": {"ms": round(part["gather"], 4),
                                          "GB/s": round(gather_gbs, 1),
                                          "frac_hbm": round(gather_gbs / peaks["hbm_gbs"], 4)},
                       "attend_compressed": {"ms": round(part["attend"], 4),
                                             "TFLOP/s": round(attn_tfs, 2),
                                             "frac_tensor": round(attn_tfs / peaks["bf16_tflops"], 4),
                                             # a launch of several ms runs under the power
                                             # cap: the sustained GEMM rate is its peak
                                             "frac_tensor_sustained": round(
                                                 attn_tfs / peaks["bf16_tflops_sustained"], 4)}}}
    del x, outs, io
    torch.cuda.empty_cache()
    return res


def run_ours(args, rank, world, local_rank):
    import kv_cache_compression_fkv_b200 as fkv
    dist = None
    torch.cuda.set_device(local_rank)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local_rank)
    from kv_cache_compression_fkv_b200 import shard
    base = wl.get(args.workload)
    if args.split == "heads":
        # strong scaling: rank r runs its contiguous range of the L*H heads of one step
        h0, h1 = shard.head_range(base.L * base.H, world, rank)
        x_cpu = shard.shard_inputs(wl.generate(base), h0, h1)
        w = shard.local_workload(base, h0, h1)
    else:
        w = replica_workload(base, rank, world)
        x_cpu = wl.generate(w)
    p = fkv.params_for(w)
    stream = torch.cuda.current_stream(dev)
    x = {k: v.to(dev) for k, v in x_cpu.items()}
    outs = fkv.allocate(p, dev)
    io = fkv.make_step_io(p, x, outs)
    flush = L2Flush(dev)

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)

    # ---- timed: fused fkv_step, inputs resident.  The clock sampler starts
    # before the warm-up, so the GPU is not left idle between warm-up and timing.
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    with ClockSampler(local_rank) as clk:
        for _ in range(args.warmup):
            fkv.step(p, x, outs, io=io)
        torch.cuda.synchronize(dev)
        st, det = fkv.read_status(outs["ws"])
        if st != 0:
            raise RuntimeError(f"device status {st} on head {det}")
        barrier()
        for i in range(args.steps):
            flush(i)
            evs[i][0].record(stream)
            fkv.step(p, x, outs, io=io)
            evs[i][1].record(stream)
        torch.cuda.synchronize(dev)
    barrier()
    step_ms = [a.elapsed_time(b) for a, b in evs]
    total_ms = max_over_ranks(sum(step_ms), dist, dev)
    clocks = clk.summary()

    # ---- per-kernel breakdown: the same kernels through the four entry points
    rope = w.granularity == "frame" and not w.static_token_mask
    # temporal RoPE band of the re-positioning compaction: 22 pairs (44 dims)
    omega = (10000.0 ** (-torch.arange(22, dtype=torch.float32) / 22)).to(dev)
    calls = entry_point_calls(fkv, p, x, outs)
    if rope:
        calls.append(fkv.marshal(fkv.compact_gather_rope, p, x["k_hist"], x["v_hist"],
                                 outs["kept_idx"], outs["kept_cnt"], omega, outs["k_comp"],
                                 outs["v_comp"], outs["ws"]))
    barrier()
    times = time_calls(calls, flush, args.steps, stream)
    barrier()
    part = dict(zip(["score", "select", "gather", "attend", "gather_rope"], times + [0.0]))

    # comparison selectors (uniform eviction / random drop), same budgets
    hc = [fkv.marshal(fkv.select_heuristic, p, "uniform", 1, x["k_per_head"], outs["kept_idx"],
                      outs["kept_cnt"], outs["ws"]),
          fkv.marshal(fkv.select_heuristic, p, "random", 1, x["k_per_head"], outs["kept_idx"],
                      outs["kept_cnt"], outs["ws"], seg_score=outs["seg_score"])]
    heur = dict(zip(["uniform", "random"], time_calls(hc, flush, args.steps, stream)))

    # ---- FP8 (e4m3) compressed cache: the same scoring and selection, then the
    # e4m3 compaction, the chunk's quantisation and the kind::f8f6f4 attention
    fp8 = None
    if (w.granularity == "frame" and not w.static_token_mask and w.dtype == "bf16" and w.D == 128
            and w.T >= 128):
        c8 = fkv.allocate_fp8(p, dev)
        out8 = torch.empty_like(outs["out"])
        calls8 = entry_point_calls(fkv, p, x, outs)[:2] + [
            fkv.marshal(fkv.compact_gather_fp8, p, x["k_hist"], x["v_hist"], outs["kept_idx"],
                        outs["kept_cnt"], c8, outs["ws"]),
            fkv.marshal(fkv.quantize_chunk_fp8, p, x["q_cur"], x["k_cur"], x["v_cur"], c8,
                        outs["ws"]),
            fkv.marshal(fkv.attend_compressed_fp8, p, c8, outs["kept_cnt"], out8, outs["ws"]),
        ]
        time_calls(calls8, flush, args.warmup, stream)  # warm-up
        fp8 = dict(zip(["score", "select", "gather", "quant", "attend"],
                       time_calls(calls8, flush, args.steps, stream)))
        st, det = fkv.read_status(outs["ws"])
        if st != 0:
            raise RuntimeError(f"device status {st} on head {det} (fp8 path)")
        fp8["step"] = sum(fp8[n] for n in ("score", "select", "gather", "quant", "attend"))
        # the same step through the one fused call (fkv_step_fp8)
        sev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        for i in range(args.steps):
            flush(i)
            sev[i][0].record(stream)
            fkv.step_fp8(p, x, outs, c8, io=io)
            sev[i][1].record(stream)
        torch.cuda.synchronize(dev)
        fp8["fused"] = statistics.mean(a_.elapsed_time(b_) for a_, b_ in sev)

    # ---- e2e: host buffers in, result out, through the same call.  Every step
    # copies its inputs from pinned host memory (H2D stream), runs fkv_step
    # (compute stream) and reads its result back (D2H stream); two buffer sets
    # let the copies of one step overlap the compute of the other.
    pinned = {k: v.pin_memory() for k, v in x_cpu.items()}
    res_keys = ("out", "kept_idx", "kept_cnt")
    out_host = [{k: torch.empty(outs[k].shape, dtype=outs[k].dtype, pin_memory=True)
                 for k in res_keys} for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in pinned.values())
    d2h = sum(t.numel() * t.element_size() for t in out_host[0].values())
    xs = [x, {k: torch.empty_like(v) for k, v in x.items()}]
    os_ = [outs, fkv.allocate(p, dev)]
    ios = [fkv.make_step_io(p, xs[b], os_[b]) for b in range(2)]
    s_h2d, s_d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    comp_done = [ev() for _ in range(args.steps)]
    h2d_done = [ev() for _ in range(args.steps)]
    d2h_done = [ev() for _ in range(args.steps)]
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    e_start.record(stream)
    s_h2d.wait_stream(stream)
    s_d2h.wait_stream(stream)
    for i in range(args.steps):
        b = i & 1
        with torch.cuda.stream(s_h2d):
            if i >= 2:  # buffer b was last read by step i-2's compute and D2H
                s_h2d.wait_event(comp_done[i - 2])
            for k, v in pinned.items():
                xs[b][k].copy_(v, non_blocking=True)
            h2d_done[i].record(s_h2d)
        stream.wait_event(h2d_done[i])
        if i >= 2:
            stream.wait_event(d2h_done[i - 2])
        fkv.step(p, xs[b], os_[b], io=ios[b])
        comp_done[i].record(stream)
        with torch.cuda.stream(s_d2h):
            s_d2h.wait_event(comp_done[i])
            for k in res_keys:
                out_host[b][k].copy_(os_[b][k], non_blocking=True)
            d2h_done[i].record(s_d2h)
    stream.wait_stream(s_h2d)
    stream.wait_stream(s_d2h)
    e_end.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = max_over_ranks(e_start.elapsed_time(e_end), dist, dev)
    for b in range(2):
        st, det = fkv.read_status(os_[b]["ws"])
        if st != 0:
            raise RuntimeError(f"device status {st} on head {det}")
    st, det = fkv.read_status(outs["ws"])
    if st != 0:
        raise RuntimeError(f"device status {st} on head {det}")

    # ---- chunk lifecycle: kDenoise denoising steps of one chunk, then the cache
    # advance (next history = the most recent kept frames + the chunk).  Two
    # policies: compress at every denoising step, or once per chunk and reuse
    # the selection (attention alone for the later steps).
    lifecycle = None
    if w.granularity == "frame" and not w.static_token_mask and w.L == 1:
        n_den = 4
        kept = int(outs["kept_cnt"].min())
        window = min(kept, w.F - w.Fc) + w.Fc
        k_next = torch.empty((w.L, w.H, window * w.T, w.D), dtype=x["k_cur"].dtype, device=dev)
        v_next = torch.empty_like(k_next)

        def advance():
            fkv.cache_advance(p, outs["k_comp"], outs["v_comp"], outs["kept_cnt"], x["k_cur"],
                              x["v_cur"], window, k_next, v_next, outs["ws"])

        def attend_only():
            fkv.attend_compressed(p, x["q_cur"], x["k_cur"], x["v_cur"], outs["k_comp"],
                                  outs["v_comp"], outs["kept_cnt"], outs["out"], outs["ws"])

        def timed(body):
            evs_ = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                    for _ in range(args.steps)]
            for i in range(args.steps):
                flush(i)
                evs_[i][0].record(stream)
                body()
                evs_[i][1].record(stream)
            torch.cuda.synchronize(dev)
            return statistics.mean(a_.elapsed_time(b_) for a_, b_ in evs_)

        every = timed(lambda: ([fkv.step(p, x, outs, io=io) for _ in range(n_den)], advance()))
        reuse = timed(lambda: (fkv.step(p, x, outs, io=io),
                               [attend_only() for _ in range(n_den - 1)], advance()))
        lifecycle = {"denoising_steps": n_den, "window_frames": window,
                     "ms_per_chunk_compress_every_step": round(every, 4),
                     "ms_per_chunk_compress_once": round(reuse, 4),
                     "chunks_per_s_compress_once": round(1e3 / reuse, 2)}
        st, det = fkv.read_status(outs["ws"])
        if st != 0:
            raise RuntimeError(f"device status {st} on head {det}")

    # heads split: the all-gather of O that gives every rank the whole output
    gather_ms = None
    if args.split == "heads" and dist is not None:
        gev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        for i in range(args.warmup + args.steps):
            if i >= args.warmup:
                gev[i - args.warmup][0].record(stream)
            shard.gather_heads(outs["out"], base.L * base.H, world)
            if i >= args.warmup:
                gev[i - args.warmup][1].record(stream)
        torch.cuda.synchronize(dev)
        gather_ms = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in gev), dist, dev)

    alg = algorithmic(w, outs["kept_cnt"].cpu(), x_cpu["head_role"] if w.granularity == "frame"
                      else torch.ones(w.L, w.H))
    peaks, peak_kind = load_peaks()
    if args.split == "heads":  # all ranks together run one whole step per step
        value = aggregate_throughput(base.L * args.steps, 1, total_ms)
        e2e_value = aggregate_throughput(base.L * args.steps, 1, e2e_ms)
    else:
        value = aggregate_throughput(w.L * args.steps, world, total_ms)
        e2e_value = aggregate_throughput(w.L * args.steps, world, e2e_ms)
    attn_tfs = alg["attn_flops"] / (part["attend"] * 1e-3) / 1e12
    gather_gbs = alg["gather_bytes"] / (part["gather"] * 1e-3) / 1e9
    score_tfs = alg["score_flops"] / (part["score"] * 1e-3) / 1e12
    score_gbs = alg["score_bytes"] / (part["score"] * 1e-3) / 1e9
    src_hash = kernel_source_hash(_attend_sources())
    traffic = committed_traffic("attend", w.name, src_hash)
    roof = {"bound": "tensor", "kernel": "attend_compressed", "achieved": round(attn_tfs, 2),
            "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
            "frac": round(attn_tfs / peaks["bf16_tflops"], 4),
            "peak_kind": f"{peak_kind} burst bf16 (cuBLAS 8192^3)",
            "traffic": traffic,
            "algorithmic_per_launch": alg["attn_flops"], "ms_per_launch": round(part["attend"], 4)}
    kernels = {
        "score_segments": {"ms": round(part["score"], 4), "TFLOP/s": round(score_tfs, 2),
                           "GB/s": round(score_gbs, 1),
                           **({"bound": "sfu", "exp2_per_s": round(alg["score_exps"] / (part["score"] * 1e-3), 1),
                               "peak_exp2_per_s": SFU_EXP2_PER_S,
                               "frac_sfu": round(alg["score_exps"] / (part["score"] * 1e-3) / SFU_EXP2_PER_S, 4)}
                              if alg["score_exps"] else {}),
                           "frac_tensor": round(score_tfs / peaks["bf16_tflops"], 4),
                           "frac_hbm": round(score_gbs / peaks["hbm_gbs"], 4)},
        "select_topk": {"ms": round(part["select"], 4)},
        "select_heuristic": {"uniform_ms": round(heur["uniform"], 4),
                             "random_ms": round(heur["random"], 4)},
        "compact_gather_rope": ({"ms": round(part["gather_rope"], 4),
                                 "GB/s": round(alg["gather_bytes"] / (part["gather_rope"] * 1e-3) / 1e9, 1),
                                 "frac_hbm": round(alg["gather_bytes"] / (part["gather_rope"] * 1e-3) / 1e9
                                                   / peaks["hbm_gbs"], 4)} if rope else None),
        "compact_gather": {"ms": round(part["gather"], 4), "GB/s": round(gather_gbs, 1),
                           "frac_hbm": round(gather_gbs / peaks["hbm_gbs"], 4),
                           "frac_hbm_spec": round(gather_gbs / SPEC_HBM_GBS, 4)},
        "attend_compressed": {"ms": round(part["attend"], 4), "TFLOP/s": round(attn_tfs, 2),
                              "frac_tensor": round(attn_tfs / peaks["bf16_tflops"], 4),
                              "frac_tensor_spec": round(attn_tfs / SPEC_BF16_TFLOPS, 4)},
        "score_plus_attend_frac_tensor": round(
            (alg["attn_flops"] + alg["score_flops"]) / ((part["attend"] + part["score"]) * 1e-3)
            / 1e12 / peaks["bf16_tflops"], 4),
    }
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 4),
        "higher_is_better": True, "scaling": "strong" if args.split == "heads" else "weak",
        "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "fp32", "data": "synthetic (seeded, Wan-shaped)",
        "config": bench_config(base, w, world, args.split,
                               {"heads_per_rank": f"{w.H} (rank {rank})",
                                "gather_out_ms": round(gather_ms, 4)} if gather_ms is not None
                               else None),
        "impl": "ours",
        "e2e": {"value": round(e2e_value, 3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": fkv.step_launches(p) * args.steps,
        "roofline": roof,
        "kernels": kernels,
        "clocks": clocks,
    }
    if lifecycle is not None:
        line["lifecycle"] = lifecycle
    if fp8 is not None:
        fp8_peak = 2.0 * peaks["bf16_tflops"]  # dense e4m3 = 2 x bf16 (nominal ratio)
        kept_rows = float((outs["kept_cnt"].cpu().to(torch.int64) * w.T).sum())
        g8_bytes = kept_rows * w.D * 3 * 2          # K and V: 2 B read, 1 B written per element
        q8_bytes = float(w.L * w.H * w.Lq * w.D * 3 * 3)  # Q, K, V of the chunk
        a8_tfs = alg["attn_flops"] / (fp8["attend"] * 1e-3) / 1e12
        line["fp8"] = {
            "ms_per_step": round(fp8["fused"], 4),
            "ms_per_step_separate_calls": round(fp8["step"], 4),
            "value_per_gpu": round(aggregate_throughput(w.L, 1, fp8["fused"]), 3), "unit": UNIT,
            "kernels": {
                "compact_gather_fp8": {"ms": round(fp8["gather"], 4),
                                       "GB/s": round(g8_bytes / (fp8["gather"] * 1e-3) / 1e9, 1),
                                       "frac_hbm": round(g8_bytes / (fp8["gather"] * 1e-3) / 1e9
                                                         / peaks["hbm_gbs"], 4)},
                "quantize_chunk_fp8": {"ms": round(fp8["quant"], 4),
                                       "GB/s": round(q8_bytes / (fp8["quant"] * 1e-3) / 1e9, 1),
                                       "frac_hbm": round(q8_bytes / (fp8["quant"] * 1e-3) / 1e9
                                                         / peaks["hbm_gbs"], 4)},
                "attend_compressed_fp8": {"ms": round(fp8["attend"], 4), "TFLOP/s": round(a8_tfs, 2),
                                          "peak": round(fp8_peak, 1),
                                          "peak_kind": f"2 x {peak_kind} burst bf16",
                                          "frac_tensor": round(a8_tfs / fp8_peak, 4),
                                          "traffic": committed_traffic(
                                              "attend_fp8", w.name,
                                              kernel_source_hash(_attend_fp8_sources()))},
            },
        }
    extra = [n for n in args.extra.split(",") if n and n != base.name] if world == 1 else []
    if extra:
        # the metric's other resolution and the other configurations, timed on the
        # same GPU after the headline workload (inputs generated outside the timing)
        line["workloads"] = {}
        with ClockSampler(local_rank) as clk_x:
            for name in extra:
                we = wl.get(name)
                line["workloads"][name] = measure_workload(
                    fkv, we, wl.generate(we), dev, min(args.steps, 10), args.warmup, flush)
        line["workloads_clocks"] = clk_x.summary()
    if world == 1:
        line["hw_rates"] = hw_rates(dev)
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(w, x_cpu, budget_s=args.cpu_budget)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return line


def _attend_sources():
    """Source files of the attention kernel (the traffic record is void once they change)."""
    return ["attend_sm100.cu", "attend_common.cuh", "sm100_common.cuh"]


def _attend_fp8_sources():
    """Source files of the e4m3 attention kernel."""
    return ["attend_fp8_sm100.cu", "attend_common.cuh", "sm100_common.cuh", "f8_common.cuh"]


# --------------------------------------------------------------------------- CPU oracle

def _oracle_head(w, x, l, h):
    """One (layer, head) of the step through the fp64 oracle, as it stands:
    scoring and selection, compaction, attention over every query row."""
    from oracle import fkv_oracle as orc
    f64 = lambda k: wl.as_float64(x[k][l, h])  # noqa: E731
    ks, _ = orc.head_keep(
        granularity=w.granularity,
        dynamic=w.granularity == "token" or bool(x["head_role"][l, h]),
        mask_row=x["static_mask"][l, h].numpy(), k=int(x["k_per_head"][l, h]),
        q_cur=f64("q_cur"), k_hist=f64("k_hist"), T=w.T, scale=w.scale,
        score_stride=w.score_stride, q_score=f64("q_score") if "q_score" in x else None,
        sink=w.sink_tokens, recent=w.recent_tokens,
        k_chunk=f64("k_cur") if w.score_with_chunk else None,
        token_static_mask=w.static_token_mask)
    seg_len = w.T if (w.granularity == "frame" and not w.static_token_mask) else 1
    keys = np.concatenate([orc.compact(f64("k_hist"), ks, seg_len), f64("k_cur")])
    vals = np.concatenate([orc.compact(f64("v_hist"), ks, seg_len), f64("v_cur")])
    orc.attention(f64("q_cur"), keys, vals, w.scale)


def _head_order(w, x):
    """(layer, head) pairs alternating dynamic and static heads, so that any
    prefix of the order has the layer's mix of the two."""
    order = [(l, h) for l in range(w.L) for h in range(w.H)]
    if w.granularity == "frame":
        role = x["head_role"]
        dyn = [lh for lh in order if role[lh]]
        sta = [lh for lh in order if not role[lh]]
        order = [v for pair in zip(dyn, sta) for v in pair] + dyn[len(sta):] + sta[len(dyn):]
    return order


def _cores():
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()


def cpu_baseline(w, x_cpu, budget_s=15.0):
    """Times the fp64 oracle, as it stands, on a bounded sample: whole heads
    (scoring, selection, compaction, attention over every query row) taken in
    order until the budget is spent; value scaled to layer-steps per second."""
    heads_done, t0 = 0, time.perf_counter()
    for (l, h) in _head_order(w, x_cpu):
        _oracle_head(w, x_cpu, l, h)
        heads_done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    layers = heads_done / w.H
    return {"value": round(layers / dt, 6), "unit": UNIT, "cores": _cores(),
            "cpu_model": cpu_model(), "kind": "oracle",
            "sample": f"{heads_done} of {w.L * w.H} heads of workload {w.name} (full oracle step "
                      f"per head, every query row), {dt:.1f} s, numpy fp64",
            "seconds": round(dt, 2)}


def run_reference(args):
    """The reference arm: the fp64 oracle, as it stands, on the host cores.
    One "step" is a bounded sample of the workload's chunk step: a fixed number
    of whole heads (one dynamic and one static head by default, every query
    row), taken in turn from the layer's alternating order so that successive
    steps walk through all of its heads.  ``ms_per_step`` is the measured wall
    time of such a step; ``value`` = the layers these steps covered (heads / H)
    per second of their total time."""
    w = wl.get(args.workload)
    x_cpu = wl.generate(w)
    order = _head_order(w, x_cpu)
    per_step = max(1, min(args.ref_heads, len(order)))
    pos, times = 0, []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        for _ in range(per_step):
            l, h = order[pos % len(order)]
            _oracle_head(w, x_cpu, l, h)
            pos += 1
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
    total_s = sum(times)
    value = (per_step * args.steps / w.H) / total_s
    cb = {"value": round(value, 6), "unit": UNIT, "cores": _cores(), "cpu_model": cpu_model(),
          "kind": "oracle",
          "sample": f"{per_step} of {w.L * w.H} heads of workload {w.name} per step (full oracle "
                    f"step per head, every query row), {args.steps} timed steps in "
                    f"{total_s:.1f} s, numpy fp64",
          "seconds": round(total_s, 2)}
    return {
        "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(1e3 * total_s / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded, Wan-shaped)",
        "config": bench_config(w, w),
        "impl": "reference", "cpu_baseline": cb,
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="480p", choices=sorted(wl.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--split", default="replicas", choices=["replicas", "heads"],
                    help="N > 1: independent replicas per GPU (weak scaling) or the heads of "
                         "one step split across GPUs (strong scaling)")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--ref-heads", type=int, default=2,
                    help="reference arm: whole heads of the workload per timed step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--extra", default="1080p,480p_30layer,token14b",
                    help="N = 1: further workloads timed after the headline one, reported "
                         "under 'workloads' (empty string: none)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)  # at least 3 untimed warm-up steps
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank != 0:
            return
        print(json.dumps(run_reference(args)), flush=True)
        return
    line = run_ours(args, rank, world, local_rank)
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
