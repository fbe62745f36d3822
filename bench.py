#!/usr/bin/env python
"""Benchmark: causal attention forward + backward (bf16) TFLOP/s on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one forward + one backward over the whole workload (default: the
long-context window B=1, H=16, T=8192, D=128 with RoPE), inputs resident in
HBM: attn_fwd_save + attn_bwd_saved, the forward's rotated q, k kept for the
backward as a training step keeps its activations (--no-save: the plain
attn_fwd + attn_bwd, which rotate q, k in both calls). Each timed step is bracketed by CUDA events on the launching stream; L2
is flushed (a 256 MiB write) between steps, outside the events; warm-up steps
repeat the timed sequence (flush included) and the NVML clock sampler starts
before them, keeping samples of the timed steps only. FLOPs follow
the nominal convention 4*B*H*T^2*D/2 forward and 2.5x that backward
(7*B*H*T^2*D per step; for packed documents the within-document figure is
reported beside it). With N > 1 (torchrun, one process per GPU) every rank
runs its own replica of the workload (weak scaling: attention has no
exchange step), the step time is the max over ranks, and value is the
aggregate. Rank 0 prints one JSON line.

--impl reference times the float64 CPU oracle on the host cores instead
(rank 0 only), each step one (batch, head) slice of the same workload.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "causal attention fwd+bwd TFLOP/s (bf16) and % of B200 dense BF16 tensor peak"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# FP32 FMA peak of the CUDA cores: 148 SMs x 128 lanes x 2 flop x 1.965 GHz.
FP32_SIMT_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) per launch from
# one ncu capture of the kernel on the workload, valid only while the kernel
# sources still hash to what was captured (sha256, first 16 hex digits).
MEASURED_TRAFFIC = {
    ("dkdv", "long_context_8k"): (687.5e6, {"bwd_sm100.cuh": "c69bb6094afca43f",
                                            "sm100.cuh": "d00797b7a9dd3426",
                                            "common.cuh": "36b3720cacd61ee7"}),
    ("dkdv", "decoder237m_layer"): (124.5e6, {"bwd_sm100.cuh": "c69bb6094afca43f",
                                              "sm100.cuh": "d00797b7a9dd3426",
                                              "common.cuh": "36b3720cacd61ee7"}),
    ("fwd", "long_context_8k"): (157.7e6, {"fwd_sm100.cuh": "a1c0ac515047a7cc",
                                           "sm100.cuh": "d00797b7a9dd3426",
                                           "common.cuh": "36b3720cacd61ee7"}),
    ("fwd", "decoder237m_layer"): (50.4e6, {"fwd_sm100.cuh": "a1c0ac515047a7cc",
                                            "sm100.cuh": "d00797b7a9dd3426",
                                            "common.cuh": "36b3720cacd61ee7"}),
    ("decode", "decode_8k_gqa"): (200.6e6, {"decode.cuh": "ed672db8f3155da3",
                                            "sm100.cuh": "d00797b7a9dd3426",
                                            "common.cuh": "36b3720cacd61ee7"}),
}


def measured_traffic(kernel: str, workload: str):
    import hashlib
    entry = MEASURED_TRAFFIC.get((kernel, workload))
    if entry is None:
        return None
    nbytes, sources = entry
    csrc = os.path.join(ROOT, "bwd_causal_sdpa_b200", "csrc")
    for name, digest in sources.items():
        with open(os.path.join(csrc, name), "rb") as f:
            if hashlib.sha256(f.read()).hexdigest()[:16] != digest:
                return None  # the kernel changed since the counters were taken
    return nbytes


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="long_context_8k")
    ap.add_argument("--kv-heads", type=int, default=None,
                    help="grouped-query attention: key/value heads (dividing the workload's H)")
    ap.add_argument("--decode", default=None,
                    help="time decode attention on this decode workload instead of the training step")
    ap.add_argument("--proj", default=None,
                    help="time the projections around the attention on this projection workload")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--bwd-route", type=int, default=0,
                    help="backward route (attn_set_backward_route): 0 default, 1 key-tile dK/dV + "
                         "query-tile dQ pass, 2 CTA-pair dK/dV (D = 128) + query-tile dQ pass")
    ap.add_argument("--no-save", action="store_true",
                    help="plain attn_fwd / attn_bwd (the backward rotates q, k again)")
    ap.add_argument("--sustain", type=float, default=0.0,
                    help="also time back-to-back steps for about this many seconds and report "
                         "them against the sustained bf16 peak (clocks and power sampled)")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------------
# FLOP accounting
# ---------------------------------------------------------------------------

def causal_unit(w) -> float:
    """One causal matmul over the workload: H*D*sum(L^2) flops (2 per MAC
    over the L^2/2 allowed pairs of each document)."""
    return w.algorithmic_flops() / 7.0


def kernel_algorithmic(name: str, w, kinds_seen) -> tuple:
    """(bound, algorithmic amount per launch, unit) for one kernel kind."""
    U = causal_unit(w)
    elem = 2 if w.dtype == "bf16" else 4
    N = w.B * w.H * w.T * w.D
    Nkv = w.B * w.kv_heads * w.T * w.D
    R = w.B * w.H * w.T
    if name == "fwd":
        return "tensor", 2 * U, "flop"
    if name == "dkdv":
        return "tensor", (4 if "dq" in kinds_seen else 5) * U, "flop"
    if name == "dq":
        return "tensor", 1 * U, "flop"
    if name == "delta":
        if w.dtype != "bf16":  # Delta only
            return "hbm", 2 * N * elem + 4 * R, "byte"
        # bf16 backward row pass: read o, dO, lse; write -Delta and -lse*log2e,
        # zero the fp32 dq accumulator; with RoPE (fp16 operands) also read v
        # for the per-head norm statistics
        v_read = Nkv * elem if w.rope_cos is not None else 0
        return "hbm", 2 * N * elem + 12 * R + 4 * N + v_read, "byte"
    if name == "rope_prep":
        return "hbm", 2 * (N + Nkv) * elem, "byte"
    if name == "dq_finalize":
        return "hbm", N * 4 + N * elem, "byte"
    return "hbm", 0, "byte"


def ideal_tiles(w) -> dict:
    """Tile products (128 queries x 128 keys, per query head) that hold at
    least one allowed (query, key) pair, and the allowed pairs themselves in
    tile units. A query tile's allowed keys form one range, from the start
    of its first row's document to its last row (rows are causal and a
    document is contiguous), so the tiles holding an allowed pair are exactly
    the key tiles of that range; the same set, seen from a key tile, is the
    query tiles from its own to the one holding its last key's document end.
    This is the least work block skipping can do at this tile size."""
    import numpy as np

    T, B, H = w.T, w.B, w.H
    nt, n64 = (T + 127) // 128, (T + 63) // 64
    tiles = blocks = 0
    for b in range(B):
        ds = np.zeros(T, dtype=np.int64)
        if w.cu_seqlens is not None:
            cu = w.cu_seqlens.astype(np.int64)
            row = cu[(cu >= b * T) & (cu <= (b + 1) * T)] - b * T
            for a, e in zip(row[:-1], row[1:]):
                ds[a:e] = a
        qt = np.arange(nt)
        first = qt * 128
        tiles += int(np.sum(qt - ds[first] // 128 + 1))
        # the forward walks keys in blocks of 64: per query tile, the blocks
        # from its first row's document start to its diagonal
        blocks += int(np.sum(np.minimum(2 * qt + 2, n64) - ds[first] // 64))
    L = np.asarray(w.doc_lengths(), dtype=np.float64)
    allowed = float(np.sum(L * (L + 1) / 2))
    return {"ideal": tiles * H, "fwd_ideal_blocks64": blocks * H,
            "allowed_pairs_in_tiles": allowed * H / (128 * 128)}


# ---------------------------------------------------------------------------
# Clock sampling (NVML, read-only) during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    REASONS = [(0x4, "sw_power_cap"), (0x8, "hw_slowdown"), (0x20, "sw_thermal_slowdown"),
               (0x40, "hw_thermal_slowdown"), (0x80, "hw_power_brake_slowdown"),
               (0x2, "applications_clocks_setting"), (0x1, "gpu_idle")]

    def __init__(self, index: int, period_s: float = 0.01, gated: bool = False):
        """Samples every ``period_s`` seconds on a thread of its own. With
        ``gated`` the thread starts (and NVML is initialised) on entry but
        keeps samples only between ``on()`` and ``off()``: entered before the
        warm-up, so nothing of its start-up falls into the timed steps."""
        self.index, self.period = index, period_s
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.power_w = []
        self._stop = threading.Event()
        self._keep = threading.Event()
        if not gated:
            self._keep.set()
        self._thr = None
        self.error = None

    def on(self):
        self._keep.set()

    def off(self):
        self._keep.clear()

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._query()  # first calls resolve NVML's entry points: keep them here
            self._thr = threading.Thread(target=self._run, daemon=True)
            self._thr.start()
        except Exception as e:  # NVML missing: report no clocks rather than guess
            self.error = repr(e)
        return self

    def _query(self):
        nv = self._nv
        mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
        watts = nv.nvmlDeviceGetPowerUsage(self._h) / 1000.0
        mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h) \
            if hasattr(nv, "nvmlDeviceGetCurrentClocksEventReasons") \
            else nv.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
        return mhz, watts, mask

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz, watts, mask = self._query()
                if self._keep.is_set():
                    self.samples.append(mhz)
                    self.power_w.append(watts)
                    for bit, name in self.REASONS:
                        if mask & bit:
                            self.reasons.add(name)
            except Exception as e:
                self.error = repr(e)
                break
            time.sleep(self.period)

    def __exit__(self, *exc):
        self._stop.set()
        if self._thr:
            self._thr.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0, "error": self.error}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples),
                "power_w_median": statistics.median(self.power_w) if self.power_w else None,
                "power_w_max": max(self.power_w) if self.power_w else None}


# ---------------------------------------------------------------------------
# CPU oracle timing (the baseline, and the reference arm)
# ---------------------------------------------------------------------------

def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [p.get("num_threads", 1) for p in threadpool_info() if p.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return 1


def oracle_slice_seconds(w, heads, outputs=None):
    """Seconds the float64 oracle takes for the forward and backward of the
    given (b, h) slices; its results go into ``outputs`` when a dict is given."""
    from oracle import attention_backward, attention_forward

    t0 = time.perf_counter()
    o, lse = attention_forward(w.q, w.k, w.v, w.rope_cos, w.rope_sin, w.cu_seqlens, w.scale,
                               heads=heads)
    dq, dk, dv = attention_backward(w.q, w.k, w.v, w.do, w.rope_cos, w.rope_sin, w.cu_seqlens,
                                    w.scale, heads=heads)
    secs = time.perf_counter() - t0
    if outputs is not None:
        outputs.update(o=o, lse=lse, dq=dq, dk=dk, dv=dv)
    return secs


def slice_errors(w, heads, ref, got):
    """Relative Frobenius error of each output over the sampled slices (dk, dv
    only when every query head has its own key/value head: with grouped heads
    the oracle's partial sums over the sample are not the whole gradient)."""
    import numpy as np

    errs = {}
    names = ["o", "lse", "dq"] + (["dk", "dv"] if w.kv_heads == w.H else [])
    for n in names:
        a = np.stack([got[n][b, h] for b, h in heads]).astype(np.float64)
        r = np.stack([ref[n][b, h] for b, h in heads])
        den = np.linalg.norm(r)
        errs[n] = float(np.linalg.norm(a - r) / (den if den > 0 else 1.0))
    return errs


def slice_flops(w, heads) -> float:
    """Nominal-convention flops of the given (b, h) slices (within-document for
    packed rows): 7 * D * sum over their documents of L^2."""
    import numpy as np
    total = 0.0
    for b, _h in heads:
        if w.cu_seqlens is None:
            total += 7.0 * w.D * w.T * w.T
        else:
            cu = w.cu_seqlens.astype(np.int64)
            L = np.diff(cu)[(cu[:-1] >= b * w.T) & (cu[:-1] < (b + 1) * w.T)].astype(np.float64)
            total += 7.0 * w.D * float((L * L).sum())
    return total


def sample_description(w, heads):
    return (f"fwd+bwd of {len(heads)} (batch, head) slice(s) {heads} of {w.cfg.name} "
            f"(T={w.T}, D={w.D}), float64 NumPy oracle")


# ---------------------------------------------------------------------------
# Arms
# ---------------------------------------------------------------------------

def max_over_ranks(x: float, world: int, device) -> float:
    """The largest of every rank's value (the job's time is its slowest
    rank's); one all-reduce on a one-element tensor on ``device`` (the GPU
    under NCCL, the CPU under gloo)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_rank_step: float, world: int, ms: float) -> float:
    """Weak scaling: every rank runs its own workload; the job's throughput is
    all ranks' flops over the slowest rank's step time."""
    return flops_per_rank_step * world / (ms / 1e3) / 1e12


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        if world == 1:
            raise SystemExit("--gpus N > 1 needs torchrun with N processes")
        raise SystemExit(f"--gpus {n_gpus} does not match the {world} launched processes")
    return world, rank, local


def run_reference(args):
    import torch
    from workloads import config_by_name, make_workload

    world, rank, _ = dist_setup(args.gpus)
    if rank != 0:
        return 0
    w = make_workload(config_by_name(args.workload))
    heads = [(0, 0)]
    for _ in range(args.warmup):
        oracle_slice_seconds(w, heads)
    secs = [oracle_slice_seconds(w, heads) for _ in range(args.steps)]
    per_step = sum(secs) / len(secs)
    value = slice_flops(w, heads) / per_step / 1e12
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": per_step * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
        "config": workload_config(w, l2="n/a (host)"),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample_description(w, heads)},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    del torch
    return 0


def workload_config(w, l2):
    c = {"workload": w.cfg.name, "B": w.B, "H": w.H, "H_kv": w.kv_heads, "T": w.T, "D": w.D,
         "rope": w.rope_cos is not None,
         "varlen": w.cu_seqlens is not None, "global_batch": w.B, "seq_len": w.T,
         "parallelism": "replicas (one independent workload per GPU)", "l2": l2,
         "flops_per_step_nominal": w.cfg.nominal_flops if (w.B, w.T, w.D) == (w.cfg.B, w.cfg.T, w.cfg.D)
         else 7.0 * w.B * w.H * w.T * w.T * w.D,
         "flops_per_step_within_documents": w.algorithmic_flops()}
    if w.cu_seqlens is not None:
        c["documents"] = int(len(w.cu_seqlens) - 1)
    return c


def run_ours(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    import bwd_causal_sdpa_b200 as A
    from bwd_causal_sdpa_b200.runner import AttnRunner
    from workloads import config_by_name, make_workload

    world, rank, local = dist_setup(args.gpus)
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()


    cfg = config_by_name(args.workload)
    w = make_workload(cfg, H_kv=args.kv_heads)
    stream = torch.cuda.Stream(dev)
    A.check(A.attn_set_backward_route(args.bwd_route), "attn_set_backward_route")
    r = AttnRunner.from_workload(w, device=dev, stream=stream, save=not args.no_save)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    peaks, peak_src = load_peaks()
    flops_step = 7.0 * w.B * w.H * w.T * w.T * w.D

    # The clock sampler starts before the warm-up (its start-up stays out of
    # the timed steps) and keeps samples of the timed region only; warm-up
    # steps are the timed steps' exact sequence, flush included.
    with ClockSampler(local, gated=True) as clocks:
        with torch.cuda.stream(stream):
            for _ in range(max(args.warmup, 0)):
                flush.zero_()
                r.forward()
                r.backward()
        st = r.status()
        if st != A.ATTN_OK:
            raise SystemExit(f"device status after warm-up: {A.error_string(st)}")

        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        torch.cuda.synchronize(dev)
        barrier()
        torch.cuda.synchronize(dev)
        A.check(A.attn_tile_counts()[0], "attn_tile_counts")  # reset the device counters
        n0 = A.attn_launch_count()
        clocks.on()
        with torch.cuda.stream(stream):
            for i in range(args.steps):
                flush.zero_()
                ev[i][0].record(stream)
                r.forward()
                r.backward()
                ev[i][1].record(stream)
        torch.cuda.synchronize(dev)
        clocks.off()
    barrier()
    torch.cuda.synchronize(dev)
    launches = A.attn_launch_count() - n0
    code, fwd_tiles, bwd_tiles, dq_tiles = A.attn_tile_counts()
    A.check(code, "attn_tile_counts")
    tiles = None
    if w.dtype == "bf16":
        tiles = ideal_tiles(w)
        tiles.update(fwd_executed_blocks64=fwd_tiles / args.steps,
                     fwd_executed=fwd_tiles / 2 / args.steps,
                     bwd_executed=bwd_tiles / args.steps, dq_pass_executed=dq_tiles / args.steps)
        tiles["fwd_over_ideal"] = tiles["fwd_executed_blocks64"] / tiles["fwd_ideal_blocks64"]
        tiles["bwd_over_ideal"] = tiles["bwd_executed"] / tiles["ideal"]
        tiles["unit"] = ("128x128 tile products per step, all query heads (device counters); "
                         "the forward also in its own 128-query x 64-key blocks")
    step_ms = [a.elapsed_time(b) for a, b in ev]
    # Per-kernel times for the roofline come from a second pass over the same
    # number of steps with an event pair around every launch (kept out of the
    # timed steps above: events between launches would stop them overlapping).
    A.check(A.attn_profile_enable(1), "attn_profile_enable")
    with torch.cuda.stream(stream):
        for i in range(args.steps):
            flush.zero_()
            r.forward()
            r.backward()
    torch.cuda.synchronize(dev)
    A.attn_profile_enable(0)
    prof = A.profile_summary()
    ms_local = sum(step_ms) / len(step_ms)
    ms = max_over_ranks(ms_local, world, dev)
    value = whole_job_tflops(flops_step, world, ms)
    st = r.status()
    if st != A.ATTN_OK:
        raise SystemExit(f"device status after timing: {A.error_string(st)}")

    # Dominant kernel: the kind with the largest summed event time.
    kinds = set(prof)
    dom = max(prof.items(), key=lambda kv: kv[1][1])[0] if prof else None
    roofline = None
    kernels = {}
    for name, (n, tot) in prof.items():
        bound, amount, u = kernel_algorithmic(name, w, kinds)
        kernels[name] = {"launches": n, "avg_ms": tot / n, "share": None, "bound": bound,
                         "algorithmic": amount, "algorithmic_unit": u}
    total_k = sum(tot for _, tot in prof.values())
    for name in kernels:
        kernels[name]["share"] = prof[name][1] / total_k if total_k else None
    if dom is not None:
        kd = kernels[dom]
        simt = w.dtype != "bf16"  # bf16 runs on the tensor cores; f32 on the CUDA cores
        if kd["bound"] == "tensor":
            achieved = kd["algorithmic"] / (kd["avg_ms"] / 1e3) / 1e12
            if simt:
                peak, unit, bound = FP32_SIMT_PEAK_TFLOPS, "TFLOP/s", "alu"
                peak_note = "fp32 FMA peak of the CUDA cores (148 SMs x 128 x 2 x 1.965 GHz)"
            else:
                peak, unit, bound = peaks["bf16_tflops"], "TFLOP/s", "tensor"
                peak_note = f"bf16_tflops burst ({peak_src})"
        else:
            achieved = kd["algorithmic"] / (kd["avg_ms"] / 1e3) / 1e9
            peak, unit, bound = peaks["hbm_gbs"], "GB/s", "hbm"
            peak_note = f"hbm_gbs ({peak_src})"
        roofline = {"bound": bound, "kernel": dom, "achieved": achieved, "peak": peak,
                    "unit": unit, "frac": achieved / peak,
                    "traffic": (measured_traffic(dom, w.cfg.name)
                                if (w.B, w.T) == (cfg.B, cfg.T) and w.kv_heads == w.H else None),
                    "traffic_unit": "bytes per launch (ncu dram read + write)",
                    "algorithmic_per_launch": kd["algorithmic"],
                    "algorithmic_unit": kd["algorithmic_unit"],
                    "peak_source": peak_note}

    # End to end through the public API with host buffers: every step copies
    # its inputs in from pinned host memory and its five results back out.
    # Steps are pipelined the way a caller overlaps them on a B200: two
    # device buffer sets, a copy-in stream, the compute stream and a copy-out
    # stream, so step i+1's inputs travel in and step i-1's results travel
    # out (the two PCIe directions run at once) while step i computes. The
    # serial figure (one stream, copy in -> compute -> copy out) is reported
    # beside it.
    e2e = None
    if not args.no_e2e:
        r2 = AttnRunner.from_workload(w, device=dev, stream=stream, save=not args.no_save)
        sets = [r, r2]
        host_in = [x.detach().to("cpu").pin_memory() for x in (r.q, r.k, r.v, r.do)]
        host_out = [[torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
                     for x in (r.o, r.lse, r.dq, r.dk, r.dv)] for _ in range(2)]
        h2d = sum(x.numel() * x.element_size() for x in host_in)
        d2h = sum(x.numel() * x.element_size() for x in host_out[0])
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev = lambda: torch.cuda.Event(enable_timing=False)
        outs = lambda rr: (rr.o, rr.lse, rr.dq, rr.dk, rr.dv)

        def pipelined(steps):
            in_done = [ev() for _ in range(steps)]
            comp_done = [ev() for _ in range(steps)]
            out_done = [ev() for _ in range(steps)]
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record(s_in)
            for i in range(steps):
                rr = sets[i % 2]
                with torch.cuda.stream(s_in):  # inputs of step i
                    if i >= 2:
                        s_in.wait_event(comp_done[i - 2])  # step i-2 done reading this set
                    for dst, src in zip((rr.q, rr.k, rr.v, rr.do), host_in):
                        dst.copy_(src, non_blocking=True)
                    in_done[i].record(s_in)
                with torch.cuda.stream(stream):  # step i's kernels
                    stream.wait_event(in_done[i])
                    if i >= 2:
                        stream.wait_event(out_done[i - 2])  # this set's results copied out
                    flush.zero_()
                    rr.forward()
                    rr.backward()
                    comp_done[i].record(stream)
                with torch.cuda.stream(s_out):  # results of step i
                    s_out.wait_event(comp_done[i])
                    for dst, src in zip(host_out[i % 2], outs(rr)):
                        dst.copy_(src, non_blocking=True)
                    out_done[i].record(s_out)
            s_out.wait_event(out_done[steps - 1])
            t1.record(s_out)
            torch.cuda.synchronize(dev)
            return t0.elapsed_time(t1) / steps

        def serial(steps):
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(steps)]
            with torch.cuda.stream(stream):
                for i in range(steps):
                    flush.zero_()
                    evs[i][0].record(stream)
                    for dst, src in zip((r.q, r.k, r.v, r.do), host_in):
                        dst.copy_(src, non_blocking=True)
                    r.forward()
                    r.backward()
                    for dst, src in zip(host_out[0], outs(r)):
                        dst.copy_(src, non_blocking=True)
                    evs[i][1].record(stream)
            torch.cuda.synchronize(dev)
            return sum(a.elapsed_time(b) for a, b in evs) / steps

        torch.cuda.synchronize(dev)
        pipelined(min(4, args.steps))  # warm-up of the streams and the second set
        barrier()
        e_ms = max_over_ranks(pipelined(args.steps), world, dev)
        barrier()
        s_ms = max_over_ranks(serial(args.steps), world, dev)
        e2e = {"value": whole_job_tflops(flops_step, world, e_ms), "unit": UNIT,
               "ms_per_step": e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "mode": "pipelined: two device buffer sets, copy-in / compute / copy-out streams",
               "serial_value": whole_job_tflops(flops_step, world, s_ms),
               "serial_ms_per_step": s_ms}
        del r2, sets

    sustained = None
    if args.sustain > 0:
        # back-to-back steps for about args.sustain seconds (steps sized from
        # the timed region), same step and flush as above, so the GPU reaches
        # its power-limited clocks; reported against the sustained peak
        n_sus = max(1, int(args.sustain * 1e3 / (ms_local + 0.05)))
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n_sus)]
        torch.cuda.synchronize(dev)
        barrier()
        with ClockSampler(local, period_s=0.05) as sclk:
            with torch.cuda.stream(stream):
                for i in range(n_sus):
                    flush.zero_()
                    evs[i][0].record(stream)
                    r.forward()
                    r.backward()
                    evs[i][1].record(stream)
            torch.cuda.synchronize(dev)
        barrier()
        s_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs) / n_sus, world, dev)
        s_val = whole_job_tflops(flops_step, world, s_ms)
        sustained = {"value": s_val, "unit": UNIT, "steps": n_sus, "ms_per_step": s_ms,
                     "timed_seconds": n_sus * s_ms / 1e3,
                     "frac_of_bf16_sustained": s_val / world / peaks["bf16_tflops_sustained"],
                     "frac_of_bf16_burst": s_val / world / peaks["bf16_tflops"],
                     "clocks": sclk.summary()}
        if r.status() != A.ATTN_OK:
            raise SystemExit("device status after the sustained run is not OK")

    cpu = None
    parity = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        heads = [(0, 0)]
        ref = {}
        secs = oracle_slice_seconds(w, heads, ref)
        cpu = {"value": slice_flops(w, heads) / secs / 1e12, "unit": UNIT,
               "cores": blas_threads(), "kind": "oracle", "seconds": secs,
               "sample": sample_description(w, heads)}
        # the timed path's own outputs (the inputs never change between
        # steps) against the oracle on the same slice
        parity = {"sample": [list(x) for x in heads],
                  "rel_fro": slice_errors(w, heads, ref, r.results()),
                  "tolerance": ({"o": 1e-2, "lse": 1e-4, "dq": 1e-2, "dk": 1e-2, "dv": 1e-2}
                                if w.dtype == "bf16" else
                                {"o": 1e-5, "lse": 1e-5, "dq": 1e-5, "dk": 1e-5, "dv": 1e-5})}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic (seeded)",
            "config": dict(workload_config(w, l2="flushed between steps (256 MiB write outside the step events)"),
                           calls=("attn_fwd_gqa + attn_bwd_gqa" if args.no_save or r.saved is None
                                  else "attn_fwd_save + attn_bwd_saved (rotated q, k kept between them)"),
                           backward_route=args.bwd_route),
            "pct_of_bf16_peak": value / world / peaks["bf16_tflops"],
            "pct_of_bf16_peak_sustained": value / world / peaks["bf16_tflops_sustained"],
            "peaks_source": peak_src,
            "value_within_documents": w.algorithmic_flops() * world / (ms / 1e3) / 1e12,
            "roofline": roofline, "kernels": kernels, "tiles": tiles, "sustained": sustained,
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches,
            "clocks": clocks.summary(), "parity": parity,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_decode(args):
    """Decode attention (one new token per sequence against a key/value
    cache): bytes of cache read per second, against the measured HBM copy
    bandwidth; L2 is flushed between steps as in the training bench."""
    import torch

    import bwd_causal_sdpa_b200 as A
    from bwd_causal_sdpa_b200.runner import DecodeRunner
    from workloads import decode_config_by_name, make_decode_workload

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = make_decode_workload(decode_config_by_name(args.decode))
    stream = torch.cuda.Stream(dev)
    r = DecodeRunner(w, device=dev, stream=stream)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    peaks, peak_src = load_peaks()
    with ClockSampler(0, gated=True) as clocks:  # started before the warm-up, as above
        with torch.cuda.stream(stream):
            for _ in range(max(args.warmup, 0)):
                flush.zero_()
                r.run()
        if r.status() != A.ATTN_OK:
            raise SystemExit("device status after warm-up is not OK")
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        torch.cuda.synchronize(dev)
        n0 = A.attn_launch_count()
        clocks.on()
        with torch.cuda.stream(stream):
            for i in range(args.steps):
                flush.zero_()
                ev[i][0].record(stream)
                r.run()
                ev[i][1].record(stream)
        torch.cuda.synchronize(dev)
        clocks.off()
    launches = A.attn_launch_count() - n0
    # per-kernel times from a separate pass (events around every launch)
    A.check(A.attn_profile_enable(1), "attn_profile_enable")
    with torch.cuda.stream(stream):
        for i in range(args.steps):
            flush.zero_()
            r.run()
    torch.cuda.synchronize(dev)
    A.attn_profile_enable(0)
    prof = A.profile_summary()
    ms = sum(a.elapsed_time(b) for a, b in ev) / args.steps
    nbytes = w.cache_bytes_read()
    gbs = nbytes / (ms / 1e3) / 1e9
    kd = prof.get("decode")
    achieved = nbytes / (kd[1] / kd[0] / 1e3) / 1e9 if kd else None
    line = {
        "metric": "decode attention: key/value cache bytes read per second", "value": gbs,
        "unit": "GB/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": w.dtype, "data": "synthetic (seeded)",
        "config": {"workload": w.cfg.name, "B": w.B, "H": w.H, "H_kv": w.H_kv, "T_max": w.T_max,
                   "D": w.D, "cache_tokens": int(w.cache_lens.sum()), "cache_bytes": nbytes,
                   "l2": "flushed between steps (256 MiB write outside the step events)"},
        "roofline": None if achieved is None else {
            "bound": "hbm", "kernel": "decode", "achieved": achieved, "peak": peaks["hbm_gbs"],
            "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
            "traffic": measured_traffic("decode", w.cfg.name),
            "peak_source": f"hbm_gbs ({peak_src})"},
        "kernels": {k: {"launches": n, "avg_ms": t / n} for k, (n, t) in prof.items()},
        "gpu_launches": launches, "clocks": clocks.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


def run_proj(args):
    """The projections around one attention layer, forward and backward: the
    QKV projection (head layout and RoPE in its epilogue), the output
    projection and their four backward products (dx, dW for each), as
    TFLOP/s of GEMM work against the measured bf16 tensor peak; L2 is flushed
    between steps as in the training bench."""
    import torch

    import bwd_causal_sdpa_b200 as A
    from bwd_causal_sdpa_b200.runner import ProjRunner
    from workloads import make_proj_workload, proj_config_by_name

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = make_proj_workload(proj_config_by_name(args.proj))
    stream = torch.cuda.Stream(dev)
    r = ProjRunner(w, device=dev, stream=stream)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    peaks, peak_src = load_peaks()

    def step():
        r.qkv()
        r.out()
        r.out_bwd()
        r.qkv_bwd()

    with ClockSampler(0, gated=True) as clocks:  # started before the warm-up, as above
        with torch.cuda.stream(stream):
            for _ in range(max(args.warmup, 0)):
                flush.zero_()
                step()
        if r.status() != A.ATTN_OK:
            raise SystemExit("device status after warm-up is not OK")
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        torch.cuda.synchronize(dev)
        n0 = A.attn_launch_count()
        clocks.on()
        with torch.cuda.stream(stream):
            for i in range(args.steps):
                flush.zero_()
                ev[i][0].record(stream)
                step()
                ev[i][1].record(stream)
        torch.cuda.synchronize(dev)
        clocks.off()
    launches = A.attn_launch_count() - n0
    A.check(A.attn_profile_enable(1), "attn_profile_enable")
    with torch.cuda.stream(stream):
        for i in range(args.steps):
            flush.zero_()
            step()
    torch.cuda.synchronize(dev)
    A.attn_profile_enable(0)
    prof = A.profile_summary()
    ms = sum(a.elapsed_time(b) for a, b in ev) / args.steps
    fl = w.flops()
    flops = sum(fl.values())
    tflops = flops / (ms / 1e3) / 1e12
    kg = prof.get("gemm")
    achieved = flops / (kg[1] / args.steps / 1e3) / 1e12 if kg else None
    c = w.cfg
    line = {
        "metric": "attention-layer projections fwd+bwd TFLOP/s (bf16 GEMMs)", "value": tflops,
        "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded)",
        "config": {"workload": c.name, "B": c.B, "T": c.T, "C": c.C, "H": c.H, "H_kv": c.H_kv,
                   "D": c.D, "rope": c.rope, "flops_per_step": flops, "flops_by_call": fl,
                   "l2": "flushed between steps (256 MiB write outside the step events)"},
        "roofline": None if achieved is None else {
            "bound": "tensor", "kernel": "gemm (all six products of a step)",
            "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
            "frac": achieved / peaks["bf16_tflops"], "traffic": None,
            "peak_source": f"bf16_tflops burst ({peak_src})"},
        "kernels": {k: {"launches": n, "avg_ms": t / n} for k, (n, t) in prof.items()},
        "gpu_launches": launches, "clocks": clocks.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse_args()
    if args.decode:
        return run_decode(args)
    if args.proj:
        return run_proj(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
