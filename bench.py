#!/usr/bin/env python
"""Benchmark of the LSH-attention hot path on B200.

Headline: forward tokens/s (B*L per second, all heads and 8 hash rounds) on
the L=65536 workload (B=1, H=8, d=64, n_buckets=1024, n_rounds=8, chunk=64,
causal, bf16), one step = hash -> sort -> chunk attention -> round combine,
inputs resident in HBM, L2 flushed (256 MB memset) between timed steps.
Also reported: fwd+bwd tokens/s with the backward's roofline (L=16384
workload and an L=65536 variant), the same forward end to end from pinned
host buffers, per-stage times, the roofline of the dominant kernel, every
other workload's forward with its roofline, recall against full attention
over rounds and bucket counts, the chunked feed-forward's positions/s with
its tensor roofline, the reversible block's forward and backward tokens/s,
clocks, and the CPU oracle timed on the host cores
(with a parity record of the head it recomputes).

``--impl reference`` times the CPU oracle (the reference arm) on a bounded
sample of the same workload.  Under torchrun every rank runs the full
workload on its own GPU (weak scaling, no data-path collective); timings are
max-reduced over ranks.
"""

from __future__ import annotations

import argparse
import dataclasses
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from lsh_attention_long_b200 import workloads as W  # noqa: E402

METRIC = "LSH-attention tokens/s (fwd, fwd+bwd) at L=65536, 8 rounds; % of roofline"
HEADLINE = "fwd_bf16_L65536"
BWD_WORKLOAD = "fwdbwd_bf16_L16384"
FLUSH_BYTES = 256 << 20
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default=HEADLINE)
    p.add_argument("--no-extras", action="store_true",
                   help="headline only: skip fwd+bwd, e2e and the CPU baseline")
    p.add_argument("--fwd-bwd", action="store_true",
                   help="only the forward + backward measurement of --workload (a "
                        "diagnostic line, not the headline)")
    p.add_argument("--recall", action="store_true",
                   help="recall of LSH attention against full attention on the clustered "
                        "L=16384 workload, over rounds and bucket counts (a report)")
    p.add_argument("--heads", type=int, default=0,
                   help="run --workload with this many heads instead of its own (a "
                        "smaller case of the same kernels, e.g. for profiling); the "
                        "line's workload name gets an _H<heads> suffix")
    p.add_argument("--ffn", action="store_true",
                   help="only the chunked feed-forward line (a diagnostic line)")
    p.add_argument("--rev", action="store_true",
                   help="only the reversible-block line (a diagnostic line)")
    p.add_argument("--shard", choices=["none", "heads"], default="none",
                   help="heads: split one problem's B*H heads over the ranks (strong "
                        "scaling) instead of a replica per rank")
    p.add_argument("--gather", action="store_true",
                   help="with --shard heads: all-gather O and lse to every rank inside "
                        "the timed step")
    p.add_argument("--ref-seconds", type=float, default=150.0,
                   help="--impl reference: CPU seconds of oracle sampling over all steps")
    return p.parse_args()


# ---------------------------------------------------------------------------
# process group (one rank per GPU; collectives only for barriers and timing)
# ---------------------------------------------------------------------------

def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def aggregate_tokens_per_s(world: int, tokens_per_rank_step: int, steps: int,
                           max_ms: float) -> float:
    """Whole-job throughput: every rank runs its own copy of the workload
    (weak scaling), timed by the slowest rank."""
    return world * tokens_per_rank_step * steps / (max_ms / 1e3)


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
# clocks during the timed regions
# ---------------------------------------------------------------------------

class ClockSampler:
    """Samples SM clock, power and clock-event reasons through NVML every
    10 ms on a background thread while the timed region runs."""

    REASONS = (("nvmlClocksEventReasonHwSlowdown", "hw_slowdown"),
               ("nvmlClocksEventReasonHwThermalSlowdown", "hw_thermal_slowdown"),
               ("nvmlClocksEventReasonSwThermalSlowdown", "sw_thermal_slowdown"),
               ("nvmlClocksEventReasonSwPowerCap", "sw_power_cap"),
               ("nvmlClocksEventReasonHwPowerBrakeSlowdown", "hw_power_brake_slowdown"))

    def __init__(self, index: int):
        self.index = index
        self.rows = []
        self.err = None
        self._stop = None
        self._thread = None

    def __enter__(self):
        import threading
        try:
            import pynvml as nv
            nv.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            phys = int(vis.split(",")[self.index]) if vis and vis.split(",")[0].isdigit() \
                else self.index
            h = nv.nvmlDeviceGetHandleByIndex(phys)
            self.smax = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: report that instead of clocks
            self.err = f"nvml unavailable: {e}"
            return self
        self._stop = threading.Event()

        def loop():
            while not self._stop.is_set():
                try:
                    self.rows.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM),
                                      nv.nvmlDeviceGetPowerUsage(h) / 1000.0,
                                      nv.nvmlDeviceGetCurrentClocksEventReasons(h)))
                except Exception as e:
                    self.err = str(e)
                    return
                time.sleep(0.01)

        self._nv = nv
        self._thread = threading.Thread(target=loop, daemon=True)
        self._thread.start()
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=5)

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [self.err or "no samples"]}
        nv = self._nv
        reasons = []
        for attr, name in self.REASONS:
            bit = getattr(nv, attr, 0)
            if any(r[2] & bit for r in self.rows):
                reasons.append(name)
        return {"sm_mhz": statistics.median(r[0] for r in self.rows), "sm_max_mhz": self.smax,
                "reasons": reasons, "samples": len(self.rows),
                "power_w_max": round(max(r[1] for r in self.rows), 1), "source": "nvml 10 ms"}


# ---------------------------------------------------------------------------
# algorithmic work per stage (per call of the stage on workload w)
# ---------------------------------------------------------------------------

def stage_work(w: W.Workload):
    s = 2 if w.dtype == "bf16" else 4
    d, R = w.d, w.n_rounds
    n_tok = w.B * w.H * w.L
    tr = n_tok * R
    return {
        # Q read once for all rounds, one u32 key written per token-round
        "hash": {"bytes": n_tok * d * s + tr * 4, "flops": tr * d * w.n_buckets},
        # read a key, write a permutation entry
        "sort": {"bytes": tr * 8, "flops": 0},
        # gather q and v rows, the perm entry and the packed key per
        # token-round; fp32 partial (o_r, lse_r) written for rounds < R-1 and
        # read back by the combine; O and lse written once
        "attend": {"bytes": tr * (2 * d * s + 8) + 2 * n_tok * (R - 1) * (4 * d + 4)
                   + n_tok * (d * s + 4),
                   "flops": tr * 8 * w.chunk * d},
        # per token-round: perm and key, q, v and dO rows, lse and G, three
        # fp32 accumulator rows read and written once; per token: the dQ, dV
        # writes and the O, dO reads of G = dO . O, spread over R rounds
        "bwd": {"bytes": tr * (4 + 4 + 3 * d * s + 8 + 3 * 4 * d) + n_tok * (2 * d * s + 3 * 4 * d),
                "flops": tr * 20 * w.chunk * d},
    }


def load_peaks():
    if os.path.exists(PEAKS_FILE):
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def device_inputs(w: W.Workload, dev):
    inp = W.make_inputs(w)
    return {k: v.to(dev) for k, v in inp.items()}


def roofline_of(w: W.Workload, stage: str, ms: float, peaks, peak_kind, traffic=None):
    """The roofline line of one stage: algorithmic work of one launch over its
    measured time, against the stage's binding peak."""
    work = stage_work(w)[stage]
    sec = ms / 1e3
    if stage == "hash" and w.dtype == "bf16" and w.n_buckets >= 256:
        tfs = work["flops"] / sec / 1e12
        return {"bound": "tensor", "kernel": stage, "achieved": round(tfs, 2),
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": round(tfs / peaks["bf16_tflops"], 4), "traffic": traffic,
                "peak_source": peak_kind}
    gbs = work["bytes"] / sec / 1e9
    return {"bound": "hbm", "kernel": stage, "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"],
            "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4), "traffic": traffic,
            "peak_source": peak_kind}


def time_forward(w: W.Workload, steps: int, warmup: int, world: int, sample_clocks: bool = False,
                 inputs=None, after_step=None):
    """hash -> sort -> attend (with the combine) on device-resident inputs, L2
    flushed before each step; CUDA events per stage on the launching stream.
    `inputs` (device Q, V, rot) replaces the workload's own, e.g. one rank's
    heads of it; `after_step(O, lse)` runs inside each timed step, after the
    attention (its time counts with the attention's).
    Returns (total ms over the steps, per-stage ms per step, clocks, outputs)."""
    import lsh_attention_long_b200 as L
    dev = torch.device("cuda", torch.cuda.current_device())
    t = inputs if inputs is not None else device_inputs(w, dev)
    Q, V, rot = t["Q"], t["V"], t["rot"]
    R, Lx = w.n_rounds, w.L
    B, H = Q.shape[:2]
    shape = L.make_shape(B, H, Lx, w.d, w.n_buckets, R, w.chunk, w.causal, Q.dtype)
    ws = L.workspace(shape, dev)
    keys = torch.empty((R, B, H, Lx), dtype=torch.int32, device=dev)
    perm = torch.empty_like(keys)
    O = torch.empty_like(Q)
    lse = torch.empty((B, H, Lx), dtype=torch.float32, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]

    def step():
        L.lsh_hash(Q, rot, w.n_buckets, keys=keys, want_buckets=False)
        ev[1].record(stream)
        L.lsh_sort(keys, w.n_buckets, perm=perm)
        ev[2].record(stream)
        L.lsh_attend_fwd(Q, V, keys, perm, w.n_buckets, w.chunk, w.causal, O=O, lse=lse, ws=ws)
        if after_step is not None:
            after_step(O, lse)

    for _ in range(warmup):
        flush.zero_()
        ev[0].record(stream)
        step()
        ev[3].record(stream)
    torch.cuda.synchronize()
    if L.lsh_device_status() != 0:
        raise RuntimeError("device status error during warm-up")
    stage_ms = {"hash": 0.0, "sort": 0.0, "attend": 0.0}
    total_ms = 0.0
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(dev.index) if sample_clocks else _NoClocks() as clocks:
        for _ in range(steps):
            flush.zero_()
            ev[0].record(stream)
            step()
            ev[3].record(stream)
            ev[3].synchronize()
            a, b, c = ev[0].elapsed_time(ev[1]), ev[1].elapsed_time(ev[2]), ev[2].elapsed_time(ev[3])
            stage_ms["hash"] += a
            stage_ms["sort"] += b
            stage_ms["attend"] += c
            total_ms += a + b + c
        torch.cuda.synchronize()
    barrier(world)
    if L.lsh_device_status() != 0:
        raise RuntimeError("device status error in the timed region")
    total_ms = max_over_ranks(total_ms, world)
    per_stage = {k: v / steps for k, v in stage_ms.items()}
    del flush, ws
    return total_ms, per_stage, clocks.summary(), {"keys": keys, "perm": perm, "O": O, "lse": lse}


class _NoClocks:
    def __enter__(self):
        return self

    def __exit__(self, *exc):
        return False

    def summary(self):
        return None


def stage_lines(w: W.Workload, per_stage: dict, peaks) -> dict:
    work = stage_work(w)
    out = {}
    for name, ms in per_stage.items():
        sec = ms / 1e3
        gbs = work[name]["bytes"] / sec / 1e9
        tfs = work[name]["flops"] / sec / 1e12
        out[name] = {"ms": round(ms, 4), "GB_s": round(gbs, 1), "TFLOP_s": round(tfs, 2),
                     "hbm_frac": round(gbs / peaks["hbm_gbs"], 4),
                     "tensor_frac": round(tfs / peaks["bf16_tflops"], 4)}
    return out


def workload_config(w: W.Workload) -> dict:
    return {"workload": w.name, "B": w.B, "H": w.H, "L": w.L, "d": w.d,
            "n_buckets": w.n_buckets, "n_rounds": w.n_rounds, "chunk": w.chunk,
            "causal": w.causal}


def run_ours(args, world, rank):
    import lsh_attention_long_b200 as L
    L.load_library()
    w = W.WORKLOADS[args.workload]
    total_ms, per_stage, clocks, outs = time_forward(w, args.steps, args.warmup, world,
                                                     sample_clocks=True)
    ms_per_step = total_ms / args.steps
    # hash_tc, sort_rows, then key_scale + attend_tc + combine
    launches_per_step = 1 + 1 + 3
    value = aggregate_tokens_per_s(world, w.B * w.L, args.steps, total_ms)
    peaks, peak_kind = load_peaks()
    stages = stage_lines(w, per_stage, peaks)
    dom = max(per_stage, key=per_stage.get)
    roof = roofline_of(w, dom, per_stage[dom], peaks, peak_kind, TRAFFIC.get((dom, w.name)))

    result = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded Gaussian Q, V, rotations)",
        "config": workload_config(w),
        "l2": "flushed between timed steps (256 MB memset)",
        "parallelism": f"replicas x{world} (independent problems per GPU)",
        "roofline": roof, "stages": stages,
        # the same rate counted in (batch, head, position, round) units
        "head_token_rounds_per_s": round(value * w.H * w.n_rounds, 1),
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if not args.no_extras:
        result["e2e"] = run_e2e(args, w, world)
        result["fwd_bwd"] = {BWD_WORKLOAD: run_fwd_bwd(args, W.WORKLOADS[BWD_WORKLOAD], world),
                             "fwd_bf16_L65536+bwd": run_fwd_bwd(args, w, world)}
        result["workloads"] = run_other_workloads(args, w, world, peaks, peak_kind)
        result["recall"] = run_recall(args)
        result["ffn"] = run_ffn(args, world)
        result["reversible"] = run_rev(args, world)
    # the head the CPU baseline recomputes, for its parity record
    result["_head0"] = {k: v[:, :1, :1].cpu() if k in ("keys", "perm") else v[:1, :1].cpu()
                        for k, v in outs.items()}
    return result


def run_sharded(args, world, rank):
    """One problem (the workload) split over the ranks by (batch, head): rank
    k runs hash -> sort -> attend on its contiguous slice of the B*H heads;
    no data-path collective, unless --gather all-gathers O and lse inside the
    timed step.  value = the whole problem's tokens per second, timed by the
    slowest rank (strong scaling: the total work is fixed)."""
    import lsh_attention_long_b200 as L
    from lsh_attention_long_b200 import shard
    L.load_library()
    w = W.WORKLOADS[args.workload]
    dev = torch.device("cuda", torch.cuda.current_device())
    full = W.make_inputs(w)
    h0, h1 = shard.head_range(w.B * w.H, world, rank)
    t = {"Q": shard.head_slice(full["Q"], world, rank).contiguous().to(dev),
         "V": shard.head_slice(full["V"], world, rank).contiguous().to(dev),
         "rot": full["rot"].to(dev)}
    after = None
    if args.gather:
        def after(O, lse):
            shard.all_gather_heads(O, w.B, w.H, world, rank)
            shard.all_gather_heads(lse, w.B, w.H, world, rank)
    total_ms, per_stage, clocks, _ = time_forward(w, args.steps, args.warmup, world,
                                                  sample_clocks=True, inputs=t, after_step=after)
    value = w.B * w.L * args.steps / (total_ms / 1e3)
    return {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 4), "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded Gaussian Q, V, rotations)", "config": workload_config(w),
        "l2": "flushed between timed steps (256 MB memset)",
        "parallelism": f"(batch, head) shards of one problem over {world} ranks; rank 0 holds "
                       f"heads [{h0}, {h1}) of {w.B * w.H}"
                       + ("; O and lse all-gathered in the timed step" if args.gather else ""),
        "stages_rank0": {k: round(v, 4) for k, v in per_stage.items()},
        "gpu_launches": 5 * args.steps, "clocks": clocks,
    }


def run_ffn(args, world):
    """The chunked feed-forward (65 536 positions, 512 -> 2048 -> 512, chunks
    of 8192) on device-resident inputs, L2 flushed between steps: positions
    per second and the tensor-pipe roofline of its two products (4 * T *
    d_model * d_ff flops per step)."""
    import lsh_attention_long_b200 as L
    dev = torch.device("cuda", torch.cuda.current_device())
    w = W.FFN_WORKLOADS["ffn_bf16_L65536"]
    t = {k: v.to(dev) for k, v in W.ffn_inputs(w.tokens, w.d_model, w.d_ff).items()}
    Y = torch.empty_like(t["X"])
    ws = L.ffn_workspace(w.tokens, w.d_model, w.d_ff, w.chunk, dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    steps = max(5, args.steps // 2)

    def step():
        L.lsh_ffn_forward(t["X"], t["W1"], t["b1"], t["W2"], t["b2"], w.chunk, Y=Y, ws=ws)

    for _ in range(max(3, args.warmup)):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    barrier(world)
    ms = 0.0
    for _ in range(steps):
        flush.zero_()
        e0.record(stream)
        step()
        e1.record(stream)
        e1.synchronize()
        ms += e0.elapsed_time(e1)
    barrier(world)
    if L.lsh_device_status() != 0:
        raise RuntimeError("device status error in the feed-forward")
    ms = max_over_ranks(ms, world) / steps
    peaks, peak_kind = load_peaks()
    tfs = 4.0 * w.tokens * w.d_model * w.d_ff / (ms / 1e3) / 1e12
    del flush, ws
    return {"value": round(world * w.tokens / (ms / 1e3), 1), "unit": "positions/s",
            "ms_per_step": round(ms, 4), "steps": steps, "config": w.describe(),
            "launches_per_step": 2 * (w.tokens // w.chunk),
            "roofline": {"bound": "tensor", "kernel": "gemm_tc_kernel (both products)",
                         "achieved": round(tfs, 1), "peak": peaks["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": round(tfs / peaks["bf16_tflops"], 4),
                         "traffic": TRAFFIC.get(("ffn", w.name)), "peak_source": peak_kind}}


def run_rev(args, world):
    """The reversible residual block (F = LSH attention, G = chunked
    feed-forward) on one batch element of L=16384 with 8 heads of 64 (d_model
    512), 256 buckets, 4 rounds, chunk 64, causal, d_ff 2048, feed-forward
    chunks of 8192: forward and backward (inputs recomputed from the outputs)
    tokens per second, device-resident, L2 flushed between steps."""
    import lsh_attention_long_b200 as L
    dev = torch.device("cuda", torch.cuda.current_device())
    B, Lx, H, nb, R, chunk, causal, d_ff, fchunk = 1, 16384, 8, 256, 4, 64, True, 2048, 8192
    D = H * 64
    g = torch.Generator().manual_seed(30)
    X1 = torch.randn(B, Lx, D, generator=g).to(dev)
    X2 = torch.randn(B, Lx, D, generator=g).to(dev)
    dY1 = torch.randn(B, Lx, D, generator=g).to(dev)
    dY2 = torch.randn(B, Lx, D, generator=g).to(dev)
    rot = W.rotations(R, 64, nb, 1, torch.bfloat16).to(dev)
    w = tuple(v.to(dev) for k, v in W.ffn_inputs(B * Lx, D, d_ff).items()
              if k in ("W1", "b1", "W2", "b2"))
    shape = L.make_shape(B, H, Lx, 64, nb, R, chunk, causal, torch.bfloat16)
    ws = L.rev_workspace(shape, d_ff, fchunk, dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    steps = max(3, args.steps // 4)
    fwd = bwd = 0.0
    for i in range(max(3, args.warmup) + steps):
        flush.zero_()
        e[0].record(stream)
        Y1, Y2, keys, perm = L.lsh_rev_forward(X1, X2, rot, *w, H, nb, chunk, causal, fchunk,
                                               ws=ws)
        e[1].record(stream)
        L.lsh_rev_backward(Y1, Y2, dY1, dY2, keys, perm, *w, H, nb, chunk, causal, fchunk, ws=ws)
        e[2].record(stream)
        e[2].synchronize()
        if i >= max(3, args.warmup):
            fwd += e[0].elapsed_time(e[1])
            bwd += e[1].elapsed_time(e[2])
    if L.lsh_device_status() != 0:
        raise RuntimeError("device status error in the reversible block")
    fwd, bwd = max_over_ranks(fwd, world) / steps, max_over_ranks(bwd, world) / steps
    del flush, ws
    return {"value": round(world * B * Lx / ((fwd + bwd) / 1e3), 1), "unit": "tokens/s",
            "ms_fwd": round(fwd, 4), "ms_bwd": round(bwd, 4), "steps": steps,
            "fwd_tokens_per_s": round(world * B * Lx / (fwd / 1e3), 1),
            "config": {"B": B, "L": Lx, "H": H, "d_model": D, "n_buckets": nb, "n_rounds": R,
                       "chunk": chunk, "causal": causal, "d_ff": d_ff, "ffn_chunk": fchunk}}


def run_other_workloads(args, headline, world, peaks, peak_kind):
    """Forward tokens/s and the dominant stage's roofline of every other
    workload (the small fp32 one, L=4096, the clustered L=16384 and the
    fwd+bwd workload's forward), timed as the headline."""
    out = {}
    steps = max(5, args.steps // 2)
    for name, w in W.WORKLOADS.items():
        if name == headline.name:
            continue
        total_ms, per_stage, _, _ = time_forward(w, steps, max(3, args.warmup), world)
        dom = max(per_stage, key=per_stage.get)
        out[name] = {"value": round(aggregate_tokens_per_s(world, w.B * w.L, steps, total_ms), 1),
                     "unit": "tokens/s", "ms_per_step": round(total_ms / steps, 4),
                     "steps": steps, "config": workload_config(w),
                     "stages": stage_lines(w, per_stage, peaks),
                     "roofline": roofline_of(w, dom, per_stage[dom], peaks, peak_kind,
                                             TRAFFIC.get((dom, name)))}
    return out


def run_e2e(args, w, world):
    """The same forward through the public API with host buffers: one
    lsh_forward_host call takes Q, V and the rotations from pinned host
    memory and returns O and lse to pinned host memory, copying and
    computing head groups in a pipeline; all of it inside the timed region."""
    import lsh_attention_long_b200 as L
    dev = torch.device("cuda", torch.cuda.current_device())
    host = {k: v.pin_memory() for k, v in W.make_inputs(w).items()}
    shape = L.make_shape(w.B, w.H, w.L, w.d, w.n_buckets, w.n_rounds, w.chunk, w.causal,
                         host["Q"].dtype)
    ws = L.forward_host_workspace(shape, dev)
    O_host = torch.empty_like(host["Q"]).pin_memory()
    lse_host = torch.empty((w.B, w.H, w.L), dtype=torch.float32).pin_memory()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    steps = max(3, args.steps // 4)

    def step():
        L.lsh_forward_host(host["Q"], host["V"], host["rot"], w.n_buckets, w.chunk, w.causal,
                           O=O_host, lse=lse_host, ws=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier(world)
    ms = 0.0
    for _ in range(steps):
        e0.record(stream)
        step()
        e1.record(stream)
        e1.synchronize()
        ms += e0.elapsed_time(e1)
    barrier(world)
    if L.lsh_device_status() != 0:
        raise RuntimeError("device status error in the end-to-end forward")
    ms = max_over_ranks(ms, world)
    bi = sum(host[k].numel() * host[k].element_size() for k in ("Q", "V", "rot"))
    bo = O_host.numel() * O_host.element_size() + lse_host.numel() * lse_host.element_size()
    return {"value": round(aggregate_tokens_per_s(world, w.B * w.L, steps, ms), 1), "unit": "tokens/s",
            "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo, "steps": steps,
            "ms_per_step": round(ms / steps, 4), "call": "lsh_forward_host (pinned host buffers)"}


def run_fwd_bwd(args, w, world):
    """Forward + backward (dQ, dV with buckets frozen) tokens/s, device-resident."""
    import lsh_attention_long_b200 as L
    dev = torch.device("cuda", torch.cuda.current_device())
    t = device_inputs(w, dev)
    if "dO" not in t:
        t["dO"] = W.gaussian(tuple(t["Q"].shape), 2, t["Q"].dtype).to(dev)
    shape = L.make_shape(w.B, w.H, w.L, w.d, w.n_buckets, w.n_rounds, w.chunk, w.causal,
                         t["Q"].dtype)
    ws = L.workspace(shape, dev)
    out = {"keys": torch.empty((w.n_rounds, w.B, w.H, w.L), dtype=torch.int32, device=dev)}
    out["perm"] = torch.empty_like(out["keys"])
    out["O"] = torch.empty_like(t["Q"])
    out["lse"] = torch.empty((w.B, w.H, w.L), dtype=torch.float32, device=dev)
    dQ, dV = torch.empty_like(t["Q"]), torch.empty_like(t["V"])
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    steps = max(1, args.steps) if args.fwd_bwd else max(3, args.steps // 4)

    def step():
        e[0].record(stream)
        L.lsh_forward(t["Q"], t["V"], t["rot"], w.n_buckets, w.chunk, w.causal, out=out, ws=ws)
        e[1].record(stream)
        L.lsh_attend_bwd(t["Q"], t["V"], out["O"], t["dO"], out["keys"], out["perm"], out["lse"],
                         w.n_buckets, w.chunk, w.causal, dQ=dQ, dV=dV, ws=ws)
        e[2].record(stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    barrier(world)
    fwd = bwd = 0.0
    for _ in range(steps):
        flush.zero_()
        step()
        e[2].synchronize()
        fwd += e[0].elapsed_time(e[1])
        bwd += e[1].elapsed_time(e[2])
    barrier(world)
    if L.lsh_device_status() != 0:
        raise RuntimeError("device status error in fwd+bwd")
    tot = max_over_ranks(fwd + bwd, world)
    peaks, peak_kind = load_peaks()
    return {"value": round(aggregate_tokens_per_s(world, w.B * w.L, steps, tot), 1), "unit": "tokens/s",
            "ms_fwd": round(fwd / steps, 4), "ms_bwd": round(bwd / steps, 4), "steps": steps,
            "config": workload_config(w),
            # the backward call (G = dO . O, key scales, the tensor-core kernel,
            # the cast) against HBM with the algorithmic bytes of stage_work
            "roofline_bwd": roofline_of(w, "bwd", bwd / steps, peaks, peak_kind,
                                        TRAFFIC.get(("bwd", w.name)))}


# ---------------------------------------------------------------------------
# recall against full attention (a report; the pages give no number for it)
# ---------------------------------------------------------------------------

def attended_mask(keys, perm, L: int, chunk: int, causal: bool, rows, b: int, h: int):
    """[len(rows), L] bool: the keys that query positions `rows` of (b, h)
    attend to in any round.  Per round the window is the query's chunk of the
    sorted row and the previous chunk (chunk 0 wraps to the last; a single
    chunk is its own window once); a key counts when it is in the query's
    bucket, is not the query itself and, if causal, is at an earlier
    position.  keys, perm: [R, B, H, L] (packed keys bucket * L + position)."""
    R = keys.shape[0]
    dev = keys.device
    nch = L // chunk
    S = rows.numel()
    mask = torch.zeros((S, L), dtype=torch.bool, device=dev)
    offs = torch.arange(chunk, device=dev)
    for r in range(R):
        k_r = keys[r, b, h].to(torch.int64) & 0xFFFFFFFF  # original order
        p_r = perm[r, b, h].to(torch.int64)               # sorted slot -> position
        inv = torch.empty_like(p_r)
        inv[p_r] = torch.arange(L, device=dev)
        ck = inv[rows] // chunk
        if nch > 1:
            prev = (ck - 1) % nch
            win = torch.cat([prev[:, None] * chunk + offs, ck[:, None] * chunk + offs], 1)
        else:
            win = ck[:, None] * chunk + offs
        tok = p_r[win]
        ok = (k_r[tok] // L == (k_r[rows] // L)[:, None]) & (tok != rows[:, None])
        if causal:
            ok &= tok < rows[:, None]
        qi = torch.arange(S, device=dev)[:, None].expand_as(tok)
        mask[qi[ok], tok[ok]] = True
    return mask


def full_attention_recall(Q, keys, perm, chunk: int, causal: bool, rows, b: int, h: int,
                          topk: int = 0):
    """Per query: the share of full shared-QK attention's probability mass
    (softmax of q_i . khat_j / sqrt(d) over every other key, earlier ones if
    causal) that falls on keys LSH attention sees in some round; with topk > 0
    instead the share of the query's topk highest-scoring keys that it sees.
    fp64.  Queries with no key at all (the first position, causal) are
    dropped."""
    q = Q[b, h].to(torch.float64)
    L, d = q.shape
    n = q.norm(dim=1, keepdim=True)
    khat = torch.where(n > 0, q / torch.where(n > 0, n, torch.ones_like(n)), torch.zeros_like(q))
    s = (q[rows] @ khat.T) / math.sqrt(d)
    cols = torch.arange(L, device=q.device)[None, :]
    allowed = cols != rows[:, None]
    if causal:
        allowed &= cols < rows[:, None]
    s = s.masked_fill(~allowed, float("-inf"))
    keep = allowed.any(1)
    seen = attended_mask(keys, perm, L, chunk, causal, rows, b, h)[keep]
    if topk > 0:
        k = min(topk, L - 1)
        idx = s[keep].topk(k, dim=1).indices
        return seen.gather(1, idx).to(torch.float64).mean(1)
    p = torch.softmax(s[keep], dim=1)
    return (p * seen).sum(1)


def run_recall(args):
    """Recall against full attention over rounds (R = 1, 2, 4, 8 at nb = 256)
    and bucket counts (nb = 64, 256, 1024 at R = 4) on the clustered
    L = 16384 workload, with the forward's time for each setting."""
    import lsh_attention_long_b200 as L
    L.load_library()
    dev = torch.device("cuda", torch.cuda.current_device())
    base = W.WORKLOADS["fwd_bf16_L16384_clustered"]
    inp = W.make_inputs(base)
    Q, V = inp["Q"].to(dev), inp["V"].to(dev)
    g = torch.Generator(device="cpu")
    g.manual_seed(7)
    rows = torch.randperm(base.L, generator=g)[:4096].sort().values.to(dev)
    out = []
    for R, nb in [(1, 256), (2, 256), (4, 256), (8, 256), (4, 64), (4, 1024)]:
        rot = W.rotations(R, base.d, nb, 1, Q.dtype).to(dev)
        res = L.lsh_forward(Q, V, rot, nb, base.chunk, base.causal)
        torch.cuda.synchronize()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        for _ in range(3):
            L.lsh_forward(Q, V, rot, nb, base.chunk, base.causal, out=res)
        ev[0].record()
        for _ in range(10):
            L.lsh_forward(Q, V, rot, nb, base.chunk, base.causal, out=res)
        ev[1].record()
        torch.cuda.synchronize()
        ms = ev[0].elapsed_time(ev[1]) / 10
        rec = torch.cat([full_attention_recall(Q, res["keys"], res["perm"], base.chunk,
                                               base.causal, rows, b, 0) for b in range(base.B)])
        top = torch.cat([full_attention_recall(Q, res["keys"], res["perm"], base.chunk,
                                               base.causal, rows, b, 0, topk=32)
                         for b in range(base.B)])
        out.append({"n_rounds": R, "n_buckets": nb, "chunk": base.chunk,
                    "recall_top32": round(float(top.mean()), 4),
                    "mass_recall": round(float(rec.mean()), 4),
                    "fwd_ms": round(ms, 4),
                    "tokens_per_s": round(base.B * base.L / (ms / 1e3), 1)})
    if L.lsh_device_status() != 0:
        raise RuntimeError("device status error in the recall sweep")
    return {"report": "recall vs full attention", "workload": base.name,
            "sample": "4096 query positions (seed 7) of head 0 in each batch element; fp64 "
                      "full attention over every other key; recall_top32 = share of each "
                      "query's 32 highest-scoring keys (about one cluster: 16384 tokens, "
                      "512 centres) seen in some round; mass_recall = share of the full "
                      "softmax mass seen (near-uniform here: unit-norm queries give scores "
                      "within +-1/8)",
            "sweep": out}


# DRAM bytes per launch from ncu (dram__bytes_read.sum + dram__bytes_write.sum)
# for the kernels as they stand, keyed by (stage, workload); absent until
# taken, and to be cleared whenever a kernel changes.  A stage's figure covers
# the launches its time covers: the attention call is fwd_prep_kernel +
# attend_tc_kernel + combine16_kernel.  Each is from one capture of the
# workload's timed step (profiles/launches_fwd_bf16_L65536.md).
TRAFFIC = {
    ("hash", "fwd_bf16_L65536"): 67661824 + 2908928,
    ("attend", "fwd_bf16_L65536"): (134232576 + 31965440) + (182373888 + 497529344)
                                   + (553657856 + 57975808),
    ("attend", "fwdbwd_bf16_L16384"): (67115264 + 6037504) + (77978368 + 85642240)
                                      + (138419712 + 14423552),
}


# ---------------------------------------------------------------------------
# CPU oracle (the reference arm and the cpu_baseline leg)
# ---------------------------------------------------------------------------

class OracleSampler:
    """Times the fp64 CPU oracle (single thread, as it stands) on a bounded
    sample of a workload and scales each stage to the whole step.

    Setup (untimed): the oracle hashes one full row (head 0, round 0) so that
    the sort and attention samples have real keys.  A timed sample is then:
    the oracle's hash of `n_tok` tokens of head 0 for round 0, its sort of
    that row, its attention for the queries of `n_chunks` chunks of that row,
    and its combine over `n_tok` tokens.  Each stage's time is scaled by the
    number of such units in the whole step (B*H*L*R tokens hashed, B*H*R rows
    sorted, B*H*R*L/c chunks attended, B*H*L tokens combined)."""

    def __init__(self, w: W.Workload):
        from oracle import oracle as cpu_oracle
        import numpy as np
        cpu_oracle.build()
        self.o, self.np, self.w = cpu_oracle, np, w
        inp = W.make_inputs(w)
        self.Q = inp["Q"][:1, :1].float().numpy()
        self.V = inp["V"][:1, :1].float().numpy()
        self.rot = inp["rot"][:1].float().numpy()
        self.keys, _, _ = cpu_oracle.lsh_hash(self.Q, self.rot, w.n_buckets)
        self.perm = cpu_oracle.lsh_sort(self.keys)

    def step(self, n_tok: int, n_chunks: int):
        w, o, np = self.w, self.o, self.np
        t0 = time.perf_counter()
        o.lsh_hash(self.Q[:, :, :n_tok], self.rot, w.n_buckets)
        t1 = time.perf_counter()
        o.lsh_sort(self.keys)
        t2 = time.perf_counter()
        o.lsh_attend_fwd_range(self.Q, self.V, self.keys, self.perm, w.chunk, w.causal, 0,
                               n_chunks)
        t3 = time.perf_counter()
        part = np.zeros((w.n_rounds, 1, 1, n_tok, w.d))
        o.lsh_combine(part, np.zeros((w.n_rounds, 1, 1, n_tok)))
        t4 = time.perf_counter()
        rows = w.B * w.H * w.n_rounds
        full = ((t1 - t0) / n_tok * w.B * w.H * w.L * w.n_rounds
                + (t2 - t1) * rows
                + (t3 - t2) / n_chunks * rows * (w.L // w.chunk)
                + (t4 - t3) / n_tok * w.B * w.H * w.L)
        return t4 - t0, full

    def describe(self, n_tok, n_chunks):
        w = self.w
        return (f"{w.name}: oracle hash of {n_tok} tokens (head 0, round 0), sort of one "
                f"{w.L}-token row, attention for {n_chunks} chunks of that row, combine of "
                f"{n_tok} tokens; each stage scaled by its unit count to the whole step "
                f"(B*H*L*R hashes, B*H*R rows, B*H*R*L/c chunks); single-threaded fp64")


def host_cpu() -> dict:
    """The host's CPU model name and logical core count, for the baseline lines."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"cpu_model": model, "nproc": os.cpu_count()}


def run_cpu_baseline(w, head0=None):
    """The oracle as it stands on one whole head (b=0, h=0) of the workload:
    hash, sort, attention and combine for all rounds, scaled by B*H.  With the
    GPU's outputs for that head (head0), the oracle's results also give a
    parity record outside the timed region: near ties among the head's hashes,
    bucket ids and permutations that differ, and the largest errors of O and
    lse (the oracle's attention fed the GPU's keys and permutations)."""
    from oracle import oracle as cpu_oracle
    cpu_oracle.build()
    import numpy as np
    inp = W.make_inputs(w)
    Q = inp["Q"][:1, :1].float().numpy()
    V = inp["V"][:1, :1].float().numpy()
    rot = inp["rot"].float().numpy()
    t0 = time.perf_counter()
    ref = cpu_oracle.lsh_forward(Q, V, rot, w.n_buckets, w.chunk, w.causal)
    sec = time.perf_counter() - t0
    full = sec * w.B * w.H
    res = {"value": round(w.B * w.L / full, 3), "unit": "tokens/s", "cores": 1,
           "kind": "oracle", **host_cpu(),
           "sample": f"one head (b=0, h=0) of {w.name}, all {w.n_rounds} rounds, full "
                     f"L={w.L}: hash, sort, attention, combine in {sec:.1f} s single-threaded "
                     f"fp64; scaled by B*H={w.B * w.H} to the whole step"}
    if head0 is not None:
        keys = head0["keys"].numpy().view(np.uint32)
        perm = head0["perm"].numpy()
        gb = keys // np.uint32(w.L)
        tie = ref["near_tie"] != 0
        diff = gb != ref["buckets"]
        o_part, lse_r = cpu_oracle.lsh_attend_fwd(Q, V, keys, perm, w.chunk, w.causal)
        O, lse = cpu_oracle.lsh_combine(o_part, lse_r)
        res["parity_head0"] = {
            "tokens_hashed": int(keys.size), "near_ties": int(tie.sum()),
            "bucket_mismatch_outside_near_ties": int((diff & ~tie).sum()),
            "near_tie_flips": int((diff & tie).sum()),
            "perm_equal_to_oracle_sort_of_gpu_keys": bool(np.array_equal(perm,
                                                                         cpu_oracle.lsh_sort(keys))),
            "O_max_abs": float(np.abs(head0["O"].float().numpy() - O).max()),
            "lse_max_abs": float(np.abs(head0["lse"].numpy() - lse).max()),
            "tol": 2e-2 if w.dtype == "bf16" else 2e-3}
    return res


def run_cpu_baseline_threads(w):
    """The same oracle, with the independent (b, h) heads of the step spread
    over host threads (one head per thread, at most one thread per core).  The
    oracle's C routines release the GIL, so the threads run in parallel.  With
    fewer cores than heads, as many heads as cores run and the time is scaled
    by the number of heads over that."""
    from concurrent.futures import ThreadPoolExecutor
    from oracle import oracle as cpu_oracle
    cpu_oracle.build()
    inp = W.make_inputs(w)
    BH = w.B * w.H
    n = max(1, min(BH, os.cpu_count() or 1))
    heads = [(i // w.H, i % w.H) for i in range(n)]
    Qs = [inp["Q"][b:b + 1, h:h + 1].float().numpy() for b, h in heads]
    Vs = [inp["V"][b:b + 1, h:h + 1].float().numpy() for b, h in heads]
    rot = inp["rot"].float().numpy()
    with ThreadPoolExecutor(max_workers=n) as pool:
        t0 = time.perf_counter()
        list(pool.map(lambda i: cpu_oracle.lsh_forward(Qs[i], Vs[i], rot, w.n_buckets, w.chunk,
                                                       w.causal), range(n)))
        sec = time.perf_counter() - t0
    full = sec * BH / n
    return {"value": round(w.B * w.L / full, 3), "unit": "tokens/s", "cores": n,
            "kind": "oracle", **host_cpu(),
            "sample": f"{n} of the {BH} heads of {w.name}, one per thread, all {w.n_rounds} "
                      f"rounds, full L={w.L}: hash, sort, attention, combine in {sec:.1f} s "
                      f"fp64; scaled by {BH}/{n} to the whole step"}


def run_reference(args, world, rank):
    w = W.WORKLOADS[args.workload]
    if rank != 0:
        return None
    s = OracleSampler(w)
    # a few minutes in all: about --ref-seconds of sampling over warm-up + timed steps
    per_step = args.ref_seconds / (args.warmup + args.steps)
    max_chunks = w.L // w.chunk
    probe_tok, probe_chunks = min(256, w.L), min(4, max_chunks)
    probe, _ = s.step(probe_tok, probe_chunks)
    scale = max(1.0, min(32.0, per_step / max(probe, 1e-3)))
    n_tok = min(int(probe_tok * scale), w.L)
    n_chunks = min(max(1, int(probe_chunks * scale)), max_chunks)
    full = []
    for i in range(args.warmup + args.steps):
        _, f = s.step(n_tok, n_chunks)
        if i >= args.warmup:
            full.append(f)
    per = sum(full) / len(full)
    value = w.B * w.L / per
    sample = s.describe(n_tok, n_chunks)
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(per * 1e3, 1), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w),
        "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": 1,
                         "kind": "oracle", "sample": sample, **host_cpu()},
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    args = parse_args()
    if args.heads > 0:
        w = W.WORKLOADS[args.workload]
        w = dataclasses.replace(w, H=args.heads, name=f"{w.name}_H{args.heads}")
        W.WORKLOADS[w.name] = w
        args.workload = w.name
    if args.impl == "reference":
        # the CPU oracle runs on rank 0 only; other ranks exit without work
        if int(os.environ.get("RANK", "0")) != 0:
            return
        res = run_reference(args, int(os.environ.get("WORLD_SIZE", "1")), 0)
        print(json.dumps(res), flush=True)
        return
    world, rank, _ = dist_setup(args.gpus)
    try:
        if not torch.cuda.is_available():
            raise SystemExit("bench.py needs a CUDA device for --impl ours")
        if args.recall:
            if rank == 0:
                print(json.dumps(run_recall(args)), flush=True)
            return
        if args.fwd_bwd:
            res = {"workload": args.workload,
                   "fwd_bwd": run_fwd_bwd(args, W.WORKLOADS[args.workload], world)}
            if rank == 0:
                print(json.dumps(res), flush=True)
            return
        if args.ffn or args.rev:
            res = {}
            if args.ffn:
                res["ffn"] = run_ffn(args, world)
            if args.rev:
                res["reversible"] = run_rev(args, world)
            if rank == 0:
                print(json.dumps(res), flush=True)
            return
        if args.shard == "heads":
            res = run_sharded(args, world, rank)
            if rank == 0:
                print(json.dumps(res), flush=True)
            return
        res = run_ours(args, world, rank)
        head0 = res.pop("_head0")
        if rank == 0 and not args.no_extras and world == 1:
            res["cpu_baseline"] = run_cpu_baseline(W.WORKLOADS[args.workload], head0)
            res["cpu_baseline_threads"] = run_cpu_baseline_threads(W.WORKLOADS[args.workload])
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
