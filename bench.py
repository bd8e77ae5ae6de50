"""HSTU jagged attention forward benchmark on B200.

Workload (default): the 8-layer HSTU stack workload at sequence lengths up to
8,320 -- 8 users with lengths uniform in [4160, 8320], 4 heads, d = 128,
N_max = 8320, causal mask, per-layer rab tables and Q/K/V/U, bf16 inputs.
One step = the attention forward (validate + tile schedule, tcgen05 attention,
LayerNorm-gate epilogue) of all 8 layers.  The metric is attention TFLOP/s
(algorithmic: 2 (d_qk + d_v) flops per allowed (query, key) pair and head),
with tokens/s alongside.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU: one process per GPU (torchrun); users are independent, so every
rank runs its own batch with no collective on the data path (weak scaling);
timing is the max over ranks.  --impl reference times the fp64 CPU oracle on
the host cores on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

FLOPS_PER_PAIR_HEAD = 2 * (128 + 128)  # QK^T and AV, d_qk = d_v = 128
TILE = 128
# dram__bytes_read.sum + dram__bytes_write.sum of one attention-kernel launch
# (layer 0 of the 8-layer stack workload) and of one paged attention launch,
# each from a single-launch capture on a B200:
#   ncu --set full --clock-control none -k regex:attn_sm100_kernel -s 2 -c 1 \
#       python bench.py --only stack --steps 2 --warmup 3 --e2e-steps 0 --no-cpu-baseline --layers 1
#   ncu --set full --clock-control none -k regex:attn_sm100_single -s 10 -c 1 \
#       python bench.py --only paged --steps 3 --warmup 3
# None whenever the kernel has changed since its counters were taken.
ATTN_TRAFFIC_BYTES = 394_607_616 + 36_452_352
PAGED_TRAFFIC_BYTES = 114_908_672 + 4_225_024


def allowed_pairs(lengths, cands=None):
    """Allowed (query, key) pairs per head: h(h+1)/2 causal history pairs plus,
    per candidate, the h history keys and itself."""
    total = 0
    for i, n in enumerate(lengths):
        c = 0 if cands is None else int(cands[i])
        h = int(n) - c
        total += h * (h + 1) // 2 + c * (h + 1)
    return total


def issued_tiles(lengths, cands=None):
    """128x128 key tiles the tensor-core kernel issues (both GEMMs), per head."""
    tiles = 0
    for i, n in enumerate(lengths):
        c = 0 if cands is None else int(cands[i])
        h = int(n) - c
        for m in range(math.ceil(int(n) / TILE)):
            q_last = min(int(n), (m + 1) * TILE) - 1
            kv_end = max(0, min(q_last + 1, h))
            tiles += math.ceil(kv_end / TILE)
    return tiles


def max_sm_mhz(device_index: int = 0) -> int:
    """clocks.max.sm from nvidia-smi (1965 MHz on this part if it cannot be read)."""
    try:
        out = subprocess.run(["nvidia-smi", "-i", str(device_index), "--query-gpu=clocks.max.sm",
                              "--format=csv,noheader,nounits"], capture_output=True, text=True, timeout=10)
        return int(out.stdout.strip().splitlines()[0])
    except Exception:
        return 1965


class ClockSampler:
    """SM clock and throttle reasons sampled during the timed region: NVML from a
    background thread every 10 ms (read-only queries), else nvidia-smi every
    100 ms.  stop() returns the median SM clock, the maximum, the reasons seen
    and the sample count."""

    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        import threading
        self.proc = None
        self.thread = None
        self.samples = []
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            bits = {"hw_slowdown": pynvml.nvmlClocksEventReasonHwSlowdown,
                    "hw_thermal_slowdown": pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                    "sw_thermal_slowdown": pynvml.nvmlClocksEventReasonSwThermalSlowdown,
                    "sw_power_cap": pynvml.nvmlClocksEventReasonSwPowerCap}
            self.stop_flag = threading.Event()

            def run():
                while not self.stop_flag.is_set():
                    try:
                        mhz = float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
                        rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                        self.samples.append((mhz, {n for n, b in bits.items() if rs & b}))
                    except Exception:
                        pass
                    self.stop_flag.wait(0.01)
            self.thread = threading.Thread(target=run, daemon=True)
            self.thread.start()
            return
        except Exception:
            self.thread = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(device_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.thread is not None:
            self.stop_flag.set()
            self.thread.join(timeout=2)
            if not self.samples:
                return None
            sm = [m for m, _ in self.samples]
            reasons = set().union(*(r for _, r in self.samples))
            return {"sm_mhz": statistics.median(sm), "sm_max_mhz": self.max_mhz or max(sm),
                    "reasons": sorted(reasons), "samples": len(sm), "source": "nvml, 10 ms"}
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        for line in out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(self.NAMES, parts[4:8]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm), "source": "nvidia-smi, 100 ms"}


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    # an earlier measurement on this part: 6.65 TB/s copy, 1.59 PFLOP/s bf16 GEMM in
    # a burst, settling near 1.4 PFLOP/s under the 1 kW power cap
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def pick_bf16_peak(peaks, clk):
    """The bf16 tensor peak that applies to a timed region: the burst figure when
    the SM clock sampled during the region stayed near its maximum (median at
    95% of it or more), else the sustained one (a long region that the power
    cap slowed)."""
    burst = float(peaks["bf16_tflops"])
    sustained = float(peaks.get("bf16_tflops_sustained", burst))
    if clk is None:
        return burst, "burst (no clock samples)"
    # the clock the region actually ran at decides: a power-cap flag in some
    # samples while the median clock held near its maximum still means burst
    hot = clk["sm_mhz"] >= 0.95 * clk["sm_max_mhz"]
    cap = ", sw_power_cap seen" if "sw_power_cap" in clk["reasons"] else ", no power cap"
    if hot:
        return burst, f"burst (median {clk['sm_mhz']:.0f} of {clk['sm_max_mhz']:.0f} MHz{cap})"
    return sustained, f"sustained (median {clk['sm_mhz']:.0f} of {clk['sm_max_mhz']:.0f} MHz, {clk['reasons']})"


def tensor_roofline(kernel, flops_per_launch, launch_ms, clk, traffic=None, issued_flops=None):
    """Roofline of a tensor-bound kernel from its per-launch CUDA-event times
    (median and spread) against the measured bf16 peak that fits the clocks."""
    peaks, kind = measured_peaks()
    med = float(np.median(launch_ms))
    achieved = flops_per_launch / (med * 1e-3) / 1e12
    peak, which = pick_bf16_peak(peaks, clk)
    r = {"kernel": kernel, "bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
         "frac": round(achieved / peak, 4), "peak_source": f"{kind} bf16_tflops, {which}",
         "frac_of_burst": round(achieved / float(peaks["bf16_tflops"]), 4),
         "frac_of_sustained": round(achieved / float(peaks.get("bf16_tflops_sustained",
                                                                 peaks["bf16_tflops"])), 4),
         "traffic": traffic, "launch_ms": round(med, 4),
         "launch_ms_p10_p90": [round(float(np.percentile(launch_ms, 10)), 4),
                               round(float(np.percentile(launch_ms, 90)), 4)],
         "launches_timed": len(launch_ms), "flops_per_launch": flops_per_launch, "statistic": "median"}
    if issued_flops is not None:
        itf = issued_flops / (med * 1e-3) / 1e12
        r["issued_tile_tflops"] = round(itf, 2)
        r["issued_frac"] = round(itf / peak, 4)
    return r


# ----------------------------------------------------------------------------
# CPU oracle baseline (bounded sample)
# ----------------------------------------------------------------------------

def oracle_sample(batch, target_s: float, seed: int = 0):
    """Time the fp64 oracle on random query rows of `batch` for about target_s."""
    import oracle
    rng = np.random.default_rng(seed)
    lengths = batch.lengths
    off = batch.seq_offsets
    # inputs converted to fp64 once, outside the timed calls
    q64, k64, v64, u64 = (t.double().numpy() for t in (batch.q, batch.k, batch.v, batch.u))
    # per-row keys of a causal row i: i + 1
    def run(nrows):
        users = rng.integers(0, batch.batch, size=nrows)
        rows = np.array([off[usr] + rng.integers(0, lengths[usr]) for usr in users], dtype=np.int64)
        keys = 0
        for r, usr in zip(rows, users):
            i = r - off[usr]
            c = 0 if batch.num_candidates is None else int(batch.num_candidates[usr])
            h = lengths[usr] - c
            keys += (i + 1) if i < h else (h + 1)
        t0 = time.perf_counter()
        oracle.attn_jagged(q64, k64, v64, u64, batch.seq_offsets, batch.timestamps, batch.num_candidates,
                           batch.rab_pos, batch.rab_ts, batch.alpha, batch.n_max, rows=rows)
        return time.perf_counter() - t0, keys * batch.num_heads * FLOPS_PER_PAIR_HEAD, nrows
    dt, _, _ = run(8)  # warm-up
    dt, flops, nrows = run(16)
    n = int(max(16, min(20000, 16 * target_s / max(dt, 1e-3))))
    dt, flops, nrows = run(n)
    return dt, flops, nrows


# ----------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------

def to_dev(x, dtype=None, device="cuda"):
    if x is None:
        return None
    if isinstance(x, np.ndarray):
        x = torch.from_numpy(np.ascontiguousarray(x))
    return x.to(device=device, dtype=dtype) if dtype is not None else x.to(device)


def rank_seed(rank: int):
    """Seed of a rank's users: rank 0 draws the workload's own users, every other
    rank a distinct set (weak scaling: the same amount of work per rank)."""
    return None if rank == 0 else 1000 + 7919 * rank


def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's time: every rank contributes its own, all get the max."""
    if world <= 1:
        return ms
    t = torch.tensor([ms], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job(flops_per_rank_step: float, tokens_per_rank_step: float, world: int, ms_step: float):
    """Whole-job throughput: all ranks' work over the slowest rank's step time."""
    return (flops_per_rank_step * world / (ms_step * 1e-3) / 1e12,
            tokens_per_rank_step * world / (ms_step * 1e-3))


WORKLOAD_TEXT = {
    "stack8_bf16": "8-layer HSTU attention, B=8 users, lengths U[4160,8320], H=4, d=128, N_max=8320, causal",
    "stack8_n8192": "8-layer HSTU attention, B=8 users, all lengths 8192, H=4, d=128, N_max=8320, causal",
    "mfalcon_bf16": "M-FALCON ranking, 2 layers, B=16 users, history U[2048,4096] + 512 candidates each "
                    "(candidates see the history and themselves), H=4, d=128, N_max=4608",
}
MIN_ROOFLINE_LAUNCHES = 56


def time_attention_stack(workload, args, rank, world, device, *, steps, warmup, e2e_steps=0, layers=None):
    """One step = the attention forward (plan, tcgen05 attention, LayerNorm-gate
    epilogue) of every layer of `workload` on per-layer inputs.  Returns the
    whole-job throughput of `steps` timed steps, the attention kernel's
    roofline from per-launch events and, with e2e_steps, the same step end to
    end from pinned host buffers."""
    import generative_recommender_attention_jagged_b200 as hstu
    from generative_recommender_attention_jagged_b200 import _lib

    seed = rank_seed(rank)  # every rank its own users
    stack = synth.attention_stack(workload, num_layers=layers, seed=seed)
    L = len(stack)
    b0 = stack[0]
    T, H, d = b0.q.shape
    stream = torch.cuda.current_stream()
    dev_layers = []
    for b in stack:
        dev_layers.append(dict(q=to_dev(b.q), k=to_dev(b.k), v=to_dev(b.v), u=to_dev(b.u),
                               rab_pos=to_dev(b.rab_pos, torch.float32), rab_ts=to_dev(b.rab_ts, torch.float32)))
    off = to_dev(b0.seq_offsets, torch.int32)
    ts = to_dev(b0.timestamps, torch.int64)
    cand = to_dev(b0.num_candidates, torch.int32)
    params = hstu.attn_params(batch=b0.batch, num_heads=H, head_dim=d, n_max=b0.n_max, total_tokens=T,
                              max_seq_len=b0.max_seq_len, dtype=b0.q.dtype, alpha=b0.alpha)
    ws_bytes = hstu.hstu_attn_workspace_size(params)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=device)
    outs = [torch.empty(T, H * d, dtype=b0.q.dtype, device=device) for _ in range(L)]

    def call(l, stage):
        x = dev_layers[l]
        return hstu.hstu_attn_fwd(x["q"], x["k"], x["v"], x["u"], off, ts, x["rab_pos"], x["rab_ts"],
                                  n_max=b0.n_max, alpha=b0.alpha, num_candidates=cand,
                                  max_seq_len=b0.max_seq_len, out=outs[l], workspace=ws, stages=stage)

    def step(ev_attn=None, ev_step=None):
        if ev_step is not None:
            ev_step[0].record(stream)
        for l in range(L):
            call(l, _lib.F_STAGE_PLAN)
            if ev_attn is not None:
                ev_attn[l][0].record(stream)
            call(l, _lib.F_STAGE_ATTN)
            if ev_attn is not None:
                ev_attn[l][1].record(stream)
            call(l, _lib.F_STAGE_EPILOGUE)
        if ev_step is not None:
            ev_step[1].record(stream)

    new_ev = lambda: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    status = hstu.hstu_check_device_error(ws)
    if status != 0:
        raise RuntimeError(f"device status {status} ({hstu.hstu_status_string(status)})")

    ev_attn = [[new_ev() for _ in range(L)] for _ in range(steps)]
    ev_step = [new_ev() for _ in range(steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(device.index if device.index is not None else 0)
    t0, t1 = new_ev()
    t0.record(stream)
    for s in range(steps):
        step(ev_attn[s], ev_step[s])
    t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    total_ms = max_over_ranks(t0.elapsed_time(t1), world, device)
    attn_ms = [a.elapsed_time(b) for row in ev_attn for a, b in row]
    step_ms = [a.elapsed_time(b) for a, b in ev_step]
    # the roofline statistic wants at least MIN_ROOFLINE_LAUNCHES launches: short
    # runs add untimed-in-`value` passes of the same steps
    while len(attn_ms) < MIN_ROOFLINE_LAUNCHES:
        extra = [new_ev() for _ in range(L)]
        step(extra)
        torch.cuda.synchronize()
        attn_ms += [a.elapsed_time(b) for a, b in extra]
    status = hstu.hstu_check_device_error(ws)
    if status != 0:
        raise RuntimeError(f"device status {status} ({hstu.hstu_status_string(status)})")

    lengths = b0.lengths
    pairs = allowed_pairs(lengths, b0.num_candidates)
    flops_layer = pairs * H * FLOPS_PER_PAIR_HEAD
    flops_step = flops_layer * L
    ms_step = total_ms / steps
    value, tokens_s = whole_job(flops_step, T * L, world, ms_step)
    tiles = issued_tiles(lengths, b0.num_candidates) * H
    issued = tiles * 2 * (2 * TILE * TILE * 128)
    traffic = ATTN_TRAFFIC_BYTES if (workload == "stack8_bf16" and ATTN_TRAFFIC_BYTES) else None
    roof = tensor_roofline("attn_sm100_kernel", flops_layer, attn_ms, clk, traffic=traffic, issued_flops=issued)

    e2e = None
    if e2e_steps > 0:
        e2e = time_e2e(stack, b0, hstu, ws, world, device, stream, e2e_steps, flops_step)
    return {"value": value, "tokens_per_s": tokens_s, "ms_per_step": ms_step,
            "ms_per_step_median": float(np.median(step_ms)),
            "ms_per_step_p10_p90": [float(np.percentile(step_ms, 10)), float(np.percentile(step_ms, 90))],
            "roofline": roof, "clocks": clk, "e2e": e2e, "b0": b0, "T": T, "H": H, "d": d, "L": L,
            "flops_step": flops_step, "launches": steps * L * 3}


def time_e2e(stack, b0, hstu, ws, world, device, stream, e2e_steps, flops_step):
    """The stack end to end through the C ABI from pinned host buffers: each
    layer's inputs copy in (host to device) and its Y copies out (device to
    host) inside the timed region, pipelined as a caller would run it."""
    L = len(stack)
    T, H, d = b0.q.shape
    host = []
    for b in stack:
        host.append({k: (v.pin_memory() if isinstance(v, torch.Tensor) else torch.from_numpy(v).pin_memory())
                     for k, v in dict(q=b.q, k=b.k, v=b.v, u=b.u, rab_pos=b.rab_pos, rab_ts=b.rab_ts).items()})
    h_off = torch.from_numpy(b0.seq_offsets.astype(np.int32)).pin_memory()
    h_ts = torch.from_numpy(b0.timestamps).pin_memory()
    h_cand = None if b0.num_candidates is None else torch.from_numpy(b0.num_candidates.astype(np.int32)).pin_memory()
    h_out = [torch.empty(T, H * d, dtype=b0.q.dtype).pin_memory() for _ in range(L)]
    # two device input sets and two output buffers: layer l + 1's inputs copy
    # in on one stream while layer l computes, and each output copies out on a
    # third stream (host-to-device and device-to-host run at once)
    d_in = [{k: torch.empty_like(v, device=device) for k, v in host[0].items()} for _ in range(2)]
    d_off = torch.empty_like(h_off, device=device)
    d_ts = torch.empty_like(h_ts, device=device)
    d_cand = None if h_cand is None else torch.empty_like(h_cand, device=device)
    d_out = [torch.empty(T, H * d, dtype=b0.q.dtype, device=device) for _ in range(2)]
    s_h2d, s_d2h = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev_in = [torch.cuda.Event() for _ in range(2)]     # inputs of buffer set j landed
    ev_used = [torch.cuda.Event() for _ in range(2)]   # compute done with buffer set j
    ev_out = [torch.cuda.Event() for _ in range(2)]    # output buffer j copied out
    for j in range(2):
        ev_used[j].record(stream)
        ev_out[j].record(stream)
    h2d = d2h = 0

    def e2e_step(count):
        nonlocal h2d, d2h
        with torch.cuda.stream(s_h2d):
            s_h2d.wait_stream(stream)
            d_off.copy_(h_off, non_blocking=True)
            d_ts.copy_(h_ts, non_blocking=True)
            if d_cand is not None:
                d_cand.copy_(h_cand, non_blocking=True)
        if count:
            h2d += h_off.numel() * 4 + h_ts.numel() * 8 + (0 if h_cand is None else h_cand.numel() * 4)
        for l in range(L):
            j = l % 2
            with torch.cuda.stream(s_h2d):
                s_h2d.wait_event(ev_used[j])
                for k_, v_ in host[l].items():
                    d_in[j][k_].copy_(v_, non_blocking=True)
                    if count:
                        h2d += v_.numel() * v_.element_size()
                ev_in[j].record(s_h2d)
            stream.wait_event(ev_in[j])
            stream.wait_event(ev_out[j])
            x = d_in[j]
            hstu.hstu_attn_fwd(x["q"], x["k"], x["v"], x["u"], d_off, d_ts, x["rab_pos"], x["rab_ts"],
                               n_max=b0.n_max, alpha=b0.alpha, num_candidates=d_cand,
                               max_seq_len=b0.max_seq_len, out=d_out[j], workspace=ws)
            ev_used[j].record(stream)
            with torch.cuda.stream(s_d2h):
                s_d2h.wait_event(ev_used[j])
                h_out[l].copy_(d_out[j], non_blocking=True)
                ev_out[j].record(s_d2h)
            if count:
                d2h += d_out[j].numel() * d_out[j].element_size()
        # the step ends when its last output is on the host
        stream.wait_stream(s_d2h)
        stream.wait_stream(s_h2d)

    e2e_step(False)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step(True)
    e1.record(stream)
    torch.cuda.synchronize()
    e_ms = max_over_ranks(e0.elapsed_time(e1), world, device)
    e_step = e_ms / e2e_steps
    return {"value": round(whole_job(flops_step, T * L, world, e_step)[0], 3), "unit": "TFLOP/s",
            "ms_per_step": round(e_step, 3), "steps": e2e_steps,
            "h2d_bytes_per_step": h2d // e2e_steps, "d2h_bytes_per_step": d2h // e2e_steps}


def run_ours(args, rank, world, device):
    r = time_attention_stack(args.workload, args, rank, world, device, steps=args.steps, warmup=args.warmup,
                             e2e_steps=args.e2e_steps, layers=args.layers)
    b0, T, H, d, L = r["b0"], r["T"], r["H"], r["d"], r["L"]
    result = {
        "metric": "HSTU attention fwd TFLOP/s + tokens/s, % of B200 BF16 peak / HBM BW",
        "value": round(r["value"], 3),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(r["ms_per_step"], 4),
        "ms_per_step_median": round(r["ms_per_step_median"], 4),
        "ms_per_step_p10_p90": [round(x, 4) for x in r["ms_per_step_p10_p90"]],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded; no dataset)",
        "config": {"workload": f"{args.workload}: {WORKLOAD_TEXT[args.workload]} (T={T})",
                   "global_batch": b0.batch * world, "total_tokens_per_gpu": T, "layers": L,
                   "parallelism": f"replicas x{world} (users sharded, no collective)",
                   "l2": "inputs larger than L2 (%d per-layer Q/K/V/U sets, %.2f GB)" %
                         (L, 4 * T * H * d * 2 * L / 1e9)},
        "tokens_per_s": round(r["tokens_per_s"], 1),
        "roofline": r["roofline"],
        "gpu_launches": r["launches"],  # per layer: plan, attention, epilogue
        "clocks": r["clocks"],
        "e2e": r["e2e"],
    }
    return result, b0


def run_config_line(workload, args, device):
    """A per-config line: the attention stack of `workload` at 1 GPU with its
    roofline, clocks and an oracle sample on the host cores."""
    steps = max(10, min(args.steps, 50))
    r = time_attention_stack(workload, args, 0, 1, device, steps=steps, warmup=args.warmup)
    b0 = r["b0"]
    line = {"workload": f"{workload}: {WORKLOAD_TEXT[workload]} (T={r['T']})", "layers": r["L"],
            "steps": steps, "tflops": round(r["value"], 2), "tokens_per_s": round(r["tokens_per_s"], 1),
            "ms_per_step": round(r["ms_per_step"], 4), "ms_per_step_median": round(r["ms_per_step_median"], 4),
            "roofline": r["roofline"], "clocks": r["clocks"], "gpu_launches": r["launches"]}
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_line(b0, 6.0)
    return line


def cpu_baseline_line(b0, seconds):
    import oracle
    oracle.build()
    dt, flops, nrows = oracle_sample(b0, seconds)
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{nrows} random query rows of layer 0 (all heads), fp64 C oracle, {dt:.1f} s"}


def run_latency_bench(args, device):
    """Tiny fp32 workload (2 users, lengths 37 and 64, H=2, d=32): latency of
    one whole forward call (validate + plan, CUDA-core attention, epilogue),
    eager through the Python binding and replayed from a CUDA graph."""
    import generative_recommender_attention_jagged_b200 as hstu
    b = synth.workload_attention("tiny_fp32")
    T, H, d = b.q.shape
    x = dict(q=to_dev(b.q), k=to_dev(b.k), v=to_dev(b.v), u=to_dev(b.u), off=to_dev(b.seq_offsets, torch.int32),
             ts=to_dev(b.timestamps, torch.int64), rp=to_dev(b.rab_pos, torch.float32),
             rt=to_dev(b.rab_ts, torch.float32))
    params = hstu.attn_params(batch=b.batch, num_heads=H, head_dim=d, n_max=b.n_max, total_tokens=T,
                              max_seq_len=b.max_seq_len, dtype=b.q.dtype, alpha=b.alpha)
    ws = torch.empty(hstu.hstu_attn_workspace_size(params), dtype=torch.uint8, device=device)
    out = torch.empty(T, H * d, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream()

    def call():
        hstu.hstu_attn_fwd(x["q"], x["k"], x["v"], x["u"], x["off"], x["ts"], x["rp"], x["rt"], n_max=b.n_max,
                           alpha=b.alpha, max_seq_len=b.max_seq_len, out=out, workspace=ws)
    n = 200
    for _ in range(10):
        call()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for e0, e1 in ev:
        e0.record(stream)
        call()
        e1.record(stream)
    torch.cuda.synchronize()
    eager_us = [1e3 * a.elapsed_time(c) for a, c in ev]
    cap = torch.cuda.Stream()
    cap.wait_stream(stream)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(cap):
        call()
        cap.synchronize()
        with torch.cuda.graph(graph, stream=cap):
            call()
    torch.cuda.synchronize()
    for _ in range(10):
        graph.replay()
    torch.cuda.synchronize()
    for e0, e1 in ev:
        e0.record(stream)
        graph.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    graph_us = [1e3 * a.elapsed_time(c) for a, c in ev]
    del graph
    if hstu.hstu_check_device_error(ws) != 0:
        raise RuntimeError("tiny workload device status")
    pairs = allowed_pairs(b.lengths, None)
    flops = pairs * H * 2 * (d + d)
    line = {"workload": f"tiny_fp32: B=2 users, lengths 37 and 64, H={H}, d={d}, N_max={b.n_max}, fp32, causal",
            "unit": "us per call (median of 200)", "eager_us": round(float(np.median(eager_us)), 2),
            "eager_us_p10_p90": [round(float(np.percentile(eager_us, q)), 2) for q in (10, 90)],
            "graph_us": round(float(np.median(graph_us)), 2),
            "graph_us_p10_p90": [round(float(np.percentile(graph_us, q)), 2) for q in (10, 90)],
            "flops_per_call": flops, "gpu_launches_per_call": 3,
            "roofline": {"kernel": "attn_simt_kernel + plan + epilogue", "bound": "latency",
                         "note": "0.7 MFLOP and a few KB: launch latency, not a unit of the GPU, bounds it"}}
    if not args.no_cpu_baseline:
        import oracle
        oracle.build()
        t0 = time.perf_counter()
        reps = 0
        while time.perf_counter() - t0 < 2.0:
            oracle.batch_attn(b)
            reps += 1
        dt = (time.perf_counter() - t0) / reps
        line["cpu_baseline"] = {"value": round(dt * 1e6, 1), "unit": "us per call", "cores": oracle.num_threads(),
                                "kind": "oracle", "sample": f"the whole tiny workload, {reps} calls"}
    return line


def run_layer_bench(args, device):
    """Single HSTU layer (32 users, lengths U[512,1024], d_model 512, H=4, d=128):
    x -> f1 = SiLU(x W1 + b1) -> attention (LayerNorm(A V) * U) -> f2 = y W2 + b2,
    all through the library.  Two input sets alternate (each layer's working set,
    ~225 MB, is larger than L2)."""
    import generative_recommender_attention_jagged_b200 as hstu
    from generative_recommender_attention_jagged_b200 import _lib
    s = synth.workload_stack("layer_bf16")
    T, dm, H, d = s.x.shape[0], s.d_model, s.num_heads, s.head_dim
    hd = H * d
    rp, rt, w = s.layers[0]
    w1 = to_dev(torch.from_numpy(w.w1).to(torch.bfloat16))
    w2 = to_dev(torch.from_numpy(w.w2).to(torch.bfloat16))
    b1, b2 = to_dev(w.b1, torch.float32), to_dev(w.b2, torch.float32)
    rp, rt = to_dev(rp, torch.float32), to_dev(rt, torch.float32)
    off, ts = to_dev(s.seq_offsets, torch.int32), to_dev(s.timestamps, torch.int64)
    lengths = np.diff(s.seq_offsets)
    xs = [to_dev(s.x), to_dev(s.x).roll(1, 0).contiguous()]
    z = torch.empty(T, 4 * hd, dtype=torch.bfloat16, device=device)
    y = torch.empty(T, hd, dtype=torch.bfloat16, device=device)
    xo = torch.empty(T, dm, dtype=torch.bfloat16, device=device)
    lin_ws = torch.empty(hstu.hstu_linear_workspace_size(hstu.api.linear_params(xs[0], w1, z, True)),
                         dtype=torch.uint8, device=device)
    params = hstu.attn_params(batch=len(lengths), num_heads=H, head_dim=d, n_max=s.n_max, total_tokens=T,
                              max_seq_len=int(lengths.max()), dtype=torch.bfloat16, alpha=s.alpha)
    attn_ws = torch.empty(hstu.hstu_attn_workspace_size(params), dtype=torch.uint8, device=device)
    u, v, q, k = (z[:, i * hd:(i + 1) * hd] for i in range(4))
    q3, k3, v3 = (t.view(T, H, d) for t in (q, k, v))
    stream = torch.cuda.current_stream()

    def attn(stage):
        hstu.hstu_attn_fwd(q3, k3, v3, u, off, ts, rp, rt, n_max=s.n_max, alpha=s.alpha,
                           max_seq_len=int(lengths.max()), out=y, workspace=attn_ws, stages=stage)

    def layer(i, ev=None):
        rec = (lambda j: ev[j].record(stream)) if ev is not None else (lambda j: None)
        rec(0)
        hstu.hstu_layer_f1(xs[i % 2], w1, b1, out=z, workspace=lin_ws)
        rec(1)
        attn(_lib.F_STAGE_PLAN)
        rec(2)
        attn(_lib.F_STAGE_ATTN)
        rec(3)
        attn(_lib.F_STAGE_EPILOGUE)
        rec(4)
        hstu.hstu_layer_f2(y, w2, b2, out=xo, workspace=lin_ws)
        rec(5)

    steps = max(56, min(args.steps, 100))
    for i in range(args.warmup):
        layer(i)
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(steps)]
    clocks = ClockSampler(device.index if device.index is not None else 0)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(steps):
        layer(i, ev[i])
    t1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if hstu.hstu_check_device_error(attn_ws) != 0 or hstu.hstu_check_device_error(lin_ws) != 0:
        raise RuntimeError("layer workload device status")
    ms_layer = t0.elapsed_time(t1) / steps
    part = lambda a, c: [e[a].elapsed_time(e[c]) for e in ev]
    f1_ms, attn_ms, f2_ms = part(0, 1), part(2, 3), part(4, 5)
    pairs = allowed_pairs(lengths, None)
    attn_flops = pairs * H * FLOPS_PER_PAIR_HEAD
    f1_flops, f2_flops = 2.0 * T * dm * 4 * hd, 2.0 * T * hd * dm
    total = attn_flops + f1_flops + f2_flops
    line = {"workload": f"layer_bf16: one HSTU layer, B={len(lengths)} users, lengths U[512,1024] (T={T}), "
                        f"d_model={dm}, H={H}, d={d}, N_max={s.n_max}: f1 -> attention -> f2",
            "steps": steps, "ms_per_layer": round(ms_layer, 4), "tokens_per_s": round(T / (ms_layer * 1e-3), 1),
            "tflops": round(total / (ms_layer * 1e-3) / 1e12, 2),
            "flops_per_layer": {"f1": f1_flops, "attention": attn_flops, "f2": f2_flops},
            "ms_median": {"f1": round(float(np.median(f1_ms)), 4), "attention": round(float(np.median(attn_ms)), 4),
                          "f2": round(float(np.median(f2_ms)), 4),
                          "plan+epilogue": round(float(np.median([a + c for a, c in zip(part(1, 2), part(3, 4))])), 4)},
            "roofline": tensor_roofline("attn_sm100_kernel", attn_flops, attn_ms, clk),
            "roofline_f1": tensor_roofline("gemm_pair_kernel (f1)", f1_flops, f1_ms, clk),
            "clocks": clk, "gpu_launches_per_layer": 5, "l2": "two alternating input sets"}
    if not args.no_cpu_baseline:
        b0 = synth.workload_attention("layer_bf16")
        line["cpu_baseline"] = cpu_baseline_line(b0, 4.0)
    return line


def run_paged_bench(args, device):
    """Paged incremental workload: 8 users, cached prefix U[6144,8192] in
    32-token pages, +64 actions +64 candidates, 8 layers with separate pools."""
    import generative_recommender_attention_jagged_b200 as hstu
    from generative_recommender_attention_jagged_b200 import _lib
    layers = synth.paged_stack(8)
    stream = torch.cuda.current_stream()
    dl = []
    for pb in layers:
        dl.append(dict(q=to_dev(pb.q), k=to_dev(pb.k), v=to_dev(pb.v), u=to_dev(pb.u),
                       off=to_dev(pb.new_offsets, torch.int32), ts=to_dev(pb.timestamps, torch.int64),
                       tso=to_dev(pb.ts_offsets, torch.int32), cand=to_dev(pb.num_candidates, torch.int32),
                       rp=to_dev(pb.rab_pos, torch.float32), rt=to_dev(pb.rab_ts, torch.float32),
                       kp=to_dev(pb.k_pool), vp=to_dev(pb.v_pool), pt=to_dev(pb.kv_page_table, torch.int32),
                       cl=to_dev(pb.cached_lens, torch.int32)))
    pb0 = layers[0]
    T = int(pb0.new_offsets[-1])
    maxc = int(pb0.cached_lens.max())
    params = hstu.attn_params(batch=pb0.batch, num_heads=4, head_dim=128, n_max=pb0.n_max, total_tokens=T,
                              max_seq_len=pb0.n_max, dtype=torch.bfloat16)
    splits = hstu.hstu_attn_paged_default_splits(params, maxc)
    ws = torch.empty(hstu.hstu_attn_paged_workspace_size(params, splits), dtype=torch.uint8, device=device)
    out = torch.empty(T, 512, dtype=torch.bfloat16, device=device)

    def call(x, stage):
        hstu.hstu_attn_fwd_paged(x["q"], x["k"], x["v"], x["u"], x["off"], x["ts"], x["tso"], x["rp"], x["rt"],
                                 x["kp"], x["vp"], x["pt"], x["cl"], n_max=pb0.n_max, num_candidates=x["cand"],
                                 num_splits=splits, out=out, workspace=ws, stages=stage)

    steps = max(10, min(args.steps, 50))
    for _ in range(3):
        for x in dl:
            call(x, 0)
    torch.cuda.synchronize()
    # whole layers as a caller runs them (three Python calls per layer: plan, attention, epilogue)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        for x in dl:
            call(x, 0)
    t1.record(stream)
    torch.cuda.synchronize()
    status = hstu.hstu_check_device_error(ws)
    if status != 0:
        raise RuntimeError(f"paged device status {status}")
    ms_layer = t0.elapsed_time(t1) / (steps * len(dl))
    # The attention kernel alone: its launches for the 8 layers captured in a CUDA
    # graph and replayed, so no host time (argument marshalling, tensor-map
    # encoding) falls between the events.  Every layer has the same users and
    # cached lengths, so one plan serves all of them.
    cap = torch.cuda.Stream()
    cap.wait_stream(stream)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(cap):
        call(dl[0], _lib.F_STAGE_PLAN)
        for x in dl:
            call(x, _lib.F_STAGE_ATTN)
        cap.synchronize()
        with torch.cuda.graph(graph, stream=cap):
            for x in dl:
                call(x, _lib.F_STAGE_ATTN)
    torch.cuda.synchronize()
    graph.replay()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    clocks = ClockSampler(device.index if device.index is not None else 0)
    for a, b in ev:
        a.record(stream)
        graph.replay()
        b.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    replay_ms = [a.elapsed_time(b) / len(dl) for a, b in ev]
    attn_ms = float(np.median(replay_ms))
    status = hstu.hstu_check_device_error(ws)
    if status != 0:
        raise RuntimeError(f"paged device status {status}")
    del graph
    kv_bytes = int(sum(2 * int(c) * 4 * 128 * 2 for c in pb0.cached_lens))
    new_bytes = T * 512 * 2 * 4 + int(pb0.ts_offsets[-1]) * 8
    alg_bytes = kv_bytes + new_bytes
    peaks, kind = measured_peaks()
    achieved = alg_bytes / (attn_ms * 1e-3) / 1e9
    return {"workload": "paged_bf16: 8 users, cached U[6144,8192] in 32-token pages, +64 actions "
                        "+64 candidates, 8 layers (separate pools), H=4, d=128, N_max=8320",
            "ms_per_layer": round(ms_layer, 4), "new_tokens_per_s": round(T / (ms_layer * 1e-3), 1),
            "splits": splits,
            "roofline": {"kernel": "attn_sm100_single_kernel (paged)", "bound": "hbm", "achieved": round(achieved, 1),
                         "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                         "frac": round(achieved / float(peaks["hbm_gbs"]), 4),
                         "peak_source": f"{kind} hbm_gbs", "bytes_per_launch": alg_bytes,
                         "launch_ms": round(attn_ms, 4),
                         "launch_ms_p10_p90": [round(float(np.percentile(replay_ms, q)), 4) for q in (10, 90)],
                         "timing": f"CUDA-graph replay of the 8 layers' attention launches, median of {steps} "
                                   f"replays", "traffic": PAGED_TRAFFIC_BYTES},
            "clocks": clk}


def run_glue_bench(args, device):
    """The layer glue around the attention at the 8-layer stack's shapes:
    f1 = SiLU(x W1 + b1) (512 -> 2048, cuBLASLt GEMM + in-place SiLU kernel)
    and f2 = y W2 + b2 (512 -> 512).  Two input sets alternate so that the
    operands (~270 MB per f1 call) do not sit in L2 between calls."""
    import generative_recommender_attention_jagged_b200 as hstu
    s = synth.workload_stack("stack8_bf16", num_layers=1)
    T = s.x.shape[0]
    _, _, w = s.layers[0]
    w1 = to_dev(torch.from_numpy(w.w1).to(torch.bfloat16))
    w2 = to_dev(torch.from_numpy(w.w2).to(torch.bfloat16))
    b1, b2 = to_dev(w.b1, torch.float32), to_dev(w.b2, torch.float32)
    xs = [to_dev(s.x), to_dev(s.x).roll(1, 0).contiguous()]
    zs = [torch.empty(T, 2048, dtype=torch.bfloat16, device=device) for _ in range(2)]
    ys = [z[:, :512] for z in zs]          # a [T, 512] view with row stride 2048, as f2 sees y after attention
    outs = [torch.empty(T, 512, dtype=torch.bfloat16, device=device) for _ in range(2)]
    ws = torch.empty(hstu.hstu_linear_workspace_size(hstu.api.linear_params(xs[0], w1, zs[0], True)),
                     dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()
    steps = max(50, min(args.steps, 100))

    samples = {}

    def timed(fn, name=None):
        for i in range(3):
            fn(i)
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        clocks = ClockSampler(device.index if device.index is not None else 0) if name else None
        for i, (a, b) in enumerate(ev):
            a.record(stream)
            fn(i)
            b.record(stream)
        torch.cuda.synchronize()
        ms = [a.elapsed_time(b) for a, b in ev]
        if name:
            samples[name] = (ms, clocks.stop())
        return float(np.median(ms))

    f1_ms = timed(lambda i: hstu.hstu_layer_f1(xs[i % 2], w1, b1, out=zs[i % 2], workspace=ws), "f1")
    f2_ms = timed(lambda i: hstu.hstu_layer_f2(ys[i % 2], w2, b2, out=outs[i % 2], workspace=ws), "f2")
    f1_lib = timed(lambda i: hstu.hstu_layer_f1(xs[i % 2], w1, b1, out=zs[i % 2], workspace=ws,
                                                force_cublas=True))
    f2_lib = timed(lambda i: hstu.hstu_layer_f2(ys[i % 2], w2, b2, out=outs[i % 2], workspace=ws,
                                                force_cublas=True))
    f1_flops, f2_flops = 2.0 * T * 512 * 2048, 2.0 * T * 512 * 512
    tf = lambda flops, ms: flops / (ms * 1e-3) / 1e12
    f1_tf, f2_tf = tf(f1_flops, f1_ms), tf(f2_flops, f2_ms)
    return {"workload": f"stack8_bf16 layer glue: T={T}, f1 512->2048 + SiLU, f2 512->512, bf16",
            "f1_ms": round(f1_ms, 4), "f2_ms": round(f2_ms, 4), "statistic": f"median of {steps} calls",
            "f1_tflops": round(f1_tf, 1), "f2_tflops": round(f2_tf, 1),
            "cublaslt": {"f1_ms": round(f1_lib, 4), "f2_ms": round(f2_lib, 4),
                         "f1_tflops": round(tf(f1_flops, f1_lib), 1), "f2_tflops": round(tf(f2_flops, f2_lib), 1),
                         "note": "cuBLASLt GEMM, bias in its epilogue, separate in-place SiLU pass for f1"},
            "roofline": tensor_roofline("gemm_pair_kernel (f1: bias + SiLU in the epilogue)", f1_flops,
                                        *samples["f1"]),
            "roofline_f2": tensor_roofline("cuBLASLt GEMM (f2 = y W2 + b2)", f2_flops, *samples["f2"])}


def run_mfalcon_bench(args, device):
    """M-FALCON: 8 users with a cached history of U[2048,4096] tokens (32-token
    pages) score 4,096 candidates each, 2,048 per microbatch."""
    import generative_recommender_attention_jagged_b200 as hstu
    rng = np.random.default_rng(1000 + 31)
    B, C, mb = 8, 4096, 2048
    cached = rng.integers(2048, 4096, size=B, endpoint=True)
    n_max = 4096 + mb
    pb = synth.paged_batch(cached, 0, C, 4, 128, n_max, rng=rng, poison=False)
    hist, hist_off, cand = [], [0], []
    for b in range(B):
        L = int(pb.cached_lens[b])
        t = pb.timestamps[pb.ts_offsets[b]:pb.ts_offsets[b + 1]]
        hist.append(t[:L])
        cand.append(t[L:])
        hist_off.append(hist_off[-1] + L)
    d = dict(q=to_dev(pb.q), k=to_dev(pb.k), v=to_dev(pb.v), u=to_dev(pb.u),
             off=to_dev(pb.new_offsets, torch.int32), hist=to_dev(np.concatenate(hist), torch.int64),
             hoff=to_dev(np.array(hist_off), torch.int32), cts=to_dev(np.concatenate(cand), torch.int64),
             rp=to_dev(pb.rab_pos, torch.float32), rt=to_dev(pb.rab_ts, torch.float32), kp=to_dev(pb.k_pool),
             vp=to_dev(pb.v_pool), pt=to_dev(pb.kv_page_table, torch.int32), cl=to_dev(pb.cached_lens, torch.int32))
    out, ws = None, None

    def call():
        nonlocal out, ws
        out, ws = hstu.hstu_mfalcon_fwd(d["q"], d["k"], d["v"], d["u"], d["off"], d["hist"], d["hoff"], d["cts"],
                                        d["rp"], d["rt"], d["kp"], d["vp"], d["pt"], d["cl"], n_max=n_max,
                                        microbatch=mb, max_candidates=C, max_cached_len=int(cached.max()),
                                        out=out, workspace=ws)
    for _ in range(2):
        call()
    torch.cuda.synchronize()
    steps = max(56, min(args.steps, 100))
    stream = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    clocks = ClockSampler(device.index if device.index is not None else 0)
    for e0, e1 in ev:
        e0.record(stream)
        call()
        e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if hstu.hstu_check_device_error(ws) != 0:
        raise RuntimeError("mfalcon device status")
    call_ms = [a.elapsed_time(b) for a, b in ev]
    ms = float(np.median(call_ms))
    flops = float(sum(C * (int(L) + 1) for L in cached)) * 4 * 2 * (128 + 128)
    tf = flops / (ms * 1e-3) / 1e12
    roof = tensor_roofline("hstu_mfalcon_fwd (whole call: gather, paged attention, epilogue, scatter)", flops,
                           call_ms, clk)
    return {"workload": f"M-FALCON: B={B} users, cached history U[2048,4096] (32-token pages), {C} candidates "
                        f"per user in microbatches of {mb}, H=4, d=128, bf16",
            "ms": round(ms, 4), "candidates_per_s": round(B * C / (ms * 1e-3), 1), "tflops": round(tf, 1),
            "roofline": roof, "clocks": clk}


def run_bwd_bench(args, device):
    """Backward of the attention core on one layer of the 32-user layer
    workload (d_q, d_k, d_v and the bias-table gradients): the default path
    (tcgen05, bf16 GEMM operands, fp32 accumulate) against the measured bf16
    peak, and the fp32 CUDA-core kernel (force_simt) beside it."""
    import generative_recommender_attention_jagged_b200 as hstu
    b = synth.workload_attention("layer_bf16", layer=0)
    T, H, d = b.q.shape
    g = torch.randn(T, H, d, device=device)
    x = dict(q=to_dev(b.q), k=to_dev(b.k), v=to_dev(b.v), off=to_dev(b.seq_offsets, torch.int32),
             ts=to_dev(b.timestamps, torch.int64), rp=to_dev(b.rab_pos, torch.float32),
             rt=to_dev(b.rab_ts, torch.float32))

    def call(force_simt):
        return hstu.hstu_attn_bwd(x["q"], x["k"], x["v"], x["off"], x["ts"], x["rp"], x["rt"], g, n_max=b.n_max,
                                  alpha=b.alpha, max_seq_len=b.max_seq_len, force_simt=force_simt)
    steps = max(20, min(args.steps, 50))
    stream = torch.cuda.current_stream()

    def timed(force_simt):
        out = call(force_simt)
        torch.cuda.synchronize()
        if hstu.hstu_check_device_error(out[-1]) != 0:
            raise RuntimeError("backward device status")
        for _ in range(3):
            call(force_simt)
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        clocks = ClockSampler(device.index if device.index is not None else 0)
        for e0, e1 in ev:
            e0.record(stream)
            call(force_simt)
            e1.record(stream)
        torch.cuda.synchronize()
        return [e0.elapsed_time(e1) for e0, e1 in ev], clocks.stop()

    pairs = allowed_pairs(b.lengths, b.num_candidates)
    flops = pairs * H * 4 * 2 * d          # d_v, d_a, d_q, d_k: four products of 2 d flops per pair
    tc_ms, tc_clk = timed(False)
    simt_ms, _ = timed(True)
    tf = lambda ms: flops / (ms * 1e-3) / 1e12
    ms_tc, ms_simt = float(np.median(tc_ms)), float(np.median(simt_ms))
    clk = max_sm_mhz()
    fma_peak = 148 * 128 * 2 * clk * 1e6 / 1e12   # fp32 FMA lanes x 2 flops x clock
    return {"workload": f"layer_bf16 backward: B={b.batch} users, lengths U[512,1024] (T={T}), H={H}, d={d}, "
                        f"bf16 on the tensor cores", "ms": round(ms_tc, 3), "tflops": round(tf(ms_tc), 2),
            "statistic": f"median of {steps} calls (each: d_o to bf16, d_q zeroing, validation, the kernel)",
            "roofline": tensor_roofline("attn_bwd_sm100_kernel (whole call)", flops, tc_ms, tc_clk),
            "fp32_cuda_cores": {"ms": round(ms_simt, 3), "tflops": round(tf(ms_simt), 2),
                                "roofline": {"kernel": "attn_bwd_tiled_kernel", "bound": "alu",
                                             "achieved": round(tf(ms_simt), 2), "peak": round(fma_peak, 1),
                                             "unit": "TFLOP/s", "frac": round(tf(ms_simt) / fma_peak, 4),
                                             "peak_source": f"148 SMs x 128 fp32 FMA lanes x 2 flops x {clk} MHz"}}}


def run_kv_append_bench(args, device):
    """KV write side after a request of the paged workload: 8 users append 64
    actions each (K and V, 4 heads x 128 bf16) into free pages."""
    import generative_recommender_attention_jagged_b200 as hstu
    rng = np.random.default_rng(1000 + 32)
    B, A, P, H, D = 8, 64, 32, 4, 128
    cached = rng.integers(6144, 8192, size=B, endpoint=True)
    max_pages = int((cached.max() + A * 64) // P + 2)
    num_pages = int(sum((c + A * 64) // P + 2 for c in cached))
    k_pool = torch.zeros(num_pages, H, P, D, dtype=torch.bfloat16, device=device)
    v_pool = torch.zeros_like(k_pool)
    k_new = torch.randn(B * A, H, D, device=device).to(torch.bfloat16)
    v_new = torch.randn(B * A, H, D, device=device).to(torch.bfloat16)
    off = torch.arange(0, B * A + 1, A, dtype=torch.int32, device=device)
    steps = max(3, min(args.steps, 50))

    def fresh():
        table = torch.full((B, max_pages), -1, dtype=torch.int32, device=device)
        pages = [(int(c) + P - 1) // P for c in cached]
        perm = torch.randperm(num_pages, device=device).to(torch.int32)
        pos = 0
        for b in range(B):
            table[b, :pages[b]] = perm[pos:pos + pages[b]]
            pos += pages[b]
        free = perm[pos:].clone()
        free = torch.cat([free, torch.zeros(pos, dtype=torch.int32, device=device)])
        return table, torch.tensor(cached, dtype=torch.int32, device=device), free, \
            torch.tensor([num_pages - pos], dtype=torch.int32, device=device)

    table, lens, free, fc = fresh()
    ws = hstu.hstu_kv_append(k_new, v_new, off, k_pool, v_pool, table, lens, free, fc)
    torch.cuda.synchronize()
    table, lens, free, fc = fresh()
    stream = torch.cuda.current_stream()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):   # each call appends one more request's actions to every user
        hstu.hstu_kv_append(k_new, v_new, off, k_pool, v_pool, table, lens, free, fc, workspace=ws)
    b.record(stream)
    torch.cuda.synchronize()
    if hstu.hstu_check_device_error(ws) != 0:
        raise RuntimeError("kv append device status")
    us = a.elapsed_time(b) / steps * 1e3
    moved = 2 * B * A * H * D * 2 * 2          # K and V, read + write
    return {"workload": f"KV append: {B} users x {A} actions, H={H}, d={D}, bf16, {P}-token pages",
            "us_per_call": round(us, 2), "bytes_per_call": moved,
            "gbs": round(moved / (us * 1e-6) / 1e9, 1),
            "note": "two launches (plan + copy) per call; at this size the call is launch-bound"}


# ----------------------------------------------------------------------------
# reference arm: the fp64 CPU oracle on the host cores
# ----------------------------------------------------------------------------

def run_reference(args):
    import oracle
    oracle.build()
    b0 = synth.workload_attention(args.workload, layer=0)
    per_step = max(2.0, 60.0 / max(1, args.steps + args.warmup))
    vals = []
    for s in range(args.warmup + args.steps):
        dt, flops, nrows = oracle_sample(b0, per_step, seed=s)
        if s >= args.warmup:
            vals.append((dt, flops, nrows))
    dt = sum(v[0] for v in vals)
    flops = sum(v[1] for v in vals)
    rows = sum(v[2] for v in vals)
    value = flops / dt / 1e12
    cores = oracle.num_threads()
    return {
        "impl": "reference",
        "metric": "HSTU attention fwd TFLOP/s + tokens/s, % of B200 BF16 peak / HBM BW",
        "value": value, "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded; no dataset)",
        "config": {"workload": f"{args.workload}: {WORKLOAD_TEXT[args.workload]} (T={b0.total_tokens})",
                   "global_batch": b0.batch, "total_tokens_per_gpu": b0.total_tokens,
                   "parallelism": "host cores (OpenMP), rank 0 only"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"{rows} random query rows of layer 0 (all heads), fp64 C oracle"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="stack8_bf16", choices=["stack8_bf16", "stack8_n8192", "mfalcon_bf16"])
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--only", choices=["stack", "paged", "glue", "next", "configs", "layer", "latency",
                                       "n8192", "mfalcon_jagged"],
                    help="run one part only (profiling captures); prints that part's JSON")
    ap.add_argument("--no-paged", action="store_true")
    ap.add_argument("--no-glue", action="store_true", help="skip the f1/f2 layer-glue timing")
    ap.add_argument("--no-next", action="store_true", help="skip the M-FALCON, KV-append and backward timings")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-config lines (configs 0, 1, 2b, 3)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--paged-only", action="store_true", help="same as --only paged")
    ap.add_argument("--glue-only", action="store_true", help="same as --only glue")
    ap.add_argument("--next-only", action="store_true", help="same as --only next")
    ap.add_argument("--layers", type=int, default=None,
                    help="fewer layers (profiling captures only; the bench line uses all of them)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    for flag, part in (("paged_only", "paged"), ("glue_only", "glue"), ("next_only", "next")):
        if getattr(args, flag):
            args.only = part

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    from generative_recommender_attention_jagged_b200 import build as hbuild
    hbuild.build()
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)

    def configs():
        return {"config0_tiny_fp32_latency": run_latency_bench(args, device),
                "config1_layer": run_layer_bench(args, device),
                "config2b_stack8_n8192": run_config_line("stack8_n8192", args, device),
                "config3_mfalcon_jagged": run_config_line("mfalcon_bf16", args, device)}

    if args.only is not None and args.only != "stack":
        parts = {"paged": lambda: {"paged": run_paged_bench(args, device)},
                 "glue": lambda: {"glue": run_glue_bench(args, device)},
                 "next": lambda: {"mfalcon": run_mfalcon_bench(args, device),
                                  "kv_append": run_kv_append_bench(args, device),
                                  "backward": run_bwd_bench(args, device)},
                 "configs": configs,
                 "layer": lambda: {"config1_layer": run_layer_bench(args, device)},
                 "latency": lambda: {"config0_tiny_fp32_latency": run_latency_bench(args, device)},
                 "n8192": lambda: {"config2b_stack8_n8192": run_config_line("stack8_n8192", args, device)},
                 "mfalcon_jagged": lambda: {"config3_mfalcon_jagged": run_config_line("mfalcon_bf16", args,
                                                                                      device)}}
        if rank == 0:
            print(json.dumps(parts[args.only]()), flush=True)
        return
    result, b0 = run_ours(args, rank, world, device)
    extras = args.only is None and world == 1 and rank == 0
    if extras and not args.no_configs:
        result.update(configs())
    if extras and not args.no_paged:
        result["paged"] = run_paged_bench(args, device)
    if extras and not args.no_glue:
        result["glue"] = run_glue_bench(args, device)
    if extras and not args.no_next:
        result["mfalcon"] = run_mfalcon_bench(args, device)
        result["kv_append"] = run_kv_append_bench(args, device)
        result["backward"] = run_bwd_bench(args, device)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        dt, flops, nrows = oracle_sample(b0, 12.0)
        result["cpu_baseline"] = {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(),
                                  "kind": "oracle",
                                  "sample": f"{nrows} random query rows of layer 0 (all 4 heads), fp64 C oracle, "
                                            f"{dt:.1f} s"}
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


if __name__ == "__main__":
    main()
