#!/usr/bin/env python3
"""Benchmark of the selective state update over a paged state pool (one JSON line).

Headline step: one ssu_decode launch over the Mamba2-2.7B-like decode workload
(batch 256 over a 512-slot pool, 80 heads, dim 64, dstate 128, one group, bf16
x/B/C/z/out, fp32 dt/A/D/dt_bias and fp32 state, softplus with dt_bias, z gate,
stateIndices a random subset of the pool). Each step reads and writes 20,480 head
states of 32 KiB: 671 MB of state per step, far above the 126 MB L2, so consecutive
steps do not hit in L2 and no flush is needed (checked at run time).

  value      seq-head updates/s over all ranks (K steps x batch x heads / max time)
  roofline   the decode kernel's algorithmic bytes / its mean launch time (CUDA events
             on the launching stream) against the measured HBM copy bandwidth
  e2e        the same metric through the public binding with the step's inputs copied
             from pinned host memory and the output copied back inside the timed region
  forms      (one GPU only) the prefill scan and the speculative replay on their own
             workloads, same timing method
  cpu_baseline  the float64 CPU oracle on a bounded sample, rank 0, one GPU only: on
             every host core (value, cores) and on one thread, with the CPU model

Multi-GPU (torchrun): replicas only -- every rank runs its own pool and batch, no data
collective; the barrier and the max-over-ranks reduction are measurement plumbing.
`--impl reference` times the CPU oracle instead (rank 0 only).
"""

from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "decode state-update HBM GB/s (% of B200 peak); seq-head updates/s at batch 256"
UNIT = "seq-head updates/s"
WORKLOAD = "mamba2_decode_b256"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0

REASON_BITS = {
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
    0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
    0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
    0x100: "display_clock_setting",
}


# ----------------------------------------------------------------------------- helpers

def measured_bf16_tflops():
    """The burst bf16 GEMM rate of MEASURED_PEAKS.json (TFLOP/s), else the fallback."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_BF16_TFLOPS, "fallback"


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


DECODE_SOURCES = ("ssu_decode.cu", "ssu_stream.cuh", "ssu_async.cuh", "ssu_common.cuh")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "ssu_decode_traffic.json")


def decode_source_hash() -> str:
    """sha256 over the decode kernel's sources, to tie an ncu traffic figure to them."""
    import hashlib
    h = hashlib.sha256()
    for name in DECODE_SOURCES:
        with open(os.path.join(ROOT, "linear_attention_recurrent_selective_b200", "csrc", name),
                  "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def recorded_traffic(batch: int):
    """DRAM bytes per decode launch measured by ncu (profiles/ssu_decode_traffic.json), or
    None when the record is missing, is for another batch, or was taken on sources other
    than the ones built now."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    if rec.get("source_sha256") != decode_source_hash() or rec.get("batch") != batch:
        return None
    try:
        return int(rec["bytes_per_launch"])
    except (KeyError, TypeError, ValueError):
        return None


def decode_bytes(batch, H, G, Dm, N, state_bytes, io_bytes):
    """Algorithmic bytes of one decode launch: every state element read and written once,
    x/z/out once per (row, head, dim), B/C once per (row, group), dt once per (row, head),
    A/D/dt_bias once per head, one index per row."""
    units = batch * H
    state = units * Dm * N * state_bytes * 2
    io = units * Dm * io_bytes * 3 + units * 4 + batch * G * N * io_bytes * 2
    return state, state + io + H * 12 + batch * 4


def world():
    return int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), \
        int(os.environ.get("LOCAL_RANK", "0"))


def max_over_ranks(x: float, device) -> float:
    """Max of a per-rank float over the process group (identity without one)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank_step: int, steps: int, n_ranks: int, seconds: float) -> float:
    """Whole-job throughput: the units every rank processed over the slowest rank's time."""
    return units_per_rank_step * steps * n_ranks / seconds


def barrier(device):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


class ClockSampler:
    """Polls SM clock and clock-event reasons via NVML while the timed region runs."""

    def __init__(self, device_index: int, period_s: float = 0.001):
        self.samples = []      # (t, sm_mhz, reasons_mask)
        self.max_mhz = None
        self._stop = threading.Event()
        self._period = period_s
        self._handle = None
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self._handle = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self._nvml = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._handle, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # NVML missing: report the absence instead of clocks
            self.error = repr(e)
        self._thread = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        n = self._nvml
        while not self._stop.is_set():
            try:
                mhz = n.nvmlDeviceGetClockInfo(self._handle, n.NVML_CLOCK_SM)
                reasons = n.nvmlDeviceGetCurrentClocksEventReasons(self._handle)
                self.samples.append((time.perf_counter(), mhz, reasons))
            except Exception:
                pass
            time.sleep(self._period)

    def start(self):
        if self._handle is not None:
            self._thread.start()
        return self

    def stop(self):
        self._stop.set()
        if self._thread.is_alive():
            self._thread.join()

    def summary(self, t0: float, t1: float):
        if self._handle is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [],
                    "note": "NVML unavailable: " + getattr(self, "error", "")}
        win = [s for s in self.samples if t0 <= s[0] <= t1]
        note = "samples inside the timed region"
        if not win:   # timed region shorter than the poll period: nearest samples
            win = sorted(self.samples, key=lambda s: min(abs(s[0] - t0), abs(s[0] - t1)))[:3]
            note = "timed region shorter than the poll period: nearest samples"
        mask = 0
        for s in win:
            mask |= s[2]
        return {"sm_mhz": statistics.median(s[1] for s in win) if win else None,
                "sm_max_mhz": self.max_mhz,
                "reasons": [v for k, v in REASON_BITS.items() if mask & k and k != 0x1],
                "samples": len(win), "note": note}


# ----------------------------------------------------------------------------- our arm

def run_decode(args, device):
    from linear_attention_recurrent_selective_b200 import ssu
    from linear_attention_recurrent_selective_b200.workloads import make_config

    overrides = {}
    if args.batch:
        overrides = dict(batch=args.batch, P=2 * args.batch)
    case = make_config(WORKLOAD, **overrides)
    d = case.to(device)
    pool = d.pool
    out = torch.empty_like(d.x)
    units = case.batch * case.H
    state_b, alg_b = decode_bytes(case.batch, case.H, case.G, case.Dm, case.N,
                                  pool.element_size(), d.x.element_size())
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    flush = state_b < 2 * l2
    flush_buf = torch.empty(4 * l2 // 4, dtype=torch.float32, device=device) if flush else None

    def step():
        ssu.ssu_decode(d.x, d.A, d.B, d.C, d.dt, pool, out, dt_bias=d.dt_bias, D=d.D, z=d.z,
                       state_indices=d.state_indices, active_batch=case.active,
                       slot_stride=case.slot_stride, P=case.P)

    stream = torch.cuda.current_stream(device)
    for _ in range(args.warmup):
        if flush:
            flush_buf.zero_()
        step()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    t_all0, t_all1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(device.index).start()
    torch.cuda.synchronize(device)
    barrier(device)
    torch.cuda.synchronize(device)
    wall0 = time.perf_counter()
    t_all0.record(stream)
    for k in range(args.steps):
        if flush:
            flush_buf.zero_()
        starts[k].record(stream)
        step()
        ends[k].record(stream)
    t_all1.record(stream)
    torch.cuda.synchronize(device)
    wall1 = time.perf_counter()
    barrier(device)
    torch.cuda.synchronize(device)
    clocks.stop()
    total_ms = t_all0.elapsed_time(t_all1)
    kern_ms = statistics.fmean(s.elapsed_time(e) for s, e in zip(starts, ends))
    res = dict(case=case, units=units, total_ms=total_ms, kern_ms=kern_ms, state_b=state_b,
               alg_b=alg_b, clocks=clocks.summary(wall0, wall1), flush=flush, l2=l2)

    # ---- end to end through the binding: pinned host inputs in, output back out.
    # Every step copies its inputs from pinned host memory and reads its output back; the
    # copies run on their own streams, double-buffered, so that step k+1's inputs arrive
    # and step k-1's output leaves while step k computes (the state pool is updated in
    # place, so the compute steps stay in order on one stream).
    host = {k: getattr(case, k).pin_memory() for k in ("x", "z", "B", "C", "dt",
                                                       "state_indices")}
    s_in, s_comp, s_out = (torch.cuda.Stream(device) for _ in range(3))
    bufs = [{k: torch.empty_like(v, device=device) for k, v in host.items()} for _ in range(2)]
    outs = [torch.empty_like(out) for _ in range(2)]
    outs_h = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    ev_in = [torch.cuda.Event() for _ in range(2)]       # inputs of buffer j have landed
    ev_done = [torch.cuda.Event() for _ in range(2)]     # compute finished with buffer j
    ev_out = [torch.cuda.Event() for _ in range(2)]      # output j has been copied out

    def e2e_step(k):
        j = k & 1
        s_in.wait_event(ev_done[j])                       # step k-2 no longer reads bufs[j]
        with torch.cuda.stream(s_in):
            for name in host:
                bufs[j][name].copy_(host[name], non_blocking=True)
        ev_in[j].record(s_in)
        s_comp.wait_event(ev_in[j])
        s_comp.wait_event(ev_out[j])                      # outs[j] of step k-2 copied out
        b = bufs[j]
        ssu.ssu_decode(b["x"], d.A, b["B"], b["C"], b["dt"], pool, outs[j], dt_bias=d.dt_bias,
                       D=d.D, z=b["z"], state_indices=b["state_indices"],
                       active_batch=case.active, slot_stride=case.slot_stride, P=case.P,
                       stream=s_comp)
        ev_done[j].record(s_comp)
        s_out.wait_event(ev_done[j])
        with torch.cuda.stream(s_out):
            outs_h[j].copy_(outs[j], non_blocking=True)
        ev_out[j].record(s_out)

    for k in range(args.warmup):
        e2e_step(k)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(device)
    barrier(device)
    e0.record(s_in)
    for k in range(args.steps):
        e2e_step(k)
    e1.record(s_out)                                      # after the last output read
    torch.cuda.synchronize(device)
    barrier(device)
    res["e2e_ms"] = e0.elapsed_time(e1)
    res["h2d"] = sum(v.numel() * v.element_size() for v in host.values())
    res["d2h"] = outs_h[0].numel() * outs_h[0].element_size()

    # ---- clock record over a longer window (not part of the reported value): the same
    # step back to back for at least 0.5 s, NVML sampled every 5 ms, so that the clock the
    # kernel ran at rests on many samples even when the timed region above is short
    n_sus = 0 if args.no_clock_window else max(10, int(0.6 / max(kern_ms / 1e3, 1e-6)))
    sus = ClockSampler(device.index, period_s=0.005).start()
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(device)
    w0 = time.perf_counter()
    s0.record(stream)
    for _ in range(n_sus):
        if flush:
            flush_buf.zero_()
        step()
    s1.record(stream)
    torch.cuda.synchronize(device)
    w1 = time.perf_counter()
    sus.stop()
    sus_ms = s0.elapsed_time(s1) / max(n_sus, 1)
    res["clocks_sustained"] = {**sus.summary(w0, w1), "steps": n_sus,
                               "seconds": round(w1 - w0, 3), "ms_per_step": sus_ms}
    return res


def time_launches(fn, steps, warmup, device):
    stream = torch.cuda.current_stream(device)
    for _ in range(warmup):
        fn()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    torch.cuda.synchronize(device)
    for k in range(steps):
        starts[k].record(stream)
        fn()
        ends[k].record(stream)
    torch.cuda.synchronize(device)
    return statistics.fmean(s.elapsed_time(e) for s, e in zip(starts, ends))


def form_prefill(args, device, batch=0):
    """Multi-token prefill (batch 16, T 512, contextLengths ~ U{1..512}), without and with
    the replay stash. Reported against the FP32 peak at the sequential form's FLOP count
    (5 per state element and token), the measure the scope table fixes; with bf16 inputs
    the library evaluates the recurrence in chunks of 128 tokens on the tensor cores, so
    the MMA work as issued (against the measured bf16 GEMM rate) and the algorithmic
    bytes (against the measured HBM copy rate) are reported beside it."""
    from linear_attention_recurrent_selective_b200 import ssu
    from linear_attention_recurrent_selective_b200.workloads import make_config

    steps, warm = max(3, min(args.steps, 50)), max(3, min(args.warmup, 5))
    case = make_config("prefill_b16_t512", **(dict(batch=batch, P=2 * batch) if batch else {}))
    d = case.to(device)
    pool = d.pool.clone()
    out = torch.empty_like(d.x)
    f = dict(dtype=torch.float32, device=device)
    b, T, H, G, Dm, N = case.batch, case.T, case.H, case.G, case.Dm, case.N
    stash = (torch.empty(b, T, H, **f), torch.empty(b, T, H, Dm, **f),
             torch.empty(b, T, G, N, **f), torch.empty(b, T, H, **f))
    tokens = int(case.context_lengths.sum())

    def prefill(st):
        ssu.ssu_prefill(d.x, d.A, d.B, d.C, d.dt, pool, out, dt_bias=d.dt_bias, D=d.D, z=d.z,
                        state_indices=d.state_indices, context_lengths=d.context_lengths,
                        stash=st, slot_stride=case.slot_stride, P=case.P)

    flop = tokens * H * Dm * N * 5       # per state element: mul + FMA update, FMA output
    sm = torch.cuda.get_device_properties(device).multi_processor_count
    alu_peak = sm * 128 * 2 * 1.965e9 / 1e12   # fp32 FMA lanes x 2 FLOP x max SM clock
    tc = (case.x.dtype == torch.bfloat16 and case.B.dtype == torch.bfloat16 and N == 128
          and Dm % 8 == 0)
    # chunked tensor-core form: per (row, head, 64-row dim tile) and chunk of 128 tokens,
    # C s^T and G X (3 pieces x 8 K-steps of M128 N64 K16 each), C B^T (8 of M128 N128 K16)
    # and B^T (w dt X) (3 x 8 of M128 N64 K16)
    chunks = int(sum(-(-int(L) // 128) for L in case.context_lengths.tolist()))
    mma_flop = chunks * H * -(-Dm // 64) * (72 * 2 * 128 * 64 * 16 + 8 * 2 * 128 * 128 * 16)
    tc_peak, tc_src = measured_bf16_tflops()
    forms = {}
    for name, st in (("prefill", None), ("prefill_stash", stash)):
        ms = time_launches(lambda: prefill(st), steps, warm, device)
        # algorithmic bytes: x, z and out (and with the stash U, dA and dt) per valid
        # token-head, B and C per token (and the stash's B), the state read (and written)
        xb = case.x.element_size()
        io = tokens * H * Dm * xb * 3 + tokens * H * 4 + tokens * G * N * xb * 2
        if st is not None:
            io += tokens * H * Dm * 4 + tokens * H * 8 + tokens * G * N * 4
        state = b * H * Dm * N * 4 * (1 if st is not None else 2)
        forms[name] = {
            "workload": "prefill_b16_t512", "batch": b, "tokens": tokens, "ms_per_launch": ms,
            "tokens_per_s": tokens / (ms / 1e3),
            "form": "chunked tensor-core" if tc else "sequential CUDA-core",
            "roofline": {"bound": "alu", "achieved": flop / (ms / 1e3) / 1e12,
                         "peak": alu_peak, "unit": "TFLOP/s",
                         "frac": flop / (ms / 1e3) / 1e12 / alu_peak, "traffic": None,
                         "peak_source": "derived: SMs x 128 FP32 lanes x 2 FLOP x 1965 MHz",
                         "flop_count": "5 per state element and token (sequential form)"},
            "hbm": {"algorithmic_bytes": io + state,
                    "achieved_gbs": (io + state) / (ms / 1e3) / 1e9,
                    "frac_of_measured": (io + state) / (ms / 1e3) / 1e9 / measured_peaks()[0]}}
        if tc:
            forms[name]["tensor"] = {"mma_flop_issued": mma_flop,
                                     "achieved_tflops": mma_flop / (ms / 1e3) / 1e12,
                                     "bf16_peak": tc_peak, "bf16_peak_source": tc_src,
                                     "frac": mma_flop / (ms / 1e3) / 1e12 / tc_peak}
    return forms


def form_replay(args, device, hbm_peak, batch=0):
    """Speculative replay (batch 64, 5 drafted tokens, acceptedLengths ~ U{0..5}); the stash
    comes from this library's prefill in stash mode. HBM bound."""
    from linear_attention_recurrent_selective_b200 import ssu
    from linear_attention_recurrent_selective_b200.workloads import make_config

    steps, warm = max(3, min(args.steps, 50)), max(3, min(args.warmup, 5))
    f = dict(dtype=torch.float32, device=device)
    rcase = make_config("spec_replay_b64_t5", **(dict(batch=batch, P=2 * batch) if batch else {}))
    rd = rcase.to(device)
    rpool = rd.pool.clone()
    b, T, H, G, Dm, N = rcase.batch, rcase.T, rcase.H, rcase.G, rcase.Dm, rcase.N
    rst = (torch.empty(b, T, H, **f), torch.empty(b, T, H, Dm, **f),
           torch.empty(b, T, G, N, **f), torch.empty(b, T, H, **f))
    rout = torch.empty_like(rd.x)
    ssu.ssu_prefill(rd.x, rd.A, rd.B, rd.C, rd.dt, rpool, rout, dt_bias=rd.dt_bias, D=rd.D,
                    z=rd.z, state_indices=rd.state_indices, stash=rst,
                    slot_stride=rcase.slot_stride, P=rcase.P)
    acc = rd.accepted_lengths
    ms = time_launches(lambda: ssu.ssu_replay(rpool, rst, acc, state_indices=rd.state_indices,
                                              slot_stride=rcase.slot_stride, P=rcase.P),
                       steps, warm, device)
    acc_h = rcase.accepted_lengths
    rows = int((acc_h > 0).sum())
    nacc = int(acc_h.sum())
    rbytes = rows * H * Dm * N * 4 * 2 + nacc * (H * (4 + 4 + Dm * 4) + G * N * 4) + b * 4
    return {"replay": {
        "workload": "spec_replay_b64_t5", "batch": b, "accepted_tokens": nacc,
        "ms_per_launch": ms, "accepted_tokens_per_s": nacc / (ms / 1e3),
        "algorithmic_bytes": rbytes,
        "roofline": {"bound": "hbm", "achieved": rbytes / (ms / 1e3) / 1e9,
                     "peak": hbm_peak, "unit": "GB/s",
                     "frac": rbytes / (ms / 1e3) / 1e9 / hbm_peak, "traffic": None}}}


def form_layers(args, device, hbm_peak):
    """Multi-layer launches and row movement on one GPU: the speculative replay over 8
    layers in one launch, the gather of the batch-256 decode rows into a dense batch, and
    the clear of one slot across 64 layers. All HBM bound."""
    from linear_attention_recurrent_selective_b200 import ssu
    from linear_attention_recurrent_selective_b200.workloads import make_config

    steps, warm = max(3, min(args.steps, 50)), max(3, min(args.warmup, 5))
    forms = {}
    f = dict(dtype=torch.float32, device=device)

    # replay over 8 layers: each layer has its own pool and stash (stash from this
    # library's prefill in stash mode, one per layer)
    layers = 8
    rcase = make_config("spec_replay_b64_t5")
    rd = rcase.to(device)
    b, T, H, G, Dm, N = rcase.batch, rcase.T, rcase.H, rcase.G, rcase.Dm, rcase.N
    pools, stashes = [], []
    for _ in range(layers):
        pool = rd.pool.clone()
        st = (torch.empty(b, T, H, **f), torch.empty(b, T, H, Dm, **f),
              torch.empty(b, T, G, N, **f), torch.empty(b, T, H, **f))
        ssu.ssu_prefill(rd.x, rd.A, rd.B, rd.C, rd.dt, pool, torch.empty_like(rd.x),
                        dt_bias=rd.dt_bias, D=rd.D, z=rd.z, state_indices=rd.state_indices,
                        stash=st, slot_stride=rcase.slot_stride, P=rcase.P)
        pools.append(pool)
        stashes.append(st)
    table = ssu.replay_layer_table(list(zip(pools, stashes)))
    acc = rd.accepted_lengths
    ms = time_launches(lambda: ssu.ssu_replay_layers(table, layers, pools[0], stashes[0], acc,
                                                     state_indices=rd.state_indices,
                                                     slot_stride=rcase.slot_stride, P=rcase.P),
                       steps, warm, device)
    acc_h = rcase.accepted_lengths
    rows, nacc = int((acc_h > 0).sum()), int(acc_h.sum())
    per_layer = rows * H * Dm * N * 4 * 2 + nacc * (H * (4 + 4 + Dm * 4) + G * N * 4) + b * 4
    forms["replay_layers"] = {
        "workload": "spec_replay_b64_t5 x 8 layers", "ms_per_launch": ms,
        "accepted_tokens_per_s": layers * nacc / (ms / 1e3),
        "roofline": {"bound": "hbm", "achieved": layers * per_layer / (ms / 1e3) / 1e9,
                     "peak": hbm_peak, "unit": "GB/s",
                     "frac": layers * per_layer / (ms / 1e3) / 1e9 / hbm_peak, "traffic": None}}
    del pools, stashes, table

    # gather of the 256 active rows of the batch-256 decode pool (2.6 MB slots)
    dcase = make_config(WORKLOAD)
    dpool = dcase.pool.to(device).view(dcase.P, dcase.slot_stride)
    dense = torch.empty(dcase.batch, dcase.slot_stride, **f)
    idx = dcase.state_indices.to(device)
    ms = time_launches(lambda: ssu.pool_gather(dpool, dense, state_indices=idx), steps, warm,
                       device)
    gbytes = 2 * dense.numel() * 4
    forms["gather"] = {
        "workload": "mamba2_decode_b256 rows -> dense batch", "ms_per_launch": ms,
        "roofline": {"bound": "hbm", "achieved": gbytes / (ms / 1e3) / 1e9, "peak": hbm_peak,
                     "unit": "GB/s", "frac": gbytes / (ms / 1e3) / 1e9 / hbm_peak,
                     "traffic": None}}
    del dpool, dense

    # clear one slot (2.6 MB of state, 40 KB of conv state) across 64 layers
    nl, P, slot_elems, conv_elems = 64, 4, 80 * 64 * 128, 10240
    recs = [torch.ones(P, slot_elems, **f) for _ in range(nl)]
    convs = [torch.ones(P, conv_elems, dtype=torch.bfloat16, device=device) for _ in range(nl)]
    ltab = ssu.layer_states_table(list(zip(recs, convs)))
    ms = time_launches(lambda: ssu.pool_clear_slot_layers(ltab, nl, P, 1, slot_elems * 4,
                                                          conv_elems * 2), steps, warm, device)
    cbytes = nl * (slot_elems * 4 + conv_elems * 2)
    forms["clear_layers"] = {
        "workload": "one slot x 64 layers (fp32 state + bf16 conv)", "ms_per_launch": ms,
        "roofline": {"bound": "hbm", "achieved": cbytes / (ms / 1e3) / 1e9, "peak": hbm_peak,
                     "unit": "GB/s", "frac": cbytes / (ms / 1e3) / 1e9 / hbm_peak,
                     "traffic": None}}
    return forms


def form_conv(args, device, hbm_peak):
    """The batch-256 decode with the causal conv1d (width 4) of its raw xBC channels fused
    in (both launches of ssu_conv_decode); HBM bound."""
    from linear_attention_recurrent_selective_b200 import ssu
    from linear_attention_recurrent_selective_b200.workloads import make_config

    steps, warm = max(3, min(args.steps, 50)), max(3, min(args.warmup, 5))
    case = make_config("mamba2_conv_decode_b256",
                       **(dict(batch=args.batch, P=2 * args.batch) if args.batch else {}))
    d = case.to(device)
    b, H, G, Dm, N, W = case.batch, case.H, case.G, case.Dm, case.N, case.width
    out = torch.empty(b, H, Dm, dtype=case.xbc.dtype, device=device)

    def step():
        ssu.ssu_conv_decode(d.xbc, d.conv_w, d.conv_state, d.A, d.dt, d.pool, out, width=W,
                            conv_strides=case.conv_strides, nheads=H, ngroups=G, dim=Dm,
                            conv_bias=d.conv_b, dt_bias=d.dt_bias, D=d.D, z=d.z,
                            state_indices=d.state_indices, slot_stride=case.slot_stride,
                            P=case.P)

    ms = time_launches(step, steps, warm, device)
    xb = case.xbc.element_size()
    cd = H * Dm + 2 * G * N
    state_b = b * H * Dm * N * case.pool.element_size() * 2
    cbytes = (state_b + 2 * b * H * Dm * xb + b * cd * xb + 2 * b * cd * (W - 1) * xb
              + cd * (W + 1) * xb + b * H * 4)
    return {"conv_decode": {
        "workload": "mamba2_conv_decode_b256", "batch": b, "width": W, "ms_per_launch": ms,
        "seq_head_updates_per_s": b * H / (ms / 1e3), "algorithmic_bytes": cbytes,
        "launches": 2,
        "roofline": {"bound": "hbm", "achieved": cbytes / (ms / 1e3) / 1e9, "peak": hbm_peak,
                     "unit": "GB/s", "frac": cbytes / (ms / 1e3) / 1e9 / hbm_peak,
                     "traffic": None}}}


def form_gdn(args, device, hbm_peak):
    """Gated delta-rule decode (batch 256, 16 key / 32 value heads, 128 x 128 fp32 state per
    value head); HBM bound."""
    from linear_attention_recurrent_selective_b200 import ssu
    from linear_attention_recurrent_selective_b200.workloads import make_gdn_config

    steps, warm = max(3, min(args.steps, 50)), max(3, min(args.warmup, 5))
    case = make_gdn_config("gdn_decode_b256",
                           **(dict(batch=args.batch, P=2 * args.batch) if args.batch else {}))
    d = case.to(device)
    b, HK, HV, K, V = case.batch, case.HK, case.HV, case.K, case.V
    out = torch.empty(b, HV, V, dtype=case.q.dtype, device=device)

    def step():
        ssu.gdn_decode(d.q, d.k, d.v, d.a, d.b, d.A_log, d.pool, out, dt_bias=d.dt_bias,
                       state_indices=d.state_indices, slot_stride=case.slot_stride, P=case.P)

    ms = time_launches(step, steps, warm, device)
    xb = case.q.element_size()
    gbytes = (b * HV * V * K * 4 * 2 + 2 * b * HK * K * xb + 2 * b * HV * V * xb
              + 2 * b * HV * xb + b * 4)
    return {"gdn_decode": {
        "workload": "gdn_decode_b256", "batch": b, "ms_per_launch": ms,
        "seq_head_updates_per_s": b * HV / (ms / 1e3), "algorithmic_bytes": gbytes,
        "roofline": {"bound": "hbm", "achieved": gbytes / (ms / 1e3) / 1e9, "peak": hbm_peak,
                     "unit": "GB/s", "frac": gbytes / (ms / 1e3) / 1e9 / hbm_peak,
                     "traffic": None}}}


def form_ddtree(args, device, hbm_peak):
    """Tree verify of one 128-node draft tree per row (batch 16, random recursive trees),
    then the replay of each row's accepted root-to-node path through acceptedNodeIds.
    With bf16 B and C the verify's dense products run on the tensor cores (three bf16
    pieces of the fp32 state per product), so its binding roofline is HBM: the algorithmic
    bytes take longer at the measured copy bandwidth than the tensor work at the measured
    bf16 GEMM rate (reported beside it as "compute"). The replay is HBM bound."""
    from linear_attention_recurrent_selective_b200 import ssu
    from linear_attention_recurrent_selective_b200.workloads import make_config

    steps, warm = max(3, min(args.steps, 50)), max(3, min(args.warmup, 5))
    case = make_config("ddtree_b16_n128")
    d = case.to(device)
    f = dict(dtype=torch.float32, device=device)
    b, T, H, G, Dm, N = case.batch, case.T, case.H, case.G, case.Dm, case.N
    out = torch.empty_like(d.x)
    st = (torch.empty(b, T, H, **f), torch.empty(b, T, H, Dm, **f),
          torch.empty(b, T, G, N, **f), torch.empty(b, T, H, **f))

    def verify():
        ssu.ssu_ddtree(d.x, d.A, d.B, d.C, d.dt, d.pool, out, d.parent_ids, d.depths, st,
                       dt_bias=d.dt_bias, D=d.D, state_indices=d.state_indices,
                       slot_stride=case.slot_stride, P=case.P)

    ms = time_launches(verify, steps, warm, device)
    pairs = int((case.depths + 1).sum())          # (node, path node) pairs of all rows
    # dense a_i = s0 . C_i per node, head and dim row; the path sums per (pair, head, dim
    # row); C_i . B_j per (pair, group)
    flop = 2 * b * H * T * Dm * N + 2 * pairs * H * Dm + 2 * pairs * G * N
    xb = case.x.element_size()
    vbytes = (b * H * Dm * N * 4 + 2 * b * T * H * Dm * xb + b * T * H * Dm * 4
              + b * T * G * N * (2 * case.B.element_size() + 4) + b * T * H * 12 + 2 * b * T * 4)
    tc_peak, tc_src = measured_bf16_tflops()
    pieces = {torch.float32: 3, torch.float16: 2, torch.bfloat16: 1}[case.pool.dtype]
    tc_flop = 2 * b * H * 128 * Dm * N * pieces        # the MMAs as issued (128 node slots)
    gbs = vbytes / (ms / 1e3) / 1e9
    forms = {"ddtree": {
        "workload": "ddtree_b16_n128", "batch": b, "nodes": b * T, "path_pairs": pairs,
        "ms_per_launch": ms, "nodes_per_s": b * T / (ms / 1e3), "algorithmic_flop": flop,
        "algorithmic_bytes": vbytes,
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s",
                     "frac": gbs / hbm_peak, "traffic": None},
        "compute": {"unit": "TFLOP/s", "algorithmic": flop / (ms / 1e3) / 1e12,
                    "tensor_issued": tc_flop / (ms / 1e3) / 1e12, "bf16_peak": tc_peak,
                    "bf16_peak_source": tc_src,
                    "tensor_floor_ms": tc_flop / (tc_peak * 1e12) * 1e3,
                    "hbm_floor_ms": vbytes / (hbm_peak * 1e9) * 1e3}}}

    pool = d.pool.clone()
    acc, ids = d.accepted_lengths, d.accepted_node_ids
    rms = time_launches(lambda: ssu.ssu_replay(pool, st, acc, state_indices=d.state_indices,
                                               slot_stride=case.slot_stride, P=case.P,
                                               accepted_node_ids=ids), steps, warm, device)
    acc_h = case.accepted_lengths
    rows, nacc = int((acc_h > 0).sum()), int(acc_h.sum())
    rbytes = rows * H * Dm * N * 4 * 2 + nacc * (H * (4 + 4 + Dm * 4) + G * N * 4) + b * 4
    forms["replay_nodes"] = {
        "workload": "ddtree_b16_n128 accepted paths", "accepted_tokens": nacc,
        "ms_per_launch": rms, "accepted_tokens_per_s": nacc / (rms / 1e3),
        "roofline": {"bound": "hbm", "achieved": rbytes / (rms / 1e3) / 1e9, "peak": hbm_peak,
                     "unit": "GB/s", "frac": rbytes / (rms / 1e3) / 1e9 / hbm_peak,
                     "traffic": None}}
    return forms


def cpu_model() -> str:
    """The host CPU's model name from /proc/cpuinfo (empty when unavailable)."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return ""


def _time_oracle_steps(oracle, case, threads, budget_s, max_steps):
    """Whole decode steps of the oracle on `threads` threads until budget_s has passed
    (at least one step). Returns (steps, seconds, threads used)."""
    used = oracle.set_threads(threads)
    pool = case.pool.clone()             # updated in place step after step, like the GPU's
    runs, t0 = 0, time.perf_counter()
    while True:
        oracle.decode_case(case, pool=pool)
        runs += 1
        el = time.perf_counter() - t0
        if el > budget_s or runs >= max_steps:
            return runs, el, used


def cpu_baseline_decode(case, budget_s=8.0):
    """The float64 oracle on whole decode steps of the same workload, timed on this host:
    on every host core (the reported value; the oracle's (row, head) units run on OpenMP
    threads) and on one thread, each for about budget_s seconds."""
    from oracle import oracle
    oracle.build()
    units = case.batch * case.H
    before = oracle.threads()
    try:
        runs_n, el_n, cores = _time_oracle_steps(oracle, case, 0, budget_s, 1000)
        runs_1, el_1, _ = _time_oracle_steps(oracle, case, 1, budget_s, 1000)
    finally:
        oracle.set_threads(before)
    model = cpu_model()
    return {"value": units * runs_n / el_n, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{runs_n} full decode step(s) of the batch-{case.batch} workload "
                      f"({units} seq-head updates each) on {cores} threads, {el_n:.1f} s",
            "host_cores": oracle.host_cores(), "cpu_model": model,
            "single_thread": {"value": units * runs_1 / el_1, "unit": UNIT, "cores": 1,
                              "sample": f"{runs_1} full decode step(s), one thread, "
                                        f"{el_1:.1f} s"}}


def config_block(case, res=None):
    c = {"workload": WORKLOAD, "batch": case.batch, "pool_slots": case.P, "nheads": case.H,
         "dim": case.Dm, "dstate": case.N, "ngroups": case.G, "state_dtype": "f32",
         "io_dtype": str(case.x.dtype).replace("torch.", ""), "z_gate": case.z is not None,
         "dt_softplus": case.dt_softplus, "parallelism": "replicas"}
    if res is not None:
        c["l2"] = (f"state per step {res['state_b'] / 1e6:.0f} MB vs L2 {res['l2'] / 1e6:.0f} MB: "
                   + ("L2 flushed between steps" if res["flush"] else "inputs larger than L2, no flush"))
    return c


def main_ours(args):
    n_world, rank, local = world()
    if n_world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local if n_world > 1 else torch.cuda.current_device())
    torch.cuda.set_device(device)
    hbm_peak, peak_src = measured_peaks()
    if args.form in ("prefill", "replay", "layers", "ddtree", "conv", "gdn"):   # one form
        if args.form == "prefill":
            forms = form_prefill(args, device, args.batch)
        elif args.form == "replay":
            forms = form_replay(args, device, hbm_peak, args.batch)
        elif args.form == "ddtree":
            forms = form_ddtree(args, device, hbm_peak)
        elif args.form == "conv":
            forms = form_conv(args, device, hbm_peak)
        elif args.form == "gdn":
            forms = form_gdn(args, device, hbm_peak)
        else:
            forms = form_layers(args, device, hbm_peak)
        if rank == 0:
            print(json.dumps({"form": args.form, "forms": forms}), flush=True)
        return

    res = run_decode(args, device)
    case = res["case"]
    t_max = max_over_ranks(res["total_ms"], device)
    e2e_max = max_over_ranks(res["e2e_ms"], device)
    value = job_throughput(res["units"], args.steps, n_world, t_max / 1e3)
    e2e_value = job_throughput(res["units"], args.steps, n_world, e2e_max / 1e3)
    achieved = res["alg_b"] / (res["kern_ms"] / 1e3) / 1e9

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": n_world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_max / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic", "config": config_block(case, res),
        "state_hbm_gbs": res["state_b"] / (res["kern_ms"] / 1e3) / 1e9,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak, "traffic": recorded_traffic(case.batch),
                     "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)"
                     if peak_src == "measured" else "fallback 6.65 TB/s",
                     "kernel": "ssu_decode_kernel", "kernel_ms": res["kern_ms"],
                     "algorithmic_bytes": res["alg_b"]},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": res["h2d"],
                "d2h_bytes_per_step": res["d2h"],
                "copies": "pinned host inputs in and the output back every step, on separate "
                          "streams, double-buffered so they overlap the neighbouring steps' "
                          "compute"},
        "gpu_launches": args.steps,
        "clocks": {**res["clocks"], "sustained": res["clocks_sustained"]},
    }
    if n_world == 1 and not args.no_forms and args.form == "all":
        line["forms"] = {**form_prefill(args, device), **form_replay(args, device, hbm_peak),
                         **form_layers(args, device, hbm_peak),
                         **form_ddtree(args, device, hbm_peak), **form_conv(args, device, hbm_peak),
                         **form_gdn(args, device, hbm_peak)}
    if n_world == 1 and rank == 0 and not args.no_cpu_baseline and args.form == "all":
        line["cpu_baseline"] = cpu_baseline_decode(case)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if n_world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ----------------------------------------------------------------------------- reference arm

def main_reference(args):
    """The float64 CPU oracle as the reference arm: rank 0 only, on every host core, each
    step the whole decode workload or, on a small host, a bounded row sample of it."""
    n_world, rank, _ = world()
    if rank != 0:
        return
    import dataclasses
    from linear_attention_recurrent_selective_b200.workloads import make_config
    from oracle import oracle
    oracle.build()
    cores = oracle.set_threads(0)
    case = make_config(WORKLOAD)
    # one probe step on a 16-row sample sets the row count: the whole run near a minute
    probe = 16
    pick = {f: getattr(case, f)[:probe].contiguous()
            for f in ("x", "z", "B", "C", "dt", "state_indices")}
    pool = case.pool.clone()             # updated in place step after step, like the GPU's
    t0 = time.perf_counter()
    oracle.decode_case(dataclasses.replace(case, batch=probe, active=probe, **pick), pool=pool)
    per_row = (time.perf_counter() - t0) / probe
    rows = max(1, min(case.batch, int(60.0 / max(1, args.steps + args.warmup) / per_row)))
    sub = case
    if rows < case.batch:
        pick = {f: getattr(case, f)[:rows].contiguous()
                for f in ("x", "z", "B", "C", "dt", "state_indices")}
        sub = dataclasses.replace(case, batch=rows, active=rows, **pick)
    for _ in range(args.warmup):
        oracle.decode_case(sub, pool=pool)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.decode_case(sub, pool=pool)
    el = time.perf_counter() - t0
    units = rows * case.H * args.steps
    value = units / el
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": n_world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_block(case), "impl": "reference",
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{rows} of {case.batch} rows x {case.H} heads per step",
                         "host_cores": oracle.host_cores(), "cpu_model": cpu_model()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def parse(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the batch (pool = 2 x batch), e.g. for a small profile")
    ap.add_argument("--no-forms", action="store_true", help="skip the prefill/replay forms")
    ap.add_argument("--form", choices=("all", "decode", "prefill", "replay", "layers", "ddtree",
                                       "conv", "gdn"),
                    default="all",
                    help="run one kernel only (for profiling); its line carries that form")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clock-window", action="store_true",
                    help="skip the >= 0.5 s clock-sampling window after the timed region "
                         "(for profiler runs)")
    a = ap.parse_args(argv)
    if a.warmup < 3 and a.impl == "ours":
        ap.error("--warmup must be at least 3")
    return a


if __name__ == "__main__":
    args = parse()
    if args.impl == "reference":
        main_reference(args)
    else:
        main_ours(args)
