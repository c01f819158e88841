#!/usr/bin/env python
"""Throughput of the SSD mixer scan on B200: tokens/s, roofline fraction,
decode-step GB/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one ssd_forward over the headline workload, long_7b (a 7B-class
Mamba-2 layer: batch 2 x 16384 tokens, 128 heads x 64, d_state 128, 8 B/C
groups, conv 4, nonzero initial state) -- the largest configuration that fits
one GPU -- with its inputs resident in HBM; the whole hot path runs in the
library's kernels (conv, dt/cumsum, chunk scan with state passing, gated
output, final state).  Rank 0 prints one JSON line.  With N > 1 (torchrun)
every rank runs its own batch -- the scan has no cross-row exchange -- so the
scaling is weak and `value` counts every rank's tokens over the slowest rank's
device time.

The timed region is the K-step loop, run R times back to back (R chosen so the
region lasts at least half a second and the clock sampler sees it); every
repetition times exactly K steps and `ms_per_step` is their mean.

Extra keys: `roofline` (dominant kernel against measured HBM bandwidth),
`forward_roofline` (whole forward against its compulsory bytes), `configs`
(the same measurement, rooflines and CPU baseline for mini_k3_mixer and
mamba3_siso), `decode` (decode_b256 single-token step, GB/s), `backward`
(ssd_backward on mini_k3_mixer), `packed_gated_norm` (the forward on a packed
in_proj input followed by the gated RMSNorm), `e2e` (host
buffers, copies inside the timed region), `cpu_baseline` (the fp64 oracle on
this host's cores), `clocks` (SM clock and throttle reasons sampled during the
timed region).  `cpu_baseline.single_thread` gives the oracle's one-thread
rate on one (row, head) pair of the workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "SSD mixer tokens/s (B·L/s) at 1 B200 and % of roofline; decode-step GB/s"
WORKLOAD = "long_7b"                        # the headline configuration
EXTRA_WORKLOADS = ("mini_k3_mixer", "mamba3_siso")
MIN_TIMED_S = 0.5                            # shortest timed region (clock samples)
DECODE_WORKLOAD = "decode_b256"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "kernel_traffic.json")


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--path", choices=["auto", "fused", "staged"], default="auto")
    p.add_argument("--no-decode", action="store_true", help="skip the decode measurement")
    p.add_argument("--no-e2e", action="store_true", help="skip the host-buffer measurement")
    p.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    p.add_argument("--no-s6", action="store_true", help="skip the Mamba-1 (S6) scan measurement")
    p.add_argument("--no-backward", action="store_true",
                   help="skip the backward and the packed-input gated-norm measurements")
    p.add_argument("--workload", default=WORKLOAD,
                   choices=["long_7b", "mini_k3_mixer", "mamba3_siso"],
                   help="the workload of the headline measurement (default long_7b)")
    p.add_argument("--min-timed-s", type=float, default=MIN_TIMED_S,
                   help="shortest timed region in seconds (the K-step loop is repeated)")
    p.add_argument("--no-extra", action="store_true",
                   help="time the headline workload only (skip mini_k3_mixer and mamba3_siso)")
    return p.parse_args(argv)


# ---------------------------------------------------------------------------------------
# distributed plumbing (one process per GPU; also exercised with gloo on CPU by the tests)
def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def dist_init(backend: str):
    import datetime
    import torch.distributed as dist
    rank, world, _ = dist_env()
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=180))
    return rank, world


def aggregate(local_ms: float, local_units: float, world: int, device=None):
    """(max over ranks of the device time, sum over ranks of the units processed)."""
    if world <= 1:
        return local_ms, local_units
    import torch
    import torch.distributed as dist
    t = torch.tensor([local_ms], dtype=torch.float64, device=device)
    u = torch.tensor([local_units], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(t.item()), float(u.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------------------------
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS)


def kernel_source_hash(path_kind: str) -> str:
    """Hash of the sources that make up the dominant kernel of a path."""
    files = {"fused": ["chunk_fused.cu", "ssd_device.cuh", "tc05.cuh"],
             "staged": ["chunk_staged.cu", "staged_rows.cuh", "ssd_device.cuh"],
             "decode": ["decode.cu", "ssd_device.cuh", "tc05.cuh"]}[path_kind]
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "selective_state_space_forward_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(kernel_key: str, path_kind: str, scale: float = 1.0):
    """DRAM bytes per launch from the committed ncu summary, or None when the
    summary is missing or was taken on other kernel sources."""
    try:
        with open(PROFILE_SUMMARY) as f:
            d = json.load(f)
        e = d[kernel_key]
    except (OSError, KeyError, ValueError):
        return None
    if e.get("source_hash") != kernel_source_hash(path_kind):
        return None
    return float(e["dram_bytes_per_launch"]) * scale


class ClockSampler:
    """SM clock and throttle reasons, sampled by NVML while the timed region runs."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._dev = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._dev = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._dev, pynvml.NVML_CLOCK_SM)
        except Exception as e:   # NVML missing: report that, keep benchmarking
            self.error = str(e)
        self._period = period_s
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._dev,
                                                                    self._nv.NVML_CLOCK_SM))
                r = self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._dev)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self._period)

    def __enter__(self):
        if self._dev is not None:
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._dev is not None:
            self._t.join()

    def summary(self):
        if self._dev is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": self.error}
        s = sorted(self.samples)
        med = s[len(s) // 2] if s else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(s)}


# ---------------------------------------------------------------------------------------
def _device_inputs(w, inp, torch):
    at = torch.bfloat16 if w.act_dtype == "bf16" else torch.float32
    dev = {}
    for k in ("x", "z", "B", "C", "conv_w", "conv_b"):
        dev[k] = None if inp.get(k) is None else torch.from_numpy(inp[k]).to(at).cuda()
    for k in ("dt_raw", "dt_bias", "A", "D", "B_norm_w", "C_norm_w", "B_bias", "C_bias"):
        dev[k] = None if inp.get(k) is None else torch.from_numpy(inp[k]).cuda()
    dev["seq_idx"] = None if inp.get("seq_idx") is None else torch.from_numpy(
        inp["seq_idx"]).cuda()
    return dev


def forward_bytes(w) -> dict:
    """Compulsory bytes of one forward of workload w (every input read once,
    every output written once, plus initial and final state)."""
    a = 2 if w.act_dtype == "bf16" else 4
    BL = w.batch * w.seqlen
    HP, GN, H = w.nheads * w.headdim, w.ngroups * w.dstate, w.nheads
    b = BL * (HP * a * 3 + 2 * GN * a + H * 4)            # x, z, out, B, C, dt_raw
    if w.a_per_token:
        b += BL * H * 4
    if w.documents != "none":
        b += BL * 4
    state = w.batch * H * w.headdim * w.dstate * 4
    b += state * (2 if w.init_state else 1)
    if w.dconv > 1:
        b += w.batch * 3 * w.conv_dim * a
    return {"bytes": b}


def main_kernel_bytes(w, path: str) -> int:
    """Algorithmic bytes of one launch of the dominant kernel of `path`."""
    a = 2 if w.act_dtype == "bf16" else 4
    BL = w.batch * w.seqlen
    HP, GN, H = w.nheads * w.headdim, w.ngroups * w.dstate, w.nheads
    nc = (w.seqlen + 63) // 64
    state = w.batch * H * w.headdim * w.dstate * 4
    seq = BL * 4 if w.documents != "none" else 0
    if path == "fused":
        # x (raw, for its conv), z, out, the conv'd B|C (or raw B, C), dt and acs, ids, state
        b = BL * (3 * HP * a + 2 * GN * a + 2 * H * 4) + seq + state
        if w.init_state:
            b += state
        if w.dconv > 1:
            b += w.batch * 3 * HP * a          # the x part of the conv history
        return b
    # staged chunk-output kernel: conv'd x|B|C (fp32) or raw, z, out, dt/acs, ids, Hin
    u = BL * (HP + 2 * GN) * (4 if w.dconv > 1 else a)
    return u + BL * (2 * HP * a + 2 * H * 4) + seq + w.batch * nc * H * w.headdim * w.dstate * 4


def _timed_loop(torch, stream, step, K: int, world: int, h=None, clk_index: int = 0,
                min_s: float = MIN_TIMED_S):
    """Run the K-step loop R times back to back inside one sampled region (R so
    that the region lasts at least min_s seconds); every repetition times exactly
    K steps with CUDA events on `stream`.  When a handle is given, its main
    kernel is bracketed by per-step events too.  Returns (mean ms per step,
    mean main-kernel ms or None, R, clocks summary, the handle's kernel launches
    in the whole timed region)."""
    probe0, probe1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    probe0.record(stream)
    for _ in range(K):
        step()
    probe1.record(stream)
    torch.cuda.synchronize()
    est = max(probe0.elapsed_time(probe1) / 1e3, 1e-6)
    R = max(1, int(-(-min_s // est)))
    if world > 1:       # every rank runs the same number of repetitions
        import torch.distributed as dist
        t = torch.tensor([R], dtype=torch.int64, device=torch.device("cuda", clk_index))
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        R = int(t.item())
    reps = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(R)]
    kev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(K)] for _ in range(R)] if h is not None else None
    for ev in [e for pair in reps for e in pair] + (
            [e for rep in kev for pair in rep for e in pair] if kev else []):
        ev.record(stream)          # materialise the events so their handles exist
    torch.cuda.synchronize()
    barrier(world)
    launches0 = h.launch_count() if h is not None else 0
    with ClockSampler(clk_index) as clk:
        for r in range(R):
            reps[r][0].record(stream)
            for i in range(K):
                if kev is not None:
                    h.set_timing_events(*kev[r][i])
                step()
            reps[r][1].record(stream)
        torch.cuda.synchronize()
    launches = (h.launch_count() - launches0) if h is not None else None
    if h is not None:
        h.set_timing_events(None, None)
    barrier(world)
    ms = sum(a.elapsed_time(b) for a, b in reps) / (R * K)
    kern = (sum(a.elapsed_time(b) for rep in kev for a, b in rep) / (R * K)) if kev else None
    return ms, kern, R, clk.summary(), launches


def bench_forward(args, torch, rank, world, local_rank, peaks, wname=WORKLOAD):
    from selective_state_space_forward_b200 import ssd
    from selective_state_space_forward_b200.synthetic import WORKLOADS, make_inputs
    w = WORKLOADS[wname]
    inp = make_inputs(w)
    dev = _device_inputs(w, inp, torch)
    h = ssd.Handle(w.nheads, w.headdim, w.dstate, w.ngroups, w.dconv, w.act_dtype,
                   a_per_token=w.a_per_token, bc_norm=w.bc_norm, max_batch=w.batch,
                   max_seqlen=w.seqlen, path=args.path)
    if w.bc_norm:
        h.set_bc_norm(dev["B_norm_w"], dev["C_norm_w"], dev["B_bias"], dev["C_bias"])
    init = None
    if inp.get("init_ssm") is not None:
        init = h.new_state(w.batch)
        ssm, _ = h.state_views(init, w.batch)
        ssm.copy_(torch.from_numpy(inp["init_ssm"]))
    fin = h.new_state(w.batch)
    out = torch.empty_like(dev["x"])
    stream = torch.cuda.current_stream()

    def step():
        h.forward(dev["x"], dev["z"], dev["dt_raw"], dev["dt_bias"], dev["A"], dev["B"],
                  dev["C"], dev["D"], dev["conv_w"], dev["conv_b"], seq_idx=dev["seq_idx"],
                  init_state=init, out=out, final_state=fin, stream=stream)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    K = args.steps
    local_ms, kern_ms, R, clocks, launches = _timed_loop(torch, stream, step, K, world, h,
                                                         local_rank, args.min_timed_s)
    h.check()
    max_ms, total_tokens = aggregate(local_ms, w.tokens, world,
                                     device=torch.device("cuda", local_rank))

    kb = main_kernel_bytes(w, h.path)
    achieved = kb / (kern_ms * 1e-3) / 1e9
    traffic = measured_traffic(f"{h.path}:{wname}", h.path)
    fb = forward_bytes(w)["bytes"]
    roof_ms = fb / (peaks["hbm_gbs"] * 1e9) * 1e3
    res = {
        "value": total_tokens / (max_ms * 1e-3),
        "ms_per_step": max_ms,
        "repeats": R,
        "tokens_per_rank": w.tokens,
        "path": h.path,
        "launches": launches,
        "launches_per_step": launches / (R * K) if launches is not None else None,
        "clocks": clocks,
        "roofline": {"bound": "hbm", "kernel": "ssd_chunk_fused" if h.path == "fused"
                     else "chunk_output_kernel", "achieved": round(achieved, 1),
                     "peak": peaks["hbm_gbs"], "peak_source": peaks["source"], "unit": "GB/s",
                     "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": traffic,
                     "algorithmic_bytes": kb, "kernel_ms": round(kern_ms, 4)},
        "forward_roofline": {"compulsory_bytes": fb, "roofline_ms": round(roof_ms, 4),
                             "roofline_tokens_per_s": w.tokens / (roof_ms * 1e-3),
                             "frac": round(roof_ms / local_ms, 4)},
    }
    return res, (w, inp, h, dev, out, fin, init)


def bench_e2e(args, torch, ctx, world, local_rank):
    """Same forward through the public call with the step's inputs in pinned host
    memory: every step's H2D copies, the call, and the D2H read of its output are
    inside the timed region.  Steps are pipelined the way a serving loop runs
    them: device inputs and outputs are double-buffered, the inputs of step k+1
    are copied in on one stream while step k computes on the handle's stream
    and step k-1's output is read back on a third (the two copy directions use
    separate copy engines).  The serial form (one stream, copy in, call, copy
    out) is timed too and reported beside it."""
    w, inp, h, dev, out, fin, init = ctx
    stream = torch.cuda.current_stream()
    keys = ["x", "z", "B", "C", "dt_raw"] + (["seq_idx"] if dev["seq_idx"] is not None else []) + (
        ["A"] if w.a_per_token else [])
    host = {k: dev[k].cpu().pin_memory() for k in keys}
    dbufs = [{k: torch.empty_like(dev[k]) for k in keys} for _ in range(2)]
    outs = [out, torch.empty_like(out)]
    houts = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    bi = sum(t.numel() * t.element_size() for t in host.values())
    bo = houts[0].numel() * houts[0].element_size()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def call(d, o):
        h.forward(d["x"], d["z"], d["dt_raw"], dev["dt_bias"], d["A"] if w.a_per_token else dev["A"],
                  d["B"], d["C"], dev["D"], dev["conv_w"], dev["conv_b"], seq_idx=d.get("seq_idx"),
                  init_state=init, out=o, final_state=fin, stream=stream)

    def step_pipelined(i):
        j = i % 2
        s_in.wait_event(ev_done[j])          # step i-2 has read this slot's inputs
        with torch.cuda.stream(s_in):
            for k in keys:
                dbufs[j][k].copy_(host[k], non_blocking=True)
        ev_in[j].record(s_in)
        stream.wait_event(ev_in[j])
        stream.wait_event(ev_out[j])         # step i-2's output has been read back
        call(dbufs[j], outs[j])
        ev_done[j].record(stream)
        s_out.wait_event(ev_done[j])
        with torch.cuda.stream(s_out):
            houts[j].copy_(outs[j], non_blocking=True)
        ev_out[j].record(s_out)

    def step_serial(i):
        for k in keys:
            dbufs[0][k].copy_(host[k], non_blocking=True)
        call(dbufs[0], outs[0])
        houts[0].copy_(outs[0], non_blocking=True)

    K = max(3, min(args.steps, 20))
    res = {}
    for name, step in (("serial", step_serial), ("pipelined", step_pipelined)):
        for i in range(3):
            step(i)
        torch.cuda.synchronize()
        barrier(world)
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        s_in.wait_event(t0)
        s_out.wait_event(t0)
        for i in range(K):
            step(i)
        stream.wait_event(ev_out[0])
        stream.wait_event(ev_out[1])
        t1.record(stream)
        torch.cuda.synchronize()
        res[name] = t0.elapsed_time(t1) / K
    max_ms, tot = aggregate(res["pipelined"], w.tokens, world, device=torch.device("cuda", local_rank))
    ser_ms, ser_tot = aggregate(res["serial"], w.tokens, world, device=torch.device("cuda", local_rank))
    return {"value": tot / (max_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": bi,
            "d2h_bytes_per_step": bo, "ms_per_step": max_ms, "steps": K,
            "pipelining": "inputs copied in on one stream, the call on the handle's stream, the output "
                          "read back on a third; device buffers double-buffered",
            "serial": {"value": ser_tot / (ser_ms * 1e-3), "ms_per_step": ser_ms}}


def bench_decode(args, torch, peaks):
    """decode_b256: a 2048-token prefill, then single-token steps; each step's
    decode kernel is timed alone with L2 flushed before it (the fp32 state is
    just above L2's size, so without the flush part of it would be re-read
    from L2)."""
    from selective_state_space_forward_b200 import ssd
    from selective_state_space_forward_b200.synthetic import WORKLOADS, make_inputs, make_step_inputs
    w = WORKLOADS[DECODE_WORKLOAD]
    inp = make_inputs(w)
    dev = _device_inputs(w, inp, torch)
    h = ssd.Handle(w.nheads, w.headdim, w.dstate, w.ngroups, w.dconv, w.act_dtype,
                   max_batch=w.batch, max_seqlen=w.seqlen, path=args.path)
    state = h.new_state(w.batch)
    h.forward(dev["x"], dev["z"], dev["dt_raw"], dev["dt_bias"], dev["A"], dev["B"], dev["C"],
              dev["D"], dev["conv_w"], dev["conv_b"], final_state=state)
    del dev["x"], dev["z"], dev["B"], dev["C"], dev["dt_raw"]
    torch.cuda.synchronize()
    torch.cuda.empty_cache()      # the prefill's inputs are not needed by the steps
    steps_in = []
    for i in range(8):
        si = make_step_inputs(w, i)
        steps_in.append({k: torch.from_numpy(v).to(torch.bfloat16 if k in "xzBC" else
                                                     torch.float32).cuda() for k, v in si.items()})
    out = torch.empty(w.batch, w.nheads * w.headdim, dtype=torch.bfloat16, device="cuda")
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def step(i):
        s = steps_in[i % len(steps_in)]
        h.step(s["x"], s["z"], s["dt_raw"], dev["dt_bias"], dev["A"], s["B"], s["C"], dev["D"],
               dev["conv_w"], dev["conv_b"], state=state, out=out, stream=stream)

    for i in range(10):
        step(i)
    n = w.decode_steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(n)]
    for a_, b_ in ev:
        a_.record(stream)
        b_.record(stream)
    torch.cuda.synchronize()
    flush.fill_(1)
    for i in range(n):
        # evict the state by READING a buffer larger than L2: a write would
        # leave dirty lines whose write-back the timed step would pay for
        flush_sum = flush.sum(dtype=torch.int64)
        h.set_timing_events(*ev[i])
        step(i)
    torch.cuda.synchronize()
    del flush_sum
    h.set_timing_events(None, None)
    h.check()
    times = sorted(a_.elapsed_time(b_) for a_, b_ in ev)
    med_ms = times[len(times) // 2]
    state_b = w.batch * w.nheads * w.headdim * w.dstate * 4
    # Size-matched reference: torch's own copy of a buffer the size of the fp32
    # state (the same bytes read and written as the state update), L2 evicted
    # the same way.  At this size a copy does not reach the long-copy peak.
    src = torch.rand(state_b // 4, device="cuda")
    dst = torch.empty_like(src)
    cev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(64)]
    for a_, b_ in cev:
        flush_sum = flush.sum(dtype=torch.int64)
        a_.record(stream)
        dst.copy_(src)
        b_.record(stream)
    torch.cuda.synchronize()
    del flush_sum, src, dst
    ctimes = sorted(a_.elapsed_time(b_) for a_, b_ in cev)
    copy_gbs = 2 * state_b / (ctimes[len(ctimes) // 2] * 1e-3) / 1e9
    conv_b = w.batch * 3 * w.conv_dim * 2
    io_b = w.batch * (3 * w.nheads * w.headdim * 2 + 2 * w.ngroups * w.dstate * 2 + w.nheads * 4)
    total = 2 * state_b + 2 * conv_b + io_b
    gbs = total / (med_ms * 1e-3) / 1e9
    return {"workload": f"{DECODE_WORKLOAD}: batch 256, 32 heads x 64, d_state 64, 8 groups, "
                        "conv 4, after a 2048-token prefill",
            "us_per_step_median": round(med_ms * 1e3, 2), "bytes_per_step": total,
            "gbs": round(gbs, 1), "frac_of_hbm": round(gbs / peaks["hbm_gbs"], 4),
            "peak_source": peaks["source"], "steps_timed": n, "l2": "evicted before each step by reading a 256 MB buffer",
            "copy_reference": {"what": "torch copy of a buffer the size of the fp32 state, L2 evicted the same way",
                               "bytes": 2 * state_b, "gbs": round(copy_gbs, 1),
                               "decode_frac_of_it": round(gbs / copy_gbs, 4)},
            "traffic": measured_traffic(f"decode:{DECODE_WORKLOAD}", "decode")}


def _event_ms(torch, fn, reps: int) -> float:
    """Median CUDA-event time of fn() on the current stream over `reps` calls."""
    ts = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    return sorted(ts)[len(ts) // 2]


def bench_backward(args, torch, peaks, wname="mini_k3_mixer"):
    """ssd_backward (zero-state prefill) over a full workload: the forward
    recompute on the staged kernels plus the backward kernels, timed as one
    call with CUDA events; the timing hook brackets the backward kernels alone.
    Compulsory bytes: x, z, B, C, dt_raw and gout read once, the fp32 gradients
    of x, z, B, C, dt_raw written once (weights and the small per-head vectors
    are negligible)."""
    from selective_state_space_forward_b200 import ssd
    from selective_state_space_forward_b200.synthetic import WORKLOADS, make_inputs, make_output_grad
    w = WORKLOADS[wname]
    inp = make_inputs(w)
    dev = _device_inputs(w, inp, torch)
    h = ssd.Handle(w.nheads, w.headdim, w.dstate, w.ngroups, w.dconv, w.act_dtype,
                   a_per_token=w.a_per_token, bc_norm=w.bc_norm, max_batch=w.batch,
                   max_seqlen=w.seqlen)
    gout = torch.from_numpy(make_output_grad(w, 11)).to(dev["x"].dtype).cuda()
    ws = torch.empty(h.backward_workspace_bytes(w.batch, w.seqlen), dtype=torch.uint8,
                     device="cuda")
    grads = {}

    def call():
        grads.update(h.backward(dev["x"], dev["z"], dev["dt_raw"], dev["dt_bias"], dev["A"],
                                dev["B"], dev["C"], dev["D"], dev["conv_w"], dev["conv_b"],
                                gout=gout, seq_idx=dev["seq_idx"], workspace=ws, grads=grads))

    for _ in range(3):
        call()
    torch.cuda.synchronize()
    ms = _event_ms(torch, call, max(5, min(args.steps, 20)))
    k0, k1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    k0.record()        # torch times only events it has recorded once itself
    k1.record()
    h.set_timing_events(k0, k1)
    call()
    torch.cuda.synchronize()
    kern_ms = k0.elapsed_time(k1)
    h.set_timing_events(None, None)
    h.check()
    a = 2 if w.act_dtype == "bf16" else 4
    BL, HP, GN, H = w.tokens, w.nheads * w.headdim, w.ngroups * w.dstate, w.nheads
    nbytes = BL * ((3 * HP + 2 * GN) * a + H * 4) + BL * (2 * HP + 2 * GN + H) * 4
    return {"workload": WORKLOAD_TEXT[wname], "ms_per_call": round(ms, 4),
            "backward_kernels_ms": round(kern_ms, 4), "tokens_per_s": BL / (ms * 1e-3),
            "roofline": {"bound": "hbm", "unit": "GB/s", "compulsory_bytes": nbytes,
                         "achieved": round(nbytes / (ms * 1e-3) / 1e9, 1),
                         "peak": peaks["hbm_gbs"], "peak_source": peaks["source"],
                         "frac": round(nbytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)},
            "arithmetic": "forward recompute on the staged kernels, then the backward kernels; "
                          "their contractions on the tensor cores (mma.sync tf32 operands, fp32 "
                          "accumulation) for bf16 activations, fp32 SIMT for fp32",
            "workspace_bytes": ws.numel()}


def bench_packed_norm(args, torch, peaks, wname="mini_k3_mixer"):
    """The forward reading a packed in_proj row [z | x | B | C | dt_raw] in place,
    followed by the gated RMSNorm (group d_inner / ngroups), against the plain
    contiguous forward on the same workload."""
    from selective_state_space_forward_b200 import ssd
    from selective_state_space_forward_b200.synthetic import WORKLOADS, make_inputs
    w = WORKLOADS[wname]
    inp = make_inputs(w)
    dev = _device_inputs(w, inp, torch)
    h = ssd.Handle(w.nheads, w.headdim, w.dstate, w.ngroups, w.dconv, w.act_dtype,
                   a_per_token=w.a_per_token, bc_norm=w.bc_norm, max_batch=w.batch,
                   max_seqlen=w.seqlen)
    bf = dev["x"].dtype
    packed = torch.cat([dev["z"], dev["x"], dev["B"], dev["C"], dev["dt_raw"].to(bf)], dim=2)
    del dev["x"], dev["z"], dev["B"], dev["C"]
    torch.cuda.empty_cache()
    HP = w.nheads * w.headdim
    weight = torch.ones(HP, device="cuda")
    out = torch.empty(w.batch, w.seqlen, HP, dtype=bf, device="cuda")
    fin = h.new_state(w.batch)
    h.set_gated_norm(weight, group_size=HP // w.ngroups)

    def call():
        h.forward_packed(packed, dev["dt_bias"], dev["A"], dev["D"], dev["conv_w"], dev["conv_b"],
                         seq_idx=dev["seq_idx"], out=out, final_state=fin)

    for _ in range(3):
        call()
    torch.cuda.synchronize()
    ms = _event_ms(torch, call, max(5, min(args.steps, 20)))
    h.check()
    fb = forward_bytes(w)["bytes"] + HP * 4
    return {"workload": WORKLOADS[wname].name + ": packed in_proj input (row stride "
                        f"{packed.shape[2]} bf16), gated RMSNorm over groups of {HP // w.ngroups}",
            "ms_per_step": round(ms, 4), "tokens_per_s": w.tokens / (ms * 1e-3),
            "forward_roofline": {"compulsory_bytes": fb,
                                 "frac": round(fb / (peaks["hbm_gbs"] * 1e9) / (ms * 1e-3), 4)},
            "note": "the norm re-reads and re-writes out once: the kernels move "
                    f"{fb + 2 * w.tokens * HP * 2} bytes against {fb} compulsory"}


# Mamba-1 selective scan (S6) at the Falcon-Mamba-7B mixer shape.
S6_SHAPE = dict(batch=2, seqlen=4096, d_inner=8192, dstate=16)


def bench_s6(args, torch, peaks, sm_mhz):
    """ssd_s6_forward over the Falcon-Mamba-7B mixer shape (bf16 u, z, B, C; fp32
    dt, A_log, D, states) drawn by the seeded generator the parity tests use,
    each call timed alone with CUDA events; the inputs (674 MB) are larger than
    L2.  Rooflines: HBM bytes, and the MUFU pipe at its rate measured on this
    GPU by a one-kernel probe (ssd_ex2_throughput), which takes the dstate
    exponentials of every (token, channel)."""
    from selective_state_space_forward_b200 import ssd
    from selective_state_space_forward_b200.synthetic import make_s6_inputs
    Bb, L, DI, N = (S6_SHAPE[k] for k in ("batch", "seqlen", "d_inner", "dstate"))
    inp = make_s6_inputs(Bb, L, DI, N, seed=9)
    dev = {k: (None if v is None else torch.from_numpy(v).to(
        torch.bfloat16 if k in ("u", "z", "B", "C") else torch.float32).cuda())
        for k, v in inp.items()}
    state = dev["init"].clone()
    out = torch.empty_like(dev["u"])

    def call():
        ssd.s6_forward(dev["u"], dev["delta"], dev["delta_bias"], dev["A_log"], dev["B"],
                       dev["C"], dev["D"], z=dev["z"], init_state=state, out=out,
                       final_state=state)

    for _ in range(3):
        call()
    torch.cuda.synchronize()
    ms = _event_ms(torch, call, max(5, min(args.steps, 20)))
    tc = Bb * L * DI
    nbytes = tc * (2 + 4 + 2 + 2) + 2 * Bb * L * N * 2 + 2 * Bb * DI * N * 4
    exps = tc * N                                   # the state decays
    rate = ssd.ex2_throughput()                     # measured exp2 results/s
    mhz = sm_mhz or 1965
    return {"workload": "falcon_mamba_7b_mixer: Mamba-1 selective scan, batch 2 x 4096 tokens, "
                        "d_inner 8192, d_state 16, bf16 u/z/B/C, fp32 dt/A/D/state",
            "ms_per_call": round(ms, 4), "tokens_per_s": Bb * L / (ms * 1e-3),
            "roofline": {"bound": "alu", "unit": "G exp2/s (MUFU)",
                         "achieved": round(exps / (ms * 1e-3) / 1e9, 1),
                         "peak": round(rate / 1e9, 1), "frac": round(exps / (ms * 1e-3) / rate, 4),
                         "peak_source": "measured by ssd_ex2_throughput on this GPU "
                                        f"({rate / 148 / (mhz * 1e6):.2f} results/clk/SM at "
                                        f"{mhz} MHz)"},
            "hbm": {"algorithmic_bytes": nbytes, "gbs": round(nbytes / (ms * 1e-3) / 1e9, 1),
                    "frac_of_hbm": round(nbytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)},
            "inputs": "make_s6_inputs(seed 9), the parity tests' generator",
            "l2": "inputs larger than L2 (674 MB), no flush"}


# ---------------------------------------------------------------------------------------
_INPUT_CACHE = {}


def _inputs(wname):
    from selective_state_space_forward_b200.synthetic import WORKLOADS, make_inputs
    if wname not in _INPUT_CACHE:
        _INPUT_CACHE[wname] = make_inputs(WORKLOADS[wname])
    return _INPUT_CACHE[wname]


def cpu_oracle_run(wname: str = WORKLOAD, max_seconds: float | None = None):
    """The fp64 oracle on this host's cores over (part of) workload `wname`.
    Returns (tokens-equivalent per second, description, threads, seconds)."""
    import oracle
    from selective_state_space_forward_b200.synthetic import WORKLOADS
    w = WORKLOADS[wname]
    inp = _inputs(wname)
    cores = oracle.default_threads()
    pairs = [(b, hh) for b in range(w.batch) for hh in range(w.nheads)]
    L = w.seqlen
    if max_seconds is not None:
        # calibrate one pair on 512 tokens, then size the sample to the budget
        t0 = time.time()
        oracle.forward(w.with_(seqlen=512).dims(), _cut(inp, 512), pairs=[(0, 0)], threads=1,
                       final=False)
        per_tok = (time.time() - t0) / 512
        npairs = min(len(pairs), cores)
        L = int(max(64, min(w.seqlen, max_seconds / max(per_tok, 1e-9))) // 64 * 64)
        pairs = pairs[:npairs]
        inp = _cut(inp, L)
    dims = w.with_(seqlen=L).dims()
    t0 = time.time()
    r = oracle.forward(dims, inp, pairs=pairs, threads=0, final=True)
    dt = time.time() - t0
    tokens_equiv = len(pairs) * L / w.nheads
    desc = (f"{len(pairs)} (row, head) pairs of {wname} over {L} tokens each "
            f"(= {tokens_equiv:.0f} full-width tokens of {w.nheads} heads), fp64")
    return tokens_equiv / dt, desc, r["threads"], dt


def cpu_oracle_single_thread(wname: str = WORKLOAD) -> dict:
    """One host thread of the oracle on one (row, head) pair of workload `wname`
    over its full length; tokens/s in full-width tokens (all heads)."""
    import oracle
    from selective_state_space_forward_b200.synthetic import WORKLOADS
    w = WORKLOADS[wname]
    t0 = time.time()
    oracle.forward(w.dims(), _inputs(wname), pairs=[(0, 0)], threads=1, final=True)
    dt = time.time() - t0
    tokens = w.seqlen / w.nheads
    return {"tokens_per_s": tokens / dt, "seconds": round(dt, 4),
            "sample": f"1 (row, head) pair x {w.seqlen} tokens of {wname}, 1 thread"}


def _cut(inp, L):
    keys = ("x", "z", "B", "C", "dt_raw", "seq_idx")
    out = {k: (v[:, :L] if (v is not None and k in keys) else v) for k, v in inp.items()}
    if inp.get("A") is not None and inp["A"].ndim == 3:      # per-token A
        out["A"] = inp["A"][:, :L]
    return out


def cpu_baseline_block(wname: str, seconds: float) -> dict:
    v, desc, threads, _ = cpu_oracle_run(wname, seconds)
    return {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": desc,
            "single_thread": cpu_oracle_single_thread(wname)}


def reference_arm(args):
    """The oracle, as it stands, timed on the host cores: each step is a
    bounded sample of the headline workload."""
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    budget = 150.0 / max(1, args.steps + args.warmup)
    for _ in range(args.warmup):
        cpu_oracle_run(args.workload, budget)
    vals, descs, threads, wall = [], None, None, 0.0
    for _ in range(args.steps):
        v, descs, threads, dt = cpu_oracle_run(args.workload, budget)
        vals.append(v)
        wall += dt
    value = sum(vals) / len(vals)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": wall / max(1, args.steps) * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_block(args.gpus, args.workload),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads,
                             "kind": "oracle", "sample": descs},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)
    return 0


WORKLOAD_TEXT = {
    "long_7b": "long_7b: 7B-class Mamba-2 layer, batch 2 x 16384 tokens per GPU, 128 heads x 64, "
               "d_state 128, 8 B/C groups, conv kernel 4, initial state N(0, 0.1), one document "
               "per row, bf16 activations, fp32 dt/A/D/state",
    "mini_k3_mixer": "mini_k3_mixer: Mamba-2 SSD mixer, batch 5 x 8192 tokens per GPU, 32 heads "
                     "x 64, d_state 64, 8 B/C groups, conv kernel 4, packed documents (geometric "
                     "lengths, mean 1500), bf16 activations, fp32 dt/A/D/state",
    "mamba3_siso": "mamba3_siso: Mamba-3-sized SISO scan, batch 4 x 4096 tokens per GPU, 80 heads "
                   "x 64, d_state 128, 1 group, no conv, per-token A floored at 1e-4, B/C RMSNorm "
                   "+ per-head bias, bf16 activations, fp32 dt/A/D/state",
}


def config_block(n, wname=WORKLOAD):
    from selective_state_space_forward_b200.synthetic import WORKLOADS
    w = WORKLOADS[wname]
    fb = forward_bytes(w)["bytes"]
    return {"workload": WORKLOAD_TEXT[wname], "global_batch": w.batch * n, "seq_len": w.seqlen,
            "parallelism": f"dp{n} (independent rows)",
            "l2": f"inputs larger than L2 ({fb / 1e6:.0f} MB per step), no flush"}


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return reference_arm(args)
    import torch
    rank, world, local_rank = dist_env()
    torch.cuda.set_device(local_rank)
    rank, world = dist_init("nccl")
    peaks = load_peaks()
    fwd, ctx = bench_forward(args, torch, rank, world, local_rank, peaks, args.workload)
    e2e = None if args.no_e2e else bench_e2e(args, torch, ctx, world, local_rank)
    del ctx
    torch.cuda.empty_cache()
    configs = {}
    if not args.no_extra:
        for wname in [n for n in (WORKLOAD,) + EXTRA_WORKLOADS if n != args.workload]:
            r, c = bench_forward(args, torch, rank, world, local_rank, peaks, wname)
            del c
            torch.cuda.empty_cache()
            configs[wname] = dict(r, config=config_block(world, wname))
    decode = None
    if not args.no_decode and rank == 0:
        torch.cuda.empty_cache()
        decode = bench_decode(args, torch, peaks)
    backward = packed = None
    if not args.no_backward and rank == 0:
        torch.cuda.empty_cache()
        backward = bench_backward(args, torch, peaks)
        torch.cuda.empty_cache()
        packed = bench_packed_norm(args, torch, peaks)
    s6 = None
    if not args.no_s6 and rank == 0:
        torch.cuda.empty_cache()
        s6 = bench_s6(args, torch, peaks, fwd["clocks"].get("sm_mhz"))
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline_block(args.workload, 20.0)
        for wname in configs:
            configs[wname]["cpu_baseline"] = cpu_baseline_block(wname, 6.0)
    if rank == 0:
        line = {"metric": METRIC, "value": fwd["value"], "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": fwd["ms_per_step"],
                "repeats": fwd["repeats"], "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": config_block(world, args.workload), "path": fwd["path"],
                "roofline": fwd["roofline"],
                "forward_roofline": fwd["forward_roofline"], "configs": configs,
                "decode": decode, "backward": backward, "packed_gated_norm": packed, "s6": s6,
                "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": fwd["launches"],
                "gpu_launches_per_step": fwd["launches_per_step"], "clocks": fwd["clocks"]}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        barrier(world)
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
