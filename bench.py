"""Benchmark of the Gated DeltaNet hot path on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl gdn|reference]
                    [--workload ragged|long]

One step = one gdn_prefill call over the whole prefill workload (default: 8
ragged requests with lengths U[1,4096], Hq=16, Hv=32, Dk=Dv=128, bf16), inputs
resident in HBM, consecutive launches alternating between two independent input
sets.  `value` is prefill tokens/s over all ranks.  After the K timed steps the
same K-launch window is repeated until a quarter second of launches has been
timed, so that the clock record covers a few dozen samples; the repeats are
reported beside the measurement.  The long-context workload (B=1, S=32768) is
timed the same way through the same call and reported under "long_prefill", and the
ragged workload with a per-key-dimension decay (g of shape [N, Hv, Dk], the per-token
kernel) under "prefill_per_key_decay".
`roofline.bound` is the roof (tensor cores or HBM) whose ideal time is longer;
both fractions are reported.  The same run
then times gdn_decode over the state-pool workload (pool [1024,32,128,128]
fp32, 256 rows with 13 padding rows) for K steps and reports its state-pool
GB/s under "decode", and gdn_conv1d (the causal conv feeding q, k, v: conv_dim
8192, K = 4, bf16) over the ragged token mix ("conv1d") and over one decode
step of 256 requests ("conv1d_decode"), in HBM GB/s.

Multi-GPU (torchrun): every rank runs an independent replica of the workload
(weak scaling, no collective on the data path); times are the max over ranks.

--impl reference times the float64 CPU oracle on a bounded sample of the same
workload on this host's cores (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "GDN prefill tokens/s (tensor-pipe %); decode state-pool GB/s vs HBM peak"
CHUNK = 64


# ----------------------------------------------------------------- helpers
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def source_digest(source: str):
    """First 16 hex of the sha256 over a kernel file and, depth first, every header of csrc/ that
    it includes with quotes (each counted once), or None when the file is missing.  A change to a
    shared device header therefore counts as a change of every kernel that includes it."""
    import hashlib
    import re
    csrc = os.path.join(ROOT, "gated_deltanet_state_gdn_b200", "csrc")
    h = hashlib.sha256()
    seen = set()

    def visit(name):
        path = os.path.join(csrc, name)
        if name in seen or not os.path.exists(path):
            return
        seen.add(name)
        data = open(path, "rb").read()
        h.update(data)
        for inc in re.findall(rb'^\s*#\s*include\s*"([^"]+)"', data, re.M):
            visit(inc.decode())

    if not os.path.exists(os.path.join(csrc, source)):
        return None
    visit(source)
    return h.hexdigest()[:16]


def ncu_traffic(profile_name: str, source: str, key: str = "traffic_bytes_per_launch"):
    """DRAM bytes recorded under `key` (per launch, or per call for a call of several launches)
    in profiles/<profile_name> by an ncu capture, or None when the kernel source changed since
    (the summary stores source_digest of the sources it was captured on)."""
    import re
    path = os.path.join(ROOT, "profiles", profile_name)
    digest = source_digest(source)
    if not (os.path.exists(path) and digest):
        return None
    text = open(path).read()
    m_t = re.search(r"^" + re.escape(key) + r":\s*(\d+)", text, re.M)
    m_h = re.search(r"^source_sha256_16:\s*([0-9a-f]+)", text, re.M)
    if not (m_t and m_h):
        return None
    return int(m_t.group(1)) if digest == m_h.group(1) else None


def prefill_flops_per_token_head(Dk, Dv, C=CHUNK):
    """Tensor-core FLOPs of the chunked form per token and value head:
    Gram K K^T and Q K^T (2 * 2 C Dk), W = T diag(b G) K (2 C Dk), U~ = T diag(b) V (2 C Dv),
    W S and Q S (2 * 2 Dk Dv), (Q K^T . M) U (2 C Dv), K~^T U (2 Dk Dv)."""
    return 6 * Dk * Dv + 2 * C * (3 * Dk + 2 * Dv)


def prefill_bytes(case):
    N = case.N
    Hq, Hv, Dk, Dv = case.dims
    esz = case.q.element_size()
    g_per_token = Hv * (Dk if case.g is not None and case.g.dim() == 3 else 1)
    b = N * (2 * Hq * Dk + 2 * Hv * Dv) * esz + N * (g_per_token + Hv) * 4  # q, k, v, out, g, beta
    st = case.B * Hv * Dv * Dk * 4
    b += st * (2 if case.initial_state is not None else 1)
    if case.cu_seqlens is not None:
        b += (case.B + 1) * 4
    return b


def decode_bytes(case):
    """HBM bytes the method must move: per live (row, head) the state read once and written
    once per store, plus q, k, v, a, b, out."""
    B, T, H, Dk = case.q.shape
    nh = case.k.shape[2]
    HV, Dv = case.v.shape[3], case.v.shape[4]
    live = int((case.read_idx >= 0).sum())
    state = Dv * Dk * 4
    if case.scatter_idx is not None:
        sc = case.scatter_idx[case.read_idx >= 0]
        stores = int((sc >= 0).sum())
    elif case.disable_state_update:
        stores = 0
    else:
        w = case.read_idx if case.write_idx is None else case.write_idx
        stores = int(((case.read_idx >= 0) & (w >= 0)).sum())
    act = live * T * (H * Dk + nh * H * Dk + nh * HV * Dv + HV * Dv) * 2 + live * T * (HV + nh * HV) * 2
    return live * HV * state + stores * HV * state + act


class ClockSampler:
    """SM clocks, power and clock-event (throttle) reasons sampled in the background.

    NVML is polled every 5 ms from a thread (reads only; nothing is set); every sample carries
    its host time, so the summary covers exactly the timed window it is asked about.  Without
    NVML it falls back to `nvidia-smi -lms 100`.
    """
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.rows = []            # (host time, sm MHz, max sm MHz, set of reason names)
        self.proc = None
        self.stop_flag = threading.Event()
        self.thread = None

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.handle = pynvml.nvmlDeviceGetHandleByIndex(self.gpu_index)
            self.max_sm = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
            self.bits = {
                "hw_slowdown": pynvml.nvmlClocksEventReasonHwSlowdown,
                "hw_thermal_slowdown": pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                "sw_thermal_slowdown": pynvml.nvmlClocksEventReasonSwThermalSlowdown,
                "sw_power_cap": pynvml.nvmlClocksEventReasonSwPowerCap,
            }
            self.thread = threading.Thread(target=self._poll_nvml, daemon=True)
            self.thread.start()
            return
        except Exception:
            self.nvml = None
        try:
            fields = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                      "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                      "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_index}", f"--query-gpu={fields}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read_smi, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _poll_nvml(self):
        nv = self.nvml
        while not self.stop_flag.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                active = {n for n, bit in self.bits.items() if mask & bit}
                self.rows.append((time.time(), float(sm), float(self.max_sm), active))
            except Exception:
                pass
            time.sleep(0.005)

    def _read_smi(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                active = {n for n, v in zip(self.NAMES, parts[5:9])
                          if v.strip().lower().startswith("active")}
                smax = float(parts[2]) if parts[2].replace(".", "").isdigit() else None
                self.rows.append((time.time(), float(parts[1]), smax, active))

    def stop(self):
        self.stop_flag.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self, window=None, label="all timed phases"):
        rows = self.rows if window is None else [r for r in self.rows
                                                   if window[0] <= r[0] <= window[1]]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0,
                    "window": label}
        reasons = set()
        for r in rows:
            reasons |= r[3]
        smax = [r[2] for r in rows if r[2] is not None]
        return {"sm_mhz": statistics.median(r[1] for r in rows),
                "sm_max_mhz": max(smax) if smax else None, "reasons": sorted(reasons),
                "samples": len(rows), "window": label,
                "source": "nvml 5 ms" if self.nvml is not None else "nvidia-smi 100 ms"}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """Max of a per-rank time over all ranks (replicas are timed independently; the job
    takes as long as its slowest rank)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: int, world: int, max_ms_per_step: float) -> float:
    """Whole-job throughput of `world` weak-scaled replicas: all ranks' units / slowest rank."""
    return units_per_rank * world / (max_ms_per_step / 1e3)


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------- GPU arms
def to_dev(t):
    return None if t is None else t.cuda(non_blocking=False)


def prefill_sets(case, nsets):
    """`nsets` independent device copies of the prefill inputs and outputs, used in turn by
    consecutive launches: by the time a set comes round again the other sets (each larger than
    L2) have streamed through L2, so no launch re-reads its initial states, gates or q/k/v from
    L2 (the rotation stands in for an L2 flush between launches)."""
    Hq, Hv, Dk, Dv = case.dims
    sets = []
    for _ in range(nsets):
        q, k, v, g, beta = map(to_dev, (case.q, case.k, case.v, case.g, case.beta))
        cu, init = to_dev(case.cu_seqlens), to_dev(case.initial_state)
        out = torch.empty((case.N, Hv, Dv), dtype=case.q.dtype, device="cuda")
        fs = torch.empty((case.B, Hv, Dv, Dk), dtype=torch.float32, device="cuda")
        sets.append((q, k, v, g, beta, cu, init, fs, out))
    return sets


def time_prefill(gdn, case, steps, warmup, world, nsets=2, min_window_s=0.25):
    """K timed gdn_prefill launches (one per step, rotating over `nsets` input sets), then
    further windows of K launches until at least `min_window_s` of launches have been timed, so
    that the clock record of the prefill covers a few dozen samples.  The first window is the
    reported measurement; the repeats are reported beside it.  Every window is bracketed by a
    barrier and a device synchronisation; per-launch CUDA events on the launching stream."""
    sets = prefill_sets(case, nsets)

    def step(i):
        q, k, v, g, beta, cu, init, fs, out = sets[i % nsets]
        gdn.gdn_prefill(q, k, v, g, beta, cu, init, fs, out, num_requests=case.B,
                        scale=case.scale, qk_l2norm=case.qk_l2norm)

    for i in range(warmup):
        step(i)
    stream = torch.cuda.current_stream()

    def window(base):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        barrier(world)
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        host0 = time.time()
        t0.record(stream)
        for i, (s, e) in enumerate(ev):
            s.record(stream)
            step(base + i)
            e.record(stream)
        t1.record(stream)
        torch.cuda.synchronize()
        host1 = time.time()
        barrier(world)
        return t0.elapsed_time(t1), [s.elapsed_time(e) for s, e in ev], (host0, host1)

    total_ms, launch_ms, (h0, h1) = window(warmup)
    repeats = []
    timed_s = total_ms / 1e3
    n = 1
    # every rank takes the same number of windows: the count follows rank 0's first window
    want = max(0, math.ceil(min_window_s / max(timed_s, 1e-6)) - 1)
    if world > 1:
        import torch.distributed as dist
        t = torch.tensor([want], dtype=torch.int64, device="cuda")
        dist.broadcast(t, 0)
        want = int(t.item())
    for _ in range(want):
        w_ms, w_launch, (_, h1) = window(warmup + n * steps)
        repeats.append(w_ms / steps)
        n += 1
    del sets
    time_prefill.window = (h0, h1)
    time_prefill.repeats = repeats
    time_prefill.launches = n * steps
    return total_ms, launch_ms


def time_prefill_e2e(gdn, case, steps, warmup, world):
    """Through the public call, from pinned host buffers, with host<->device copies inside.

    Every step copies that step's inputs (q, k, v, g, beta, cu_seqlens, initial state) from
    pinned host memory, runs gdn_prefill and copies the outputs and final states back to
    pinned host memory.  Steps are pipelined the way a serving loop would run them: two sets
    of device buffers, the host-to-device copies on one stream, the call on a second and the
    device-to-host copies on a third, ordered by events, so that step i+1's input copy
    overlaps step i's kernel and output copy.  Nothing is skipped: every step moves all of
    its bytes both ways.
    """
    hin = [case.q, case.k, case.v, case.g, case.beta, case.cu_seqlens, case.initial_state]
    hin = [None if t is None else t.pin_memory() for t in hin]
    Hq, Hv, Dk, Dv = case.dims
    dins = [[None if t is None else torch.empty_like(t, device="cuda") for t in hin]
            for _ in range(2)]
    outs = [torch.empty((case.N, Hv, Dv), dtype=case.q.dtype, device="cuda") for _ in range(2)]
    fss = [torch.empty((case.B, Hv, Dv, Dk), dtype=torch.float32, device="cuda") for _ in range(2)]
    hout = [torch.empty(outs[0].shape, dtype=outs[0].dtype).pin_memory() for _ in range(2)]
    hfs = [torch.empty(fss[0].shape, dtype=torch.float32).pin_memory() for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in hin if t is not None)
    d2h = hout[0].numel() * hout[0].element_size() + hfs[0].numel() * hfs[0].element_size()
    s_in, s_run, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    copied = [torch.cuda.Event() for _ in range(2)]    # inputs of buffer set j on the device
    consumed = [torch.cuda.Event() for _ in range(2)]  # the call has read buffer set j
    done = [torch.cuda.Event() for _ in range(2)]      # outputs of set j written
    drained = [torch.cuda.Event() for _ in range(2)]   # outputs of set j copied to the host
    used = [False, False]

    def step(i):
        j = i % 2
        with torch.cuda.stream(s_in):
            if used[j]:
                s_in.wait_event(consumed[j])
            for d, h in zip(dins[j], hin):
                if d is not None:
                    d.copy_(h, non_blocking=True)
            copied[j].record(s_in)
        with torch.cuda.stream(s_run):
            s_run.wait_event(copied[j])
            if used[j]:
                s_run.wait_event(drained[j])
            q, k, v, g, b, cu, init = dins[j]
            gdn.gdn_prefill(q, k, v, g, b, cu, init, fss[j], outs[j], num_requests=case.B,
                            scale=case.scale, qk_l2norm=case.qk_l2norm, stream=s_run)
            consumed[j].record(s_run)
            done[j].record(s_run)
        with torch.cuda.stream(s_out):
            s_out.wait_event(done[j])
            hout[j].copy_(outs[j], non_blocking=True)
            hfs[j].copy_(fss[j], non_blocking=True)
            drained[j].record(s_out)
        used[j] = True

    main = torch.cuda.current_stream()
    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(main)
    for st in (s_in, s_run, s_out):
        st.wait_event(t0)
    for i in range(steps):
        step(warmup + i)
    for st in (s_in, s_run, s_out):
        ev = torch.cuda.Event()
        ev.record(st)
        main.wait_event(ev)
    t1.record(main)
    torch.cuda.synchronize()
    barrier(world)
    return t0.elapsed_time(t1), h2d, d2h


def time_decode(gdn, case, steps, warmup, world, graph=False, npools=1):
    """Per-launch CUDA events around back-to-back launches; with graph=True the `steps` launches
    are captured in one CUDA graph (for launches short enough that the Python call would
    otherwise show in the events), replayed once untimed and once timed, and the mean per launch
    is returned for every step.  With npools > 1 consecutive launches use `npools` independent
    copies of the pool (and of the inputs), so that one lap of the rotation moves more bytes than
    L2 holds and no launch finds its slots still in L2 from an earlier launch."""
    B, T, H, Dk = case.q.shape
    HV, Dv = case.v.shape[3], case.v.shape[4]
    sets = []
    for _ in range(npools):
        q, k, v, a, b = map(to_dev, (case.q, case.k, case.v, case.a, case.b))
        out = torch.zeros((B, T, HV, Dv), dtype=torch.bfloat16, device="cuda")
        sets.append((q, k, v, a, b, to_dev(case.pool), out))
    A_log, dt_bias = to_dev(case.A_log), to_dev(case.dt_bias)
    ri, wi, si = to_dev(case.read_idx), to_dev(case.write_idx), to_dev(case.scatter_idx)

    def step(i, stream=None):
        q, k, v, a, b, pool, out = sets[i % npools]
        gdn.gdn_decode(q, k, v, pool, ri, A_log, a, dt_bias, b, scale=case.scale, out=out,
                       scatter_idx=si, use_qk_l2norm=case.use_qk_l2norm, write_idx=wi,
                       stream=stream)

    for i in range(warmup):
        step(i)
    stream = torch.cuda.current_stream()
    barrier(world)
    torch.cuda.synchronize()
    if graph:
        side = torch.cuda.Stream()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(side):
            with torch.cuda.graph(g, stream=side):
                for i in range(steps):
                    step(i, side)
        torch.cuda.synchronize()
        g.replay()   # first replay uploads the graph: untimed
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        per = e0.elapsed_time(e1) / steps
        del g, sets
        return [per] * steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for i, (s, e) in enumerate(ev):
        s.record(stream)
        step(i)
        e.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    del sets
    return [s.elapsed_time(e) for s, e in ev]


def conv_bytes(case):
    """HBM bytes the conv must move: x read and out written once, each request's window read
    and written once, the weights once."""
    N, C = case.x.shape
    K = case.weight.shape[1]
    esz = case.x.element_size()
    lens = (case.row_offsets[1:].to(torch.int64) - case.row_offsets[:-1].to(torch.int64))
    live = int((lens > 0).sum())
    return 2 * N * C * esz + 2 * live * C * (K - 1) * esz + C * K * esz


def time_conv(gdn, case, steps, warmup, world, graph=False, nsets=1):
    """Per-launch CUDA events around back-to-back launches; with graph=True the `steps`
    launches are captured in one CUDA graph (host launch cost out of the way for small calls)
    and the mean per launch is returned for every step.  With nsets > 1 consecutive launches
    use `nsets` independent copies of x, the window pool and out, so that one lap of the
    rotation moves more bytes than L2 holds."""
    w, si, ro = map(to_dev, (case.weight, case.slot_idx, case.row_offsets))
    sets = []
    for _ in range(nsets):
        x, st = to_dev(case.x), to_dev(case.conv_state)
        sets.append((x, st, torch.empty_like(x)))

    def step(i, stream=None):
        x, st, out = sets[i % nsets]
        gdn.gdn_conv1d(x, w, st, si, ro, out, stream=stream)

    for i in range(warmup):
        step(i)
    stream = torch.cuda.current_stream()
    barrier(world)
    torch.cuda.synchronize()
    if graph:
        side = torch.cuda.Stream()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(side):
            with torch.cuda.graph(g, stream=side):
                for i in range(steps):
                    step(i, side)
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        per = e0.elapsed_time(e1) / steps
        del g
        return [per] * steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for i, (s, e) in enumerate(ev):
        s.record(stream)
        step(i)
        e.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    del sets
    return [s.elapsed_time(e) for s, e in ev]


# ---------------------------------------------------------------- CPU oracle
def cpu_oracle_sample(case, target_s=10.0, repeats=1, threads=None, warmup=0):
    """Time the float64 oracle on a bounded sample of the prefill workload: the first L
    tokens of the packed stream with every head; L is grown until one run takes ~target_s/8,
    then scaled so that one run is ~target_s (at most the whole stream).  The calibrated
    sample then runs `warmup` times untimed and `repeats` times timed, and the median rate of
    the timed runs is reported.  threads: host threads for the oracle's (request, head) units
    (default: all cores)."""
    import oracle
    oracle.build()
    threads = oracle.max_threads() if threads is None else int(threads)
    Hq, Hv, Dk, Dv = case.dims
    start = 0 if case.cu_seqlens is None else int(case.cu_seqlens[0])
    total = case.N - start

    def run(L):
        sl = slice(start, start + L)
        q = case.q[sl].to(torch.float64).numpy()
        k = case.k[sl].to(torch.float64).numpy()
        v = case.v[sl].to(torch.float64).numpy()
        g = case.g[sl].to(torch.float64).numpy()
        b = case.beta[sl].to(torch.float64).numpy()
        init = None if case.initial_state is None else \
            case.initial_state[:1].to(torch.float64).numpy()
        t = time.perf_counter()
        oracle.prefill(q, k, v, g, b, None, init, B=1, scale=case.scale,
                       qk_l2norm=case.qk_l2norm, threads=threads)
        return time.perf_counter() - t

    L = 16
    dt = run(L)
    while dt < target_s / 8 and L * 2 <= total:
        L *= 2
        dt = run(L)
    L_final = max(1, min(total, int(L * (target_s / max(dt, 1e-6)))))
    for _ in range(max(0, warmup)):
        run(L_final)
    times = [run(L_final) for _ in range(max(1, repeats))]
    dt = statistics.median(times)
    return {"value": L_final / dt, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"first {L_final} tokens of the packed stream run as one request, "
                      f"all {Hv} value heads ({Hq} query/key heads), float64, {dt:.2f} s per run"
                      + (f", median of {len(times)} runs" if len(times) > 1 else ""),
            "runs": len(times), "warmup_runs": max(0, warmup)}


def prefill_roofline(gdn, case, launch_ms, peaks, sm_mhz, traffic):
    """Roofline of one prefill workload from its per-launch CUDA-event times.

    The kernel is held to both of its roofs: the tensor cores (algorithmic FLOPs of the chunk
    form against the measured bf16 peak) and HBM (algorithmic bytes against the measured copy
    bandwidth).  `bound` is the roof whose ideal time is the longer one, and `frac` is taken
    against it; both fractions are reported."""
    Hq, Hv, Dk, Dv = case.dims
    avg_s = statistics.mean(launch_ms) / 1e3
    per_key = case.g is not None and case.g.dim() == 3
    if not gdn.prefill_uses_chunked(case.q.dtype, Hv, Dk, Dv, decay_per_key=per_key):
        byts = prefill_bytes(case)
        ach = byts / avg_s / 1e9
        return {"kernel": "gdn_prefill_seq", "bound": "hbm", "achieved": ach,
                "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": ach / peaks["hbm_gbs"],
                "traffic": None, "algorithmic_bytes": byts, "ms_per_launch": avg_s * 1e3,
                "peak_source": peaks["source"],
                "note": "per-token recurrence: one dependent step per token per head, so its "
                        "time follows the longest request, not the bytes"}
    flops = case.N * Hv * prefill_flops_per_token_head(Dk, Dv)
    byts = prefill_bytes(case)
    tc_peak, hbm_peak = peaks["bf16_tflops"], peaks["hbm_gbs"]
    t_tc = flops / (tc_peak * 1e12)
    t_hbm = byts / (hbm_peak * 1e9)
    tc = {"achieved": flops / avg_s / 1e12, "peak": tc_peak, "unit": "TFLOP/s",
          "frac": flops / avg_s / 1e12 / tc_peak, "ideal_us": t_tc * 1e6,
          "algorithmic_flops": flops}
    hbm = {"achieved": byts / avg_s / 1e9, "peak": hbm_peak, "unit": "GB/s",
           "frac": byts / avg_s / 1e9 / hbm_peak, "ideal_us": t_hbm * 1e6,
           "algorithmic_bytes": byts}
    b = tc if t_tc >= t_hbm else hbm
    return {"kernel": "gdn_prefill_kd" if per_key else "gdn_prefill_chunk",
            "bound": "tensor" if t_tc >= t_hbm else "hbm",
            "achieved": b["achieved"], "peak": b["peak"], "unit": b["unit"], "frac": b["frac"],
            "traffic": traffic, "tensor": tc, "hbm": hbm,
            "ms_per_launch": avg_s * 1e3,
            "kcycles_per_launch": None if sm_mhz is None else avg_s * 1e3 * sm_mhz,
            "peak_source": peaks["source"] + " (burst bf16; copy bandwidth)"}


def profile_phase(gdn, workloads, args):
    """Run one phase for `--steps` steps after `--warmup` (under a profiler); prints timings."""
    if args.phase == "prefill":
        case = make_case(args.workload)
        # no repeat windows: under a profiler every launch counts
        total_ms, launch_ms = time_prefill(gdn, case, args.steps, args.warmup, 1, min_window_s=0.0)
        print(json.dumps({"phase": "prefill", "workload": case.name,
                          "ms_per_launch": statistics.mean(launch_ms)}), flush=True)
    elif args.phase == "conv":
        for ccase in (workloads.conv_ragged_case(), workloads.conv_decode_case()):
            cms = time_conv(gdn, ccase, args.steps, args.warmup, 1)
            print(json.dumps({"phase": "conv", "workload": ccase.name,
                              "ms_per_launch": statistics.mean(cms)}), flush=True)
    else:
        for dcase, graph in ((workloads.decode_pool_case(), False), (workloads.mtp_case(), True)):
            dms = time_decode(gdn, dcase, args.steps, args.warmup, 1, graph=graph)
            print(json.dumps({"phase": "decode", "workload": dcase.name,
                              "ms_per_launch": statistics.mean(dms)}), flush=True)
    return 0


# ---------------------------------------------------------------------- main
def make_case(name):
    from gated_deltanet_state_gdn_b200 import workloads
    if name == "ragged":
        return workloads.ragged_prefill_case()
    if name == "long":
        return workloads.long_prefill_case()
    if name == "ragged_per_key":
        return workloads.ragged_prefill_case(decay_per_key=True)
    raise ValueError(name)


def workload_config(case, name):
    Hq, Hv, Dk, Dv = case.dims
    return {"workload": case.name, "requests": case.B, "tokens": case.N,
            "lengths": "U[1,4096] seeded" if name.startswith("ragged") else str(case.N),
            "Hq": Hq, "Hv": Hv, "Dk": Dk, "Dv": Dv, "chunk": CHUNK,
            "l2": "inputs larger than L2 (q+k+v+out > 126 MB), and consecutive launches "
                  "alternate between two independent input sets, so no launch re-reads "
                  "initial states, gates or q/k/v left in L2 by the previous one"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="gdn", choices=["gdn", "reference"])
    ap.add_argument("--workload", default="ragged", choices=["ragged", "long", "ragged_per_key"])
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-conv", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-long", action="store_true", help="skip the long-context prefill line")
    ap.add_argument("--no-per-key", action="store_true",
                    help="skip the per-key-dimension decay prefill line")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--phase", default="all", choices=["all", "prefill", "decode", "conv"],
                    help="prefill or decode alone (for profiling); 'all' for the JSON line")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return 0
        case = make_case(args.workload)
        # W untimed and K timed steps of one calibrated sample each, sized so that the run
        # stays near 90 s
        per_step = min(2.5, max(0.2, 90.0 / max(1, args.steps + args.warmup)))
        base = cpu_oracle_sample(case, target_s=per_step, repeats=args.steps, warmup=args.warmup)
        val = base["value"]
        print(json.dumps({
            "impl": "reference", "metric": METRIC, "value": val, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": case.N / val * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(case, args.workload), "cpu_baseline": base,
            "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}), flush=True)
        return 0

    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    import gated_deltanet_state_gdn_b200 as gdn
    from gated_deltanet_state_gdn_b200 import workloads
    gdn.lib()
    peaks = load_peaks()

    if args.phase != "all":
        return profile_phase(gdn, workloads, args)

    case = make_case(args.workload)
    Hq, Hv, Dk, Dv = case.dims
    clocks = ClockSampler(int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[0])
                          if os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")[0].isdigit()
                          else local)
    clocks.start()
    total_ms, launch_ms = time_prefill(gdn, case, args.steps, args.warmup, world)
    prefill_window = time_prefill.window
    prefill_repeats = time_prefill.repeats
    launches = time_prefill.launches
    max_ms = max_over_ranks(total_ms, world)
    ms_per_step = max_ms / args.steps
    tokens = case.N * world
    value = job_throughput(case.N, world, ms_per_step)
    prefill_clocks = clocks.summary(prefill_window, "prefill timed windows")
    traffic = ncu_traffic("prefill_chunk_ragged_prefill.md", "prefill_chunk.cu") \
        if args.workload == "ragged" else None
    roof = prefill_roofline(gdn, case, launch_ms, peaks, prefill_clocks["sm_mhz"], traffic)
    roof["repeat_windows_ms_per_launch"] = prefill_repeats

    # the long-context workload (B = 1, S = 32768) through the same call, in the same run
    long_prefill = None
    if args.workload == "ragged" and not args.no_long:
        lcase = make_case("long")
        l_total, l_launch = time_prefill(gdn, lcase, args.steps, args.warmup, world)
        l_clocks = clocks.summary(time_prefill.window, "long-context prefill timed windows")
        l_max = max_over_ranks(l_total, world) / args.steps
        long_prefill = {
            "workload": lcase.name, "tokens": lcase.N, "ms_per_step": l_max,
            "value": job_throughput(lcase.N, world, l_max), "unit": "tokens/s",
            "roofline": prefill_roofline(
                gdn, lcase, l_launch, peaks, l_clocks["sm_mhz"],
                ncu_traffic("prefill_chunk_long_split.md", "prefill_chunk.cu",
                            "traffic_bytes_per_call")),
            "repeat_windows_ms_per_launch": time_prefill.repeats, "clocks": l_clocks}
        # a call that takes the sequence split launches three kernels: two passes and the
        # composition of the segment maps
        Hq_l, Hv_l, Dk_l, Dv_l = lcase.dims
        splits = gdn.lib().gdn_prefill_workspace_size(lcase.B, lcase.N, Hq_l, Hv_l, Dk_l, Dv_l,
                                                      gdn.GDN_BF16, 0) > 0
        long_prefill["kernels_per_call"] = 3 if splits else 1
        if long_prefill["roofline"].get("traffic") is not None:
            long_prefill["roofline"]["traffic_scope"] = \
                "one call: both passes and the composition of the segment maps"
        launches += time_prefill.launches * long_prefill["kernels_per_call"]
        del lcase

    # the per-key-dimension decay over the ragged workload's shapes (its tensor-core kernel)
    per_key = None
    if args.workload == "ragged" and not args.no_per_key:
        pcase = workloads.ragged_prefill_case(decay_per_key=True)
        p_steps = max(3, args.steps // 10)
        p_total, p_launch = time_prefill(gdn, pcase, p_steps, args.warmup, world,
                                         min_window_s=0.0)
        p_max = max_over_ranks(p_total, world) / p_steps
        per_key = {
            "workload": pcase.name, "tokens": pcase.N, "steps": p_steps, "ms_per_step": p_max,
            "value": job_throughput(pcase.N, world, p_max), "unit": "tokens/s",
            "roofline": prefill_roofline(gdn, pcase, p_launch, peaks, None,
                                         ncu_traffic("prefill_kd_ragged_per_key.md", "prefill_kd.cu"))}
        launches += time_prefill.launches
        del pcase

    decode = decode_mtp = None
    if not args.no_decode:
        dcase = workloads.decode_pool_case()
        dms = time_decode(gdn, dcase, args.steps, args.warmup, world)
        dmax = max_over_ranks(sum(dms), world) / args.steps
        dbytes = decode_bytes(dcase)
        gbs = dbytes * world / (dmax / 1e3) / 1e9
        per_gpu = dbytes / (statistics.mean(dms) / 1e3) / 1e9
        decode = {"workload": dcase.name, "value": gbs, "unit": "GB/s",
                  "bytes_per_step": dbytes, "ms_per_step": dmax,
                  "frac": per_gpu / peaks["hbm_gbs"], "peak": peaks["hbm_gbs"],
                  "peak_source": peaks["source"]}
        launches += args.steps
        del dcase
        # MTP / Gated DeltaProduct: T = 4 tokens, 2 Householder sub-steps, per-token scatter
        mcase = workloads.mtp_case()
        mms = time_decode(gdn, mcase, args.steps, args.warmup, world, graph=True, npools=4)
        mmax = max_over_ranks(sum(mms), world) / args.steps
        mbytes = decode_bytes(mcase)
        decode_mtp = {"workload": mcase.name, "value": mbytes * world / (mmax / 1e3) / 1e9,
                      "unit": "GB/s", "bytes_per_step": mbytes, "ms_per_step": mmax,
                      "frac": mbytes / (statistics.mean(mms) / 1e3) / 1e9 / peaks["hbm_gbs"],
                      "peak": peaks["hbm_gbs"], "peak_source": peaks["source"],
                      "timing": "one CUDA graph of K launches rotating over 4 independent "
                                "256 MB pools (690 MB moved per lap > L2): no slot is "
                                "rewritten while an earlier write of it can still sit in L2"}
        launches += args.steps
        del mcase

    conv = conv_dec = None
    if not args.no_conv:
        for key, ccase, graph, note in (
                ("conv1d", workloads.conv_ragged_case(), False,
                 "back-to-back launches, working set > L2 (steady-state HBM traffic)"),
                ("conv1d_decode", workloads.conv_decode_case(), True,
                 "one CUDA graph of K launches rotating over 6 independent copies of x, the "
                 "window pool and out (202 MB moved per lap > L2)")):
            cms = time_conv(gdn, ccase, args.steps, args.warmup, world, graph=graph,
                            nsets=6 if graph else 1)
            cmax = max_over_ranks(sum(cms), world) / args.steps
            cbytes = conv_bytes(ccase)
            per_gpu = cbytes / (statistics.mean(cms) / 1e3) / 1e9
            obj = {"workload": ccase.name, "value": cbytes * world / (cmax / 1e3) / 1e9,
                   "unit": "GB/s", "bytes_per_step": cbytes, "ms_per_step": cmax,
                   "frac": per_gpu / peaks["hbm_gbs"], "peak": peaks["hbm_gbs"],
                   "peak_source": peaks["source"], "timing": note}
            if key == "conv1d":
                obj["traffic"] = ncu_traffic("conv1d_ragged.md", "conv1d.cu")
                conv = obj
            else:
                conv_dec = obj
            launches += args.steps
            del ccase
    clocks.stop()

    e2e = None
    if not args.no_e2e:
        e_steps = max(4, args.steps // 2)
        e_ms, h2d, d2h = time_prefill_e2e(gdn, case, e_steps, args.warmup, world)
        e_max = max_over_ranks(e_ms, world) / e_steps
        e2e = {"value": tokens / (e_max / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e_max}
        launches += e_steps

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_oracle_sample(case, target_s=args.cpu_seconds)
        # the same oracle on one host thread, a shorter sample
        one = cpu_oracle_sample(case, target_s=max(1.0, args.cpu_seconds / 3), threads=1)
        cpu["single_thread"] = {"value": one["value"], "unit": one["unit"], "cores": 1,
                                "sample": one["sample"]}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": dict(workload_config(case, args.workload),
                                                parallelism=f"replicas{world}"),
            "roofline": roof, "long_prefill": long_prefill, "prefill_per_key_decay": per_key,
            "decode": decode, "decode_mtp": decode_mtp, "conv1d": conv,
            "conv1d_decode": conv_dec,
            "e2e": e2e, "cpu_baseline": cpu,
            "clocks": prefill_clocks,
            "clocks_all_phases": clocks.summary(),
            "gpu_launches": launches,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
