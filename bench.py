"""Benchmark of liblisa on B200: the LISA decode step of a 7B-shaped layer at 16K context.

Workload (one "step" = one pass of the whole hot path over one batch): the
fused decode step — cache append, linear-state update and read-out, indexer
scan over the full context, top-M, sparse attention over the selected rows
and the gate — for B=8 sequences at context 16384 (28 query / 4 KV heads,
head dim 128, 8 indexer heads of dim 64, M=2048), bf16 activations, fp32
linear state built by a prefill of the same seeded tokens.

Timing: W untimed warm-up steps, then K steps, each timed with CUDA events on
the launching stream.  Instead of flushing L2, the inputs are larger than L2:
four copies of the whole decode state (caches, linear state, step inputs) at
distinct addresses are used in rotation, so each step's ~55 MB of traffic was
last touched three steps (~165 MB, more than the 126 MB L2) earlier.  Each timed
step replays a CUDA graph captured from the lisa_decode_step call of its state
copy (`--no-graphs`: the call itself); the end-to-end line calls the API
directly.  A barrier and a device synchronise bracket the timed region; the
reported time is the maximum over ranks.  Under torchrun each rank
runs its own replica of the workload (weak scaling; the path has no exchange).

`--impl reference` times the CPU oracle (plain fp64 C++) on the host cores on
a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "LISA decode tok/s @16K ctx (7B-shape layer), prefill tok/s, % of HBM roofline"
UNIT = "tok/s"


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), float(pk["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


def decode_bytes(wl, elu1: bool = False) -> dict:
    """Algorithmic HBM bytes of one decode step (per sequence and total).

    Keys are read once (k_I scan over the n cached positions), only the
    min(M, n) selected K/V rows are gathered, the fp32 state (and, with the
    elu+1 feature map, its normaliser z) is read and written once, plus the
    step's small inputs and outputs."""
    n, M = wl.n, wl.M
    scan = n * wl.H_Ik * wl.d_I * 2
    gather = min(M, n) * wl.H_kv * wl.d * 2 * 2
    state = wl.H_kv * wl.d * wl.d * 4 * 2 + (wl.H_kv * wl.d * 4 * 2 if elu1 else 0)
    small = (wl.H_q * wl.d * 2 * 2          # q, o
             + wl.H_q * wl.d * 2            # q_L (aliases q, counted once more for the LA read)
             + wl.H_kv * wl.d * 2 * 2 * 2   # k_new, v_new read + written to the cache
             + wl.H_I * wl.d_I * 2          # q_I
             + wl.d_I * wl.H_Ik * 2 * 2     # k_I_new read + written
             + wl.H_I * 4 + wl.H_q * 2)     # w, gate logits
    per_seq = scan + gather + state + small
    return dict(scan=scan, gather=gather, state=state, small=small, per_seq=per_seq,
                total=per_seq * wl.B)


DECODE_KERNELS_PER_STEP = 1  # k_decode_coop: the whole step in one cooperative launch
DECODE_SOURCES = ("decode_coop.cu", "attend_core.cuh", "decode_linear.cuh", "sm100_ptx.cuh",
                  "tma_host.cuh", "lisa_internal.cuh", "lisa_fast.cuh")


def _kernel_source_hash() -> str:
    """Hash of the sources the decode-step kernels are compiled from: a
    recorded DRAM traffic figure applies only to the kernels it was taken on."""
    h = hashlib.sha256()
    for name in DECODE_SOURCES:
        with open(os.path.join(ROOT, "hybrid_linear_top_lightning_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def _profiled_traffic(wl):
    """DRAM bytes of one decode step (one k_decode_coop launch) from the
    committed ncu summary, if it was taken on the current kernel sources; else
    None."""
    path = os.path.join(ROOT, "profiles", "decode_coop_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except Exception:
        return None
    if rec.get("kernel_source_sha") != _kernel_source_hash():
        return None
    if rec.get("workload") != wl.name:
        return None
    return float(rec["dram_bytes_per_launch"])


class ClockSampler:
    """nvidia-smi clock and throttle-reason samples, each stamped with the host
    time it arrived, so that the samples inside the timed region can be told
    from those around it."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str, period_ms: int = 100):
        self.gpu = gpu_id
        self.period_ms = period_ms
        self.proc = None
        self.samples = []  # (host time, line)
        self._reader = None

    def _read(self):
        for ln in self.proc.stdout:
            if ln.strip():
                self.samples.append((time.time(), ln))

    def __enter__(self):
        import threading

        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", str(self.period_ms)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True, bufsize=1)
            self._reader = threading.Thread(target=self._read, daemon=True)
            self._reader.start()
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            if self._reader is not None:
                self._reader.join(timeout=5)
        return False

    def summary(self, t0=None, t1=None):
        """Median SM clock, maximum clock and throttle reasons of the samples
        that arrived between host times t0 and t1 (all samples if not given)."""
        sm, smax, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ts, ln in self.samples:
            if t0 is not None and not (t0 <= ts <= t1):
                continue
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm),
                "period_ms": self.period_ms, "window": "samples inside the timed region"}


def time_blocks(run_block, stream, min_seconds: float, max_blocks: int = 4000):
    """Runs blocks (each `run_block(k)` issues one block of K back-to-back
    steps) with a CUDA event at every block boundary and no host
    synchronisation in between, until about `min_seconds` have passed on the
    device; returns the device time of each block (ms) and the host times at
    which the timed region started and ended.  The caller brackets it with a
    barrier and a synchronise."""
    import torch

    # size the run from one untimed block
    a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a_.record(stream)
    run_block(0)
    b_.record(stream)
    torch.cuda.synchronize()
    est = max(a_.elapsed_time(b_), 1e-3)
    blocks = int(min(max_blocks, max(1, math.ceil(min_seconds * 1e3 / est))))
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(blocks + 1)]
    torch.cuda.synchronize()
    t0 = time.time()
    ev[0].record(stream)
    for k in range(blocks):
        run_block(k)
        ev[k + 1].record(stream)
    torch.cuda.synchronize()
    t1 = time.time()
    return [ev[k].elapsed_time(ev[k + 1]) for k in range(blocks)], t0, t1


# ----------------------------------------------------------------------------- ranks
def max_over_ranks(x: float, device=None, world: int = 1) -> float:
    """The maximum of x over all ranks of the default process group (x itself
    when there is only one rank): a multi-rank time is the slowest rank's."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: int, world: int, steps: int, total_ms: float) -> float:
    """Whole-job throughput: the units every rank processed over all timed
    steps, divided by the slowest rank's time."""
    return world * units_per_rank * steps / (total_ms / 1e3)


# ----------------------------------------------------------------------------- GPU arm
def _setup_decode(wl, device):
    import torch

    from hybrid_linear_top_lightning_b200 import inputs, lisa

    gen = inputs.Generator(wl)
    n, p, B = wl.n, wl.n - 1, wl.B
    bf = torch.bfloat16
    kc = torch.empty(B, n, wl.H_kv, wl.d, dtype=bf, device=device)
    vc = torch.empty_like(kc)
    kIc = torch.empty(B, n, wl.H_Ik, wl.d_I, dtype=bf, device=device)
    for b in range(B):
        kc[b] = torch.from_numpy(gen.k(b, 0, n)).to(bf)
        vc[b] = torch.from_numpy(gen.v(b, 0, n)).to(bf)
        kIc[b] = torch.from_numpy(gen.k_I(b, 0, n)).to(bf)
    host = {
        "q": gen.batch("q", p, n), "q_I": gen.batch("q_I", p, n), "w": gen.batch("w", p, n),
        "gate": gen.batch("gate", p, n),
        "k_new": np.ascontiguousarray(kc[:, p:].float().cpu().numpy()),
        "v_new": np.ascontiguousarray(vc[:, p:].float().cpu().numpy()),
        "k_I_new": np.ascontiguousarray(kIc[:, p:].float().cpu().numpy()),
    }
    # linear state of the n-1 cached tokens, built by the library's own prefill
    S = torch.zeros(B, wl.H_kv, wl.d, wl.d, dtype=torch.float32, device=device)
    Dp = lisa.make_dims(B, p, 0, n, wl.H_q, wl.H_kv, wl.d, wl.H_I, wl.H_Ik, wl.d_I, wl.M,
                        chunk=wl.chunk)
    ws_p = lisa.workspace(Dp, lisa.LISA_OP_LINEAR_PREFILL, device)
    o_tmp = torch.empty(B, p, wl.H_q, wl.d, dtype=bf, device=device)
    q_tmp = torch.zeros(B, p, wl.H_q, wl.d, dtype=bf, device=device)
    lisa.lisa_linear_prefill(Dp, q_tmp, kc[:, :p].contiguous(), vc[:, :p].contiguous(), S, None,
                             o_tmp, ws_p)
    del o_tmp, q_tmp, ws_p
    dev = {k: torch.from_numpy(v).to(torch.float32 if k == "w" else bf).to(device)
           for k, v in host.items()}
    return kc, vc, kIc, S, dev, host


def _packed_inputs(tensors, alloc):
    """One flat byte buffer from `alloc(nbytes)` holding every tensor of
    `tensors` (same dtypes and shapes) at 256-byte-aligned offsets, so that a
    step's inputs move in one copy.  Returns (flat buffer, dict of views)."""
    import torch

    lay, off = {}, 0
    for k, t in tensors.items():
        nb = t.numel() * t.element_size()
        lay[k] = (off, nb)
        off += (nb + 255) & ~255
    flat = alloc(off)
    views = {}
    for k, t in tensors.items():
        o, nb = lay[k]
        views[k] = flat[o:o + nb].view(t.dtype).view(t.shape)
        views[k].copy_(t)
    return flat, views


def run_gpu(args, wl, rank, world, device):
    import torch
    import torch.distributed as dist

    from hybrid_linear_top_lightning_b200 import lisa

    torch.manual_seed(0)
    kc0, vc0, kIc0, S0, dv0, host = _setup_decode(wl, device)
    # a step's inputs live in one device buffer per state copy (views into it),
    # so the end-to-end line moves them host to device in one copy
    dev_alloc = lambda nb: torch.empty(nb, dtype=torch.uint8, device=device)  # noqa: E731
    B, n, p = wl.B, wl.n, wl.n - 1
    D = lisa.make_dims(B, 1, p, n, wl.H_q, wl.H_kv, wl.d, wl.H_I, wl.H_Ik, wl.d_I, wl.M)
    stream = torch.cuda.current_stream()

    # R copies of the whole decode state at distinct addresses; step i uses copy
    # i % R, so each step's ~55 MB was last touched R-1 steps (> L2) earlier.
    copies = []
    for r in range(args.rotate):
        if r == 0:
            kc, vc, kIc, S = kc0, vc0, kIc0, S0
        else:
            kc, vc, kIc, S = kc0.clone(), vc0.clone(), kIc0.clone(), S0.clone()
        flat, dv = _packed_inputs(dv0, dev_alloc)
        ws = lisa.workspace(D, lisa.LISA_OP_DECODE_STEP, device)
        o = torch.empty(B, 1, wl.H_q, wl.d, dtype=torch.bfloat16, device=device)
        a = lisa.decode_args(dv["q"], dv["k_new"], dv["v_new"], dv["q_I"], dv["k_I_new"],
                             dv["w"], wl.H_I, dv["q"], dv["k_new"], dv["v_new"], dv["gate"],
                             kc, vc, kIc, S, None, o)
        copies.append(dict(dv=dv, flat=flat, ws=ws, o=o, a=a, S=S, kc=kc, vc=vc, kIc=kIc))

    def step(i):
        c = copies[i % len(copies)]
        lisa.lisa_decode_step(D, c["a"], c["ws"], stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    for c in copies:
        assert lisa.lisa_check_status(c["ws"], stream) == lisa.LISA_OK

    def run_block(k):  # noqa: ARG001
        for i in range(args.steps):
            step(i)

    graph = None
    if args.graphs:
        # one CUDA graph holding the K steps of a block (cycling through the
        # state copies): a timed block is one graph launch, so the host's launch
        # cost stays off the GPU, and each step's kernel is a programmatic
        # dependent of the one before it (its launch and shared-memory set-up
        # overlap the previous step's end)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for i in range(args.steps):
                lisa.lisa_decode_step(D, copies[i % len(copies)]["a"], copies[i % len(copies)]["ws"])
        stream = torch.cuda.current_stream()

        def run_block(k):  # noqa: F811,ARG001
            graph.replay()

        for _ in range(max(1, args.warmup // max(1, args.steps)) + 1):
            run_block(0)
        torch.cuda.synchronize()
        for c in copies:
            assert lisa.lisa_check_status(c["ws"], stream) == lisa.LISA_OK

    # The K timed steps run back to back between CUDA events on the launching
    # stream (an event pair around every step would add its own gap to each
    # step).  Blocks of K steps repeat, with an event at each block boundary and
    # no host synchronisation between them, until about --min-seconds of device
    # time have passed, so that the clock samples taken inside the timed region
    # are many; the reported time is the median block's.
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
    except Exception:
        gpu_id = str(device.index)
    with ClockSampler(gpu_id) as clk:
        blocks, w0, w1 = time_blocks(run_block, stream, args.min_seconds)
    if world > 1:
        dist.barrier()
    for c in copies:
        assert lisa.lisa_check_status(c["ws"], stream) == lisa.LISA_OK
    total_ms = max_over_ranks(statistics.median(blocks), device, world)
    del graph

    # ---- end to end through the public API with host buffers: every step
    # copies its inputs (packed in one pinned buffer laid out like the device
    # one) host to device in one copy, runs lisa_decode_step and reads o back
    pinned, _ = _packed_inputs(
        {k: torch.from_numpy(np.ascontiguousarray(v)).to(torch.float32 if k == "w" else torch.bfloat16)
         for k, v in host.items()},
        lambda nb: torch.empty(nb, dtype=torch.uint8).pin_memory())
    o_host = torch.empty(copies[0]["o"].shape, dtype=torch.bfloat16).pin_memory()
    h2d = pinned.numel()
    d2h = o_host.numel() * o_host.element_size()

    # The copies run on their own stream, pipelined as a serving loop would:
    # step i+1's inputs go up while step i's kernel runs (into the state copy
    # step i+1 uses, once the kernel that last read it is done), and o of step
    # i comes down after that kernel.  Every step's bytes still cross inside the
    # timed region, which ends when the last read-back has landed.
    R = len(copies)
    cstream = torch.cuda.Stream(device)
    up = [torch.cuda.Event() for _ in range(R)]    # inputs of the copy's next step landed
    done = [torch.cuda.Event() for _ in range(R)]  # the copy's last kernel finished
    used = [False] * R

    def upload(j):
        slot = j % R
        if used[slot]:
            cstream.wait_event(done[slot])
        with torch.cuda.stream(cstream):
            copies[slot]["flat"].copy_(pinned, non_blocking=True)
        up[slot].record(cstream)

    def e2e_run(count):
        upload(0)
        for i in range(count):
            slot = i % R
            if i + 1 < count:
                upload(i + 1)
            stream.wait_event(up[slot])
            lisa.lisa_decode_step(D, copies[slot]["a"], copies[slot]["ws"], stream)
            done[slot].record(stream)
            used[slot] = True
            cstream.wait_event(done[slot])
            with torch.cuda.stream(cstream):
                o_host.copy_(copies[slot]["o"], non_blocking=True)
        stream.wait_stream(cstream)

    e2e_run(max(1, args.warmup))
    torch.cuda.synchronize()
    e_st = torch.cuda.Event(enable_timing=True)
    e_en = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e_st.record(stream)
    e2e_run(args.steps)
    e_en.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e_st.elapsed_time(e_en), device, world)

    extra = run_next_rows(args, wl, copies, D, stream) if args.next_rows else {}

    bytes_ = decode_bytes(wl)
    avg_s = total_ms / 1e3 / args.steps
    hbm_peak, _, peak_kind = _peaks()
    achieved = bytes_["total"] / avg_s / 1e9
    value = job_throughput(B, world, args.steps, total_ms)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded Philox inputs, 1% planted heavy keys)",
        "config": {"workload": wl.name, "B": B, "context": n, "H_q": wl.H_q, "H_kv": wl.H_kv,
                   "d": wl.d, "H_I": wl.H_I, "d_I": wl.d_I, "M": wl.M,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": f"inputs larger than L2: {args.rotate} copies of the decode state "
                         f"(caches, state, inputs) used in rotation, "
                         f"{args.rotate} x {bytes_['total'] / 1e6:.1f} MB touched per cycle",
                   "step": "decode step: append, linear update+readout, indexer scan, "
                           "top-M, sparse attention, gate (one cooperative kernel)",
                   "launch": "one CUDA graph of the K lisa_decode_step calls of a block, "
                             "each kernel a programmatic dependent of the previous one"
                             if args.graphs else "lisa_decode_step from the host"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak, "peak_kind": peak_kind,
                     "frac_of_8TBs": achieved / 8000.0,
                     "traffic": _profiled_traffic(wl),
                     "algorithmic_bytes_per_launch": bytes_["total"],
                     "kernel": "decode step: one lisa_decode_step call = one k_decode_coop "
                               "launch (cooperative, one CTA per SM)",
                     "launch_us": avg_s * 1e6},
        "e2e": {"value": job_throughput(B, world, args.steps, e2e_ms), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "timing": {"blocks": len(blocks), "steps_per_block": args.steps,
                   "block_ms_median": statistics.median(blocks), "block_ms_min": min(blocks),
                   "block_ms_max": max(blocks), "timed_region_s": w1 - w0,
                   "what": "blocks of K steps back to back, an event at each block boundary; "
                           "value and ms_per_step from the median block (max over ranks)"},
        "gpu_launches": DECODE_KERNELS_PER_STEP * args.steps * len(blocks),
        "clocks": clk.summary(w0, w1),
    }
    line.update(extra)
    return line


# ----------------------------------------------------------------------------- helpers
def graph_timed(calls, steps: int, warmup: int):
    """Captures one CUDA graph issuing every call once (each a closure issuing
    one library call on the current stream, typically one per state copy) and
    replays it: enough untimed replays for `warmup` calls, then enough for at
    least `steps` calls between one event pair on the launching stream.
    Returns the device time per call in ms."""
    import torch

    for c in calls:
        c()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for c in calls:
            c()
    cur = torch.cuda.current_stream()
    per = len(calls)
    for _ in range(max(1, math.ceil(warmup / per))):
        g.replay()
    torch.cuda.synchronize()
    reps = max(1, math.ceil(steps / per))
    a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a_.record(cur)
    for _ in range(reps):
        g.replay()
    b_.record(cur)
    torch.cuda.synchronize()
    ms = a_.elapsed_time(b_) / (reps * per)
    del g
    return ms


def hbm_roof(nbytes: float, ms: float) -> dict:
    hbm_peak, _, peak_kind = _peaks()
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"bound": "hbm", "algorithmic_bytes_per_launch": nbytes, "achieved": gbs,
            "peak": hbm_peak, "unit": "GB/s", "frac": gbs / hbm_peak, "peak_kind": peak_kind,
            "traffic": None}


def device_decode_state(wl, device, seed: int):
    """Seeded synthetic decode state drawn on the device with torch's generator,
    for the timing-only lines (drawing 32 sequences of 64K tokens through the
    per-block host streams would take minutes).  Same recipe as the workload
    generator: N(0, sigma^2) values, 1% of positions per sequence planted with
    3 sigma sqrt(dim) along one shared unit direction in k and k_I, bf16."""
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(seed)
    bf = torch.bfloat16
    B, n = wl.B, wl.n

    def rn(*shape, scale=wl.sigma):
        return (torch.randn(*shape, generator=g, device=device, dtype=torch.float32) * scale).to(bf)

    kc = torch.empty(B, n, wl.H_kv, wl.d, dtype=bf, device=device)
    vc = torch.empty_like(kc)
    kI = torch.empty(B, n, wl.H_Ik, wl.d_I, dtype=bf, device=device)
    u = torch.randn(wl.d, generator=g, device=device)
    uI = torch.randn(wl.d_I, generator=g, device=device)
    u, uI = u / u.norm(), uI / uI.norm()
    cnt = n // 100
    for b in range(B):  # one sequence at a time keeps the fp32 temporaries small
        kc[b] = rn(n, wl.H_kv, wl.d)
        vc[b] = rn(n, wl.H_kv, wl.d)
        kI[b] = rn(n, wl.H_Ik, wl.d_I)
        if cnt:
            pos = torch.randperm(n, generator=g, device=device)[:cnt]
            kc[b, pos] = (kc[b, pos].float() + 3 * wl.sigma * math.sqrt(wl.d) * u).to(bf)
            kI[b, pos] = (kI[b, pos].float() + 3 * wl.sigma * math.sqrt(wl.d_I) * uI).to(bf)
    p = n - 1
    step = {"q": rn(B, 1, wl.H_q, wl.d), "q_I": rn(B, 1, wl.H_I, wl.d_I),
            "w": torch.rand(B, 1, wl.H_I, generator=g, device=device),
            "gate": rn(B, 1, wl.H_q, scale=1.0),
            "k_new": kc[:, p:].clone(), "v_new": vc[:, p:].clone(), "k_I_new": kI[:, p:].clone()}
    S = torch.randn(B, wl.H_kv, wl.d, wl.d, generator=g, device=device) * 0.05
    return kc, vc, kI, S, step


def coop_decode_kernel(B: int, n: int, window_M: int = 0, sms: int = 148) -> str:
    """Which decode kernel the library's dispatch picks for B sequences at
    context n: the cooperative kernel while each CTA's share of the positions
    fits its shared memory (at most 8192), else the four-kernel form."""
    m = min(window_M, n) if window_M else n
    ncta = max(1, min(sms // max(1, B), (m + 15) // 16))
    kpc = (-(-m // ncta) + 15) // 16 * 16
    return ("k_decode_coop" if B <= sms and kpc <= 8192
            else "k_decode_scan, k_decode_select, k_decode_attend, k_decode_combine")


def run_sweep(args, device):
    """The long-context decode sweep: B=32 sequences at every context of 4K-64K
    with both budgets (tok/s and HBM fraction per point), the Stage-1 window
    step at the same budgets (the sparse branch alone, no indexer scan: its
    cost must stay flat in the context), and dense causal attention over the
    same caches (the O(n) reference line)."""
    import torch

    from hybrid_linear_top_lightning_b200 import inputs, lisa

    points, dense, window = [], [], {}
    for n in inputs.SWEEP_CTX:
        wl0 = inputs.sweep_workload(n, min(inputs.SWEEP_M))
        kc0, vc0, kI0, S0, st0 = device_decode_state(wl0, device, seed=1000 + n)
        ncopy = int(min(4, max(1, math.ceil(400e6 / decode_bytes(wl0)["total"]))))
        copies = []
        for r in range(ncopy):
            if r == 0:
                c = dict(kc=kc0, vc=vc0, kI=kI0, S=S0, st=st0)
            else:
                c = dict(kc=kc0.clone(), vc=vc0.clone(), kI=kI0.clone(), S=S0.clone(),
                         st={k: v.clone() for k, v in st0.items()})
            c["o"] = torch.empty(wl0.B, 1, wl0.H_q, wl0.d, dtype=torch.bfloat16, device=device)
            copies.append(c)
        for M in inputs.SWEEP_M:
            wl = inputs.sweep_workload(n, M)
            D = lisa.make_dims(wl.B, 1, n - 1, n, wl.H_q, wl.H_kv, wl.d, wl.H_I, wl.H_Ik, wl.d_I, M)
            calls_d, calls_w = [], []
            for c in copies:
                st = c["st"]
                a = lisa.decode_args(st["q"], st["k_new"], st["v_new"], st["q_I"], st["k_I_new"],
                                     st["w"], wl.H_I, st["q"], st["k_new"], st["v_new"],
                                     st["gate"], c["kc"], c["vc"], c["kI"], c["S"], None, c["o"])
                ws = lisa.workspace(D, lisa.LISA_OP_DECODE_STEP, device)
                calls_d.append(lambda a=a, ws=ws: lisa.lisa_decode_step(D, a, ws))
                calls_w.append(lambda a=a, ws=ws: lisa.lisa_decode_step_window(D, a, ws))
                c.setdefault("ws", []).append(ws)
            ms_d = graph_timed(calls_d, args.steps, args.warmup)
            ms_w = graph_timed(calls_w, args.steps, args.warmup)
            for c in copies:
                for ws in c.pop("ws"):
                    assert lisa.lisa_check_status(ws) == lisa.LISA_OK
            db, wb = decode_bytes(wl), window_bytes(wl)
            points.append({"context": n, "M": M, "B": wl.B, "us_per_step": ms_d * 1e3,
                           "value": wl.B / (ms_d / 1e3), "unit": "tok/s",
                           "kernel": coop_decode_kernel(wl.B, n),
                           "l2": f"{ncopy} state copies in rotation",
                           "roofline": hbm_roof(db["total"], ms_d)})
            window.setdefault(M, []).append({"context": n, "us_per_step": ms_w * 1e3,
                                             "kernel": coop_decode_kernel(wl.B, n, M),
                                             "roofline": hbm_roof(wb["total"], ms_w)})
        # dense causal attention over the same caches (one query token per sequence)
        Dd = lisa.make_dims(wl0.B, 1, n - 1, n, wl0.H_q, wl0.H_kv, wl0.d, wl0.H_I, wl0.H_Ik,
                            wl0.d_I, wl0.M)
        calls, wss = [], []
        for c in copies:
            ws = lisa.workspace(Dd, lisa.LISA_OP_DENSE_ATTN, device)
            wss.append(ws)
            calls.append(lambda c=c, ws=ws: lisa.lisa_dense_attn(Dd, c["st"]["q"], c["kc"],
                                                                c["vc"], c["o"], ws))
        ms = graph_timed(calls, max(4, args.steps // 4), args.warmup)
        for ws in wss:
            assert lisa.lisa_check_status(ws) == lisa.LISA_OK
        nbytes = wl0.B * (n * wl0.H_kv * wl0.d * 2 * 2 + 2 * wl0.H_q * wl0.d * 2)
        dense.append({"context": n, "B": wl0.B, "us_per_call": ms * 1e3,
                      "value": wl0.B / (ms / 1e3), "unit": "tok/s",
                      "roofline": hbm_roof(nbytes, ms)})
        del copies, kc0, vc0, kI0, S0, st0
        torch.cuda.empty_cache()
    # the O(M)-not-O(n) check: at a fixed budget the sparse branch's time stays
    # flat across the contexts (window step), while the full step grows with
    # the indexer scan (128 bytes per cached token per sequence)
    flat = {}
    for M, rows in window.items():
        us = [r["us_per_step"] for r in rows]
        full = [p["us_per_step"] for p in points if p["M"] == M]
        flat[str(M)] = {"contexts": [r["context"] for r in rows], "window_us": us,
                        "window_max_over_min": max(us) / min(us), "decode_us": full,
                        "decode_max_over_min": max(full) / min(full),
                        "scan_bytes_per_seq": [128 * r["context"] for r in rows],
                        "gather_bytes_per_seq": [min(int(M), r["context"]) * 2048 for r in rows]}
    return {"what": "decode step at B=32 over every (context, budget) point, with the "
                    "Stage-1 window step at the same budgets and dense causal attention "
                    "(lisa_dense_attn) on the same caches",
            "data": "seeded synthetic caches drawn on the device (torch generator; the "
                    "workload recipe: N(0, 1/128), 1% planted heavy keys, bf16)",
            "points": points, "dense": dense,
            "window": {str(M): rows for M, rows in window.items()},
            "o_of_m_check": flat}


# ----------------------------------------------------------------------------- next rows
def window_bytes(wl) -> dict:
    """Algorithmic HBM bytes of one sliding-window decode step: the last M K/V
    rows (contiguous), the state read and written, the step's small tensors."""
    M = min(wl.M, wl.n)
    gather = M * wl.H_kv * wl.d * 2 * 2
    state = wl.H_kv * wl.d * wl.d * 4 * 2
    small = wl.H_q * wl.d * 2 * 3 + wl.H_kv * wl.d * 2 * 2 * 2 + wl.H_q * 2
    per_seq = gather + state + small
    return dict(per_seq=per_seq, total=per_seq * wl.B)


def run_next_rows(args, wl, copies, D, stream):
    """The Stage-1 sliding-window decode step and the segment state transfer,
    on the same decode state: device-timed lines with their HBM rooflines."""
    import torch

    from hybrid_linear_top_lightning_b200 import lisa

    hbm_peak, _, peak_kind = _peaks()
    out = {}
    # ---- sliding-window decode step (no indexer), one graph over the copies
    cur = torch.cuda.current_stream()
    ms = graph_timed([lambda c=c: lisa.lisa_decode_step_window(D, c["a"], c["ws"]) for c in copies],
                     args.steps, args.warmup)
    for c in copies:
        assert lisa.lisa_check_status(c["ws"], cur) == lisa.LISA_OK
    wb = window_bytes(wl)
    out["window"] = {
        "what": "decode step with the Stage-1 sliding window (last M positions, no indexer): "
                "lisa_decode_step_window, one cooperative kernel",
        "value": wl.B / (ms / 1e3), "unit": "tok/s", "us_per_step": ms * 1e3,
        "roofline": {"bound": "hbm", "algorithmic_bytes_per_launch": wb["total"],
                     "achieved": wb["total"] / (ms / 1e3) / 1e9, "peak": hbm_peak, "unit": "GB/s",
                     "frac": wb["total"] / (ms / 1e3) / 1e9 / hbm_peak, "peak_kind": peak_kind,
                     "traffic": None}}
    # ---- the elu+1 feature map with its normaliser z (the same state copies,
    # a positive z each); the step also advances z
    De = lisa.make_dims(wl.B, 1, wl.n - 1, wl.n, wl.H_q, wl.H_kv, wl.d, wl.H_I, wl.H_Ik,
                        wl.d_I, wl.M, phi=lisa.LISA_PHI_ELU1_NORM)
    calls = []
    for c in copies:
        dv = c["dv"]
        z = torch.rand(wl.B, wl.H_kv, wl.d, device=stream.device) * 20.0 + 1.0
        ae = lisa.decode_args(dv["q"], dv["k_new"], dv["v_new"], dv["q_I"], dv["k_I_new"],
                              dv["w"], wl.H_I, dv["q"], dv["k_new"], dv["v_new"], dv["gate"],
                              c["kc"], c["vc"], c["kIc"], c["S"], z, c["o"])
        calls.append(lambda ae=ae, ws=c["ws"]: lisa.lisa_decode_step(De, ae, ws))
    ms = graph_timed(calls, args.steps, args.warmup)
    for c in copies:
        assert lisa.lisa_check_status(c["ws"], cur) == lisa.LISA_OK
    eb = decode_bytes(wl, elu1=True)
    out["elu1"] = {
        "what": "decode step with the elu+1 feature map and its normaliser "
                "(phi = LISA_PHI_ELU1_NORM), one cooperative kernel",
        "value": wl.B / (ms / 1e3), "unit": "tok/s", "us_per_step": ms * 1e3,
        "roofline": hbm_roof(eb["total"], ms)}

    # ---- the paper's indexer form: a key per indexer head (H_Ik = H_I = 8), w = 1
    from hybrid_linear_top_lightning_b200 import inputs

    wl8 = wl.with_(H_Ik=wl.H_I)
    gen8 = inputs.Generator(wl8)
    n, p, B = wl.n, wl.n - 1, wl.B
    kI8 = torch.empty(B, n, wl.H_I, wl.d_I, dtype=torch.bfloat16, device=stream.device)
    for b in range(B):
        kI8[b] = torch.from_numpy(gen8.k_I(b, 0, n)).to(torch.bfloat16)
    D8 = lisa.make_dims(B, 1, p, n, wl.H_q, wl.H_kv, wl.d, wl.H_I, wl.H_I, wl.d_I, wl.M)
    w1 = torch.ones(B, 1, wl.H_I, device=stream.device)
    pf = []
    for i, c in enumerate(copies):
        kc8 = kI8 if i == 0 else kI8.clone()
        kI_new = kc8[:, p:].clone()
        dv = c["dv"]
        a8 = lisa.decode_args(dv["q"], dv["k_new"], dv["v_new"], dv["q_I"], kI_new, w1, wl.H_I,
                              dv["q"], dv["k_new"], dv["v_new"], dv["gate"], c["kc"], c["vc"], kc8,
                              c["S"], None, c["o"])
        pf.append(dict(a=a8, ws=lisa.workspace(D8, lisa.LISA_OP_DECODE_STEP, stream.device)))
    ms = graph_timed([lambda c=c: lisa.lisa_decode_step(D8, c["a"], c["ws"]) for c in pf],
                     args.steps, args.warmup)
    for c in pf:
        assert lisa.lisa_check_status(c["ws"], cur) == lisa.LISA_OK
    pb = decode_bytes(wl8)
    out["paper_form"] = {
        "what": "decode step with the paper's indexer form: a key per indexer head "
                "(H_Ik = H_I = 8, 1 KB of k_I per token), unweighted head sum",
        "value": B / (ms / 1e3), "unit": "tok/s", "us_per_step": ms * 1e3,
        "roofline": {"bound": "hbm", "algorithmic_bytes_per_launch": pb["total"],
                     "achieved": pb["total"] / (ms / 1e3) / 1e9, "peak": hbm_peak, "unit": "GB/s",
                     "frac": pb["total"] / (ms / 1e3) / 1e9 / hbm_peak, "peak_kind": peak_kind,
                     "traffic": None}}
    del pf, kI8

    # ---- segment state transfer over B x H_kv states of d x d fp32; 16 sets of
    # (S, S_start, grad_sum) in rotation (201 MB, larger than L2)
    shape = (wl.B, wl.H_kv, wl.d, wl.d)
    states = [tuple(torch.randn(shape, device=stream.device) for _ in range(3)) for _ in range(16)]
    for t in range(1, args.warmup + 1):
        for S, S0, G in states:
            lisa.lisa_state_transfer(D, S, S0, G, t, 0.25, stream)
    torch.cuda.synchronize()
    # one graph of 16 calls (a call is a few microseconds: shorter than a host launch)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for S, S0, G in states:
            lisa.lisa_state_transfer(D, S, S0, G, args.warmup + 1, 0.25)
    g.replay()
    torch.cuda.synchronize()
    reps = max(4, args.steps // 8)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(reps)]
    for a_, b_ in ev:
        a_.record(cur)
        g.replay()
        b_.record(cur)
    torch.cuda.synchronize()
    ms = sum(a_.elapsed_time(b_) for a_, b_ in ev) / (reps * len(states))
    st_bytes = 6 * wl.B * wl.H_kv * wl.d * wl.d * 4
    out["state_transfer"] = {
        "what": "segment state transfer and correction (Eq. 6-9) over B x H_kv states of d x d fp32",
        "us_per_call": ms * 1e3,
        "l2": "16 state sets in rotation (201 MB, larger than L2); a CUDA graph of 16 calls replayed",
        "roofline": {"bound": "hbm", "algorithmic_bytes_per_launch": st_bytes,
                     "achieved": st_bytes / (ms / 1e3) / 1e9, "peak": hbm_peak, "unit": "GB/s",
                     "frac": st_bytes / (ms / 1e3) / 1e9 / hbm_peak, "peak_kind": peak_kind,
                     "traffic": None}}
    del states, g

    # ---- one recurrent step of the linear branch alone (lisa_linear_decode) at
    # the headline shape; 64 state sets in rotation (134 MB, larger than L2)
    nsets = 64
    sets = [dict(S=torch.randn(shape, device=stream.device) * 0.05,
                 q=torch.randn(wl.B, 1, wl.H_q, wl.d, device=stream.device).to(torch.bfloat16),
                 k=torch.randn(wl.B, 1, wl.H_kv, wl.d, device=stream.device).to(torch.bfloat16),
                 v=torch.randn(wl.B, 1, wl.H_kv, wl.d, device=stream.device).to(torch.bfloat16),
                 o=torch.empty(wl.B, 1, wl.H_q, wl.d, device=stream.device, dtype=torch.bfloat16))
            for _ in range(nsets)]
    ms = graph_timed([lambda c=c: lisa.lisa_linear_decode(D, c["q"], c["k"], c["v"], c["S"], None, c["o"])
                      for c in sets], args.steps, args.warmup)
    ld_bytes = 2 * wl.B * wl.H_kv * wl.d * wl.d * 4 + 2 * wl.B * (2 * wl.H_q + 2 * wl.H_kv) * wl.d
    out["linear_decode"] = {
        "what": "one recurrent step of the linear branch (lisa_linear_decode, identity map): "
                "S += phi(k)^T v, o = phi(q) S over B x H_kv states of d x d fp32",
        "us_per_call": ms * 1e3,
        "l2": f"{nsets} state sets in rotation ({nsets * wl.B * wl.H_kv * wl.d * wl.d * 4 / 1e6:.0f} MB, "
              "larger than L2); a CUDA graph of one call per set replayed",
        "roofline": {"bound": "hbm", "algorithmic_bytes_per_launch": ld_bytes,
                     "achieved": ld_bytes / (ms / 1e3) / 1e9, "peak": hbm_peak, "unit": "GB/s",
                     "frac": ld_bytes / (ms / 1e3) / 1e9 / hbm_peak, "peak_kind": peak_kind,
                     "traffic": None}}
    return out


# ----------------------------------------------------------------------------- channel gate
def run_gate_channel(args, device, T_prefill=None):
    """The per-channel gate (Sec. 3.3 Eq. 5) at the 7B width (3584 channels,
    D_h 3584): the 16384-token prefill on the tensor cores (TFLOP/s) and the
    8-token decode, which streams W_g once (GB/s).  L2 is flushed before every
    timed prefill call; the decode calls rotate over copies of W_g larger than
    L2 together."""
    import numpy as np
    import torch

    from hybrid_linear_top_lightning_b200 import inputs, lisa

    hbm_peak, tc_peak, peak_kind = _peaks()
    out = {}
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()
    for label, wl in (("prefill", inputs.PREFILL_7B), ("decode", inputs.DECODE_7B)):
        T = wl.n if label == "prefill" else 1
        if label == "prefill" and T_prefill:
            T = T_prefill
        D_h = N = wl.H_q * wl.d
        gen = inputs.Generator(wl)
        h = torch.from_numpy(np.stack([gen.hidden(b, 0, T, D_h) for b in range(wl.B)]))
        h = h.to(torch.bfloat16).to(device)
        W = torch.from_numpy(gen.gate_weight(D_h)).to(torch.bfloat16).to(device)
        o_lin = torch.from_numpy(np.stack([gen.branch("o_lin", b, 0, T) for b in range(wl.B)]))
        o_lin = o_lin.to(torch.bfloat16).to(device)
        o_sp = torch.from_numpy(np.stack([gen.branch("o_sp", b, 0, T) for b in range(wl.B)]))
        o_sp = o_sp.to(torch.bfloat16).to(device)
        o = torch.empty_like(o_lin)
        D = lisa.make_dims(wl.B, T, 0, T, wl.H_q, wl.H_kv, wl.d, wl.H_I, wl.H_Ik, wl.d_I, wl.M)
        ws = lisa.workspace(D, lisa.LISA_OP_GATE_CHANNEL, device)
        for _ in range(args.warmup):
            lisa.lisa_gate_channel(D, D_h, h, W, o_lin, o_sp, o, ws, stream)
        torch.cuda.synchronize()
        if label == "prefill":
            reps = max(3, min(args.steps, 20))
            tot = 0.0
            for _ in range(reps):
                flush.fill_(1)  # evict the previous call's data from L2
                a_ = torch.cuda.Event(enable_timing=True)
                b_ = torch.cuda.Event(enable_timing=True)
                a_.record(stream)
                lisa.lisa_gate_channel(D, D_h, h, W, o_lin, o_sp, o, ws, stream)
                b_.record(stream)
                torch.cuda.synchronize()
                tot += a_.elapsed_time(b_)
            ms = tot / reps
        else:
            # a call is a few microseconds, shorter than a host launch: one graph of
            # 8 calls over 8 copies of W_g (207 MB in rotation, larger than L2)
            Ws = [W] + [W.clone() for _ in range(7)]
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for Wc in Ws:
                    lisa.lisa_gate_channel(D, D_h, h, Wc, o_lin, o_sp, o, ws)
            g.replay()
            torch.cuda.synchronize()
            reps = max(4, args.steps // 4)
            a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a_.record(stream)
            for _ in range(reps):
                g.replay()
            b_.record(stream)
            torch.cuda.synchronize()
            ms = a_.elapsed_time(b_) / (reps * len(Ws))
            del g, Ws
        assert lisa.lisa_check_status(ws, stream) == lisa.LISA_OK
        tokens = wl.B * T
        nbytes = 2 * (tokens * D_h + N * D_h + 3 * tokens * N)
        flops = 2.0 * tokens * N * D_h
        if label == "prefill":
            roof = {"bound": "tensor", "algorithmic_flops_per_launch": flops,
                    "achieved": flops / (ms / 1e3) / 1e12, "peak": tc_peak, "unit": "TFLOP/s",
                    "frac": flops / (ms / 1e3) / 1e12 / tc_peak, "peak_kind": peak_kind,
                    "traffic": None}
        else:
            roof = {"bound": "hbm", "algorithmic_bytes_per_launch": nbytes,
                    "achieved": nbytes / (ms / 1e3) / 1e9, "peak": hbm_peak, "unit": "GB/s",
                    "frac": nbytes / (ms / 1e3) / 1e9 / hbm_peak, "peak_kind": peak_kind,
                    "traffic": None}
        out[label] = {"tokens": tokens, "channels": N, "D_h": D_h, "us_per_call": ms * 1e3,
                      "value": tokens / (ms / 1e3), "unit": "tok/s", "roofline": roof}
        del h, W, o_lin, o_sp, o, ws
    out["what"] = ("per-channel gate g = sigmoid(W_g h) mixing the branches (Eq. 5): "
                   "lisa_gate_channel, 7B width")
    return out


# ----------------------------------------------------------------------------- prefill
def prefill_work(wl) -> dict:
    """Algorithmic work of one causal prefill of wl.n tokens per sequence: causal
    indexer pairs, key visits of the sparse attention (sum over rows of
    min(M, t+1)) and the chunk GEMMs of the linear branch (flops, all B)."""
    n, M = wl.n, wl.M
    pairs = n * (n + 1) // 2
    visits = sum(min(M, t + 1) for t in range(n))
    indexer = pairs * wl.H_I * wl.d_I * 2
    sparse = visits * wl.H_q * wl.d * 2 * 2
    C = wl.chunk
    nc = (n + C - 1) // C
    # per chunk and KV head: K^T V (d x d x C); per query head: Q S (C x d x d),
    # Q K^T (C x C x d, causal half) and P V (C x C x d, causal half)
    lin = nc * (wl.H_kv * 2 * wl.d * wl.d * C
                + wl.H_q * (2 * C * wl.d * wl.d + 2 * 2 * (C * (C + 1) // 2) * wl.d))
    # the masked tensor-core attention runs 128-query x 64-key tiles: every
    # 64-key tile of a 128-row query tile's causal range that one of its rows
    # selects from (all of them for these selections) costs the full tile
    tiles = sum((min((qt + 1) * 128, n) + 63) // 64 for qt in range((n + 127) // 128))
    sparse_tiles = tiles * wl.H_q * 128 * 64 * wl.d * 2 * 2
    return dict(pairs=pairs * wl.B, visits=visits * wl.B, indexer=indexer * wl.B,
                sparse=sparse * wl.B, linear=lin * wl.B, sparse_tiles=sparse_tiles * wl.B,
                total=(indexer + sparse + lin) * wl.B)


def run_prefill(args, wl, device):
    """Times one whole-module prefill (lisa_prefill) of the 7B-shaped layer and,
    separately, each of its four stages; L2 is flushed before every timed call."""
    import torch

    from hybrid_linear_top_lightning_b200 import inputs, lisa

    gen = inputs.Generator(wl)
    n, B, bf = wl.n, wl.B, torch.bfloat16

    def dv(name, dt=bf):
        return torch.from_numpy(gen.batch(name, 0, n)).to(dt).to(device)

    q, k, v, qI, kI = dv("q"), dv("k"), dv("v"), dv("q_I"), dv("k_I")
    w, gl = dv("w", torch.float32), dv("gate")
    D = lisa.make_dims(B, n, 0, n, wl.H_q, wl.H_kv, wl.d, wl.H_I, wl.H_Ik, wl.d_I, wl.M,
                       chunk=wl.chunk)
    S = torch.zeros(B, wl.H_kv, wl.d, wl.d, device=device)
    o = torch.empty(B, n, wl.H_q, wl.d, dtype=bf, device=device)
    o_sp, o_lin = torch.empty_like(o), torch.empty_like(o)
    idx = torch.empty(B, n, wl.M, dtype=torch.int32, device=device)
    cnt = torch.empty(B, n, dtype=torch.int32, device=device)
    De = lisa.make_dims(B, n, 0, n, wl.H_q, wl.H_kv, wl.d, wl.H_I, wl.H_Ik, wl.d_I, wl.M,
                        chunk=wl.chunk, phi=lisa.LISA_PHI_ELU1_NORM)
    z = torch.zeros(B, wl.H_kv, wl.d, device=device)
    ws = lisa.workspace(D, lisa.LISA_OP_PREFILL, device)
    args_p = lisa.prefill_args(q, k, v, qI, kI, w, wl.H_I, q, k, v, gl, S, None, o, idx, cnt)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()

    stages = {
        "whole": lambda: lisa.lisa_prefill(D, args_p, ws, stream),
        "topm": lambda: lisa.lisa_topm(D, qI, kI, w, wl.H_I, idx, cnt, ws, stream),
        "sparse_attn": lambda: lisa.lisa_sparse_attn(D, q, k, v, idx, cnt, o_sp, ws, stream),
        "linear": lambda: lisa.lisa_linear_prefill(D, q, k, v, S, None, o_lin, ws, stream),
        "linear_elu1": lambda: lisa.lisa_linear_prefill(De, q, k, v, S, z, o_lin, ws, stream),
        "gate": lambda: lisa.lisa_gate_fuse(D, gl, o_lin, o_sp, o, stream),
    }
    steps = max(1, args.prefill_steps)
    times = {}
    for name, fn in stages.items():
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(steps):
            flush.fill_(1)  # evict the previous call's data from L2
            a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a_.record(stream)
            fn()
            b_.record(stream)
            torch.cuda.synchronize()
            ts.append(a_.elapsed_time(b_))
        times[name] = statistics.median(ts)
        assert lisa.lisa_check_status(ws, stream) == lisa.LISA_OK
    work = prefill_work(wl)
    _, tc_burst, peak_kind = _peaks()
    whole_s = times["whole"] / 1e3
    idx_tf = work["indexer"] / (times["topm"] / 1e3) / 1e12
    lin_tf = work["linear"] / (times["linear"] / 1e3) / 1e12
    lin_e_tf = work["linear"] / (times["linear_elu1"] / 1e3) / 1e12
    sp_tf = work["sparse"] / (times["sparse_attn"] / 1e3) / 1e12
    sp_tile_tf = work["sparse_tiles"] / (times["sparse_attn"] / 1e3) / 1e12
    return {
        "workload": wl.name, "B": B, "n": n, "M": wl.M, "H_q": wl.H_q, "H_kv": wl.H_kv,
        "value": B * n / whole_s, "unit": "tok/s", "ms": times["whole"], "steps": steps,
        "stage_ms": {k_: v_ for k_, v_ in times.items() if k_ != "whole"},
        "stage_note": "linear_elu1 is the linear branch with the elu+1 feature map and its "
                      "normaliser (not part of the whole-module time, which uses the identity)",
        "gpu_launches_per_prefill": 7,
        "l2": "256 MB buffer written before every timed call",
        "work": {"indexer_gflop": work["indexer"] / 1e9, "sparse_gflop": work["sparse"] / 1e9,
                 "sparse_tile_gflop": work["sparse_tiles"] / 1e9,
                 "linear_gflop": work["linear"] / 1e9},
        "roofline": {
            "bound": "tensor", "unit": "TFLOP/s", "peak": tc_burst, "peak_kind": peak_kind,
            "achieved": work["total"] / whole_s / 1e12,
            "frac": work["total"] / whole_s / 1e12 / tc_burst,
            "indexer_tflops_incl_select": idx_tf, "indexer_frac_incl_select": idx_tf / tc_burst,
            "linear_tflops": lin_tf, "linear_frac": lin_tf / tc_burst,
            "linear_elu1_tflops": lin_e_tf, "linear_elu1_frac": lin_e_tf / tc_burst,
            "sparse_attn_tflops_selected": sp_tf, "sparse_attn_frac_selected": sp_tf / tc_burst,
            "sparse_attn_tflops_tiles": sp_tile_tf, "sparse_attn_frac_tiles": sp_tile_tf / tc_burst,
            "sparse_attn_note": "selected = the selected (query, key) pairs' products; tiles = "
                                "the products the tensor cores run over whole 128x64 tiles "
                                "(unselected keys are dropped in the softmax)",
            "traffic": None},
    }


# ----------------------------------------------------------------------------- CPU oracle
_ORACLE_INPUTS = {}


def _oracle_inputs(wl, seqs: int):
    """The seeded inputs of `seqs` sequences of the decode workload (drawn once)."""
    from hybrid_linear_top_lightning_b200 import inputs

    key = (wl.name, seqs)
    if key not in _ORACLE_INPUTS:
        gen = inputs.Generator(wl.with_(B=seqs))
        n, p = wl.n, wl.n - 1
        x = {k: gen.batch(k, 0, n) for k in ("k", "v", "k_I")}
        x.update({k: gen.batch(k, p, n) for k in ("q", "q_I", "w", "gate")})
        rng = np.random.default_rng(0)
        x["S0"] = rng.standard_normal((seqs, wl.H_kv, wl.d, wl.d)) * 0.1
        _ORACLE_INPUTS[key] = x
    return _ORACLE_INPUTS[key]


def oracle_decode_sample(wl, seqs: int, budget_s: float):
    """Time the oracle's decode step on `seqs` sequences of the workload, repeated
    until about `budget_s` seconds have passed.  Returns (tok/s, threads, note)."""
    from oracle import ref

    x = _oracle_inputs(wl, seqs)
    n, p = wl.n, wl.n - 1
    D = ref.Dims(B=seqs, T=1, n_past=p, N_max=n, H_q=wl.H_q, H_kv=wl.H_kv, d=wl.d, H_I=wl.H_I,
                 H_Ik=wl.H_Ik, d_I=wl.d_I, M=wl.M)
    kc, vc = x["k"], x["v"]
    reps = 0
    t0 = time.perf_counter()
    while True:
        ref.forward(D, x["q"], kc, vc, x["q_I"], x["k_I"], x["w"], wl.H_I, x["q"], kc[:, p:],
                    vc[:, p:], x["gate"], S0=x["S0"])
        reps += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    tok_s = reps * seqs / el
    thr = ref.num_threads()
    return tok_s, thr, (f"{reps} oracle decode steps of {seqs} sequences at context {n} "
                        f"(the full step per sequence: indexer over every key, full sort, "
                        f"sparse attention, linear branch, gate) in {el:.1f} s on {thr} "
                        f"thread(s)")


def oracle_prefill_sample(wl, stride: int, budget_s: float):
    """Time the oracle's whole module on every `stride`-th query row of one
    causal prefill of the workload (each sampled row: the indexer over all its
    causal keys, a full sort, sparse attention and the gate; the linear
    recurrence runs over every token), repeated until about `budget_s` seconds
    have passed.  Returns (sampled rows per second, threads, note)."""
    from hybrid_linear_top_lightning_b200 import inputs
    from oracle import ref

    gen = inputs.Generator(wl)
    n = wl.n
    x = {k: gen.batch(k, 0, n) for k in ("q", "k", "v", "q_I", "k_I", "w", "gate")}
    D = ref.Dims(B=wl.B, T=n, n_past=0, N_max=n, H_q=wl.H_q, H_kv=wl.H_kv, d=wl.d, H_I=wl.H_I,
                 H_Ik=wl.H_Ik, d_I=wl.d_I, M=wl.M)
    rows = np.arange(stride - 1, n, stride, dtype=np.int32)
    reps = 0
    t0 = time.perf_counter()
    while True:
        ref.forward(D, x["q"], x["k"], x["v"], x["q_I"], x["k_I"], x["w"], wl.H_I, x["q"], x["k"],
                    x["v"], x["gate"], rows=rows)
        reps += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    thr = ref.num_threads()
    return reps * rows.size * wl.B / el, thr, (
        f"{reps} oracle prefill pass(es) over every {stride}th query row ({rows.size} rows) of "
        f"the {n}-token prefill (per sampled row: indexer over its causal keys, full sort, sparse "
        f"attention, gate; the linear recurrence over all {n} tokens) in {el:.1f} s on {thr} "
        f"thread(s)")


def run_reference(args, wl):
    # rank 0 is the only worker of this arm, so it takes every core it may run
    # on (a multi-process launcher sets OMP_NUM_THREADS=1 for each rank)
    from oracle import ref
    ref.set_num_threads(len(os.sched_getaffinity(0)))
    tok_s, cores, note = oracle_decode_sample(wl, seqs=wl.B, budget_s=max(5.0, args.cpu_seconds))
    return {
        "metric": METRIC, "value": tok_s, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": wl.B / tok_s * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "B": wl.B, "context": wl.n, "M": wl.M},
        "impl": "reference",
        "cpu_baseline": {"value": tok_s, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": note},
        "e2e": {"value": tok_s, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="lisa", choices=["lisa", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--min-seconds", type=float, default=1.5,
                    help="device time of the timed region: blocks of --steps steps repeat "
                         "until it has passed (clock samples inside it)")
    ap.add_argument("--no-sweep", dest="sweep", action="store_false",
                    help="skip the long-context sweep (B=32, contexts 4K-64K, both budgets, "
                         "window and dense lines)")
    ap.add_argument("--rotate", type=int, default=4,
                    help="copies of the decode state used in rotation (inputs larger than L2)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graphs", dest="graphs", action="store_false",
                    help="launch every timed decode step from the host instead of replaying "
                         "a captured CUDA graph")
    ap.add_argument("--no-next-rows", dest="next_rows", action="store_false",
                    help="skip the sliding-window step and state-transfer lines")
    ap.add_argument("--prefill-steps", type=int, default=3,
                    help="timed calls per stage of the 7B prefill line (0: skip it)")
    ap.add_argument("--prefill-n", type=int, default=0,
                    help="prefill length of the prefill line (default: the 7B workload's 16384)")
    ap.add_argument("--prefill-only", action="store_true",
                    help="time only the prefill line and print it (for profiling runs)")
    ap.add_argument("--gate-only", action="store_true",
                    help="time only the per-channel gate lines and print them (for profiling)")
    ap.add_argument("--gate-T", type=int, default=0,
                    help="prefill tokens of the channel-gate line (default: 16384)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    from hybrid_linear_top_lightning_b200 import inputs

    wl = inputs.DECODE_7B
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, wl)), flush=True)
        return

    import torch
    import torch.distributed as dist

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
    try:
        wl_p = inputs.PREFILL_7B
        if args.prefill_n > 0:
            wl_p = wl_p.with_(n=args.prefill_n, name=f"prefill_7b_n{args.prefill_n}")
        if args.prefill_only:
            if rank == 0:
                print(json.dumps({"prefill": run_prefill(args, wl_p, device)}), flush=True)
            return
        if args.gate_only:
            if rank == 0:
                print(json.dumps({"gate_channel": run_gate_channel(args, device, args.gate_T)}),
                      flush=True)
            return
        line = run_gpu(args, wl, rank, world, device)
        if args.next_rows:
            line["gate_channel"] = run_gate_channel(args, device)
        if args.prefill_steps > 0:
            line["prefill"] = run_prefill(args, wl_p, device)
        if args.sweep:
            line["sweep"] = run_sweep(args, device)
            line["prefill_1p5b"] = run_prefill(args, inputs.PREFILL_1P5B, device)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            from oracle import ref
            ref.set_num_threads(len(os.sched_getaffinity(0)))
            tok_s, cores, note = oracle_decode_sample(wl, seqs=wl.B, budget_s=args.cpu_seconds)
            ref.set_num_threads(1)
            tok_1, _, note_1 = oracle_decode_sample(wl, seqs=wl.B,
                                                    budget_s=max(2.0, args.cpu_seconds / 2))
            ref.set_num_threads(cores)
            line["cpu_baseline"] = {"value": tok_s, "unit": UNIT, "cores": cores,
                                    "kind": "oracle", "sample": note,
                                    "single_thread": {"value": tok_1, "unit": UNIT, "cores": 1,
                                                      "sample": note_1}}
            if "prefill" in line:
                pt, pc, pnote = oracle_prefill_sample(wl_p, stride=16, budget_s=args.cpu_seconds)
                line["prefill"]["cpu_baseline"] = {"value": pt, "unit": "tok/s", "cores": pc,
                                                   "kind": "oracle", "sample": pnote}
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
