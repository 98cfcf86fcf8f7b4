#!/usr/bin/env python
"""Throughput of the fused QK-RMSNorm + RoPE forward + backward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...      (the CPU oracle, as the reference arm)

A step is one forward and one backward over one batch of the workload
(default: the largest single-GPU configuration, partial RoPE at long
context: one row of 65,536 tokens, 32 query / 8 KV heads of dim 128, rotary
on the first 32 dims, bf16 I/O). Inputs are resident in HBM before timing.
Each rank keeps a ring of input/output sets (four, more for small
workloads); step i runs the forward on set i and the backward on set i - 2
(a layer's backward comes after the rest of the forward in training), so no
kernel finds its inputs in the 126 MB L2. K steps are timed with CUDA events
between a barrier and a synchronize on both sides, with no event between the
launches; then K forward launches alone and K backward launches alone, back
to back, give the per-kernel times for the roofline. N > 1 (torchrun): weak scaling,
each rank its own batch, no collective on the data path; the time is the
max over ranks.

Rank 0 prints one JSON line. ``per_config`` times the other workloads the
same way (their own rings, forward and backward each). ``e2e`` repeats the
step through the public Python API from pinned host buffers (inputs copied
in, every output copied back, inside the timed region; two device slots and
three streams let one step's host-to-device copies overlap the previous
step's device-to-host copies). ``cpu_baseline``
times the CPU oracle on a bounded sample of the same workload, on one host
core and on all of them.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import platform
import statistics
import sys
import threading
import time
from concurrent.futures import ThreadPoolExecutor

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "QK-norm+RoPE fwd+bwd tokens/s and HBM GB/s (% of B200 peak), 1 GPU"
FALLBACK_HBM_GBS = 6650.0
NSETS, LAG = 4, 2  # ring of input sets; the backward runs LAG steps behind
L2_BYTES = 126 * 1024 * 1024
# the workloads timed beside the headline one (one GPU each); the tiny fp32
# case is a parity check, not a throughput workload
PER_CONFIG = ("qwen2.5-0.5b", "llama3-8b-qknorm", "partial-rope-64k", "bfd-packed")
KERNEL_SOURCES = ["qk_rmsnorm_rope_norm_b200/csrc/qknr_kernels.cuh",
                  "qk_rmsnorm_rope_norm_b200/csrc/qknr_pipe.cuh",
                  "qk_rmsnorm_rope_norm_b200/csrc/qknr_api.cu"]


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def env_rank():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback (6.65 TB/s, earlier measurement on this pool)"


def source_hash():
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, or None when the
    kernel sources changed since it was captured."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        e = d[kernel][workload]
        if e.get("source_sha256") != source_hash():
            return None
        return float(e["dram_bytes_per_launch"])
    except Exception:
        return None


# ----------------------------------------------------------------- clocks
REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
           0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
           0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
           0x100: "display_clock_setting"}


class ClockSampler:
    """NVML samples of the SM clock and clock-event reasons, every few ms,
    while the timed region runs."""

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.ok = False
        self.samples = []
        self.period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = self._handle(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report clocks as unknown
            log("clock sampler unavailable:", e)

    def _handle(self, idx):
        nv = self.nv
        try:
            p = torch.cuda.get_device_properties(idx)
            bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
            return nv.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
            phys = int(vis.split(",")[idx]) if vis and vis.split(",")[0].isdigit() else idx
            return nv.nvmlDeviceGetHandleByIndex(phys)

    def sample(self):
        nv = self.nv
        sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
        try:
            r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        self.samples.append((sm, r))

    def _run(self):
        while not self._stop.is_set():
            try:
                self.sample()
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._stop = threading.Event()
            self.sample()
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self._t.join()
            self.sample()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unknown: no NVML"]}
        busy = [s for s in self.samples if not (s[1] & 0x1)] or self.samples
        mask = 0
        for _, r in busy:
            mask |= r
        reasons = [n for b, n in REASONS.items() if mask & b]
        return {"sm_mhz": statistics.median(s[0] for s in busy), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples)}


# ------------------------------------------------------- multi-rank plumbing
def rank_seed(w, rank: int) -> int:
    """Each rank draws its own batch (weak scaling): seed 1000*index + 100*rank."""
    return workloads.seed_for(w) + 100 * rank


def max_over_ranks(values, world: int, device) -> list:
    """Element-wise max of per-rank timings (the job is as slow as its
    slowest rank); a no-op on one rank."""
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def aggregate_tokens_per_s(world: int, tokens_per_rank: int, ms_per_step: float) -> float:
    """Whole-job throughput: every rank processes its own batch each step."""
    return world * tokens_per_rank / (ms_per_step / 1e3)


# ---------------------------------------------------------------- our arm
class Set:
    """Device buffers of one batch: inputs, forward outputs, gradients. With
    layout "qkv", q and k are slices of a fused QKV projection buffer
    [B, S, (Hq + 2 Hkv) D] and dq, dk slices of a dQKV buffer (the V slots
    are never touched by the op)."""

    def __init__(self, inp: workloads.Inputs, dev, layout: str = "dense"):
        w = inp.w
        self.q, self.k = inp.q.to(dev), inp.k.to(dev)
        if layout == "qkv":
            import qk_rmsnorm_rope_norm_b200 as qknr
            width = (w.Hq + 2 * w.Hkv) * w.D
            self.qkv = torch.zeros((w.B, w.S, width), dtype=self.q.dtype, device=dev)
            q, k, _ = qknr.split_qkv(self.qkv, w.Hq, w.Hkv)
            q.copy_(self.q)
            k.copy_(self.k)
            self.q, self.k = q, k
        self.gq, self.gk = inp.gamma_q.to(dev), inp.gamma_k.to(dev)
        self.pos = None if inp.pos is None else inp.pos.to(dev)
        self.dqo, self.dko = inp.dq_out.to(dev), inp.dk_out.to(dev)
        self.qo = torch.empty(self.q.shape, dtype=self.q.dtype, device=dev)
        self.ko = torch.empty(self.k.shape, dtype=self.k.dtype, device=dev)
        self.rq = torch.empty((w.B, w.S, w.Hq), dtype=torch.float32, device=dev)
        self.rk = torch.empty((w.B, w.S, w.Hkv), dtype=torch.float32, device=dev)
        self.dq = torch.empty(self.q.shape, dtype=self.q.dtype, device=dev)
        self.dk = torch.empty(self.k.shape, dtype=self.k.dtype, device=dev)
        if layout == "qkv":
            self.dqkv = torch.zeros_like(self.qkv)
            self.dq, self.dk, _ = qknr.split_qkv(self.dqkv, w.Hq, w.Hkv)
        self.dgq = torch.empty(w.D, dtype=torch.float32, device=dev)
        self.dgk = torch.empty(w.D, dtype=torch.float32, device=dev)


def ring_sets(w, nsets: int) -> int:
    """Input sets in the ring: at least ``nsets``, and enough that ~2.5x the
    126 MB L2 of other traffic passes between two touches of a set even in a
    loop of one direction alone."""
    cb = workloads.contract_bytes(w)
    need = int(2.5 * L2_BYTES / max(1, min(cb["fwd"], cb["bwd"]))) + 2
    return max(nsets, min(need, 16))


def measure(w, inp, dev, steps: int, warmup: int, nsets: int, layout: str = "dense",
            world: int = 1, clocks=None):
    """Time ``steps`` fwd + bwd steps of workload ``w`` on a ring of input
    sets (after ``warmup`` untimed steps), with events only at the two ends
    of the timed region (the step time: the kernels run back to back, each
    one's prologue overlapping the previous one's tail). Then each direction
    alone: ``steps`` forward launches back to back, and ``steps`` backward
    launches, each loop timed by events at its ends (the per-kernel times).
    Returns the step total, the mean forward and mean backward launch
    milliseconds, the max over ranks when ``world`` > 1."""
    import qk_rmsnorm_rope_norm_b200 as qknr
    cfg = dict(rotary_dim=w.rotary_dim, theta=w.theta, eps=w.eps)
    sets = [Set(inp, dev, layout) for _ in range(nsets)]
    stream = torch.cuda.current_stream(dev)
    fwd = [qknr.prepare_fwd(s.q, s.k, s.gq, s.gk, s.pos, s.qo, s.ko, s.rq, s.rk, **cfg)
           for s in sets]
    bwd = [qknr.prepare_bwd(s.q, s.k, s.gq, s.gk, s.pos, s.rq, s.rk, s.dqo, s.dko, s.dq,
                            s.dk, s.dgq, s.dgk, **cfg) for s in sets]
    K, W = steps, warmup

    def step(i):
        fwd[i % nsets]()
        bwd[(i - LAG) % nsets]()

    def events():
        return torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    for i in range(W):
        step(i)
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    t0, t1 = events()
    with (clocks if clocks is not None else _Null()):
        t0.record(stream)
        for i in range(K):
            step(W + i)
        t1.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    total_ms = t0.elapsed_time(t1)
    per = []
    for calls in (fwd, bwd):
        for i in range(3):
            calls[i % nsets]()
        a, b = events()
        a.record(stream)
        for i in range(K):
            calls[(W + i) % nsets]()
        b.record(stream)
        torch.cuda.synchronize(dev)
        per.append(a.elapsed_time(b) / K)
    del fwd, bwd, sets
    return max_over_ranks([total_ms, per[0], per[1]], world, dev)


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *exc):
        return False


def run_ours(args, w, inp, rank, local_rank, world):
    import qk_rmsnorm_rope_norm_b200 as qknr
    dev = torch.device("cuda", local_rank)
    qknr.load_library()
    cfg = dict(rotary_dim=w.rotary_dim, theta=w.theta, eps=w.eps)
    clocks = ClockSampler(local_rank)  # NVML start-up stays outside the timed region
    nsets = ring_sets(w, args.sets) if args.sets == NSETS else args.sets
    total_ms, fwd_ms, bwd_ms = measure(w, inp, dev, args.steps, args.warmup, nsets,
                                       args.layout, world, clocks)
    torch.cuda.empty_cache()
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, w, inp, dev, cfg, world)
    cb = workloads.contract_bytes(w, with_pos=inp.pos is not None)
    floor = {"fwd_ms": copy_floor_ms(cb["fwd"], dev), "bwd_ms": copy_floor_ms(cb["bwd"], dev)}
    return dict(total_ms=total_ms, fwd_ms=fwd_ms, bwd_ms=bwd_ms, nsets=nsets,
                clocks=clocks.summary(), e2e=e2e, floor=floor)


def device_limits(dev):
    """SM count and opt-in shared memory per block of ``dev`` (for the plan)."""
    p = torch.cuda.get_device_properties(dev)
    return p.multi_processor_count, int(getattr(p, "shared_memory_per_block_optin", 0) or 0)


def kernels_of(w, dev, layout: str = "dense"):
    """The forward and backward kernels the library launches for ``w``."""
    import qk_rmsnorm_rope_norm_b200 as qknr
    sms, optin = device_limits(dev)
    strided = 3 if layout == "qkv" else 0
    return tuple(qknr.kernel_name(kind, w.B, w.S, w.Hq, w.Hkv, w.D, w.rotary_dim,
                                  w.torch_dtype, strided, sms, optin) for kind in ("fwd", "bwd"))


def per_config_line(w, inp, fwd_ms, bwd_ms, peak, dev, steps):
    cb = workloads.contract_bytes(w, with_pos=inp.pos is not None)
    kf, kb = kernels_of(w, dev)
    tok = inp.real_tokens

    def one(ms, nbytes, kern):
        gbs = nbytes / (ms / 1e3) / 1e9
        return {"ms": ms, "gbs": gbs, "frac": gbs / peak, "tokens_per_s": tok / (ms / 1e3),
                "bytes_per_launch": nbytes, "kernel": kern}

    return {"fwd": one(fwd_ms, cb["fwd"], kf), "bwd": one(bwd_ms, cb["bwd"], kb),
            "fwd_bwd_tokens_per_s": tok / ((fwd_ms + bwd_ms) / 1e3), "tokens": tok,
            "steps": steps}


def run_per_config(args, main_w, main_r, rank, dev, peak):
    """Every throughput workload on its own ring, timed like the main step;
    the headline workload's entry repeats the main measurement."""
    out = {}
    for name in PER_CONFIG:
        if name == main_w.name:
            w, inp = main_w, main_inp_cache[0]
            fwd_ms, bwd_ms, steps = main_r["fwd_ms"], main_r["bwd_ms"], args.steps
        else:
            base = workloads.WORKLOADS[name]
            inp = workloads.make_inputs(base, seed=rank_seed(base, rank))
            w = inp.w
            steps = args.per_config_steps
            total_ms, fwd_ms, bwd_ms = measure(w, inp, dev, steps, max(3, args.warmup),
                                               ring_sets(w, NSETS))
            torch.cuda.empty_cache()
        out[name] = per_config_line(w, inp, fwd_ms, bwd_ms, peak, dev, steps)
        out[name]["ms_per_step"] = (main_r["total_ms"] / args.steps if name == main_w.name
                                    else total_ms / steps)
    return out


main_inp_cache = [None]


def run_variants(args, w, inp, dev, peak):
    """The other entry points on the same workload, each timed like the main
    step's per-kernel loops (a ring of input sets, launches back to back,
    CUDA events at the loop ends, mean over the launches): the fused op on Q / K slices of a fused QKV buffer, the
    NoPE op (qk_norm_*), the mean-centred form (qk_layernorm_rope_*), the
    statistic alone (qk_rms_stats) and the rotation alone, forward and
    inverse (qk_rope_apply). Bytes are each call's contract bytes."""
    import qk_rmsnorm_rope_norm_b200 as qknr
    lib = qknr.load_library()
    cfg = dict(rotary_dim=w.rotary_dim, theta=w.theta, eps=w.eps)
    stream = torch.cuda.current_stream(dev)
    n_launch = max(50, min(args.steps, 400))
    e = w.elem_bytes
    rows = inp.q.numel() // w.D + inp.k.numel() // w.D
    T = w.B * w.S
    pos_b = 4 * T if inp.pos is not None else 0
    cb = workloads.contract_bytes(w, with_pos=inp.pos is not None)
    cb_nope = workloads.contract_bytes(w, with_pos=False)

    def timed(calls):
        for c in calls[:3]:
            c()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for i in range(n_launch):
            calls[i % len(calls)]()
        b.record(stream)
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b) / n_launch

    def line(ms, nbytes):
        gbs = nbytes / (ms / 1e3) / 1e9
        return {"ms": ms, "gbs": gbs, "frac": gbs / peak, "bytes_per_launch": nbytes}

    out = {}
    nsets = ring_sets(w, args.sets)
    qkv = [Set(inp, dev, "qkv") for _ in range(nsets)]
    f = [qknr.prepare_fwd(s.q, s.k, s.gq, s.gk, s.pos, s.qo, s.ko, s.rq, s.rk, **cfg) for s in qkv]
    b = [qknr.prepare_bwd(s.q, s.k, s.gq, s.gk, s.pos, s.rq, s.rk, s.dqo, s.dko, s.dq, s.dk,
                          s.dgq, s.dgk, **cfg) for s in qkv]
    out["fused_qkv_layout"] = {"fwd": line(timed(f), cb["fwd"]), "bwd": line(timed(b), cb["bwd"]),
                               "entry": "qk_norm_rope_fwd_strided / qk_norm_rope_bwd_strided"}
    del qkv, f, b
    dense = [Set(inp, dev) for _ in range(nsets)]
    P = qknr._ptr
    dt = 0 if w.dtype == "f32" else 1
    st = qknr._stream(None)

    def nope_fwd(s):
        a = (P(s.q), P(s.k), P(s.gq), P(s.gk), P(s.qo), P(s.ko), P(s.rq), P(s.rk), w.B, w.S,
             w.Hq, w.Hkv, w.D, float(w.eps), dt, st)
        return qknr.PreparedCall(lib.qk_norm_fwd, a, "qk_norm_fwd", s)

    def nope_bwd(s):
        a = (P(s.q), P(s.k), P(s.gq), P(s.gk), P(s.rq), P(s.rk), P(s.dqo), P(s.dko), P(s.dq),
             P(s.dk), P(s.dgq), P(s.dgk), w.B, w.S, w.Hq, w.Hkv, w.D, float(w.eps), dt, st)
        return qknr.PreparedCall(lib.qk_norm_bwd, a, "qk_norm_bwd", s)

    def rope(s, inverse):
        a = (P(s.q), P(s.k), P(s.pos), P(s.qo), P(s.ko), w.B, w.S, w.Hq, w.Hkv, w.D,
             w.rotary_dim, float(w.theta), 1 if inverse else 0, dt, st)
        return qknr.PreparedCall(lib.qk_rope_apply, a, "qk_rope_apply", s)

    out["nope_qk_norm"] = {"fwd": line(timed([nope_fwd(s) for s in dense]), cb_nope["fwd"]),
                           "bwd": line(timed([nope_bwd(s) for s in dense]), cb_nope["bwd"]),
                           "entry": "qk_norm_fwd / qk_norm_bwd"}
    ln = dict(cfg, norm="layer")
    f = [qknr.prepare_fwd(s.q, s.k, s.gq, s.gk, s.pos, s.qo, s.ko, s.rq, s.rk, **ln) for s in dense]
    b = [qknr.prepare_bwd(s.q, s.k, s.gq, s.gk, s.pos, s.rq, s.rk, s.dqo, s.dko, s.dq, s.dk,
                          s.dgq, s.dgk, **ln) for s in dense]
    out["qk_layernorm_rope"] = {"fwd": line(timed(f), cb["fwd"]), "bwd": line(timed(b), cb["bwd"]),
                                "entry": "qk_layernorm_rope_fwd / qk_layernorm_rope_bwd"}
    rope_bytes = 2 * rows * w.D * e + pos_b
    def stats(s):
        a = (P(s.q), P(s.k), P(s.rq), P(s.rk), w.B, w.S, w.Hq, w.Hkv, w.D, float(w.eps), dt, st)
        return qknr.PreparedCall(lib.qk_rms_stats, a, "qk_rms_stats", s)

    out["rms_stats"] = {"fwd": line(timed([stats(s) for s in dense]),
                                    rows * w.D * e + 4 * rows),
                        "entry": "qk_rms_stats"}
    out["rope_only"] = {"fwd": line(timed([rope(s, False) for s in dense]), rope_bytes),
                        "inverse": line(timed([rope(s, True) for s in dense]), rope_bytes),
                        "entry": "qk_rope_apply"}
    out.update(layerwise_variants(w, dense, dev, timed, line))
    return out


def layerwise_variants(w, dense, dev, timed, line):
    """Layerwise (all-heads) QK-norm on the same rows, gamma over the full
    hidden vector and one statistic per token and tensor. "one_pass": one
    rank holds every head, one launch each way. "tp_phases": the sequence a
    tensor-parallel rank runs (stats, then normalise; dots, then backward),
    here with every head on one GPU and no exchange between the phases, so it
    times the extra pass over the rows that sharding costs. "tp_rank": the
    same sequence on one rank's head slice (TP 8, 4 or 2), the shape a real
    sharded rank runs. "tp_chunked": the binding's chunked exchange schedule.
    Bytes are the op's contract bytes (each row read once and written once,
    dy read once, rstd [T] per tensor)."""
    import qk_rmsnorm_rope_norm_b200 as qknr
    lib = qknr.load_library()
    P = qknr._ptr
    dt = 0 if w.dtype == "f32" else 1
    st = qknr._stream(None)
    T = w.B * w.S
    e = w.elem_bytes
    H = w.Hq + w.Hkv
    pos_b = 4 * T if dense[0].pos is not None else 0
    gbytes = H * w.D * e
    fwd_b = 2 * T * H * w.D * e + 4 * T * (int(w.Hq > 0) + int(w.Hkv > 0)) + pos_b + gbytes
    bwd_b = 3 * T * H * w.D * e + 4 * T * (int(w.Hq > 0) + int(w.Hkv > 0)) + pos_b + gbytes
    gq, gk = workloads.layerwise_gamma(w, 17)
    gq, gk = gq.to(dev), gk.to(dev)
    bufs = []
    for s in dense:
        bufs.append(dict(rq=torch.empty(T, device=dev), rk=torch.empty(T, device=dev),
                         sq=torch.empty(T, device=dev), sk=torch.empty(T, device=dev),
                         dgq=torch.empty(w.Hq * w.D, device=dev),
                         dgk=torch.empty(w.Hkv * w.D, device=dev)))

    def fwd(s, b, sums):
        sq, sk = (P(b["sq"]), P(b["sk"])) if sums else (None, None)
        return (P(s.q), P(s.k), P(gq), P(gk), P(s.pos), sq, sk, P(s.qo), P(s.ko), P(b["rq"]),
                P(b["rk"]), w.B, w.S, w.Hq, w.Hkv, w.Hq, w.Hkv, w.D, w.rotary_dim,
                float(w.theta), float(w.eps), dt, st)

    def bwd(s, b, sums):
        sq, sk = (P(b["sq"]), P(b["sk"])) if sums else (None, None)
        return (P(s.q), P(s.k), P(gq), P(gk), P(s.pos), P(b["rq"]), P(b["rk"]), P(s.dqo),
                P(s.dko), sq, sk, P(s.dq), P(s.dk), P(b["dgq"]), P(b["dgk"]), w.B, w.S, w.Hq,
                w.Hkv, w.Hq, w.Hkv, w.D, w.rotary_dim, float(w.theta), dt, st)

    def stats(s, b):
        return (P(s.q), P(s.k), P(b["sq"]), P(b["sk"]), w.B, w.S, w.Hq, w.Hkv, w.D, dt, st)

    def dots(s, b):
        return (P(s.q), P(s.k), P(gq), P(gk), P(s.pos), P(b["rq"]), P(b["rk"]), P(s.dqo),
                P(s.dko), P(b["sq"]), P(b["sk"]), w.B, w.S, w.Hq, w.Hkv, w.D, w.rotary_dim,
                float(w.theta), dt, st)

    C = qknr.PreparedCall

    def seq(*calls):
        def run():
            for c in calls:
                c()
        return run

    one_f = [C(lib.qk_layerwise_norm_rope_fwd, fwd(s, b, False), "lw fwd", s)
             for s, b in zip(dense, bufs)]
    one_b = [C(lib.qk_layerwise_norm_rope_bwd, bwd(s, b, False), "lw bwd", s)
             for s, b in zip(dense, bufs)]
    two_f = [seq(C(lib.qk_layerwise_stats, stats(s, b), "lw stats", s),
                 C(lib.qk_layerwise_norm_rope_fwd, fwd(s, b, True), "lw fwd", s))
             for s, b in zip(dense, bufs)]
    two_b = [seq(C(lib.qk_layerwise_bwd_dots, dots(s, b), "lw dots", s),
                 C(lib.qk_layerwise_norm_rope_bwd, bwd(s, b, True), "lw bwd", s))
             for s, b in zip(dense, bufs)]
    def no_exchange(buf, span):  # one GPU: the sums are already the totals
        return None

    def graphed(fn):
        # the chunked schedule's host work (a few calls and events per chunk)
        # would dominate short calls; a training step captures it in a CUDA
        # graph, and so does this measurement: one capture, timed replays
        fn()
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        torch.cuda.synchronize(dev)
        keep.append(g)
        return g.replay

    keep = []

    def chunked_f(s):
        return graphed(lambda: qknr.layerwise_chunked_fwd(
            s.q, s.k, gq, gk, s.pos, rotary_dim=w.rotary_dim, theta=w.theta, eps=w.eps,
            Hq_total=w.Hq, Hkv_total=w.Hkv, exchange=no_exchange,
            chunks=qknr.DEFAULT_EXCHANGE_CHUNKS))

    def chunked_b(s, b):
        return graphed(lambda: qknr.layerwise_chunked_bwd(
            s.q, s.k, gq, gk, s.pos, b["rq"], b["rk"], s.dqo, s.dko, rotary_dim=w.rotary_dim,
            theta=w.theta, Hq_total=w.Hq, Hkv_total=w.Hkv, exchange=no_exchange,
            chunks=qknr.DEFAULT_EXCHANGE_CHUNKS))

    # one rank of a tensor-parallel group on its own head slice: the two
    # phases it runs (stats, then normalise; dots, then backward), with the
    # exchange between them a no-op on one GPU. TP = the largest of 8, 4, 2
    # that divides both head counts.
    tp = next((t for t in (8, 4, 2) if w.Hq % t == 0 and w.Hkv % t == 0), 1)
    hq, hk = w.Hq // tp, w.Hkv // tp
    gq_r, gk_r = gq[: hq * w.D], gk[: hk * w.D]
    ranks = []
    for s in dense:
        r = dict(q=s.q[:, :, :hq].contiguous(), k=s.k[:, :, :hk].contiguous(),
                 dqo=s.dqo[:, :, :hq].contiguous(), dko=s.dko[:, :, :hk].contiguous(),
                 pos=s.pos, rq=torch.empty(T, device=dev), rk=torch.empty(T, device=dev),
                 dgq=torch.empty(hq * w.D, device=dev), dgk=torch.empty(hk * w.D, device=dev))
        r.update(qo=torch.empty_like(r["q"]), ko=torch.empty_like(r["k"]),
                 dq=torch.empty_like(r["q"]), dk=torch.empty_like(r["k"]))
        # one checked pass through the Python API validates every buffer
        r["sq"], r["sk"] = qknr.qk_layerwise_stats(r["q"], r["k"])
        qknr.qk_layerwise_norm_rope_fwd(r["q"], r["k"], gq_r, gk_r, r["pos"], r["sq"], r["sk"],
                                        rotary_dim=w.rotary_dim, theta=w.theta, eps=w.eps,
                                        Hq_total=w.Hq, Hkv_total=w.Hkv, q_out=r["qo"],
                                        k_out=r["ko"], rstd_q=r["rq"], rstd_k=r["rk"])
        qknr.qk_layerwise_norm_rope_bwd(r["q"], r["k"], gq_r, gk_r, r["pos"], r["rq"], r["rk"],
                                        r["dqo"], r["dko"], r["sq"], r["sk"],
                                        rotary_dim=w.rotary_dim, theta=w.theta, Hq_total=w.Hq,
                                        Hkv_total=w.Hkv, dq=r["dq"], dk=r["dk"],
                                        dgamma_q=r["dgq"], dgamma_k=r["dgk"])
        ranks.append(r)
    torch.cuda.synchronize(dev)
    rank_f = [seq(C(lib.qk_layerwise_stats,
                    (P(r["q"]), P(r["k"]), P(r["sq"]), P(r["sk"]), w.B, w.S, hq, hk, w.D, dt, st),
                    "lw stats", r),
                  C(lib.qk_layerwise_norm_rope_fwd,
                    (P(r["q"]), P(r["k"]), P(gq_r), P(gk_r), P(r["pos"]), P(r["sq"]), P(r["sk"]),
                     P(r["qo"]), P(r["ko"]), P(r["rq"]), P(r["rk"]), w.B, w.S, hq, hk, w.Hq,
                     w.Hkv, w.D, w.rotary_dim, float(w.theta), float(w.eps), dt, st),
                    "lw fwd", r))
              for r in ranks]
    rank_b = [seq(C(lib.qk_layerwise_bwd_dots,
                    (P(r["q"]), P(r["k"]), P(gq_r), P(gk_r), P(r["pos"]), P(r["rq"]), P(r["rk"]),
                     P(r["dqo"]), P(r["dko"]), P(r["sq"]), P(r["sk"]), w.B, w.S, hq, hk, w.D,
                     w.rotary_dim, float(w.theta), dt, st),
                    "lw dots", r),
                  C(lib.qk_layerwise_norm_rope_bwd,
                    (P(r["q"]), P(r["k"]), P(gq_r), P(gk_r), P(r["pos"]), P(r["rq"]), P(r["rk"]),
                     P(r["dqo"]), P(r["dko"]), P(r["sq"]), P(r["sk"]), P(r["dq"]), P(r["dk"]),
                     P(r["dgq"]), P(r["dgk"]), w.B, w.S, hq, hk, w.Hq, w.Hkv, w.D,
                     w.rotary_dim, float(w.theta), dt, st),
                    "lw bwd", r))
              for r in ranks]
    Hr = hq + hk
    fwd_r = 2 * T * Hr * w.D * e + 4 * T * 2 + pos_b + Hr * w.D * e
    bwd_r = 3 * T * Hr * w.D * e + 4 * T * 2 + pos_b + Hr * w.D * e
    rank_line = {"fwd": line(timed(rank_f), fwd_r), "bwd": line(timed(rank_b), bwd_r),
                 "tp": tp, "heads": f"{hq} + {hk}",
                 "entry": f"one rank of a TP={tp} group on its {hq} + {hk} head slice: "
                          "qk_layerwise_stats + _fwd; qk_layerwise_bwd_dots + _bwd (the "
                          "exchange between them a no-op); bytes are the slice's one-pass bytes"}
    del ranks

    return {
        "layerwise_tp_rank": rank_line,
        "layerwise_one_pass": {"fwd": line(timed(one_f), fwd_b), "bwd": line(timed(one_b), bwd_b),
                               "entry": "qk_layerwise_norm_rope_fwd / _bwd, sums NULL"},
        "layerwise_tp_phases": {"fwd": line(timed(two_f), fwd_b),
                                "bwd": line(timed(two_b), bwd_b),
                                "entry": "qk_layerwise_stats + _fwd; qk_layerwise_bwd_dots + _bwd"},
        "layerwise_tp_chunked": {
            "fwd": line(timed([chunked_f(s) for s in dense]), fwd_b),
            "bwd": line(timed([chunked_b(s, b) for s, b in zip(dense, bufs)]), bwd_b),
            "entry": f"layerwise_chunked_fwd / _bwd, up to {qknr.DEFAULT_EXCHANGE_CHUNKS} token "
                     f"chunks of >= {qknr.MIN_CHUNK_TOKENS} tokens and >= "
                     f"{qknr.MIN_CHUNK_BYTES >> 20} MiB of rows, side-stream exchange (here a "
                     "no-op: one GPU holds every head), captured in a CUDA graph and replayed"},
    }


def copy_floor_ms(traffic_bytes: int, dev, n: int = 20) -> float:
    """Median time of a device-to-device copy moving the same DRAM bytes
    (traffic/2 read + traffic/2 written), each launch after an L2 flush:
    the practical floor for a single launch of that size on this GPU."""
    half = max(16, traffic_bytes // 2) // 2 * 2
    src = torch.empty(half // 2, dtype=torch.bfloat16, device=dev)
    dst = torch.empty_like(src)
    flush = torch.empty(256 * 1024 * 1024 // 4, device=dev)
    ts = []
    for i in range(n + 3):
        flush.fill_(float(i))
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        dst.copy_(src)
        b.record()
        torch.cuda.synchronize(dev)
        if i >= 3:
            ts.append(a.elapsed_time(b))
    del src, dst, flush
    return statistics.median(ts)


def run_e2e(args, w, inp, dev, cfg, world):
    """Public API from pinned host buffers: every step copies its inputs
    host -> device, runs the forward and the backward, and copies all their
    results device -> host. Two slots of device buffers and three streams
    pipeline the steps the way a training loop's loader does: step i + 1's
    inputs cross PCIe host -> device while step i's results cross it device
    -> host (the link is full duplex), and a step's kernels run in between.
    Every step still moves all of its bytes both ways."""
    import qk_rmsnorm_rope_norm_b200 as qknr
    host_in = {n: getattr(inp, n).pin_memory() for n in ("q", "k", "dq_out", "dk_out")}
    gq, gk = inp.gamma_q.to(dev), inp.gamma_k.to(dev)
    pos = None if inp.pos is None else inp.pos.to(dev)
    out_shapes = {"q_out": (inp.q.shape, inp.q.dtype), "k_out": (inp.k.shape, inp.k.dtype),
                  "rstd_q": ((w.B, w.S, w.Hq), torch.float32),
                  "rstd_k": ((w.B, w.S, w.Hkv), torch.float32),
                  "dq": (inp.q.shape, inp.q.dtype), "dk": (inp.k.shape, inp.k.dtype),
                  "dgamma_q": ((w.D,), torch.float32), "dgamma_k": ((w.D,), torch.float32)}
    host_out = {n: torch.empty(s, dtype=dt).pin_memory() for n, (s, dt) in out_shapes.items()}
    slots = []
    for _ in range(2):
        d = {n: torch.empty_like(t, device=dev) for n, t in host_in.items()}
        d.update({n: torch.empty(s, dtype=dt, device=dev) for n, (s, dt) in out_shapes.items()})
        slots.append(d)
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out.values())
    s_in, s_run, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    ev = {(k, i): torch.cuda.Event() for k in ("in", "run", "out") for i in range(2)}
    used = [False, False]

    def step(i):
        sl = i % 2
        d = slots[sl]
        with torch.cuda.stream(s_in):
            if used[sl]:
                s_in.wait_event(ev["run", sl])  # the slot's inputs are read
            for n, t in host_in.items():
                d[n].copy_(t, non_blocking=True)
            ev["in", sl].record(s_in)
        s_run.wait_event(ev["in", sl])
        if used[sl]:
            s_run.wait_event(ev["out", sl])  # the slot's results are out
        qknr.qk_norm_rope_fwd(d["q"], d["k"], gq, gk, pos, q_out=d["q_out"], k_out=d["k_out"],
                              rstd_q=d["rstd_q"], rstd_k=d["rstd_k"], stream=s_run, **cfg)
        qknr.qk_norm_rope_bwd(d["q"], d["k"], gq, gk, pos, d["rstd_q"], d["rstd_k"],
                              d["dq_out"], d["dk_out"], dq=d["dq"], dk=d["dk"],
                              dgamma_q=d["dgamma_q"], dgamma_k=d["dgamma_k"], stream=s_run,
                              **cfg)
        ev["run", sl].record(s_run)
        s_out.wait_event(ev["run", sl])
        with torch.cuda.stream(s_out):
            for n, t in host_out.items():
                t.copy_(d[n], non_blocking=True)
            ev["out", sl].record(s_out)
        used[sl] = True

    E = max(1, min(args.steps, args.e2e_steps))
    for i in range(3):
        step(i)
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s_in)
    for i in range(E):
        step(3 + i)
    b.record(s_out)  # after the last step's results reached the host
    torch.cuda.synchronize(dev)
    ms = max_over_ranks([a.elapsed_time(b) / E], world, dev)[0]
    return dict(ms=ms, steps=E, h2d=h2d, d2h=d2h)


# ------------------------------------------------------- the CPU oracle
def host_cores() -> int:
    """Cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return platform.processor() or "unknown"


def oracle_rate(inp, budget_s: float, threads: int, tokens_per_call: int = 256,
                rounds=None):
    """Time the CPU oracle (fwd + bwd, unmodified) on consecutive token chunks
    of the workload with ``threads`` host threads, each taking the next chunk
    until ``budget_s`` seconds of wall time have passed (or, with ``rounds``,
    exactly ``rounds`` chunks per thread). The oracle is C called through
    ctypes, which releases the GIL, so the threads run on separate cores.
    Returns (tokens, wall seconds, per-round wall times)."""
    import oracle
    w = inp.w
    T = w.B * w.S
    m_all = oracle.positions(None if inp.pos is None else inp.pos.numpy(), w.B, w.S)
    q = inp.q.reshape(T, w.Hq, w.D)
    k = inp.k.reshape(T, w.Hkv, w.D)
    dqo = inp.dq_out.reshape(T, w.Hq, w.D)
    dko = inp.dk_out.reshape(T, w.Hkv, w.D)
    orc = oracle.get()
    lock = threading.Lock()
    nxt = [0]

    def chunk():
        with lock:
            t0 = nxt[0]
            t1 = min(T, t0 + tokens_per_call)
            nxt[0] = t1 % T
        m = m_all[t0:t1]
        orc.fwd(q[t0:t1], k[t0:t1], inp.gamma_q, inp.gamma_k, m, w.rotary_dim, w.theta, w.eps)
        orc.bwd(q[t0:t1], k[t0:t1], inp.gamma_q, inp.gamma_k, m, dqo[t0:t1], dko[t0:t1],
                w.rotary_dim, w.theta, w.eps)
        return t1 - t0

    def worker(deadline, n):
        done, calls = 0, 0
        while (n is None and time.perf_counter() < deadline) or (n is not None and calls < n):
            done += chunk()
            calls += 1
        return done

    per_round = []
    with ThreadPoolExecutor(threads) as ex:
        if rounds is None:
            c = time.perf_counter()
            done = sum(ex.map(worker, [c + budget_s] * threads, [None] * threads))
            wall = time.perf_counter() - c
        else:
            done, wall = 0, 0.0
            for _ in range(rounds):
                c = time.perf_counter()
                done += sum(ex.map(worker, [0.0] * threads, [1] * threads))
                dt = time.perf_counter() - c
                per_round.append(dt)
                wall += dt
    return done, wall, per_round


def cpu_baseline(inp, budget_s: float) -> dict:
    """The oracle on all host cores (the reported value) and on one core."""
    cores = host_cores()
    d1, s1, _ = oracle_rate(inp, budget_s / 2, 1)
    dn, sn, _ = oracle_rate(inp, budget_s / 2, cores)
    return {"value": dn / sn, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "nproc": os.cpu_count(), "cpu_model": cpu_model(),
            "one_core": {"value": d1 / s1, "cores": 1, "tokens": d1, "seconds": s1},
            "sample": f"consecutive 256-token chunks of the workload, fwd + bwd, unmodified "
                      f"fp64 C oracle; {cores} threads (one per core): {dn} tokens in "
                      f"{sn:.1f} s; one thread: {d1} tokens in {s1:.1f} s"}


cfg_args = None


def config_of(w, inp, world):
    return {"workload": w.name, "B": w.B, "S": w.S, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D,
            "rotary_dim": w.rotary_dim, "theta": w.theta, "eps": w.eps, "io_dtype": w.dtype,
            "tokens_per_step": inp.real_tokens,
            "l2": f"ring of {ring_sets(w, NSETS)} input sets, bwd lags fwd by {LAG} steps: "
                  f"inputs not L2-resident (>= 2.5x 126 MB of traffic between touches)"
                  if getattr(cfg_args, "sets", NSETS) == NSETS else
                  f"{cfg_args.sets} input set(s): profiling run, inputs may be L2-resident",
            "layout": getattr(cfg_args, "layout", "dense"),
            "parallelism": f"dp{world} (weak, no data-path collective)"}


def run_reference(args, w, inp, rank, world):
    """The reference arm: the CPU oracle as it stands, on every host core,
    rank 0 only. A step is one round in which every core runs the oracle
    (fwd + bwd) on the next 256-token chunk of the workload."""
    if rank != 0:
        return
    cores = host_cores()
    oracle_rate(inp, 0.0, cores, rounds=args.warmup)
    done, spent, per_round = oracle_rate(inp, 0.0, cores, rounds=args.steps)
    v = done / spent
    ms = 1000.0 * spent / args.steps
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_of(w, inp, 1),
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "nproc": os.cpu_count(), "cpu_model": cpu_model(),
                         "sample": f"each step: {cores} threads (one per core) each run the "
                                   f"unmodified fp64 C oracle, fwd + bwd, on the next 256 "
                                   f"consecutive tokens of the workload"},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=workloads.BENCH_WORKLOAD,
                    choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--seq-len", type=int, default=0,
                    help="override S of the workload (smaller profiling captures; the "
                         "line's config records it)")
    ap.add_argument("--sets", type=int, default=NSETS,
                    help="input sets in the ring (4 keeps inputs out of L2; 1 for small "
                         "profiling footprints)")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cpu-budget-s", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--per-config-steps", type=int, default=200,
                    help="timed steps of each other workload in per_config")
    ap.add_argument("--no-per-config", action="store_true")
    ap.add_argument("--variants", action="store_true",
                    help="also time the fused-QKV, NoPE and rotation-only entry points")
    ap.add_argument("--layout", choices=["dense", "qkv"], default="dense",
                    help="dense [B,S,H,D] q/k, or q/k read from (and dq/dk written into) "
                         "fused QKV buffers")
    args = ap.parse_args()
    global cfg_args
    cfg_args = args
    if args.sets < 1:
        ap.error("--sets must be >= 1")
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank, local_rank, world = env_rank()
    w = workloads.WORKLOADS[args.workload]
    over = {"S": args.seq_len} if args.seq_len > 0 and not w.packed else {}
    inp = workloads.make_inputs(w, seed=rank_seed(w, rank), **over)
    w = inp.w
    main_inp_cache[0] = inp

    if args.impl == "reference":
        run_reference(args, w, inp, rank, world)
        return

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
    r = run_ours(args, w, inp, rank, local_rank, world)
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank != 0:
        return

    peak, peak_src = hbm_peak()
    per_config = None
    if world == 1 and not args.no_per_config:
        per_config = run_per_config(args, w, r, rank, dev, peak)
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(inp, args.cpu_budget_s)

    cb = workloads.contract_bytes(w, with_pos=inp.pos is not None)
    tokens = inp.real_tokens
    ms = r["total_ms"] / args.steps
    value = aggregate_tokens_per_s(world, tokens, ms)
    fwd_gbs = cb["fwd"] / (r["fwd_ms"] / 1e3) / 1e9
    bwd_gbs = cb["bwd"] / (r["bwd_ms"] / 1e3) / 1e9
    step_gbs = (cb["fwd"] + cb["bwd"]) / (ms / 1e3) / 1e9
    fwd_kernel, bwd_kernel = kernels_of(w, dev, args.layout)
    # the dominant kernel: the one with the larger share of the step
    dom = "bwd" if r["bwd_ms"] >= r["fwd_ms"] else "fwd"
    dom_kernel = bwd_kernel if dom == "bwd" else fwd_kernel
    dom_gbs = bwd_gbs if dom == "bwd" else fwd_gbs
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "io_dtype": w.dtype, "data": "synthetic", "config": config_of(w, inp, world),
        "hbm": {"fwd_gbs": fwd_gbs, "bwd_gbs": bwd_gbs, "step_gbs": step_gbs,
                "fwd_frac": fwd_gbs / peak, "bwd_frac": bwd_gbs / peak,
                "step_frac": step_gbs / peak, "peak_gbs": peak, "peak_source": peak_src,
                "copy_floor": {
                    "what": "torch copy_ moving the same DRAM bytes, one launch after an "
                            "L2 flush (the practical floor at this size)",
                    "fwd_gbs": cb["fwd"] / (r["floor"]["fwd_ms"] / 1e3) / 1e9,
                    "bwd_gbs": cb["bwd"] / (r["floor"]["bwd_ms"] / 1e3) / 1e9,
                    "fwd_frac_of_copy": r["floor"]["fwd_ms"] / r["fwd_ms"],
                    "bwd_frac_of_copy": r["floor"]["bwd_ms"] / r["bwd_ms"]}},
        "per_kernel_timing": f"fwd.ms and bwd.ms: {args.steps} launches of each direction "
                             f"alone, back to back on the same ring, events at the loop ends",
        "fwd": {"ms": r["fwd_ms"], "tokens_per_s": aggregate_tokens_per_s(world, tokens, r["fwd_ms"]),
                "bytes_per_launch": cb["fwd"], "kernel": fwd_kernel},
        "bwd": {"ms": r["bwd_ms"], "tokens_per_s": aggregate_tokens_per_s(world, tokens, r["bwd_ms"]),
                "bytes_per_launch": cb["bwd"], "kernel": bwd_kernel},
        "roofline": {"bound": "hbm", "kernel": dom_kernel, "direction": dom, "achieved": dom_gbs,
                     "peak": peak, "unit": "GB/s", "frac": dom_gbs / peak,
                     "traffic": ncu_traffic(dom_kernel, w.name),
                     "algorithmic_bytes": cb[dom], "peak_source": peak_src},
        "clocks": r["clocks"],
        # per step: the forward, the kernel that clears dgamma, the backward
        "gpu_launches": 3 * args.steps,
    }
    if r["e2e"] is not None:
        e = r["e2e"]
        line["e2e"] = {"value": aggregate_tokens_per_s(world, tokens, e["ms"]), "unit": "tokens/s",
                       "h2d_bytes_per_step": e["h2d"], "d2h_bytes_per_step": e["d2h"],
                       "ms_per_step": e["ms"], "steps": e["steps"],
                       "schedule": "public API calls on pinned host buffers; two device "
                                   "buffer slots and three streams, so step i+1's "
                                   "host-to-device copies overlap step i's device-to-host "
                                   "copies"}
    line["cpu_baseline"] = cpu
    if per_config is not None:
        line["per_config"] = per_config
    if args.variants and world == 1:
        line["variants"] = run_variants(args, w, inp, dev, peak)
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
