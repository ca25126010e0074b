#!/usr/bin/env python
"""HLA prefill and decode benchmark on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one pass of the hot path over synthetic inputs already resident in HBM:
  * prefill of the dense 0.8B-like layer (B=1, H=16, T=16384, C=64, d=128, bf16,
    bias -2 with spread route inputs, no skipping): pools, gates, chunk
    transitions, gated composition, read-out;
  * one decode step of 64 sequences with 32768-token contexts (512 cached A_j/B_j
    per head, H=16, d=128, bf16, bias -2, threshold 0.05: every chunk active).
The L2 cache is flushed before each timed phase (a 256 MiB write, then a 256 MiB read so
that the write's dirty lines go back to HBM outside the timed region; untimed).  Each
phase is timed with CUDA events on the launching stream; per-stage times come from
the library's own event pairs (hla_profile_*), on the same stream.

``value`` is prefill tokens/s (whole job: every rank runs an independent replica,
weak scaling, max time over ranks); the decode numbers are in ``decode``.  The
``reference`` arm times the CPU oracle on a bounded sample of the same workloads.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "HLA prefill tokens/s (% bf16 tensor peak); decode tokens/s at 32K (% HBM BW)"
L2_FLUSH_BYTES = 256 << 20
# algorithmic flops per chunk at C=64, d=128 (see the kernel headers):
#   transition: K K^T 2C^2d + Wb, Ub 2*2C^2d + A, B 2*2Cd^2  (triangular solve ignored)
#   read-out:   Q S^T, Wb S^T 2*2Cd^2 + Q K^T 2C^2d + P X 2C^2d
FLOP_TRANSITION = 3 * 2 * 64 * 64 * 128 + 2 * 2 * 64 * 128 * 128
FLOP_READOUT = 2 * 2 * 64 * 128 * 128 + 2 * 2 * 64 * 64 * 128


PREFILL_WORKLOADS = {
    "dense": lambda syn: syn.PREFILL_0P8B,
    "sparse": lambda syn: syn.SPARSE_LONG,
    "gdn": lambda syn: syn.GDN_REDUCTION,
}


def rank_env():
    """(world, rank, local_rank) from the torchrun environment (1, 0, 0 alone)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(values, device="cpu"):
    """Element-wise maximum of per-rank timings (one all_reduce(MAX) when a process
    group of more than one rank is up; the values themselves otherwise)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def whole_job_rate(units_per_rank, ms_max, world):
    """Weak-scaling throughput: every rank runs an independent replica of the same
    work, so the job processes world x units in the slowest rank's time."""
    return units_per_rank * world / (ms_max * 1e-3)


# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) from one ncu
# capture of each kernel, keyed by the kernel and tagged with the SHA-256 prefix of
# the kernel's source files at capture time.  A figure is reported only while those
# sources are unchanged.
#   compose: one full-size launch on the dense 0.8B-like prefill
#   decode_main: a 4-sequence decode (64 of the 1024 (sequence, head) streams of the
#     32K-context step), scaled by 16; per stream it equals the algorithmic bytes
NCU_TRAFFIC = {
    "compose": (2.0470e9, {"compose_tc.cu": "4b50659baac7102a", "tc_common.cuh": "c10beda371c1dd4b"}),
    # gate + stream kernels of one step, captured on 4 (dense) and 8 (planted) of the
    # 64 sequences and scaled by the sequence count (the traffic is per sequence)
    "decode_main": (3.4638e10, {"decode_stream.cu": "8916b84931f22b4f", "tc_common.cuh": "c10beda371c1dd4b"}),
    "decode_planted": (5.447e8, {"decode_stream.cu": "8916b84931f22b4f", "tc_common.cuh": "c10beda371c1dd4b"}),
}

# Datasheet figures of one B200, reported beside the measured denominators: dense
# bf16 tensor throughput 2.25 PFLOP/s (without 2:4 sparsity) and HBM3e bandwidth of
# about 8 TB/s (7.7 TB/s in the HGX configuration).
DATASHEET_BF16_TFLOPS = 2250.0
DATASHEET_HBM_GBS = 8000.0


def ncu_traffic(kernel):
    """The recorded traffic of `kernel` (bytes per launch), or None if there is no
    capture or its sources have changed since."""
    import hashlib
    rec = NCU_TRAFFIC.get(kernel)
    if rec is None:
        return None
    nbytes, files = rec
    for name, tag in files.items():
        path = os.path.join(ROOT, "gated_delta_rule_transitions_b200", "csrc", name)
        try:
            with open(path, "rb") as f:
                if hashlib.sha256(f.read()).hexdigest()[:16] != tag:
                    return None
        except OSError:
            return None
    return nbytes


def _peaks():
    """(HBM GB/s, bf16 burst TFLOP/s, bf16 sustained TFLOP/s, source).  The measured
    copy bandwidth and cuBLAS bf16 throughput of this GPU pool when the measurement
    file is present; otherwise an earlier measurement on the same pool, labelled
    "fallback" in the output line and announced on stderr."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), "measured"
    except Exception as e:
        print(f"bench.py: no measured peaks ({type(e).__name__}); using the fallback figures 6650 GB/s and "
              f"1590 / 1400 TFLOP/s, labelled 'fallback'", file=sys.stderr)
        return 6650.0, 1590.0, 1400.0, "fallback"


class ClockSampler:
    """SM clocks, power and throttle reasons sampled during the timed region.

    Reads NVML every 5 ms from a thread (read-only queries; no setting is changed),
    on the NVML device whose PCI bus id matches the CUDA device; falls back to
    polling nvidia-smi when NVML is unavailable."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4))

    def __init__(self, cuda_index: int):
        self.cuda_index = cuda_index
        self.samples = []  # (sm_mhz, max_mhz, power_w, reason_bits)
        self.source = None
        self._stop = threading.Event()
        self._t = None

    def _nvml_handle(self):
        """NVML handle of the CUDA device: matched by UUID, else by PCI bus id."""
        import pynvml
        import torch
        pynvml.nvmlInit()
        p = torch.cuda.get_device_properties(self.cuda_index)
        uuid = str(getattr(p, "uuid", "")).lower().removeprefix("gpu-")
        bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
        for i in range(pynvml.nvmlDeviceGetCount()):
            h = pynvml.nvmlDeviceGetHandleByIndex(i)
            u = pynvml.nvmlDeviceGetUUID(h)
            u = (u.decode() if isinstance(u, bytes) else u).lower().removeprefix("gpu-")
            b = pynvml.nvmlDeviceGetPciInfo(h).busId
            b = (b.decode() if isinstance(b, bytes) else b).lower()
            if (uuid and u == uuid) or b.endswith(bus[-12:]):
                return pynvml, h
        raise RuntimeError(f"no NVML device matches uuid {uuid} / bus {bus}")

    def _run_nvml(self, nv, h):
        mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        while not self._stop.is_set():
            self._sample_nvml(nv, h, mx)
            self._stop.wait(0.005)

    def _run_smi(self):
        fields = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
                  "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                  "clocks_event_reasons.sw_power_cap")
        while not self._stop.is_set():
            try:
                out = subprocess.run(["nvidia-smi", "-i", str(self.cuda_index), f"--query-gpu={fields}",
                                      "--format=csv,noheader,nounits"], capture_output=True, text=True,
                                     timeout=5).stdout.strip().split(",")
                bits = 0
                for (_, bit), flag in zip(self.REASONS, out[3:7]):
                    bits |= bit if flag.strip() == "Active" else 0
                self.samples.append((float(out[0]), float(out[1]), float(out[2]), bits))
            except Exception:
                pass
            self._stop.wait(0.2)

    def _sample_nvml(self, nv, h, mx):
        try:
            sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
            pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
            rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
            self.samples.append((float(sm), float(mx), pw, int(rs)))
        except Exception:
            pass

    def __enter__(self):
        try:
            nv, h = self._nvml_handle()
            self.source = "nvml"
            self._nv = (nv, h, nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            self._t = threading.Thread(target=self._run_nvml, args=(nv, h), daemon=True)
        except Exception as e:
            self.source = f"nvidia-smi (nvml: {type(e).__name__}: {str(e)[:80]})"
            self._t = threading.Thread(target=self._run_smi, daemon=True)
        self._t.start()
        return self

    def __exit__(self, *a):
        if getattr(self, "_nv", None) is not None:
            self._sample_nvml(*self._nv)   # at least one sample inside the region
        self._stop.set()
        self._t.join(timeout=10)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0,
                    "source": self.source}
        reasons = sorted({name for *_, bits in self.samples for name, bit in self.REASONS if bits & bit})
        return {"sm_mhz": statistics.median(s[0] for s in self.samples),
                "sm_max_mhz": max(s[1] for s in self.samples),
                "power_w_max": round(max(s[2] for s in self.samples), 1),
                "reasons": reasons, "samples": len(self.samples), "source": self.source}


# ----------------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------------

def build_decode_cache(hla, syn, torch, w, max_chunks, group=8, cache_format="dense"):
    """Fill a decode cache for w.B sequences of w.T-token contexts through the public
    API: hla_prefill with every earlier-chunk weight 0 writes the cache (A/B/key pools
    do not depend on gates) without the quadratic composition."""
    cfg = hla.make_config(w.B, w.H, w.T, w.C, w.d, w.dtype, "routed", w.tau, w.bias, w.thr, cache_format=cache_format,
                          pool_window=w.window, decay=w.decay)
    cache = hla.Cache(cfg, max_chunks)
    gcfg = hla.make_config(group, w.H, w.T, w.C, w.d, w.dtype, "zero", w.tau, w.bias, w.thr,
                           cache_format=cache_format, pool_window=w.window, decay=w.decay)
    ws = torch.empty(hla.prefill_workspace_bytes(gcfg), dtype=torch.uint8, device="cuda")
    first_ctx = None
    for b0 in range(0, w.B, group):
        ctx = syn.make_context_group(w, b0, group, device="cuda")
        if b0 == 0:
            first_ctx = {k: v[:2].clone() for k, v in ctx.items()}
        holder = cache.slice(b0, group)
        o = torch.empty_like(ctx["q"])
        hla.hla_prefill(gcfg, ctx["q"], ctx["k"], ctx["v"], ctx["alpha"], ctx["beta"], o, cache=holder,
                        q_route=ctx.get("q_route"), k_route=ctx.get("k_route"), workspace=ws)
        del ctx, o
    torch.cuda.synchronize()
    del ws
    return cache, first_ctx


def _stage_avg(stages, name, calls):
    """Device milliseconds of one stage per call (a stage may launch several kernels)."""
    ms, n = stages.get(name, (0.0, 0))
    return ms / calls if n and calls else None


def measure_decode_planted(hla, syn, torch, stream, l2_flush, steps, warmup):
    """The planted 32K decode step (the step of the 32K decode with planted route
    inputs: about 4 of the 512 cached chunks active per (sequence, head)).  Timed on
    its own after the main loop: `steps` steps with CUDA events on the launching
    stream, the L2 flushed (untimed) before each.  The active chunks are counted on
    the first warm-up step from its decode workspace, pre-filled with a sentinel:
    the entries the kernel writes are exactly the active ones."""
    wd = syn.DECODE_32K_PLANTED
    max_chunks = wd.T // wd.C + 1
    cache, _ = build_decode_cache(hla, syn, torch, wd, max_chunks, group=8)
    dcfg = hla.make_config(wd.B, wd.H, 1, wd.C, wd.d, wd.dtype, wd.gate_mode, wd.tau, wd.bias, wd.thr)
    nbytes = hla.decode_workspace_bytes(dcfg, max_chunks)
    dws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    toks = [{k: v.cuda() for k, v in t.items()} for t in syn.make_decode_tokens(wd, warmup + steps)]
    n = wd.B * wd.H * max_chunks
    od = torch.empty_like(toks[0]["q"])
    active = None
    for i in range(warmup):
        t = toks[i]
        if i == 0:
            dws.view(torch.int32).fill_(-7)
        hla.hla_decode_step(dcfg, cache, t["q"], t["k"], t["v"], t["alpha"], t["beta"], od, q_route=t["q_route"],
                            k_route=t["k_route"], workspace=dws)
        if i == 0:
            active = (dws.view(torch.int32)[:n] != -7).view(wd.B, wd.H, max_chunks).sum(-1).cpu()
        l2_flush()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    hla.hla_profile_read(reset=True)
    hla.hla_profile_enable(True)
    for s_ in range(steps):
        t = toks[warmup + s_]
        ev[s_][0].record(stream)
        hla.hla_decode_step(dcfg, cache, t["q"], t["k"], t["v"], t["alpha"], t["beta"], od, q_route=t["q_route"],
                            k_route=t["k_route"], workspace=dws)
        ev[s_][1].record(stream)
        l2_flush()
    torch.cuda.synchronize()
    hla.hla_profile_enable(False)
    stages = hla.hla_profile_read(reset=True)
    ms = sum(a.elapsed_time(b) for a, b in ev) / steps
    n_ctx = wd.T // wd.C
    per_chunk = 2 * wd.d * wd.d * 2
    act_total = int(active.sum())
    nbytes_alg = act_total * per_chunk + wd.B * wd.H * n_ctx * wd.d * 4
    kern = _stage_avg(stages, "decode", steps)
    del cache, dws
    torch.cuda.empty_cache()
    return wd, ms, kern, act_total, nbytes_alg, stages


def measure_sparse_prefill(hla, syn, torch, stream, l2_flush, steps, warmup):
    """The long sparse prefill (B=1, H=32, T=131072, C=64, d=128, bf16, planted
    route inputs, threshold 0.05), timed on its own after the main loop: `steps`
    prefills with CUDA events on the launching stream, the L2 flushed (untimed)
    before each.  Inputs are generated on the device (5 x 1 GiB)."""
    wp = syn.SPARSE_LONG
    inp = syn.make_gdn_inputs(wp, device="cuda")
    inp["q_route"], inp["k_route"] = syn.make_route_inputs(wp, device="cuda")
    cfg = hla.make_config(wp.B, wp.H, wp.T, wp.C, wp.d, wp.dtype, wp.gate_mode, wp.tau, wp.bias, wp.thr)
    ws = torch.empty(hla.prefill_workspace_bytes(cfg), dtype=torch.uint8, device="cuda")
    o = torch.empty_like(inp["q"])
    N = wp.N
    acnt = torch.empty((wp.B, wp.H, N), dtype=torch.int32, device="cuda")

    def run(**kw):
        hla.hla_prefill(cfg, inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], o, q_route=inp["q_route"],
                        k_route=inp["k_route"], workspace=ws, **kw)

    for _ in range(warmup):
        run()
        l2_flush()
    run(active_cnt_out=acnt, active_idx_out=torch.empty((wp.B, wp.H, N, N), dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    pairs = int(acnt.sum().item())
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    hla.hla_profile_read(reset=True)
    hla.hla_profile_enable(True)
    for s_ in range(steps):
        l2_flush()
        ev[s_][0].record(stream)
        run()
        ev[s_][1].record(stream)
    torch.cuda.synchronize()
    hla.hla_profile_enable(False)
    stages = hla.hla_profile_read(reset=True)
    ms = sum(a.elapsed_time(b) for a, b in ev) / steps
    # the CPU oracle's sample: the first 16384 tokens of four heads
    sample = {k: inp[k][:, :16384, :4].cpu() for k in ("q", "k", "v", "alpha", "beta", "q_route", "k_route")}
    del inp, ws, o
    torch.cuda.empty_cache()
    return wp, ms, pairs, stages, sample


def run_ours(args):
    import torch
    import torch.distributed as dist

    import gated_delta_rule_transitions_b200 as pkg
    import hla_synth as syn

    hla = pkg._hla
    world, rank, local = rank_env()
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    hbm_gbs, bf16_tf, bf16_tf_sus, peak_src = _peaks()
    stream = torch.cuda.current_stream()

    # ---- prefill workload (inputs resident in HBM) ----
    wp = PREFILL_WORKLOADS[args.prefill_workload](syn)
    if args.prefill_T:
        wp = wp.with_(T=args.prefill_T, name=f"{wp.name}_T{args.prefill_T}")
    if args.chunk != wp.C:
        wp = wp.with_(C=args.chunk, name=wp.name.replace("_C64_", f"_C{args.chunk}_"))
    if args.pool_window:
        wp = wp.with_(window=args.pool_window, name=f"{wp.name}_window{args.pool_window}")
    if args.decay != "scalar":
        wp = wp.with_(decay=args.decay, name=f"{wp.name}_{args.decay}_decay")
    # the long sparse workload is generated on the device (5 x 1 GiB of inputs)
    gen_dev = "cuda" if wp.B * wp.T * wp.H * wp.d > (1 << 28) else "cpu"
    inp = syn.make_gdn_inputs(wp, device=gen_dev)
    qr, kr = syn.make_route_inputs(wp, device=gen_dev)
    inp["q_route"], inp["k_route"] = qr, kr
    inp = {k: v for k, v in inp.items() if v is not None}
    host = {k: v.contiguous().cpu().pin_memory() for k, v in inp.items()}
    dev = {k: v.cuda() for k, v in host.items()}
    del inp
    inp = host
    pcfg = hla.make_config(wp.B, wp.H, wp.T, wp.C, wp.d, wp.dtype, wp.gate_mode, wp.tau, wp.bias, wp.thr,
                           pool_window=wp.window, decay=wp.decay)
    pws = torch.empty(hla.prefill_workspace_bytes(pcfg), dtype=torch.uint8, device="cuda")
    o = torch.empty_like(dev["q"])
    o_host = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    N = wp.N
    acnt = torch.empty((wp.B, wp.H, N), dtype=torch.int32, device="cuda")

    def prefill():
        hla.hla_prefill(pcfg, dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"], o,
                        q_route=dev.get("q_route"), k_route=dev.get("k_route"), workspace=pws)

    # ---- decode workload ----
    wd = syn.DECODE_32K_PLANTED if args.decode_workload == "planted" else syn.DECODE_32K
    if args.decode_B or args.decode_ctx:
        B_ = args.decode_B or wd.B
        T_ = args.decode_ctx or wd.T
        wd = wd.with_(B=B_, T=T_, name=f"decode_bf16_{B_}seq_ctx{T_}_H16_C64_d128_thr0.05"
                                       + ("_planted" if args.decode_workload == "planted" else ""))
    if args.skip_decode:
        wd = wd.with_(B=8, T=64 * 4, name="decode_skipped")
    if args.decode_cache != "dense":
        wd = wd.with_(name=f"{wd.name}_{args.decode_cache}_cache")
    if args.chunk != wd.C:
        wd = wd.with_(C=args.chunk, name=wd.name.replace("_C64_", f"_C{args.chunk}_"))
    if args.pool_window:
        wd = wd.with_(window=args.pool_window, name=f"{wd.name}_window{args.pool_window}")
    if args.decay != "scalar":
        wd = wd.with_(decay=args.decay, name=f"{wd.name}_{args.decay}_decay")
    max_chunks = wd.T // wd.C + 1
    cache, ctx0 = build_decode_cache(hla, syn, torch, wd, max_chunks, group=min(8, wd.B),
                                     cache_format=args.decode_cache)
    torch.cuda.empty_cache()
    dcfg = hla.make_config(wd.B, wd.H, 1, wd.C, wd.d, wd.dtype, wd.gate_mode, wd.tau, wd.bias, wd.thr,
                           cache_format=args.decode_cache, pool_window=wd.window, decay=wd.decay)
    dws = torch.empty(hla.decode_workspace_bytes(dcfg, max_chunks), dtype=torch.uint8, device="cuda")
    ntok = args.warmup + args.steps + 1
    toks_host = [{k: v.contiguous().pin_memory() for k, v in t.items()} for t in syn.make_decode_tokens(wd, ntok)]
    toks = [{k: v.cuda() for k, v in t.items()} for t in toks_host]
    od = torch.empty_like(toks[0]["q"])
    od_host = torch.empty(od.shape, dtype=od.dtype).pin_memory()
    step_idx = [0]

    def decode():
        t = toks[step_idx[0]]
        step_idx[0] += 1
        hla.hla_decode_step(dcfg, cache, t["q"], t["k"], t["v"], t["alpha"], t["beta"], od,
                            q_route=t.get("q_route"), k_route=t.get("k_route"), workspace=dws)

    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    flush_read = torch.ones(L2_FLUSH_BYTES // 8, dtype=torch.int64, device="cuda")

    def l2_flush():
        # write a buffer larger than L2, then read another: the dirty lines of the write
        # go back to HBM here, outside the timed region, and the next phase starts with
        # a cache of clean, unrelated lines
        flush.zero_()
        flush_read.sum()

    for _ in range(max(args.warmup, 0)):
        prefill()
        l2_flush()
        decode()
        l2_flush()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()

    # active pairs of the prefill (for the algorithmic flop count)
    hla.hla_prefill(pcfg, dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"], o,
                    q_route=dev.get("q_route"), k_route=dev.get("k_route"), workspace=pws, active_cnt_out=acnt,
                    active_idx_out=torch.empty((wp.B, wp.H, N, N), dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    active_pairs = int(acnt.sum().item())

    # routing diagnostics (mass and effective support per query chunk) on the same
    # gates, timed alone: it reads the lower triangle of the N x N gate rows
    gates_full = torch.empty((wp.B, wp.H, N, N), dtype=torch.float32, device="cuda")
    hla.hla_prefill(pcfg, dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"], o,
                    q_route=dev.get("q_route"), k_route=dev.get("k_route"), workspace=pws, gates_out=gates_full)
    mass = torch.empty((wp.B, wp.H, N), dtype=torch.float32, device="cuda")
    support = torch.empty_like(mass)
    for _ in range(3):
        hla.hla_gate_support(pcfg, gates_full, mass, support)
    l2_flush()
    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ev_s[0].record(stream)
    for _ in range(20):
        hla.hla_gate_support(pcfg, gates_full, mass, support)
    ev_s[1].record(stream)
    torch.cuda.synchronize()
    support_us = ev_s[0].elapsed_time(ev_s[1]) / 20 * 1e3
    diagnostics = {"gate_support_us": support_us, "gate_rows": wp.B * wp.H * N,
                   "support_median": float(support.median().item()), "mass_median": float(mass.median().item())}
    del gates_full

    hla.hla_profile_read(reset=True)
    hla.hla_profile_enable(True)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(4 * args.steps)]
    with ClockSampler(local) as clocks:
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        for s in range(args.steps):
            e = ev[2 * s]
            e[0].record(stream)
            prefill()
            e[1].record(stream)
            l2_flush()
            e = ev[2 * s + 1]
            e[0].record(stream)
            decode()
            e[1].record(stream)
            l2_flush()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
    hla.hla_profile_enable(False)
    stages = hla.hla_profile_read(reset=True)
    pre_ms = sum(ev[2 * s][0].elapsed_time(ev[2 * s][1]) for s in range(args.steps)) / args.steps
    dec_ms = sum(ev[2 * s + 1][0].elapsed_time(ev[2 * s + 1][1]) for s in range(args.steps)) / args.steps
    pre_ms, dec_ms = max_over_ranks([pre_ms, dec_ms], device="cuda")

    # ---- end to end through the public API with host buffers ----
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(2)]
    reps = max(1, min(args.steps, 5))
    e2e_pre = e2e_dec = 0.0
    for _ in range(reps):
        l2_flush()
        e2e_ev[0][0].record(stream)
        for k in dev:
            dev[k].copy_(host[k], non_blocking=True)
        prefill()
        o_host.copy_(o, non_blocking=True)
        e2e_ev[0][1].record(stream)
        l2_flush()
        e2e_ev[1][0].record(stream)
        t_, th = toks[-1], toks_host[-1]
        for k in t_:
            t_[k].copy_(th[k], non_blocking=True)
        hla.hla_decode_step(dcfg, cache, t_["q"], t_["k"], t_["v"], t_["alpha"], t_["beta"], od,
                            q_route=t_.get("q_route"), k_route=t_.get("k_route"), workspace=dws)
        od_host.copy_(od, non_blocking=True)
        e2e_ev[1][1].record(stream)
        torch.cuda.synchronize()
        e2e_pre += e2e_ev[0][0].elapsed_time(e2e_ev[0][1]) / reps
        e2e_dec += e2e_ev[1][0].elapsed_time(e2e_ev[1][1]) / reps
    e2e_pre, e2e_dec = max_over_ranks([e2e_pre, e2e_dec], device="cuda")
    h2d_pre = sum(v.numel() * v.element_size() for v in host.values())
    d2h_pre = o.numel() * o.element_size()
    h2d_dec = sum(v.numel() * v.element_size() for v in toks_host[0].values())
    d2h_dec = od.numel() * od.element_size()

    # ---- roofline of the dominant kernels ----
    d = wp.d
    if wp.gate_mode == "one":
        # every gate one: the library composes by a prefix scan, N-1 steps per head
        comp_units = wp.B * wp.H * max(N - 1, 0)
        comp_what = f"{comp_units} scan steps (gates all one)"
    else:
        comp_units = active_pairs
        comp_what = f"{active_pairs} active pairs"
    flops_compose = comp_units * 2.0 * d ** 3
    # transitions and read-out per 64-token sub-chunk; at C > 64 also the merge of
    # s = C / 64 sub-chunk transitions per complete chunk (2 (s - 1) products) and the
    # advance of the composed state to the later sub-chunks (s - 1 products per chunk)
    n_sub = (wp.T + 63) // 64
    s_sub = wp.C // 64
    flops_other = wp.B * wp.H * (n_sub * (FLOP_TRANSITION + FLOP_READOUT)
                                 + (2 * (wp.T // wp.C) + N) * (s_sub - 1) * 2.0 * d ** 3)
    comp_avg = _stage_avg(stages, "compose", args.steps) or 0.0
    comp_tf = flops_compose / (comp_avg * 1e-3) / 1e12 if comp_avg > 0 else None
    n_ctx = wd.T // wd.C
    if args.decode_cache == "factored":
        per_chunk = 3 * wd.C * wd.d * 2 + (wd.C + 4) * 4   # K, Wb, Ub bf16 + scales
    else:
        per_chunk = 2 * wd.d * wd.d * 2                      # A, B bf16
    key_reps = wd.C // wd.window if wd.window else 1
    bytes_decode = wd.B * wd.H * (n_ctx * (per_chunk + key_reps * wd.d * 4))
    dmain_avg = _stage_avg(stages, "decode", args.steps) or 0.0
    dec_gbs = bytes_decode / (dmain_avg * 1e-3) / 1e9 if dmain_avg > 0 else None
    if args.decode_workload == "planted":
        dec_gbs = None  # the active chunks are counted by the planted extra line only
    launches = sum(n for (_, n) in stages.values())

    tokens_pre = wp.B * wp.T
    tokens_dec = wd.B
    out = {
        "metric": METRIC,
        "value": whole_job_rate(tokens_pre, pre_ms, world),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": pre_ms + dec_ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded; shapes and distributions of the HLA workloads; no dataset)",
        "config": {"workload": wp.name, "decode_workload": wd.name, "prefill_ms": pre_ms, "decode_ms": dec_ms,
                   "active_pairs": active_pairs, "parallelism": f"replicas x{world} (no data-path collective)",
                   "l2": "flushed before every timed phase (256 MiB write, then a 256 MiB read that "
                         "leaves only clean lines; untimed)"},
        "roofline": {"kernel": "compose", "bound": "tensor", "achieved": comp_tf, "peak": bf16_tf,
                     "unit": "TFLOP/s", "frac": (comp_tf / bf16_tf) if comp_tf else None,
                     "traffic": ncu_traffic("compose"), "traffic_unit": "bytes per launch (ncu dram read+write)",
                     "peak_source": f"{peak_src} bf16 dense (burst)",
                     "sustained": {"peak": bf16_tf_sus,
                                   "frac": (comp_tf / bf16_tf_sus) if comp_tf else None,
                                   "source": f"{peak_src} bf16 dense, seconds-long loop under the power cap"},
                     "datasheet": {"peak": DATASHEET_BF16_TFLOPS,
                                   "frac": (comp_tf / DATASHEET_BF16_TFLOPS) if comp_tf else None,
                                   "source": "B200 datasheet, dense bf16"},
                     "algorithmic": f"{comp_what} x 2 d^3 = {flops_compose:.4g} flop per launch",
                     "prefill_frac_of_peak": (flops_compose + flops_other) / (pre_ms * 1e-3) / 1e12 / bf16_tf},
        "decode": {"value": whole_job_rate(tokens_dec, dec_ms, world), "unit": "tokens/s", "ms_per_step": dec_ms,
                   "roofline": {"kernel": "decode (gate and stream kernels of the step)", "bound": "hbm", "achieved": dec_gbs, "peak": hbm_gbs,
                                "unit": "GB/s", "frac": (dec_gbs / hbm_gbs) if dec_gbs else None,
                                "traffic": ncu_traffic("decode_main") if args.decode_cache == "dense" else None,
                                "traffic_unit": "bytes per step (ncu dram read+write, gate and stream kernels)",
                                "peak_source": f"{peak_src} HBM copy",
                                "datasheet": {"peak": DATASHEET_HBM_GBS,
                                              "frac": (dec_gbs / DATASHEET_HBM_GBS) if dec_gbs else None,
                                              "source": "B200 datasheet HBM3e (about 8 TB/s)"},
                                "algorithmic": f"{bytes_decode:.4g} bytes per launch ({n_ctx} active chunks "
                                               f"({args.decode_cache} cache) + key pools per sequence and head)"},
                   "e2e": {"value": whole_job_rate(tokens_dec, e2e_dec, world), "unit": "tokens/s",
                           "h2d_bytes_per_step": h2d_dec, "d2h_bytes_per_step": d2h_dec}},
        "stages_ms_per_step": {k: v[0] / args.steps for k, v in stages.items() if v[1]},
        "e2e": {"value": whole_job_rate(tokens_pre, e2e_pre, world), "unit": "tokens/s", "h2d_bytes_per_step": h2d_pre,
                "d2h_bytes_per_step": d2h_pre},
        "diagnostics": diagnostics,
        "gpu_launches": launches,
        "clocks": clocks.summary(),
    }
    sparse_sample = None
    if not args.no_extra_lines:
        del cache, dws
        torch.cuda.empty_cache()
        # the planted 32K decode: about 4 active chunks per (sequence, head)
        wdp, ms_dp, kern_dp, act_dp, bytes_dp, st_dp = measure_decode_planted(
            hla, syn, torch, stream, l2_flush, args.steps, args.warmup)
        ms_dp, kern_dp = max_over_ranks([ms_dp, kern_dp or 0.0], device="cuda")
        gbs_dp = bytes_dp / (kern_dp * 1e-3) / 1e9 if kern_dp > 0 else None
        out["decode_sparse"] = {
            "workload": wdp.name, "value": whole_job_rate(wdp.B, ms_dp, world), "unit": "tokens/s",
            "ms_per_step": ms_dp, "active_chunks_mean": act_dp / (wdp.B * wdp.H),
            "roofline": {"kernel": "decode (gate and stream kernels of the step)", "bound": "hbm", "achieved": gbs_dp, "peak": hbm_gbs,
                         "unit": "GB/s", "frac": (gbs_dp / hbm_gbs) if gbs_dp else None,
                         "peak_source": f"{peak_src} HBM copy",
                         "datasheet": {"peak": DATASHEET_HBM_GBS,
                                       "frac": (gbs_dp / DATASHEET_HBM_GBS) if gbs_dp else None},
                         "algorithmic": f"{bytes_dp:.4g} bytes per launch ({act_dp} active A_j/B_j of 64 KiB, "
                                        f"counted on the first warm-up step, + all {wdp.T // wdp.C} key pools of "
                                        f"512 B per sequence and head)", "traffic": ncu_traffic("decode_planted"),
                         "traffic_unit": "bytes per step (ncu dram read+write, gate and stream kernels)"},
            "stages_ms_per_step": {k: v[0] / args.steps for k, v in st_dp.items() if v[1]}}
        # the long sparse prefill (B=1, H=32, T=131072, planted, threshold 0.05)
        wsp, ms_sp, pairs_sp, st_sp, sparse_sample = measure_sparse_prefill(
            hla, syn, torch, stream, l2_flush, args.steps, args.warmup)
        (ms_sp,) = max_over_ranks([ms_sp], device="cuda")
        bthd = wsp.B * wsp.T * wsp.H * wsp.d
        n_sub = wsp.T // 64
        flops_sp = pairs_sp * 2.0 * wsp.d ** 3 + wsp.B * wsp.H * n_sub * (FLOP_TRANSITION + FLOP_READOUT)
        ab_bytes = wsp.B * wsp.H * (wsp.T // wsp.C) * 2 * wsp.d * wsp.d * 2
        bytes_sp = 6 * bthd * 2 + 2 * ab_bytes   # q, k, v, route inputs in, o out; A/B written once, read once
        tf_sp = flops_sp / (ms_sp * 1e-3) / 1e12
        gbs_sp = bytes_sp / (ms_sp * 1e-3) / 1e9
        comp_sp = _stage_avg(st_sp, "compose", args.steps)
        out["sparse_prefill"] = {
            "workload": wsp.name, "value": whole_job_rate(wsp.B * wsp.T, ms_sp, world), "unit": "tokens/s",
            "ms": ms_sp, "active_pairs": pairs_sp,
            "roofline_tensor": {"achieved": tf_sp, "peak": bf16_tf, "unit": "TFLOP/s", "frac": tf_sp / bf16_tf,
                                "peak_source": f"{peak_src} bf16 dense (burst)",
                                "datasheet": {"peak": DATASHEET_BF16_TFLOPS, "frac": tf_sp / DATASHEET_BF16_TFLOPS},
                                "algorithmic": f"{flops_sp:.4g} flop per prefill ({pairs_sp} active pairs x 2 d^3 "
                                               f"+ transitions and read-out of {n_sub} chunks per head)"},
            "roofline_hbm": {"achieved": gbs_sp, "peak": hbm_gbs, "unit": "GB/s", "frac": gbs_sp / hbm_gbs,
                             "peak_source": f"{peak_src} HBM copy",
                             "datasheet": {"peak": DATASHEET_HBM_GBS, "frac": gbs_sp / DATASHEET_HBM_GBS},
                             "algorithmic": f"{bytes_sp:.4g} bytes per prefill (q, k, v, two route inputs read "
                                            f"and o written once; every A_c/B_c written once and read once)"},
            "compose_tflops": (pairs_sp * 2.0 * wsp.d ** 3 / (comp_sp * 1e-3) / 1e12) if comp_sp else None,
            "stages_ms_per_step": {k: v[0] / args.steps for k, v in st_sp.items() if v[1]}}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(inp, wp, wd, ctx0, toks_host, torch, sparse_sample)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


# ----------------------------------------------------------------------------------
# CPU oracle (baseline and reference arm)
# ----------------------------------------------------------------------------------

def _limit_blas_threads():
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:
        pass


def _oracle_prefill_worker(job):
    """One (sequence, head) of the oracle prefill; returns its wall time (s)."""
    _limit_blas_threads()
    from oracle import hla_oracle as ho
    arrays, params, window = job
    t0 = time.perf_counter()
    ho.hla_prefill_head(*arrays[:5], *params, arrays[5], arrays[6], pool_window=window)
    return time.perf_counter() - t0


def _oracle_decode_worker(job):
    """Oracle decode head built from one context (untimed), then one timed step."""
    _limit_blas_threads()
    from oracle import hla_oracle as ho
    ctx, params, tok, window = job
    head = ho.HlaDecodeHead.from_prefill(*ctx, *params, pool_window=window)
    t0 = time.perf_counter()
    head.step(*tok)
    return time.perf_counter() - t0


_REASSOC_TRANS = None


def _oracle_decode_reassoc_worker(job):
    """The decode read-out of `pairs` (sequence, head) pairs in the oracle's
    reassociated mat-vec form (decode_output_backward) over every cached chunk;
    returns the wall time (s).  The cached transitions are seeded random matrices
    of the cache's shape (the work does not depend on their values), made once per
    worker outside the timed region."""
    global _REASSOC_TRANS
    _limit_blas_threads()
    from oracle import hla_oracle as ho
    pairs, n_chunks, d, seed = job
    if _REASSOC_TRANS is None or len(_REASSOC_TRANS) != n_chunks:
        rng = np.random.default_rng(seed)
        _REASSOC_TRANS = [(rng.standard_normal((d, d)) / d, rng.standard_normal((d, d)) / d) for _ in range(n_chunks)]
    rng = np.random.default_rng(seed + 1)
    g = rng.uniform(0.05, 0.2, n_chunks)
    x = rng.standard_normal(d)
    y0 = np.zeros(d)
    active = list(range(n_chunks))
    t0 = time.perf_counter()
    for _ in range(pairs):
        ho.decode_output_backward(_REASSOC_TRANS, g, active, x, y0)
    return time.perf_counter() - t0


def _oracle_sparse_head_worker(job):
    """One head of the long sparse prefill by the oracle; returns its wall time (s)."""
    return _oracle_prefill_worker(job)


class OraclePool:
    """Worker processes for the oracle on the host cores, one BLAS thread each.
    Started with the spawn method: the parent may already hold a CUDA context."""

    def __init__(self, jobs_hint):
        import multiprocessing as mp
        self.n = max(1, min(os.cpu_count() or 1, jobs_hint))
        self.pool = mp.get_context("spawn").Pool(self.n, initializer=_limit_blas_threads)

    def map(self, fn, jobs):
        return self.pool.map(fn, jobs, chunksize=1)

    def close(self):
        self.pool.close()
        self.pool.join()


def _prefill_jobs(inp, wp, pairs):
    def f(name, b, h, dt):
        t = inp.get(name)
        return None if t is None else t[b, :, h].float().numpy().astype(dt)
    params = (wp.C, wp.tau, wp.bias, wp.thr, wp.gate_mode)
    return [((f("q", b, h, np.float64), f("k", b, h, np.float64), f("v", b, h, np.float64),
              f("alpha", b, h, np.float64), f("beta", b, h, np.float64),
              f("q_route", b, h, np.float32), f("k_route", b, h, np.float32)), params, wp.window) for (b, h) in pairs]


def _decode_jobs(ctx, wd, tok, pairs):
    params = (wd.C, wd.tau, wd.bias, wd.thr, wd.gate_mode)
    jobs = []
    for (b, h) in pairs:
        c = tuple(ctx[n][b, :, h].float().cpu().numpy().astype(np.float64) for n in ("q", "k", "v", "alpha", "beta"))
        a_bh = tok["alpha"][b, h]
        t = (tok["q"][b, h].double().numpy(), tok["k"][b, h].double().numpy(), tok["v"][b, h].double().numpy(),
             a_bh.double().numpy() if a_bh.dim() else float(a_bh), float(tok["beta"][b, h]))
        jobs.append((c, params, t, wd.window))
    return jobs


def _cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown CPU"


def cpu_baseline(inp, wp, wd, ctx0, toks_host, torch, sparse_sample=None):
    """The oracle on the host cores: the full prefill (every (sequence, head) of the
    prompt, one per worker process), one decode step of a sample of (sequence,
    head) pairs in the definition form, the whole decode step in the reassociated
    mat-vec form, and (given its sample) four heads of the long sparse prefill."""
    pairs_p = [(b, h) for b in range(wp.B) for h in range(wp.H)]
    pairs_d = [(b, h) for b in range(min(2, wd.B)) for h in range(8)]
    pool = OraclePool(max(len(pairs_p), len(pairs_d)))
    try:
        t0 = time.perf_counter()
        pool.map(_oracle_prefill_worker, _prefill_jobs(inp, wp, pairs_p))
        tp = time.perf_counter() - t0
        td = pool.map(_oracle_decode_worker, _decode_jobs(ctx0, wd, toks_host[0], pairs_d))
        # the whole decode step (all B x H pairs) in the reassociated form, split over the workers
        n_pairs = wd.B * wd.H
        per = [n_pairs // pool.n + (1 if i < n_pairs % pool.n else 0) for i in range(pool.n)]
        # each worker times its own share (its set-up of the cached matrices excluded);
        # the step takes as long as the slowest share
        tr = max(pool.map(_oracle_decode_reassoc_worker, [(p_, wd.T // wd.C, wd.d, 11) for p_ in per]))
        sparse = None
        if sparse_sample is not None:
            import hla_synth as syn
            ws_ = syn.SPARSE_LONG
            nh, ts_ = sparse_sample["q"].shape[2], sparse_sample["q"].shape[1]
            ts = pool.map(_oracle_sparse_head_worker,
                          _prefill_jobs(sparse_sample, ws_.with_(T=ts_), [(0, h) for h in range(nh)]))
            # head-tokens per second on `cores` workers, extrapolated linearly to the whole
            # prompt (the token rule dominates the oracle's time on this sparse workload)
            rate = pool.n * ts_ / max(ts)
            sparse = {"value": rate * ws_.T / (ws_.H * ws_.T), "unit": "tokens/s", "kind": "oracle",
                      "sample": f"the first {ts_} tokens of {nh} of the {ws_.H} heads, one per worker (slowest "
                                f"{max(ts):.1f} s); tokens/s of the whole prompt on {pool.n} workers, scaled "
                                f"linearly in tokens and heads"}
    finally:
        pool.close()
    td_mean = statistics.mean(td)
    res = {"value": wp.B * wp.T / tp, "unit": "tokens/s", "cores": pool.n, "kind": "oracle",
            "sample": f"prefill: the whole prompt ({wp.B * wp.H} (sequence, head) pairs of T={wp.T}, "
                      f"{tp:.1f} s wall on {pool.n} worker processes); decode: one step of {len(pairs_d)} "
                      f"(sequence, head) pairs of the 32K context ({td_mean:.3f} s each), tokens/s = cores / "
                      f"(H x time per pair); {_cpu_model()}",
            "decode": {"value": pool.n / (wd.H * td_mean), "unit": "tokens/s"},
            "decode_reassociated": {"value": wd.B / tr, "unit": "tokens/s", "kind": "oracle (reassociated mat-vec form)",
                                    "sample": f"the whole step: {wd.B * wd.H} (sequence, head) pairs x "
                                              f"{wd.T // wd.C} cached chunks by decode_output_backward on "
                                              f"{pool.n} workers (slowest share {tr:.2f} s); cached "
                                              f"transitions are seeded matrices of the cache's shape"}}
    if sparse is not None:
        res["sparse_prefill"] = sparse
    return res


def run_reference(args):
    """The oracle as it stands, on the host cores, on the same workloads; rank 0
    only.  Each step is the whole prefill prompt (every (sequence, head) in parallel
    worker processes) plus one decode step of a sample of (sequence, head) pairs."""
    world, rank, _ = rank_env()
    if rank != 0:
        return
    import torch
    import hla_synth as syn
    wp = syn.PREFILL_0P8B
    wd = syn.DECODE_32K
    inp = syn.make_gdn_inputs(wp)
    inp["q_route"], inp["k_route"] = syn.make_route_inputs(wp)
    # decode context of 1 sequence (CPU generator; same shapes and distributions)
    ctx = syn.make_gdn_inputs(wd.with_(B=1), device="cpu")
    tok = syn.make_decode_tokens(wd.with_(B=1), 1)[0]
    pairs_p = [(b, h) for b in range(wp.B) for h in range(wp.H)]
    pairs_d = [(0, h) for h in range(min(8, wd.H))]
    pool = OraclePool(len(pairs_p))
    jobs_p = _prefill_jobs(inp, wp, pairs_p)
    jobs_d = _decode_jobs(ctx, wd, tok, pairs_d)
    times_p, times_d = [], []
    try:
        for s in range(args.warmup + args.steps):
            t0 = time.perf_counter()
            pool.map(_oracle_prefill_worker, jobs_p)
            tp = time.perf_counter() - t0
            td = statistics.mean(pool.map(_oracle_decode_worker, jobs_d)) if (s < 1 or s >= args.warmup) else 0.0
            if s >= args.warmup:
                times_p.append(tp)
                times_d.append(td)
    finally:
        pool.close()
    tp = statistics.mean(times_p)
    td = statistics.mean(times_d)
    val = wp.B * wp.T / tp
    out = {"impl": "reference", "metric": METRIC, "value": val, "unit": "tokens/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": tp * 1e3, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": wp.name, "decode_workload": wd.name},
           "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": pool.n, "kind": "oracle",
                            "sample": f"each step: the whole T={wp.T} prefill ({len(pairs_p)} (sequence, head) "
                                      f"pairs on {pool.n} worker processes) and one decode step of "
                                      f"{len(pairs_d)} (sequence, head) pairs of one 32K context; {_cpu_model()}"},
           "decode": {"value": pool.n / (wd.H * td), "unit": "tokens/s"},
           "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra-lines", action="store_true",
                    help="skip the planted 32K decode and the long sparse prefill (timed after the main loop)")
    # smaller variants for profiling captures (the default is the full workload)
    ap.add_argument("--prefill-T", type=int, default=None, help="prefill tokens (default: the workload's)")
    ap.add_argument("--prefill-workload", choices=sorted(PREFILL_WORKLOADS), default="dense",
                    help="dense: the 0.8B-like layer (the metric's workload); sparse: B=1, H=32, T=131072 "
                         "with planted gates; gdn: B=4, H=16, T=4096 with all gates one")
    ap.add_argument("--decode-B", type=int, default=None, help="decode sequences (default 64)")
    ap.add_argument("--decode-ctx", type=int, default=None, help="decode context tokens (default 32768)")
    ap.add_argument("--skip-decode", action="store_true")
    ap.add_argument("--decode-workload", choices=["dense", "planted"], default="dense",
                    help="main decode line: every cached chunk active (dense) or the planted routes "
                         "(about 4 active chunks per sequence and head)")
    ap.add_argument("--decode-cache", choices=["dense", "factored"], default="dense",
                    help="dense: A_j/B_j d x d (the metric's workload); factored: K_j, Wb_j, Ub_j per chunk")
    ap.add_argument("--chunk", type=int, choices=[64, 128, 256], default=64,
                    help="chunk size C of both workloads (the metric's workloads use 64)")
    ap.add_argument("--pool-window", type=int, default=0,
                    help="key window representatives of this many tokens (0: one pool per chunk)")
    ap.add_argument("--decay", choices=["scalar", "channel"], default="scalar",
                    help="scalar: one decay per token (the metric's workloads); channel: one per key channel")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
