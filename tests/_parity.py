"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI
and the oracle on the same seeded inputs, and assert the bars.

Bars: max-abs <= 1e-4 on the float32 path; relative L2 <= 2e-2 on the bf16 path,
asserted for every (sequence, head) on its own (a pooled norm over many heads could
hide one wrong head).  Every check records the error it reached; the session's
worst case per test is printed at the end of the run and, when HLA_PARITY_LOG names
a file, written there as JSON lines."""
from __future__ import annotations

import json
import os

import numpy as np
import torch

import hla_synth as syn
from oracle import hla_oracle as ho

TOL_F32_MAXABS = 1e-4   # fp32 path: max-abs error against the fp64 oracle
TOL_BF16_RELL2 = 2e-2   # bf16 path: relative L2 error over the output tensor


def np64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def np32(t):
    return t.detach().float().cpu().numpy().astype(np.float32)


def rel_l2(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


# (test id, what, kind, achieved, bar) of every check in this process
MARGINS: list[tuple[str, str, str, float, float]] = []


def _record(what, kind, err, bar):
    test = os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0]
    MARGINS.append((test, what, kind, float(err), float(bar)))
    path = os.environ.get("HLA_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"test": test, "what": what, "kind": kind, "err": float(err), "bar": float(bar)})
                    + "\n")


def check_f32(got, ref, what="output", tol=TOL_F32_MAXABS):
    """float32 path: max-abs error against the oracle."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = float(np.abs(got - ref).max()) if got.size else 0.0
    _record(what, "maxabs", err, tol)
    assert err <= tol, f"{what}: max-abs {err:.3e} > {tol:.1e}"
    return err


def _heads(got, ref, layout, nh):
    """(label, got, ref) per (sequence, head).  layout "bthd": [B,T,H,d] tensors;
    "bhd": [B,H,d] (one decode step); "steps": [steps * nh, d] rows, step-major over
    nh (sequence, head) pairs (chained decode steps); "head": already one head."""
    if layout == "steps":
        g = got.reshape(-1, nh, got.shape[-1])
        r = ref.reshape(-1, nh, ref.shape[-1])
        for j in range(nh):
            yield f"pair{j}", g[:, j], r[:, j]
    elif layout == "bthd":
        for b in range(got.shape[0]):
            for h in range(got.shape[2]):
                yield f"b{b}h{h}", got[b, :, h], ref[b, :, h]
    elif layout == "bhd":
        for b in range(got.shape[0]):
            for h in range(got.shape[1]):
                yield f"b{b}h{h}", got[b, h], ref[b, h]
    else:
        yield "", got, ref


def check_bf16(got, ref, what="output", layout="head", tol=TOL_BF16_RELL2, nh=1):
    """bf16 path: relative L2 error, asserted for every (sequence, head) of `layout`
    on its own; returns the worst one."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    worst, where = 0.0, ""
    for label, g, r in _heads(got, ref, layout, nh):
        e = rel_l2(g, r)
        if e > worst or not where:
            worst, where = e, label
    _record(what, "rel_l2_per_head", worst, tol)
    assert worst <= tol, f"{what}: relative L2 {worst:.3e} > {tol:.1e} at {where}"
    return worst


def gpu_inputs(w: syn.Workload, T=None, B=None):
    inp = syn.make_gdn_inputs(w, T=T, B=B)
    qr, kr = syn.make_route_inputs(w, T=T, B=B)
    inp["q_route"], inp["k_route"] = qr, kr
    return inp


def to_cuda(inp):
    return {k: (None if v is None else v.cuda().contiguous()) for k, v in inp.items()}


def run_prefill(hla, w: syn.Workload, inp, user_gates=None, cache=None, cache_format="dense"):
    B, T, H, d = inp["q"].shape
    N = (T + w.C - 1) // w.C
    cfg = hla.make_config(B, H, T, w.C, d, w.dtype, w.gate_mode, w.tau, w.bias, w.thr, cache_format=cache_format,
                          pool_window=w.window, decay=w.decay)
    g = to_cuda(inp)
    o = torch.empty_like(g["q"])
    gates = torch.empty((B, H, N, N), dtype=torch.float32, device="cuda")
    aidx = torch.empty((B, H, N, N), dtype=torch.int32, device="cuda")
    acnt = torch.empty((B, H, N), dtype=torch.int32, device="cuda")
    ug = None if user_gates is None else user_gates.cuda().contiguous()
    hla.hla_prefill(cfg, g["q"], g["k"], g["v"], g["alpha"], g["beta"], o, q_route=g["q_route"],
                    k_route=g["k_route"], user_gates=ug, gates_out=gates, active_idx_out=aidx,
                    active_cnt_out=acnt, cache=cache)
    torch.cuda.synchronize()
    return o.cpu(), gates.cpu(), aidx.cpu(), acnt.cpu()


def oracle_prefill_head(w: syn.Workload, inp, b, h, user_gates=None, query_chunks=None):
    f = lambda name: None if inp.get(name) is None else np64(inp[name][b, :, h])
    return ho.hla_prefill_head(
        f("q"), f("k"), f("v"), np64(inp["alpha"][b, :, h]), np64(inp["beta"][b, :, h]), w.C,
        w.tau, w.bias, w.thr, w.gate_mode,
        None if inp.get("q_route") is None else np32(inp["q_route"][b, :, h]),
        None if inp.get("k_route") is None else np32(inp["k_route"][b, :, h]),
        None if user_gates is None else user_gates[b, h].numpy(),
        query_chunks=query_chunks, pool_window=w.window)


def check_routing_exact(res, gates, aidx, acnt, b, h):
    """Gates bit-exact, active lists identical."""
    G = gates[b, h].numpy()
    assert np.array_equal(G.view(np.uint32), res.gates.view(np.uint32)), \
        f"gates differ at {np.argwhere(G != res.gates)[:5]}"
    for i, act in enumerate(res.active):
        n = int(acnt[b, h, i])
        assert n == len(act), (i, n, len(act))
        assert np.array_equal(aidx[b, h, i, :n].numpy(), act)
        assert np.all(aidx[b, h, i, n:].numpy() == -1)
