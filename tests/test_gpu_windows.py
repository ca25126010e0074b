"""GPU parity with window representatives (the pages' gate: a log-sum-exp over a
chunk's window representatives inside the sigmoid; "Methodology in Plain English"
para. 2, window 32 by default per "Main Findings").

Window pools, gates and active lists are bit-exact against the oracle's binary32
recipe; outputs within max-abs 1e-4 (float32 path) or relative L2 2e-2 (bf16)."""
import numpy as np
import pytest
import torch

import hla_synth as syn
from oracle import hla_oracle as ho
from tests import _parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hla():
    import gated_delta_rule_transitions_b200 as m
    m.lib()
    return m._hla


def _check_prefill(hla, w):
    inp = P.gpu_inputs(w)
    o, gates, aidx, acnt = P.run_prefill(hla, w, inp)
    B, T, H, _ = inp["q"].shape
    ref = np.zeros(tuple(inp["v"].shape))
    for b in range(B):
        for h in range(H):
            r = P.oracle_prefill_head(w, inp, b, h)
            ref[b, :, h] = r.o
            P.check_routing_exact(r, gates, aidx, acnt, b, h)
    got = P.np64(o)
    if w.dtype == "f32":
        P.check_f32(got, ref)
    else:
        P.check_bf16(got, ref, layout="bthd")
    st, code = hla.hla_device_status()
    assert st == 0 and code == 0
    return gates


@pytest.mark.parametrize("C,window,T,thr", [
    (256, 32, 256 * 5 + 77, 0.0),     # the pages' defaults: 8 windows per chunk
    (256, 32, 256 * 6, 0.3),
    (64, 32, 64 * 9 + 30, 0.0),
    (128, 8, 128 * 4 + 64, 0.2),      # 16 windows per chunk (the maximum)
])
def test_bf16_window_gates(hla, C, window, T, thr):
    w = syn.PREFILL_0P8B.with_(B=2, H=2, T=T, C=C, window=window, thr=thr)
    gates = _check_prefill(hla, w)
    N = w.N
    low = gates.numpy()[:, :, np.tril_indices(N, -1)[0], np.tril_indices(N, -1)[1]]
    assert np.all((low > 0.0) & (low <= 1.0))


def test_f32_window_gates_planted(hla):
    w = syn.SPARSE_LONG.with_(B=1, H=2, T=64 * 14 + 9, C=64, dtype="f32", d=64, topics=3, window=16)
    _check_prefill(hla, w)


def test_routing_window_pools_bit_exact(hla):
    w = syn.PREFILL_0P8B.with_(B=1, H=3, T=128 * 6 + 40, C=128, window=32, thr=0.2)
    inp = P.gpu_inputs(w)
    B, T, H, d = inp["q"].shape
    N, W = w.N, w.C // w.window
    cfg = hla.make_config(B, H, T, w.C, d, w.dtype, "routed", w.tau, w.bias, w.thr, pool_window=w.window)
    g = P.to_cuda(inp)
    rq = torch.empty((B, H, N, d), dtype=torch.float32, device="cuda")
    rk = torch.full((B, H, N * W, d), float("nan"), dtype=torch.float32, device="cuda")
    gates = torch.empty((B, H, N, N), dtype=torch.float32, device="cuda")
    hla.hla_routing(cfg, g["q_route"], g["k_route"], rq, rk, gates_out=gates)
    torch.cuda.synchronize()
    rk = rk.cpu().numpy()
    for h in range(H):
        ref = ho.window_pools(P.np32(inp["k_route"][0, :, h]), w.C, w.window, w.tau)   # complete chunks
        got = rk[0, h, :ref.shape[0] * W].reshape(ref.shape)
        assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
        rqr = ho.route_pools(P.np32(inp["q_route"][0, :, h]), w.C, w.tau)
        assert np.array_equal(rq[0, h].cpu().numpy().view(np.uint32), rqr.view(np.uint32))
        G = ho.gate_matrix(rqr, ref, d, w.bias)
        assert np.array_equal(gates[0, h].cpu().numpy().view(np.uint32), G.view(np.uint32))


@pytest.mark.parametrize("dtype,d,C,window,T0,steps,fmt", [
    ("f32", 64, 64, 16, 64 * 3 + 60, 7, "dense"),      # CUDA-core decode, closes chunk 3 at step 4
    ("bf16", 128, 128, 32, 128 * 2 + 125, 6, "dense"),  # TMA-streamed decode, closes at step 3
    ("bf16", 128, 64, 32, 64 * 4 + 61, 6, "factored"),  # factored cache
])
def test_decode_window_gates(hla, dtype, d, C, window, T0, steps, fmt):
    w = syn.DECODE_32K.with_(B=2, H=2, T=T0, C=C, dtype=dtype, d=d, thr=0.2, bias=-0.5, route="spread",
                             window=window)
    inp = P.gpu_inputs(w)
    maxc = T0 // C + 2
    cfg = hla.make_config(w.B, w.H, T0, C, d, dtype, "routed", w.tau, w.bias, w.thr, cache_format=fmt,
                          pool_window=window)
    cache = hla.Cache(cfg, max_chunks=maxc)
    P.run_prefill(hla, w, inp, cache=cache, cache_format=fmt)
    heads = {}
    for b in range(w.B):
        for h in range(w.H):
            f = lambda n: inp[n][b, :, h]
            heads[(b, h)] = ho.HlaDecodeHead.from_prefill(
                P.np64(f("q")), P.np64(f("k")), P.np64(f("v")), P.np64(f("alpha")), P.np64(f("beta")), C,
                w.tau, w.bias, w.thr, "routed", P.np32(f("q_route")), P.np32(f("k_route")), pool_window=window)
    dcfg = hla.make_config(w.B, w.H, 1, C, d, dtype, "routed", w.tau, w.bias, w.thr, cache_format=fmt,
                           pool_window=window)
    g = torch.Generator().manual_seed(91)
    tdt = syn.torch_dtype(w)
    got, ref = [], []
    for tk in syn.make_decode_tokens(w, steps):
        qr = (torch.randn((w.B, w.H, d), generator=g) * 1.4).to(tdt)
        kr = (qr.float() + 0.3 * torch.randn((w.B, w.H, d), generator=g)).to(tdt)
        gt = {k: v.cuda().contiguous() for k, v in tk.items()}
        o = torch.empty_like(gt["q"])
        hla.hla_decode_step(dcfg, cache, gt["q"], gt["k"], gt["v"], gt["alpha"], gt["beta"], o,
                            q_route=qr.cuda(), k_route=kr.cuda())
        torch.cuda.synchronize()
        o = P.np64(o)
        for (b, h), st in heads.items():
            ref.append(st.step(P.np64(tk["q"][b, h]), P.np64(tk["k"][b, h]), P.np64(tk["v"][b, h]),
                               float(tk["alpha"][b, h]), float(tk["beta"][b, h]),
                               P.np32(qr[b, h]), P.np32(kr[b, h])))
            got.append(o[b, h])
    got, ref = np.stack(got), np.stack(ref)
    if dtype == "f32":
        P.check_f32(got, ref)
    else:
        P.check_bf16(got, ref, layout="steps", nh=len(heads))
    st, code = hla.hla_device_status()
    assert st == 0 and code == 0
    W = C // window
    rk = cache.view("rk", (w.B, w.H, maxc, W, d), torch.float32).cpu().numpy()
    for (b, h), st_ in heads.items():
        assert len(st_.rk) == (T0 + steps) // C
        for j in range(len(st_.rk)):
            assert np.array_equal(rk[b, h, j].view(np.uint32), st_.rk[j].view(np.uint32))


def test_window_gates_16_row_tiles(hla):
    """Enough query chunks for the 16-row tiles of the windowed gate kernel (at least
    two CTAs per SM): B=1, H=20, 256 chunks of 64 tokens, window 32.  Gates and
    active lists bit-exact on two heads (the routing call alone)."""
    w = syn.PREFILL_0P8B.with_(B=1, H=20, T=64 * 256, C=64, window=32, thr=0.3)
    inp = P.gpu_inputs(w)
    B, T, H, d = inp["q"].shape
    N, W = w.N, w.C // w.window
    assert (N // 16) * B * H >= 2 * 148
    cfg = hla.make_config(B, H, T, w.C, d, w.dtype, "routed", w.tau, w.bias, w.thr, pool_window=w.window)
    g = P.to_cuda(inp)
    rq = torch.empty((B, H, N, d), dtype=torch.float32, device="cuda")
    rk = torch.empty((B, H, N * W, d), dtype=torch.float32, device="cuda")
    gates = torch.empty((B, H, N, N), dtype=torch.float32, device="cuda")
    aidx = torch.empty((B, H, N, N), dtype=torch.int32, device="cuda")
    acnt = torch.empty((B, H, N), dtype=torch.int32, device="cuda")
    hla.hla_routing(cfg, g["q_route"], g["k_route"], rq, rk, gates_out=gates, active_idx_out=aidx,
                    active_cnt_out=acnt)
    torch.cuda.synchronize()
    for h in (0, 13):
        rqr = ho.route_pools(P.np32(inp["q_route"][0, :, h]), w.C, w.tau)
        rkw = ho.window_pools(P.np32(inp["k_route"][0, :, h]), w.C, w.window, w.tau)
        G = ho.gate_matrix(rqr, rkw, d, w.bias)
        res = ho.HeadResult(o=None, gates=G, active=ho.active_lists(G, w.thr), rq=rqr, rk=rkw)
        P.check_routing_exact(res, gates.cpu(), aidx.cpu(), acnt.cpu(), 0, h)
