"""GPU parity of the decode step against the oracle (through the C ABI).

A prefill writes the cache; chained decode steps (crossing a chunk boundary, so a
chunk is closed into the cache) are compared token by token with the oracle's
decode state, which follows the definition (forward composition of S_in, then the
token rule over the open chunk).  Cached key pools must be bit-exact."""
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


def _route_tokens(B, H, d, steps, seed, dtype):
    g = torch.Generator().manual_seed(seed)
    out = []
    for _ in range(steps):
        mu = torch.randn((B, H, d), generator=g) * 1.4
        out.append((mu.to(dtype), (mu + 0.3 * torch.randn((B, H, d), generator=g)).to(dtype)))
    return out


@pytest.mark.parametrize("dtype,d,mode,thr,route", [
    ("f32", 64, "routed", 0.05, False),
    ("f32", 64, "routed", 0.4, True),
    ("bf16", 128, "routed", 0.05, False),
    ("bf16", 128, "routed", 0.4, True),
    ("bf16", 128, "one", 0.0, False),
    ("f32", 64, "zero", 0.0, False),
])
def test_decode_chain_matches_oracle(hla, dtype, d, mode, thr, route):
    T0 = 64 * 3 + 58
    steps = 9  # closes chunk 3 after 6 steps, then opens chunk 4
    w = syn.DECODE_32K.with_(B=2, H=2, T=T0, dtype=dtype, d=d, gate_mode=mode, thr=thr,
                             route="spread" if route else "default", bias=-0.5 if route else -2.0)
    inp = P.gpu_inputs(w)
    cfg = hla.make_config(w.B, w.H, T0, 64, d, dtype, mode, w.tau, w.bias, w.thr)
    cache = hla.Cache(cfg, max_chunks=8)
    P.run_prefill(hla, w, inp, cache=cache)
    toks = syn.make_decode_tokens(w, steps)
    tdt = syn.torch_dtype(w)
    routes = _route_tokens(w.B, w.H, d, steps, 77, tdt) if route else [(None, None)] * steps
    heads = {}
    for b in range(w.B):
        for h in range(w.H):
            f = lambda n: None if inp.get(n) is None else inp[n][b, :, h]
            heads[(b, h)] = ho.HlaDecodeHead.from_prefill(
                P.np64(f("q")), P.np64(f("k")), P.np64(f("v")), P.np64(f("alpha")), P.np64(f("beta")), 64,
                w.tau, w.bias, w.thr, mode,
                None if f("q_route") is None else P.np32(f("q_route")),
                None if f("k_route") is None else P.np32(f("k_route")))
    dcfg = hla.make_config(w.B, w.H, 1, 64, d, dtype, mode, w.tau, w.bias, w.thr)
    errs = []
    for s, tk in enumerate(toks):
        g = {k: v.cuda().contiguous() for k, v in tk.items()}
        qr, kr = routes[s]
        o = torch.empty_like(g["q"])
        hla.hla_decode_step(dcfg, cache, g["q"], g["k"], g["v"], g["alpha"], g["beta"], o,
                            q_route=None if qr is None else qr.cuda(), k_route=None if kr is None else kr.cuda())
        torch.cuda.synchronize()
        o = P.np64(o)
        for (b, h), st in heads.items():
            ref = st.step(P.np64(tk["q"][b, h]), P.np64(tk["k"][b, h]), P.np64(tk["v"][b, h]),
                          float(tk["alpha"][b, h]), float(tk["beta"][b, h]),
                          None if qr is None else P.np32(qr[b, h]), None if kr is None else P.np32(kr[b, h]))
            errs.append((o[b, h], ref))
    got = np.stack([e[0] for e in errs])
    ref = np.stack([e[1] for e in errs])
    if dtype == "f32":
        P.check_f32(got, ref)
    else:
        P.check_bf16(got, ref, layout="steps", nh=len(heads))
    st, code = hla.hla_device_status()
    assert st == 0 and code == 0
    # counters and the closed chunk's key pool
    n = cache.view("n_chunks", (w.B,), torch.int32).cpu()
    m = cache.view("m_partial", (w.B,), torch.int32).cpu()
    assert n.tolist() == [4] * w.B and m.tolist() == [(T0 + steps) % 64] * w.B
    rk = cache.view("rk", (w.B, w.H, 8, d), torch.float32).cpu().numpy()
    for (b, h), st_ in heads.items():
        for j in range(4):
            assert np.array_equal(rk[b, h, j].view(np.uint32), st_.rk[j].view(np.uint32))


@pytest.mark.parametrize("mode,thr,route", [("routed", 0.05, False), ("routed", 0.4, True), ("one", 0.0, False)])
def test_decode_factored_cache_matches_oracle(hla, mode, thr, route):
    """Decode from a factored cache (K_j, Wb_j, Ub_j and the scales per closed chunk):
    prefill hand-off, chained steps that close a chunk (the closing step writes the
    new chunk's factors), outputs against the oracle and against the same steps on a
    dense cache."""
    T0 = 64 * 3 + 58
    steps = 9
    w = syn.DECODE_32K.with_(B=2, H=2, T=T0, gate_mode=mode, thr=thr,
                             route="spread" if route else "default", bias=-0.5 if route else -2.0)
    inp = P.gpu_inputs(w)
    caches = {}
    for fmt in ("factored", "dense"):
        cfg = hla.make_config(w.B, w.H, T0, 64, 128, "bf16", mode, w.tau, w.bias, w.thr, cache_format=fmt)
        caches[fmt] = hla.Cache(cfg, max_chunks=8)
        P.run_prefill(hla, w.with_(), inp, cache=caches[fmt], cache_format=fmt)
    toks = syn.make_decode_tokens(w, steps)
    routes = _route_tokens(w.B, w.H, 128, steps, 77, torch.bfloat16) if route else [(None, None)] * steps
    heads = {}
    for b in range(w.B):
        for h in range(w.H):
            f = lambda n: None if inp.get(n) is None else inp[n][b, :, h]
            heads[(b, h)] = ho.HlaDecodeHead.from_prefill(
                P.np64(f("q")), P.np64(f("k")), P.np64(f("v")), P.np64(f("alpha")), P.np64(f("beta")), 64,
                w.tau, w.bias, w.thr, mode,
                None if f("q_route") is None else P.np32(f("q_route")),
                None if f("k_route") is None else P.np32(f("k_route")))
    got, dense, ref = [], [], []
    for s_, tk in enumerate(toks):
        g = {k: v.cuda().contiguous() for k, v in tk.items()}
        qr, kr = routes[s_]
        outs = {}
        for fmt, cache in caches.items():
            dcfg = hla.make_config(w.B, w.H, 1, 64, 128, "bf16", mode, w.tau, w.bias, w.thr, cache_format=fmt)
            o = torch.empty_like(g["q"])
            hla.hla_decode_step(dcfg, cache, g["q"], g["k"], g["v"], g["alpha"], g["beta"], o,
                                q_route=None if qr is None else qr.cuda(), k_route=None if kr is None else kr.cuda())
            outs[fmt] = o
        torch.cuda.synchronize()
        for (b, h), st_ in heads.items():
            got.append(P.np64(outs["factored"][b, h]))
            dense.append(P.np64(outs["dense"][b, h]))
            ref.append(st_.step(P.np64(tk["q"][b, h]), P.np64(tk["k"][b, h]), P.np64(tk["v"][b, h]),
                                float(tk["alpha"][b, h]), float(tk["beta"][b, h]),
                                None if qr is None else P.np32(qr[b, h]), None if kr is None else P.np32(kr[b, h])))
    got, dense, ref = np.stack(got), np.stack(dense), np.stack(ref)
    P.check_bf16(got, ref, layout="steps", nh=len(heads))
    P.check_bf16(got, dense, "factored vs dense cache", layout="steps", nh=len(heads))
    st, code = hla.hla_device_status()
    assert st == 0 and code == 0
    n = caches["factored"].view("n_chunks", (w.B,), torch.int32).cpu().tolist()
    assert n == [(T0 + steps) // 64] * w.B


@pytest.mark.parametrize("dtype,d,fmt", [("bf16", 128, "dense"), ("f32", 64, "dense"), ("bf16", 128, "factored")])
def test_decode_ragged_positions(hla, dtype, d, fmt):
    """Sequences at different positions in one cache: each is prefilled on its own
    (prompts of 202 and 370 tokens) into its slice of the cache, then chained decode
    steps advance both together; they close chunks at different steps.  Every output
    is compared with that sequence's oracle decode head."""
    lens = [64 * 3 + 10, 64 * 5 + 50]
    steps = 60
    base = syn.DECODE_32K.with_(B=1, H=2, dtype=dtype, d=d, thr=0.05, bias=-0.5, route="spread")
    cfg2 = hla.make_config(2, base.H, max(lens), 64, d, dtype, "routed", base.tau, base.bias, base.thr,
                           cache_format=fmt)
    cache = hla.Cache(cfg2, max_chunks=8)
    heads = {}
    for b, T_b in enumerate(lens):
        w = base.with_(T=T_b, seed=11 + b)
        inp = P.gpu_inputs(w)
        P.run_prefill(hla, w, inp, cache=cache.slice(b, 1), cache_format=fmt)
        for h in range(w.H):
            f = lambda n: None if inp.get(n) is None else inp[n][0, :, h]
            heads[(b, h)] = ho.HlaDecodeHead.from_prefill(
                P.np64(f("q")), P.np64(f("k")), P.np64(f("v")), P.np64(f("alpha")), P.np64(f("beta")), 64,
                w.tau, w.bias, w.thr, "routed", P.np32(f("q_route")), P.np32(f("k_route")))
    dcfg = hla.make_config(2, base.H, 1, 64, d, dtype, "routed", base.tau, base.bias, base.thr, cache_format=fmt)
    toks = syn.make_decode_tokens(base.with_(B=2), steps)
    routes = _route_tokens(2, base.H, d, steps, 91, syn.torch_dtype(base))
    got, ref = [], []
    for s_, tk in enumerate(toks):
        g = {k: v.cuda().contiguous() for k, v in tk.items()}
        qr, kr = routes[s_]
        o = torch.empty_like(g["q"])
        hla.hla_decode_step(dcfg, cache, g["q"], g["k"], g["v"], g["alpha"], g["beta"], o, q_route=qr.cuda(),
                            k_route=kr.cuda())
        torch.cuda.synchronize()
        o = P.np64(o)
        for (b, h), st_ in heads.items():
            got.append(o[b, h])
            ref.append(st_.step(P.np64(tk["q"][b, h]), P.np64(tk["k"][b, h]), P.np64(tk["v"][b, h]),
                                float(tk["alpha"][b, h]), float(tk["beta"][b, h]), P.np32(qr[b, h]),
                                P.np32(kr[b, h])))
    got, ref = np.stack(got), np.stack(ref)
    if dtype == "f32":
        P.check_f32(got, ref)
    else:
        P.check_bf16(got, ref, layout="steps", nh=len(heads))
    st, code = hla.hla_device_status()
    assert st == 0 and code == 0
    n = cache.view("n_chunks", (2,), torch.int32).cpu().tolist()
    m = cache.view("m_partial", (2,), torch.int32).cpu().tolist()
    assert n == [(T + steps) // 64 for T in lens] and m == [(T + steps) % 64 for T in lens]


def test_decode_cache_full_is_reported(hla):
    w = syn.DECODE_32K.with_(B=1, H=1, T=64 * 2 + 63, dtype="f32", d=64)
    inp = P.gpu_inputs(w)
    cfg = hla.make_config(1, 1, w.T, 64, 64, "f32", "routed", 1.0, -2.0, 0.05)
    cache = hla.Cache(cfg, max_chunks=2)
    P.run_prefill(hla, w, inp, cache=cache)
    tk = syn.make_decode_tokens(w, 1)[0]
    g = {k: v.cuda().contiguous() for k, v in tk.items()}
    o = torch.empty_like(g["q"])
    hla.hla_decode_step(hla.make_config(1, 1, 1, 64, 64, "f32", "routed", 1.0, -2.0, 0.05), cache,
                        g["q"], g["k"], g["v"], g["alpha"], g["beta"], o)
    st, code = hla.hla_device_status(clear=True)
    assert st == hla.HLA_ERR_WORKSPACE and code & 4
    st, code = hla.hla_device_status(clear=True)
    assert st == 0 and code == 0


def test_full_size_decode_sampled(hla):
    """The 32K decode step at full size (64 sequences x 32768-token contexts, 512
    cached chunks per head, H=16, d=128, bf16, threshold 0.05): the cache is built
    as bench.py builds it, one decode step runs over all sequences, and two
    (sequence, head) outputs are compared with the oracle's decode head built from
    the same context (definition form: forward composition over all 512 chunks)."""
    import os
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    w = syn.DECODE_32K
    max_chunks = w.T // w.C + 1
    cache, ctx = bench.build_decode_cache(hla, syn, torch, w, max_chunks, group=8)
    try:
        dcfg = hla.make_config(w.B, w.H, 1, w.C, w.d, w.dtype, w.gate_mode, w.tau, w.bias, w.thr)
        tok = syn.make_decode_tokens(w, 1)[0]
        g = {k: v.cuda().contiguous() for k, v in tok.items()}
        o = torch.empty_like(g["q"])
        hla.hla_decode_step(dcfg, cache, g["q"], g["k"], g["v"], g["alpha"], g["beta"], o)
        torch.cuda.synchronize()
        st, code = hla.hla_device_status()
        assert st == hla.HLA_OK, code
        n = cache.view("n_chunks", (w.B,), torch.int32).cpu()
        m = cache.view("m_partial", (w.B,), torch.int32).cpu()
        assert torch.all(n == w.T // w.C) and torch.all(m == 1)
        for (b, h) in ((0, 0), (1, 9)):
            f = lambda name: P.np64(ctx[name][b, :, h])
            head = ho.HlaDecodeHead.from_prefill(f("q"), f("k"), f("v"), f("alpha"), f("beta"), w.C, w.tau,
                                                 w.bias, w.thr, w.gate_mode)
            ref = head.step(P.np64(tok["q"][b, h]), P.np64(tok["k"][b, h]), P.np64(tok["v"][b, h]),
                            float(tok["alpha"][b, h]), float(tok["beta"][b, h]))
            P.check_bf16(P.np64(o[b, h]), ref)
    finally:
        del cache
        torch.cuda.empty_cache()


def test_full_size_planted_decode_sampled(hla):
    """The planted 32K decode step at full size (64 sequences x 32768-token contexts,
    H=16, d=128, bf16, bias -4, threshold 0.05, planted route inputs: the open chunk
    matches about 4 of the 512 cached chunks).  The step's active lists are read
    from the decode workspace (pre-filled with a sentinel, so the entries the kernel
    wrote are exactly the active ones) and must equal the oracle's, with bit-exact
    gates; sampled (sequence, head) outputs are compared with the oracle's decode
    head built from the same context (forward composition over the active chunks)."""
    import os
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    w = syn.DECODE_32K_PLANTED
    max_chunks = w.T // w.C + 1
    cache, ctx = bench.build_decode_cache(hla, syn, torch, w, max_chunks, group=8)
    try:
        dcfg = hla.make_config(w.B, w.H, 1, w.C, w.d, w.dtype, w.gate_mode, w.tau, w.bias, w.thr)
        tok = syn.make_decode_tokens(w, 1)[0]
        g = {k: v.cuda().contiguous() for k, v in tok.items()}
        o = torch.empty_like(g["q"])
        nbytes = hla.decode_workspace_bytes(dcfg, max_chunks)
        ws = torch.full((nbytes // 4,), -7, dtype=torch.int32, device="cuda")
        hla.hla_decode_step(dcfg, cache, g["q"], g["k"], g["v"], g["alpha"], g["beta"], o,
                            q_route=g["q_route"], k_route=g["k_route"], workspace=ws)
        torch.cuda.synchronize()
        st, code = hla.hla_device_status()
        assert st == hla.HLA_OK, code
        n = w.B * w.H * max_chunks
        g_off = ((n * 4 + 255) // 256) * 256 // 4
        idx = ws[:n].view(w.B, w.H, max_chunks).cpu()
        gts = ws[g_off:g_off + n].view(torch.float32).view(w.B, w.H, max_chunks).cpu()
        counts = (idx != -7).sum(-1)
        assert 1.0 <= counts.float().mean() <= 12.0, counts.float().mean()
        for (b, h) in ((0, 0), (1, 9), (0, 15)):
            f = lambda name: P.np64(ctx[name][b, :, h])
            r32 = lambda name: P.np32(ctx[name][b, :, h])
            head = ho.HlaDecodeHead.from_prefill(f("q"), f("k"), f("v"), f("alpha"), f("beta"), w.C, w.tau,
                                                 w.bias, w.thr, w.gate_mode, r32("q_route"), r32("k_route"))
            ref = head.step(P.np64(tok["q"][b, h]), P.np64(tok["k"][b, h]), P.np64(tok["v"][b, h]),
                            float(tok["alpha"][b, h]), float(tok["beta"][b, h]),
                            P.np32(tok["q_route"][b, h]), P.np32(tok["k_route"][b, h]))
            P.check_bf16(P.np64(o[b, h]), ref, "planted decode output")
            # the oracle's gates of this step: its open chunk now holds the new token
            g_ref = head.gates()
            act_ref = head.active(g_ref)
            c = int(counts[b, h])
            assert idx[b, h, :c].tolist() == [int(j) for j in act_ref]
            assert np.array_equal(gts[b, h, :c].numpy().view(np.uint32),
                                  np.asarray(g_ref[act_ref], np.float32).view(np.uint32))
    finally:
        del cache
        torch.cuda.empty_cache()
