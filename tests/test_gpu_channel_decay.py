"""GPU parity with channel-wise decay (a decay per key channel, the KDA-style decay
named in the Gated DeltaNet-2 abstract on the HLA listing page):
  S_t = S_{t-1} Diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T.

With bf16 and d = 128 the prefill runs on the tensor cores (the decays folded into
prepared keys and queries per 64-token sub-chunk); with float32 or d = 64, and in
gdn_chunk_transitions and the decode close, the transitions and read-out run the token
rule row by row on CUDA cores.  The composition and the gates are those of the scalar
path.  Bars as elsewhere: gates and lists bit-exact, outputs max-abs 1e-4 (float32) or
relative L2 2e-2 (bf16) per head; bf16 transitions relative L2 1e-2 per matrix."""
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
    assert inp["alpha"].dim() == 4
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


@pytest.mark.parametrize("C,T,thr", [(64, 64 * 6 + 21, 0.0), (256, 256 * 3 + 100, 0.3), (128, 128 * 4, 0.0)])
def test_bf16_channel_decay_prefill(hla, C, T, thr):
    _check_prefill(hla, syn.PREFILL_0P8B.with_(B=2, H=2, T=T, C=C, thr=thr, decay="channel"))


def test_f32_channel_decay_prefill_planted(hla):
    w = syn.SPARSE_LONG.with_(B=1, H=2, T=64 * 12 + 7, dtype="f32", d=64, topics=3, decay="channel")
    _check_prefill(hla, w)


@pytest.mark.parametrize("dtype,d", [("f32", 64), ("bf16", 128)])
def test_channel_decay_gates_one_is_the_token_rule(hla, dtype, d):
    w = syn.GDN_REDUCTION.with_(B=2, H=2, T=64 * 4 + 9, dtype=dtype, d=d, decay="channel")
    inp = P.gpu_inputs(w)
    o, *_ = P.run_prefill(hla, w, inp)
    for b in range(2):
        for h in range(2):
            ref, _ = ho.gdn_recurrent(P.np64(inp["q"][b, :, h]), P.np64(inp["k"][b, :, h]),
                                      P.np64(inp["v"][b, :, h]), P.np64(inp["alpha"][b, :, h]),
                                      P.np64(inp["beta"][b, :, h]))
            got = P.np64(o[b, :, h])
            if dtype == "f32":
                P.check_f32(got, ref)
            else:
                P.check_bf16(got, ref)


@pytest.mark.parametrize("dtype,d,C", [
    ("f32", 64, 64),
    ("f32", 128, 128),    # d = 128: four rows per group of eight threads, G = 32
    ("bf16", 128, 64),
    ("bf16", 128, 256),   # the decode close and gdn_chunk_transitions at C > 64
])
def test_channel_decay_transitions(hla, dtype, d, C):
    """A_c and B_c of every chunk, one by one, against the oracle's literal token-rule
    transition (not only through gated outputs, where small gates dilute an error)."""
    w = syn.TINY_F32.with_(B=1, H=2, T=C * 2 + 5, C=C, dtype=dtype, d=d, decay="channel")
    inp = P.gpu_inputs(w)
    B, H, T = 1, 2, w.T
    cfg = hla.make_config(B, H, T, C, d, dtype, decay="channel")
    g = P.to_cuda(inp)
    A = torch.empty((B, H, T // C, d, d), dtype=syn.torch_dtype(w), device="cuda")
    Bm = torch.empty_like(A)
    hla.gdn_chunk_transitions(cfg, g["k"], g["v"], g["alpha"], g["beta"], A, Bm)
    torch.cuda.synchronize()
    A, Bm = P.np64(A), P.np64(Bm)
    for h in range(H):
        for c in range(T // C):
            sl = slice(C * c, C * c + C)
            Ar, Br = ho.chunk_transition(P.np64(inp["k"][0, sl, h]), P.np64(inp["v"][0, sl, h]),
                                         P.np64(inp["alpha"][0, sl, h]), P.np64(inp["beta"][0, sl, h]))
            if dtype == "f32":
                P.check_f32(A[0, h, c], Ar, "transition")
                P.check_f32(Bm[0, h, c], Br, "transition")
            else:
                P.check_bf16(A[0, h, c], Ar, "transition", tol=1e-2)
                P.check_bf16(Bm[0, h, c], Br, "transition", tol=1e-2)


@pytest.mark.parametrize("dtype,d,C,T0,steps", [
    ("f32", 64, 64, 64 * 3 + 60, 7),      # CUDA-core decode, closes a chunk at step 4
    ("bf16", 128, 64, 64 * 2 + 62, 5),    # TMA-streamed decode, closes at step 2
    ("bf16", 128, 128, 128 + 126, 4),     # 128-token chunks
])
def test_channel_decay_decode(hla, dtype, d, C, T0, steps):
    w = syn.DECODE_32K.with_(B=2, H=2, T=T0, C=C, dtype=dtype, d=d, thr=0.05, decay="channel")
    inp = P.gpu_inputs(w)
    maxc = T0 // C + 2
    cfg = hla.make_config(w.B, w.H, T0, C, d, dtype, "routed", w.tau, w.bias, w.thr, decay="channel")
    cache = hla.Cache(cfg, max_chunks=maxc)
    P.run_prefill(hla, w, inp, cache=cache)
    heads = {}
    for b in range(w.B):
        for h in range(w.H):
            f = lambda n: inp[n][b, :, h]
            heads[(b, h)] = ho.HlaDecodeHead.from_prefill(
                P.np64(f("q")), P.np64(f("k")), P.np64(f("v")), P.np64(f("alpha")), P.np64(f("beta")), C,
                w.tau, w.bias, w.thr)
    dcfg = hla.make_config(w.B, w.H, 1, C, d, dtype, "routed", w.tau, w.bias, w.thr, decay="channel")
    got, ref = [], []
    for tk in syn.make_decode_tokens(w, steps):
        assert tk["alpha"].shape == (w.B, w.H, d)
        gt = {k: v.cuda().contiguous() for k, v in tk.items()}
        o = torch.empty_like(gt["q"])
        hla.hla_decode_step(dcfg, cache, gt["q"], gt["k"], gt["v"], gt["alpha"], gt["beta"], o)
        torch.cuda.synchronize()
        o = P.np64(o)
        for (b, h), st in heads.items():
            ref.append(st.step(P.np64(tk["q"][b, h]), P.np64(tk["k"][b, h]), P.np64(tk["v"][b, h]),
                               P.np64(tk["alpha"][b, h]), float(tk["beta"][b, h])))
            got.append(o[b, h])
    got, ref = np.stack(got), np.stack(ref)
    if dtype == "f32":
        P.check_f32(got, ref)
    else:
        P.check_bf16(got, ref, layout="steps", nh=len(heads))
    st, code = hla.hla_device_status()
    assert st == 0 and code == 0
    n = cache.view("n_chunks", (w.B,), torch.int32).cpu()
    assert n.tolist() == [(T0 + steps) // C] * w.B


def test_full_size_channel_decay_sampled(hla):
    """Dense 0.8B-like layer at full size (T=16384, H=16, d=128, bf16) with a decay
    per key channel: gates bit-exact on two heads, sampled query chunks against the
    oracle."""
    w = syn.PREFILL_0P8B.with_(decay="channel")
    inp = P.gpu_inputs(w)
    o, gates, aidx, acnt = P.run_prefill(hla, w, inp)
    for h in (0, 9):
        sample = [0, 1, 37, 128, 255]
        r = P.oracle_prefill_head(w, inp, 0, h, query_chunks=sample)
        P.check_routing_exact(r, gates, aidx, acnt, 0, h)
        rows = np.concatenate([np.arange(64 * i, 64 * i + 64) for i in sample])
        P.check_bf16(P.np64(o[0, rows, h]), r.o[rows])


def test_bf16_d64_channel_decay(hla):
    """bf16 storage with d = 64 (CUDA-core composition, float32 states read by the
    token-rule read-out)."""
    _check_prefill(hla, syn.PREFILL_0P8B.with_(B=1, H=2, T=64 * 5 + 33, d=64, thr=0.2, decay="channel"))


@pytest.mark.parametrize("C,T", [(64, 64 * 5 + 7), (256, 256 * 2 + 64 + 3)])
def test_channel_decay_tensor_core_cache_transitions(hla, C, T):
    """The A_c, B_c that a bf16, d = 128 prefill with a decay per channel writes into a
    dense cache (tensor-core transitions of the 64-token sub-chunks, merged at C > 64),
    chunk by chunk against the oracle's literal token-rule transition."""
    w = syn.PREFILL_0P8B.with_(B=1, H=2, T=T, C=C, decay="channel")
    inp = P.gpu_inputs(w)
    cfg = hla.make_config(1, 2, T, C, 128, "bf16", "routed", w.tau, w.bias, w.thr, decay="channel")
    cache = hla.Cache(cfg, max_chunks=T // C + 1)
    P.run_prefill(hla, w, inp, cache=cache)
    st, code = hla.hla_device_status()
    assert st == 0 and code == 0
    n = T // C
    # the closed chunks' slots only (the slot after them has not been written)
    A = P.np64(cache.view("A", (1, 2, n + 1, 128, 128), torch.bfloat16)[:, :, :n])
    Bm = P.np64(cache.view("Bm", (1, 2, n + 1, 128, 128), torch.bfloat16)[:, :, :n])
    for h in range(2):
        for c in range(n):
            sl = slice(C * c, C * c + C)
            Ar, Br = ho.chunk_transition(P.np64(inp["k"][0, sl, h]), P.np64(inp["v"][0, sl, h]),
                                         P.np64(inp["alpha"][0, sl, h]), P.np64(inp["beta"][0, sl, h]))
            P.check_bf16(A[0, h, c], Ar, "transition", tol=1e-2)
            P.check_bf16(Bm[0, h, c], Br, "transition", tol=1e-2)
