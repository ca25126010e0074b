"""GPU parity at chunk sizes C = 128 and 256 (the pages' default chunk is 256 tokens,
HLA summary page, "Main Findings", chunk-size ablation).

The library works on 64-token sub-chunks: their WY transitions are merged into the
chunk's transition, the composition runs over chunks, and the composed state is
advanced to every sub-chunk for the read-out.  The oracle knows nothing of
sub-chunks: it pools, gates, composes and reads out over chunks of C tokens by the
definition.  Bars as elsewhere: gates and active lists bit-exact, outputs max-abs
1e-4 (float32 path) or relative L2 2e-2 (bf16 path)."""
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


def _check_prefill(hla, w, tol_f32=True):
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


# T values: several chunks plus a partial chunk that holds complete sub-chunks and a
# ragged one; exactly whole chunks; a prompt shorter than one chunk.
@pytest.mark.parametrize("C,T", [(128, 128 * 4 + 64 + 17), (256, 256 * 3), (256, 256 * 2 + 3 * 64 + 9), (256, 100)])
def test_bf16_tensor_core_spread(hla, C, T):
    _check_prefill(hla, syn.PREFILL_0P8B.with_(B=2, H=2, T=T, C=C))


@pytest.mark.parametrize("C,T", [(128, 128 * 5 + 70), (256, 256 * 2 + 130)])
def test_f32_cuda_core_thresholded(hla, C, T):
    w = syn.SPARSE_LONG.with_(B=1, H=2, T=T, C=C, dtype="f32", d=64, topics=3)
    _check_prefill(hla, w)


def test_bf16_d64_cuda_core(hla):
    _check_prefill(hla, syn.PREFILL_0P8B.with_(B=1, H=2, T=128 * 3 + 40, C=128, d=64))


def test_bf16_planted_sparse_c256(hla):
    w = syn.SPARSE_LONG.with_(B=1, H=2, T=256 * 8 + 64, C=256, topics=3)
    _check_prefill(hla, w)


@pytest.mark.parametrize("dtype,C", [("f32", 128), ("bf16", 256), ("bf16", 128)])
def test_gates_one_is_native_gdn(hla, dtype, C):
    """All gates one (the prefix-scan composition over chunks) equals the plain
    sequential gated delta rule, whatever the chunk size."""
    d = 64 if dtype == "f32" else 128
    w = syn.GDN_REDUCTION.with_(B=2, H=2, T=C * 3 + 64 + 9, C=C, dtype=dtype, d=d)
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


@pytest.mark.parametrize("dtype,d,C", [("f32", 64, 128), ("bf16", 128, 256)])
def test_gdn_chunk_transitions_long(hla, dtype, d, C):
    w = syn.TINY_F32.with_(dtype=dtype, d=d, B=1, H=2, T=C * 2 + 11, C=C)
    inp = P.gpu_inputs(w)
    B, H, T = 1, 2, w.T
    cfg = hla.make_config(B, H, T, C, d, dtype)
    g = P.to_cuda(inp)
    tdt = syn.torch_dtype(w)
    A = torch.empty((B, H, T // C, d, d), dtype=tdt, device="cuda")
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
                P.check_f32(A[0, h, c], Ar)
                P.check_f32(Bm[0, h, c], Br)
            else:
                P.check_bf16(A[0, h, c], Ar, "transition", tol=1e-2)
                P.check_bf16(Bm[0, h, c], Br, "transition", tol=1e-2)


@pytest.mark.parametrize("dtype,d,C,T0,steps", [
    ("f32", 64, 128, 128 * 2 + 120, 10),   # closes chunk 2 at step 8
    ("bf16", 128, 128, 128 * 3 + 123, 7),  # closes chunk 3 at step 5
    ("bf16", 128, 256, 256 + 250, 9),      # closes chunk 1 at step 6
])
def test_decode_long_chunks(hla, dtype, d, C, T0, steps):
    """Prefill into a dense cache (chunk transitions merged from sub-chunks straight
    into the cache), then decode steps that close a chunk by the token rule."""
    w = syn.DECODE_32K.with_(B=2, H=2, T=T0, C=C, dtype=dtype, d=d, thr=0.05)
    inp = P.gpu_inputs(w)
    maxc = T0 // C + 2
    cfg = hla.make_config(w.B, w.H, T0, C, d, dtype, "routed", w.tau, w.bias, w.thr)
    cache = hla.Cache(cfg, max_chunks=maxc)
    P.run_prefill(hla, w, inp, cache=cache)
    heads = {}
    for b in range(w.B):
        for h in range(w.H):
            f = lambda n: inp[n][b, :, h]
            heads[(b, h)] = ho.HlaDecodeHead.from_prefill(
                P.np64(f("q")), P.np64(f("k")), P.np64(f("v")), P.np64(f("alpha")), P.np64(f("beta")), C,
                w.tau, w.bias, w.thr)
    dcfg = hla.make_config(w.B, w.H, 1, C, d, dtype, "routed", w.tau, w.bias, w.thr)
    got, ref = [], []
    for tk in syn.make_decode_tokens(w, steps):
        g = {k: v.cuda().contiguous() for k, v in tk.items()}
        o = torch.empty_like(g["q"])
        hla.hla_decode_step(dcfg, cache, g["q"], g["k"], g["v"], g["alpha"], g["beta"], o)
        torch.cuda.synchronize()
        o = P.np64(o)
        for (b, h), st in heads.items():
            ref.append(st.step(P.np64(tk["q"][b, h]), P.np64(tk["k"][b, h]), P.np64(tk["v"][b, h]),
                               float(tk["alpha"][b, h]), float(tk["beta"][b, h])))
            got.append(o[b, h])
    got, ref = np.stack(got), np.stack(ref)
    if dtype == "f32":
        P.check_f32(got, ref)
    else:
        P.check_bf16(got, ref, layout="steps", nh=len(heads))
    st, code = hla.hla_device_status()
    assert st == 0 and code == 0
    n = cache.view("n_chunks", (w.B,), torch.int32).cpu()
    m = cache.view("m_partial", (w.B,), torch.int32).cpu()
    assert n.tolist() == [(T0 + steps) // C] * w.B and m.tolist() == [(T0 + steps) % C] * w.B
    rk = cache.view("rk", (w.B, w.H, maxc, d), torch.float32).cpu().numpy()
    for (b, h), st_ in heads.items():
        for j in range(len(st_.rk)):
            assert np.array_equal(rk[b, h, j].view(np.uint32), st_.rk[j].view(np.uint32))


def test_full_size_c256_window32_sampled(hla):
    """The pages' defaults at the dense 0.8B-like layer's full size (T=16384, H=16,
    d=128, bf16, 256-token chunks, window-32 representatives): all gates and active
    lists bit-exact on two heads; sampled query chunks against the oracle."""
    w = syn.PREFILL_0P8B.with_(C=256, window=32)
    inp = P.gpu_inputs(w)
    o, gates, aidx, acnt = P.run_prefill(hla, w, inp)
    for h in (0, 9):
        sample = [0, 1, 17, 40, 63]
        r = P.oracle_prefill_head(w, inp, 0, h, query_chunks=sample)
        P.check_routing_exact(r, gates, aidx, acnt, 0, h)
        rows = np.concatenate([np.arange(256 * i, 256 * i + 256) for i in sample])
        P.check_bf16(P.np64(o[0, rows, h]), r.o[rows])
