"""Edge cases of the chunk-size, window and decay options against the oracle:
prompts shorter than one 64-token sub-chunk, caller-given and all-zero gates with
long chunks, windows on the float32 path, and decoding from an empty cache."""
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


def _prefill_vs_oracle(hla, w, user_gates=None):
    inp = P.gpu_inputs(w)
    o, gates, aidx, acnt = P.run_prefill(hla, w, inp, user_gates=user_gates) if user_gates is not None \
        else P.run_prefill(hla, w, inp)
    B, T, H, _ = inp["q"].shape
    ref = np.zeros(tuple(inp["v"].shape))
    for b in range(B):
        for h in range(H):
            r = P.oracle_prefill_head(w, inp, b, h, user_gates=user_gates)
            ref[b, :, h] = r.o
            P.check_routing_exact(r, gates, aidx, acnt, b, h)
    got = P.np64(o)
    if w.dtype == "f32":
        P.check_f32(got, ref)
    else:
        P.check_bf16(got, ref, layout="bthd")
    st, code = hla.hla_device_status()
    assert st == 0 and code == 0


@pytest.mark.parametrize("T,dtype,d", [(40, "bf16", 128), (1, "bf16", 128), (50, "f32", 64)])
def test_prompt_shorter_than_a_sub_chunk_c256(hla, T, dtype, d):
    _prefill_vs_oracle(hla, syn.PREFILL_0P8B.with_(B=2, H=2, T=T, C=256, dtype=dtype, d=d))


def test_user_gates_c256(hla):
    w = syn.PREFILL_0P8B.with_(B=1, H=2, T=256 * 4 + 70, C=256, gate_mode="user", thr=0.3)
    _prefill_vs_oracle(hla, w, user_gates=syn.make_user_gates(w))


def test_zero_gates_c128_windows(hla):
    _prefill_vs_oracle(hla, syn.PREFILL_0P8B.with_(B=1, H=2, T=128 * 3 + 9, C=128, gate_mode="zero", window=32))


def test_f32_windows_d64_c128(hla):
    _prefill_vs_oracle(hla, syn.PREFILL_0P8B.with_(B=1, H=2, T=128 * 4 + 17, C=128, dtype="f32", d=64,
                                                   window=16, thr=0.2))


def test_decode_from_an_empty_cache_c256_windows(hla):
    """No prefill: 260 decode steps from an empty cache at C = 256 with window-32
    representatives close the first chunk by the token rule and go on past it."""
    C, d, steps = 256, 128, 260
    w = syn.DECODE_32K.with_(B=1, H=2, T=1, C=C, thr=0.05, bias=-0.5, window=32)
    cfg = hla.make_config(w.B, w.H, 1, C, d, "bf16", "routed", w.tau, w.bias, w.thr, pool_window=32)
    cache = hla.Cache(cfg, max_chunks=3)
    heads = {(0, h): ho.HlaDecodeHead(C, d, d, w.tau, w.bias, w.thr, pool_window=32) for h in range(w.H)}
    got, ref = [], []
    for tk in syn.make_decode_tokens(w, steps):
        g = {k: v.cuda().contiguous() for k, v in tk.items()}
        o = torch.empty_like(g["q"])
        hla.hla_decode_step(cfg, cache, g["q"], g["k"], g["v"], g["alpha"], g["beta"], o)
        o = P.np64(o)
        for (b, h), st in heads.items():
            ref.append(st.step(P.np64(tk["q"][b, h]), P.np64(tk["k"][b, h]), P.np64(tk["v"][b, h]),
                               float(tk["alpha"][b, h]), float(tk["beta"][b, h])))
            got.append(o[b, h])
    torch.cuda.synchronize()
    P.check_bf16(np.stack(got), np.stack(ref), layout="steps", nh=len(heads))
    n = cache.view("n_chunks", (1,), torch.int32).cpu()
    m = cache.view("m_partial", (1,), torch.int32).cpu()
    assert n.tolist() == [1] and m.tolist() == [steps - C]
    st, code = hla.hla_device_status()
    assert st == 0 and code == 0
