"""hla_decode_step_static (scratch in the library's fixed device array) against
hla_decode_step (caller workspace), through the C ABI.

Two caches start from the same prefill (the second is a byte copy of the first);
each then takes the same two decode tokens, one entry point per cache.  The first
token fills the open chunk, so that step also closes it into the cache; the second
opens the next chunk.  Outputs must agree within the parity tolerances, and the
cache counters exactly; around the second static call the device's free memory and
torch's allocated bytes must not move.  The file is named to be collected last, and it also
passes alone in a fresh process (the first call on the device does the set-up)."""
import pytest
import torch

import hla_synth as syn
from tests import _parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hla():
    import gated_delta_rule_transitions_b200 as m
    m.lib()
    return m._hla


@pytest.mark.parametrize("dtype,d,mode,thr,route", [
    ("bf16", 128, "routed", 0.05, True),
    ("f32", 64, "routed", 0.3, False),
    ("bf16", 128, "one", 0.0, False),
])
def test_static_scratch_decode_matches_workspace_decode(hla, dtype, d, mode, thr, route):
    T0 = 64 * 3 + 63
    w = syn.DECODE_32K.with_(B=3, H=2, T=T0, dtype=dtype, d=d, gate_mode=mode, thr=thr,
                             route="spread" if route else "default", bias=-0.5 if route else -2.0)
    inp = P.gpu_inputs(w)
    cfg = hla.make_config(w.B, w.H, T0, 64, d, dtype, mode, w.tau, w.bias, w.thr)
    ref_cache = hla.Cache(cfg, max_chunks=6)
    P.run_prefill(hla, w, inp, cache=ref_cache)
    st_cache = hla.Cache(cfg, max_chunks=6)
    st_cache.mem.copy_(ref_cache.mem)
    torch.cuda.synchronize()

    dcfg = hla.make_config(w.B, w.H, 1, 64, d, dtype, mode, w.tau, w.bias, w.thr)
    toks = syn.make_decode_tokens(w, 2)
    gen = torch.Generator().manual_seed(5)
    for step, tk in enumerate(toks):
        g = {k: v.cuda().contiguous() for k, v in tk.items()}
        qr = kr = None
        if route:
            mu = torch.randn((w.B, w.H, d), generator=gen) * 1.4
            qr = mu.to(g["q"].dtype).cuda()
            kr = (mu + 0.3 * torch.randn((w.B, w.H, d), generator=gen)).to(g["q"].dtype).cuda()
        o_ref = torch.empty_like(g["q"])
        o_st = torch.empty_like(g["q"])
        hla.hla_decode_step(dcfg, ref_cache, g["q"], g["k"], g["v"], g["alpha"], g["beta"], o_ref,
                            q_route=qr, k_route=kr)
        torch.cuda.synchronize()
        before = (torch.cuda.memory_allocated(), torch.cuda.mem_get_info()[0])
        hla.hla_decode_step_static(dcfg, st_cache, g["q"], g["k"], g["v"], g["alpha"], g["beta"], o_st,
                                   q_route=qr, k_route=kr)
        torch.cuda.synchronize()
        after = (torch.cuda.memory_allocated(), torch.cuda.mem_get_info()[0])
        if step > 0:
            # past the set-up of the first call in this process: no device memory
            # taken by torch's allocator or by any other allocation on the device
            assert after == before, (before, after)
        a, b = P.np64(o_st), P.np64(o_ref)
        if dtype == "f32":
            P.check_f32(a, b, "static vs workspace decode")
        else:
            P.check_bf16(a, b, "static vs workspace decode", layout="bhd")
    for field in ("n_chunks", "m_partial"):
        got = st_cache.view(field, (w.B,), torch.int32).cpu()
        ref = ref_cache.view(field, (w.B,), torch.int32).cpu()
        assert torch.equal(got, ref)
    assert int(ref_cache.view("n_chunks", (w.B,), torch.int32)[0]) == 4
    st, code = hla.hla_device_status()
    assert st == hla.HLA_OK, code
