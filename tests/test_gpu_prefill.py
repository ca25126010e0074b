"""GPU parity of the prefill path against the oracle (through the C ABI).

Bars: gates and active lists bit-exact; outputs max-abs <= 1e-4 on the float32 path
and relative L2 <= 2e-2 on the bf16 path (over the whole output tensor)."""
import numpy as np
import pytest
import torch

import hla_synth as syn
from oracle import hla_oracle as ho
from oracle import routing_recipe as rr
from tests import _parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hla():
    import gated_delta_rule_transitions_b200 as m
    m.lib()
    return m._hla


def _oracle_all(w, inp, user_gates=None):
    B, T, H, _ = inp["q"].shape
    o = np.zeros(tuple(inp["v"].shape), np.float64)
    res = {}
    for b in range(B):
        for h in range(H):
            r = P.oracle_prefill_head(w, inp, b, h, user_gates)
            o[b, :, h] = r.o
            res[(b, h)] = r
    return o, res


def test_tiny_f32_prefill(hla):
    w = syn.TINY_F32
    inp = P.gpu_inputs(w)
    o, gates, aidx, acnt = P.run_prefill(hla, w, inp)
    ref, res = _oracle_all(w, inp)
    P.check_f32(P.np64(o), ref)
    for (b, h), r in res.items():
        P.check_routing_exact(r, gates, aidx, acnt, b, h)


@pytest.mark.parametrize("T", [64 * 5, 64 * 5 + 17, 40])
def test_bf16_spread_gates_ragged(hla, T):
    w = syn.PREFILL_0P8B.with_(B=2, H=2, T=T)
    inp = P.gpu_inputs(w)
    o, gates, aidx, acnt = P.run_prefill(hla, w, inp)
    ref, res = _oracle_all(w, inp)
    P.check_bf16(P.np64(o), ref, layout="bthd")
    for (b, h), r in res.items():
        P.check_routing_exact(r, gates, aidx, acnt, b, h)
    g = np.concatenate([r.gates[np.tril_indices(r.gates.shape[0], -1)] for r in res.values()])
    if g.size > 10:
        assert g.min() < 0.2 and g.max() > 0.5  # spread over (0, 1)


def test_f32_routed_thresholded(hla):
    w = syn.SPARSE_LONG.with_(B=1, H=2, T=64 * 12, dtype="f32", d=64, topics=3)
    inp = P.gpu_inputs(w)
    o, gates, aidx, acnt = P.run_prefill(hla, w, inp)
    ref, res = _oracle_all(w, inp)
    P.check_f32(P.np64(o), ref)
    skipped = 0
    for (b, h), r in res.items():
        P.check_routing_exact(r, gates, aidx, acnt, b, h)
        skipped += sum(i - len(a) for i, a in enumerate(r.active))
    assert skipped > 0


def test_bf16_planted_sparse(hla):
    w = syn.SPARSE_LONG.with_(B=1, H=2, T=64 * 20, topics=4)
    inp = P.gpu_inputs(w)
    o, gates, aidx, acnt = P.run_prefill(hla, w, inp)
    ref, res = _oracle_all(w, inp)
    P.check_bf16(P.np64(o), ref, layout="bthd")
    for (b, h), r in res.items():
        P.check_routing_exact(r, gates, aidx, acnt, b, h)
        kept = [len(a) for a in r.active]
        assert 0 < sum(kept) < sum(range(len(kept)))


def test_bf16_planted_sparse_odd_chunks(hla):
    """Skipping with an odd number of query chunks (one unpaired chain in the pairing
    order), several sequences and heads, and a ragged last chunk."""
    w = syn.SPARSE_LONG.with_(B=2, H=3, T=64 * 20 + 5, topics=5)
    inp = P.gpu_inputs(w)
    o, gates, aidx, acnt = P.run_prefill(hla, w, inp)
    ref, res = _oracle_all(w, inp)
    P.check_bf16(P.np64(o), ref, layout="bthd")
    skipped = 0
    for (b, h), r in res.items():
        P.check_routing_exact(r, gates, aidx, acnt, b, h)
        skipped += sum(i - len(a) for i, a in enumerate(r.active))
    assert skipped > 0


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_gates_one_is_native_gdn(hla, dtype):
    w = syn.GDN_REDUCTION.with_(B=2, H=2, T=64 * 4 + 9, dtype=dtype, d=64 if dtype == "f32" else 128)
    inp = P.gpu_inputs(w)
    o, gates, aidx, acnt = P.run_prefill(hla, w, inp)
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


def test_gates_zero_is_intra_chunk_only(hla):
    w = syn.TINY_F32.with_(gate_mode="zero", T=64 * 3 + 5)
    inp = P.gpu_inputs(w)
    o, *_ = P.run_prefill(hla, w, inp)
    for h in range(2):
        for c in range(4):
            sl = slice(64 * c, min(64 * c + 64, w.T))
            ref, _ = ho.gdn_recurrent(P.np64(inp["q"][0, sl, h]), P.np64(inp["k"][0, sl, h]),
                                      P.np64(inp["v"][0, sl, h]), P.np64(inp["alpha"][0, sl, h]),
                                      P.np64(inp["beta"][0, sl, h]))
            P.check_f32(P.np64(o[0, sl, h]), ref)


def test_identity_tokens_give_zero_output(hla):
    w = syn.TINY_F32
    inp = P.gpu_inputs(w)
    inp["alpha"] = torch.ones_like(inp["alpha"])
    inp["beta"] = torch.zeros_like(inp["beta"])
    o, *_ = P.run_prefill(hla, w, inp)
    assert torch.count_nonzero(o) == 0


def test_user_gates(hla):
    w = syn.TINY_F32.with_(gate_mode="user", thr=0.3)
    inp = P.gpu_inputs(w)
    ug = syn.make_user_gates(w)
    o, gates, aidx, acnt = P.run_prefill(hla, w, inp, user_gates=ug)
    ref, res = _oracle_all(w, inp, user_gates=ug)
    P.check_f32(P.np64(o), ref)
    for (b, h), r in res.items():
        P.check_routing_exact(r, gates, aidx, acnt, b, h)


@pytest.mark.parametrize("dtype,d", [("f32", 64), ("f32", 128), ("bf16", 128), ("bf16", 64)])
def test_gdn_chunk_transitions(hla, dtype, d):
    w = syn.TINY_F32.with_(dtype=dtype, d=d, B=2, H=3, T=64 * 3 + 11)
    inp = P.gpu_inputs(w)
    B, T, H = 2, w.T, 3
    cfg = hla.make_config(B, H, T, 64, d, dtype)
    g = P.to_cuda(inp)
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    A = torch.empty((B, H, T // 64, d, d), dtype=tdt, device="cuda")
    Bm = torch.empty_like(A)
    hla.gdn_chunk_transitions(cfg, g["k"], g["v"], g["alpha"], g["beta"], A, Bm)
    torch.cuda.synchronize()
    A, Bm = P.np64(A), P.np64(Bm)
    for b in range(B):
        for h in range(H):
            for c in range(T // 64):
                sl = slice(64 * c, 64 * c + 64)
                Ar, Br = ho.chunk_transition(P.np64(inp["k"][b, sl, h]), P.np64(inp["v"][b, sl, h]),
                                             P.np64(inp["alpha"][b, sl, h]), P.np64(inp["beta"][b, sl, h]))
                if dtype == "f32":
                    P.check_f32(A[b, h, c], Ar)
                    P.check_f32(Bm[b, h, c], Br)
                else:
                    # bf16 operands and storage: relative L2 per matrix well inside the
                    # output tolerance
                    P.check_bf16(A[b, h, c], Ar, "transition", tol=1e-2)
                    P.check_bf16(Bm[b, h, c], Br, "transition", tol=1e-2)


def test_gdn_chunk_transitions_many_heads(hla):
    """More chunks than persistent CTAs with few chunks per head (N = 3, 150 heads):
    every CTA steps through several (b, h) positions, wrapping across sequences."""
    w = syn.TINY_F32.with_(dtype="bf16", d=128, B=3, H=50, T=64 * 2 + 5)
    inp = P.gpu_inputs(w)
    B, H, T = 3, 50, w.T
    cfg = hla.make_config(B, H, T, 64, 128, "bf16")
    g = P.to_cuda(inp)
    A = torch.empty((B, H, T // 64, 128, 128), dtype=torch.bfloat16, device="cuda")
    Bm = torch.empty_like(A)
    hla.gdn_chunk_transitions(cfg, g["k"], g["v"], g["alpha"], g["beta"], A, Bm)
    torch.cuda.synchronize()
    A, Bm = P.np64(A), P.np64(Bm)
    for b in range(B):
        for h in (0, 1, 17, H - 1):
            for c in range(T // 64):
                sl = slice(64 * c, 64 * c + 64)
                Ar, Br = ho.chunk_transition(P.np64(inp["k"][b, sl, h]), P.np64(inp["v"][b, sl, h]),
                                             P.np64(inp["alpha"][b, sl, h]), P.np64(inp["beta"][b, sl, h]))
                P.check_bf16(A[b, h, c], Ar, "transition", tol=1e-2)
                P.check_bf16(Bm[b, h, c], Br, "transition", tol=1e-2)


def test_gdn_chunk_transitions_strong_decay(hla):
    """Chunks whose accumulated decay exceeds e^80 (the pair decays then come from one
    exponential per pair, not from per-token factors) next to weakly decaying ones.
    Where the chunk's decay is beyond e^-60, A_c is of the order of gamma_C, at the
    bottom of the float32 / bf16 range, so A_c is checked in absolute terms there and
    B_c (of order one: the last tokens' keys barely decay) relatively."""
    w = syn.TINY_F32.with_(dtype="bf16", d=128, B=1, H=2, T=64 * 4)
    inp = P.gpu_inputs(w)
    gen = torch.Generator().manual_seed(77)
    # log alpha per chunk: about -0.05 (weak), -2 (|l| reaches about 128), -1.3 (about
    # 83 at the end of the chunk), and -40 on a single token of an otherwise weak chunk
    la = torch.empty(1, w.T, 2)
    la[:, 0:64] = -0.05
    la[:, 64:128] = -2.0
    la[:, 128:192] = -1.3
    la[:, 192:256] = -0.05
    la[:, 224] = -40.0
    la = la * (1.0 + 0.1 * torch.rand(la.shape, generator=gen))
    inp["alpha"] = torch.exp(la).float().contiguous()
    cfg = hla.make_config(1, 2, w.T, 64, 128, "bf16")
    g = P.to_cuda(inp)
    A = torch.empty((1, 2, w.T // 64, 128, 128), dtype=torch.bfloat16, device="cuda")
    Bm = torch.empty_like(A)
    hla.gdn_chunk_transitions(cfg, g["k"], g["v"], g["alpha"], g["beta"], A, Bm)
    torch.cuda.synchronize()
    A, Bm = P.np64(A), P.np64(Bm)
    for h in range(2):
        for c in range(w.T // 64):
            sl = slice(64 * c, 64 * c + 64)
            Ar, Br = ho.chunk_transition(P.np64(inp["k"][0, sl, h]), P.np64(inp["v"][0, sl, h]),
                                         P.np64(inp["alpha"][0, sl, h]), P.np64(inp["beta"][0, sl, h]))
            if -np.log(P.np64(inp["alpha"][0, sl, h])).sum() > 60.0:
                assert np.abs(A[0, h, c]).max() <= 1e-20 and np.abs(Ar).max() <= 1e-20
            else:
                P.check_bf16(A[0, h, c], Ar, "transition", tol=1e-2)
            P.check_bf16(Bm[0, h, c], Br, "transition", tol=1e-2)


@pytest.mark.parametrize("dtype,d,T", [("f32", 64, 64 * 7 + 3), ("bf16", 128, 64 * 9)])
def test_routing_bit_exact(hla, dtype, d, T):
    w = syn.PREFILL_0P8B.with_(B=2, H=3, T=T, dtype=dtype, d=d, thr=0.3)
    inp = P.gpu_inputs(w)
    B, H, N = 2, 3, (T + 63) // 64
    cfg = hla.make_config(B, H, T, 64, d, dtype, "routed", w.tau, w.bias, w.thr)
    g = P.to_cuda(inp)
    rq = torch.empty((B, H, N, d), device="cuda")
    rk = torch.empty_like(rq)
    gates = torch.empty((B, H, N, N), device="cuda")
    aidx = torch.empty((B, H, N, N), dtype=torch.int32, device="cuda")
    acnt = torch.empty((B, H, N), dtype=torch.int32, device="cuda")
    hla.hla_routing(cfg, g["q_route"], g["k_route"], rq, rk, gates, aidx, acnt)
    torch.cuda.synchronize()
    for b in range(B):
        for h in range(H):
            qr = P.np32(inp["q_route"][b, :, h])
            kr = P.np32(inp["k_route"][b, :, h])
            rq_ref = ho.route_pools(qr, 64, w.tau)
            rk_ref = ho.route_pools(kr, 64, w.tau)
            assert np.array_equal(rq[b, h].cpu().numpy().view(np.uint32), rq_ref.view(np.uint32))
            assert np.array_equal(rk[b, h].cpu().numpy().view(np.uint32), rk_ref.view(np.uint32))
            G = ho.gate_matrix(rq_ref, rk_ref, d, w.bias)
            act = ho.active_lists(G, w.thr)
            res = ho.HeadResult(o=None, gates=G, active=act, rq=rq_ref, rk=rk_ref)
            P.check_routing_exact(res, gates.cpu(), aidx.cpu(), acnt.cpu(), b, h)


@pytest.mark.parametrize("d,H,T,tau,scale", [
    # tau = 0.05 and large route values: pools whose shifted values fall below -86
    # (the exp's zero branch) and scores whose exp overflows or underflows
    (128, 3, 64 * 8 + 5, 0.05, 30.0),
    # enough 64-row gate tiles to fill the GPU at d = 64 (the 64-row kernel)
    (64, 37, 64 * 512, 1.0, 1.0),
    # several pool tiles per warp of the staged pool kernel, ending in a partial chunk
    (128, 4, 64 * 1000 + 17, 1.0, 1.0),
])
def test_routing_bit_exact_ranges(hla, d, H, T, tau, scale):
    gen = torch.Generator().manual_seed(123)
    N = (T + 63) // 64
    if scale > 1.0:
        # chunks of route keys around +scale or -scale (alternating), queries around
        # +scale: pooled scores of either sign and far beyond the exp's range
        sign = torch.where(torch.arange(T) // 64 % 2 == 0, 1.0, -1.0)[None, :, None, None]
        qr = (scale * (0.1 * torch.randn(1, T, H, d, generator=gen) + 1.0)).to(torch.bfloat16)
        kr = (scale * (0.1 * torch.randn(1, T, H, d, generator=gen) + sign)).to(torch.bfloat16)
    else:
        qr = torch.randn(1, T, H, d, generator=gen).to(torch.bfloat16)
        kr = torch.randn(1, T, H, d, generator=gen).to(torch.bfloat16)
    bias, thr = -1.0, 0.3
    cfg = hla.make_config(1, H, T, 64, d, "bf16", "routed", tau, bias, thr)
    rq = torch.empty((1, H, N, d), device="cuda")
    rk = torch.empty_like(rq)
    gates = torch.empty((1, H, N, N), device="cuda")
    aidx = torch.empty((1, H, N, N), dtype=torch.int32, device="cuda")
    acnt = torch.empty((1, H, N), dtype=torch.int32, device="cuda")
    hla.hla_routing(cfg, qr.cuda(), kr.cuda(), rq, rk, gates, aidx, acnt)
    torch.cuda.synchronize()
    for h in (0, H - 1):
        rq_ref = ho.route_pools(P.np32(qr[0, :, h]), 64, tau)
        rk_ref = ho.route_pools(P.np32(kr[0, :, h]), 64, tau)
        assert np.array_equal(rq[0, h].cpu().numpy().view(np.uint32), rq_ref.view(np.uint32))
        assert np.array_equal(rk[0, h].cpu().numpy().view(np.uint32), rk_ref.view(np.uint32))
        G = ho.gate_matrix(rq_ref, rk_ref, d, bias)
        if scale > 1.0:
            low = np.tril(np.ones_like(G, dtype=bool), -1)
            assert (G[low] == 0.0).any() and (G[low] == 1.0).any()  # both saturations reached
        res = ho.HeadResult(o=None, gates=G, active=ho.active_lists(G, thr), rq=rq_ref, rk=rk_ref)
        P.check_routing_exact(res, gates.cpu(), aidx.cpu(), acnt.cpu(), 0, h)


def test_full_size_prefill_sampled(hla):
    """Dense 0.8B-like layer (T=16384, H=16, d=128, bf16): all gates bit-exact on
    two heads; sampled query chunks against the oracle."""
    w = syn.PREFILL_0P8B
    inp = P.gpu_inputs(w)
    o, gates, aidx, acnt = P.run_prefill(hla, w, inp)
    for h in (0, 9):
        sample = [0, 1, 37, 128, 255]
        r = P.oracle_prefill_head(w, inp, 0, h, query_chunks=sample)
        P.check_routing_exact(r, gates, aidx, acnt, 0, h)
        rows = np.concatenate([np.arange(64 * i, 64 * i + 64) for i in sample])
        P.check_bf16(P.np64(o[0, rows, h]), r.o[rows])


def test_full_size_gdn_reduction_sampled(hla):
    """Native-GDN reduction at full size (B=4, H=16, T=4096, d=128, bf16, all gates
    one): whole sequences of two (b, h) pairs against the sequential gated delta rule."""
    w = syn.GDN_REDUCTION
    inp = P.gpu_inputs(w)
    o, gates, aidx, acnt = P.run_prefill(hla, w, inp)
    assert torch.all(acnt[:, :, 1:] > 0)
    for (b, h) in ((0, 0), (3, 11)):
        ref, _ = ho.gdn_recurrent(P.np64(inp["q"][b, :, h]), P.np64(inp["k"][b, :, h]),
                                  P.np64(inp["v"][b, :, h]), P.np64(inp["alpha"][b, :, h]),
                                  P.np64(inp["beta"][b, :, h]))
        P.check_bf16(P.np64(o[b, :, h]), ref)


def test_full_size_sparse_prefill_sampled(hla):
    """Long sparse prefill at full size (B=1, H=32, T=131072, 2048 chunks, bf16,
    planted route inputs, threshold 0.05).  Inputs are generated on the device (the
    oracle reads the sampled heads back); gates and active lists bit-exact on two
    heads, sampled query chunks against the oracle, and the planted sparsity
    (about 8 active earlier chunks per query chunk on average) is checked."""
    w = syn.SPARSE_LONG
    inp = syn.make_gdn_inputs(w, device="cuda")
    inp["q_route"], inp["k_route"] = syn.make_route_inputs(w, device="cuda")
    o, gates, aidx, acnt = P.run_prefill(hla, w, inp)
    mean_active = float(acnt.double().mean())
    assert 4.0 <= mean_active <= 12.0, mean_active
    for h in (0, 21):
        sample = [0, 1, 700, 1500, 2047]
        r = P.oracle_prefill_head(w, inp, 0, h, query_chunks=sample)
        P.check_routing_exact(r, gates, aidx, acnt, 0, h)
        rows = np.concatenate([np.arange(64 * i, 64 * i + 64) for i in sample])
        P.check_bf16(P.np64(o[0, rows, h]), r.o[rows])
