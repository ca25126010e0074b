"""GPU parity of the routing diagnostics (hla_gate_support) against the oracle.

Mass and effective support per query chunk are float32 sums on the GPU and float64
sums of the same binary32 gates in the oracle: they agree to a relative 1e-5 (a
float32 butterfly over at most a few thousand terms in [0, 1] errs by far less)."""
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


@pytest.mark.parametrize("w", [
    syn.PREFILL_0P8B.with_(B=2, H=2, T=64 * 40 + 7),                      # dense, spread gates
    syn.SPARSE_LONG.with_(B=1, H=3, T=64 * 70, topics=6),                 # planted, thresholded
    syn.PREFILL_0P8B.with_(B=1, H=2, T=256 * 9 + 100, C=256, thr=0.3),    # long chunks, thresholded
])
def test_gate_support_matches_oracle(hla, w):
    inp = P.gpu_inputs(w)
    o, gates, aidx, acnt = P.run_prefill(hla, w, inp)
    B, T, H, d = inp["q"].shape
    N = w.N
    cfg = hla.make_config(B, H, T, w.C, d, w.dtype, w.gate_mode, w.tau, w.bias, w.thr)
    g = gates.cuda()
    mass = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    sup = torch.empty_like(mass)
    hla.hla_gate_support(cfg, g, mass, sup)
    torch.cuda.synchronize()
    mass, sup = mass.cpu().numpy(), sup.cpu().numpy()
    for b in range(B):
        for h in range(H):
            # the oracle's own gates (pools and gates by the binary32 recipe)
            qr = inp["q_route"] if inp.get("q_route") is not None else inp["q"]
            kr = inp["k_route"] if inp.get("k_route") is not None else inp["k"]
            rq = ho.route_pools(P.np32(qr[b, :, h]), w.C, w.tau)
            rk = ho.route_pools(P.np32(kr[b, :, h]), w.C, w.tau)
            G = ho.gate_matrix(rq, rk, d, w.bias, w.gate_mode)
            m_ref, s_ref = ho.gate_support(G, w.thr)
            assert np.all(np.abs(mass[b, h] - m_ref) <= 1e-5 * np.maximum(1.0, np.abs(m_ref)))
            assert np.all(np.abs(sup[b, h] - s_ref) <= 1e-5 * np.maximum(1.0, np.abs(s_ref)))
            # the kept count bounds the support (Cauchy-Schwarz) and equals the list length
            kept = acnt[b, h].numpy()
            assert np.all(sup[b, h] <= kept + 1e-3)
    if w.thr > 0:
        assert np.median(sup) < np.median(acnt.numpy()) + 1e-3
