"""Pins for the fp64 HLA oracle (CPU only).

Each test pins the oracle to something other than itself: the plain token-by-token
gated delta rule, exact rational brute force with explicit per-token matrices,
closed forms, special cases and invariants that the definition fixes.  Source
passages: HLA summary page, "Methodology in Plain English" (affine per-token rule;
exact chunk summaries; weight 1 keeps the transition, weight 0 leaves the state
untouched; current chunk weight one, future masked; threshold skip is exact) and
"Key Contributions" 2-3.
"""
from fractions import Fraction

import numpy as np
import pytest

from oracle import hla_oracle as ho
from oracle import brute
from oracle import routing_recipe as rr


def _head(rng, T, dk, dv=None, bf16_like=False):
    dv = dk if dv is None else dv
    q = rng.standard_normal((T, dk))
    k = rng.standard_normal((T, dk))
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((T, dv))
    alpha = np.exp(-np.log1p(np.exp(rng.standard_normal(T) - 3.0)))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal(T)))
    if bf16_like:
        q, k, v = (x.astype(np.float32) for x in (q, k, v))
    return q, k, v, alpha, beta


# ---- chunk transitions ------------------------------------------------------------

@pytest.mark.parametrize("n,d,dv", [(8, 5, 6), (16, 12, 12), (64, 128, 128)])
def test_wy_form_equals_literal_transition(n, d, dv):
    rng = np.random.default_rng(n + d)
    _, k, v, a, b = _head(rng, n, d, dv)
    A, B = ho.chunk_transition(k, v, a, b)
    A2, B2, Wb, Ub, ell = ho.chunk_transition_wy(k, v, a, b)
    assert np.abs(A - A2).max() <= 1e-12
    assert np.abs(B - B2).max() <= 1e-12


def test_composition_law_two_chunks():
    rng = np.random.default_rng(11)
    _, k, v, a, b = _head(rng, 16, 6)
    A1, B1 = ho.chunk_transition(k[:8], v[:8], a[:8], b[:8])
    A2, B2 = ho.chunk_transition(k[8:], v[8:], a[8:], b[8:])
    A, B = ho.chunk_transition(k, v, a, b)
    assert np.abs(A - A1 @ A2).max() <= 1e-13
    assert np.abs(B - (B1 @ A2 + B2)).max() <= 1e-13


def test_long_chunk_is_product_of_its_64_token_pieces():
    # a chunk of 256 tokens acts as its four 64-token pieces applied in order:
    # A = A1 A2 A3 A4 and B = ((B1 A2 + B2) A3 + B3) A4 + B4 (affine maps compose)
    rng = np.random.default_rng(21)
    _, k, v, a, b = _head(rng, 256, 10)
    A, B = ho.chunk_transition(k, v, a, b)
    Ap, Bp = np.eye(10), np.zeros((10, 10))
    for p in range(4):
        sl = slice(64 * p, 64 * p + 64)
        Ai, Bi = ho.chunk_transition(k[sl], v[sl], a[sl], b[sl])
        Ap, Bp = Ap @ Ai, Bp @ Ai + Bi
    assert np.abs(A - Ap).max() <= 1e-13
    assert np.abs(B - Bp).max() <= 1e-12


def test_transition_contraction():
    # eigenvalues of I - beta k k^T lie in [1 - beta, 1] for unit k, so ||A_c||_2 <= gamma_C
    rng = np.random.default_rng(12)
    for _ in range(5):
        _, k, v, a, b = _head(rng, 64, 32)
        A, _ = ho.chunk_transition(k, v, a, b)
        gamma = np.prod(a)
        assert np.linalg.norm(A, 2) <= gamma * (1 + 1e-12)


def test_identity_transition_alpha1_beta0():
    rng = np.random.default_rng(13)
    q, k, v, _, _ = _head(rng, 24, 8)
    a = np.ones(24)
    b = np.zeros(24)
    A, B = ho.chunk_transition(k[:8], v[:8], a[:8], b[:8])
    assert np.array_equal(A, np.eye(8)) and np.array_equal(B, np.zeros((8, 8)))
    r = ho.hla_prefill_head(q, k, v, a, b, 8, bias=1.0)
    assert np.array_equal(r.o, np.zeros_like(r.o))


# ---- prefill reductions ----------------------------------------------------------

def test_T1_closed_form():
    rng = np.random.default_rng(14)
    q, k, v, a, b = _head(rng, 1, 16)
    r = ho.hla_prefill_head(q, k, v, a, b, 64)
    np.testing.assert_allclose(r.o[0], b[0] * (k[0] @ q[0]) * v[0], rtol=1e-14, atol=1e-15)


def test_single_chunk_equals_gdn():
    rng = np.random.default_rng(15)
    q, k, v, a, b = _head(rng, 50, 16)
    r = ho.hla_prefill_head(q, k, v, a, b, 64, bias=-3.0)
    o, _ = ho.gdn_recurrent(q, k, v, a, b)
    assert np.abs(r.o - o).max() <= 1e-13


@pytest.mark.parametrize("T,C", [(64, 8), (70, 8), (600, 256), (300, 128)])
def test_gates_one_is_native_gdn(T, C):
    rng = np.random.default_rng(16 + T)
    q, k, v, a, b = _head(rng, T, 12)
    r = ho.hla_prefill_head(q, k, v, a, b, C, gate_mode=ho.GATES_ONE)
    o, _ = ho.gdn_recurrent(q, k, v, a, b)
    assert np.abs(r.o - o).max() <= 1e-12


def test_gates_zero_leaves_intra_chunk_only():
    rng = np.random.default_rng(17)
    q, k, v, a, b = _head(rng, 40, 12)
    r = ho.hla_prefill_head(q, k, v, a, b, 8, gate_mode=ho.GATES_ZERO)
    for c in range(5):
        sl = slice(8 * c, 8 * c + 8)
        o, _ = ho.gdn_recurrent(q[sl], k[sl], v[sl], a[sl], b[sl])
        assert np.abs(r.o[sl] - o).max() <= 1e-14


def test_two_chunks_output_affine_in_gate():
    rng = np.random.default_rng(18)
    q, k, v, a, b = _head(rng, 16, 6)
    outs = []
    for g in (0.0, 0.3, 1.0):
        ug = np.zeros((2, 2))
        ug[1, 0] = g
        outs.append(ho.hla_prefill_head(q, k, v, a, b, 8, gate_mode=ho.GATES_USER, user_gates=ug).o)
    # S_in(1) = g B_0, chunk 1 output is affine in g (gates are binary32 values)
    interp = outs[0] + float(np.float32(0.3)) * (outs[2] - outs[0])
    assert np.abs(outs[1] - interp).max() <= 1e-13
    # chunk 0 never sees the gate
    assert np.array_equal(outs[0][:8], outs[2][:8])
    # with g = 1 the state entering chunk 1 is B_0: compare against the token rule
    o, S8 = ho.gdn_recurrent(q[:8], k[:8], v[:8], a[:8], b[:8])
    o2, _ = ho.gdn_recurrent(q[8:], k[8:], v[8:], a[8:], b[8:], S0=S8)
    assert np.abs(outs[2][8:] - o2).max() <= 1e-13


def test_skip_is_exactly_identity():
    rng = np.random.default_rng(19)
    T, d, C = 96, 8, 8
    q, k, v, a, b = _head(rng, T, d)
    qr = rng.standard_normal((T, d)) * 2
    kr = rng.standard_normal((T, d)) * 2
    r0 = ho.hla_prefill_head(q, k, v, a, b, C, bias=-1.0, q_route=qr, k_route=kr)
    thr = float(np.median(r0.gates[np.tril_indices(T // C, -1)]))
    r = ho.hla_prefill_head(q, k, v, a, b, C, bias=-1.0, thr=thr, q_route=qr, k_route=kr)
    skipped = sum(i - len(x) for i, x in enumerate(r.active))
    assert skipped > 10
    ug = np.where(r.gates >= np.float32(thr), r.gates, 0).astype(np.float64)
    r2 = ho.hla_prefill_head(q, k, v, a, b, C, gate_mode=ho.GATES_USER, user_gates=ug, thr=0.0)
    assert np.array_equal(r.o, r2.o)


def test_future_chunks_do_not_change_past_outputs():
    rng = np.random.default_rng(20)
    q, k, v, a, b = _head(rng, 64, 8)
    r1 = ho.hla_prefill_head(q, k, v, a, b, 8, bias=0.5)
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    v2[40:] += 3.0
    k2[40:] = np.roll(k2[40:], 1, axis=1)
    r2 = ho.hla_prefill_head(q2, k2, v2, a, b, 8, bias=0.5)
    assert np.array_equal(r1.o[:40], r2.o[:40])


# ---- brute force ----------------------------------------------------------------

def _frac(x):
    return Fraction(float(x))


@pytest.mark.parametrize("T,C,d", [(8, 2, 2), (8, 4, 3), (7, 4, 2), (6, 2, 4)])
def test_exact_rational_brute_force(T, C, d):
    rng = np.random.default_rng(100 + T * C * d)
    q, k, v, a, b = _head(rng, T, d)
    N = (T + C - 1) // C
    ug = np.tril(rng.uniform(0, 1, (N, N)), -1).astype(np.float32)   # gates are binary32
    r = ho.hla_prefill_head(q, k, v, a, b, C, gate_mode=ho.GATES_USER, user_gates=ug)
    F = lambda M: [[_frac(x) for x in row] for row in np.atleast_2d(M)]
    ob = brute.hla_brute(F(q), F(k), F(v), [_frac(x) for x in a], [_frac(x) for x in b], C,
                         [[_frac(x) for x in row] for row in ug], zero=Fraction(0), one=Fraction(1))
    exact = np.array([[float(x) for x in row] for row in ob])
    assert np.abs(r.o - exact).max() <= 1e-13


def test_brute_force_with_routed_thresholded_gates():
    rng = np.random.default_rng(21)
    T, C, d = 8, 2, 4
    q, k, v, a, b = _head(rng, T, d)
    qr = (rng.standard_normal((T, d)) * 3).astype(np.float32)
    kr = (rng.standard_normal((T, d)) * 3).astype(np.float32)
    r = ho.hla_prefill_head(q, k, v, a, b, C, bias=-0.5, thr=0.4, q_route=qr, k_route=kr)
    assert any(len(x) < i for i, x in enumerate(r.active))
    gates = [[float(g) for g in row] for row in r.gates]
    ob = brute.hla_brute(q.tolist(), k.tolist(), v.tolist(), a.tolist(), b.tolist(), C, gates,
                         active=[list(x) for x in r.active])
    assert np.abs(r.o - np.array(ob)).max() <= 1e-13
    # gates come from pools of the route tokens of each chunk
    rq = np.stack([rr.lme_pool32(qr[c * C:(c + 1) * C], 1.0) for c in range(4)])
    assert np.array_equal(r.rq, rq)


# ---- decode -----------------------------------------------------------------------

def _steps(rng, n, d):
    out = []
    for _ in range(n):
        q, k, v, a, b = _head(rng, 1, d)
        out.append((q[0], k[0], v[0], a[0], b[0]))
    return out


@pytest.mark.parametrize("T0,window", [(16, 0), (21, 0), (21, 4), (19, 2)])
def test_decode_matches_prefill_of_extended_sequence(T0, window):
    rng = np.random.default_rng(22 + T0)
    C, d = 8, 6
    q, k, v, a, b = _head(rng, T0, d)
    qr = rng.standard_normal((T0, d)) * 2
    kr = rng.standard_normal((T0, d)) * 2
    st = ho.HlaDecodeHead.from_prefill(q, k, v, a, b, C, bias=-0.5, thr=0.3,
                                       q_route=qr, k_route=kr, pool_window=window)
    toks = _steps(rng, 12, d)   # crosses a chunk boundary
    for s, (tq, tk, tv, ta, tb) in enumerate(toks):
        tqr = rng.standard_normal(d) * 2
        tkr = rng.standard_normal(d) * 2
        o = st.step(tq, tk, tv, ta, tb, tqr, tkr)
        q = np.vstack([q, tq]); k = np.vstack([k, tk]); v = np.vstack([v, tv])
        a = np.append(a, ta); b = np.append(b, tb)
        qr = np.vstack([qr, tqr]); kr = np.vstack([kr, tkr])
        ref = ho.hla_prefill_head(q, k, v, a, b, C, bias=-0.5, thr=0.3, q_route=qr,
                                  k_route=kr, query_chunks=[(len(a) - 1) // C], pool_window=window)
        assert np.abs(o - ref.o[-1]).max() <= 1e-12
    # closed chunks in the cache equal the literal transitions and pools
    n = len(a) // C
    assert len(st.trans) == n
    A, B = ho.chunk_transition(k[(n - 1) * C:n * C], v[(n - 1) * C:n * C], a[(n - 1) * C:n * C],
                               b[(n - 1) * C:n * C])
    assert np.abs(st.trans[-1][0] - A).max() <= 1e-14
    last = kr[(n - 1) * C:n * C].astype(np.float32)
    if window:
        for u in range(C // window):
            assert np.array_equal(st.rk[-1][u], rr.lme_pool32(last[u * window:(u + 1) * window], 1.0))
    else:
        assert np.array_equal(st.rk[-1], rr.lme_pool32(last, 1.0))


def test_decode_backward_chain_equals_forward_composition():
    rng = np.random.default_rng(23)
    C, d, T = 8, 6, 64
    q, k, v, a, b = _head(rng, T, d)
    trans = [ho.chunk_transition(k[c * C:(c + 1) * C], v[c * C:(c + 1) * C], a[c * C:(c + 1) * C],
                                 b[c * C:(c + 1) * C]) for c in range(8)]
    g = rng.uniform(0, 1, 8)
    active = [0, 2, 3, 6, 7]
    x = rng.standard_normal(d)
    S = np.zeros((d, d))
    for j in active:
        S = S + g[j] * ((S @ trans[j][0] + trans[j][1]) - S)
    y = ho.decode_output_backward(trans, g, active, x, np.zeros(d))
    assert np.abs(y - S @ x).max() <= 1e-13


def test_decode_partial_chunk_sweep_closed_form():
    # right-to-left sweep over buffered tokens gives A_p q and B_p q
    rng = np.random.default_rng(24)
    d, m = 6, 5
    _, k, v, a, b = _head(rng, m, d)
    qv = rng.standard_normal(d)
    Ap, Bp = ho.chunk_transition(k, v, a, b)
    x = qv.copy()
    y0 = np.zeros(d)
    for t in reversed(range(m)):
        y0 += b[t] * v[t] * (k[t] @ x)
        x = a[t] * (x - b[t] * k[t] * (k[t] @ x))
    assert np.abs(x - Ap @ qv).max() <= 1e-14
    assert np.abs(y0 - Bp @ qv).max() <= 1e-14


# ---- effective support of the routing (order-2 effective number) ------------------

def test_support_of_equal_gates_is_their_count():
    # n kept gates of equal value g: (n g)^2 / (n g^2) = n, mass n g
    G = np.zeros((6, 6), np.float32)
    for i in range(6):
        G[i, :i] = 0.375
    mass, sup = ho.gate_support(G, 0.0)
    assert sup.tolist() == [0.0, 1.0, 2.0, 3.0, 4.0, 5.0]
    assert mass.tolist() == [0.375 * i for i in range(6)]


def test_support_counts_only_kept_chunks_and_is_scale_free():
    G = np.zeros((4, 4), np.float32)
    G[3, :3] = [0.9, 0.02, 0.9]          # the middle chunk is below the threshold
    G[2, :2] = [0.5, 0.0]
    mass, sup = ho.gate_support(G, 0.05)
    assert sup[3] == 2.0 and mass[3] == pytest.approx(1.8, abs=1e-7)
    assert sup[2] == 1.0                  # one kept chunk
    assert sup[1] == 0.0 and mass[1] == 0.0   # g = 0 < 0.05: nothing kept
    _, sup_all = ho.gate_support(G, 0.0)
    # without a threshold the small gate counts a little: 1.82^2 / (2 * 0.81 + 0.0004)
    assert sup_all[3] == pytest.approx(1.82 ** 2 / (2 * 0.9 ** 2 + 0.02 ** 2), rel=1e-6)
    _, sup_half = ho.gate_support(G * np.float32(0.5), 0.0)
    assert np.allclose(sup_half, sup_all, rtol=1e-12)


def test_support_lies_between_one_and_the_kept_count():
    # Cauchy-Schwarz: (sum g)^2 <= n sum g^2, with equality for equal gates
    rng = np.random.default_rng(31)
    G = rng.uniform(0.0, 1.0, (40, 40)).astype(np.float32)
    mass, sup = ho.gate_support(G, 0.3)
    for i in range(40):
        n = int((G[i, :i] >= np.float32(0.3)).sum())
        if n == 0:
            assert sup[i] == 0.0
        else:
            assert 1.0 - 1e-12 <= sup[i] <= n + 1e-12


# ---- channel-wise decay (KDA-style: S Diag(alpha_t)(I - beta k k^T) + beta v k^T) -----

def _channel_alpha(rng, T, d):
    return np.exp(-np.log1p(np.exp(rng.standard_normal((T, d)) - 3.0)))


@pytest.mark.parametrize("T,C,d", [(8, 2, 2), (7, 4, 3)])
def test_channel_decay_exact_rational_brute_force(T, C, d):
    rng = np.random.default_rng(300 + T * C * d)
    q, k, v, _, b = _head(rng, T, d)
    a = _channel_alpha(rng, T, d)
    N = (T + C - 1) // C
    ug = np.tril(rng.uniform(0, 1, (N, N)), -1).astype(np.float32)
    r = ho.hla_prefill_head(q, k, v, a, b, C, gate_mode=ho.GATES_USER, user_gates=ug)
    F = lambda M: [[_frac(x) for x in row] for row in np.atleast_2d(M)]
    ob = brute.hla_brute(F(q), F(k), F(v), F(a), [_frac(x) for x in b], C,
                         [[_frac(x) for x in row] for row in ug], zero=Fraction(0), one=Fraction(1))
    exact = np.array([[float(x) for x in row] for row in ob])
    assert np.abs(r.o - exact).max() <= 1e-13


def test_channel_decay_with_equal_channels_is_scalar_decay():
    rng = np.random.default_rng(301)
    q, k, v, a, b = _head(rng, 40, 6)
    r1 = ho.hla_prefill_head(q, k, v, a, b, 8, bias=-1.0, thr=0.3)
    r2 = ho.hla_prefill_head(q, k, v, np.repeat(a[:, None], 6, axis=1), b, 8, bias=-1.0, thr=0.3)
    assert np.abs(r1.o - r2.o).max() <= 1e-12


def test_channel_decay_without_edits_is_diagonal():
    # beta = 0: no edit, so A_c = Diag(prod_t alpha_t) and B_c = 0
    rng = np.random.default_rng(302)
    _, k, v, _, _ = _head(rng, 9, 5)
    a = _channel_alpha(rng, 9, 5)
    A, B = ho.chunk_transition(k, v, a, np.zeros(9))
    assert np.abs(A - np.diag(np.prod(a, axis=0))).max() <= 1e-15
    assert np.abs(B).max() == 0.0


def test_channel_decay_decode_matches_prefill():
    rng = np.random.default_rng(303)
    C, d, T0 = 8, 5, 13
    q, k, v, _, b = _head(rng, T0, d)
    a = _channel_alpha(rng, T0, d)
    st = ho.HlaDecodeHead.from_prefill(q, k, v, a, b, C, bias=-0.5, thr=0.2)
    for _ in range(6):   # closes chunk 1 at the third step
        tq, tk, tv, _, tb = _head(rng, 1, d)
        ta = _channel_alpha(rng, 1, d)
        o = st.step(tq[0], tk[0], tv[0], ta[0], tb[0])
        q = np.vstack([q, tq]); k = np.vstack([k, tk]); v = np.vstack([v, tv])
        a = np.vstack([a, ta]); b = np.append(b, tb)
        ref = ho.hla_prefill_head(q, k, v, a, b, C, bias=-0.5, thr=0.2, query_chunks=[(len(b) - 1) // C])
        assert np.abs(o - ref.o[-1]).max() <= 1e-12
    assert len(st.trans) == 2


@pytest.mark.parametrize("n,d,dv", [(8, 5, 6), (16, 12, 12), (64, 128, 128)])
def test_channel_wy_form_equals_literal_transition(n, d, dv):
    """The chunkwise WY form with the decays folded into the keys (kt = gamma o k,
    kh = k / gamma) reaches the token rule's (A, B) with a decay per key channel."""
    rng = np.random.default_rng(100 + n + d)
    _, k, v, _, b = _head(rng, n, d, dv)
    a = _channel_alpha(rng, n, d)
    A, B = ho.chunk_transition(k, v, a, b)
    A2, B2, Wb, Ub, ell = ho.chunk_transition_wy_channel(k, v, a, b)
    assert np.abs(A - A2).max() <= 1e-12
    assert np.abs(B - B2).max() <= 1e-12


def test_channel_wy_form_with_equal_channels_is_the_scalar_wy_form():
    rng = np.random.default_rng(7)
    _, k, v, a, b = _head(rng, 16, 8)
    A1, B1, W1, U1, _ = ho.chunk_transition_wy(k, v, a, b)
    A2, B2, W2, U2, _ = ho.chunk_transition_wy_channel(k, v, np.repeat(a[:, None], 8, axis=1), b)
    for x, y in ((A1, A2), (B1, B2), (W1, W2), (U1, U2)):
        assert np.abs(x - y).max() <= 1e-13


@pytest.mark.parametrize("n,d", [(8, 5), (64, 32)])
def test_channel_wy_readout_equals_token_rule(n, d):
    """O = Qt S0^T + tril(Qt Kh^T)(Ub - Wb S0^T) equals the token rule run from S0
    with a decay per key channel, output o_t = S_t q_t."""
    rng = np.random.default_rng(200 + n)
    q, k, v, _, b = _head(rng, n, d)
    a = _channel_alpha(rng, n, d)
    S0 = rng.standard_normal((d, d))
    o, _ = ho.gdn_recurrent(q, k, v, a, b, S0=S0)
    _, _, Wb, Ub, ell = ho.chunk_transition_wy_channel(k, v, a, b)
    O = ho.chunk_readout_wy_channel(q, k, Wb, Ub, ell, S0)
    assert np.abs(O - o).max() <= 1e-12
