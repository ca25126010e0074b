"""Oracle, part 1: Hybrid Linear Attention (HLA) over Gated DeltaNet, in fp64.

TEST INFRASTRUCTURE ONLY.  This is the plain, slow, obviously-correct CPU statement
of what the GPU hot path computes.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it; the
product path never does, and it shares no code with the CUDA library.

Source passages (HLA: Expressive Hybrid Linear Attention via Chunk-Wise Dynamic
Mixing, ai.info AI summary page):
* "Methodology in Plain English", first paragraph: the gated delta rule updates the
  state at every token by an affine rule (a matrix that decays and edits the old
  state, plus an additive key-value write); affine maps compose, so a whole chunk is
  summarised exactly by one (matrix, additive term) pair.
* Same section, third paragraph: a chunk's weight interpolates its full transition
  with the identity (weight 1 = original transition, weight 0 = incoming state
  untouched); the current chunk always has weight one and uses its own causal
  prefix as is; future chunks are masked out.
* Same section, fourth paragraph: historical weights below the inference threshold
  are set to zero without renormalisation, so skipping that transition is exact.
* "Key Contributions" 2-3 and the "Authors' abstract": each completed chunk is an
  exact affine state transition; prefill and autoregressive decoding algorithms.

Precise reading (the pages give prose only):
* per head, state S is d_v x d_k; token rule
  S_t = S_{t-1} * alpha_t (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,  o_t = S_t q_t
  (no 1/sqrt(d) on q);
* chunk c (tokens cC .. cC+C-1) acts as S -> S A_c + B_c, computed here LITERALLY by
  running the token rule (A_c from the homogeneous rule started at I, B_c from the
  full rule started at 0);
* query chunk i: S <- 0; for j = 0 .. i-1 ascending: S <- S + g_ij((S A_j + B_j) - S);
  this is S_in(i); a j with g_ij below the threshold has g_ij = 0 and is the identity;
* output: run the token rule from S_in(i) over chunk i's tokens, o_t = S_t q_t;
* gates g_ij (j < i) come from the binary32 routing recipe (``routing_recipe``) on
  per-chunk log-mean-exp pools of the route inputs (default: q and k), all tokens
  of each chunk (the pool is not causal inside a chunk); a final partial chunk pools
  its own m tokens.

All arithmetic here is float64 except the routing recipe, which is binary32 by
definition.  Inputs (bf16 or fp32) are upcast exactly.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

from . import routing_recipe as rr

GATES_ROUTED = "routed"
GATES_ONE = "one"
GATES_ZERO = "zero"
GATES_USER = "user"


# ----------------------------------------------------------------------------------
# Token recurrence and chunk transitions
# ----------------------------------------------------------------------------------

def gdn_token_step(S, k, v, alpha, beta):
    """One token of the gated delta rule: S Diag(alpha) (I - beta k k^T) + beta v k^T.

    ``alpha`` is a scalar (Gated DeltaNet: S alpha (I - beta k k^T) + beta v k^T) or a
    vector over the d_k key channels (channel-wise decay, the KDA-style decay named in
    the Gated DeltaNet-2 abstract on the HLA listing page: the state's key channels
    decay each at its own rate before the delta-rule edit)."""
    if np.ndim(alpha) == 0:
        Sk = S @ k
        return alpha * (S - beta * np.outer(Sk, k)) + beta * np.outer(v, k)
    Sa = S * np.asarray(alpha, np.float64)[None, :]
    return Sa - beta * np.outer(Sa @ k, k) + beta * np.outer(v, k)


def _alpha_of(a):
    """A buffered decay as float (scalar) or float64 vector (channel-wise)."""
    return float(a) if np.ndim(a) == 0 else np.asarray(a, np.float64)


def gdn_recurrent(q, k, v, alpha, beta, S0=None):
    """Plain token-by-token gated delta rule for one head.

    q, k: [T, d_k]; v: [T, d_v]; alpha: [T] or [T, d_k] (channel-wise); beta: [T].
    Returns (o [T, d_v], S_T)."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    alpha = np.asarray(alpha, np.float64)
    beta = np.asarray(beta, np.float64)
    T, dk = k.shape
    dv = v.shape[1]
    S = np.zeros((dv, dk)) if S0 is None else np.array(S0, np.float64)
    o = np.zeros((T, dv))
    for t in range(T):
        S = gdn_token_step(S, k[t], v[t], alpha[t], beta[t])
        o[t] = S @ q[t]
    return o, S


def chunk_transition(k, v, alpha, beta):
    """Exact affine transition (A, B) of one chunk, S -> S A + B, by running the
    token rule: A from the homogeneous rule (no write) started at I, B from the full
    rule started at 0.  k: [n, d_k], v: [n, d_v].  Returns A [d_k, d_k], B [d_v, d_k]."""
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    n, dk = k.shape
    dv = v.shape[1]
    A = np.eye(dk)
    B = np.zeros((dv, dk))
    for t in range(n):
        A = gdn_token_step(A, k[t], np.zeros(dk), alpha[t], beta[t])
        B = gdn_token_step(B, k[t], v[t], alpha[t], beta[t])
    return A, B


def chunk_transition_wy(k, v, alpha, beta):
    """The same (A, B) through the chunkwise WY/UT form (the form the GPU uses).

    With l_t = sum_{s<=t} log alpha_s, gamma_t = exp(l_t), Gamma_ts = exp(l_t - l_s):
      L = strictly-lower part of diag(beta) (Gamma o K K^T)
      T = (I + L)^{-1} diag(beta)
      Wb = T diag(gamma) K,  Ub = T V,  D = diag(gamma_n / gamma_t)
      A = gamma_n I - Wb^T D K,  B = Ub^T D K.
    Returns (A, B, Wb, Ub, l)."""
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    alpha = np.asarray(alpha, np.float64)
    beta = np.asarray(beta, np.float64)
    n, dk = k.shape
    ell = np.cumsum(np.log(alpha))
    gamma = np.exp(ell)
    Gam = np.exp(ell[:, None] - ell[None, :])
    L = np.tril(beta[:, None] * Gam * (k @ k.T), -1)
    T = np.linalg.solve(np.eye(n) + L, np.diag(beta))
    Wb = T @ (gamma[:, None] * k)
    Ub = T @ v
    Dk = np.exp(ell[-1] - ell)[:, None] * k
    A = gamma[-1] * np.eye(dk) - Wb.T @ Dk
    B = Ub.T @ Dk
    return A, B, Wb, Ub, ell


def chunk_transition_wy_channel(k, v, alpha, beta):
    """(A, B) of one chunk under channel-wise decay (alpha [n, d_k]) through the
    chunkwise WY/UT form with the decays folded into the keys.

    With l_t = sum_{s<=t} log alpha_s (a vector over key channels), gamma_t = exp(l_t):
    the state after token t from S_0 is S_0 Diag(gamma_t) + sum_{s<=t} u_s (k_s o
    gamma_t / gamma_s)^T with u_t = beta_t (v_t - S_{t-1} Diag(alpha_t) k_t).  Writing
    kt_t = gamma_t o k_t and kh_s = k_s / gamma_s, the coupling of u_t to u_s (s < t) is
    beta_t (kt_t . kh_s), so
      L = strictly-lower part of diag(beta) Kt Kh^T
      T = (I + L)^{-1} diag(beta)
      Wb = T Kt,  Ub = T V,  Kc = rows k_s o gamma_n / gamma_s
      A = Diag(gamma_n) - Wb^T Kc,  B = Ub^T Kc.
    With equal channels it is ``chunk_transition_wy``.  The entries of Kt Kh^T are
    formed here as sum_c k_t[c] k_s[c] exp(l_t[c] - l_s[c]) (every factor at most 1 for
    s < t).  Returns (A, B, Wb, Ub, l) with l [n, d_k]."""
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    alpha = np.asarray(alpha, np.float64)
    beta = np.asarray(beta, np.float64)
    n, dk = k.shape
    ell = np.cumsum(np.log(alpha), axis=0)             # [n, d_k]
    gamma = np.exp(ell)
    # [t, s, c] = gamma_t / gamma_s for s < t, else 0
    lower = np.tri(n, n, -1)[:, :, None] > 0
    ratio = np.exp(np.where(lower, ell[:, None, :] - ell[None, :, :], -np.inf))
    L = beta[:, None] * np.einsum("tc,sc,tsc->ts", k, k, ratio)
    T = np.linalg.solve(np.eye(n) + L, np.diag(beta))
    Wb = T @ (gamma * k)
    Ub = T @ v
    Kc = np.exp(ell[-1][None, :] - ell) * k
    A = np.diag(gamma[-1]) - Wb.T @ Kc
    B = Ub.T @ Kc
    return A, B, Wb, Ub, ell


def chunk_readout_wy_channel(q, k, Wb, Ub, ell, S0):
    """Outputs of one chunk from its incoming state S0 under channel-wise decay, in
    the WY form (the form a tensor-core read-out uses): with qt_t = gamma_t o q_t,
      O = Qt S0^T + tril(Qt Kh^T) (Ub - Wb S0^T)     (diagonal included),
    where (Qt Kh^T)_ts = sum_c q_t[c] k_s[c] exp(l_t[c] - l_s[c]).  Returns O [n, d_v]."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    n = q.shape[0]
    gamma = np.exp(ell)
    lower = np.tri(n, n, 0)[:, :, None] > 0
    ratio = np.exp(np.where(lower, ell[:, None, :] - ell[None, :, :], -np.inf))
    P = np.einsum("tc,sc,tsc->ts", q, k, ratio)
    U = Ub - Wb @ np.asarray(S0, np.float64).T
    return (gamma * q) @ np.asarray(S0, np.float64).T + P @ U


# ----------------------------------------------------------------------------------
# Routing (binary32 recipe)
# ----------------------------------------------------------------------------------

def chunk_bounds(T: int, C: int):
    N = (T + C - 1) // C
    return [(c * C, min(T, (c + 1) * C)) for c in range(N)]


def route_pools(x_route, C: int, tau: float):
    """Per-chunk log-mean-exp pools of one head's route tokens [T, d] -> [N, d] f32."""
    x = np.asarray(x_route, np.float32)
    T = x.shape[0]
    full = T // C
    # complete chunks pooled side by side (each chunk on its own, same steps)
    out = [rr.lme_pool32(x[:full * C].reshape(full, C, -1), tau)] if full else []
    if T > full * C:
        out.append(rr.lme_pool32(x[full * C:], tau)[None])
    return np.concatenate(out).astype(np.float32)


def window_pools(x_route, C: int, window: int, tau: float):
    """Window representatives of one head's complete chunks: every chunk of C tokens
    is split into W = C / window windows, each pooled on its own by the log-mean-exp
    pool.  x_route [T, d] -> [T // C, W, d] f32."""
    x = np.asarray(x_route, np.float32)
    nc = x.shape[0] // C
    W = C // window
    if nc == 0:
        return np.zeros((0, W, x.shape[1]), np.float32)
    r = rr.lme_pool32(x[:nc * C].reshape(nc * W, window, -1), tau)
    return r.reshape(nc, W, -1).astype(np.float32)


def gate_matrix(rq, rk, d: int, bias: float, mode: str = GATES_ROUTED, user=None):
    """Raw gates G [N, N] (binary32) with G[i, j] meaningful for j < i, zero elsewhere
    (the current chunk's own weight is 1 by definition and is not a gate).  rk is
    [N_k, d] (one representative per chunk) or [N_k, W, d] (window representatives,
    combined by a log-sum-exp inside the sigmoid); N_k may be smaller than N when
    only the complete chunks have key representatives."""
    N = rq.shape[0]
    if mode == GATES_ROUTED and np.ndim(rk) == 3:
        G = np.zeros((N, N), np.float32)
        nk = rk.shape[0]
        if nk:
            G[:, :nk] = rr.gate_matrix_window32(rq, rk, d, bias)
    elif mode == GATES_ROUTED:
        G = rr.gate_matrix32(rq, rk, d, bias)
    elif mode == GATES_ONE:
        G = np.ones((N, N), np.float32)
    elif mode == GATES_ZERO:
        G = np.zeros((N, N), np.float32)
    elif mode == GATES_USER:
        G = np.asarray(user, np.float32).copy()
    else:
        raise ValueError(mode)
    return np.tril(G, -1).astype(np.float32)


def active_lists(G, thr: float):
    """Ascending active chunk indices per query chunk: {j < i : G[i, j] >= thr} for
    thr > 0; for thr <= 0 every j < i is active (nothing is skipped)."""
    N = G.shape[0]
    thr32 = np.float32(thr)
    out = []
    for i in range(N):
        js = np.arange(i)
        if thr > 0:
            js = js[G[i, :i] >= thr32]
        out.append(js.astype(np.int32))
    return out


def gate_support(G, thr: float):
    """Routing mass and effective support per query chunk ("Key Contributions" 3 and
    "Methodology in Plain English" para. 4: an order-2 effective number, the inverse
    sum of squares, of the chunks a query accesses).

    Over the chunks j < i that are kept (every one for thr <= 0, else G[i, j] >= thr):
    mass_i = sum_j g_ij and support_i = mass_i^2 / sum_j g_ij^2 (0 with nothing
    kept).  float64 sums of the binary32 gates.  Returns (mass [N], support [N])."""
    G = np.asarray(G, np.float32)
    N = G.shape[0]
    mass = np.zeros(N)
    support = np.zeros(N)
    for i in range(N):
        g = G[i, :i].astype(np.float64)
        if thr > 0:
            g = g[G[i, :i] >= np.float32(thr)]
        m, q = g.sum(), (g * g).sum()
        mass[i] = m
        support[i] = m * m / q if q > 0 else 0.0
    return mass, support


# ----------------------------------------------------------------------------------
# Prefill
# ----------------------------------------------------------------------------------

def compose_state(trans, gates_row, active):
    """S_in for one query chunk: S <- 0; for j in active (ascending):
    S <- S + g_j ((S A_j + B_j) - S)."""
    dv, dk = trans[0][1].shape
    S = np.zeros((dv, dk))
    for j in active:
        A, B = trans[j]
        g = float(gates_row[j])
        S = S + g * ((S @ A + B) - S)
    return S


@dataclass
class HeadResult:
    o: np.ndarray                 # [T, d_v] float64
    gates: np.ndarray             # [N, N] float32 raw gates (j < i), 0 elsewhere
    active: list                  # per query chunk: ascending int32 active j
    rq: np.ndarray                # [N, d] float32 pools
    rk: np.ndarray                # [N, d] float32 pools
    trans: list = field(default_factory=list)  # [(A_j, B_j)] for complete chunks


def hla_prefill_head(q, k, v, alpha, beta, C, tau=1.0, bias=0.0, thr=0.0,
                     gate_mode=GATES_ROUTED, q_route=None, k_route=None,
                     user_gates=None, query_chunks=None, trans=None, pool_window=0):
    """HLA prefill for one (sequence, head).  q, k: [T, d_k]; v: [T, d_v].

    ``pool_window`` > 0: each chunk's key side is represented by its C / pool_window
    window pools and the gate takes a log-sum-exp over them (``gate_window32``).

    ``query_chunks``: if given, only those query chunks' outputs are computed (the rest
    of ``o`` is NaN) -- used for sampled checks at full size.  ``trans``: optional
    precomputed list of (A_j, B_j); by default built literally by ``chunk_transition``.
    """
    q = np.asarray(q, np.float64)
    k64 = np.asarray(k, np.float64)
    v64 = np.asarray(v, np.float64)
    alpha = np.asarray(alpha, np.float64)
    beta = np.asarray(beta, np.float64)
    T, dk = k64.shape
    dv = v64.shape[1]
    bounds = chunk_bounds(T, C)
    N = len(bounds)
    qr = q if q_route is None else q_route
    kr = k if k_route is None else k_route
    rq = route_pools(qr, C, tau)
    rk = window_pools(kr, C, pool_window, tau) if pool_window else route_pools(kr, C, tau)
    G = gate_matrix(rq, rk, dk, bias, gate_mode, user_gates)
    act = active_lists(G, thr)
    n_complete = T // C
    if trans is None:
        need = N if query_chunks is None else max(query_chunks)
        need = min(need, n_complete)
        trans = [chunk_transition(k64[a:b], v64[a:b], alpha[a:b], beta[a:b])
                 for (a, b) in bounds[:need]]
    o = np.full((T, dv), np.nan)
    chunks = range(N) if query_chunks is None else query_chunks
    for i in chunks:
        a, b = bounds[i]
        S = compose_state(trans, G[i], act[i]) if i > 0 else np.zeros((dv, dk))
        o[a:b], _ = gdn_recurrent(q[a:b], k64[a:b], v64[a:b], alpha[a:b], beta[a:b], S0=S)
    return HeadResult(o=o, gates=G, active=act, rq=rq, rk=rk, trans=trans)


def hla_prefill(q, k, v, alpha, beta, C, tau=1.0, bias=0.0, thr=0.0,
                gate_mode=GATES_ROUTED, q_route=None, k_route=None, user_gates=None, pool_window=0):
    """Batched prefill over [B, T, H, d] inputs (alpha, beta: [B, T, H];
    user_gates: [B, H, N, N]).  Returns (o [B, T, H, d_v], {(b, h): HeadResult})."""
    Bn, T, H, _ = np.shape(q)
    dv = np.shape(v)[3]
    o = np.zeros((Bn, T, H, dv))
    res = {}
    for b in range(Bn):
        for h in range(H):
            r = hla_prefill_head(
                q[b, :, h], k[b, :, h], v[b, :, h], alpha[b, :, h], beta[b, :, h], C,
                tau, bias, thr, gate_mode,
                None if q_route is None else q_route[b, :, h],
                None if k_route is None else k_route[b, :, h],
                None if user_gates is None else user_gates[b, h], pool_window=pool_window)
            o[b, :, h] = r.o
            res[(b, h)] = r
    return o, res


# ----------------------------------------------------------------------------------
# Decode
# ----------------------------------------------------------------------------------

class HlaDecodeHead:
    """Decode state of one (sequence, head): cached complete-chunk transitions and
    key pools, plus the partial chunk's buffered tokens.

    ``step`` takes one token and returns o_t by the definition: gates of the partial
    chunk's query pool (over its m tokens so far) against every cached key pool,
    threshold, forward composition of S_in over the active chunks, then the token
    rule over the buffered tokens from S_in.  When the partial chunk reaches C tokens
    it is closed: its transition and key pool are appended to the cache."""

    def __init__(self, C, d_k, d_v, tau=1.0, bias=0.0, thr=0.0, gate_mode=GATES_ROUTED, pool_window=0):
        self.C, self.dk, self.dv = C, d_k, d_v
        self.tau, self.bias, self.thr, self.mode = tau, bias, thr, gate_mode
        self.window = pool_window
        self.trans = []       # [(A_j, B_j)] float64
        self.rk = []          # [d] float32 pools ([W, d] window pools with pool_window > 0)
        self.buf = []         # [(q, k, v, alpha, beta, q_route, k_route)]

    @classmethod
    def from_prefill(cls, q, k, v, alpha, beta, C, tau=1.0, bias=0.0, thr=0.0,
                     gate_mode=GATES_ROUTED, q_route=None, k_route=None, trans=None, pool_window=0):
        """Cache state after a prefill of one head's T tokens."""
        T, dk = np.shape(k)
        dv = np.shape(v)[1]
        st = cls(C, dk, dv, tau, bias, thr, gate_mode, pool_window)
        qr = q if q_route is None else q_route
        kr = k if k_route is None else k_route
        n = T // C
        k64 = np.asarray(k, np.float64)
        v64 = np.asarray(v, np.float64)
        if trans is None:
            trans = [chunk_transition(k64[c * C:(c + 1) * C], v64[c * C:(c + 1) * C],
                                      alpha[c * C:(c + 1) * C], beta[c * C:(c + 1) * C])
                     for c in range(n)]
        st.trans = list(trans[:n])
        st.rk = [st._key_rep(np.asarray(kr[c * C:(c + 1) * C], np.float32)) for c in range(n)]
        for t in range(n * C, T):
            st.buf.append((q[t], k[t], v[t], alpha[t], beta[t], qr[t], kr[t]))
        return st

    def _key_rep(self, krs):
        """Key representative(s) of one closed chunk's C route keys."""
        if self.window:
            return window_pools(krs, self.C, self.window, self.tau)[0]
        return rr.lme_pool32(krs, self.tau)

    def gates(self):
        """Raw binary32 gates of the partial chunk against all cached chunks."""
        n = len(self.trans)
        if n == 0:
            return np.zeros(0, np.float32)
        if self.mode == GATES_ONE:
            return np.ones(n, np.float32)
        if self.mode == GATES_ZERO:
            return np.zeros(n, np.float32)
        qr = np.stack([np.asarray(b[5], np.float32) for b in self.buf])
        rq = rr.lme_pool32(qr, self.tau)
        if self.window:
            return rr.gate_window32(rq[None, :], np.stack(self.rk), self.dk, self.bias)
        return rr.gate32(rq[None, :], np.stack(self.rk), self.dk, self.bias)

    def active(self, g):
        js = np.arange(len(g))
        if self.thr > 0:
            js = js[g >= np.float32(self.thr)]
        return js

    def step(self, q, k, v, alpha, beta, q_route=None, k_route=None):
        qr = q if q_route is None else q_route
        kr = k if k_route is None else k_route
        self.buf.append((q, k, v, alpha, beta, qr, kr))
        g = self.gates()
        act = self.active(g)
        S = np.zeros((self.dv, self.dk))
        for j in act:
            A, B = self.trans[j]
            S = S + float(g[j]) * ((S @ A + B) - S)
        for (_q, _k, _v, _a, _b, _qr, _kr) in self.buf:
            S = gdn_token_step(S, np.asarray(_k, np.float64), np.asarray(_v, np.float64),
                               _alpha_of(_a), float(_b))
        o = S @ np.asarray(q, np.float64)
        if len(self.buf) == self.C:
            self.close_chunk()
        return o

    def close_chunk(self):
        ks = np.stack([np.asarray(b[1], np.float64) for b in self.buf])
        vs = np.stack([np.asarray(b[2], np.float64) for b in self.buf])
        al = np.array([_alpha_of(b[3]) for b in self.buf])
        be = np.array([float(b[4]) for b in self.buf])
        krs = np.stack([np.asarray(b[6], np.float32) for b in self.buf])
        self.trans.append(chunk_transition(ks, vs, al, be))
        self.rk.append(self._key_rep(krs))
        self.buf = []


def decode_output_backward(trans, g, active, xq, y0):
    """Reassociated decode read-out (the form the GPU uses), for cross-checks:
    S_in x = sum_j g_j B_j prod_{l>j} ((1-g_l) I + g_l A_l) x, evaluated right to left:
    for j in active, descending: y += g_j B_j x; x <- (1-g_j) x + g_j A_j x.
    Returns y + y0."""
    x = np.asarray(xq, np.float64).copy()
    y = np.zeros(trans[0][1].shape[0]) if trans else np.zeros_like(x)
    for j in sorted(active, reverse=True):
        A, B = trans[j]
        gj = float(g[j])
        y = y + gj * (B @ x)
        x = (1.0 - gj) * x + gj * (A @ x)
    return y + y0
