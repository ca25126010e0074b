"""Oracle, part 3: brute force for tiny inputs, in pure Python (no numpy).

TEST INFRASTRUCTURE ONLY (same import rule as the rest of ``oracle/``).

Every per-token map is written out as an explicit matrix,
  M_t = alpha_t (I - beta_t k_t k_t^T)   (d_k x d_k; Diag(alpha_t)(...) for a
                                          channel-wise decay)
  N_t = beta_t v_t k_t^T                  (d_v x d_k)
so that the token rule is S_t = S_{t-1} M_t + N_t (HLA summary page, "Methodology in
Plain English": a matrix that decays and edits the old state plus an additive
write).  Chunk transitions are formed as explicit products of these matrices,
gated by interpolating with the identity, and the result is read out token by token.
Works on floats or ``fractions.Fraction`` (exact rational arithmetic).

This is deliberately a different computation from ``hla_oracle``: it never calls a
library matmul, and it builds the chunk transitions as products of per-token
matrices rather than by running the rule on a state.
"""
from __future__ import annotations


def _zeros(r, c, z):
    return [[z for _ in range(c)] for _ in range(r)]


def _eye(n, z, one):
    m = _zeros(n, n, z)
    for i in range(n):
        m[i][i] = one
    return m


def _mm(a, b, z):
    r, k, c = len(a), len(b), len(b[0])
    out = _zeros(r, c, z)
    for i in range(r):
        for j in range(c):
            acc = z
            for t in range(k):
                acc = acc + a[i][t] * b[t][j]
            out[i][j] = acc
    return out


def _add(a, b):
    return [[x + y for x, y in zip(ra, rb)] for ra, rb in zip(a, b)]


def _scale(s, a):
    return [[s * x for x in r] for r in a]


def _mv(a, x, z):
    out = []
    for row in a:
        acc = z
        for p, q in zip(row, x):
            acc = acc + p * q
        out.append(acc)
    return out


def token_matrices(k, v, alpha, beta, z, one):
    """Per-token (M_t, N_t) as explicit nested lists.  ``alpha`` is one number, or a
    list over the key channels (channel-wise decay: M_t = Diag(alpha)(I - beta k k^T),
    row r scaled by alpha[r])."""
    dk = len(k)
    M = _eye(dk, z, one)
    for r in range(dk):
        a_r = alpha[r] if isinstance(alpha, (list, tuple)) else alpha
        for c in range(dk):
            M[r][c] = a_r * (M[r][c] - beta * k[r] * k[c])
    N = [[beta * v[r] * k[c] for c in range(dk)] for r in range(len(v))]
    return M, N


def hla_brute(q, k, v, alpha, beta, C, gates, active=None, zero=0.0, one=1.0):
    """HLA output for one head by explicit per-token matrices.

    q, k: list of T lists (d_k); v: list of T lists (d_v); alpha, beta: lists of T;
    gates: gates[i][j] for j < i (the weights actually used, after thresholding);
    active: optional per-query-chunk iterable of j (default all j < i).
    Returns o as a list of T lists (d_v)."""
    T = len(k)
    dk = len(k[0])
    dv = len(v[0])
    N = (T + C - 1) // C
    # (A_c, B_c) as explicit products over each complete chunk.
    trans = []
    for c in range(T // C):
        A = _eye(dk, zero, one)
        Bm = _zeros(dv, dk, zero)
        for t in range(c * C, (c + 1) * C):
            M, Nt = token_matrices(k[t], v[t], alpha[t], beta[t], zero, one)
            A = _mm(A, M, zero)
            Bm = _add(_mm(Bm, M, zero), Nt)
        trans.append((A, Bm))
    o = []
    for i in range(N):
        S = _zeros(dv, dk, zero)
        js = range(i) if active is None else active[i]
        for j in js:
            g = gates[i][j]
            A, Bm = trans[j]
            # gated transition: S ((1-g) I + g A) + g B
            Ag = _add(_scale(one - g, _eye(dk, zero, one)), _scale(g, A))
            S = _add(_mm(S, Ag, zero), _scale(g, Bm))
        for t in range(i * C, min(T, (i + 1) * C)):
            M, Nt = token_matrices(k[t], v[t], alpha[t], beta[t], zero, one)
            S = _add(_mm(S, M, zero), Nt)
            o.append(_mv(S, q[t], zero))
    return o
