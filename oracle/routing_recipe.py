"""Oracle, part 2: the bit-level fp32 routing recipe (log-mean-exp pools and gates).

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import this module;
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` do.

Source passages
---------------
* HLA (ai.info summary of "HLA: Expressive Hybrid Linear Attention via Chunk-Wise
  Dynamic Mixing"), "Overview": the routing gates are *log-mean-exp pooled*.
* Same page, "Methodology in Plain English": a query is compared against the chunk
  representatives and the score is squashed through a sigmoid, giving one weight in
  (0, 1) per historical chunk; the weights are independent sigmoids, not a
  normalised distribution; at inference a historical weight below a threshold is
  set to zero without renormalisation.

Reading taken: the representative of chunk c is the per-channel pool
``r = tau * log(mean_t exp(x_t / tau))`` over the chunk's route tokens, and the gate
is ``g_ij = sigmoid(<r^q_i, r^k_j> / sqrt(d) + b)``.

Why a bit-level recipe
----------------------
Gates decide which chunks are skipped, so the CPU and the GPU must take that
decision on identical bits.  The recipe below uses only IEEE-754 binary32 operations
that are correctly rounded: +, -, *, /, the fused multiply-add ``fma(a, b, c)``
(``a*b + c`` rounded once), and exact scaling by powers of two.  Every conforming
implementation of the same sequence of operations therefore produces the same bits.
``fma32`` below is that operation, emulated exactly with float64 arithmetic.
``exp`` and ``log`` are written here from their mathematical definitions:

* ``exp32`` -- Cody & Waite argument reduction ``x = n*ln2 + r``: ``n`` is the
  integer nearest (ties to even) to the exact product ``x*log2e``; ``r`` is
  ``fma(-n, ln2_lo, fma(-n, ln2_hi, x))`` with ``ln 2`` split into a
  16-significant-bit head and a tail; then the degree-7 Taylor polynomial of
  ``e^r`` in Horner form, one fma per step; then exact scaling by ``2^n``.  Inputs
  above 88 give +inf, inputs below -86 give 0 (so no subnormal result is ever
  formed).
* ``log32`` -- split ``x = m * 2^e`` with ``m`` in [sqrt(1/2), sqrt(2)), then
  ``log m = 2 atanh(f)``, ``f = (m-1)/(m+1)``, summed as the odd series up to f^15
  with separately rounded products and sums, plus ``e*ln2`` (head exact, tail
  rounded).

Constants are derived below from the mathematics (``1/k!``, ``1/(2k+1)``, ``ln 2``),
each rounded once to binary32.

The pooled values, dot products and gates returned here are the reference bits that
the GPU routing must reproduce exactly.
"""
from __future__ import annotations

import math

import numpy as np

F32 = np.float32

# ---- constants, from the mathematics, each rounded once to binary32 ----------------

_LN2 = math.log(2.0)  # double-precision ln 2


def _ln2_split() -> tuple[np.float32, np.float32]:
    """Head of ln 2 with 16 significant bits (low 8 of 24 mantissa bits cleared),
    and the binary32 rounding of the remainder."""
    head_bits = np.array([_LN2], dtype=np.float32).view(np.uint32)[0] & np.uint32(0xFFFFFF00)
    head = np.array([head_bits], dtype=np.uint32).view(np.float32)[0]
    tail = F32(_LN2 - float(head))
    return F32(head), tail


LN2_HI, LN2_LO = _ln2_split()
LOG2E = F32(1.0 / _LN2)
EXP_COEF = [F32(1.0 / math.factorial(k)) for k in range(8)]  # 1/0! .. 1/7!
ODD_RECIP = [F32(1.0 / (2 * k + 1)) for k in range(8)]  # 1/1, 1/3, .., 1/15
SQRT_HALF = F32(math.sqrt(0.5))
EXP_HI = F32(88.0)
EXP_LO = F32(-86.0)


def _f32(x):
    return np.asarray(x, dtype=np.float32)


def fma32(a, b, c):
    """Binary32 fused multiply-add, elementwise: the exact a*b + c rounded once to
    nearest (ties to even).

    The product of two binary32 values is exact in float64 (48 significant bits).
    The float64 sum ``s`` is the float64 value nearest to the exact sum, and the
    exact remainder ``e = (a*b + c) - s`` follows from the two-sum identity.  No
    binary32 rounding boundary (a midpoint between neighbours) can lie strictly
    between the exact sum and ``s``, so rounding ``s`` to binary32 is already correct
    unless ``s`` sits exactly on a midpoint; there the exact sum is on the side given
    by the sign of ``e`` (or on the midpoint itself when ``e`` is zero, where ties go
    to the even neighbour, as the float64 -> binary32 conversion does).
    """
    a, b, c = np.broadcast_arrays(_f32(a), _f32(b), _f32(c))
    p = a.astype(np.float64) * b.astype(np.float64)
    c64 = c.astype(np.float64)
    s = p + c64
    bv = s - p
    e = (p - (s - bv)) + (c64 - bv)
    r = s.astype(np.float32)
    d = s - r.astype(np.float64)
    toward = np.where(d > 0, np.float32(np.inf), np.float32(-np.inf))
    nb = np.nextafter(r, toward)
    tie = (d != 0) & (s + s == r.astype(np.float64) + nb.astype(np.float64))
    fix = tie & (e != 0) & (np.sign(e) == np.sign(d))
    return np.where(fix, nb, r).astype(np.float32)


def exp32(x):
    """e^x on binary32 arrays by the recipe above (elementwise, vectorised)."""
    x = _f32(x)
    # nearest integer to the exact product (float64 holds it exactly)
    n = np.rint(x.astype(np.float64) * np.float64(LOG2E)).astype(np.float32)
    r = fma32(-n, LN2_LO, fma32(-n, LN2_HI, x))
    p = EXP_COEF[7]
    for c in EXP_COEF[6::-1]:
        p = fma32(p, r, c)  # one rounding per step
    ni = np.clip(n, -126, 127).astype(np.int32)
    scale = ((ni + 127).astype(np.uint32) << np.uint32(23)).view(np.float32)
    out = (p * scale).astype(np.float32)
    out = np.where(x > EXP_HI, F32(np.inf), out)
    out = np.where(x < EXP_LO, F32(0.0), out)
    return out.astype(np.float32)


def log32(x):
    """Natural log on positive normal binary32 arrays by the recipe above."""
    x = _f32(x)
    mant, e = np.frexp(x)  # mant in [0.5, 1), exact
    mant = mant.astype(np.float32)
    e = e.astype(np.int32)
    low = mant < SQRT_HALF
    mant = np.where(low, mant * F32(2.0), mant).astype(np.float32)
    e = np.where(low, e - 1, e)
    f = (mant - F32(1.0)) / (mant + F32(1.0))
    f2 = f * f
    p = ODD_RECIP[7]
    for c in ODD_RECIP[6:0:-1]:  # 1/13 .. 1/3
        p = p * f2 + c
    t = (f * f2) * p
    log_m = (f + t) * F32(2.0)
    ef = e.astype(np.float32)
    out = ef * LN2_HI + (log_m + ef * LN2_LO)
    return out.astype(np.float32)


def lme_pool32(x, tau: float, n_tokens=None):
    """Per-channel log-mean-exp pool over axis -2 (tokens) of a binary32 array.

    ``x``: [..., n, d].  Returns [..., d].  Steps, in order:
    inv_tau = 1/tau; m = max_t (x_t * inv_tau);
    s = sum over ascending t of exp32(fma(x_t, inv_tau, -m)), one rounding per add,
    starting at 0;  r = tau * (m + log32(s / n)).
    """
    x = _f32(x)
    n = x.shape[-2] if n_tokens is None else n_tokens
    tau32 = F32(tau)
    inv_tau = F32(1.0) / tau32
    y = x[..., :n, :] * inv_tau
    m = y[..., 0, :]
    for t in range(1, n):
        m = np.maximum(m, y[..., t, :])
    s = np.zeros_like(m)
    for t in range(n):
        s = s + exp32(fma32(x[..., t, :], inv_tau, -m))
    mean = s / F32(n)
    return (tau32 * (m + log32(mean))).astype(np.float32)


def gate_scale(d: int) -> np.float32:
    """c_d = 1/sqrt(d), computed in double and rounded once."""
    return F32(1.0 / math.sqrt(float(d)))


def dot32(a, b):
    """Sequential binary32 dot over the last axis: acc = 0; acc = fma(a[c], b[c], acc),
    c ascending (one rounding per step)."""
    a = _f32(a)
    b = _f32(b)
    a, b = np.broadcast_arrays(a, b)
    acc = np.zeros(a.shape[:-1], dtype=np.float32)
    for c in range(a.shape[-1]):
        acc = fma32(a[..., c], b[..., c], acc)
    return acc


def gate32(rq, rk, d: int, bias: float):
    """g = 1 / (1 + exp32(-z)), z = fma(dot32(rq, rk), c_d, bias), all binary32."""
    dot = dot32(rq, rk)
    z = fma32(dot, gate_scale(d), F32(bias))
    return (F32(1.0) / (F32(1.0) + exp32(-z))).astype(np.float32)


def gate_matrix32(rq, rk, d: int, bias: float):
    """All pairs: rq [N_q, d], rk [N_k, d] -> G [N_q, N_k] by the recipe (no masking)."""
    rq = _f32(rq)
    rk = _f32(rk)
    return gate32(rq[:, None, :], rk[None, :, :], d, bias)


def gate_window32(rq, rkw, d: int, bias: float):
    """Gate against a chunk summarised by W window representatives (the pages'
    log-sum-exp over a chunk's representatives, then a sigmoid).  rq [..., d],
    rkw [..., W, d].  Steps, all binary32:
    t_u = dot32(rq, rk_u) * c_d (one rounding); m = max_u t_u;
    s = sum over ascending u of exp32(t_u - m), one rounding per add, from 0;
    z = (m + log32(s)) + bias (two roundings); g = 1 / (1 + exp32(-z))."""
    rq = _f32(rq)
    rkw = _f32(rkw)
    t = (dot32(rq[..., None, :], rkw) * gate_scale(d)).astype(np.float32)
    m = t.max(axis=-1)
    s = np.zeros_like(m)
    for u in range(t.shape[-1]):
        s = (s + exp32((t[..., u] - m).astype(np.float32))).astype(np.float32)
    z = ((m + log32(s)).astype(np.float32) + F32(bias)).astype(np.float32)
    return (F32(1.0) / (F32(1.0) + exp32(-z))).astype(np.float32)


def gate_matrix_window32(rq, rkw, d: int, bias: float):
    """All pairs: rq [N_q, d], rkw [N_k, W, d] -> G [N_q, N_k] by gate_window32."""
    rq = _f32(rq)
    rkw = _f32(rkw)
    return gate_window32(rq[:, None, :], rkw[None, :, :, :], d, bias)


# ---- fp64 statements of the same quantities (to measure the recipe's own error) -----

def lme_pool64(x, tau: float):
    x = np.asarray(x, dtype=np.float64)
    return tau * np.log(np.mean(np.exp(x / tau), axis=-2))


def gate64(rq, rk, d: int, bias: float):
    rq = np.asarray(rq, dtype=np.float64)
    rk = np.asarray(rk, dtype=np.float64)
    z = np.sum(rq * rk, axis=-1) / math.sqrt(d) + bias
    return 1.0 / (1.0 + np.exp(-z))


def gate_window64(rq, rkw, d: int, bias: float):
    """sigmoid(log sum_u exp(<rq, rk_u> / sqrt(d)) + bias) in float64."""
    rq = np.asarray(rq, dtype=np.float64)
    rkw = np.asarray(rkw, dtype=np.float64)
    t = np.sum(rq[..., None, :] * rkw, axis=-1) / math.sqrt(d)
    m = t.max(axis=-1)
    z = m + np.log(np.sum(np.exp(t - m[..., None]), axis=-1)) + bias
    return 1.0 / (1.0 + np.exp(-z))
