"""Seeded synthetic inputs for HLA prefill and decode.

This module holds input generators only -- none of the method's arithmetic -- and
is the one piece shared by the oracle-side tests, the GPU tests and ``bench.py``.

All tensors use the layouts of the C ABI: q, k, v, route inputs ``[B, T, H, d]``;
alpha, beta ``[B, T, H]`` float32.  Value distributions:

* q, k ~ N(0, 1), then L2-normalised per token (unit keys keep I - beta k k^T a
  contraction); v ~ N(0, 1);
* alpha_t = exp(-softplus(N(0,1) - 3)), beta_t = sigmoid(N(0,1)); with channel-wise
  decay alpha_t is a vector over the key channels, each entry drawn the same way;
* bf16 workloads round q, k, v (and route inputs) to bf16 after normalisation
  (round to nearest even); alpha, beta stay float32.

Route inputs (the "projected query" the router compares against the chunk
representatives) are optional and default to q and k.  Two recipes make the gates
non-trivial:

* ``spread``: per chunk and head a centre mu ~ N(0, 2 I) plus per-token noise
  N(0, 0.25 I); with bias -2 the gates spread over (0, 1).
* ``planted``: every chunk j gets a topic c_j ~ U{0..P-1}; its route tokens are
  s e_{c_j} + 0.1 N(0, I) with s = 9.51 (s^2 / sqrt(128) = 8); with bias -4 same-topic
  pairs give g ~ 0.98 and the rest g ~ 0.018.

Generation uses ``torch.Generator`` seeded with the workload's seed, on the CPU by
default; very large workloads may be generated on the GPU (``device='cuda'``) --
those values differ from the CPU stream and tests that compare against the oracle
copy the sampled slices back to the host.
"""
from __future__ import annotations

from dataclasses import dataclass, replace
import math

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int
    C: int
    d: int
    dtype: str            # "f32" or "bf16"
    tau: float = 1.0
    bias: float = 0.0
    thr: float = 0.0
    gate_mode: str = "routed"   # routed | one | zero | user
    route: str = "default"      # default | spread | planted
    seed: int = 0
    topics: int = 128
    window: int = 0             # key window representatives of `window` tokens (0: one per chunk)
    decay: str = "scalar"       # scalar (one alpha per token) | channel (one per key channel)

    @property
    def N(self) -> int:
        return (self.T + self.C - 1) // self.C

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads (shapes and distributions as described above).
TINY_F32 = Workload("tiny_f32_B1_H2_T256_C64_d64", 1, 2, 256, 64, 64, "f32", 1.0, 0.0, 0.0, seed=0)
GDN_REDUCTION = Workload("gdn_reduction_bf16_B4_H16_T4096_C64_d128", 4, 16, 4096, 64, 128, "bf16",
                         1.0, 0.0, 0.0, gate_mode="one", seed=1)
PREFILL_0P8B = Workload("prefill_bf16_B1_H16_T16384_C64_d128_dense", 1, 16, 16384, 64, 128, "bf16",
                        1.0, -2.0, 0.0, route="spread", seed=2)
DECODE_32K = Workload("decode_bf16_64seq_ctx32768_H16_C64_d128_thr0.05", 64, 16, 32768, 64, 128, "bf16",
                      1.0, -2.0, 0.05, seed=3)
SPARSE_LONG = Workload("sparse_prefill_bf16_B1_H32_T131072_C64_d128_thr0.05", 1, 32, 131072, 64, 128,
                       "bf16", 1.0, -4.0, 0.05, route="planted", seed=5)
# The decode step of DECODE_32K with planted route inputs (the recipe of SPARSE_LONG):
# the open chunk matches about 512 / 128 = 4 of the 512 cached chunks.
DECODE_32K_PLANTED = Workload("decode_bf16_64seq_ctx32768_H16_C64_d128_thr0.05_planted", 64, 16, 32768, 64, 128,
                              "bf16", 1.0, -4.0, 0.05, route="planted", seed=4)

WORKLOADS = {w.name: w for w in (TINY_F32, GDN_REDUCTION, PREFILL_0P8B, DECODE_32K, SPARSE_LONG,
                                 DECODE_32K_PLANTED)}


def torch_dtype(w: Workload):
    return torch.float32 if w.dtype == "f32" else torch.bfloat16


def _l2n(x):
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)


def make_gdn_inputs(w: Workload, T: int | None = None, B: int | None = None, device="cpu",
                    seed: int | None = None):
    """q, k, v [B,T,H,d] (workload dtype), alpha [B,T,H] (or [B,T,H,d] with channel-wise
    decay) and beta [B,T,H] float32."""
    T = w.T if T is None else T
    B = w.B if B is None else B
    g = torch.Generator(device=device)
    g.manual_seed(w.seed if seed is None else seed)
    shape = (B, T, w.H, w.d)
    q = _l2n(torch.randn(shape, generator=g, device=device))
    k = _l2n(torch.randn(shape, generator=g, device=device))
    v = torch.randn(shape, generator=g, device=device)
    a_raw = torch.randn((B, T, w.H), generator=g, device=device)
    b_raw = torch.randn((B, T, w.H), generator=g, device=device)
    if w.decay == "channel":
        a_raw = torch.randn((B, T, w.H, w.d), generator=g, device=device)
    alpha = torch.exp(-torch.nn.functional.softplus(a_raw - 3.0)).float()
    beta = torch.sigmoid(b_raw).float()
    dt = torch_dtype(w)
    return dict(q=q.to(dt), k=k.to(dt), v=v.to(dt), alpha=alpha.contiguous(), beta=beta.contiguous())


def make_route_inputs(w: Workload, T: int | None = None, B: int | None = None, device="cpu",
                      seed: int | None = None):
    """q_route, k_route [B,T,H,d] or (None, None) for the default (route = q, k)."""
    T = w.T if T is None else T
    B = w.B if B is None else B
    if w.route == "default":
        return None, None
    g = torch.Generator(device=device)
    g.manual_seed((w.seed if seed is None else seed) + 1000003)
    N = (T + w.C - 1) // w.C
    dt = torch_dtype(w)
    shape = (B, T, w.H, w.d)
    # chunk id of each token
    cid = torch.arange(T, device=device) // w.C
    if w.route == "spread":
        outs = []
        for _ in range(2):
            mu = torch.randn((B, N, w.H, w.d), generator=g, device=device) * math.sqrt(2.0)
            eps = torch.randn(shape, generator=g, device=device) * 0.5
            outs.append((mu[:, cid] + eps).to(dt))
        return outs[0], outs[1]
    if w.route == "planted":
        s = 9.51
        topic = torch.randint(0, w.topics, (B, N, w.H), generator=g, device=device)
        onehot = torch.nn.functional.one_hot(topic, w.d).float() * s   # [B,N,H,d]
        outs = []
        for _ in range(2):
            eps = torch.randn(shape, generator=g, device=device) * 0.1
            outs.append((onehot[:, cid] + eps).to(dt))
        return outs[0], outs[1]
    raise ValueError(w.route)


def make_user_gates(w: Workload, device="cpu", seed: int | None = None):
    """Fixed (input-independent) chunk weights [B,H,N,N] in (0,1), float32."""
    g = torch.Generator(device=device)
    g.manual_seed((w.seed if seed is None else seed) + 7919)
    return torch.rand((w.B, w.H, w.N, w.N), generator=g, device=device).float()


def make_decode_tokens(w: Workload, steps: int, device="cpu", seed: int | None = None):
    """Per-step new tokens: list of dicts with q, k, v [B,H,d], alpha [B,H] (or [B,H,d]
    with channel-wise decay), beta [B,H].  With planted route inputs each dict also
    holds q_route, k_route [B,H,d] (see ``make_decode_route_tokens``)."""
    g = torch.Generator(device=device)
    g.manual_seed((w.seed if seed is None else seed) + 4242)
    dt = torch_dtype(w)
    out = []
    for _ in range(steps):
        q = _l2n(torch.randn((w.B, w.H, w.d), generator=g, device=device))
        k = _l2n(torch.randn((w.B, w.H, w.d), generator=g, device=device))
        v = torch.randn((w.B, w.H, w.d), generator=g, device=device)
        a = torch.exp(-torch.nn.functional.softplus(
            torch.randn((w.B, w.H) + ((w.d,) if w.decay == "channel" else ()), generator=g, device=device)
            - 3.0)).float()
        b = torch.sigmoid(torch.randn((w.B, w.H), generator=g, device=device)).float()
        out.append(dict(q=q.to(dt), k=k.to(dt), v=v.to(dt), alpha=a, beta=b))
    if w.route == "planted":
        for tok, (qr, kr) in zip(out, make_decode_route_tokens(w, steps, device=device, seed=seed)):
            tok["q_route"], tok["k_route"] = qr, kr
    return out


def make_decode_route_tokens(w: Workload, steps: int, device="cpu", seed: int | None = None):
    """Planted route inputs of the decode tokens that follow a w.T-token context:
    list of (q_route, k_route) [B,H,d].  Token t of the decode (position w.T + t)
    belongs to chunk (w.T + t) // C; each such chunk gets a topic c ~ U{0..topics-1}
    per (sequence, head), and its route tokens are s e_c + 0.1 N(0, I) (s = 9.51),
    the recipe of ``make_route_inputs``."""
    assert w.route == "planted", w.route
    g = torch.Generator(device=device)
    g.manual_seed((w.seed if seed is None else seed) + 2718281)
    dt = torch_dtype(w)
    s = 9.51
    first = w.T // w.C
    n_chunks = (w.T + steps - 1) // w.C - first + 1
    topic = torch.randint(0, w.topics, (n_chunks, w.B, w.H), generator=g, device=device)
    onehot = torch.nn.functional.one_hot(topic, w.d).float() * s   # [n_chunks, B, H, d]
    out = []
    for t in range(steps):
        c = (w.T + t) // w.C - first
        pair = []
        for _ in range(2):
            eps = torch.randn((w.B, w.H, w.d), generator=g, device=device) * 0.1
            pair.append((onehot[c] + eps).to(dt))
        out.append((pair[0], pair[1]))
    return out


def make_context_group(w: Workload, b0: int, nb: int, device="cuda"):
    """Decode context (prompt) of sequences b0 .. b0+nb-1, generated on ``device``
    with a generator seeded by (seed, b0): q, k, v [nb, T, H, d], alpha, beta
    [nb, T, H]; with spread or planted route inputs also q_route, k_route
    [nb, T, H, d] (``make_route_inputs`` seeded by (seed, b0)).  Used to build large
    decode caches group by group."""
    g = torch.Generator(device=device)
    g.manual_seed(w.seed * 1000003 + b0)
    shape = (nb, w.T, w.H, w.d)
    dt = torch_dtype(w)
    q = _l2n(torch.randn(shape, generator=g, device=device)).to(dt)
    k = _l2n(torch.randn(shape, generator=g, device=device)).to(dt)
    v = torch.randn(shape, generator=g, device=device).to(dt)
    a_raw = torch.randn((nb, w.T, w.H), generator=g, device=device)
    b_raw = torch.randn((nb, w.T, w.H), generator=g, device=device)
    if w.decay == "channel":
        a_raw = torch.randn((nb, w.T, w.H, w.d), generator=g, device=device)
    alpha = torch.exp(-torch.nn.functional.softplus(a_raw - 3.0)).float()
    beta = torch.sigmoid(b_raw).float()
    out = dict(q=q, k=k, v=v, alpha=alpha, beta=beta)
    if w.route != "default":
        out["q_route"], out["k_route"] = make_route_inputs(w, B=nb, device=device, seed=w.seed * 1000003 + b0 + 17)
    return out
