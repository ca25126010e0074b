"""C ABI checks that need no GPU: the library loads, exports every symbol that
include/hla.h declares, sizes its cache and workspaces by the stated arithmetic,
and rejects bad arguments on the host before any launch."""
import ctypes
import json
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hla.h")


@pytest.fixture(scope="module")
def hla():
    from gated_delta_rule_transitions_b200 import _hla
    from gated_delta_rule_transitions_b200 import build as b
    b.build()
    return _hla


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^[A-Za-z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(", src, flags=re.M)
    return sorted(set(n for n in names if n not in ("defined",)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("gdn_chunk_transitions", "hla_prefill", "hla_decode_step", "hla_routing",
              "hla_prefill_workspace_bytes", "hla_cache_bytes", "hla_cache_init",
              "hla_decode_workspace_bytes", "hla_last_error", "hla_device_status"):
        assert n in names


def test_library_exports_every_declared_symbol(hla):
    L = hla.lib()
    for n in declared_functions():
        assert hasattr(L, n), n
    assert set(hla.EXPORTS) <= set(declared_functions())


def cfg(hla, **kw):
    base = dict(B=1, H=1, T=4096, C=64, d=128, dtype="bf16")
    base.update(kw)
    return hla.make_config(**base)


def test_cache_bytes_match_affine_state_arithmetic(hla):
    """Main Findings (affine-state memory): the per-chunk A and B, d x d each at 2
    bytes, reproduce the page's 2 MiB KV figure and its 100/50/25/12.5% table."""
    gold = json.load(open(os.path.join(ROOT, "tests", "golden", "affine_state_memory.json")))
    d = gold["head_dim"]
    c = cfg(hla, d=d)
    per_chunk = hla.cache_bytes(c, 101) - hla.cache_bytes(c, 100)
    rk_bytes = d * 4  # float32 key pool per chunk (routing only)
    ab_bytes = per_chunk - rk_bytes
    assert ab_bytes == 2 * d * d * 2
    kv = gold["context_tokens"] * 2 * d * 2
    assert kv == gold["kv_cache_bytes_per_layer_head"]
    for C, frac in gold["affine_state_fraction_of_kv"].items():
        chunks = gold["context_tokens"] // int(C)
        assert chunks * ab_bytes / kv == pytest.approx(frac, abs=0)
    # float32 storage doubles the A/B part
    c32 = cfg(hla, d=d, dtype="f32")
    assert hla.cache_bytes(c32, 101) - hla.cache_bytes(c32, 100) - rk_bytes == 2 * d * d * 4


def test_decode_workspace_and_cache_sizes(hla):
    c = hla.make_config(64, 16, 1, 64, 128, "bf16")
    # config of a 64-sequence, 512-chunk decode: 32 GiB of A/B
    nb = hla.cache_bytes(c, 512)
    assert nb >= 64 * 16 * 512 * 2 * 128 * 128 * 2
    assert nb < 64 * 16 * 512 * 2 * 128 * 128 * 2 * 1.02
    # active lists and gates per (sequence, head, chunk), one list length per (sequence, head)
    assert hla.decode_workspace_bytes(c, 512) == 2 * 64 * 16 * 512 * 4 + 64 * 16 * 4


def test_prefill_workspace_grows_with_T(hla):
    a = hla.prefill_workspace_bytes(cfg(hla, T=1024))
    b = hla.prefill_workspace_bytes(cfg(hla, T=2048))
    assert 0 < a < b


@pytest.mark.parametrize("kw,status", [
    (dict(C=32), 2), (dict(C=96), 2), (dict(C=512), 2), (dict(d=96), 2), (dict(T=0), 1), (dict(B=0), 1),
    (dict(tau=0.0), 1),
])
def test_bad_config_rejected_on_host(hla, kw, status):
    c = cfg(hla, **kw)
    P = ctypes.c_void_p(0x100000)
    st = hla.lib().gdn_chunk_transitions(ctypes.byref(c), P, P, P, P, P, P, None)
    assert st == status
    assert hla.last_error() != ""
    assert hla.prefill_workspace_bytes(c) == 0


def test_null_and_misaligned_pointers_rejected(hla):
    c = cfg(hla, T=256)
    P = ctypes.c_void_p(0x100000)
    L = hla.lib()
    assert L.gdn_chunk_transitions(ctypes.byref(c), None, P, P, P, P, P, None) == hla.HLA_ERR_INVALID_ARG
    assert "k is NULL" in hla.last_error()
    bad = ctypes.c_void_p(0x100008)
    assert L.gdn_chunk_transitions(ctypes.byref(c), P, bad, P, P, P, P, None) == hla.HLA_ERR_INVALID_ARG
    assert "aligned" in hla.last_error()


def test_small_workspace_rejected_before_launch(hla):
    c = cfg(hla, T=256)
    P = ctypes.c_void_p(0x100000)
    need = hla.prefill_workspace_bytes(c)
    st = hla.lib().hla_prefill(ctypes.byref(c), P, P, P, P, P, None, None, None, P, None, None, None, None,
                               P, need - 256, None)
    assert st == hla.HLA_ERR_WORKSPACE
    assert "workspace too small" in hla.last_error()


def test_user_gates_required_in_user_mode(hla):
    c = cfg(hla, T=256, gate_mode="user")
    P = ctypes.c_void_p(0x100000)
    st = hla.lib().hla_prefill(ctypes.byref(c), P, P, P, P, P, None, None, None, P, None, None, None, None,
                               P, 1 << 40, None)
    assert st == hla.HLA_ERR_INVALID_ARG and "user_gates" in hla.last_error()


def test_decode_rejects_user_gates_and_foreign_cache(hla):
    c = cfg(hla, T=1, gate_mode="user")
    P = ctypes.c_void_p(0x100000)
    cache = hla.HlaCache()
    st = hla.lib().hla_decode_step(ctypes.byref(c), ctypes.byref(cache), P, P, P, P, P, None, None, P, P, 1 << 30,
                                   None)
    assert st == hla.HLA_ERR_UNSUPPORTED
    c = cfg(hla, T=1)
    st = hla.lib().hla_decode_step(ctypes.byref(c), ctypes.byref(cache), P, P, P, P, P, None, None, P, P, 1 << 30,
                                   None)
    assert st == hla.HLA_ERR_INVALID_ARG and "different config" in hla.last_error()


def test_python_binding_refuses_cpu_tensors(hla):
    import torch
    c = cfg(hla, T=64, d=64, dtype="f32")
    x = torch.zeros(1, 64, 1, 64)
    with pytest.raises(ValueError, match="CUDA"):
        hla.gdn_chunk_transitions(c, x, x, x[..., 0], x[..., 0], x, x)


def test_static_decode_rejects_scratch_beyond_its_array(hla):
    """hla_decode_step_static has 8 MiB of fixed scratch (8 B per sequence, head and
    cached chunk, plus 4 B per sequence and head); a larger cache is refused on the
    host (the fake aligned pointers are never read)."""
    c = cfg(hla, B=64, H=16, T=1)
    cache = hla.HlaCache()
    cache.B, cache.H, cache.C, cache.d, cache.dtype = 64, 16, 64, 128, 1
    cache.max_chunks = (1 << 20) // (64 * 16) + 1
    for f in ("A", "Bm", "rk", "buf_k", "buf_v", "buf_qr", "buf_kr", "buf_alpha", "buf_beta", "n_chunks",
              "m_partial"):
        setattr(cache, f, 256)
    P = ctypes.c_void_p(256)
    st = hla.lib().hla_decode_step_static(ctypes.byref(c), ctypes.byref(cache), P, P, P, P, P, None, None, P,
                                          None)
    assert st == hla.HLA_ERR_WORKSPACE and "static array" in hla.last_error()


def test_bounded_wait_check_limit_checked_on_host(hla):
    for bad in (0, 100001):
        st = hla.lib().hla_check_bounded_wait(bad, 0, None)
        assert st == hla.HLA_ERR_INVALID_ARG and "limit_us" in hla.last_error()


def test_cache_slice_offsets_follow_the_sequence_major_layout(hla):
    """hla_cache_slice advances every buffer by b0 sequences of the layout that
    include/hla.h documents ([B, H, max_chunks, d, d] A/Bm, [B, H, max_chunks, d]
    key pools, [B, H, C, d] / [B, H, C] open-chunk buffers, [B] counters)."""
    c = hla.HlaCache()
    c.B, c.H, c.C, c.d, c.dtype, c.max_chunks = 4, 2, 64, 128, 1, 3
    fields = ("A", "Bm", "rk", "buf_k", "buf_v", "buf_qr", "buf_kr", "buf_alpha", "buf_beta", "n_chunks",
              "m_partial")
    for i, f in enumerate(fields):
        setattr(c, f, (i + 1) << 32)
    out = hla.HlaCache()
    assert hla.lib().hla_cache_slice(ctypes.byref(c), 2, 2, ctypes.byref(out)) == hla.HLA_OK
    per_seq = {"A": 2 * 3 * 128 * 128 * 2, "Bm": 2 * 3 * 128 * 128 * 2, "rk": 2 * 3 * 128 * 4,
               "buf_k": 2 * 64 * 128 * 2, "buf_v": 2 * 64 * 128 * 2, "buf_qr": 2 * 64 * 128 * 2,
               "buf_kr": 2 * 64 * 128 * 2, "buf_alpha": 2 * 64 * 4, "buf_beta": 2 * 64 * 4, "n_chunks": 4,
               "m_partial": 4}
    assert out.B == 2 and out.H == 2 and out.max_chunks == 3
    for i, f in enumerate(fields):
        assert getattr(out, f) == ((i + 1) << 32) + 2 * per_seq[f], f
    for b0, nb in ((-1, 1), (0, 0), (3, 2), (4, 1)):
        assert hla.lib().hla_cache_slice(ctypes.byref(c), b0, nb, ctypes.byref(out)) == hla.HLA_ERR_INVALID_ARG


def test_factored_cache_sizes_and_slices(hla):
    """A factored cache stores K_j, Wb_j, Ub_j (C x d each) and C + 4 float32 scales
    per closed chunk instead of the two d x d matrices."""
    dense = cfg(hla, B=2, H=3, T=1)
    fact = cfg(hla, B=2, H=3, T=1, cache_format="factored")
    mc = 5
    per_chunk_dense = 2 * 128 * 128 * 2
    per_chunk_fact = 3 * 64 * 128 * 2 + (64 + 4) * 4
    diff = hla.cache_bytes(dense, mc) - hla.cache_bytes(fact, mc)
    # the rest of the layout is identical; 256-byte alignment of 2 vs 4 sub-buffers
    assert abs(diff - 2 * 3 * mc * (per_chunk_dense - per_chunk_fact)) <= 4 * 256
    c = hla.HlaCache()
    c.B, c.H, c.C, c.d, c.dtype, c.max_chunks, c.format = 4, 2, 64, 128, 1, 3, 1
    for i, f in enumerate(("Kf", "Wf", "Uf", "df")):
        setattr(c, f, (i + 1) << 32)
    for f in ("rk", "buf_k", "buf_v", "buf_qr", "buf_kr", "buf_alpha", "buf_beta", "n_chunks", "m_partial"):
        setattr(c, f, 1 << 40)
    out = hla.HlaCache()
    assert hla.lib().hla_cache_slice(ctypes.byref(c), 1, 2, ctypes.byref(out)) == hla.HLA_OK
    assert out.Kf == (1 << 32) + 2 * 3 * 64 * 128 * 2
    assert out.df == (4 << 32) + 2 * 3 * 68 * 4
    assert not out.A and not out.Bm


def test_factored_cache_needs_bf16_d128(hla):
    c = cfg(hla, B=1, H=1, T=1, d=64, dtype="f32", cache_format="factored")
    out = hla.HlaCache()
    st = hla.lib().hla_cache_init(ctypes.byref(c), 4, ctypes.c_void_p(1 << 20), 1 << 30, ctypes.byref(out), None)
    assert st == hla.HLA_ERR_UNSUPPORTED and "factored" in hla.last_error()


@pytest.mark.parametrize("C", [128, 256])
def test_long_chunks_accepted(hla, C):
    """Chunks of 128 and 256 tokens (the pages' default is 256): the prefill workspace
    holds the gates of N = T / C chunks and the transitions of the T / 64 sub-chunks."""
    T = 4096
    c = cfg(hla, T=T, C=C)
    ws = hla.prefill_workspace_bytes(c)
    assert ws > 0
    N, d = T // C, 128
    # at least: A/B of the chunks and of the sub-chunks (bf16), the state entering
    # every sub-chunk and the gate rows of the chunks
    assert ws >= (N + T // 64) * 2 * d * d * 2 + (T // 64) * d * d * 4 + 2 * N * N * 4
    assert hla.cache_bytes(c, 8) > 0
    # the decode cache holds C-token buffers of the open chunk
    c64 = cfg(hla, T=1, C=64)
    cC = cfg(hla, T=1, C=C)
    assert hla.cache_bytes(cC, 8) - hla.cache_bytes(c64, 8) >= 4 * (C - 64) * d * 2


def test_factored_cache_needs_c64(hla):
    c = cfg(hla, B=1, H=1, T=1, C=128, cache_format="factored")
    out = hla.HlaCache()
    st = hla.lib().hla_cache_init(ctypes.byref(c), 4, ctypes.c_void_p(1 << 20), 1 << 30, ctypes.byref(out), None)
    assert st == hla.HLA_ERR_UNSUPPORTED and "C = 64" in hla.last_error()


def test_gate_support_needs_an_output(hla):
    c = cfg(hla, T=256)
    P = ctypes.c_void_p(0x100000)
    st = hla.lib().hla_gate_support(ctypes.byref(c), P, None, None, None)
    assert st == hla.HLA_ERR_INVALID_ARG and "both NULL" in hla.last_error()
    st = hla.lib().hla_gate_support(ctypes.byref(c), None, P, P, None)
    assert st == hla.HLA_ERR_INVALID_ARG and "gates is NULL" in hla.last_error()


@pytest.mark.parametrize("C,w,ok", [(64, 32, True), (64, 16, True), (256, 32, True), (256, 16, True),
                                    (256, 8, False), (64, 64, False), (64, 4, False), (64, 48, False)])
def test_pool_window_shapes(hla, C, w, ok):
    """Window representatives: 8 <= w < C, w divides C, at most 16 windows per chunk."""
    c = cfg(hla, T=1024, C=C, pool_window=w)
    assert (hla.prefill_workspace_bytes(c) > 0) == ok
    if not ok:
        P = ctypes.c_void_p(0x100000)
        assert hla.lib().gdn_chunk_transitions(ctypes.byref(c), P, P, P, P, P, P, None) == hla.HLA_ERR_UNSUPPORTED
        assert "pool_window" in hla.last_error()


def test_window_pools_enlarge_the_key_cache(hla):
    d = 128
    base = cfg(hla, T=1, C=256)
    win = cfg(hla, T=1, C=256, pool_window=32)
    per_chunk = lambda c: hla.cache_bytes(c, 101) - hla.cache_bytes(c, 100)
    assert per_chunk(win) - per_chunk(base) == 7 * d * 4   # 8 window pools instead of one


def test_decay_mode_checks(hla):
    assert hla.prefill_workspace_bytes(cfg(hla, T=1024, decay="channel")) > 0
    assert hla.prefill_workspace_bytes(cfg(hla, T=1024, decay=2)) == 0
    # channel-wise decay keeps d decays per buffered token in the decode cache
    d = 128
    c1 = cfg(hla, T=1, C=64)
    c2 = cfg(hla, T=1, C=64, decay="channel")
    assert hla.cache_bytes(c2, 8) - hla.cache_bytes(c1, 8) >= 64 * (d - 1) * 4
    out = hla.HlaCache()
    c3 = cfg(hla, B=1, H=1, T=1, decay="channel", cache_format="factored")
    st = hla.lib().hla_cache_init(ctypes.byref(c3), 4, ctypes.c_void_p(1 << 20), 1 << 30, ctypes.byref(out), None)
    assert st == hla.HLA_ERR_UNSUPPORTED and "scalar decay" in hla.last_error()


@pytest.mark.parametrize("window,decay", [(32, 0), (0, 1), (16, 1)])
def test_cache_slice_offsets_with_windows_and_channel_decay(hla, window, decay):
    """Window representatives keep C / w key pools per closed chunk and channel-wise
    decay keeps d decays per buffered token; a slice advances those buffers by b0
    sequences of the larger layouts (C = 64, d = 128, bf16)."""
    c = hla.HlaCache()
    c.B, c.H, c.C, c.d, c.dtype, c.max_chunks = 4, 2, 64, 128, 1, 3
    c.pool_window, c.decay_mode = window, decay
    fields = ("A", "Bm", "rk", "buf_k", "buf_v", "buf_qr", "buf_kr", "buf_alpha", "buf_beta", "n_chunks",
              "m_partial")
    for i, f in enumerate(fields):
        setattr(c, f, (i + 1) << 32)
    out = hla.HlaCache()
    assert hla.lib().hla_cache_slice(ctypes.byref(c), 1, 3, ctypes.byref(out)) == hla.HLA_OK
    reps = 64 // window if window else 1
    adim = 128 if decay else 1
    per_seq = {"A": 2 * 3 * 128 * 128 * 2, "Bm": 2 * 3 * 128 * 128 * 2, "rk": 2 * 3 * reps * 128 * 4,
               "buf_k": 2 * 64 * 128 * 2, "buf_v": 2 * 64 * 128 * 2, "buf_qr": 2 * 64 * 128 * 2,
               "buf_kr": 2 * 64 * 128 * 2, "buf_alpha": 2 * 64 * adim * 4, "buf_beta": 2 * 64 * 4,
               "n_chunks": 4, "m_partial": 4}
    for i, f in enumerate(fields):
        assert getattr(out, f) == ((i + 1) << 32) + per_seq[f], f
    # the cache block grows by exactly those buffers
    base = hla.cache_bytes(cfg(hla, B=4, H=2, T=1, C=64), 3)
    grown = hla.cache_bytes(cfg(hla, B=4, H=2, T=1, C=64, pool_window=window, decay=decay), 3)
    assert grown - base >= 4 * (per_seq["rk"] - 2 * 3 * 128 * 4) + 4 * (per_seq["buf_alpha"] - 2 * 64 * 4)
