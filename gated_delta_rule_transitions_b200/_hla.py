"""ctypes binding of libhla.so (argument marshalling only).

Every function here forwards to the C entry point of the same name in
``include/hla.h``.  Tensors are passed as raw device pointers; PyTorch supplies
device memory and the current CUDA stream.  There is no CPU fallback: if the
library or a CUDA device is missing, calls raise.
"""
from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libhla.so")

HLA_OK = 0
HLA_ERR_INVALID_ARG = 1
HLA_ERR_UNSUPPORTED = 2
HLA_ERR_WORKSPACE = 3
HLA_ERR_CUDA = 4
HLA_ERR_TIMEOUT = 5
STATUS_NAMES = {0: "HLA_OK", 1: "HLA_ERR_INVALID_ARG", 2: "HLA_ERR_UNSUPPORTED", 3: "HLA_ERR_WORKSPACE",
                4: "HLA_ERR_CUDA", 5: "HLA_ERR_TIMEOUT"}

HLA_F32 = 0
HLA_BF16 = 1
HLA_CACHE_DENSE = 0
HLA_CACHE_FACTORED = 1
CACHE_FORMATS = {"dense": HLA_CACHE_DENSE, "factored": HLA_CACHE_FACTORED}
GATE_MODES = {"routed": 0, "one": 1, "zero": 2, "user": 3}
DECAY_MODES = {"scalar": 0, "channel": 1}


class HlaConfig(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("T", ctypes.c_int32), ("C", ctypes.c_int32),
                ("dk", ctypes.c_int32), ("dv", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("gate_mode", ctypes.c_int32), ("cache_format", ctypes.c_int32), ("tau", ctypes.c_float),
                ("bias", ctypes.c_float), ("skip_threshold", ctypes.c_float), ("pool_window", ctypes.c_int32),
                ("decay_mode", ctypes.c_int32)]


class HlaCache(ctypes.Structure):
    _fields_ = [("max_chunks", ctypes.c_int32), ("B", ctypes.c_int32), ("H", ctypes.c_int32),
                ("C", ctypes.c_int32), ("d", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("format", ctypes.c_int32), ("pool_window", ctypes.c_int32), ("decay_mode", ctypes.c_int32),
                ("A", ctypes.c_void_p), ("Bm", ctypes.c_void_p), ("Kf", ctypes.c_void_p), ("Wf", ctypes.c_void_p),
                ("Uf", ctypes.c_void_p), ("df", ctypes.c_void_p), ("rk", ctypes.c_void_p),
                ("buf_k", ctypes.c_void_p), ("buf_v", ctypes.c_void_p), ("buf_qr", ctypes.c_void_p),
                ("buf_kr", ctypes.c_void_p), ("buf_alpha", ctypes.c_void_p), ("buf_beta", ctypes.c_void_p),
                ("n_chunks", ctypes.c_void_p), ("m_partial", ctypes.c_void_p)]


class HlaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


_lib = None

_P = ctypes.c_void_p
_SIGS = {
    "hla_last_error": ([], ctypes.c_char_p),
    "hla_cache_bytes": ([ctypes.POINTER(HlaConfig), ctypes.c_int32], ctypes.c_size_t),
    "hla_cache_init": ([ctypes.POINTER(HlaConfig), ctypes.c_int32, _P, ctypes.c_size_t, ctypes.POINTER(HlaCache), _P],
                       ctypes.c_int),
    "hla_cache_slice": ([ctypes.POINTER(HlaCache), ctypes.c_int32, ctypes.c_int32, ctypes.POINTER(HlaCache)],
                        ctypes.c_int),
    "hla_prefill_workspace_bytes": ([ctypes.POINTER(HlaConfig)], ctypes.c_size_t),
    "hla_decode_workspace_bytes": ([ctypes.POINTER(HlaConfig), ctypes.c_int32], ctypes.c_size_t),
    "gdn_chunk_transitions": ([ctypes.POINTER(HlaConfig), _P, _P, _P, _P, _P, _P, _P], ctypes.c_int),
    "hla_routing": ([ctypes.POINTER(HlaConfig), _P, _P, _P, _P, _P, _P, _P, _P], ctypes.c_int),
    "hla_gate_support": ([ctypes.POINTER(HlaConfig), _P, _P, _P, _P], ctypes.c_int),
    "hla_prefill": ([ctypes.POINTER(HlaConfig), _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                     ctypes.POINTER(HlaCache), _P, ctypes.c_size_t, _P], ctypes.c_int),
    "hla_decode_step": ([ctypes.POINTER(HlaConfig), ctypes.POINTER(HlaCache), _P, _P, _P, _P, _P, _P, _P, _P, _P,
                         ctypes.c_size_t, _P], ctypes.c_int),
    "hla_decode_step_static": ([ctypes.POINTER(HlaConfig), ctypes.POINTER(HlaCache), _P, _P, _P, _P, _P, _P, _P,
                                _P, _P], ctypes.c_int),
    "hla_device_status": ([ctypes.c_int32, ctypes.POINTER(ctypes.c_uint32)], ctypes.c_int),
    "hla_check_bounded_wait": ([ctypes.c_uint32, ctypes.c_int32, _P], ctypes.c_int),
    "hla_profile_enable": ([ctypes.c_int32], ctypes.c_int),
    "hla_profile_read": ([_P, _P, ctypes.c_int32], ctypes.c_int),
}

STAGES = ("pools", "gates", "transitions", "compose", "readout", "cache", "decode", "decode_close", "chain")

# Every symbol that include/hla.h declares (checked by the CPU tests).
EXPORTS = tuple(_SIGS)


def lib():
    """Load libhla.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"libhla.so not built at {_LIB_PATH}; run "
                               "`python -m gated_delta_rule_transitions_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        for name, (args, res) in _SIGS.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def last_error() -> str:
    return lib().hla_last_error().decode()


def _check(status: int):
    if status != HLA_OK:
        raise HlaError(status, last_error())


def make_config(B, H, T, C=64, d=128, dtype="bf16", gate_mode="routed", tau=1.0, bias=0.0,
                skip_threshold=0.0, cache_format="dense", pool_window=0, decay="scalar") -> HlaConfig:
    dt = {"bf16": HLA_BF16, "f32": HLA_F32, torch.bfloat16: HLA_BF16, torch.float32: HLA_F32}[dtype]
    gm = GATE_MODES[gate_mode] if isinstance(gate_mode, str) else int(gate_mode)
    cf = CACHE_FORMATS[cache_format] if isinstance(cache_format, str) else int(cache_format)
    dm = DECAY_MODES[decay] if isinstance(decay, str) else int(decay)
    return HlaConfig(B, H, T, C, d, d, dt, gm, cf, tau, bias, skip_threshold, pool_window, dm)


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if not t.is_cuda:
        raise ValueError("libhla takes CUDA device tensors only (no CPU path)")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def cache_bytes(cfg: HlaConfig, max_chunks: int) -> int:
    return int(lib().hla_cache_bytes(ctypes.byref(cfg), max_chunks))


def prefill_workspace_bytes(cfg: HlaConfig) -> int:
    return int(lib().hla_prefill_workspace_bytes(ctypes.byref(cfg)))


def decode_workspace_bytes(cfg: HlaConfig, max_chunks: int) -> int:
    return int(lib().hla_decode_workspace_bytes(ctypes.byref(cfg), max_chunks))


class CacheSlice:
    """Sequences [b0, b0 + nb) of a Cache (see Cache.slice)."""

    def __init__(self):
        self.struct = HlaCache()
        self.parent = None
        self.max_chunks = 0


class Cache:
    """A decode cache: one caller-owned device block plus the C struct of views."""

    def __init__(self, cfg: HlaConfig, max_chunks: int, device="cuda", stream=None):
        nbytes = cache_bytes(cfg, max_chunks)
        if nbytes == 0:
            raise HlaError(HLA_ERR_UNSUPPORTED, "unsupported cache config")
        self.mem = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.struct = HlaCache()
        _check(lib().hla_cache_init(ctypes.byref(cfg), max_chunks, _ptr(self.mem), nbytes,
                                    ctypes.byref(self.struct), _stream(stream)))
        self.cfg = cfg
        self.max_chunks = max_chunks

    def slice(self, b0: int, nb: int):
        """The cache of sequences [b0, b0 + nb) (shares this cache's memory)."""
        sub = CacheSlice()
        sub.parent = self
        sub.max_chunks = self.max_chunks
        _check(lib().hla_cache_slice(ctypes.byref(self.struct), b0, nb, ctypes.byref(sub.struct)))
        return sub

    def view(self, field: str, shape, dtype):
        """Torch view of one cache buffer (for tests and inspection)."""
        off = getattr(self.struct, field) - self.mem.data_ptr()
        n = 1
        for s in shape:
            n *= s
        es = torch.empty((), dtype=dtype).element_size()
        return self.mem[off:off + n * es].view(dtype).view(*shape)


def gdn_chunk_transitions(cfg, k, v, alpha, beta, A_out, B_out, stream=None):
    _check(lib().gdn_chunk_transitions(ctypes.byref(cfg), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta),
                                       _ptr(A_out), _ptr(B_out), _stream(stream)))


def hla_routing(cfg, q_route, k_route, rq_out, rk_out, gates_out=None, active_idx_out=None,
                active_cnt_out=None, stream=None):
    _check(lib().hla_routing(ctypes.byref(cfg), _ptr(q_route), _ptr(k_route), _ptr(rq_out), _ptr(rk_out),
                             _ptr(gates_out), _ptr(active_idx_out), _ptr(active_cnt_out), _stream(stream)))


def hla_gate_support(cfg, gates, mass_out=None, support_out=None, stream=None):
    """Routing mass and effective support per query chunk from a gate matrix."""
    _check(lib().hla_gate_support(ctypes.byref(cfg), _ptr(gates), _ptr(mass_out), _ptr(support_out),
                                  _stream(stream)))


def hla_prefill(cfg, q, k, v, alpha, beta, o, q_route=None, k_route=None, user_gates=None, gates_out=None,
                active_idx_out=None, active_cnt_out=None, cache: Cache | None = None, workspace=None,
                stream=None):
    if workspace is None:
        workspace = torch.empty(max(prefill_workspace_bytes(cfg), 256), dtype=torch.uint8, device=q.device)
    _check(lib().hla_prefill(ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta),
                             _ptr(q_route), _ptr(k_route), _ptr(user_gates), _ptr(o), _ptr(gates_out),
                             _ptr(active_idx_out), _ptr(active_cnt_out),
                             ctypes.byref(cache.struct) if cache is not None else None,
                             _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))
    return o


def hla_decode_step(cfg, cache: Cache, q, k, v, alpha, beta, o, q_route=None, k_route=None, workspace=None,
                    stream=None):
    if workspace is None:
        workspace = torch.empty(max(decode_workspace_bytes(cfg, cache.max_chunks), 256), dtype=torch.uint8,
                                device=q.device)
    _check(lib().hla_decode_step(ctypes.byref(cfg), ctypes.byref(cache.struct), _ptr(q), _ptr(k), _ptr(v),
                                 _ptr(alpha), _ptr(beta), _ptr(q_route), _ptr(k_route), _ptr(o),
                                 _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))
    return o


def hla_decode_step_static(cfg, cache: Cache, q, k, v, alpha, beta, o, q_route=None, k_route=None, stream=None):
    """hla_decode_step with the library's fixed device scratch array: allocates nothing."""
    _check(lib().hla_decode_step_static(ctypes.byref(cfg), ctypes.byref(cache.struct), _ptr(q), _ptr(k), _ptr(v),
                                        _ptr(alpha), _ptr(beta), _ptr(q_route), _ptr(k_route), _ptr(o),
                                        _stream(stream)))
    return o


def hla_device_status(clear: bool = True):
    code = ctypes.c_uint32(0)
    st = lib().hla_device_status(1 if clear else 0, ctypes.byref(code))
    return st, int(code.value)


def hla_check_bounded_wait(limit_us: int, complete: bool, stream=None):
    """Enqueue the library's bounded-wait check (see include/hla.h)."""
    _check(lib().hla_check_bounded_wait(int(limit_us), 1 if complete else 0, _stream(stream)))


def hla_profile_enable(on: bool = True):
    _check(lib().hla_profile_enable(1 if on else 0))


def hla_profile_read(reset: bool = True):
    """Accumulated per-stage device milliseconds and kernel launches since the last reset."""
    n = len(STAGES)
    ms = (ctypes.c_float * n)()
    la = (ctypes.c_int32 * n)()
    _check(lib().hla_profile_read(ctypes.cast(ms, ctypes.c_void_p), ctypes.cast(la, ctypes.c_void_p),
                                  1 if reset else 0))
    return {STAGES[i]: (float(ms[i]), int(la[i])) for i in range(n)}
