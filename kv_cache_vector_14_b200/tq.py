"""ctypes binding of libtq (include/tq.h), with the C ABI's names.

Argument marshalling only: every step of encode and attention runs in the CUDA
kernels of ``libtq.so``.  Tensors are PyTorch device tensors (PyTorch owns the
memory and the streams); there is no CPU fallback -- if ``libtq.so`` is missing
the first call raises.
"""
from __future__ import annotations

import ctypes as C
import os
import threading

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libtq.so")
BLOCK_T = 64

TQ_OK, TQ_ERR_INVALID_ARG, TQ_ERR_UNSUPPORTED, TQ_ERR_CUDA, TQ_ERR_WORKSPACE, TQ_ERR_DEVICE_CHECK = range(6)
TQ_F32, TQ_BF16, TQ_F16 = 0, 1, 2

EXPORTED = ("tq_params_host", "tq_init", "tq_destroy", "tq_get_params", "tq_head_dim", "tq_block_bytes",
            "tq_cache_bytes", "tq_encode_k", "tq_encode_v", "tq_attend_workspace_bytes", "tq_attend_decode",
            "tq_append_attend", "tq_prefill_workspace_bytes", "tq_attend_prefill", "tq_attend_decode_polar",
            "tq_attend_decode_static", "tq_device_status", "tq_set_decode_events", "tq_set_decode_path", "tq_set_wait_limit", "tq_attend_path",
            "tq_decode_plan", "tq_status_string")


class TQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {tq_status_string(status)} (status {status})")


class tq_cache(C.Structure):
    _fields_ = [("base", C.c_void_p), ("B", C.c_int64), ("Hkv", C.c_int64), ("Tcap", C.c_int64),
                ("block_table", C.c_void_p), ("pool_blocks", C.c_int64)]


_lock = threading.Lock()
_lib = None


def lib() -> C.CDLL:
    """Load the in-tree libtq.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(f"{LIB_PATH} is missing: build it with `python -m kv_cache_vector_14_b200.build`")
            L = C.CDLL(LIB_PATH)
            P, i64, i32, st = C.c_void_p, C.c_int64, C.c_int, C.c_int
            L.tq_params_host.argtypes = [i32, C.c_uint64, P, P, P, P]
            L.tq_params_host.restype = st
            L.tq_init.argtypes = [i32, C.c_uint64, C.POINTER(C.c_void_p)]
            L.tq_init.restype = st
            L.tq_destroy.argtypes = [P]
            L.tq_destroy.restype = st
            L.tq_get_params.argtypes = [P, P, P, P, P]
            L.tq_get_params.restype = st
            L.tq_head_dim.argtypes = [P]
            L.tq_head_dim.restype = i32
            L.tq_block_bytes.argtypes = [i32, i32]
            L.tq_block_bytes.restype = C.c_size_t
            L.tq_cache_bytes.argtypes = [i32, i32, i64, i64, i64]
            L.tq_cache_bytes.restype = C.c_size_t
            for name in ("tq_encode_k", "tq_encode_v"):
                f = getattr(L, name)
                f.argtypes = [P, P, i32, i64, i64, i64, i64, i64, i64, C.POINTER(tq_cache), i64, P]
                f.restype = st
            L.tq_attend_workspace_bytes.argtypes = [P, i64, i64, i64, i64]
            L.tq_attend_workspace_bytes.restype = C.c_size_t
            L.tq_attend_decode.argtypes = [P, P, i32, i64, i64, C.POINTER(tq_cache), C.POINTER(tq_cache), P, i64,
                                           C.c_float, P, P, C.c_size_t, P]
            L.tq_attend_decode.restype = st
            L.tq_attend_decode_static.argtypes = [P, P, i32, i64, i64, C.POINTER(tq_cache), C.POINTER(tq_cache), P,
                                                  i64, C.c_float, P, P]
            L.tq_attend_decode_static.restype = st
            L.tq_attend_decode_polar.argtypes = L.tq_attend_decode.argtypes
            L.tq_attend_decode_polar.restype = st
            L.tq_append_attend.argtypes = [P, P, P, i32, i64, i64, i64, i64, C.POINTER(tq_cache),
                                           C.POINTER(tq_cache), i64, P, i32, i64, C.c_float, P, P, C.c_size_t, P]
            L.tq_append_attend.restype = st
            L.tq_prefill_workspace_bytes.argtypes = [P, i64, i64, i64]
            L.tq_prefill_workspace_bytes.restype = C.c_size_t
            L.tq_attend_prefill.argtypes = [P, P, i32, i64, i64, i64, C.POINTER(tq_cache), C.POINTER(tq_cache), i64,
                                            C.c_float, P, P, C.c_size_t, P]
            L.tq_attend_prefill.restype = st
            L.tq_device_status.argtypes = [P, P]
            L.tq_device_status.restype = st
            L.tq_set_decode_events.argtypes = [P, P, P]
            L.tq_set_decode_events.restype = st
            L.tq_set_decode_path.argtypes = [P, i32]
            L.tq_set_decode_path.restype = st
            L.tq_set_wait_limit.argtypes = [P, i32]
            L.tq_set_wait_limit.restype = st
            L.tq_attend_path.argtypes = [P, i64, i64]
            L.tq_attend_path.restype = C.c_char_p
            L.tq_decode_plan.argtypes = [i32, i32, i64, i64, i64, i64, i32, C.POINTER(i32), C.POINTER(i64),
                                         C.POINTER(i64), C.POINTER(i64), C.POINTER(i32)]
            L.tq_decode_plan.restype = st
            L.tq_status_string.argtypes = [i32]
            L.tq_status_string.restype = C.c_char_p
            _lib = L
    return _lib


def _check(status: int, where: str) -> None:
    if status != TQ_OK:
        raise TQError(status, where)


def _np_ptr(a: np.ndarray):
    return a.ctypes.data_as(C.c_void_p)


def _stream(stream):
    if stream is None:
        import torch
        return C.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return C.c_void_p(stream)
    return C.c_void_p(stream.cuda_stream)


def _dtype_code(t) -> int:
    import torch
    m = {torch.float32: TQ_F32, torch.bfloat16: TQ_BF16, torch.float16: TQ_F16}
    if t.dtype not in m:
        raise TypeError(f"unsupported dtype {t.dtype}")
    return m[t.dtype]


# ------------------------------------------------------------------ constants

def tq_status_string(status: int) -> str:
    return lib().tq_status_string(status).decode()


def tq_params_host(head_dim: int, seed: int = 0) -> dict:
    D = np.zeros(head_dim, dtype=np.int8)
    S = np.zeros((head_dim, head_dim), dtype=np.float32)
    c8 = np.zeros(8, dtype=np.float32)
    b7 = np.zeros(7, dtype=np.float32)
    _check(lib().tq_params_host(head_dim, seed, _np_ptr(D), _np_ptr(S), _np_ptr(c8), _np_ptr(b7)), "tq_params_host")
    return {"D": D, "S": S, "c8": c8, "b7": b7}


def tq_init(head_dim: int, seed: int = 0) -> C.c_void_p:
    h = C.c_void_p()
    _check(lib().tq_init(head_dim, seed, C.byref(h)), "tq_init")
    return h


def tq_destroy(h) -> None:
    _check(lib().tq_destroy(h), "tq_destroy")


def tq_get_params(h) -> dict:
    d = lib().tq_head_dim(h)
    D = np.zeros(d, dtype=np.int8)
    S = np.zeros((d, d), dtype=np.float32)
    c8 = np.zeros(8, dtype=np.float32)
    b7 = np.zeros(7, dtype=np.float32)
    _check(lib().tq_get_params(h, _np_ptr(D), _np_ptr(S), _np_ptr(c8), _np_ptr(b7)), "tq_get_params")
    return {"D": D, "S": S, "c8": c8, "b7": b7}


def tq_head_dim(h) -> int:
    return int(lib().tq_head_dim(h))


def tq_block_bytes(head_dim: int, is_k: bool) -> int:
    return int(lib().tq_block_bytes(head_dim, 1 if is_k else 0))


def tq_cache_bytes(head_dim: int, is_k: bool, B: int, Hkv: int, Tcap: int) -> int:
    return int(lib().tq_cache_bytes(head_dim, 1 if is_k else 0, B, Hkv, Tcap))


# ------------------------------------------------------------------ caches

class Cache:
    """A compressed K or V cache in a PyTorch-owned uint8 device buffer."""

    def __init__(self, head_dim: int, is_k: bool, B: int, Hkv: int, Tcap: int, device="cuda", buf=None,
                 block_table=None, pool_blocks: int = 0):
        """Contiguous cache, or (block_table: device int32 [B*Hkv, Tcap/64]) a
        paged cache whose buffer is a pool of pool_blocks blocks."""
        import torch
        if block_table is not None:
            if block_table.dtype != torch.int32 or tuple(block_table.shape) != (B * Hkv, Tcap // 64) or \
                    not block_table.is_contiguous():
                raise ValueError("block_table must be contiguous int32 [B*Hkv, Tcap/64]")
            nbytes = pool_blocks * tq_block_bytes(head_dim, is_k)
        else:
            nbytes = tq_cache_bytes(head_dim, is_k, B, Hkv, Tcap)
        if nbytes == 0 and B * Hkv > 0:
            raise ValueError("Tcap must be a positive multiple of 64 and head_dim 64, 128 or 256")
        self.head_dim, self.is_k, self.B, self.Hkv, self.Tcap = head_dim, is_k, B, Hkv, Tcap
        self.block_table, self.pool_blocks = block_table, pool_blocks
        self.buf = buf if buf is not None else torch.zeros(max(nbytes, 16), dtype=torch.uint8, device=device)
        table = C.c_void_p(block_table.data_ptr()) if block_table is not None else None
        self.struct = tq_cache(C.c_void_p(self.buf.data_ptr()), B, Hkv, Tcap, table, pool_blocks)

    @property
    def nbytes(self) -> int:
        if self.block_table is not None:
            return self.pool_blocks * tq_block_bytes(self.head_dim, self.is_k)
        return tq_cache_bytes(self.head_dim, self.is_k, self.B, self.Hkv, self.Tcap)


# ------------------------------------------------------------------ hot calls

def _encode(fn, name, h, x, cache: Cache, t0: int, stream):
    if x.dim() != 4 or x.stride(-1) != 1:
        raise ValueError(f"{name}: x must be [B, Hkv, Tnew, d] with a contiguous last dim")
    B, Hkv, Tnew, _ = x.shape
    sb, sh, st, _ = x.stride()
    _check(fn(h, C.c_void_p(x.data_ptr()), _dtype_code(x), B, Hkv, Tnew, sb, sh, st, C.byref(cache.struct), t0,
              _stream(stream)), name)


def tq_encode_k(h, x, kc: Cache, t0: int = 0, stream=None) -> None:
    _encode(lib().tq_encode_k, "tq_encode_k", h, x, kc, t0, stream)


def tq_encode_v(h, x, vc: Cache, t0: int = 0, stream=None) -> None:
    _encode(lib().tq_encode_v, "tq_encode_v", h, x, vc, t0, stream)


def tq_attend_workspace_bytes(h, B: int, Hq: int, Hkv: int, Tmax: int) -> int:
    return int(lib().tq_attend_workspace_bytes(h, B, Hq, Hkv, Tmax))


def tq_attend_decode(h, q, kc: Cache, vc: Cache, out, ws, T: int = 0, seq_lens=None, scale: float = 1.0,
                     stream=None) -> None:
    if q.dim() != 3 or not q.is_contiguous():
        raise ValueError("tq_attend_decode: q must be contiguous [B, Hq, d]")
    B, Hq, _ = q.shape
    sl = C.c_void_p(seq_lens.data_ptr()) if seq_lens is not None else None
    _check(lib().tq_attend_decode(h, C.c_void_p(q.data_ptr()), _dtype_code(q), B, Hq, C.byref(kc.struct),
                                  C.byref(vc.struct), sl, T, float(scale), C.c_void_p(out.data_ptr()),
                                  C.c_void_p(ws.data_ptr()), ws.numel() * ws.element_size(), _stream(stream)),
           "tq_attend_decode")


def tq_attend_decode_polar(h, q, kc: Cache, vc: Cache, out, ws, T: int = 0, seq_lens=None, scale: float = 1.0,
                           stream=None) -> None:
    """Attention with a PolarQuant-only K cache (a V-layout cache written by
    tq_encode_v): scores without the QJL term."""
    if q.dim() != 3 or not q.is_contiguous():
        raise ValueError("tq_attend_decode_polar: q must be contiguous [B, Hq, d]")
    if kc.is_k:
        raise ValueError("tq_attend_decode_polar: kc must be a V-layout cache (encoded with tq_encode_v)")
    B, Hq, _ = q.shape
    sl = C.c_void_p(seq_lens.data_ptr()) if seq_lens is not None else None
    _check(lib().tq_attend_decode_polar(h, C.c_void_p(q.data_ptr()), _dtype_code(q), B, Hq, C.byref(kc.struct),
                                        C.byref(vc.struct), sl, T, float(scale), C.c_void_p(out.data_ptr()),
                                        C.c_void_p(ws.data_ptr()), ws.numel() * ws.element_size(),
                                        _stream(stream)), "tq_attend_decode_polar")


def tq_append_attend(h, k_new, v_new, kc: Cache, vc: Cache, t0: int, q, out, ws, scale: float = 1.0,
                     stream=None) -> None:
    """Fused decode step: append k_new/v_new ([B, Hkv, Tnew, d], same dtype and
    strides) at positions [t0, t0 + Tnew), then attend over t0 + Tnew tokens."""
    if k_new.dim() != 4 or k_new.stride(-1) != 1 or k_new.shape != v_new.shape or \
            k_new.stride() != v_new.stride() or k_new.dtype != v_new.dtype:
        raise ValueError("tq_append_attend: k_new, v_new must be [B, Hkv, Tnew, d] with equal dtype and strides")
    if q.dim() != 3 or not q.is_contiguous():
        raise ValueError("tq_append_attend: q must be contiguous [B, Hq, d]")
    Tnew = k_new.shape[2]
    sb, sh, st, _ = k_new.stride()
    _check(lib().tq_append_attend(h, C.c_void_p(k_new.data_ptr()), C.c_void_p(v_new.data_ptr()),
                                  _dtype_code(k_new), Tnew, sb, sh, st, C.byref(kc.struct), C.byref(vc.struct), t0,
                                  C.c_void_p(q.data_ptr()), _dtype_code(q), q.shape[1], float(scale),
                                  C.c_void_p(out.data_ptr()), C.c_void_p(ws.data_ptr()),
                                  ws.numel() * ws.element_size(), _stream(stream)), "tq_append_attend")


def tq_prefill_workspace_bytes(h, B: int, Lq: int, Hq: int) -> int:
    return int(lib().tq_prefill_workspace_bytes(h, B, Lq, Hq))


def tq_attend_prefill(h, q, kc: Cache, vc: Cache, T0: int, out, ws, scale: float = 1.0, stream=None) -> None:
    """Causal attention of a chunk of queries q [B, Lq, Hq, d] (query i over
    tokens [0, T0 + i]) over the compressed caches; out fp32 [B, Lq, Hq, d]."""
    if q.dim() != 4 or not q.is_contiguous():
        raise ValueError("tq_attend_prefill: q must be contiguous [B, Lq, Hq, d]")
    B, Lq, Hq, _ = q.shape
    _check(lib().tq_attend_prefill(h, C.c_void_p(q.data_ptr()), _dtype_code(q), B, Lq, Hq, C.byref(kc.struct),
                                   C.byref(vc.struct), T0, float(scale), C.c_void_p(out.data_ptr()),
                                   C.c_void_p(ws.data_ptr()), ws.numel() * ws.element_size(), _stream(stream)),
           "tq_attend_prefill")


def tq_device_status(h, stream=None) -> int:
    return int(lib().tq_device_status(h, _stream(stream)))


def tq_set_decode_events(h, ev_start=None, ev_stop=None) -> None:
    """Time the split-K kernel of later tq_attend_decode calls with torch.cuda.Event pairs."""
    a = C.c_void_p(ev_start.cuda_event) if ev_start is not None else None
    b = C.c_void_p(ev_stop.cuda_event) if ev_stop is not None else None
    _check(lib().tq_set_decode_events(h, a, b), "tq_set_decode_events")


def tq_set_wait_limit(h, first_wait: int) -> None:
    """Diagnostics: polls of each decode warp's first mbarrier wait (< 0: full bound)."""
    _check(lib().tq_set_wait_limit(h, int(first_wait)), "tq_set_wait_limit")


def tq_set_decode_path(h, path: str) -> None:
    """"auto" (tensor-core kernel where supported, cost-model partition), "simt",
    "split" (tensor-core kernel, uniform split grid) or "streamk" (tensor-core
    kernel, stream-K grid wherever it fits)."""
    _check(lib().tq_set_decode_path(h, {"auto": 0, "simt": 1, "split": 2, "streamk": 3}[path]),
           "tq_set_decode_path")


def tq_attend_path(h, Hq: int, Hkv: int) -> str:
    return lib().tq_attend_path(h, Hq, Hkv).decode()


def tq_decode_plan(num_sms: int, d: int, B: int, Hq: int, Hkv: int, T: int, equal_len: bool = True) -> dict:
    """The decode work partition for these sizes on a GPU of num_sms SMs (host only):
    partial slots per query head, tokens per uniform split, stream-K CTAs (0: the
    uniform grid) and chunks per unit, tokens per chunk."""
    ns, ct = C.c_int32(), C.c_int32()
    stt, skc, skn = C.c_int64(), C.c_int64(), C.c_int64()
    _check(lib().tq_decode_plan(num_sms, d, B, Hq, Hkv, T, int(equal_len), C.byref(ns), C.byref(stt), C.byref(skc),
                                C.byref(skn), C.byref(ct)), "tq_decode_plan")
    return {"nsplit": ns.value, "split_tokens": stt.value, "streamk_ctas": skc.value, "streamk_chunks": skn.value,
            "chunk_tokens": ct.value}
