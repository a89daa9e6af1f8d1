"""CPU oracle for TurboQuant KV-cache compression and compressed-cache decode
attention (float64, plain loops in ``tq_oracle.c``).

TEST INFRASTRUCTURE ONLY.  The tests, the smoke check and the CPU-baseline leg
of the benchmark may import this package; the library path never does.  It
shares no code with the CUDA library (``kv_cache_vector_14_b200``) and neither
imports the other.

This module only marshals numpy arrays into the C functions; every step of the
method lives in ``tq_oracle.c``, which cites the page passage it follows.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tq_oracle.c")
_LIB = os.path.join(_HERE, "_liborc.so")
_lock = threading.Lock()
_lib = None

BLOCK_T = 64


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/_liborc.so`` (gcc, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-D_DEFAULT_SOURCE",
             "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _L():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = C.CDLL(_LIB)
            P = C.c_void_p
            i64 = C.c_int64
            lib.orc_rng.restype = C.c_uint64
            lib.orc_rng.argtypes = [C.c_uint64, C.c_uint64]
            lib.orc_to_fp16.restype = C.c_uint16
            lib.orc_to_fp16.argtypes = [C.c_double]
            lib.orc_from_fp16.restype = C.c_double
            lib.orc_from_fp16.argtypes = [C.c_uint16]
            lib.orc_lloyd_max_std.restype = C.c_int
            lib.orc_lloyd_max_std.argtypes = [C.c_int, P]
            lib.orc_params.restype = None
            lib.orc_params.argtypes = [C.c_int, C.c_uint64, P, P, P, P]
            lib.orc_fwht.restype = None
            lib.orc_fwht.argtypes = [P, C.c_int]
            lib.orc_encode.restype = None
            lib.orc_encode.argtypes = [C.c_int, P, P, P, P, P, i64, C.c_int, P, P, P, P, P, P]
            lib.orc_sketch_given_codes.restype = None
            lib.orc_sketch_given_codes.argtypes = [C.c_int, P, P, P, P, P, i64, P, P, P]
            lib.orc_block_bytes.restype = i64
            lib.orc_block_bytes.argtypes = [C.c_int, C.c_int]
            lib.orc_pack.restype = None
            lib.orc_pack.argtypes = [C.c_int, C.c_int, i64, i64, P, P, P, P, P]
            lib.orc_unpack.restype = None
            lib.orc_unpack.argtypes = [C.c_int, C.c_int, i64, i64, P, P, P, P, P]
            lib.orc_attend.restype = None
            lib.orc_attend.argtypes = [C.c_int, C.c_int, P, P, P, P, i64, P, P, P, P, P, P,
                                       C.c_double, P]
            lib.orc_scores.restype = None
            lib.orc_scores.argtypes = [C.c_int, P, P, P, P, i64, P, P, P, P, C.c_double, P]
            lib.orc_to_fp16_array.restype = None
            lib.orc_to_fp16_array.argtypes = [P, i64, P]
            lib.orc_num_threads.restype = C.c_int
            lib.orc_num_threads.argtypes = []
            lib.orc_set_threads.restype = None
            lib.orc_set_threads.argtypes = [C.c_int]
            _lib = lib
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(C.c_void_p)


def rng(seed: int, i: int) -> int:
    """Draw number ``i`` of the counter-based SplitMix64 stream ``seed``."""
    return int(_L().orc_rng(seed & (2**64 - 1), i))


def to_fp16_bits(x) -> np.ndarray:
    """IEEE binary16 round-to-nearest-even of float64 values, as uint16 bits."""
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    h = np.zeros(a.shape, dtype=np.uint16)
    _L().orc_to_fp16_array(_p(a), a.size, _p(h))
    return h


def from_fp16_bits(h) -> np.ndarray:
    f = _L().orc_from_fp16
    a = np.asarray(h, dtype=np.uint16)
    return np.array([f(int(v)) for v in a.ravel()], dtype=np.float64).reshape(a.shape)


def round_fp16(x) -> np.ndarray:
    return from_fp16_bits(to_fp16_bits(x))


def lloyd_max_std(levels: int = 8):
    """Lloyd-Max levels for N(0,1) (unscaled, unrounded) and the iteration count."""
    c = np.zeros(levels, dtype=np.float64)
    it = _L().orc_lloyd_max_std(levels, _p(c))
    return c, it


def params(d: int, seed: int = 0) -> dict:
    """Sign diagonal D, JL matrix S (m x d, m = d), centroids c8, boundaries b7."""
    D = np.zeros(d, dtype=np.int8)
    S = np.zeros((d, d), dtype=np.float64)
    c8 = np.zeros(8, dtype=np.float64)
    b7 = np.zeros(7, dtype=np.float64)
    _L().orc_params(d, seed & (2**64 - 1), _p(D), _p(S), _p(c8), _p(b7))
    return {"d": d, "seed": seed, "D": D, "S": S, "c8": c8, "b7": b7}


def fwht(v) -> np.ndarray:
    """Orthonormal natural-order Walsh-Hadamard transform along the last axis."""
    a = np.array(v, dtype=np.float64, order="C")
    d = a.shape[-1]
    flat = a.reshape(-1, d)
    for row in flat:
        _L().orc_fwht(_p(row), d)
    return flat.reshape(a.shape)


def encode(x, prm: dict, with_qjl: bool) -> dict:
    """Encode rows of x ([N, d], any float dtype, converted exactly to float64).

    Returns idx [N,d] u8, sig [N,m] u8 (K only), n and gamma (float64, unrounded),
    nh and gh (their fp16 bits as stored), y [N,d] and z [N,m] (K only)."""
    d = prm["d"]
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float64).reshape(-1, d))
    N = x.shape[0]
    idx = np.zeros((N, d), dtype=np.uint8)
    sig = np.zeros((N, d), dtype=np.uint8)
    n = np.zeros(N, dtype=np.float64)
    g = np.zeros(N, dtype=np.float64)
    y = np.zeros((N, d), dtype=np.float64)
    z = np.zeros((N, d), dtype=np.float64)
    _L().orc_encode(d, _p(prm["D"]), _p(prm["S"]), _p(prm["c8"]), _p(prm["b7"]), _p(x), N,
                    1 if with_qjl else 0, _p(idx), _p(sig), _p(n), _p(g), _p(y), _p(z))
    out = {"idx": idx, "n": n, "nh": to_fp16_bits(n), "y": y}
    if with_qjl:
        out.update(sig=sig, gamma=g, gh=to_fp16_bits(g), z=z)
    return out


def sketch_given_codes(prm: dict, y, idx, nonzero) -> dict:
    """Residual norm and JL signs of rows y ([N, d]) quantised to the given codes."""
    d = prm["d"]
    y = np.ascontiguousarray(y, dtype=np.float64).reshape(-1, d)
    idx = np.ascontiguousarray(idx, dtype=np.uint8).reshape(-1, d)
    nz = np.ascontiguousarray(nonzero, dtype=np.uint8).reshape(-1)
    N = y.shape[0]
    sig = np.zeros((N, d), dtype=np.uint8)
    g = np.zeros(N, dtype=np.float64)
    z = np.zeros((N, d), dtype=np.float64)
    _L().orc_sketch_given_codes(d, _p(prm["S"]), _p(prm["c8"]), _p(y), _p(idx), _p(nz), N,
                                _p(sig), _p(g), _p(z))
    return {"sig": sig, "gamma": g, "gh": to_fp16_bits(g), "z": z}


def block_bytes(d: int, is_k: bool) -> int:
    return int(_L().orc_block_bytes(d, 1 if is_k else 0))


def pack(d: int, is_k: bool, t0: int, idx, sig, nh, gh, blocks: np.ndarray) -> None:
    """Write tokens [t0, t0+T) of one sequence into its block array (uint8, in place)."""
    idx = np.ascontiguousarray(idx, dtype=np.uint8)
    T = idx.shape[0]
    sig = np.ascontiguousarray(sig if sig is not None else np.zeros((T, d)), dtype=np.uint8)
    nh = np.ascontiguousarray(nh, dtype=np.uint16)
    gh = np.ascontiguousarray(gh if gh is not None else np.zeros(T), dtype=np.uint16)
    assert blocks.dtype == np.uint8 and blocks.flags["C_CONTIGUOUS"]
    _L().orc_pack(d, 1 if is_k else 0, t0, T, _p(idx), _p(sig), _p(nh), _p(gh), _p(blocks))


def unpack(d: int, is_k: bool, t0: int, T: int, blocks: np.ndarray) -> dict:
    """Read tokens [t0, t0+T) of one sequence from its block array."""
    blocks = np.ascontiguousarray(blocks, dtype=np.uint8)
    idx = np.zeros((T, d), dtype=np.uint8)
    sig = np.zeros((T, d), dtype=np.uint8)
    nh = np.zeros(T, dtype=np.uint16)
    gh = np.zeros(T, dtype=np.uint16)
    _L().orc_unpack(d, 1 if is_k else 0, t0, T, _p(blocks), _p(idx), _p(sig), _p(nh), _p(gh))
    out = {"idx": idx, "nh": nh}
    if is_k:
        out.update(sig=sig, gh=gh)
    return out


def half_bits_to_float(h) -> np.ndarray:
    """Decode stored fp16 bit patterns (vectorised through numpy's binary16 type)."""
    return np.asarray(h, dtype=np.uint16).view(np.float16).astype(np.float64)


def attend(prm: dict, q, kc: dict, vc: dict, scale: float) -> np.ndarray:
    """Decode attention of G query heads (q [G, d]) over one unpacked KV head.

    kc: dict(idx [T,d], sig [T,m], nh [T] fp16 bits, gh [T] fp16 bits)
    vc: dict(idx [T,d], nh [T] fp16 bits).  Returns out [G, d] float64."""
    d = prm["d"]
    q = np.ascontiguousarray(np.asarray(q, dtype=np.float64).reshape(-1, d))
    G = q.shape[0]
    T = kc["idx"].shape[0]
    nk = np.ascontiguousarray(half_bits_to_float(kc["nh"]))
    gk = np.ascontiguousarray(half_bits_to_float(kc["gh"]))
    nv = np.ascontiguousarray(half_bits_to_float(vc["nh"]))
    ik = np.ascontiguousarray(kc["idx"], dtype=np.uint8)
    sg = np.ascontiguousarray(kc["sig"], dtype=np.uint8)
    iv = np.ascontiguousarray(vc["idx"], dtype=np.uint8)
    out = np.zeros((G, d), dtype=np.float64)
    if T == 0:
        return out
    _L().orc_attend(d, G, _p(prm["D"]), _p(prm["S"]), _p(prm["c8"]), _p(q), T,
                    _p(ik), _p(sg), _p(nk), _p(gk), _p(iv), _p(nv), float(scale), _p(out))
    return out


def scores(prm: dict, q, kc: dict, scale: float) -> np.ndarray:
    """Pre-softmax scores s_t of one query head (q [d]) over an unpacked K head."""
    d = prm["d"]
    q = np.ascontiguousarray(np.asarray(q, dtype=np.float64).reshape(d))
    T = kc["idx"].shape[0]
    s = np.zeros(max(T, 1), dtype=np.float64)
    nk = np.ascontiguousarray(half_bits_to_float(kc["nh"]))
    gk = np.ascontiguousarray(half_bits_to_float(kc["gh"]))
    _L().orc_scores(d, _p(prm["D"]), _p(prm["S"]), _p(prm["c8"]), _p(q), T,
                    _p(np.ascontiguousarray(kc["idx"], dtype=np.uint8)),
                    _p(np.ascontiguousarray(kc["sig"], dtype=np.uint8)), _p(nk), _p(gk),
                    float(scale), _p(s))
    return s[:T]


def num_threads() -> int:
    return int(_L().orc_num_threads())


def set_threads(n: int) -> None:
    """Threads the oracle's parallel loops use from now on (n <= 0: all cores)."""
    _L().orc_set_threads(int(n))
