"""Helpers for the GPU parity tests: run the library through its C ABI, read the
packed caches back, and compare with the oracle under the stated criteria.

Criteria:
  * codes and sign bits bit-exact, except coordinates whose float64 rotated
    value lies within 1e-6 of a decision boundary, and JL projections with
    |S r| < 1e-6 (signs are compared against the sketch of the residual of
    the library's own codes, so a code decided differently inside its window
    does not count against the signs); the excluded mismatches must also be
    at most 1e-5 of the total;
  * stored fp16 norms within one fp16 unit in the last place;
  * attention outputs: per (batch, query head) row, ||o - r||_inf / ||r||_inf <= 1e-3
    (the largest per-element relative error over elements above 1e-3 of their
    row's largest magnitude is printed beside it).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
from kv_cache_vector_14_b200 import tq

EPS_WINDOW = 1e-6
BUDGET = 1e-5
ATT_TOL = 1e-3


def torch_input(x: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    if dtype == "bf16":
        t = t.to(torch.bfloat16)          # exact: values are already bf16-representable
    elif dtype == "f16":
        t = t.to(torch.float16)
    return t.to(device)


def encode_gpu(h, d: int, x: torch.Tensor, Tcap: int, t0: int = 0, kc=None, vc=None, which="kv"):
    B, Hkv, T, _ = x.shape
    if "k" in which:
        kc = kc or tq.Cache(d, True, B, Hkv, Tcap)
        tq.tq_encode_k(h, x, kc, t0)
    if "v" in which:
        vc = vc or tq.Cache(d, False, B, Hkv, Tcap)
        tq.tq_encode_v(h, x, vc, t0)
    return kc, vc


def unpack_cache(cache: tq.Cache, t0: int, T: int, seqs=None) -> dict:
    """Unpack tokens [t0, t0+T) of every (b, h) (or of the listed (b, h) pairs)."""
    d, is_k = cache.head_dim, cache.is_k
    raw = cache.buf.cpu().numpy()
    nb = cache.Tcap // 64
    bb = O.block_bytes(d, is_k)
    seqs = seqs if seqs is not None else [(b, h) for b in range(cache.B) for h in range(cache.Hkv)]
    out = {"idx": np.zeros((len(seqs), T, d), np.uint8), "nh": np.zeros((len(seqs), T), np.uint16)}
    if is_k:
        out["sig"] = np.zeros((len(seqs), T, d), np.uint8)
        out["gh"] = np.zeros((len(seqs), T), np.uint16)
    for n, (b, h) in enumerate(seqs):
        s = (b * cache.Hkv + h) * nb
        u = O.unpack(d, is_k, t0, T, raw[s * bb:(s + nb) * bb])
        for k in out:
            out[k][n] = u[k]
    return out


def half_ulps(a, b) -> np.ndarray:
    return np.abs(np.asarray(a, np.int64) - np.asarray(b, np.int64))


def check_encode(prm: dict, x: np.ndarray, gk: dict | None, gv: dict | None) -> dict:
    """x: [N, d] float64 inputs; gk/gv: unpacked library fields flattened to [N, ...]."""
    d = prm["d"]
    x = np.asarray(x, np.float64).reshape(-1, d)
    e = O.encode(x, prm, with_qjl=gk is not None)
    near = np.zeros(e["y"].shape, dtype=bool)
    for b in prm["b7"]:                       # one boundary at a time (bounded host memory)
        near |= np.abs(e["y"] - b) < EPS_WINDOW
    stats = {"vectors": x.shape[0], "near_boundary": int(near.sum())}
    for name, g in (("k", gk), ("v", gv)):
        if g is None:
            continue
        mism = g["idx"].reshape(e["idx"].shape) != e["idx"]
        bad = mism & ~near
        assert not bad.any(), f"{name}: {int(bad.sum())} code mismatches outside the 1e-6 window"
        assert mism.sum() <= BUDGET * mism.size, f"{name}: {int(mism.sum())} code mismatches"
        assert half_ulps(g["nh"].ravel(), e["nh"]).max() <= 1, f"{name}: norm off by > 1 fp16 ulp"
        stats[f"{name}_code_mismatch"] = int(mism.sum())
    if gk is not None:
        gidx = gk["idx"].reshape(e["idx"].shape)
        rows = np.flatnonzero(np.any(gidx != e["idx"], axis=1))
        sig, z, gh = e["sig"].copy(), e["z"].copy(), e["gh"].copy()
        if rows.size:
            s = O.sketch_given_codes(prm, e["y"][rows], gidx[rows], e["n"][rows] > 0)
            sig[rows], z[rows], gh[rows] = s["sig"], s["z"], s["gh"]
        smis = gk["sig"].reshape(sig.shape) != sig
        bad = smis & ~(np.abs(z) < EPS_WINDOW)
        assert not bad.any(), f"{int(bad.sum())} sign mismatches outside |S r| < 1e-6"
        assert smis.sum() <= BUDGET * smis.size, f"{int(smis.sum())} sign mismatches"
        assert half_ulps(gk["gh"].ravel(), gh).max() <= 1, "gamma off by > 1 fp16 ulp"
        stats["sign_mismatch"] = int(smis.sum())
        stats["near_zero_projection"] = int((np.abs(z) < EPS_WINDOW).sum())
    return stats


def oracle_attend(prm: dict, q: np.ndarray, ku: dict, vu: dict, Hkv: int, seq_lens, scale: float) -> np.ndarray:
    """q [B, Hq, d] float64; ku/vu unpacked [B*Hkv, T, ...]; returns [B, Hq, d]."""
    B, Hq, d = q.shape
    G = Hq // Hkv
    out = np.zeros((B, Hq, d))
    for b in range(B):
        T = int(seq_lens[b])
        for h in range(Hkv):
            n = b * Hkv + h
            kc = {k: v[n, :T] for k, v in ku.items()}
            vc = {k: v[n, :T] for k, v in vu.items()}
            out[b, h * G:(h + 1) * G] = O.attend(prm, q[b, h * G:(h + 1) * G], kc, vc, scale)
    return out


def rel_err_rows(out: np.ndarray, ref: np.ndarray) -> np.ndarray:
    o = out.reshape(-1, out.shape[-1])
    r = ref.reshape(-1, ref.shape[-1])
    den = np.abs(r).max(axis=1)
    num = np.abs(o - r).max(axis=1)
    return np.where(den > 0, num / np.where(den > 0, den, 1), num)


def rel_err_elements(out: np.ndarray, ref: np.ndarray, floor: float = 1e-3) -> float:
    """Largest per-element relative error |o - r| / |r| over the elements whose
    |r| is at least `floor` times their row's ||r||_inf (reported beside the
    per-row criterion; elements near zero are left out since their relative
    error is unbounded)."""
    o = out.reshape(-1, out.shape[-1])
    r = ref.reshape(-1, ref.shape[-1])
    big = np.abs(r) >= floor * np.abs(r).max(axis=1, keepdims=True)
    big &= np.abs(r) > 0
    if not big.any():
        return 0.0
    return float((np.abs(o - r)[big] / np.abs(r)[big]).max())


def attend_gpu(h, q: torch.Tensor, kc, vc, T: int = 0, seq_lens=None, scale=1.0):
    B, Hq, d = q.shape
    Tmax = kc.Tcap if seq_lens is not None else T
    nbytes = tq.tq_attend_workspace_bytes(h, B, Hq, kc.Hkv, Tmax)
    ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=q.device)
    out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    tq.tq_attend_decode(h, q, kc, vc, out, ws, T=T, seq_lens=seq_lens, scale=scale)
    return out
