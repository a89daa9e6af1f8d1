"""Seeded synthetic inputs for the five workloads (K/V vectors and queries).

This module draws random numbers with the workloads' shapes and value
distributions and nothing else: it holds none of the compression or attention
arithmetic, so both the CUDA library's tests/benchmark and the CPU oracle's
tests may use it.

Recipe (one ``numpy.random.SeedSequence(seed)`` per workload, spawned into
independent streams for K, V, queries, outlier channels and per-token norms):
  * K and V entries are iid N(0, 1) in fp32;
  * 4 outlier channels per KV head are drawn without replacement from the
    outlier stream and multiplied by 20;
  * where a workload has log-normal per-token norms, each (token, head) vector
    of K (and, independently, of V) is multiplied by exp(N(0, 0.5^2));
  * bf16 workloads round the fp32 values to bf16 (round to nearest even);
  * queries are iid N(0, 1), rounded to bf16 where the workload says so.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np


@dataclass(frozen=True)
class Workload:
    key: str
    title: str
    B: int
    Hq: int
    Hkv: int
    d: int
    T: int
    kv_dtype: str          # "f32" or "bf16"
    q_dtype: str           # "f32" or "bf16"
    lognormal_norms: bool
    seed: int
    scale: float
    steps: int = 0         # append-and-attend steps (0: none)
    extra: dict = field(default_factory=dict)


WORKLOADS = {
    "c1": Workload("c1", "single head: encode 1024 K/V (fp32, 4 outlier channels x20) + one decode",
                   B=1, Hq=1, Hkv=1, d=128, T=1024, kv_dtype="f32", q_dtype="f32",
                   lognormal_norms=False, seed=0, scale=1.0 / math.sqrt(128)),
    "c2": Workload("c2", "encode only: B=1, 8 KV heads, d=128, 32768 tokens, bf16, outliers, log-normal norms",
                   B=1, Hq=8, Hkv=8, d=128, T=32768, kv_dtype="bf16", q_dtype="bf16",
                   lognormal_norms=True, seed=1, scale=1.0 / math.sqrt(128)),
    "c3": Workload("c3", "decode GQA: B=1, Hq=32/Hkv=8, d=128, 40960-token compressed cache, bf16 query",
                   B=1, Hq=32, Hkv=8, d=128, T=40960, kv_dtype="bf16", q_dtype="bf16",
                   lognormal_norms=True, seed=2, scale=1.0 / math.sqrt(128)),
    "c4": Workload("c4", "long-context decode: B=4, Hq=16/Hkv=8, d=128, 102400 tokens per sequence",
                   B=4, Hq=16, Hkv=8, d=128, T=102400, kv_dtype="f32", q_dtype="bf16",
                   lognormal_norms=False, seed=3, scale=1.0 / math.sqrt(128)),
    "c5": Workload("c5", "append-and-attend: B=16, Hq=32/Hkv=8, d=256, cache from 8192 tokens, 256 steps",
                   B=16, Hq=32, Hkv=8, d=256, T=8192, kv_dtype="f32", q_dtype="f32",
                   lognormal_norms=False, seed=4, scale=1.0 / 16.0, steps=256),
}

_K, _V, _Q, _OUT, _NORM = range(5)


def _streams(seed: int):
    return [np.random.Generator(np.random.PCG64(s)) for s in np.random.SeedSequence(seed).spawn(5)]


def bf16_round(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 (ties to even); returns fp32 holding them."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16) << 16
    nan = np.isnan(a)
    out = r.astype(np.uint32).view(np.float32).copy()
    out[nan] = np.nan
    return out


def outlier_channels(w: Workload) -> np.ndarray:
    """[Hkv, 4] channel indices scaled x20 (same for K and V, and for all batches)."""
    g = _streams(w.seed)[_OUT]
    return np.stack([g.choice(w.d, size=4, replace=False) for _ in range(w.Hkv)])


def kv(w: Workload, which: str, t0: int = 0, t1: int | None = None, batches=None) -> np.ndarray:
    """K or V vectors of tokens [t0, t1) as fp32 array [B, Hkv, t1 - t0, d].

    The full sequence is Tfull = T + steps tokens; each (b, h) row draws its
    Tfull vectors from the K (or V) stream in order, so slices are consistent."""
    assert which in ("k", "v")
    Tfull = w.T + w.steps
    t1 = Tfull if t1 is None else t1
    assert 0 <= t0 <= t1 <= Tfull
    bs = list(range(w.B)) if batches is None else list(batches)
    st = _streams(w.seed)
    g = st[_K if which == "k" else _V]
    gn = st[_NORM]
    oc = outlier_channels(w)
    out = np.empty((len(bs), w.Hkv, t1 - t0, w.d), dtype=np.float32)
    # draw the whole (B, Hkv, Tfull, d) tensor row by row in a fixed order
    for b in range(w.B):
        for h in range(w.Hkv):
            row = g.standard_normal((Tfull, w.d), dtype=np.float32)
            if w.lognormal_norms:
                lk = gn.standard_normal(2 * Tfull)  # K and V factors interleaved
                fac = np.exp(0.5 * lk[(0 if which == "k" else 1)::2]).astype(np.float32)
            if b in bs:
                r = row[t0:t1]
                r[:, oc[h]] *= 20.0
                if w.lognormal_norms:
                    r *= fac[t0:t1, None]
                out[bs.index(b), h] = r
    if w.kv_dtype == "bf16":
        out = bf16_round(out)
    return out


def queries(w: Workload, step: int | None = None) -> np.ndarray:
    """Queries [B, Hq, d] (fp32 values, bf16-rounded where the workload says so).

    For the append-and-attend workload, ``step`` selects the step's query."""
    g = _streams(w.seed)[_Q]
    nsteps = max(w.steps, 1)
    qa = g.standard_normal((nsteps, w.B, w.Hq, w.d), dtype=np.float32)
    q = qa[0 if step is None else step]
    if w.q_dtype == "bf16":
        q = bf16_round(q)
    return np.ascontiguousarray(q)


def queries_all(w: Workload) -> np.ndarray:
    """Every step's queries at once, [steps, B, Hq, d] (same values as queries(w, s))."""
    g = _streams(w.seed)[_Q]
    qa = g.standard_normal((max(w.steps, 1), w.B, w.Hq, w.d), dtype=np.float32)
    if w.q_dtype == "bf16":
        qa = bf16_round(qa)
    return np.ascontiguousarray(qa)


def gaussian(shape, seed: int) -> np.ndarray:
    """Plain iid N(0,1) fp32 array for small ad-hoc cases."""
    return np.random.Generator(np.random.PCG64(seed)).standard_normal(shape, dtype=np.float32)
