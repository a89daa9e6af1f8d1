"""Pins for the CPU oracle: each check compares the oracle with something other
than itself (a printed value, a textbook table, a library routine, a closed
form, brute force), chosen so that a dropped term, a wrong sign or index, or a
transposed operand in the oracle fails at least one of them."""
import math

import numpy as np
import pytest
import scipy.integrate
import scipy.linalg
import scipy.special
import scipy.stats
import torch

import oracle as O
from kv_cache_vector_14_b200 import synthetic


def _levels_from_golden(golden):
    rows = golden("max1960_gaussian_8level.txt")
    lv = np.array([float(v) for k, v in rows if k == "level"])
    th = np.array([float(v) for k, v in rows if k == "threshold"])
    mse = [float(v) for k, v in rows if k == "mse"][0]
    return lv, th, mse


# ---------------------------------------------------------------- RNG

def test_splitmix64_published_vector(golden):
    for i, hx in golden("splitmix64_seed0.txt"):
        assert O.rng(0, int(i)) == int(hx, 16)


def test_params_distribution():
    """D is a fair +-1 diagonal; S entries are N(0,1) (KS test, moments)."""
    p = O.params(256, seed=7)
    D, S = p["D"].astype(np.float64), p["S"].ravel()
    assert set(np.unique(D)) <= {-1.0, 1.0}
    assert abs(D.mean()) < 5 / math.sqrt(256)
    assert abs(S.mean()) < 5 / math.sqrt(S.size)
    assert abs(S.var() - 1.0) < 5 * math.sqrt(2.0 / S.size)
    assert scipy.stats.kstest(S, "norm").pvalue > 1e-4
    # fp32-rounded values
    assert np.array_equal(S, S.astype(np.float32).astype(np.float64))
    # different seeds give different matrices; same seed reproduces
    assert not np.array_equal(O.params(128, 1)["S"], O.params(128, 2)["S"])
    assert np.array_equal(O.params(128, 3)["S"], O.params(128, 3)["S"])


# ---------------------------------------------------------------- codebook

def test_lloyd_max_textbook(golden):
    lv, th, mse = _levels_from_golden(golden)
    c, it = O.lloyd_max_std(8)
    assert it < 100000
    assert np.allclose(np.abs(c[4:]), lv, atol=5e-4)
    assert np.allclose(-c[:4][::-1], lv, atol=5e-4)
    mids = 0.5 * (c[:-1] + c[1:])
    assert np.allclose(mids[4:], th, atol=5e-4)
    # MSE by numerical integration (scipy quad), compared with the table
    edges = np.concatenate([[-np.inf], mids, [np.inf]])
    tot = 0.0
    for k in range(8):
        tot += scipy.integrate.quad(lambda x: (x - c[k]) ** 2 * scipy.stats.norm.pdf(x),
                                    edges[k], edges[k + 1], epsabs=1e-13)[0]
    assert abs(tot - mse) < 5e-5


def test_lloyd_max_optimality_conditions():
    """Each level is the conditional mean of its cell (quad), edges are midpoints."""
    c, _ = O.lloyd_max_std(8)
    edges = np.concatenate([[-np.inf], 0.5 * (c[:-1] + c[1:]), [np.inf]])
    for k in range(8):
        num = scipy.integrate.quad(lambda x: x * scipy.stats.norm.pdf(x), edges[k], edges[k + 1],
                                   epsabs=1e-14)[0]
        den = scipy.stats.norm.cdf(edges[k + 1]) - scipy.stats.norm.cdf(edges[k])
        assert abs(num / den - c[k]) < 1e-9


@pytest.mark.parametrize("d", [64, 128, 256])
def test_codebook_scaled_fp16(golden, d):
    lv, th, _ = _levels_from_golden(golden)
    p = O.params(d, 0)
    c8, b7 = p["c8"], p["b7"]
    std, _ = O.lloyd_max_std(8)
    sym = 0.5 * (std[::-1] * -1 + std)   # exact antisymmetric version
    # centroids are the fp16 rounding of level / sqrt(d) (numpy's binary16 as reference)
    ref = (sym / math.sqrt(d)).astype(np.float16).astype(np.float64)
    assert np.array_equal(c8, ref)
    assert np.array_equal(c8, -c8[::-1])
    assert np.all(np.diff(c8) > 0)
    assert np.allclose(np.abs(c8[4:]) * math.sqrt(d), lv, atol=5e-4)
    assert np.array_equal(b7, 0.5 * (c8[:-1] + c8[1:]))
    assert b7[3] == 0.0
    assert np.allclose(b7[4:] * math.sqrt(d), th, atol=1e-3)
    # boundaries are exact in fp32 (so GPU and oracle compare against the same numbers)
    assert np.array_equal(b7, b7.astype(np.float32).astype(np.float64))


def test_fp16_rounding_matches_numpy():
    g = np.random.default_rng(5)
    x = np.concatenate([g.standard_normal(20000) * 10.0 ** g.integers(-9, 5, 20000),
                        [0.0, -0.0, 65504.0, 65519.99, 6.1e-5, 5.96e-8, 2.98e-8, 1.0 + 2 ** -11,
                         1.0 + 3 * 2 ** -11, 2049.0, 2051.0]])
    x = x[np.abs(x) < 65520]
    ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(O.to_fp16_bits(x), ref)
    assert np.array_equal(O.from_fp16_bits(ref), ref.view(np.float16).astype(np.float64))


# ---------------------------------------------------------------- transform

@pytest.mark.parametrize("d", [2, 4, 8, 16, 32, 64, 128, 256])
def test_fwht_equals_sylvester(d):
    H = scipy.linalg.hadamard(d).astype(np.float64) / math.sqrt(d)
    v = np.random.default_rng(d).standard_normal((5, d))
    assert np.allclose(O.fwht(v), v @ H.T, atol=1e-12)
    I = np.eye(d)
    Hm = O.fwht(I)                       # rows: H e_i = column i of H
    assert np.allclose(Hm @ Hm.T, I, atol=1e-12)       # orthonormal
    assert np.allclose(O.fwht(O.fwht(v)), v, atol=1e-12)  # involutive
    assert np.allclose(np.linalg.norm(O.fwht(v), axis=1), np.linalg.norm(v, axis=1), atol=1e-12)


# ---------------------------------------------------------------- encode

def _dense_HD(p):
    d = p["d"]
    return (scipy.linalg.hadamard(d).astype(np.float64) / math.sqrt(d)) * p["D"].astype(np.float64)[None, :]


@pytest.mark.parametrize("d", [64, 128, 256])
def test_encode_steps_against_library_routines(d):
    p = O.params(d, 11)
    x = synthetic.gaussian((300, d), seed=d).astype(np.float64)
    x[:, :4] *= 20.0
    e = O.encode(x, p, with_qjl=True)
    n = np.linalg.norm(x, axis=1)
    assert np.allclose(e["n"], n, rtol=1e-14)
    y = (x / n[:, None]) @ _dense_HD(p).T                      # y = H D x/||x||
    assert np.allclose(e["y"], y, atol=1e-13)
    idx = np.searchsorted(p["b7"], e["y"], side="right")       # #{b_i <= y}, ties up
    assert np.array_equal(e["idx"], idx)
    r = e["y"] - p["c8"][e["idx"]]
    assert np.allclose(e["gamma"], np.linalg.norm(r, axis=1), rtol=1e-13)
    z = r @ p["S"].T                                           # z = S r (rows of S)
    assert np.allclose(e["z"], z, atol=1e-12)
    assert np.array_equal(e["sig"], (e["z"] >= 0).astype(np.uint8))
    # stored norms: fp16 of the float64 values
    assert np.array_equal(e["nh"], e["n"].astype(np.float16).view(np.uint16))
    assert np.array_equal(e["gh"], e["gamma"].astype(np.float16).view(np.uint16))
    # V path: same codes and norm, no sketch
    v = O.encode(x, p, with_qjl=False)
    assert np.array_equal(v["idx"], e["idx"]) and np.array_equal(v["n"], e["n"])
    assert "sig" not in v


def test_encode_zero_vector():
    p = O.params(128, 0)
    x = np.zeros((2, 128))
    x[1, 5] = 3.0
    e = O.encode(x, p, with_qjl=True)
    assert np.all(e["idx"][0] == 4) and np.all(e["sig"][0] == 1)
    assert e["n"][0] == 0.0 and e["gamma"][0] == 0.0
    assert e["n"][1] == 3.0


def test_encode_roundtrip_mse():
    """Relative MSE of x ~ n D H c[idx] is the Gaussian 8-level MSE (~0.0345)."""
    d = 128
    p = O.params(d, 0)
    x = synthetic.gaussian((10000, d), seed=1).astype(np.float64)
    e = O.encode(x, p, with_qjl=False)
    xt = e["n"][:, None] * (p["c8"][e["idx"]] @ _dense_HD(p))   # (H D)^T = D H
    rel = np.sum((x - xt) ** 2, axis=1) / np.sum(x ** 2, axis=1)
    assert abs(rel.mean() - 0.03454) < 0.05 * 0.03454


@pytest.mark.parametrize("d", [64, 128, 256])
def test_encode_mse_equals_sphere_marginal_integral(d):
    """A unit vector's coordinates after the rotation are those of a uniform
    point on the sphere S^(d-1): density proportional to (1 - y^2)^((d-3)/2)
    on [-1, 1].  The expected relative error ||x - n D H c[idx]||^2 / ||x||^2
    is therefore d times the integral of (y - c_k)^2 over each cell k of the
    codebook; the oracle's mean over 10^4 Gaussian vectors (reconstructed
    through the dense transform) must match it within five standard errors.
    This holds at each head dim (0.03344, 0.03398, 0.03426 at d = 64, 128,
    256, approaching the Gaussian 0.03454)."""
    p = O.params(d, 0)
    logc = scipy.special.gammaln(d / 2) - 0.5 * math.log(math.pi) - scipy.special.gammaln((d - 1) / 2)
    dens = lambda y: math.exp(logc + (d - 3) / 2 * math.log1p(-y * y))
    edges = [-1.0] + [float(b) for b in p["b7"]] + [1.0]
    expect = d * sum(scipy.integrate.quad(lambda y, k=k: (y - p["c8"][k]) ** 2 * dens(y), edges[k], edges[k + 1],
                                          epsabs=1e-15, limit=200)[0] for k in range(8))
    x = synthetic.gaussian((10000, d), seed=1).astype(np.float64)
    e = O.encode(x, p, with_qjl=False)
    xt = e["n"][:, None] * (p["c8"][e["idx"]] @ _dense_HD(p))   # (H D)^T = D H
    rel = np.sum((x - xt) ** 2, axis=1) / np.sum(x ** 2, axis=1)
    se = rel.std() / math.sqrt(rel.size)
    assert abs(rel.mean() - expect) < 5 * se, (rel.mean(), expect, se)
    assert 5 * se < 0.02 * expect                  # the check can tell a wrong cell or centroid


@pytest.mark.parametrize("d", [64, 128])
def test_qjl_estimator_unbiased(d):
    """E_S[ gamma sqrt(pi/2)/m <S q', 2 sigma - 1> ] = <q', r>, with the oracle's
    own sign bits and score routine; bound 5 sqrt(pi/(2 m N)) ||q'|| ||r||."""
    N = 1500
    x = synthetic.gaussian((1, d), seed=3).astype(np.float64)
    w = synthetic.gaussian((N, d), seed=4).astype(np.float64)
    errs, bounds, trues = [], [], []
    for s in range(N):
        p = O.params(d, 1000 + s)
        e = O.encode(x, p, with_qjl=True)
        r = e["y"][0] - p["c8"][e["idx"][0]]
        qp = r / np.linalg.norm(r) + 0.5 * w[s] / np.linalg.norm(w[s])   # q' correlated with r
        q = p["D"] * O.fwht(qp)                                           # q = D H q'
        kc = {"idx": e["idx"], "sig": e["sig"],
              "nh": np.array([0x3C00], dtype=np.uint16),                  # n = 1
              "gh": O.to_fp16_bits(np.array([np.linalg.norm(r)]))}
        g_hat = O.half_bits_to_float(kc["gh"])[0]
        s_t = O.scores(p, q, kc, scale=1.0)[0]
        est = s_t - qp @ p["c8"][e["idx"][0]]            # QJL part of the score
        true = qp @ r * g_hat / np.linalg.norm(r)
        errs.append(est - true)
        trues.append(true)
        bounds.append(np.linalg.norm(qp) * g_hat)
    errs = np.array(errs)
    tol = 5 * math.sqrt(math.pi / (2 * d * N)) * max(bounds)
    assert abs(errs.mean()) < tol
    assert np.mean(trues) > 20 * tol      # the test has power against a wrong constant or sign


def test_polar_only_scores_shrink_qjl_scores_unbiased():
    """PolarQuant-only versus QJL-corrected K scores (the page's two K flows).
    Over random sign diagonals and JL matrices (parameter seeds), the score
    without the QJL term, n <q', c[idx]>, regresses on the exact <q, x> with
    slope E<y_hat, y> = 1 - D_mse: the centroid condition makes the residual
    r = y - y_hat average to zero in each cell, so E<y_hat, r> = 0 and
    E<y_hat, y> = E||y_hat||^2 = 1 - E||r||^2.  Adding the QJL term (an
    unbiased estimate of <q', r>) restores slope 1.  D_mse = 0.03454 is the
    8-level Gaussian quantiser's MSE (pinned above); the tolerance 0.01 is
    about five standard errors for 12800 samples."""
    d, nseeds, T = 128, 200, 64
    x = synthetic.gaussian((T, d), seed=21).astype(np.float64)
    q = synthetic.gaussian((d,), seed=22).astype(np.float64)
    exact = x @ q
    sp, sq = [], []
    for s in range(nseeds):
        p = O.params(d, 5000 + s)
        e = O.encode(x, p, with_qjl=True)
        kc = {"idx": e["idx"], "sig": e["sig"], "nh": e["nh"], "gh": e["gh"]}
        sq.append(O.scores(p, q, kc, 1.0))
        sp.append(O.scores(p, q, dict(kc, gh=np.zeros_like(e["gh"])), 1.0))
    sp, sq = np.concatenate(sp), np.concatenate(sq)
    ex = np.tile(exact, nseeds)
    slope_polar = (sp @ ex) / (ex @ ex)
    slope_qjl = (sq @ ex) / (ex @ ex)
    assert abs(slope_qjl - 1.0) < 0.01
    assert abs(slope_polar - (1.0 - 0.03454)) < 0.01
    assert slope_qjl - slope_polar > 0.02          # the two estimators are told apart


# ---------------------------------------------------------------- layout

@pytest.mark.parametrize("d", [64, 128, 256])
def test_bits_per_dim_and_pack_roundtrip(golden, d):
    for cache, hd, bpd in golden("bits_per_dim.txt"):
        if int(hd) == d:
            bb = O.block_bytes(d, cache == "K")
            assert 8 * bb / (64 * d) == float(bpd)
    assert 8 * O.block_bytes(d, True) / (64 * d) == (3 * d + d + 32) / d
    assert 8 * O.block_bytes(d, False) / (64 * d) == (3 * d + 16) / d
    g = np.random.default_rng(d)
    T, t0, Tcap = 150, 37, 192
    idx = g.integers(0, 8, (T, d), dtype=np.uint8)
    sig = g.integers(0, 2, (T, d), dtype=np.uint8)
    nh = g.integers(0, 2 ** 16, T, dtype=np.uint16)
    gh = g.integers(0, 2 ** 16, T, dtype=np.uint16)
    for is_k in (True, False):
        blocks = np.zeros(Tcap // 64 * O.block_bytes(d, is_k), dtype=np.uint8)
        O.pack(d, is_k, t0, idx, sig if is_k else None, nh, gh if is_k else None, blocks)
        u = O.unpack(d, is_k, t0, T, blocks)
        assert np.array_equal(u["idx"], idx) and np.array_equal(u["nh"], nh)
        if is_k:
            assert np.array_equal(u["sig"], sig) and np.array_equal(u["gh"], gh)
        # tokens outside [t0, t0 + T) stay zero
        full = O.unpack(d, is_k, 0, Tcap, blocks)
        assert not full["idx"][:t0].any() and not full["idx"][t0 + T:].any()
        assert not full["nh"][:t0].any() and not full["nh"][t0 + T:].any()
        # packing in pieces (appends) gives the same blocks as one bulk pack
        part = np.zeros_like(blocks)
        for a, b in ((0, 1), (1, 30), (30, 31), (31, T)):
            O.pack(d, is_k, t0 + a, idx[a:b], sig[a:b] if is_k else None, nh[a:b], gh[a:b] if is_k else None, part)
        assert np.array_equal(part, blocks)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_layout_is_a_bijection(d):
    """Every (coordinate, code bit) and every sign lands on its own bit of the record."""
    seen = set()
    for j in range(d):
        for b in range(3):
            idx = np.zeros((1, d), dtype=np.uint8)
            idx[0, j] = 1 << b
            blocks = np.zeros(O.block_bytes(d, False), dtype=np.uint8)
            O.pack(d, False, 0, idx, None, np.zeros(1, np.uint16), None, blocks)
            bits = np.flatnonzero(np.unpackbits(blocks[: 3 * d // 8], bitorder="little"))
            assert len(bits) == 1
            seen.add(int(bits[0]))
    assert len(seen) == 3 * d
    seen = set()
    for j in range(d):
        sig = np.zeros((1, d), dtype=np.uint8)
        sig[0, j] = 1
        blocks = np.zeros(O.block_bytes(d, True), dtype=np.uint8)
        O.pack(d, True, 0, np.zeros((1, d), np.uint8), sig, np.zeros(1, np.uint16),
               np.zeros(1, np.uint16), blocks)
        off = 64 * 3 * d // 8
        bits = np.flatnonzero(np.unpackbits(blocks[off: off + d // 8], bitorder="little"))
        assert len(bits) == 1
        seen.add(int(bits[0]))
    assert len(seen) == d


# ---------------------------------------------------------------- attention

def _random_cache(d, T, seed, gamma_zero=False):
    g = np.random.default_rng(seed)
    kc = {"idx": g.integers(0, 8, (T, d), dtype=np.uint8),
          "sig": g.integers(0, 2, (T, d), dtype=np.uint8),
          "nh": O.to_fp16_bits(g.uniform(0.5, 3.0, T)),
          "gh": O.to_fp16_bits(np.zeros(T) if gamma_zero else g.uniform(0.05, 0.3, T))}
    vc = {"idx": g.integers(0, 8, (T, d), dtype=np.uint8),
          "nh": O.to_fp16_bits(g.uniform(0.5, 3.0, T))}
    return kc, vc


@pytest.mark.parametrize("d,T,G", [(64, 5, 2), (128, 1, 1), (128, 7, 2), (128, 16, 4), (256, 9, 3)])
def test_attend_bruteforce(d, T, G):
    """Per-token dequantisation in the original domain, explicit QJL term, library
    softmax, per-token inverse transforms -- against the oracle's rotated-domain
    accumulation with one inverse transform."""
    p = O.params(d, 21)
    kc, vc = _random_cache(d, T, seed=T)
    q = synthetic.gaussian((G, d), seed=G).astype(np.float64)
    scale = 1.0 / math.sqrt(d)
    HD = _dense_HD(p)
    nk, gk, nv = (O.half_bits_to_float(kc["nh"]), O.half_bits_to_float(kc["gh"]),
                  O.half_bits_to_float(vc["nh"]))
    ref = np.zeros((G, d))
    for g in range(G):
        s = np.zeros(T)
        u = p["S"] @ (HD @ q[g])
        for t in range(T):
            k_t = nk[t] * (HD.T @ p["c8"][kc["idx"][t]])          # n D H c[idx]
            corr = nk[t] * gk[t] * math.sqrt(math.pi / 2) / d * (u @ (2.0 * kc["sig"][t] - 1.0))
            s[t] = scale * (q[g] @ k_t + corr)
        pr = scipy.special.softmax(s)
        for t in range(T):
            ref[g] += pr[t] * nv[t] * (HD.T @ p["c8"][vc["idx"][t]])
    out = O.attend(p, q, kc, vc, scale)
    assert np.allclose(out, ref, atol=1e-12, rtol=1e-11)


def test_attend_gamma_zero_is_sdpa():
    """With gamma = 0 the score is the plain dot product with the dequantised key;
    the output must equal torch's scaled_dot_product_attention in float64."""
    d, T, G = 128, 64, 4
    p = O.params(d, 5)
    kc, vc = _random_cache(d, T, seed=9, gamma_zero=True)
    q = synthetic.gaussian((G, d), seed=2).astype(np.float64) * 3.0
    HD = _dense_HD(p)
    K = O.half_bits_to_float(kc["nh"])[:, None] * (p["c8"][kc["idx"]] @ HD)
    V = O.half_bits_to_float(vc["nh"])[:, None] * (p["c8"][vc["idx"]] @ HD)
    scale = 0.37
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(K)[None], torch.from_numpy(V)[None],
        scale=scale)[0].numpy()
    out = O.attend(p, q, kc, vc, scale)
    assert np.allclose(out, ref, atol=1e-12, rtol=1e-10)


def test_attend_empty_and_gqa_independence():
    d = 128
    p = O.params(d, 1)
    kc, vc = _random_cache(d, 0, seed=0)
    out = O.attend(p, np.ones((2, d)), kc, vc, 0.1)
    assert np.all(out == 0.0)
    kc, vc = _random_cache(d, 33, seed=1)
    q = synthetic.gaussian((4, d), seed=8).astype(np.float64)
    allh = O.attend(p, q, kc, vc, 0.2)
    for g in range(4):
        assert np.array_equal(allh[g], O.attend(p, q[g:g + 1], kc, vc, 0.2)[0])


def test_layout_hand_worked_entries(golden):
    """Single-entry records against words worked out by hand from the written layout."""
    rows = golden("layout_single_entries.txt")
    cases = {}
    for kind, hd, j, val, widx, whex in rows:
        cases.setdefault((kind, int(hd), int(j), int(val)), {})[int(widx)] = int(whex, 16)
    for (kind, d, j, val), words in cases.items():
        idx = np.zeros((1, d), np.uint8)
        sig = np.zeros((1, d), np.uint8)
        (idx if kind == "code" else sig)[0, j] = val
        blocks = np.zeros(O.block_bytes(d, True), dtype=np.uint8)
        O.pack(d, True, 0, idx, sig, np.zeros(1, np.uint16), np.zeros(1, np.uint16), blocks)
        if kind == "code":
            rec = blocks[: 3 * d // 8].view(np.uint32)
        else:
            off = 64 * 3 * d // 8
            rec = blocks[off: off + d // 8].view(np.uint32)
        expect = np.zeros_like(rec)
        for w, v in words.items():
            expect[w] = v
        assert np.array_equal(rec, expect), (kind, d, j, val, [hex(x) for x in rec])
