"""GPU parity: the CUDA library (through its C ABI) against the float64 oracle on
the same seeded inputs, for the five workloads and their edge cases."""
import dataclasses
import math

import numpy as np
import pytest
import torch

import oracle as O
from kv_cache_vector_14_b200 import synthetic, tq
from gpu_util import (ATT_TOL, attend_gpu, check_encode, encode_gpu, oracle_attend, rel_err_elements, rel_err_rows,
                      torch_input, unpack_cache)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def handles(libtq):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    hs = {d: tq.tq_init(d, 0) for d in (64, 128, 256)}
    yield hs
    torch.cuda.synchronize()
    for h in hs.values():
        tq.tq_destroy(h)


@pytest.fixture(params=["auto", "simt"])
def decode_path(request, handles):
    """Run a test once with the default (tensor-core where supported) decode
    kernel and once with the SIMT kernel forced."""
    for h in handles.values():
        tq.tq_set_decode_path(h, request.param)
    yield request.param
    for h in handles.values():
        tq.tq_set_decode_path(h, "auto")


@pytest.fixture(scope="module")
def prms():
    return {d: O.params(d, 0) for d in (64, 128, 256)}


def _flat(u: dict) -> dict:
    return {k: v.reshape((-1,) + v.shape[2:]) for k, v in u.items()}


def _x64(x: np.ndarray) -> np.ndarray:
    return x.astype(np.float64).reshape(-1, x.shape[-1])


@pytest.mark.parametrize("d", [64, 128, 256])
def test_params_on_device(handles, d):
    p, hp = tq.tq_get_params(handles[d]), tq.tq_params_host(d, 0)
    for k in ("D", "S", "c8", "b7"):
        assert np.array_equal(p[k], hp[k])


# ------------------------------------------------------------------ encode

def test_encode_single_head_fp32(handles, prms):
    w = synthetic.WORKLOADS["c1"]
    for which in ("k", "v"):
        x = synthetic.kv(w, which)
        kc, vc = encode_gpu(handles[128], 128, torch_input(x, w.kv_dtype), Tcap=w.T, which=which)
        g = _flat(unpack_cache(kc if which == "k" else vc, 0, w.T))
        st = check_encode(prms[128], _x64(x), g if which == "k" else None, g if which == "v" else None)
        print(which, st)


def test_encode_bf16_8heads_32768_full(handles, prms):
    """The encode-only workload at full size: every vector is compared."""
    w = synthetic.WORKLOADS["c2"]
    xk, xv = synthetic.kv(w, "k"), synthetic.kv(w, "v")
    kc, _ = encode_gpu(handles[128], 128, torch_input(xk, "bf16"), Tcap=w.T, which="k")
    _, vc = encode_gpu(handles[128], 128, torch_input(xv, "bf16"), Tcap=w.T, which="v")
    print("K", check_encode(prms[128], _x64(xk), _flat(unpack_cache(kc, 0, w.T)), None))
    print("V", check_encode(prms[128], _x64(xv), None, _flat(unpack_cache(vc, 0, w.T))))


def test_encode_d256_sampled(handles, prms):
    """d = 256 (append-and-attend workload's initial cache), two heads compared in full."""
    w = synthetic.WORKLOADS["c5"]
    x = synthetic.kv(w, "k", 0, w.T, batches=[0, 5])
    kc, vc = encode_gpu(handles[256], 256, torch_input(x, "f32"), Tcap=w.T)
    seqs = [(0, 0), (1, 7)]
    gk, gv = unpack_cache(kc, 0, w.T, seqs), unpack_cache(vc, 0, w.T, seqs)
    xs = np.stack([x[0, 0], x[1, 7]])
    print(check_encode(prms[256], _x64(xs), _flat(gk), _flat(gv)))


def test_encode_gqa_40960_full(handles, prms):
    """The 40960-token GQA workload's cache (B=1, 8 kv heads, bf16 K and V with
    outliers and log-normal norms): every K and V vector of every head compared
    with the oracle's encode."""
    w = synthetic.WORKLOADS["c3"]
    xk, xv = synthetic.kv(w, "k"), synthetic.kv(w, "v")
    kc, _ = encode_gpu(handles[128], 128, torch_input(xk, w.kv_dtype), Tcap=w.T, which="k")
    _, vc = encode_gpu(handles[128], 128, torch_input(xv, w.kv_dtype), Tcap=w.T, which="v")
    print("K", check_encode(prms[128], _x64(xk), _flat(unpack_cache(kc, 0, w.T)), None))
    print("V", check_encode(prms[128], _x64(xv), None, _flat(unpack_cache(vc, 0, w.T))))


def test_encode_long_context_b4_102400_sampled(handles, prms):
    """The long-context workload's cache (B=4, 8 kv heads, 102400 fp32 tokens with
    outliers: the benchmark's own cache, encoded in the benchmark's launch
    configuration): four whole sequences, the first and the last among them,
    compared with the oracle's encode over all 102400 tokens."""
    w = synthetic.WORKLOADS["c4"]
    seqs = [(0, 0), (1, 3), (2, 6), (w.B - 1, w.Hkv - 1)]
    for which in ("k", "v"):
        x = synthetic.kv(w, which)
        c = encode_gpu(handles[128], 128, torch_input(x, w.kv_dtype), Tcap=w.T, which=which)[0 if which == "k" else 1]
        g = _flat(unpack_cache(c, 0, w.T, seqs))
        xs = np.stack([x[b, hk] for b, hk in seqs])
        del x, c
        st = check_encode(prms[128], _x64(xs), g if which == "k" else None, g if which == "v" else None)
        print(which.upper(), st)


def test_encode_d64_bench_sampled(handles, prms):
    """The head_dim 64 benchmark workload's cache (B=4, 8 kv heads, 102400 bf16
    tokens, outliers and log-normal norms): two whole sequences, the last among
    them, against the oracle's encode."""
    w = synthetic.Workload("d64", "d64 bench", B=4, Hq=16, Hkv=8, d=64, T=102400, kv_dtype="bf16",
                           q_dtype="bf16", lognormal_norms=True, seed=640, scale=0.125)
    seqs = [(0, 0), (w.B - 1, w.Hkv - 1)]
    for which in ("k", "v"):
        x = synthetic.kv(w, which)
        c = encode_gpu(handles[64], 64, torch_input(x, w.kv_dtype), Tcap=w.T, which=which)[0 if which == "k" else 1]
        g = _flat(unpack_cache(c, 0, w.T, seqs))
        xs = np.stack([x[b, hk] for b, hk in seqs])
        del x, c
        st = check_encode(prms[64], _x64(xs), g if which == "k" else None, g if which == "v" else None)
        print(which.upper(), st)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
def test_encode_ragged_offsets_strides(handles, prms, d, dtype):
    B, Hkv, T, t0, Tcap = 2, 3, 77, 50, 192
    base = synthetic.gaussian((B, T, Hkv, d), seed=d + len(dtype))     # [B, T, H, d]: strided heads
    base[..., 3] *= 20.0
    if dtype == "bf16":
        base = synthetic.bf16_round(base)
    elif dtype == "f16":
        base = base.astype(np.float16).astype(np.float32)
    xt = torch_input(base, dtype).permute(0, 2, 1, 3)                    # view [B, H, T, d]
    assert not xt.is_contiguous()
    kc, vc = encode_gpu(handles[d], d, xt, Tcap=Tcap, t0=t0)
    x = base.transpose(0, 2, 1, 3)
    print(check_encode(prms[d], _x64(x), _flat(unpack_cache(kc, t0, T)), _flat(unpack_cache(vc, t0, T))))
    # tokens outside [t0, t0 + T) are untouched (buffers started as zeros)
    for c in (kc, vc):
        u = unpack_cache(c, 0, Tcap)
        for k, v in u.items():
            assert not np.any(v[:, :t0]) and not np.any(v[:, t0 + T:]), k


def test_encode_zero_and_special_vectors(handles, prms):
    d = 128
    x = np.zeros((1, 1, 5, d), np.float32)
    x[0, 0, 1, 7] = 3.0
    x[0, 0, 2] = 1e-3
    x[0, 0, 3] = synthetic.gaussian((d,), seed=1) * 1000.0
    x[0, 0, 4, :64] = -2.0
    kc, vc = encode_gpu(handles[d], d, torch_input(x, "f32"), Tcap=64)
    gk, gv = _flat(unpack_cache(kc, 0, 5)), _flat(unpack_cache(vc, 0, 5))
    assert np.all(gk["idx"][0] == 4) and np.all(gk["sig"][0] == 1)
    assert gk["nh"][0] == 0 and gk["gh"][0] == 0 and gv["nh"][0] == 0
    print(check_encode(prms[d], _x64(x), gk, gv))


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("paged", [False, True])
def test_encode_tensor_core_rotation_path(handles, prms, d, dtype, paged):
    """Bulk encodes of contiguous bf16 / fp16 input of at least 16384 vectors
    (the rotation on the tensor cores, quantisation from tensor memory) at
    head_dim 64 and 128: 18000 vectors (a ragged last tile), a token offset that
    straddles cache blocks, special vectors (zero, one-hot, tiny, large,
    half-constant), contiguous and paged caches; every vector against the
    oracle's encode, and tokens outside the written range stay untouched."""
    B, Hkv, T, t0 = 1, 3, 6000, 37
    Tcap, NB = 6080, 95
    x = synthetic.gaussian((B, Hkv, T, d), seed=770 + len(dtype) + d)
    x[..., 5] *= 20.0
    x[0, 0, 0] = 0.0
    x[0, 0, 1] = 0.0
    x[0, 0, 1, 7] = 3.0
    x[0, 1, 2] = 1e-3
    x[0, 1, 3] *= 1000.0
    x[0, 2, 4] = 0.0
    x[0, 2, 4, :d // 2] = -2.0
    x = synthetic.bf16_round(x) if dtype == "bf16" else x.astype(np.float16).astype(np.float32)
    xt = torch_input(x, dtype)
    assert xt.is_contiguous() and B * Hkv * T >= 16384
    if paged:
        pool = 2 * B * Hkv * NB + 3
        perm = np.random.default_rng(11).permutation(pool).astype(np.int32)
        kt = torch.from_numpy(perm[:B * Hkv * NB].reshape(B * Hkv, NB).copy()).cuda()
        vt = torch.from_numpy(perm[B * Hkv * NB:2 * B * Hkv * NB].reshape(B * Hkv, NB).copy()).cuda()
        kc = tq.Cache(d, True, B, Hkv, Tcap, block_table=kt, pool_blocks=pool)
        vc = tq.Cache(d, False, B, Hkv, Tcap, block_table=vt, pool_blocks=pool)
    else:
        kc, vc = tq.Cache(d, True, B, Hkv, Tcap), tq.Cache(d, False, B, Hkv, Tcap)
    tq.tq_encode_k(handles[d], xt, kc, t0)
    tq.tq_encode_v(handles[d], xt, vc, t0)
    torch.cuda.synchronize()
    assert tq.tq_device_status(handles[d]) == tq.TQ_OK
    if paged:                      # logical order, as a contiguous cache would hold it
        kl, vl = tq.Cache(d, True, B, Hkv, Tcap), tq.Cache(d, False, B, Hkv, Tcap)
        kl.buf.copy_(_gather_blocks(kc, kt))
        vl.buf.copy_(_gather_blocks(vc, vt))
        kc, vc = kl, vl
    gk, gv = _flat(unpack_cache(kc, t0, T)), _flat(unpack_cache(vc, t0, T))
    assert np.all(gk["idx"][0] == 4) and np.all(gk["sig"][0] == 1)
    assert gk["nh"][0] == 0 and gk["gh"][0] == 0 and gv["nh"][0] == 0
    print(check_encode(prms[d], _x64(x), gk, gv))
    for c in (kc, vc):
        u = unpack_cache(c, 0, Tcap)
        for k, v in u.items():
            assert not np.any(v[:, :t0]) and not np.any(v[:, t0 + T:]), k


@pytest.mark.parametrize("d", [64, 128, 256])
def test_append_one_token_at_a_time_equals_bulk(handles, d):
    """Bulk encodes (over 4 vectors per SM: the tiled kernel) and one-token
    appends (the small-batch kernel) write identical bytes."""
    B, Hkv, T, Tcap = 2, 4, 130, 192
    x = torch_input(synthetic.gaussian((B, Hkv, T, d), seed=3), "f32")
    kb, vb = encode_gpu(handles[d], d, x, Tcap=Tcap)
    ka, va = tq.Cache(d, True, B, Hkv, Tcap), tq.Cache(d, False, B, Hkv, Tcap)
    for t in range(T):
        encode_gpu(handles[d], d, x[:, :, t:t + 1], Tcap=Tcap, t0=t, kc=ka, vc=va)
    torch.cuda.synchronize()
    assert torch.equal(ka.buf, kb.buf) and torch.equal(va.buf, vb.buf)


# ------------------------------------------------------------------ attention

def _attend_case(h, prm, w, x_k, x_v, q, T, Tcap, seq_lens=None):
    d = w.d
    kc, _ = encode_gpu(h, d, torch_input(x_k, w.kv_dtype), Tcap=Tcap, which="k")
    _, vc = encode_gpu(h, d, torch_input(x_v, w.kv_dtype), Tcap=Tcap, which="v")
    qt = torch_input(q, w.q_dtype)
    sl = torch.tensor(seq_lens, dtype=torch.int32, device="cuda") if seq_lens is not None else None
    out = attend_gpu(h, qt, kc, vc, T=T, seq_lens=sl, scale=w.scale).cpu().numpy()
    ku, vu = unpack_cache(kc, 0, Tcap), unpack_cache(vc, 0, Tcap)
    lens = seq_lens if seq_lens is not None else [T] * q.shape[0]
    ref = oracle_attend(prm, q.astype(np.float64), ku, vu, kc.Hkv, lens, w.scale)
    err = rel_err_rows(out, ref)
    return out, ref, err


def test_attend_single_head(decode_path, handles, prms):
    w = synthetic.WORKLOADS["c1"]
    out, ref, err = _attend_case(handles[128], prms[128], w, synthetic.kv(w, "k"), synthetic.kv(w, "v"),
                                 synthetic.queries(w), w.T, w.T)
    print("max rel err", err.max(), "per element", rel_err_elements(out, ref))
    assert err.max() <= ATT_TOL


def test_attend_gqa_32_8_40960_full(decode_path, handles, prms):
    w = synthetic.WORKLOADS["c3"]
    out, ref, err = _attend_case(handles[128], prms[128], w, synthetic.kv(w, "k"), synthetic.kv(w, "v"),
                                 synthetic.queries(w), w.T, w.T)
    print("max rel err", err.max(), "per element", rel_err_elements(out, ref))
    assert err.max() <= ATT_TOL


def test_attend_long_context_b4_102400_full(decode_path, handles, prms):
    """The benchmark's workload and launch configuration, every output compared."""
    w = synthetic.WORKLOADS["c4"]
    out, ref, err = _attend_case(handles[128], prms[128], w, synthetic.kv(w, "k"), synthetic.kv(w, "v"),
                                 synthetic.queries(w), w.T, w.T)
    print("max rel err", err.max(), "per element", rel_err_elements(out, ref), "path",
          tq.tq_attend_path(handles[128], w.Hq, w.Hkv), decode_path)
    assert err.max() <= ATT_TOL


def test_append_and_attend_loop_d256(handles, prms):
    """256 append-and-attend steps from 8192 tokens (B=16, Hq=32/Hkv=8, d=256);
    several steps checked against the oracle; the grown cache equals a bulk encode."""
    w = synthetic.WORKLOADS["c5"]
    h, d = handles[256], 256
    Tend = w.T + w.steps
    Tcap = (Tend + 63) // 64 * 64
    xk = torch_input(synthetic.kv(w, "k"), "f32")
    xv = torch_input(synthetic.kv(w, "v"), "f32")
    kc, vc = tq.Cache(d, True, w.B, w.Hkv, Tcap), tq.Cache(d, False, w.B, w.Hkv, Tcap)
    tq.tq_encode_k(h, xk[:, :, :w.T], kc, 0)
    tq.tq_encode_v(h, xv[:, :, :w.T], vc, 0)
    check = {0: None, 1: None, 127: None, w.steps - 1: None}
    ws = torch.empty(tq.tq_attend_workspace_bytes(h, w.B, w.Hq, w.Hkv, Tend), dtype=torch.uint8, device="cuda")
    out = torch.empty((w.B, w.Hq, d), dtype=torch.float32, device="cuda")
    for s in range(w.steps):
        T = w.T + s
        tq.tq_encode_k(h, xk[:, :, T:T + 1], kc, T)
        tq.tq_encode_v(h, xv[:, :, T:T + 1], vc, T)
        q = torch_input(synthetic.queries(w, s), w.q_dtype)
        tq.tq_attend_decode(h, q, kc, vc, out, ws, T=T + 1, scale=w.scale)
        if s in check:
            check[s] = out.cpu().numpy().copy()
    ku, vu = unpack_cache(kc, 0, Tend), unpack_cache(vc, 0, Tend)
    for s, o in check.items():
        T = w.T + s + 1
        ref = oracle_attend(prms[d], synthetic.queries(w, s).astype(np.float64), ku, vu, w.Hkv, [T] * w.B, w.scale)
        err = rel_err_rows(o, ref)
        print("step", s, "max rel err", err.max())
        assert err.max() <= ATT_TOL
    kb, vb = encode_gpu(h, d, xk, Tcap=Tcap)
    _, vb = encode_gpu(h, d, xv, Tcap=Tcap, which="v")
    torch.cuda.synchronize()
    assert torch.equal(kb.buf, kc.buf) and torch.equal(vb.buf, vc.buf)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("G,T0,Lq", [(4, 0, 20), (2, 100, 37), (1, 64, 5), (8, 300, 17), (3, 70, 23), (16, 129, 9)])
def test_attend_prefill_matches_oracle(handles, prms, d, G, T0, Lq):
    """Chunked prefill: query i of the chunk attends causally over tokens
    [0, T0 + i]; every query row equals the oracle's attention over T0 + i + 1
    tokens within the tolerance (ragged row tiles, queries at the cache start,
    all group sizes)."""
    h = handles[d]
    B, Hkv = 2, 2
    Hq, T = Hkv * G, T0 + Lq
    Tcap = (T + 63) // 64 * 64
    x = synthetic.gaussian((2, B, Hkv, T, d), seed=81 + G)
    x[:, :, :, :, 5] *= 20.0                                     # an outlier channel
    kc, vc = tq.Cache(d, True, B, Hkv, Tcap), tq.Cache(d, False, B, Hkv, Tcap)
    tq.tq_encode_k(h, torch_input(x[0], "f32"), kc, 0)
    tq.tq_encode_v(h, torch_input(x[1], "f32"), vc, 0)
    q = synthetic.gaussian((B, Lq, Hq, d), seed=82)
    ws = torch.empty(tq.tq_prefill_workspace_bytes(h, B, Lq, Hq), dtype=torch.uint8, device="cuda")
    out = torch.full((B, Lq, Hq, d), float("nan"), dtype=torch.float32, device="cuda")
    scale = 1.0 / np.sqrt(d)
    tq.tq_attend_prefill(h, torch_input(q, "bf16"), kc, vc, T0, out, ws, scale=scale)
    got = out.cpu().numpy()
    ku, vu = unpack_cache(kc, 0, T), unpack_cache(vc, 0, T)
    qb = synthetic.bf16_round(q).astype(np.float64)
    worst = 0.0
    for i in range(Lq):
        ref = oracle_attend(prms[d], qb[:, i], ku, vu, Hkv, [T0 + i + 1] * B, scale)
        worst = max(worst, float(rel_err_rows(got[:, i], ref).max()))
    print("prefill max rel err", worst)
    assert worst <= ATT_TOL
    assert tq.tq_device_status(h) == tq.TQ_OK


@pytest.mark.parametrize("d", [64, 128])
def test_attend_prefill_bench_size_sampled_rows(handles, prms, d):
    """The benchmark's prefill workloads and launch configuration (c3's cache:
    B=1, Hq=32/Hkv=8, 40960 tokens, at d = 128 and with the same recipe at
    d = 64; the last 512 tokens' queries as one chunk): sampled query rows of
    two kv heads (first, middle, last query of the chunk) against the oracle's
    decode over T0 + i + 1 tokens, and every output finite."""
    w = synthetic.WORKLOADS["c3"]
    if d != w.d:
        w = dataclasses.replace(w, d=d, scale=1.0 / math.sqrt(d))
    B, Hq, Hkv, T = w.B, w.Hq, w.Hkv, w.T
    G, Lq = Hq // Hkv, 512
    T0 = T - Lq
    h = handles[d]
    kc, _ = encode_gpu(h, d, torch_input(synthetic.kv(w, "k"), w.kv_dtype), Tcap=T, which="k")
    _, vc = encode_gpu(h, d, torch_input(synthetic.kv(w, "v"), w.kv_dtype), Tcap=T, which="v")
    q = synthetic.bf16_round(synthetic.gaussian((B, Lq, Hq, d), seed=11))
    ws = torch.empty(tq.tq_prefill_workspace_bytes(h, B, Lq, Hq), dtype=torch.uint8, device="cuda")
    out = torch.full((B, Lq, Hq, d), float("nan"), dtype=torch.float32, device="cuda")
    tq.tq_attend_prefill(h, torch_input(q, "bf16"), kc, vc, T0, out, ws, scale=w.scale)
    got = out.cpu().numpy()
    assert np.all(np.isfinite(got))
    worst = 0.0
    for hk in (0, Hkv - 1):
        ku, vu = unpack_cache(kc, 0, T, [(0, hk)]), unpack_cache(vc, 0, T, [(0, hk)])
        for i in (0, Lq // 2, Lq - 1):
            kcs = {k: v[0, :T0 + i + 1] for k, v in ku.items()}
            vcs = {k: v[0, :T0 + i + 1] for k, v in vu.items()}
            ref = O.attend(prms[d], q[0, i, hk * G:(hk + 1) * G].astype(np.float64), kcs, vcs, w.scale)
            worst = max(worst, float(rel_err_rows(got[0, i, hk * G:(hk + 1) * G], ref).max()))
    print("prefill bench-size sampled max rel err", worst)
    assert worst <= ATT_TOL
    assert tq.tq_device_status(h) == tq.TQ_OK


@pytest.mark.parametrize("d", [64, 128, 256])
def test_attend_prefill_paged_equals_contiguous(handles, d):
    """Prefill over paged caches (random block tables) gives the same output,
    bit for bit, as over contiguous caches holding the same blocks."""
    h = handles[d]
    B, Hkv, G, T0, Lq, Tcap = 2, 2, 4, 150, 40, 192
    Hq, NB = Hkv * G, Tcap // 64
    x = torch_input(synthetic.gaussian((2, B, Hkv, T0 + Lq, d), seed=91), "f32")
    kc, vc = tq.Cache(d, True, B, Hkv, Tcap), tq.Cache(d, False, B, Hkv, Tcap)
    perm = np.random.default_rng(3).permutation(2 * B * Hkv * NB).astype(np.int32)
    kt = torch.from_numpy(perm[:B * Hkv * NB].reshape(B * Hkv, NB).copy()).cuda()
    vt = torch.from_numpy(perm[B * Hkv * NB:].reshape(B * Hkv, NB).copy()).cuda()
    kp = tq.Cache(d, True, B, Hkv, Tcap, block_table=kt, pool_blocks=2 * B * Hkv * NB)
    vp = tq.Cache(d, False, B, Hkv, Tcap, block_table=vt, pool_blocks=2 * B * Hkv * NB)
    for k_, v_ in ((kc, vc), (kp, vp)):
        tq.tq_encode_k(h, x[0], k_, 0)
        tq.tq_encode_v(h, x[1], v_, 0)
    q = torch_input(synthetic.gaussian((B, Lq, Hq, d), seed=92), "f32")
    ws = torch.empty(tq.tq_prefill_workspace_bytes(h, B, Lq, Hq), dtype=torch.uint8, device="cuda")
    outs = []
    for k_, v_ in ((kc, vc), (kp, vp)):
        o = torch.empty((B, Lq, Hq, d), dtype=torch.float32, device="cuda")
        tq.tq_attend_prefill(h, q, k_, v_, T0, o, ws, scale=0.1)
        outs.append(o)
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1])
    assert tq.tq_device_status(h) == tq.TQ_OK


def _gather_blocks(cache: tq.Cache, table: torch.Tensor) -> torch.Tensor:
    """The pool blocks of a paged cache in logical order ([B][Hkv][Tcap/64])."""
    bb = O.block_bytes(cache.head_dim, cache.is_k)
    pool = cache.buf[:cache.pool_blocks * bb].view(cache.pool_blocks, bb)
    return pool.index_select(0, table.flatten().long()).flatten()


@pytest.mark.parametrize("d", [64, 128, 256])
def test_paged_cache_matches_contiguous(handles, prms, d):
    """Paged caches (blocks scattered over a pool by a random table) hold the
    same bytes per logical block as contiguous caches after bulk encodes and
    one-token appends; attention over them (the fused step) gives the same
    output bit for bit as the separate calls on contiguous caches, and the
    oracle's within the tolerance."""
    h = handles[d]
    B, Hkv, G, T0, S, Tcap = 2, 3, 4, 150, 3, 256
    Hq, NB = Hkv * G, Tcap // 64
    pool = 2 * B * Hkv * NB + 5
    perm = np.random.default_rng(7).permutation(pool).astype(np.int32)
    kt = torch.from_numpy(perm[:B * Hkv * NB].reshape(B * Hkv, NB).copy()).cuda()
    vt = torch.from_numpy(perm[B * Hkv * NB:2 * B * Hkv * NB].reshape(B * Hkv, NB).copy()).cuda()
    kp = tq.Cache(d, True, B, Hkv, Tcap, block_table=kt, pool_blocks=pool)
    vp = tq.Cache(d, False, B, Hkv, Tcap, block_table=vt, pool_blocks=pool)
    kc, vc = tq.Cache(d, True, B, Hkv, Tcap), tq.Cache(d, False, B, Hkv, Tcap)
    x = torch_input(synthetic.gaussian((2, B, Hkv, T0 + S, d), seed=61), "bf16")
    q = torch_input(synthetic.gaussian((S, B, Hq, d), seed=62), "f32")
    for k_, v_ in ((kc, vc), (kp, vp)):
        tq.tq_encode_k(h, x[0, :, :, :T0], k_, 0)
        tq.tq_encode_v(h, x[1, :, :, :T0], v_, 0)
    ws = torch.empty(tq.tq_attend_workspace_bytes(h, B, Hq, Hkv, Tcap), dtype=torch.uint8, device="cuda")
    scale = 1.0 / np.sqrt(d)
    for s in range(S):
        t0 = T0 + s
        ref = torch.empty((B, Hq, d), dtype=torch.float32, device="cuda")
        out = torch.full((B, Hq, d), float("nan"), dtype=torch.float32, device="cuda")
        tq.tq_encode_k(h, x[0, :, :, t0:t0 + 1], kc, t0)
        tq.tq_encode_v(h, x[1, :, :, t0:t0 + 1], vc, t0)
        tq.tq_attend_decode(h, q[s], kc, vc, ref, ws, T=t0 + 1, scale=scale)
        tq.tq_append_attend(h, x[0, :, :, t0:t0 + 1], x[1, :, :, t0:t0 + 1], kp, vp, t0, q[s], out, ws,
                            scale=scale)
        torch.cuda.synchronize()
        assert torch.equal(out, ref), f"step {s}"
    assert torch.equal(_gather_blocks(kp, kt), kc.buf) and torch.equal(_gather_blocks(vp, vt), vc.buf)
    T = T0 + S
    oref = oracle_attend(prms[d], q[S - 1].double().cpu().numpy(), unpack_cache(kc, 0, T), unpack_cache(vc, 0, T),
                         Hkv, [T] * B, scale)
    assert rel_err_rows(out.cpu().numpy(), oref).max() <= ATT_TOL
    assert tq.tq_device_status(h) == tq.TQ_OK


def test_paged_cache_bad_table_entry_is_a_device_check(handles):
    """A block-table entry outside the pool is caught by the kernels' own
    check: nothing is written through it, reads go to block 0 (valid memory),
    and tq_device_status reports the failed check once."""
    d, h = 128, handles[128]
    table = torch.tensor([[0, 2]], dtype=torch.int32, device="cuda")     # block 2 is outside a 2-block pool
    kp = tq.Cache(d, True, 1, 1, 128, block_table=table, pool_blocks=2)
    vp = tq.Cache(d, False, 1, 1, 128, block_table=table, pool_blocks=2)
    x = torch_input(synthetic.gaussian((1, 1, 128, d), seed=71), "f32")
    tq.tq_encode_k(h, x, kp, 0)
    tq.tq_encode_v(h, x, vp, 0)
    assert tq.tq_device_status(h) == tq.TQ_ERR_DEVICE_CHECK
    assert tq.tq_device_status(h) == tq.TQ_OK                                 # the check word was cleared
    for c in (kp, vp):
        bb = O.block_bytes(d, c.is_k)
        assert torch.any(c.buf[:bb] != 0) and not torch.any(c.buf[bb:2 * bb] != 0)
    q = torch_input(synthetic.gaussian((1, 4, d), seed=72), "f32")
    ws = torch.empty(tq.tq_attend_workspace_bytes(h, 1, 4, 1, 128), dtype=torch.uint8, device="cuda")
    out = torch.empty((1, 4, d), dtype=torch.float32, device="cuda")
    tq.tq_attend_decode(h, q, kp, vp, out, ws, T=128, scale=1.0 / np.sqrt(d))
    assert tq.tq_device_status(h) == tq.TQ_ERR_DEVICE_CHECK
    assert torch.isfinite(out).all()


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("G,T0,Tnew", [(2, 0, 1), (4, 63, 1), (1, 64, 3), (8, 200, 2), (4, 1000, 1), (16, 100, 1)])
def test_fused_append_attend_equals_separate_calls(handles, d, G, T0, Tnew):
    """tq_append_attend writes the same cache bytes and outputs, bit for bit, as
    tq_encode_k + tq_encode_v + tq_attend_decode, over several steps, with the
    new tokens at the start, middle and end of chunks and splits."""
    h = handles[d]
    B, Hkv, S = 2, 2, 4
    Hq = Hkv * G
    Tend = T0 + S * Tnew
    Tcap = (Tend + 63) // 64 * 64
    x = torch_input(synthetic.gaussian((2, B, Hkv, Tend, d), seed=11 + G), "bf16")
    q = torch_input(synthetic.gaussian((S, B, Hq, d), seed=12), "f32")
    caches = []
    for _ in range(2):
        kc, vc = tq.Cache(d, True, B, Hkv, Tcap), tq.Cache(d, False, B, Hkv, Tcap)
        if T0:
            tq.tq_encode_k(h, x[0, :, :, :T0], kc, 0)
            tq.tq_encode_v(h, x[1, :, :, :T0], vc, 0)
        caches.append((kc, vc))
    ws = torch.empty(tq.tq_attend_workspace_bytes(h, B, Hq, Hkv, Tend), dtype=torch.uint8, device="cuda")
    for s in range(S):
        t0 = T0 + s * Tnew
        (kc, vc), (kf, vf) = caches
        ref = torch.empty((B, Hq, d), dtype=torch.float32, device="cuda")
        out = torch.full((B, Hq, d), float("nan"), dtype=torch.float32, device="cuda")
        tq.tq_encode_k(h, x[0, :, :, t0:t0 + Tnew], kc, t0)
        tq.tq_encode_v(h, x[1, :, :, t0:t0 + Tnew], vc, t0)
        tq.tq_attend_decode(h, q[s], kc, vc, ref, ws, T=t0 + Tnew, scale=1.0 / np.sqrt(d))
        tq.tq_append_attend(h, x[0, :, :, t0:t0 + Tnew], x[1, :, :, t0:t0 + Tnew], kf, vf, t0, q[s], out, ws,
                            scale=1.0 / np.sqrt(d))
        torch.cuda.synchronize()
        assert torch.equal(out, ref), f"step {s}"
        assert torch.equal(kf.buf, kc.buf) and torch.equal(vf.buf, vc.buf), f"step {s}"
    assert tq.tq_device_status(h) == tq.TQ_OK


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("fused", [False, True])
def test_append_and_attend_graph_replay_equals_eager(handles, d, fused):
    """The append-and-attend step sequence (separate calls, or the fused
    tq_append_attend) captured in a CUDA graph and replayed gives the same
    outputs, bit for bit, as launching it eagerly."""
    h = handles[d]
    B, Hq, Hkv, T0, S = 2, 8, 2, 200, 12
    Tcap = (T0 + S + 63) // 64 * 64
    xk = torch_input(synthetic.gaussian((B, Hkv, T0 + S, d), seed=5), "f32")
    xv = torch_input(synthetic.gaussian((B, Hkv, T0 + S, d), seed=6), "f32")
    q = torch_input(synthetic.gaussian((S, B, Hq, d), seed=7), "bf16")
    kc, vc = tq.Cache(d, True, B, Hkv, Tcap), tq.Cache(d, False, B, Hkv, Tcap)
    tq.tq_encode_k(h, xk[:, :, :T0], kc, 0)
    tq.tq_encode_v(h, xv[:, :, :T0], vc, 0)
    ws = torch.empty(tq.tq_attend_workspace_bytes(h, B, Hq, Hkv, T0 + S), dtype=torch.uint8, device="cuda")
    out = torch.zeros((S, B, Hq, d), dtype=torch.float32, device="cuda")

    def sequence():
        for s in range(S):
            T = T0 + s
            if fused:
                tq.tq_append_attend(h, xk[:, :, T:T + 1], xv[:, :, T:T + 1], kc, vc, T, q[s], out[s], ws,
                                    scale=1.0 / np.sqrt(d))
                continue
            tq.tq_encode_k(h, xk[:, :, T:T + 1], kc, T)
            tq.tq_encode_v(h, xv[:, :, T:T + 1], vc, T)
            tq.tq_attend_decode(h, q[s], kc, vc, out[s], ws, T=T + 1, scale=1.0 / np.sqrt(d))

    sequence()
    torch.cuda.synchronize()
    ref, kref, vref = out.clone(), kc.buf.clone(), vc.buf.clone()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        sequence()
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        sequence()
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    assert torch.equal(kc.buf, kref) and torch.equal(vc.buf, vref)
    assert tq.tq_device_status(h) == tq.TQ_OK
    del g


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("G", [1, 2, 3, 4, 6, 8, 16])
def test_attend_group_sizes_and_ragged_lengths(decode_path, handles, prms, d, G):
    Hkv, B, Tcap = 2, 3, 320
    w = synthetic.Workload("t", "edge", B=B, Hq=Hkv * G, Hkv=Hkv, d=d, T=Tcap, kv_dtype="f32", q_dtype="f32",
                           lognormal_norms=False, seed=d + G, scale=1.0 / math.sqrt(d))
    xk, xv = synthetic.kv(w, "k"), synthetic.kv(w, "v")
    q = synthetic.queries(w)
    lens = [1, 65, Tcap]
    out, ref, err = _attend_case(handles[d], prms[d], w, xk, xv, q, 0, Tcap, seq_lens=lens)
    assert err.max() <= ATT_TOL
    lens = [0, 200, 17]
    out, ref, err = _attend_case(handles[d], prms[d], w, xk, xv, q, 0, Tcap, seq_lens=lens)
    assert np.all(out[0] == 0.0)
    assert err.max() <= ATT_TOL


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("G", [1, 2, 4, 8, 16])
def test_attend_polar_only_k(decode_path, handles, prms, d, G):
    """PolarQuant-only K (a V-layout K cache from tq_encode_v): the kernels'
    attention equals the oracle's with gamma = 0 (no QJL term), ragged lengths;
    the K cache holds the oracle's V-flow codes and norms."""
    Hkv, B, Tcap = 2, 3, 320
    Hq = Hkv * G
    h = handles[d]
    xk = torch_input(synthetic.gaussian((B, Hkv, Tcap, d), seed=31 + G), "f32")
    xv = torch_input(synthetic.gaussian((B, Hkv, Tcap, d), seed=41 + G), "f32")
    kc, vc = tq.Cache(d, False, B, Hkv, Tcap), tq.Cache(d, False, B, Hkv, Tcap)
    tq.tq_encode_v(h, xk, kc, 0)
    tq.tq_encode_v(h, xv, vc, 0)
    q = synthetic.gaussian((B, Hq, d), seed=51)
    lens = [0, 129, 301]
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    ws = torch.empty(tq.tq_attend_workspace_bytes(h, B, Hq, Hkv, Tcap), dtype=torch.uint8, device="cuda")
    out = torch.full((B, Hq, d), float("nan"), dtype=torch.float32, device="cuda")
    scale = 1.0 / np.sqrt(d)
    tq.tq_attend_decode_polar(h, torch_input(q, "f32"), kc, vc, out, ws, seq_lens=sl, scale=scale)
    ku, vu = unpack_cache(kc, 0, Tcap), unpack_cache(vc, 0, Tcap)
    if G == 1:
        print(check_encode(prms[d], xk.double().cpu().numpy().reshape(-1, d), None, _flat(ku)))
    ku = {"idx": ku["idx"], "nh": ku["nh"], "sig": np.ones(ku["idx"].shape, np.uint8),
          "gh": np.zeros_like(ku["nh"])}
    ref = oracle_attend(prms[d], q.astype(np.float64), ku, vu, Hkv, lens, scale)
    err = rel_err_rows(out.cpu().numpy(), ref)
    print("polar-only K max rel err", err.max())
    assert err.max() <= ATT_TOL
    assert tq.tq_device_status(h) == tq.TQ_OK


def test_attend_d64_bench_size_sampled(handles, prms):
    """The benchmark's head_dim 64 workload in its launch configuration (B=4,
    Hq=16/Hkv=8, T=102400, bf16 K/V with outliers and log-normal norms, bf16
    queries): encode and decode on the GPU, two sampled sequences' outputs
    against the oracle over all 102400 tokens, every output finite."""
    w = synthetic.Workload("d64", "d64 bench", B=4, Hq=16, Hkv=8, d=64, T=102400, kv_dtype="bf16",
                           q_dtype="bf16", lognormal_norms=True, seed=640, scale=0.125)
    h, d = handles[64], 64
    kc, _ = encode_gpu(h, d, torch_input(synthetic.kv(w, "k"), w.kv_dtype), Tcap=w.T, which="k")
    _, vc = encode_gpu(h, d, torch_input(synthetic.kv(w, "v"), w.kv_dtype), Tcap=w.T, which="v")
    q = synthetic.queries(w)
    out = attend_gpu(h, torch_input(q, w.q_dtype), kc, vc, T=w.T, scale=w.scale).cpu().numpy()
    assert np.all(np.isfinite(out))
    G = w.Hq // w.Hkv
    worst = 0.0
    for b, hk in ((0, 0), (3, 7)):
        ku, vu = unpack_cache(kc, 0, w.T, [(b, hk)]), unpack_cache(vc, 0, w.T, [(b, hk)])
        ref = O.attend(prms[d], q[b, hk * G:(hk + 1) * G].astype(np.float64),
                       {k: v[0] for k, v in ku.items()}, {k: v[0] for k, v in vu.items()}, w.scale)
        worst = max(worst, float(rel_err_rows(out[b, hk * G:(hk + 1) * G], ref).max()))
    print("d64 bench-size sampled max rel err", worst)
    assert worst <= ATT_TOL
    assert tq.tq_device_status(h) == tq.TQ_OK


def test_attend_d64_many_splits(decode_path, handles, prms):
    """head_dim 64 over 20000 tokens (many splits and chunks, a ragged tail) with
    outlier channels and log-normal norms: every output row against the
    oracle, both decode kernels."""
    w = synthetic.Workload("t", "d64", B=2, Hq=16, Hkv=4, d=64, T=20000, kv_dtype="bf16", q_dtype="bf16",
                           lognormal_norms=True, seed=64, scale=0.125)
    out, ref, err = _attend_case(handles[64], prms[64], w, synthetic.kv(w, "k"), synthetic.kv(w, "v"),
                                 synthetic.queries(w), w.T, 20032)
    print("d64 max rel err", err.max(), "path", tq.tq_attend_path(handles[64], w.Hq, w.Hkv), decode_path)
    assert err.max() <= ATT_TOL
    assert tq.tq_device_status(handles[64]) == tq.TQ_OK


@pytest.mark.parametrize("qdt", ["f32", "bf16", "f16"])
def test_attend_query_dtypes(decode_path, handles, prms, qdt):
    w = synthetic.Workload("t", "qdt", B=1, Hq=8, Hkv=2, d=128, T=500, kv_dtype="bf16", q_dtype=qdt,
                           lognormal_norms=True, seed=9, scale=0.1)
    q = synthetic.queries(w)
    if qdt == "f16":
        q = q.astype(np.float16).astype(np.float32)
    out, ref, err = _attend_case(handles[128], prms[128], w, synthetic.kv(w, "k"), synthetic.kv(w, "v"), q,
                                 w.T, 512)
    assert err.max() <= ATT_TOL


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("G", [1, 4, 12])
@pytest.mark.parametrize("paged", [False, True])
def test_streamk_partition_matches_split_and_oracle(handles, prms, d, G, paged):
    """The stream-K grid (equal shares of the units' chunks laid end to end,
    CTAs that straddle two units with their warps divided between them, a
    partial slot per overlapping CTA, unused slots emptied by the unit's last
    CTA) against the uniform split grid of the same kernel (1e-5) and against
    the oracle, with head groups (G = 12), paged caches and a ragged tail; then
    a fused append step on the stream-K grid equals the separate calls bit for
    bit."""
    h = handles[d]
    B, Hkv, T, Tcap = 3, 5, 3001, 3072
    Hq, NB = Hkv * G, Tcap // 64
    x = synthetic.gaussian((2, B, Hkv, T + 1, d), seed=90 + d + G)
    xt = torch_input(x, "bf16")
    kc, vc = tq.Cache(d, True, B, Hkv, Tcap), tq.Cache(d, False, B, Hkv, Tcap)
    if paged:
        pool = 2 * B * Hkv * NB + 3
        perm = np.random.default_rng(d + G).permutation(pool).astype(np.int32)
        kt = torch.from_numpy(perm[:B * Hkv * NB].reshape(B * Hkv, NB).copy()).cuda()
        vt = torch.from_numpy(perm[B * Hkv * NB:2 * B * Hkv * NB].reshape(B * Hkv, NB).copy()).cuda()
        ka = tq.Cache(d, True, B, Hkv, Tcap, block_table=kt, pool_blocks=pool)
        va = tq.Cache(d, False, B, Hkv, Tcap, block_table=vt, pool_blocks=pool)
    else:
        ka, va = tq.Cache(d, True, B, Hkv, Tcap), tq.Cache(d, False, B, Hkv, Tcap)
    for k_, v_ in ((kc, vc), (ka, va)) if paged else ((ka, va),):
        tq.tq_encode_k(h, xt[0, :, :, :T], k_, 0)
        tq.tq_encode_v(h, xt[1, :, :, :T], v_, 0)
    if not paged:
        kc, vc = ka, va
    q = synthetic.gaussian((B, Hq, d), seed=91)
    qt = torch_input(q, "f32")
    ws = torch.empty(tq.tq_attend_workspace_bytes(h, B, Hq, Hkv, Tcap), dtype=torch.uint8, device="cuda")
    scale = 1.0 / np.sqrt(d)
    outs = {}
    try:
        for path in ("split", "streamk"):
            tq.tq_set_decode_path(h, path)
            out = torch.full((B, Hq, d), float("nan"), dtype=torch.float32, device="cuda")
            tq.tq_attend_decode(h, qt, ka, va, out, ws, T=T, scale=scale)
            outs[path] = out.cpu().numpy()
        # one fused append step on the stream-K grid against the separate calls
        ref = torch.empty((B, Hq, d), dtype=torch.float32, device="cuda")
        fused = torch.full((B, Hq, d), float("nan"), dtype=torch.float32, device="cuda")
        kb, vb = ka.buf.clone(), va.buf.clone()
        tq.tq_encode_k(h, xt[0, :, :, T:T + 1], ka, T)
        tq.tq_encode_v(h, xt[1, :, :, T:T + 1], va, T)
        tq.tq_attend_decode(h, qt, ka, va, ref, ws, T=T + 1, scale=scale)
        ka.buf.copy_(kb)
        va.buf.copy_(vb)
        tq.tq_append_attend(h, xt[0, :, :, T:T + 1], xt[1, :, :, T:T + 1], ka, va, T, qt, fused, ws, scale=scale)
        torch.cuda.synchronize()
    finally:
        tq.tq_set_decode_path(h, "auto")
    assert np.all(np.isfinite(outs["streamk"]))
    assert rel_err_rows(outs["streamk"], outs["split"]).max() <= 1e-5
    oref = oracle_attend(prms[d], q.astype(np.float64), unpack_cache(kc, 0, T), unpack_cache(vc, 0, T), Hkv,
                         [T] * B, scale)
    err = rel_err_rows(outs["streamk"], oref)
    print("stream-K max rel err", err.max())
    assert err.max() <= ATT_TOL
    assert torch.equal(fused, ref)
    assert tq.tq_device_status(h) == tq.TQ_OK


@pytest.mark.parametrize("d", [64, 128, 256])
def test_streamk_polar_only_k(handles, prms, d):
    """PolarQuant-only K (no QJL bit) on the stream-K grid against the uniform
    grid (1e-5) and the oracle with gamma = 0, sequences of one length with a
    ragged tail, two query heads per kv head."""
    h = handles[d]
    B, Hkv, G, T, Tcap = 2, 5, 2, 2501, 2560
    Hq = Hkv * G
    xk = torch_input(synthetic.gaussian((B, Hkv, Tcap, d), seed=81 + d), "bf16")
    xv = torch_input(synthetic.gaussian((B, Hkv, Tcap, d), seed=82 + d), "bf16")
    kc, vc = tq.Cache(d, False, B, Hkv, Tcap), tq.Cache(d, False, B, Hkv, Tcap)
    tq.tq_encode_v(h, xk, kc, 0)
    tq.tq_encode_v(h, xv, vc, 0)
    q = synthetic.gaussian((B, Hq, d), seed=83)
    ws = torch.empty(tq.tq_attend_workspace_bytes(h, B, Hq, Hkv, Tcap), dtype=torch.uint8, device="cuda")
    scale = 1.0 / np.sqrt(d)
    outs = {}
    try:
        for path in ("split", "streamk"):
            tq.tq_set_decode_path(h, path)
            out = torch.full((B, Hq, d), float("nan"), dtype=torch.float32, device="cuda")
            tq.tq_attend_decode_polar(h, torch_input(q, "f32"), kc, vc, out, ws, T=T, scale=scale)
            outs[path] = out.cpu().numpy()
    finally:
        tq.tq_set_decode_path(h, "auto")
    assert rel_err_rows(outs["streamk"], outs["split"]).max() <= 1e-5
    ku, vu = unpack_cache(kc, 0, T), unpack_cache(vc, 0, T)
    ku = {"idx": ku["idx"], "nh": ku["nh"], "sig": np.ones(ku["idx"].shape, np.uint8), "gh": np.zeros_like(ku["nh"])}
    ref = oracle_attend(prms[d], q.astype(np.float64), ku, vu, Hkv, [T] * B, scale)
    err = rel_err_rows(outs["streamk"], ref)
    print("stream-K polar-only K max rel err", err.max())
    assert err.max() <= ATT_TOL
    assert tq.tq_device_status(h) == tq.TQ_OK


def test_split_count_invariance(decode_path, handles):
    """Different split plans (by T, or by Tcap through seq_lens) agree within 1e-5."""
    d, B, Hq, Hkv, T, Tcap = 128, 2, 8, 2, 3000, 8192
    h = handles[d]
    x = torch_input(synthetic.gaussian((B, Hkv, Tcap, d), seed=4), "f32")
    kc, vc = encode_gpu(h, d, x, Tcap=Tcap)
    q = torch_input(synthetic.gaussian((B, Hq, d), seed=5), "f32")
    a = attend_gpu(h, q, kc, vc, T=T, scale=0.2).cpu().numpy()
    b = attend_gpu(h, q, kc, vc, seq_lens=torch.full((B,), T, dtype=torch.int32, device="cuda"),
                   scale=0.2).cpu().numpy()
    assert tq.tq_attend_workspace_bytes(h, B, Hq, Hkv, T) != tq.tq_attend_workspace_bytes(h, B, Hq, Hkv, Tcap)
    assert rel_err_rows(a, b).max() <= 1e-5


def test_group_heads_equal_separate_heads(decode_path, handles):
    """Query heads sharing a KV head give what each gives alone against that head."""
    d, T = 128, 700
    h = handles[d]
    x = synthetic.gaussian((1, 2, T, d), seed=6)
    kc, vc = encode_gpu(h, d, torch_input(x, "f32"), Tcap=768)
    q = torch_input(synthetic.gaussian((1, 8, d), seed=7), "f32")
    full = attend_gpu(h, q, kc, vc, T=T, scale=0.3).cpu().numpy()
    k1, v1 = encode_gpu(h, d, torch_input(x[:, 1:2], "f32"), Tcap=768)
    for g in range(4):
        one = attend_gpu(h, q[:, 4 + g:5 + g].contiguous(), k1, v1, T=T, scale=0.3).cpu().numpy()
        assert rel_err_rows(one[0, 0], full[0, 4 + g]).max() <= 1e-5


@pytest.mark.parametrize("d,G", [(128, 4), (128, 2), (64, 2), (256, 4), (128, 8)])
@pytest.mark.parametrize("path", ["auto", "streamk"])
def test_bounded_wait_give_up_path(handles, prms, d, G, path):
    """Every wait in the attention kernel is bounded.  With the first-wait
    budget set to zero polls every warp gives up at its first staged chunk: the
    call completes, the check word reports the failed wait, the outputs are
    finite (the warps' tokens are left out), and after the budget is restored
    the same handle computes the attention again and matches the oracle.  Also
    on the stream-K grid, where some warps give up before crossing into a
    second sequence."""
    h = handles[d]
    B, Hkv, T = 2, 2, 777
    Hq, Tcap = Hkv * G, 832
    x = synthetic.gaussian((2, B, Hkv, Tcap, d), seed=17)
    kc, vc = tq.Cache(d, True, B, Hkv, Tcap), tq.Cache(d, False, B, Hkv, Tcap)
    tq.tq_encode_k(h, torch_input(x[0], "f32"), kc, 0)
    tq.tq_encode_v(h, torch_input(x[1], "f32"), vc, 0)
    q = synthetic.gaussian((B, Hq, d), seed=18)
    assert tq.tq_device_status(h) == tq.TQ_OK
    try:
        tq.tq_set_decode_path(h, path)
        tq.tq_set_wait_limit(h, 0)
        out = attend_gpu(h, torch_input(q, "f32"), kc, vc, T=T, scale=0.1)
        assert tq.tq_device_status(h) == tq.TQ_ERR_DEVICE_CHECK
        assert torch.isfinite(out).all()
        tq.tq_set_wait_limit(h, -1)
        assert tq.tq_device_status(h) == tq.TQ_OK
        out = attend_gpu(h, torch_input(q, "f32"), kc, vc, T=T, scale=0.1).cpu().numpy()
        assert tq.tq_device_status(h) == tq.TQ_OK
    finally:
        tq.tq_set_wait_limit(h, -1)
        tq.tq_set_decode_path(h, "auto")
    ref = oracle_attend(prms[d], q.astype(np.float64), unpack_cache(kc, 0, Tcap), unpack_cache(vc, 0, Tcap), Hkv,
                        [T] * B, 0.1)
    assert rel_err_rows(out, ref).max() <= ATT_TOL


def test_attend_argument_errors(handles):
    h = handles[128]
    kc, vc = tq.Cache(128, True, 1, 2, 64), tq.Cache(128, False, 1, 2, 64)
    out = torch.empty((1, 4, 128), device="cuda")
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    with pytest.raises(tq.TQError) as e:
        tq.tq_attend_decode(h, torch.zeros((1, 5, 128), device="cuda"), kc, vc, out, ws, T=10)   # Hq % Hkv
    assert e.value.status == tq.TQ_ERR_INVALID_ARG
    q = torch.zeros((1, 4, 128), device="cuda")
    with pytest.raises(tq.TQError) as e:
        tq.tq_attend_decode(h, q, kc, vc, out, ws[:16], T=10)
    assert e.value.status == tq.TQ_ERR_WORKSPACE
    with pytest.raises(tq.TQError) as e:
        tq.tq_attend_decode(h, q, kc, vc, out, ws, T=65)           # T > Tcap
    assert e.value.status == tq.TQ_ERR_INVALID_ARG
    with pytest.raises(tq.TQError) as e:
        tq.tq_attend_decode(h, q, kc, vc, out, ws[1:], T=10)       # misaligned workspace
    assert e.value.status == tq.TQ_ERR_INVALID_ARG
    x = torch.zeros((1, 2, 10, 128), device="cuda")
    with pytest.raises(tq.TQError) as e:
        tq.tq_encode_k(h, x, kc, t0=60)                            # past Tcap
    assert e.value.status == tq.TQ_ERR_INVALID_ARG
    h2 = handles[256]
    k2, v2 = tq.Cache(256, True, 1, 2, 64), tq.Cache(256, False, 1, 2, 64)
    with pytest.raises(tq.TQError) as e:                           # prefill past Tcap
        tq.tq_attend_prefill(h2, torch.zeros((1, 3, 4, 256), device="cuda"), k2, v2, 62,
                             torch.empty((1, 3, 4, 256), device="cuda"), ws)
    assert e.value.status == tq.TQ_ERR_INVALID_ARG
    with pytest.raises(ValueError):                                # a K cache is not a PolarQuant-only K cache
        tq.tq_attend_decode_polar(h, q, kc, vc, out, ws, T=10)
    assert tq.tq_device_status(h) == tq.TQ_OK
