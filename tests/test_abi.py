"""Host-side checks of the C ABI, no GPU needed: the library loads, exports every
entry point include/tq.h declares, and its host-only calls agree with the oracle."""
import os
import re

import numpy as np
import pytest

import oracle as O
from kv_cache_vector_14_b200 import tq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "tq.h")).read()
    return sorted(set(re.findall(r"^TQ_API\s+[\w\s\*]+?\b(tq_\w+)\s*\(", src, flags=re.M)))


def test_exports_every_declared_symbol(libtq):
    names = declared_symbols()
    assert len(names) >= 14
    assert set(names) == set(tq.EXPORTED)
    for n in names:
        assert hasattr(libtq, n), n


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("seed", [0, 1, 12345, 2**63 + 7])
def test_params_host_bit_identical_to_oracle(libtq, d, seed):
    p = tq.tq_params_host(d, seed)
    o = O.params(d, seed)
    assert np.array_equal(p["D"], o["D"])
    assert np.array_equal(p["S"].astype(np.float64), o["S"])
    assert np.array_equal(p["c8"].astype(np.float64), o["c8"])
    assert np.array_equal(p["b7"].astype(np.float64), o["b7"])


def test_sizes_and_bits_per_dim(libtq, golden):
    for cache, hd, bpd in golden("bits_per_dim.txt"):
        is_k = cache == "K"
        assert tq.tq_block_bytes(int(hd), is_k) == O.block_bytes(int(hd), is_k)
        assert 8 * tq.tq_cache_bytes(int(hd), is_k, 3, 5, 640) / (3 * 5 * 640 * int(hd)) == float(bpd)
    for d in (64, 128, 256):
        for is_k in (True, False):
            assert tq.tq_block_bytes(d, is_k) == O.block_bytes(d, is_k)
            assert tq.tq_block_bytes(d, is_k) % 16 == 0
    assert tq.tq_block_bytes(32, True) == 0 and tq.tq_block_bytes(512, False) == 0
    assert tq.tq_cache_bytes(128, True, 1, 1, 100) == 0      # Tcap not a multiple of 64
    assert tq.tq_cache_bytes(128, True, 1, 1, 0) == 0


@pytest.mark.parametrize("d", [64, 128, 256])
def test_codebook_is_exactly_antisymmetric(libtq, d):
    """The encode kernels find the cell and the centroid from |y| alone; that
    needs c[7-k] = -c[k], b[6-k] = -b[k] and b[3] = 0 exactly in fp32, and exact
    differences of adjacent centroids (all checked on the library's constants)."""
    p = tq.tq_params_host(d, 0)
    c, b = np.asarray(p["c8"], np.float32), np.asarray(p["b7"], np.float32)
    assert b[3] == 0.0
    assert all(c[7 - k] == -c[k] for k in range(8)) and all(b[6 - k] == -b[k] for k in range(7))
    for k in (4, 5, 6):
        assert np.float64(c[k + 1]) - np.float64(c[k]) == np.float64(np.float32(c[k + 1] - c[k]))


def test_cache_struct_layout():
    """tq_cache as declared in include/tq.h: base, B, Hkv, Tcap, block_table,
    pool_blocks, 8 bytes each."""
    import ctypes as C
    assert C.sizeof(tq.tq_cache) == 48
    assert [getattr(tq.tq_cache, f).offset for f, _ in tq.tq_cache._fields_] == [0, 8, 16, 24, 32, 40]


def test_host_argument_errors(libtq):
    for bad_d in (32, 96, 512):
        with pytest.raises(tq.TQError) as e:
            tq.tq_params_host(bad_d, 0)
        assert e.value.status == tq.TQ_ERR_INVALID_ARG
    L = libtq
    c = tq.tq_cache(None, 1, 1, 64)
    import ctypes as C
    assert L.tq_encode_k(None, None, 0, 1, 1, 1, 0, 0, 0, C.byref(c), 0, None) == tq.TQ_ERR_INVALID_ARG
    assert L.tq_attend_decode(None, None, 0, 1, 1, C.byref(c), C.byref(c), None, 1, 1.0, None, None, 0,
                              None) == tq.TQ_ERR_INVALID_ARG
    assert L.tq_append_attend(None, None, None, 0, 1, 0, 0, 0, C.byref(c), C.byref(c), 0, None, 0, 1, 1.0,
                              None, None, 0, None) == tq.TQ_ERR_INVALID_ARG
    assert L.tq_append_attend(None, None, None, 0, 1, 0, 0, 0, None, None, 0, None, 0, 1, 1.0,
                              None, None, 0, None) == tq.TQ_ERR_INVALID_ARG
    assert L.tq_attend_workspace_bytes(None, 1, 1, 1, 64) == 0
    assert L.tq_attend_prefill(None, None, 0, 1, 1, 1, C.byref(c), C.byref(c), 0, 1.0, None, None, 0,
                               None) == tq.TQ_ERR_INVALID_ARG
    assert L.tq_prefill_workspace_bytes(None, 1, 1, 1) == 0
    assert L.tq_destroy(None) == tq.TQ_OK
    assert L.tq_head_dim(None) == 0
    for s in range(6):
        assert tq.tq_status_string(s)
    assert tq.tq_status_string(99) == "unknown status"


def test_oracle_sketch_given_codes_matches_encode():
    p = O.params(128, 3)
    x = np.random.default_rng(0).standard_normal((50, 128))
    e = O.encode(x, p, with_qjl=True)
    s = O.sketch_given_codes(p, e["y"], e["idx"], e["n"] > 0)
    assert np.array_equal(s["sig"], e["sig"]) and np.array_equal(s["gamma"], e["gamma"])
    idx2 = e["idx"].copy()
    idx2[:, 0] = (idx2[:, 0] + 1) % 8
    s2 = O.sketch_given_codes(p, e["y"], idx2, e["n"] > 0)
    r = e["y"] - p["c8"][idx2]
    assert np.allclose(s2["z"], r @ p["S"].T, atol=1e-12)
