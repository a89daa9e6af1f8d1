"""tq_attend_decode_static: decode attention for callers that cannot allocate
device memory when they run (plugins handed only input/output pointers, serving
loops with a fixed memory budget, deployments that forbid allocation after
start-up).  Its scratch is an array inside the library, so the call takes no
workspace.  This test calls it through the C ABI, twice in a row with different
queries, and checks each output against tq_attend_decode with a caller
workspace on the same inputs (both run the same kernels with the same split
plan, so the outputs must be identical bit for bit); it also checks that sizes needing more scratch
than the array holds are refused.  It lives in its own file, collected last."""
import ctypes as C

import numpy as np
import pytest
import torch

from kv_cache_vector_14_b200 import synthetic, tq

pytestmark = pytest.mark.gpu

def _rows_rel(a: np.ndarray, b: np.ndarray) -> float:
    a = a.reshape(-1, a.shape[-1])
    b = b.reshape(-1, b.shape[-1])
    return float((np.abs(a - b).max(axis=1) / np.maximum(np.abs(b).max(axis=1), 1e-30)).max())


def _static_call(L, h, q, kc, vc, out, T, scale):
    return L.tq_attend_decode_static(h, C.c_void_p(q.data_ptr()), tq.TQ_F32, q.shape[0], q.shape[1],
                                     C.byref(kc.struct), C.byref(vc.struct), None, T, C.c_float(scale),
                                     C.c_void_p(out.data_ptr()),
                                     C.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("d,G", [(128, 4), (256, 2)])
def test_static_scratch_decode_matches_workspace_decode(libtq, d, G):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L = libtq
    B, Hkv, T, Tcap, scale = 2, 2, 1000, 1024, 1.0 / np.sqrt(d)
    Hq = Hkv * G
    h = tq.tq_init(d, 0)
    try:
        x = torch.from_numpy(synthetic.gaussian((2, B, Hkv, Tcap, d), seed=d)).cuda()
        kc, vc = tq.Cache(d, True, B, Hkv, Tcap), tq.Cache(d, False, B, Hkv, Tcap)
        tq.tq_encode_k(h, x[0], kc, 0)
        tq.tq_encode_v(h, x[1], vc, 0)
        ws = torch.empty(tq.tq_attend_workspace_bytes(h, B, Hq, Hkv, T), dtype=torch.uint8, device="cuda")
        for call in range(2):
            q = torch.from_numpy(synthetic.gaussian((B, Hq, d), seed=100 + call)).cuda()
            ref = torch.empty((B, Hq, d), dtype=torch.float32, device="cuda")
            tq.tq_attend_decode(h, q, kc, vc, ref, ws, T=T, scale=scale)
            out = torch.full((B, Hq, d), float("nan"), dtype=torch.float32, device="cuda")
            assert _static_call(L, h, q, kc, vc, out, T, scale) == tq.TQ_OK
            torch.cuda.synchronize()
            assert torch.equal(out, ref), f"call {call}: {_rows_rel(out.cpu().numpy(), ref.cpu().numpy())}"
        assert tq.tq_device_status(h) == tq.TQ_OK
    finally:
        tq.tq_destroy(h)


def test_static_scratch_rejects_sizes_beyond_its_array(libtq):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L = libtq
    d, B, Hq, Hkv, Tcap = 128, 512, 32, 8, 64
    h = tq.tq_init(d, 0)
    try:
        assert tq.tq_attend_workspace_bytes(h, B, Hq, Hkv, Tcap) > (8 << 20)
        kc, vc = tq.Cache(d, True, B, Hkv, Tcap), tq.Cache(d, False, B, Hkv, Tcap)
        q = torch.zeros((B, Hq, d), dtype=torch.float32, device="cuda")
        out = torch.zeros((B, Hq, d), dtype=torch.float32, device="cuda")
        assert _static_call(L, h, q, kc, vc, out, Tcap, 0.1) == tq.TQ_ERR_WORKSPACE
        torch.cuda.synchronize()
        assert not torch.any(out != 0)
    finally:
        tq.tq_destroy(h)
