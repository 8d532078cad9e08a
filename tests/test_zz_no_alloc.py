"""la_prefill_noalloc: the prefill entry point for callers that cannot allocate.

Some callers cannot call cudaMalloc at all: an engine that owns every byte of
device memory up front (a serving runtime with a fixed memory plan, a plugin
living inside another framework's caching allocator), or a path where a
cudaMalloc would synchronise the device.  For them la_prefill_noalloc takes
no workspace and draws the scratch of the intra-sequence split from a static
buffer inside the library.  This test calls it through the C ABI twice in a
row -- the second call reuses a buffer still holding the first call's data --
and checks each result against la_prefill given a caller-allocated workspace,
and every unit of it against the float64 oracle, within the bf16 tolerance
the other parity tests use.

Kept in a file of its own, collected last, so that a run stopping at the
first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import recurrent_decode_la_b200 as la
from gpu_util import BF16_TOL, nerr, prefill_vs_oracle
from recurrent_decode_la_b200 import inputs

pytestmark = pytest.mark.gpu


def _noalloc(lib):
    fn = lib.la_prefill_noalloc
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    fn.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i64, i32, i32, vp, i32, i64, i32, vp]
    fn.restype = ctypes.c_int
    return fn


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return la.load_library()


def test_noalloc_prefill_matches_prefill_twice(lib):
    fn = _noalloc(lib)
    dev = torch.device("cuda")
    stream = torch.cuda.current_stream().cuda_stream
    # two calls in a row with different shapes and inputs; both few enough
    # units that the intra-sequence split (and so the scratch) is used
    for seed, (B, H, T, d, chunk) in enumerate([(1, 4, 8192, 128, 128), (1, 8, 3000, 128, 64)]):
        need = la.la_prefill_workspace_size(torch.bfloat16, B, H, T, d, d, 0, chunk)
        assert 0 < need <= 64 * 1024 * 1024
        q_h, k_h, v_h = inputs.random_qkv(100 + seed, B, H, T, d, d, dtype=torch.bfloat16)
        q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
        S0 = torch.from_numpy(
            np.random.default_rng(seed).standard_normal((B * H, d, d)).astype(np.float32) * 0.05).to(dev)

        # the existing entry point, caller-allocated workspace
        o_ref = torch.empty_like(v)
        st_ref = S0.clone()
        ws = torch.empty(need, dtype=torch.uint8, device=dev)
        la.la_prefill(q, k, v, o_ref, st_ref, chunk=chunk, workspace=ws)

        # the entry point that allocates nothing (output NaN until written)
        o = torch.full_like(v, float("nan"))
        st = S0.clone()
        status = fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), st.data_ptr(), la.LA_BF16,
                    B, H, T, d, d, None, 0, 0, chunk, stream)
        assert status == la.LA_OK, la.la_status_string(status)
        assert la.la_device_status() == la.LA_OK

        assert nerr(o, o_ref.float().cpu().numpy()) <= BF16_TOL
        assert nerr(st, st_ref.cpu().numpy()) <= BF16_TOL
        (e,), _ = prefill_vs_oracle(q_h, k_h, v_h, [(o, st)], S0=S0.cpu().numpy())
        assert e["nonfinite"] == 0 and e["O"] <= BF16_TOL and e["S"] <= BF16_TOL, e
