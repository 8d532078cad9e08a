"""The few-token prefill (at most 16 tokens per unit from a saved state: the
multi-token form of decode) against the float64 oracle: dense and packed
layouts, both dtypes, d_k != d_v, empty sequences, a sequence longer than the
promised max_seqlen (reported, its unit left untouched), agreement with the
chunked kernels, and prefill + short continuation == one longer prefill."""
import numpy as np
import pytest
import torch

import recurrent_decode_la_b200 as la
from gpu_util import BF16_TOL, F32_TOL, gpu_prefill, nerr, run_in_child, tol_for
from oracle import la_oracle as ora
from recurrent_decode_la_b200 import inputs

pytestmark = pytest.mark.gpu


def _state(seed, *shape):
    return torch.from_numpy((np.random.default_rng(seed).standard_normal(shape) * 0.05).astype(np.float32))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (32, 64), (96, 8)])
@pytest.mark.parametrize("T", [1, 2, 5, 16])
def test_short_dense(dtype, dk, dv, T):
    assert la.la_prefill_kernel(dtype, T, dk, dv) == "short"
    B, H = 3, 5
    q, k, v = inputs.random_qkv(T * 31 + dk + dv, B, H, T, dk, dv, dtype=dtype)
    S0 = _state(T + dk, B, H, dk, dv)
    O_ref, S_ref = ora.recurrent(q, k, v, S0)
    o, S = gpu_prefill(q, k, v, S0=S0)
    tol = tol_for(dtype)
    assert nerr(o, O_ref) <= tol
    assert nerr(S.reshape(S_ref.shape), S_ref) <= tol


@pytest.mark.parametrize("max_len", [4, 16])
def test_short_packed_with_empty_sequences(max_len):
    H, d = 4, 128
    lens = np.random.default_rng(max_len).integers(0, max_len + 1, size=300)
    lens[[0, 7, 299]] = 0
    lens[5] = max_len
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    q, k, v = inputs.random_qkv(77, 1, H, int(cu[-1]), d, d, dtype=torch.bfloat16)
    S0 = _state(3, len(lens), H, d, d)
    assert la.la_prefill_kernel(torch.bfloat16, max_len, d, d) == "short"
    O_ref, S_ref = ora.recurrent(q, k, v, S0, cu_seqlens=cu.numpy())
    o, S = gpu_prefill(q, k, v, S0=S0, cu=cu, max_seqlen=max_len)
    assert nerr(o, O_ref) <= BF16_TOL
    assert nerr(S.reshape(S_ref.shape), S_ref) <= BF16_TOL
    S = S.reshape(S_ref.shape).cpu()
    for n in (0, 7, 299):
        assert torch.equal(S[n], S0[n])  # empty sequence: state untouched


def test_short_sequence_longer_than_promised_is_reported():
    """max_seqlen = 4 promised, one sequence has 12 rows: that unit is left as
    it was and la_device_status reports LA_ERR_INVALID_ARG; the others are
    computed."""
    H, d = 2, 64
    lens = np.array([3, 12, 4, 1])
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    T = int(cu[-1])
    q, k, v = inputs.random_qkv(5, 1, H, T, d, d, dtype=torch.float32)
    S0 = _state(9, len(lens), H, d, d)
    O_ref, S_ref = ora.recurrent(q, k, v, S0, cu_seqlens=cu.numpy())
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o = torch.zeros_like(vd)
    st = S0.reshape(-1, d, d).cuda()
    la.la_prefill(qd, kd, vd, o, st, cu_seqlens=cu.cuda(), max_seqlen=4)
    assert la.la_device_status() == la.LA_ERR_INVALID_ARG
    assert la.la_device_status() == la.LA_OK  # reported once, then cleared
    st = st.reshape(len(lens), H, d, d).cpu()
    assert torch.equal(st[1], S0[1])
    assert torch.count_nonzero(o[0, :, 3:15]) == 0
    for n in (0, 2, 3):
        assert nerr(st[n], S_ref[n]) <= F32_TOL
    keep = np.r_[0:3, 15:T]
    assert nerr(o[0][:, keep], O_ref[0][:, keep]) <= F32_TOL


def test_short_matches_chunked_kernels():
    """The same 16-token prefill through the few-token kernel and, in a child
    process started with LINATTN_SHORT=0, through the chunked tensor-core
    kernel: both match the oracle."""
    B, H, T, d, seed = 2, 8, 16, 128, 21
    assert la.la_prefill_kernel(torch.bfloat16, T, d, d) == "short"
    res = {"short": None, "tc": run_in_child("prefill", {"LINATTN_SHORT": "0"}, dtype="bf16", B=B, H=H, T=T, d=d,
                                             seed=seed)}
    assert res["tc"]["kernel"] == "tc"
    q, k, v = inputs.random_qkv(seed, B, H, T, d, d, dtype=torch.bfloat16)
    S0 = torch.from_numpy((np.random.default_rng(seed).standard_normal((B, H, d, d)) * 0.05).astype(np.float32))
    O_ref, S_ref = ora.recurrent(q, k, v, S0)
    o, S = gpu_prefill(q, k, v, S0=S0)
    res["short"] = {"o": nerr(o, O_ref), "S": nerr(S.reshape(S_ref.shape), S_ref)}
    for name, e in res.items():
        assert e["o"] <= BF16_TOL and e["S"] <= BF16_TOL, (name, e)


def test_prefill_then_short_continuation_equals_longer_prefill():
    """Speculative-decoding shape: a prompt, then 8 tokens at once from the
    saved state; same as prefilling all the rows in one call."""
    B, H, T, n, d = 2, 4, 300, 8, 128
    q, k, v = inputs.random_qkv(13, B, H, T + n, d, d, dtype=torch.bfloat16)
    O_ref, S_ref = ora.recurrent(q, k, v)
    _, S = gpu_prefill(q[:, :, :T], k[:, :, :T], v[:, :, :T])
    assert la.la_prefill_kernel(torch.bfloat16, n, d, d) == "short"
    o = torch.empty(B, H, n, d, dtype=torch.bfloat16, device="cuda")
    la.la_prefill(q[:, :, T:].contiguous().cuda(), k[:, :, T:].contiguous().cuda(),
                  v[:, :, T:].contiguous().cuda(), o, S)
    assert la.la_device_status() == la.LA_OK
    assert nerr(o, O_ref[:, :, T:]) <= BF16_TOL
    assert nerr(S.reshape(S_ref.shape), S_ref) <= BF16_TOL


# Many units (768, more than the SMs: one column block per unit, and at
# d_k <= 64 the 128-thread CTAs).
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (32, 64), (96, 8)])
@pytest.mark.parametrize("T", [1, 8, 13])
def test_short_many_units_dense(dtype, dk, dv, T):
    B, H = 16, 48
    assert la.la_prefill_kernel(dtype, T, dk, dv) == "short"
    q, k, v = inputs.random_qkv(T * 7 + dk + 3 * dv, B, H, T, dk, dv, dtype=dtype)
    S0 = _state(T + 2 * dk, B, H, dk, dv)
    O_ref, S_ref = ora.recurrent(q, k, v, S0)
    o, S = gpu_prefill(q, k, v, S0=S0)
    tol = tol_for(dtype)
    assert nerr(o, O_ref) <= tol
    assert nerr(S.reshape(S_ref.shape), S_ref) <= tol


@pytest.mark.parametrize("d", [128, 64])
def test_short_many_units_packed_too_long_and_empty(d):
    """Many packed units (800; at d = 64 the 128-thread CTAs): empty
    sequences keep their state, a sequence longer than the promised
    max_seqlen is reported and left untouched, the others match the
    oracle."""
    H, max_len = 4, 8
    lens = np.random.default_rng(4).integers(0, max_len + 1, size=200)
    lens[[0, 50, 199]] = 0
    lens[77] = 11  # longer than promised
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    T = int(cu[-1])
    q, k, v = inputs.random_qkv(91, 1, H, T, d, d, dtype=torch.bfloat16)
    S0 = _state(17, len(lens), H, d, d)
    O_ref, S_ref = ora.recurrent(q, k, v, S0, cu_seqlens=cu.numpy())
    o = torch.zeros(1, H, T, d, dtype=torch.bfloat16, device="cuda")
    st = S0.reshape(-1, d, d).cuda()
    la.la_prefill(q.cuda(), k.cuda(), v.cuda(), o, st, cu_seqlens=cu.cuda(), max_seqlen=max_len)
    assert la.la_device_status() == la.LA_ERR_INVALID_ARG
    st = st.reshape(len(lens), H, d, d).cpu()
    assert torch.equal(st[77], S0[77])
    for n in (0, 50, 199):
        assert torch.equal(st[n], S0[n])
    a, b = int(cu[77]), int(cu[78])
    assert torch.count_nonzero(o[0, :, a:b]) == 0
    keep_units = [n for n in range(len(lens)) if n != 77]
    assert nerr(st[keep_units], S_ref[keep_units]) <= BF16_TOL
    keep = np.r_[0:a, b:T]
    assert nerr(o[0][:, keep].float().cpu(), O_ref[0][:, keep]) <= BF16_TOL
