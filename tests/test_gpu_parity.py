"""Parity of the CUDA path (called through the C ABI) with the float64 oracle.

Bars: bit-exact on the slides' integer trace; max |gpu - oracle| / max |oracle|
<= 1e-4 for fp32 inputs and <= 2e-2 for bf16 inputs (fp32 accumulation), for
the prefill output O, the decode outputs o and the final state S.
"""
import numpy as np
import pytest
import torch

import recurrent_decode_la_b200 as la
from oracle import la_oracle as ora
from recurrent_decode_la_b200 import inputs
from gpu_util import (BF16_TOL, F32_TOL, decode_tokens, decode_vs_oracle, gpu_decode_run, gpu_prefill, nerr,
                      prefill_vs_oracle)

pytestmark = pytest.mark.gpu

WL = inputs.WORKLOADS


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    la.load_library()
    yield
    torch.cuda.synchronize()
    assert la.la_device_status() == la.LA_OK


def _example_tensors(golden, dtype):
    k = torch.tensor(golden["k"], dtype=torch.float32)
    v = torch.tensor(golden["v"], dtype=torch.float32)
    return (k.clone()[None, None].to(dtype), k[None, None].to(dtype), v[None, None].to(dtype))


# ----------------------------------------------------- the slides' trace ----

@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("chunk", [1, 2, 4, 8])
def test_worked_example_bit_exact(golden, dtype, chunk):
    q, k, v = _example_tensors(golden, dtype)
    o, S = gpu_prefill(q, k, v, chunk=chunk)
    assert torch.equal(o.float().cpu()[0, 0], torch.tensor(golden["chunk4"]["o"], dtype=torch.float32))
    assert torch.equal(S.cpu()[0], torch.tensor(golden["chunk4"]["S8"], dtype=torch.float32))


def test_worked_example_handoffs_c2(golden):
    """Prefill the first 2, 4, 6 tokens: the states handed off are S_2, S_4, S_6."""
    q, k, v = _example_tensors(golden, torch.float32)
    for n, key in ((2, "S2"), (4, "S4"), (6, "S6")):
        _, S = gpu_prefill(q[:, :, :n], k[:, :, :n], v[:, :, :n], chunk=2)
        assert torch.equal(S.cpu()[0], torch.tensor(golden["chunk2"]["handoffs"][key], dtype=torch.float32))


def test_worked_example_decode_bit_exact(golden):
    """Token-by-token decode of the trace reproduces every o_t and S_8."""
    q, k, v = _example_tensors(golden, torch.float32)
    st = torch.zeros(1, 2, 2, device="cuda")
    outs = []
    for t in range(8):
        o = torch.empty(1, 1, 2, device="cuda")
        la.la_decode_step(q[0, :, t].cuda()[None], k[0, :, t].cuda()[None], v[0, :, t].cuda()[None], o, st)
        outs.append(o.cpu()[0, 0])
    assert torch.equal(torch.stack(outs), torch.tensor(golden["chunk4"]["o"], dtype=torch.float32))
    assert torch.equal(st.cpu()[0], torch.tensor(golden["chunk4"]["S8"], dtype=torch.float32))


# ------------------------------------------------ tiny fp32 workload ----

def test_tiny_f32_prefill_and_decode():
    wl = WL["tiny_f32_b1h1_t64_d16"]
    q, k, v, _ = inputs.prefill_inputs(wl)
    O_ref, S_ref = ora.recurrent(q, k, v)
    o, S = gpu_prefill(q, k, v, chunk=wl.chunk)
    assert nerr(o, O_ref) <= F32_TOL
    assert nerr(S.reshape(S_ref.shape), S_ref) <= F32_TOL
    Sd = S.clone()
    Sr = S_ref.reshape(1, 16, 16)
    for step in range(wl.decode_steps):
        dq, dk_, dv = inputs.decode_token(wl, step, units=1)
        od = torch.empty(1, 1, 16, device="cuda")
        la.la_decode_step(dq.cuda()[None], dk_.cuda()[None], dv.cuda()[None], od, Sd)
        o_ref, Sr = ora.decode_step(dq, dk_, dv, Sr)
        assert nerr(od[0], o_ref) <= F32_TOL
    assert nerr(Sd, Sr) <= F32_TOL


# ------------------------------------- tensor-core path, several tiles ----

@pytest.mark.parametrize("d,chunk", [(64, 16), (128, 16), (64, 32), (128, 32),
                                     (64, 64), (128, 64), (64, 128), (128, 128)])
@pytest.mark.parametrize("T", [1, 63, 64, 333])
def test_tc_prefill_random_state(d, chunk, T):
    assert la.la_prefill_path(torch.bfloat16, d, d, chunk) == "tc"
    B, H = 2, 3
    q, k, v = inputs.random_qkv(7 * T + d + chunk, B, H, T, d, d, dtype=torch.bfloat16)
    S0 = torch.from_numpy(np.random.default_rng(T).standard_normal((B, H, d, d)).astype(np.float32)) * 0.05
    O_ref, S_ref = ora.recurrent(q, k, v, S0)
    o, S = gpu_prefill(q, k, v, S0=S0, chunk=chunk)
    assert nerr(o, O_ref) <= BF16_TOL
    assert nerr(S.reshape(S_ref.shape), S_ref) <= BF16_TOL


@pytest.mark.parametrize("B,H,T,d,chunk", [(1, 4, 4096, 128, 128), (1, 2, 2000, 128, 64),
                                           (2, 3, 1111, 64, 128), (1, 1, 8192, 64, 64),
                                           (1, 2, 1500, 128, 32), (1, 3, 777, 64, 16)])
def test_intra_sequence_split(B, H, T, d, chunk):
    """Few units: each sequence is split into segments that start from S_0 plus
    the K^T V sums of the earlier sub-segments.  Same result as no split."""
    ws = la.la_prefill_workspace_size(torch.bfloat16, B, H, T, d, d, 0, chunk)
    assert ws > 0
    q, k, v = inputs.random_qkv(T + d, B, H, T, d, d, dtype=torch.bfloat16)
    S0 = torch.from_numpy(np.random.default_rng(T).standard_normal((B, H, d, d)).astype(np.float32)) * 0.05
    O_ref, S_ref = ora.recurrent(q, k, v, S0)
    o, S = gpu_prefill(q, k, v, S0=S0, chunk=chunk)
    assert nerr(o, O_ref) <= BF16_TOL
    assert nerr(S.reshape(S_ref.shape), S_ref) <= BF16_TOL
    o2, S2 = gpu_prefill(q, k, v, S0=S0, chunk=chunk, workspace=False)
    assert nerr(o2, O_ref) <= BF16_TOL
    assert nerr(S2.reshape(S_ref.shape), S_ref) <= BF16_TOL


def test_tc_vs_simt_same_inputs():
    """Two kernels, six chunk sizes, one result (chunking never changes it)."""
    q, k, v = inputs.random_qkv(3, 1, 4, 200, 64, 64, dtype=torch.bfloat16)
    O_ref, S_ref = ora.recurrent(q, k, v)
    paths = {8: "simt", 16: "tc", 32: "tc", 48: "simt", 64: "tc", 128: "tc"}
    for chunk, path in paths.items():
        assert la.la_prefill_path(torch.bfloat16, 64, 64, chunk) == path, chunk
        o, S = gpu_prefill(q, k, v, chunk=chunk)
        assert nerr(o, O_ref) <= BF16_TOL, chunk
        assert nerr(S.reshape(S_ref.shape), S_ref) <= BF16_TOL, chunk


def test_misaligned_bf16_runs_simt_and_matches():
    B, H, T, d = 1, 2, 100, 64
    q, k, v = inputs.random_qkv(5, B, H, T, d, d, dtype=torch.bfloat16)
    O_ref, S_ref = ora.recurrent(q, k, v)
    buf = torch.empty(3 * q.numel() + 1, dtype=torch.bfloat16, device="cuda")
    qd = buf[1:1 + q.numel()].view_as(q)
    kd = buf[1 + q.numel():1 + 2 * q.numel()].view_as(q)
    vd = buf[1 + 2 * q.numel():].view_as(q)
    qd.copy_(q.cuda()); kd.copy_(k.cuda()); vd.copy_(v.cuda())
    assert la.la_prefill_path(torch.bfloat16, d, d, 64, qd, kd, vd, qd) == "simt"
    o = torch.empty(B, H, T, d, dtype=torch.bfloat16, device="cuda")
    S = torch.zeros(B * H, d, d, device="cuda")
    la.la_prefill(qd, kd, vd, o, S, chunk=64)
    assert la.la_device_status() == la.LA_OK
    assert nerr(o, O_ref) <= BF16_TOL
    assert nerr(S.reshape(S_ref.shape), S_ref) <= BF16_TOL


# ----------------------------------------------------- edge cases ----

def test_empty_and_degenerate():
    d = 64
    S0 = torch.randn(2, d, d, device="cuda")
    st = S0.clone()
    z = torch.empty(1, 2, 0, d, dtype=torch.bfloat16, device="cuda")
    la.la_prefill(z, z, z, z.clone(), st, chunk=64)          # T = 0: no-op
    assert torch.equal(st, S0)
    with pytest.raises(la.LinAttnError) as e:                  # d above 128
        big = torch.zeros(1, 1, 4, 256, dtype=torch.bfloat16, device="cuda")
        la.la_prefill(big, big, big, big.clone(), torch.zeros(1, 256, 256, device="cuda"))
    assert e.value.status == la.LA_ERR_UNSUPPORTED
    lib = la.load_library()
    assert lib.la_prefill(None, None, None, None, None, 1, 1, 1, 8, 64, 64, None, 0, 0, 64, None, 0, None) \
        == la.LA_ERR_INVALID_ARG
    assert lib.la_decode_step(None, None, None, None, None, 1, 1, 1, 64, 64, None) == la.LA_ERR_INVALID_ARG
    assert lib.la_prefill(None, None, None, None, None, 7, 1, 1, 8, 64, 64, None, 0, 0, 64, None, 0, None) \
        == la.LA_ERR_INVALID_ARG
    assert la.la_device_status() == la.LA_OK


def test_varlen_small_with_empty_sequences():
    H, d = 3, 128
    lens = [70, 0, 64, 1, 200, 5]
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    q, k, v = inputs.random_qkv(9, 1, H, int(cu[-1]), d, d, dtype=torch.bfloat16)
    S0 = torch.from_numpy(np.random.default_rng(0).standard_normal((len(lens), H, d, d)).astype(np.float32)) * 0.05
    O_ref, S_ref = ora.recurrent(q, k, v, S0, cu_seqlens=cu.numpy())
    for chunk in (16, 32, 64, 128):
        o, S = gpu_prefill(q, k, v, S0=S0, cu=cu, chunk=chunk, max_seqlen=max(lens))
        assert nerr(o, O_ref) <= BF16_TOL
        assert nerr(S.reshape(S_ref.shape), S_ref) <= BF16_TOL
        assert torch.equal(S.reshape(S_ref.shape)[1].cpu(), S0[1])  # empty sequence untouched


@pytest.mark.parametrize("n_seqs,H,max_len,d,chunk", [(40, 8, 700, 128, 128), (40, 8, 700, 64, 64),
                                                     (40, 8, 700, 128, 32), (5000, 1, 24, 64, 64)])
def test_varlen_dynamic_walk(n_seqs, H, max_len, d, chunk):
    """More units than SMs, mixed lengths: with the workspace the persistent
    CTAs claim packed units from a counter, longest sequences first (up to
    4096 sequences; beyond, in order).  Every unit must still be computed
    exactly once, with the same arithmetic: the result equals the static walk
    bit for bit (outputs start as NaN, so a skipped unit would show) and
    matches the oracle."""
    lens = np.random.default_rng(d + chunk + n_seqs).integers(0, max_len, size=n_seqs)
    lens[[3, 17]] = 0
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    T = int(cu[-1])
    nb = la.la_prefill_workspace_size(torch.bfloat16, 1, H, T, d, d, n_seqs, chunk)
    assert nb == 256 + (((n_seqs * 4 + 255) // 256) * 256 if n_seqs <= 4096 else 0)
    q, k, v = inputs.random_qkv(11 + d, 1, H, T, d, d, dtype=torch.bfloat16)
    S0 = torch.from_numpy(np.random.default_rng(1).standard_normal((n_seqs, H, d, d)).astype(np.float32)) * 0.05
    O_ref, S_ref = ora.recurrent(q, k, v, S0, cu_seqlens=cu.numpy())
    res = []
    for use_ws in (True, False, True):
        qd, kd, vd, cud = q.cuda(), k.cuda(), v.cuda(), cu.cuda()
        o = torch.full_like(vd, float("nan"))
        st = S0.reshape(-1, d, d).cuda()
        ws = torch.empty(nb, dtype=torch.uint8, device="cuda") if use_ws else None
        la.la_prefill(qd, kd, vd, o, st, cu_seqlens=cud, max_seqlen=int(lens.max()), chunk=chunk, workspace=ws)
        assert la.la_device_status() == la.LA_OK
        res.append((o, st))
    for o, st in res[1:]:
        assert torch.equal(res[0][0], o)
        assert torch.equal(res[0][1], st)
    assert nerr(res[0][0], O_ref) <= BF16_TOL
    assert nerr(res[0][1].reshape(S_ref.shape), S_ref) <= BF16_TOL


def test_prefill_then_decode_equals_longer_prefill():
    B, H, T, n, d = 2, 4, 150, 12, 128
    q, k, v = inputs.random_qkv(17, B, H, T + n, d, d, dtype=torch.bfloat16)
    o_long, S_long = gpu_prefill(q, k, v, chunk=64)
    _, S = gpu_prefill(q[:, :, :T], k[:, :, :T], v[:, :, :T], chunk=64)
    S = S.reshape(B, H, d, d)
    for t in range(T, T + n):
        od = torch.empty(B, H, d, dtype=torch.bfloat16, device="cuda")
        la.la_decode_step(q[:, :, t].cuda().contiguous(), k[:, :, t].cuda().contiguous(),
                          v[:, :, t].cuda().contiguous(), od, S)
        assert nerr(od, o_long[:, :, t].float().cpu().numpy()) <= BF16_TOL
    assert nerr(S, S_long.reshape(B, H, d, d).cpu().numpy()) <= BF16_TOL
    O_ref, S_ref = ora.recurrent(q, k, v)
    assert nerr(S, S_ref) <= BF16_TOL


# ------------------------------------------- the five workloads ----
#
# Every unit of every workload is compared with the oracle (streamed over
# batches of units), and decode runs every step on every unit, starting from
# the oracle's own prefill states: the errors below cover the whole path,
# prefill then decode.  Outputs start as NaN, so a unit or step the kernels
# skipped fails.

def _report(name, **errs):
    print(f"{name}: " + ", ".join(f"{k}={v:.3e}" if isinstance(v, float) else f"{k}={v}" for k, v in errs.items()))


def _assert_ok(errs, tol):
    for e in errs if isinstance(errs, list) else [errs]:
        assert e["nonfinite"] == 0, e
        for key, val in e.items():
            if key != "nonfinite":
                assert val <= tol, e


def test_workload_b4h8_t2048_d64_full():
    wl = WL["b4h8_t2048_d64"]
    q, k, v, _ = inputs.prefill_inputs(wl)
    assert la.la_prefill_path(wl.torch_dtype, wl.d, wl.d, wl.chunk) == "tc"
    o, S = gpu_prefill(q, k, v, chunk=wl.chunk)
    (e,), S_ref = prefill_vs_oracle(q, k, v, [(o, S)])
    units = inputs.decode_units(wl)
    dq, dk_, dv = decode_tokens(wl, wl.decode_steps, units)
    od = gpu_decode_run(S.reshape(units, wl.d, wl.d), dq, dk_, dv)
    ed = decode_vs_oracle(dq, dk_, dv, od, S, S_ref)
    _report(wl.name, prefill_O=e["O"], prefill_S=e["S"], decode_o=ed["o"], decode_S=ed["S"])
    _assert_ok([e, ed], BF16_TOL)


def test_workload_b8h16_t8192_d128_all_units():
    """All 128 units at C = 32, 64 and 128 (one oracle pass for the three),
    then the full 256 decode steps on all 128 states from C = 128 (the bench's
    default) and from C = 64 (the workload's listed chunk)."""
    wl = WL["b8h16_t8192_d128_knorm"]
    q, k, v, _ = inputs.prefill_inputs(wl)
    runs = {c: gpu_prefill(q, k, v, chunk=c) for c in (32, 64, 128)}
    errs, S_ref = prefill_vs_oracle(q, k, v, list(runs.values()))
    for c, e in zip(runs, errs):
        _report(f"{wl.name} C={c}", prefill_O=e["O"], prefill_S=e["S"])
    units = inputs.decode_units(wl)
    dq, dk_, dv = decode_tokens(wl, wl.decode_steps, units)
    dec = {}
    for c in (128, 64):
        S = runs[c][1].reshape(units, wl.d, wl.d)
        od = gpu_decode_run(S, dq, dk_, dv)
        dec[c] = decode_vs_oracle(dq, dk_, dv, od, S, S_ref)
        _report(f"{wl.name} decode after C={c}", decode_o=dec[c]["o"], decode_S=dec[c]["S"])
    _assert_ok(errs + list(dec.values()), BF16_TOL)


def test_workload_b1h32_t131072_d128_all_units():
    """All 32 units of the long sequences (the split into segments is taken:
    32 units on a GPU of more than 64 SMs)."""
    wl = WL["b1h32_t131072_d128"]
    q, k, v, _ = inputs.prefill_inputs(wl)
    o, S = gpu_prefill(q, k, v, chunk=wl.chunk)
    (e,), _ = prefill_vs_oracle(q, k, v, [(o, S)])
    _report(wl.name, prefill_O=e["O"], prefill_S=e["S"])
    _assert_ok(e, BF16_TOL)


def test_workload_varlen64_h32_d128_all_units():
    """All 2048 packed (sequence, head) units, then the 64 x 32 final states
    repeated 4 times -> 256 x 32 decode units, all 512 steps on all of them."""
    wl = WL["varlen64_h32_d128"]
    q, k, v, cu = inputs.prefill_inputs(wl)
    lens = (cu[1:] - cu[:-1]).numpy()
    o, S = gpu_prefill(q, k, v, cu=cu, chunk=wl.chunk, max_seqlen=int(lens.max()))
    (e,), S_ref = prefill_vs_oracle(q, k, v, [(o, S)], cu=cu.numpy())
    _report(wl.name, prefill_O=e["O"], prefill_S=e["S"])
    del o, q, k, v
    units = inputs.decode_units(wl)
    Sdec = S.reshape(-1, wl.d, wl.d).repeat(wl.decode_repeat, 1, 1).contiguous()
    S_ref_dec = np.tile(S_ref, (wl.decode_repeat, 1, 1))
    dq, dk_, dv = decode_tokens(wl, wl.decode_steps, units)
    od = gpu_decode_run(Sdec, dq, dk_, dv)
    ed = decode_vs_oracle(dq, dk_, dv, od, Sdec, S_ref_dec)
    _report(f"{wl.name} decode", decode_o=ed["o"], decode_S=ed["S"])
    _assert_ok([e, ed], BF16_TOL)
