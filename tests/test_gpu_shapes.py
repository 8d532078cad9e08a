"""GPU parity on the less travelled shapes: every decode kernel (column split,
one CTA per unit, scalar), decode at thousands of units, and the fp32
CUDA-core prefill with d_k != d_v and odd sizes.  Each compares the CUDA path
with the float64 oracle on the same seeded inputs."""
import numpy as np
import pytest
import torch

import recurrent_decode_la_b200 as la
from gpu_util import BF16_TOL, F32_TOL, decode_steps_vs_oracle, gpu_prefill, nerr, run_in_child, tol_for
from oracle import la_oracle as ora
from recurrent_decode_la_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("dk,dv,env", [
    (128, 128, None),                                   # column split
    (64, 64, None),
    (128, 128, {"LINATTN_DECODE_COLBLOCKS": "0"}),      # one CTA per unit, vector loads
    (64, 32, {"LINATTN_DECODE_COLBLOCKS": "0"}),
    (5, 7, None),                                       # scalar kernel (d_v not a multiple of 4)
    (48, 80, None),
    (128, 6, None),
])
def test_decode_kernels(dtype, dk, dv, env):
    """Each decode kernel against the oracle; a kernel chosen through an
    environment switch runs in a child process (switches are read once per
    process)."""
    if env:
        errs = run_in_child("decode", env, dtype="bf16" if dtype == torch.bfloat16 else "f32",
                            dk=dk, dv=dv, steps=4, seed=dk * 7 + dv)
    else:
        errs = decode_steps_vs_oracle(dtype, 2, 3, dk, dv, 4, seed=dk * 7 + dv)
    tol = tol_for(dtype)
    assert errs["o"] <= tol and errs["S"] <= tol, errs


def test_decode_8192_units_sampled():
    """The packed workload's decode shape: 8192 units of d = 128 (one CTA per
    unit, no column split), two steps, sampled units against the oracle."""
    B, H, d = 256, 32, 128
    rng = np.random.default_rng(5)
    S0 = torch.from_numpy((rng.standard_normal((B, H, d, d)) * 0.05).astype(np.float32))
    st = S0.cuda()
    sample = [(0, 0), (17, 5), (128, 31), (255, 30)]
    toks = [inputs.random_qkv(900 + i, B, H, 1, d, d, dtype=torch.bfloat16) for i in range(2)]
    outs = []
    for q, k, v in toks:
        o = torch.empty(B, H, d, dtype=torch.bfloat16, device="cuda")
        la.la_decode_step(q[:, :, 0].contiguous().cuda(), k[:, :, 0].contiguous().cuda(),
                          v[:, :, 0].contiguous().cuda(), o, st)
        outs.append(o.cpu())
    assert la.la_device_status() == la.LA_OK
    for b, h in sample:
        S = S0[b, h].double().numpy()
        for i, (q, k, v) in enumerate(toks):
            o_ref, S = ora.decode_step(q[b, h, 0].float().numpy(), k[b, h, 0].float().numpy(),
                                       v[b, h, 0].float().numpy(), S)
            assert nerr(outs[i][b, h], o_ref) <= BF16_TOL, (b, h, i)
        assert nerr(st[b, h], S) <= BF16_TOL, (b, h)


@pytest.mark.parametrize("dk,dv", [(5, 7), (48, 80), (128, 128), (96, 32)])
@pytest.mark.parametrize("chunk", [16, 64])
@pytest.mark.parametrize("T", [1, 100])
def test_f32_prefill_cuda_cores(dk, dv, chunk, T):
    """fp32 inputs run the CUDA-core kernel (fp32 arithmetic throughout)."""
    assert la.la_prefill_path(torch.float32, dk, dv, chunk) == "simt"
    B, H = 2, 2
    q, k, v = inputs.random_qkv(dk + dv + T, B, H, T, dk, dv, dtype=torch.float32)
    S0 = torch.from_numpy(np.random.default_rng(T).standard_normal((B, H, dk, dv)).astype(np.float32)) * 0.05
    O_ref, S_ref = ora.recurrent(q, k, v, S0)
    o, S = gpu_prefill(q, k, v, S0=S0, chunk=chunk)
    assert nerr(o, O_ref) <= F32_TOL
    assert nerr(S.reshape(S_ref.shape), S_ref) <= F32_TOL


@pytest.mark.parametrize("dk,dv", [(32, 32), (96, 96), (64, 128)])
def test_bf16_prefill_outside_tensor_core_shapes(dk, dv):
    """bf16 shapes the tensor-core kernel does not take (d not in {64, 128},
    d_k != d_v) run the CUDA-core kernel with fp32 accumulation."""
    assert la.la_prefill_path(torch.bfloat16, dk, dv, 64) == "simt"
    B, H, T = 1, 3, 150
    q, k, v = inputs.random_qkv(dk * 3 + dv, B, H, T, dk, dv, dtype=torch.bfloat16)
    O_ref, S_ref = ora.recurrent(q, k, v)
    o, S = gpu_prefill(q, k, v, chunk=64)
    assert nerr(o, O_ref) <= BF16_TOL
    assert nerr(S.reshape(S_ref.shape), S_ref) <= BF16_TOL
