"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and
compare with the float64 oracle on the same seeded inputs."""
from __future__ import annotations

import numpy as np
import torch

import recurrent_decode_la_b200 as la
from oracle import la_oracle as ora
from recurrent_decode_la_b200 import inputs

BF16_TOL = 2e-2   # max |gpu - oracle| / max |oracle|, bf16 inputs, fp32 accumulation
F32_TOL = 1e-4    # same, fp32 inputs


def tol_for(dtype: torch.dtype) -> float:
    return BF16_TOL if dtype == torch.bfloat16 else F32_TOL


def nerr(x, ref) -> float:
    """Max-abs error normalised by max |ref| (0 when both are empty)."""
    x = np.asarray(x.detach().float().cpu().double().numpy() if hasattr(x, "detach") else x, np.float64)
    ref = np.asarray(ref, np.float64)
    if ref.size == 0:
        return 0.0
    scale = np.abs(ref).max()
    diff = np.abs(x - ref).max()
    return float(diff / scale) if scale > 0 else float(diff)


def gpu_prefill(q, k, v, S0=None, cu=None, chunk=0, max_seqlen=0, workspace=True):
    """Copy CPU tensors to the GPU, run la_prefill (with the workspace the
    library asks for, unless workspace=False), return (O, S_T) on the GPU."""
    dev = torch.device("cuda")
    qd, kd, vd = (x.to(dev).contiguous() for x in (q, k, v))
    o = torch.empty_like(vd)
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    units = (cu.numel() - 1) * H if cu is not None else B * H
    st = torch.empty(units, dk, dv, dtype=torch.float32, device=dev)
    la.la_state_init(st, None if S0 is None else S0.reshape(units, dk, dv).to(dev).float().contiguous())
    cud = cu.to(dev) if cu is not None else None
    ws = None
    if workspace:
        nbytes = la.la_prefill_workspace_size(q.dtype, B, H, T, dk, dv,
                                              0 if cu is None else cu.numel() - 1, chunk)
        if nbytes:
            ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    la.la_prefill(qd, kd, vd, o, st, cu_seqlens=cud, max_seqlen=max_seqlen, chunk=chunk, workspace=ws)
    assert la.la_device_status() == la.LA_OK
    return o, st


def oracle_units(wl, units, S0=None):
    """Oracle O and S_T of selected units of a workload (inputs regenerated)."""
    out = []
    for u in units:
        q, k, v = inputs.unit_qkv(wl, u)
        s0 = np.zeros((wl.d, wl.d)) if S0 is None else S0[u]
        O, S = ora.recurrent(q[None, None], k[None, None], v[None, None], np.asarray(s0)[None, None])
        out.append((O[0, 0], S[0, 0]))
    return out
