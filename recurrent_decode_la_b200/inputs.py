"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module holds no arithmetic of the method: it only draws random numbers
and lays them out.  Both the CUDA path and the float64 oracle receive the
arrays it returns (the oracle after an exact upcast to float64).

Recipe (same for every workload):
  * every (tensor, unit) block is drawn from its own numpy PCG64 stream keyed
    by ``SeedSequence([seed, tensor_id, unit])``, so any single unit can be
    regenerated on the host without drawing the others;
  * entries are N(0, 1) / sqrt(d) in float32, then cast to the workload dtype
    (bf16 rounds to nearest even);
  * where ``k_l2norm`` is set, every key row is divided by its L2 norm in
    float32 before the cast;
  * variable-length batches draw their lengths uniformly from
    [len_min, len_max] with their own generator;
  * decode tokens of step s are drawn per step, shaped [units, d].

Tensor ids: 0 = q, 1 = k, 2 = v, 3 = initial state, 10/11/12 = decode q/k/v.
"""
from __future__ import annotations

import concurrent.futures
import dataclasses
import functools
import math
import os
from typing import Optional

import numpy as np
import torch

_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: shapes, dtype, chunk size and seed."""
    name: str
    B: int
    H: int
    T: int
    d: int
    chunk: int
    dtype: str
    seed: int
    k_l2norm: bool = False
    decode_steps: int = 0
    # variable-length batch (B must be 1; T is then the packed total)
    num_seqs: int = 0
    len_min: int = 0
    len_max: int = 0
    # decode batch when it differs from the prefill units (repeat factor)
    decode_repeat: int = 1

    @property
    def torch_dtype(self) -> torch.dtype:
        return _DT[self.dtype]

    @property
    def varlen(self) -> bool:
        return self.num_seqs > 0


# The five workloads the method is measured and checked on, named by what they
# are.  The pages' own 8-token example lives in tests/golden/.
WORKLOADS = {
    "tiny_f32_b1h1_t64_d16": Workload(
        "tiny_f32_b1h1_t64_d16", B=1, H=1, T=64, d=16, chunk=16, dtype="f32",
        seed=1000, decode_steps=8),
    "b4h8_t2048_d64": Workload(
        "b4h8_t2048_d64", B=4, H=8, T=2048, d=64, chunk=64, dtype="bf16",
        seed=1001, decode_steps=256),
    "b8h16_t8192_d128_knorm": Workload(
        "b8h16_t8192_d128_knorm", B=8, H=16, T=8192, d=128, chunk=64,
        dtype="bf16", seed=1002, k_l2norm=True, decode_steps=256),
    "b1h32_t131072_d128": Workload(
        "b1h32_t131072_d128", B=1, H=32, T=131072, d=128, chunk=128,
        dtype="bf16", seed=1003),
    "varlen64_h32_d128": Workload(
        "varlen64_h32_d128", B=1, H=32, T=0, d=128, chunk=64, dtype="bf16",
        seed=1004, num_seqs=64, len_min=512, len_max=16384,
        decode_steps=512, decode_repeat=4),
}


def _gen(seed: int, tensor_id: int, index: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(
        np.random.SeedSequence([seed, tensor_id, index])))


def _randn(seed: int, tensor_id: int, index: int, *shape: int) -> torch.Tensor:
    g = _gen(seed, tensor_id, index)
    return torch.from_numpy(g.standard_normal(shape, dtype=np.float32))


def _block(seed: int, tensor_id: int, index: int, rows: int, d: int,
           l2norm: bool = False) -> torch.Tensor:
    x = _randn(seed, tensor_id, index, rows, d)
    if l2norm:
        x = x / x.norm(dim=-1, keepdim=True).clamp_min(1e-30)
    else:
        x = x / math.sqrt(d)
    return x


def varlen_lengths(wl: Workload) -> torch.Tensor:
    """Seeded sequence lengths, uniform on [len_min, len_max] (int64)."""
    g = _gen(wl.seed, 20, 0)
    return torch.from_numpy(g.integers(wl.len_min, wl.len_max + 1, wl.num_seqs,
                                       dtype=np.int64))


def cu_seqlens(wl: Workload) -> torch.Tensor:
    """Offsets (int32, num_seqs + 1 entries) of the packed sequences."""
    lens = varlen_lengths(wl)
    cu = torch.zeros(wl.num_seqs + 1, dtype=torch.int64)
    cu[1:] = torch.cumsum(lens, 0)
    return cu.to(torch.int32)


@functools.lru_cache(maxsize=16)
def _cu_cached(wl: Workload) -> torch.Tensor:
    return cu_seqlens(wl)


def total_tokens(wl: Workload) -> int:
    return int(cu_seqlens(wl)[-1]) if wl.varlen else wl.T


def n_units(wl: Workload) -> int:
    return (wl.num_seqs if wl.varlen else wl.B) * wl.H


def unit_rows(wl: Workload, unit: int) -> tuple[int, int, int]:
    """(group, first row, length) of ``unit`` in the [*, group, rows, d] layout.

    Dense: group = b*H + h, rows 0..T-1.  Varlen: unit n*H + h is head h of
    sequence n, rows cu[n]..cu[n+1]-1 of head h.
    """
    if not wl.varlen:
        return unit, 0, wl.T
    cu = _cu_cached(wl)
    n, h = divmod(unit, wl.H)
    return h, int(cu[n]), int(cu[n + 1] - cu[n])


def unit_qkv(wl: Workload, unit: int, dtype: Optional[torch.dtype] = None):
    """q, k, v rows of one unit (CPU, workload dtype), regenerated on their own."""
    dt = dtype or wl.torch_dtype
    _, _, L = unit_rows(wl, unit)
    q = _block(wl.seed, 0, unit, L, wl.d).to(dt)
    k = _block(wl.seed, 1, unit, L, wl.d, wl.k_l2norm).to(dt)
    v = _block(wl.seed, 2, unit, L, wl.d).to(dt)
    return q, k, v


def prefill_inputs(wl: Workload, dtype: Optional[torch.dtype] = None):
    """Full q, k, v on the CPU in the [B, H, T, d] layout ([1, H, T_total, d]
    for a variable-length batch), plus cu_seqlens (or None)."""
    dt = dtype or wl.torch_dtype
    d = wl.d
    if not wl.varlen:
        shape = (wl.B, wl.H, wl.T, d)
        cu = None
    else:
        cu = cu_seqlens(wl)
        shape = (1, wl.H, int(cu[-1]), d)
    q = torch.empty(shape, dtype=dt)
    k = torch.empty(shape, dtype=dt)
    v = torch.empty(shape, dtype=dt)
    qf, kf, vf = (x.view(-1, shape[2], d) for x in (q, k, v))

    def fill(u: int) -> None:
        g, r0, L = unit_rows(wl, u)
        qf[g, r0:r0 + L], kf[g, r0:r0 + L], vf[g, r0:r0 + L] = unit_qkv(wl, u, dt)

    # The generators release the GIL while drawing, so units fill in parallel;
    # every unit has its own stream, so the result does not depend on order.
    with concurrent.futures.ThreadPoolExecutor(max_workers=min(32, os.cpu_count() or 1)) as ex:
        list(ex.map(fill, range(n_units(wl))))
    return q, k, v, cu


def initial_state(wl: Workload, units: int, scale: float = 1.0) -> torch.Tensor:
    """A random non-zero initial state [units, d, d] float32 (tests of S_in)."""
    return (_randn(wl.seed, 3, 0, units, wl.d, wl.d) * scale).to(torch.float32)


def decode_units(wl: Workload) -> int:
    return n_units(wl) * wl.decode_repeat


def decode_token(wl: Workload, step: int, units: Optional[int] = None,
                 dtype: Optional[torch.dtype] = None):
    """q, k, v of decode step ``step``: each [units, d] (CPU, workload dtype)."""
    dt = dtype or wl.torch_dtype
    n = units if units is not None else decode_units(wl)
    q = _block(wl.seed, 10, step, n, wl.d).to(dt)
    k = _block(wl.seed, 11, step, n, wl.d, wl.k_l2norm).to(dt)
    v = _block(wl.seed, 12, step, n, wl.d).to(dt)
    return q, k, v


def random_qkv(seed: int, B: int, H: int, T: int, dk: int, dv: int,
               dtype: torch.dtype = torch.float32, distinct_qk: bool = True):
    """Small random q, k, v [B, H, T, d] for property tests (N(0,1)/sqrt(d))."""
    q = _randn(seed, 0, 0, B, H, T, dk) / math.sqrt(dk)
    k = _randn(seed, 1, 0, B, H, T, dk) / math.sqrt(dk)
    v = _randn(seed, 2, 0, B, H, T, dv) / math.sqrt(dv)
    if not distinct_qk:
        q = k.clone()
    return q.to(dtype), k.to(dtype), v.to(dtype)
