"""The seeded input generators shared by the tests, smoke() and bench.py.

The sampled parity tests regenerate single units of the large workloads on
the host and compare them with the CUDA path's output for the whole batch;
that only means something if a unit regenerated alone is exactly its slice of
the batch.  These tests check that, the determinism the expected values rely
on, the packed-batch offsets, and the value distributions the workloads name.
"""
import dataclasses
import math

import numpy as np
import torch

from recurrent_decode_la_b200 import inputs

WL = inputs.WORKLOADS


def _small_varlen():
    return dataclasses.replace(WL["varlen64_h32_d128"], name="varlen_small", H=3, d=16, num_seqs=7,
                               len_min=0, len_max=40)


def test_prefill_inputs_are_deterministic():
    wl = WL["tiny_f32_b1h1_t64_d16"]
    a = inputs.prefill_inputs(wl)
    b = inputs.prefill_inputs(wl)
    for x, y in zip(a[:3], b[:3]):
        assert torch.equal(x, y)


def test_unit_regenerated_alone_equals_its_slice_dense():
    wl = WL["b4h8_t2048_d64"]
    q, k, v, cu = inputs.prefill_inputs(wl)
    assert cu is None and q.shape == (4, 8, 2048, 64) and q.dtype == torch.bfloat16
    for u in (0, 13, 31):
        b, h = divmod(u, wl.H)
        uq, uk, uv = inputs.unit_qkv(wl, u)
        assert torch.equal(uq, q[b, h]) and torch.equal(uk, k[b, h]) and torch.equal(uv, v[b, h])


def test_unit_regenerated_alone_equals_its_slice_packed():
    wl = _small_varlen()
    q, k, v, cu = inputs.prefill_inputs(wl)
    lens = (cu[1:] - cu[:-1]).numpy()
    assert cu[0] == 0 and (lens >= 0).all() and (lens <= 40).all() and int(cu[-1]) == q.shape[2]
    for u in range(inputs.n_units(wl)):
        g, r0, L = inputs.unit_rows(wl, u)
        n, h = divmod(u, wl.H)
        assert (g, r0, L) == (h, int(cu[n]), int(lens[n]))
        uq, uk, uv = inputs.unit_qkv(wl, u)
        assert torch.equal(uq, q[0, g, r0:r0 + L]) and torch.equal(uk, k[0, g, r0:r0 + L])
        assert torch.equal(uv, v[0, g, r0:r0 + L])


def test_packed_lengths_of_the_packed_workload():
    wl = WL["varlen64_h32_d128"]
    lens = inputs.varlen_lengths(wl).numpy()
    cu = inputs.cu_seqlens(wl).numpy()
    assert len(lens) == 64 and lens.min() >= 512 and lens.max() <= 16384
    assert cu.dtype == np.int32 and (np.diff(cu) == lens).all() and cu[-1] == lens.sum()
    assert inputs.total_tokens(wl) == int(lens.sum())


def test_keys_are_l2_normalised_where_the_workload_says_so():
    wl = WL["b8h16_t8192_d128_knorm"]
    q, k, _ = inputs.unit_qkv(wl, 37, dtype=torch.float32)
    assert torch.allclose(k.norm(dim=-1), torch.ones(wl.T), atol=1e-5)
    assert abs(float(q.norm(dim=-1).mean()) - 1.0) < 0.05   # N(0, 1/d) rows: norm about 1


def test_values_are_standard_normal_over_sqrt_d():
    wl = WL["b1h32_t131072_d128"]
    q, _, v = inputs.unit_qkv(wl, 5, dtype=torch.float32)
    for x in (q, v):
        x = x.double() * math.sqrt(wl.d)
        assert abs(float(x.mean())) < 0.01
        assert abs(float(x.var()) - 1.0) < 0.01


def test_decode_tokens_are_prefix_consistent():
    """A decode step drawn for fewer units is the prefix of the full draw (the
    oracle samples the first units of large decode batches this way)."""
    wl = WL["b8h16_t8192_d128_knorm"]
    full = inputs.decode_token(wl, 3)
    part = inputs.decode_token(wl, 3, units=9)
    assert full[0].shape == (inputs.decode_units(wl), wl.d)
    for a, b in zip(part, full):
        assert torch.equal(a, b[:9])
    assert not torch.equal(inputs.decode_token(wl, 4)[0], full[0])


def test_distinct_streams_per_tensor_and_unit():
    wl = WL["b4h8_t2048_d64"]
    q0, k0, v0 = inputs.unit_qkv(wl, 0, dtype=torch.float32)
    q1, _, _ = inputs.unit_qkv(wl, 1, dtype=torch.float32)
    assert not torch.equal(q0, k0) and not torch.equal(q0, q1)
    # q and k of the same unit are uncorrelated
    c = float((q0 * k0).sum() / (q0.norm() * k0.norm()))
    assert abs(c) < 0.02
