"""The full-coverage comparison helpers of the GPU parity tests, checked on
the CPU: fed the oracle's own results they report (near) zero error; a
single wrong element anywhere, or a NaN (a row no kernel wrote), fails the
bound.  Dense and packed layouts, decode sequences, small row budgets so
that the streaming crosses batch boundaries."""
import numpy as np
import torch

import gpu_util as gu
from oracle import la_oracle as ora
from recurrent_decode_la_b200 import inputs


def test_prefill_compare_dense_catches_one_wrong_element_and_nan():
    q, k, v = inputs.random_qkv(3, 2, 3, 50, 8, 6, dtype=torch.bfloat16)
    S0 = np.random.default_rng(0).standard_normal((2, 3, 8, 6)) * 0.1
    O, S = ora.recurrent(q, k, v, S0)
    o_t, S_t = torch.from_numpy(O).float(), torch.from_numpy(S).float().reshape(6, 8, 6)
    (e,), S_ref = gu.prefill_vs_oracle(q, k, v, [(o_t, S_t)], S0=S0, rows_budget=64)
    assert e["O"] < 1e-6 and e["S"] < 1e-6 and e["nonfinite"] == 0
    assert np.array_equal(S_ref.reshape(S.shape), S)
    bad = o_t.clone()
    bad[1, 2, 49, 3] += 1.0                     # last row of the last unit
    errs, _ = gu.prefill_vs_oracle(q, k, v, [(o_t, S_t), (bad, S_t)], S0=S0, rows_budget=64)
    assert errs[0]["O"] < 1e-6 and errs[1]["O"] > gu.BF16_TOL
    nan = o_t.clone()
    nan[0, 1, 7, 0] = float("nan")
    (e,), _ = gu.prefill_vs_oracle(q, k, v, [(nan, S_t)], S0=S0)
    assert e["nonfinite"] == 1 and not e["O"] <= gu.BF16_TOL


def test_prefill_compare_packed_with_empty_sequence():
    cu = np.array([0, 10, 10, 33, 60])
    q, k, v = inputs.random_qkv(4, 1, 2, 60, 8, 8, dtype=torch.float32)
    O, S = ora.recurrent(q, k, v, cu_seqlens=cu)
    (e,), S_ref = gu.prefill_vs_oracle(q, k, v, [(torch.from_numpy(O), torch.from_numpy(S))], cu=cu,
                                       rows_budget=20)
    assert e == {"O": 0.0, "S": 0.0, "nonfinite": 0}
    assert np.array_equal(S_ref.reshape(S.shape), S)
    bad = torch.from_numpy(O).clone()
    bad[0, 1, 32, 5] -= 1.0                     # last row of sequence 2, head 1
    (e,), _ = gu.prefill_vs_oracle(q, k, v, [(bad, torch.from_numpy(S))], cu=cu, rows_budget=20)
    assert e["O"] > gu.F32_TOL


def test_decode_compare_matches_step_by_step_decode():
    steps, units, d = 7, 5, 8
    g = torch.Generator().manual_seed(1)
    dq, dk_, dv = (torch.randn(steps, units, d, generator=g) for _ in range(3))
    S0 = np.random.default_rng(1).standard_normal((units, d, d))
    Sg, outs = S0.copy(), []
    for t in range(steps):
        o, Sg = ora.decode_step(dq[t].numpy(), dk_[t].numpy(), dv[t].numpy(), Sg)
        outs.append(o)
    od = torch.from_numpy(np.stack(outs))
    assert gu.decode_vs_oracle(dq, dk_, dv, od, torch.from_numpy(Sg), S0, units_budget=2) == \
        {"o": 0.0, "S": 0.0, "nonfinite": 0}
    od[6, 4, 0] += 0.5                          # last step, last unit
    assert gu.decode_vs_oracle(dq, dk_, dv, od, torch.from_numpy(Sg), S0, units_budget=2)["o"] > gu.F32_TOL
