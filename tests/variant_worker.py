"""Checks that need a tuning switch of the library set in the environment.

The library reads its switches (LINATTN_SHORT, LINATTN_DECODE_COLBLOCKS, ...)
once per process, so a test of another kernel choice runs one of these
checks in a child process (``gpu_util.run_in_child``), which prints its
result as one JSON line.  Not collected by pytest (no test_ prefix).

    python tests/variant_worker.py <check> '<json kwargs>'
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))
sys.path.insert(0, HERE)

import torch  # noqa: E402

import recurrent_decode_la_b200 as la  # noqa: E402
from gpu_util import decode_steps_vs_oracle, gpu_prefill, nerr  # noqa: E402
from oracle import la_oracle as ora  # noqa: E402
from recurrent_decode_la_b200 import inputs  # noqa: E402

_DT = {"bf16": torch.bfloat16, "f32": torch.float32}


def check_decode(dtype, dk, dv, steps, seed):
    """Decode steps against the oracle with whatever decode kernel the
    environment selects."""
    return decode_steps_vs_oracle(_DT[dtype], 2, 3, dk, dv, steps, seed)


def check_prefill(dtype, B, H, T, d, seed):
    """One dense prefill from a random state against the oracle, with the
    kernel the environment selects; reports which kernel that was."""
    import numpy as np
    q, k, v = inputs.random_qkv(seed, B, H, T, d, d, dtype=_DT[dtype])
    S0 = torch.from_numpy((np.random.default_rng(seed).standard_normal((B, H, d, d)) * 0.05).astype(np.float32))
    O_ref, S_ref = ora.recurrent(q, k, v, S0)
    o, S = gpu_prefill(q, k, v, S0=S0)
    return {"kernel": la.la_prefill_kernel(_DT[dtype], T, d, d), "o": nerr(o, O_ref),
            "S": nerr(S.reshape(S_ref.shape), S_ref)}


CHECKS = {"decode": check_decode, "prefill": check_prefill}

if __name__ == "__main__":
    la.load_library()
    res = CHECKS[sys.argv[1]](**json.loads(sys.argv[2]))
    print(json.dumps(res), flush=True)
