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
    o = torch.full_like(vd, float("nan"))  # a row the kernels skip stays NaN
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


def decode_steps_vs_oracle(dtype, B, H, dk, dv, steps, seed):
    """Run `steps` decode tokens from a random state through la_decode_step
    and the same tokens through the oracle; return the normalised errors of
    the outputs (all steps) and of the final state."""
    rng = np.random.default_rng(seed)
    S0 = (rng.standard_normal((B, H, dk, dv)) * 0.05).astype(np.float32)
    toks = [inputs.random_qkv(seed * 100 + i, B, H, 1, dk, dv, dtype=dtype) for i in range(steps)]
    st = torch.from_numpy(S0).cuda()
    outs = []
    for q, k, v in toks:
        o = torch.full((B, H, dv), float("nan"), dtype=dtype, device="cuda")
        la.la_decode_step(q[:, :, 0].contiguous().cuda(), k[:, :, 0].contiguous().cuda(),
                          v[:, :, 0].contiguous().cuda(), o, st)
        outs.append(o)
    assert la.la_device_status() == la.LA_OK
    S = S0.astype(np.float64)
    refs = []
    for q, k, v in toks:
        o_ref, S = ora.decode_step(q[:, :, 0].float().numpy(), k[:, :, 0].float().numpy(),
                                   v[:, :, 0].float().numpy(), S)
        refs.append(o_ref)
    return {"o": nerr(torch.stack(outs), np.stack(refs)), "S": nerr(st.reshape(S.shape), S)}


def run_in_child(check: str, env: dict, **kwargs) -> dict:
    """Run one check of tests/variant_worker.py in a fresh process whose
    environment adds `env`.  The library reads its tuning switches once per
    process, so a test of another kernel choice runs in a process of its
    own.  Returns the check's JSON result."""
    import json
    import os
    import subprocess
    import sys
    here = os.path.dirname(os.path.abspath(__file__))
    r = subprocess.run([sys.executable, os.path.join(here, "variant_worker.py"), check, json.dumps(kwargs)],
                       env=dict(os.environ, **env), capture_output=True, text=True, timeout=900,
                       cwd=os.path.dirname(here))
    if r.returncode != 0:
        raise AssertionError(f"{check} failed in the child process:\n{r.stdout}\n{r.stderr}")
    return json.loads(r.stdout.strip().splitlines()[-1])


# ---------------------------------------------------------------------------
# Full-coverage comparison with the oracle, streamed over batches of units so
# that float64 copies of the whole workload are never held at once.  The
# normalised error is global, as the tolerance is stated: the largest
# |gpu - oracle| over every element of every unit, divided by the largest
# |oracle| over the same elements.
# ---------------------------------------------------------------------------

class GlobalErr:
    """Running max |gpu - ref| and max |ref| over many blocks."""

    def __init__(self):
        self.diff = 0.0
        self.scale = 0.0
        self.nonfinite = 0

    def add(self, x, ref):
        x = np.asarray(x, np.float64)
        ref = np.asarray(ref, np.float64)
        bad = ~np.isfinite(x)
        self.nonfinite += int(bad.sum())
        if ref.size:
            self.scale = max(self.scale, float(np.abs(ref).max()))
            self.diff = max(self.diff, float(np.abs(np.where(bad, np.inf, x - ref)).max()))

    @property
    def value(self) -> float:
        return self.diff / self.scale if self.scale > 0 else self.diff


def unit_row_ranges(B, H, T, cu=None):
    """(group, first row, rows) of every unit: dense unit b*H + h is group
    b*H + h, rows 0..T-1; packed unit n*H + h is head h, rows cu[n]..cu[n+1]-1."""
    if cu is None:
        return [(u, 0, T) for u in range(B * H)]
    cu = np.asarray(cu, np.int64)
    return [(h, int(cu[n]), int(cu[n + 1] - cu[n])) for n in range(len(cu) - 1) for h in range(H)]


def _batches(ranges, rows_budget):
    batch, rows = [], 0
    for u, (_, _, L) in enumerate(ranges):
        batch.append(u)
        rows += L
        if rows >= rows_budget:
            yield batch
            batch, rows = [], 0
    if batch:
        yield batch


def _f64_rows(x, ranges, units):
    """Rows of the given units from x [groups, rows, d] (CPU or CUDA),
    concatenated, as a float64 numpy array."""
    parts = [x[g, r0:r0 + L] for g, r0, L in (ranges[u] for u in units)]
    cat = torch.cat(parts) if parts else x[0, :0]
    return cat.to("cpu").double().numpy()


def prefill_vs_oracle(q, k, v, results, S0=None, cu=None, rows_budget=1 << 21):
    """Compare every unit of one or more GPU prefills of the same inputs with
    the oracle.  q, k, v: the CPU inputs given to the GPU ([B,H,T,d], or
    [1,H,T_total,d] with cu).  results: list of (o, S) from the GPU (o shaped
    like v, S with units * d_k * d_v elements).  S0: initial states (None =
    zero).  Returns (per-result list of {"O": err, "S": err, "nonfinite": n},
    oracle final states [units, d_k, d_v] float64)."""
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    ranges = unit_row_ranges(B, H, T, cu)
    n_units = len(ranges)
    qf, kf, vf = (x.reshape(-1, T, x.shape[-1]) for x in (q, k, v))
    S0f = None if S0 is None else np.asarray(S0, np.float64).reshape(n_units, dk, dv)
    S_ref = np.zeros((n_units, dk, dv))
    errs = [(GlobalErr(), GlobalErr()) for _ in results]
    outs = [(o.reshape(-1, T, dv), S.reshape(n_units, dk, dv)) for o, S in results]
    for units in _batches(ranges, rows_budget):
        lens = np.array([ranges[u][2] for u in units], np.int64)
        starts = np.concatenate([[0], np.cumsum(lens)[:-1]]).astype(np.int64)
        s0 = np.zeros((len(units), dk, dv)) if S0f is None else S0f[units]
        Ob, Sb = ora.recurrent_units(_f64_rows(qf, ranges, units), _f64_rows(kf, ranges, units),
                                     _f64_rows(vf, ranges, units), s0, starts, lens)
        S_ref[units] = Sb
        for (eo, es), (o, S) in zip(errs, outs):
            eo.add(_f64_rows(o, ranges, units), Ob)
            es.add(S[units].double().cpu().numpy(), Sb)
    return [{"O": eo.value, "S": es.value, "nonfinite": eo.nonfinite + es.nonfinite} for eo, es in errs], S_ref


def decode_vs_oracle(dq, dk_, dv, od, S_gpu, S_start_ref, units_budget=1024):
    """Compare every step of every unit of a GPU decode run with the oracle.
    dq, dk_, dv: the CPU decode tokens [steps, units, d]; od: the GPU outputs
    [steps, units, d_v] (CUDA); S_gpu: the GPU states after the last step;
    S_start_ref: the oracle states [units, d_k, d_v] the run starts from (the
    oracle's own prefill states, so the whole path is checked).  The oracle
    runs each unit's token sequence through the recurrence, which is the
    decode step applied once per token.  Returns {"o": err, "S": err,
    "nonfinite": n}."""
    steps, n_units, dkk = dq.shape
    dvv = dv.shape[-1]
    eo, es = GlobalErr(), GlobalErr()
    Sg = S_gpu.reshape(n_units, dkk, dvv)
    for u0 in range(0, n_units, units_budget):
        u1 = min(n_units, u0 + units_budget)
        nb = u1 - u0

        def seq(x):  # [steps, nb, d] -> [nb * steps, d] float64, unit-major
            return x[:, u0:u1].transpose(0, 1).reshape(nb * steps, x.shape[-1]).double().numpy()

        starts = np.arange(nb, dtype=np.int64) * steps
        lens = np.full(nb, steps, dtype=np.int64)
        ob, Sb = ora.recurrent_units(seq(dq), seq(dk_), seq(dv), S_start_ref[u0:u1], starts, lens)
        eo.add(od[:, u0:u1].transpose(0, 1).reshape(nb * steps, dvv).double().cpu().numpy(), ob)
        es.add(Sg[u0:u1].double().cpu().numpy(), Sb)
    return {"o": eo.value, "S": es.value, "nonfinite": eo.nonfinite + es.nonfinite}


def gpu_decode_run(state, dq, dk_, dv):
    """Decode steps on the GPU through la_decode_step: state [units, d_k, d_v]
    (CUDA, updated in place); dq, dk_, dv CPU tokens [steps, units, d].
    Returns the outputs [steps, units, d_v] (CUDA; NaN until written)."""
    steps, units, _ = dq.shape
    qd, kd, vd = dq.cuda(), dk_.cuda(), dv.cuda()
    od = torch.full((steps, units, dv.shape[-1]), float("nan"), dtype=dv.dtype, device="cuda")
    for i in range(steps):
        la.la_decode_step(qd[i][:, None], kd[i][:, None], vd[i][:, None], od[i][:, None], state)
    assert la.la_device_status() == la.LA_OK
    return od


def decode_tokens(wl, steps, units):
    """The workload's decode tokens for `steps` steps, stacked [steps, units, d]
    (CPU, workload dtype); drawn in parallel, each step from its own stream."""
    import concurrent.futures
    import os
    with concurrent.futures.ThreadPoolExecutor(max_workers=min(32, os.cpu_count() or 1)) as ex:
        toks = list(ex.map(lambda s: inputs.decode_token(wl, s, units=units), range(steps)))
    return tuple(torch.stack([t[i] for t in toks]) for i in range(3))
