"""Float64 CPU oracle for causal linear attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  The product (the CUDA library and its
Python binding) never imports it and shares no code with it.

Everything here follows the slides "Chunking, causality, and parallel prefill"
(English edition; the French twin "Chunking, causalite et prefill parallele"
prints the same numbers):

* :func:`recurrent` -- the definition.  The literal token-by-token recurrence
  S_t = S_{t-1} + k_t v_t^T, o_t = q_t^T S_t (sections "Naive recurrence" and
  "Incoming and outgoing state"), run in plain C in float64
  (``la_oracle.c``).  GPU results are compared against this.
* :func:`decode_step` -- the same recurrence for one token (section "Prefill
  and decode": the triangle is 1x1, only the state read and the local term
  remain).
* :func:`chunked` -- the slides' chunkwise algorithm in the slides' order
  (section "Split into chunks" and "Worked case -- full trace"): per chunk,
  M = tril(Q K^T); O = M V + Q S_in; S_out = S_in + K^T V.  It exists to pin
  the method (chunk-size independence, the two bugs of the trace), not to be
  fast.
* :func:`bruteforce` -- the closed form over the whole sequence at once,
  O = tril(Q K^T) V + Q S_0 and S_T = S_0 + K^T V, for short sequences.
* :func:`recurrent_py` -- the recurrence in pure-Python loops, for tiny cases.

Readings of the slides taken here (each pinned by a test in
``tests/test_oracle_pins.py``):

* inter-chunk term is Q S_in (the mechanism-map diagram prints "K.S"; the
  text reads the state through q_t^T S, and only Q S reproduces the
  recurrence when q != k);
* the diagonal is inside the triangle (o_1 = v_1 in the trace);
* no feature map, no normaliser, no 1/sqrt(d) scale inside the method
  (o_3 = v_1 + v_3 in the trace);
* the state is d_k x d_v with rows indexed by the key dimension;
* masked entries contribute exactly zero (multiplicative mask);
* a last chunk shorter than C simply has fewer rows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "la_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liblaoracle.so")

_lib = None
_lock = threading.Lock()


def build(force: bool = False) -> str:
    """Compile ``la_oracle.c`` with gcc (float64, OpenMP, no fast-math)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared",
               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            path = build()
            lib = ctypes.CDLL(path)
            lib.la_oracle_recurrent.restype = ctypes.c_int
            lib.la_oracle_recurrent.argtypes = [
                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int]
            lib.la_oracle_max_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def max_threads() -> int:
    """Threads the C oracle's OpenMP loop uses (for the CPU-baseline report)."""
    return int(_load().la_oracle_max_threads())


def _f64(x) -> np.ndarray:
    """Exact upcast to a C-contiguous float64 array (bf16/fp32 -> f64 is exact)."""
    if hasattr(x, "detach"):  # a torch tensor on the CPU
        x = x.detach().to("cpu")
        import torch
        x = x.to(torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def recurrent_units(q, k, v, state, row_start, row_len):
    """Run the recurrence on independent units given by row ranges.

    q, k: [rows, d_k]; v: [rows, d_v]; state: [n_units, d_k, d_v] (S_0, not
    modified).  Unit u covers rows row_start[u] .. row_start[u]+row_len[u]-1.
    Returns (o [rows, d_v], S_T [n_units, d_k, d_v]); rows no unit covers are 0.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    S = _f64(state).copy()
    rows, dk = q.shape
    dv = v.shape[1]
    if k.shape != (rows, dk) or v.shape[0] != rows:
        raise ValueError("q/k/v row counts differ")
    n_units = S.shape[0]
    if S.shape != (n_units, dk, dv):
        raise ValueError("state shape must be [n_units, d_k, d_v]")
    rs = np.ascontiguousarray(np.asarray(row_start, dtype=np.int64))
    rl = np.ascontiguousarray(np.asarray(row_len, dtype=np.int64))
    if rs.shape != (n_units,) or rl.shape != (n_units,):
        raise ValueError("row_start/row_len must have one entry per unit")
    if n_units and (rs.min() < 0 or rl.min() < 0 or (rs + rl).max() > rows):
        raise ValueError("unit row range outside the arrays")
    o = np.zeros((rows, dv), dtype=np.float64)
    rc = _load().la_oracle_recurrent(
        q.ctypes.data, k.ctypes.data, v.ctypes.data, o.ctypes.data,
        S.ctypes.data, n_units, rs.ctypes.data, rl.ctypes.data, dk, dv)
    if rc != 0:
        raise ValueError("la_oracle_recurrent rejected its arguments")
    return o, S


def recurrent(q, k, v, S0=None, cu_seqlens=None):
    """The definition: token-by-token recurrence, float64.

    Dense: q, k [B, H, T, d_k]; v [B, H, T, d_v]; S0 [B, H, d_k, d_v] or None
    (zero state).  Varlen: B must be 1, ``cu_seqlens`` (N+1 offsets) splits the
    T axis into N sequences; S0 and the returned state are [N, H, d_k, d_v].
    Returns (O shaped like v, S_T).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens is None:
        n_units = B * H
        row_start = np.arange(n_units, dtype=np.int64) * T
        row_len = np.full(n_units, T, dtype=np.int64)
        st_shape = (B, H, dk, dv)
    else:
        if B != 1:
            raise ValueError("varlen input needs B == 1")
        cu = np.asarray(cu_seqlens, dtype=np.int64)
        N = cu.shape[0] - 1
        if cu[0] != 0 or cu[-1] != T or np.any(np.diff(cu) < 0):
            raise ValueError("cu_seqlens must rise from 0 to T")
        # unit (n, h) -> rows h*T + cu[n] ..; state index n*H + h
        n_idx, h_idx = np.meshgrid(np.arange(N), np.arange(H), indexing="ij")
        row_start = (h_idx * T + cu[:-1][n_idx]).reshape(-1)
        row_len = (cu[1:] - cu[:-1])[n_idx].reshape(-1)
        n_units = N * H
        st_shape = (N, H, dk, dv)
    if S0 is None:
        S0 = np.zeros(st_shape, dtype=np.float64)
    S0 = _f64(S0).reshape(n_units, dk, dv)
    o, S = recurrent_units(q.reshape(-1, dk), k.reshape(-1, dk),
                           v.reshape(-1, dv), S0, row_start, row_len)
    return o.reshape(v.shape), S.reshape(st_shape)


def decode_step(q, k, v, S):
    """One decode token per unit: S' = S + k v^T, o = q^T S'.

    q, k: [..., d_k]; v: [..., d_v]; S: [..., d_k, d_v].  Returns (o, S').
    """
    q, k, v, S = _f64(q), _f64(k), _f64(v), _f64(S)
    lead = q.shape[:-1]
    dk, dv = q.shape[-1], v.shape[-1]
    n = int(np.prod(lead)) if lead else 1
    o, S1 = recurrent_units(q.reshape(n, dk), k.reshape(n, dk),
                            v.reshape(n, dv), S.reshape(n, dk, dv),
                            np.arange(n, dtype=np.int64),
                            np.ones(n, dtype=np.int64))
    return o.reshape(lead + (dv,)), S1.reshape(lead + (dk, dv))


# --------------------------------------------------------------------------
# The chunkwise algorithm, step by step, in the slides' order.  Each step is
# its own function so that the tests can plant a mistake in exactly one step
# and check that the pins catch it.
# --------------------------------------------------------------------------

def intra_scores(Qc, Kc):
    """Q K^T of one chunk (C x C): every query of the chunk against every key."""
    return Qc @ Kc.T


def causal_mask(A):
    """Keep j <= i (diagonal included); entries above it contribute exactly 0
    (section "Causal triangle": above the diagonal is forbidden by
    construction, not a computed zero)."""
    return np.tril(A)


def inter_term(Qc, Kc, S_in):
    """The incoming-state read, q_t^T S_in for every row of the chunk
    (section "Incoming and outgoing state")."""
    return Qc @ S_in


def carry(S_in, Kc, Vc):
    """The one serial hop: S_out = S_in + K^T V (section "Split into chunks")."""
    return S_in + Kc.T @ Vc


def chunked_unit(Q, K, V, C, S0=None, steps=None):
    """Chunkwise prefill of one unit: Q, K [T, d_k], V [T, d_v], chunk size C.

    Returns (O [T, d_v], S_T, handoffs) where ``handoffs`` lists the state
    after every chunk (S_C, S_2C, ..., S_T): one entry per sequential
    transition.  ``steps`` may replace any of intra_scores / causal_mask /
    inter_term / carry (tests only: planting a mistake).
    """
    st = {"intra_scores": intra_scores, "causal_mask": causal_mask,
          "inter_term": inter_term, "carry": carry}
    if steps:
        st.update(steps)
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    T, dk = Q.shape
    dv = V.shape[1]
    if C < 1:
        raise ValueError("chunk size must be >= 1")
    S = np.zeros((dk, dv)) if S0 is None else _f64(S0).copy()
    O = np.zeros((T, dv))
    handoffs = []
    for c0 in range(0, T, C):
        c1 = min(c0 + C, T)
        Qc, Kc, Vc = Q[c0:c1], K[c0:c1], V[c0:c1]
        M = st["causal_mask"](st["intra_scores"](Qc, Kc))
        O[c0:c1] = M @ Vc + st["inter_term"](Qc, Kc, S)
        S = st["carry"](S, Kc, Vc)
        handoffs.append(S.copy())
    return O, S, handoffs


def chunked(q, k, v, C, S0=None, cu_seqlens=None):
    """Chunkwise prefill over [B, H, T, d] (or varlen, as in :func:`recurrent`)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    O = np.zeros(v.shape)
    if cu_seqlens is None:
        S_T = np.zeros((B, H, dk, dv)) if S0 is None else _f64(S0).copy()
        for b in range(B):
            for h in range(H):
                O[b, h], S_T[b, h], _ = chunked_unit(q[b, h], k[b, h], v[b, h],
                                                     C, S_T[b, h])
        return O, S_T
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    N = cu.shape[0] - 1
    S_T = np.zeros((N, H, dk, dv)) if S0 is None else _f64(S0).copy()
    for n in range(N):
        a, b_ = cu[n], cu[n + 1]
        for h in range(H):
            O[0, h, a:b_], S_T[n, h], _ = chunked_unit(
                q[0, h, a:b_], k[0, h, a:b_], v[0, h, a:b_], C, S_T[n, h])
    return O, S_T


def bruteforce(Q, K, V, S0=None):
    """Closed form over a whole unit: O = tril(Q K^T) V + Q S_0, S_T = S_0 + K^T V.

    Q, K [T, d_k], V [T, d_v].  Builds the full T x T triangle, so keep T small.
    """
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    dk, dv = Q.shape[1], V.shape[1]
    S0 = np.zeros((dk, dv)) if S0 is None else _f64(S0)
    O = np.tril(Q @ K.T) @ V + Q @ S0
    return O, S0 + K.T @ V


def recurrent_py(Q, K, V, S0=None):
    """Pure-Python loops over one unit (tiny cases only)."""
    T, dk = len(Q), len(Q[0]) if len(Q) else 0
    dv = len(V[0]) if len(V) else 0
    S = [[0.0] * dv for _ in range(dk)] if S0 is None else \
        [[float(S0[i][j]) for j in range(dv)] for i in range(dk)]
    O = []
    for t in range(T):
        for i in range(dk):
            for j in range(dv):
                S[i][j] += float(K[t][i]) * float(V[t][j])
        O.append([sum(float(Q[t][i]) * S[i][j] for i in range(dk))
                  for j in range(dv)])
    return O, S
