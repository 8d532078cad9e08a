"""Pins of the float64 oracle against what the slides and the mathematics fix.

Sources (slides "Chunking, causality, and parallel prefill"):
  * "Worked case -- full trace": 8 tokens, d = 2, C = 4, q_t = k_t, S_0 = 0,
    every output, S_4 and S_8 printed (tests/golden/worked_example.json);
  * "Transfer challenge" and its instructor answer: C = 2 hands off S_2, S_4,
    S_6 with the printed values, o_5..o_8 unchanged;
  * "Chunk size" visual support: transitions 8/C and triangle C^2;
  * the two bugs of the trace: dropping the incoming state gives o_5 = [0,1],
    a full (unmasked) chunk matrix gives o_5 = [4,5];
  * "Causal triangle": j <= i, diagonal included, future entries contribute 0.
Mathematics: the closed form O = tril(Q K^T) V + Q S_0 (brute force), the
d = 1 case as a cumulative sum, and invariants (chunk-size independence,
prefill then decode equals a longer prefill, continuation, varlen equals
separate runs).

Every plausible single mistake (dropped term, transposed operand, wrong
diagonal, read before update) is planted in a copy of the oracle below and
must fail at least one pin.
"""
import numpy as np
import pytest
import torch

from oracle import la_oracle as ora
from recurrent_decode_la_b200 import inputs


def _example(golden):
    k = np.array(golden["k"], dtype=np.float64)
    v = np.array(golden["v"], dtype=np.float64)
    q = k.copy()  # the trace states q_t = k_t
    S0 = np.array(golden["S0"], dtype=np.float64)
    return q, k, v, S0


def _as4(x):
    return x[None, None]


# ---------------------------------------------------------------- pins ----

def pin_worked_example(run, golden) -> bool:
    """run(q, k, v, S0) -> (O [8,2], S_8).  Exact equality (integers)."""
    q, k, v, S0 = _example(golden)
    O, S8 = run(q, k, v, S0)
    return (np.array_equal(np.asarray(O), np.array(golden["chunk4"]["o"], float))
            and np.array_equal(np.asarray(S8), np.array(golden["chunk4"]["S8"], float)))


def pin_random_vs_bruteforce(run, seed=7, T=37, dk=5, dv=3) -> bool:
    """Random q != k, random S_0: must equal the closed form to 1e-12."""
    q, k, v = (x[0, 0].double().numpy() for x in inputs.random_qkv(seed, 1, 1, T, dk, dv))
    S0 = np.random.default_rng(seed).standard_normal((dk, dv))
    O, S = run(q, k, v, S0)
    Ob, Sb = ora.bruteforce(q, k, v, S0)
    return (np.abs(np.asarray(O) - Ob).max() < 1e-12
            and np.abs(np.asarray(S) - Sb).max() < 1e-12)


def _run_recurrent_c(q, k, v, S0):
    O, S = ora.recurrent(_as4(q), _as4(k), _as4(v), _as4(S0))
    return O[0, 0], S[0, 0]


def _run_chunked(C, steps=None):
    def run(q, k, v, S0):
        O, S, _ = ora.chunked_unit(q, k, v, C, S0, steps=steps)
        return O, S
    return run


# ------------------------------------------------------- the definition ----

def test_worked_example_recurrent_exact(golden):
    assert pin_worked_example(_run_recurrent_c, golden)
    q, k, v, S0 = _example(golden)
    _, S4 = ora.recurrent(_as4(q[:4]), _as4(k[:4]), _as4(v[:4]), _as4(S0))
    assert np.array_equal(S4[0, 0], np.array(golden["chunk4"]["S4"], float))


def test_worked_example_python_twin_exact(golden):
    def run(q, k, v, S0):
        O, S = ora.recurrent_py(q, k, v, S0)
        return np.array(O), np.array(S)
    assert pin_worked_example(run, golden)


def test_worked_example_chunk4_trace(golden):
    q, k, v, S0 = _example(golden)
    O, S8, hand = ora.chunked_unit(q, k, v, 4, S0)
    g = golden["chunk4"]
    assert np.array_equal(O, np.array(g["o"], float))
    assert np.array_equal(hand[0], np.array(g["S4"], float))
    assert np.array_equal(S8, np.array(g["S8"], float))
    assert len(hand) == g["transitions"]
    # the masked score matrix of chunk 1 as printed
    M = ora.causal_mask(ora.intra_scores(q[:4], k[:4]))
    assert np.array_equal(M, np.array(g["masked_scores_chunk1"], float))
    # inter-chunk term of chunk 2 for t5, t6: q^T S_4 = [3,4], [5,5]
    inter = ora.inter_term(q[4:6], k[4:6], hand[0])
    assert np.array_equal(inter, np.array(g["inter_term_chunk2_first_two_rows"], float))


def test_transfer_challenge_chunk2(golden):
    q, k, v, S0 = _example(golden)
    O, S8, hand = ora.chunked_unit(q, k, v, 2, S0)
    g = golden["chunk2"]
    assert np.array_equal(hand[0], np.array(g["handoffs"]["S2"], float))
    assert np.array_equal(hand[1], np.array(g["handoffs"]["S4"], float))
    assert np.array_equal(hand[2], np.array(g["handoffs"]["S6"], float))
    assert np.array_equal(O[4:], np.array(g["o5_to_o8"], float))
    # three hand-offs between four chunks, each of fixed size d x d
    assert len(hand) - 1 == g["state_handoffs_between_chunks"]
    assert all(h.shape == (2, 2) for h in hand)


def test_chunk_size_table(golden):
    q, k, v, S0 = _example(golden)
    tab = golden["chunk_size_table"]
    ref, _ = _run_recurrent_c(q, k, v, S0)
    for C, trans, cells in zip(tab["C"], tab["transitions"], tab["triangle_cells"]):
        O, S, hand = ora.chunked_unit(q, k, v, C, S0)
        assert np.array_equal(O, ref), C
        assert len(hand) == trans
        assert ora.intra_scores(q[:C], k[:C]).size == cells


def test_bugs_of_the_trace_reproduce_printed_values(golden):
    q, k, v, S0 = _example(golden)
    bug1 = {"inter_term": lambda Qc, Kc, S: np.zeros((Qc.shape[0], S.shape[1]))}
    O1, _, _ = ora.chunked_unit(q, k, v, 4, S0, steps=bug1)
    assert np.array_equal(O1[4], np.array(golden["bug1_drop_incoming_state"]["o5"], float))
    bug2 = {"causal_mask": lambda A: A}
    O2, _, _ = ora.chunked_unit(q, k, v, 4, S0, steps=bug2)
    assert np.array_equal(O2[4], np.array(golden["bug2_full_mask_in_chunk"]["o5"], float))


# ------------------------------------------------ mutants must be caught ----

CHUNK_MUTANTS = {
    "drop_incoming_state": {"inter_term": lambda Qc, Kc, S: np.zeros((Qc.shape[0], S.shape[1]))},
    "full_matrix_no_mask": {"causal_mask": lambda A: A},
    "diagonal_excluded": {"causal_mask": lambda A: np.tril(A, -1)},
    "upper_triangle": {"causal_mask": lambda A: np.triu(A)},
    "inter_term_reads_K": {"inter_term": lambda Qc, Kc, S: Kc @ S},
    "carry_dropped": {"carry": lambda S, Kc, Vc: S},
    # S accumulates V^T K instead of K^T V (only shape-valid when d_k == d_v)
    "carry_transposed": {"carry": lambda S, Kc, Vc: S + Vc.T @ Kc
                         if S.shape[0] == S.shape[1] else S + 2.0 * (Kc.T @ Vc)},
    "scores_transposed": {"intra_scores": lambda Qc, Kc: Kc @ Qc.T},
    "carry_sign": {"carry": lambda S, Kc, Vc: S - Kc.T @ Vc},
}


@pytest.mark.parametrize("name", sorted(CHUNK_MUTANTS))
def test_chunk_mutant_fails_a_pin(name, golden):
    run = _run_chunked(4, CHUNK_MUTANTS[name])
    caught = (not pin_worked_example(run, golden)) or (not pin_random_vs_bruteforce(run)) \
        or (not pin_random_vs_bruteforce(_run_chunked(3, CHUNK_MUTANTS[name]), T=11, dk=4, dv=4))
    assert caught, name


def _rec_read_before_update(q, k, v, S0):
    S = np.array(S0, float).copy()
    O = []
    for t in range(len(q)):
        O.append(q[t] @ S)
        S = S + np.outer(k[t], v[t])
    return np.array(O), S


def _rec_transposed_update(q, k, v, S0):
    S = np.array(S0, float).copy()
    O = []
    for t in range(len(q)):
        S = S + np.outer(v[t], k[t]) if S.shape[0] == S.shape[1] else S + np.outer(k[t], v[t]) * 2
        O.append(q[t] @ S)
    return np.array(O), S


def _rec_transposed_read(q, k, v, S0):
    S = np.array(S0, float).copy()
    O = []
    for t in range(len(q)):
        S = S + np.outer(k[t], v[t])
        O.append(S @ q[t] if S.shape[0] == S.shape[1] else (q[t] @ S) * 2)
    return np.array(O), S


@pytest.mark.parametrize("mut", [_rec_read_before_update, _rec_transposed_update,
                                 _rec_transposed_read])
def test_recurrence_mutant_fails_a_pin(mut, golden):
    caught = (not pin_worked_example(mut, golden)) or \
        (not pin_random_vs_bruteforce(mut, T=9, dk=3, dv=3))
    assert caught, mut.__name__


def test_real_oracle_passes_all_pins(golden):
    assert pin_worked_example(_run_recurrent_c, golden)
    assert pin_random_vs_bruteforce(_run_recurrent_c)
    for C in (1, 2, 3, 4, 5, 16, 37, 64):
        assert pin_random_vs_bruteforce(_run_chunked(C)), C


# ------------------------------------------------------ Q.S versus K.S ----

def test_inter_term_is_q_dot_s_not_k_dot_s():
    """The mechanism map prints 'K.S_in'; the text reads q_t^T S.  With q != k
    only Q.S reproduces the recurrence the slides call exact."""
    q, k, v = (x[0, 0].double().numpy() for x in inputs.random_qkv(11, 1, 1, 24, 4, 4))
    ref, Sref = _run_recurrent_c(q, k, v, np.zeros((4, 4)))
    O, S, _ = ora.chunked_unit(q, k, v, 8)
    assert np.abs(O - ref).max() < 1e-12 and np.abs(S - Sref).max() < 1e-12
    Ok, _, _ = ora.chunked_unit(q, k, v, 8, steps={"inter_term": lambda Qc, Kc, S: Kc @ S})
    assert np.abs(Ok - ref).max() > 1e-3


# ------------------------------------------------------ closed forms ----

@pytest.mark.parametrize("T,dk,dv", [(1, 1, 1), (7, 3, 5), (64, 16, 16), (200, 8, 4), (256, 2, 9)])
def test_recurrent_equals_bruteforce(T, dk, dv):
    q, k, v = (x[0, 0].double().numpy() for x in inputs.random_qkv(T * 31 + dk, 1, 1, T, dk, dv))
    S0 = np.random.default_rng(T).standard_normal((dk, dv))
    O, S = _run_recurrent_c(q, k, v, S0)
    Ob, Sb = ora.bruteforce(q, k, v, S0)
    scale = max(1.0, np.abs(Ob).max())
    assert np.abs(O - Ob).max() / scale < 1e-12
    assert np.abs(S - Sb).max() / max(1.0, np.abs(Sb).max()) < 1e-12


def test_d1_is_a_cumulative_sum():
    rng = np.random.default_rng(3)
    T = 50
    q, k, v = rng.standard_normal((3, T, 1))
    s0 = rng.standard_normal()
    O, S = _run_recurrent_c(q, k, v, np.array([[s0]]))
    expect = q[:, 0] * (s0 + np.cumsum(k[:, 0] * v[:, 0]))
    assert np.abs(O[:, 0] - expect).max() < 1e-12
    assert abs(S[0, 0] - (s0 + np.sum(k[:, 0] * v[:, 0]))) < 1e-12


def test_one_hot_keys_make_state_rows_sums_of_values():
    """With keys e_i, row i of S is the sum of v over tokens whose key is e_i
    (how S_4 = [[3,4],[5,5]] is read off the trace)."""
    rng = np.random.default_rng(5)
    T, d = 30, 6
    idx = rng.integers(0, d, T)
    k = np.eye(d)[idx]
    v = rng.standard_normal((T, d))
    _, S = _run_recurrent_c(k, k, v, np.zeros((d, d)))
    for i in range(d):
        assert np.abs(S[i] - v[idx == i].sum(0)).max() < 1e-12


# -------------------------------------------------------- invariants ----

@pytest.mark.parametrize("T", [1, 5, 16, 33, 64])
def test_chunk_size_independence_ragged(T):
    q, k, v = (x[0, 0].double().numpy() for x in inputs.random_qkv(100 + T, 1, 1, T, 6, 5))
    S0 = np.random.default_rng(T).standard_normal((6, 5))
    ref, Sref = _run_recurrent_c(q, k, v, S0)
    for C in (1, 2, 3, 4, 7, 16, T, T + 3):
        O, S, hand = ora.chunked_unit(q, k, v, C, S0)
        assert np.abs(O - ref).max() < 1e-12, C
        assert np.abs(S - Sref).max() < 1e-12, C
        assert len(hand) == -(-T // C)


def test_prefill_then_decode_equals_longer_prefill():
    B, H, T, n, d = 2, 3, 20, 6, 8
    q, k, v = (x.double().numpy() for x in inputs.random_qkv(21, B, H, T + n, d, d))
    O_long, S_long = ora.recurrent(q, k, v)
    O, S = ora.recurrent(q[:, :, :T], k[:, :, :T], v[:, :, :T])
    for t in range(T, T + n):
        o, S = ora.decode_step(q[:, :, t], k[:, :, t], v[:, :, t], S)
        assert np.abs(o - O_long[:, :, t]).max() < 1e-12
    assert np.abs(S - S_long).max() < 1e-12


def test_decode_reads_state_plus_local_term():
    """o = q^T S_prev + (q . k) v, the instructor's reading of the 1x1 case."""
    rng = np.random.default_rng(9)
    q, k = rng.standard_normal((2, 4, 7))
    v = rng.standard_normal((4, 5))
    S = rng.standard_normal((4, 7, 5))
    o, S1 = ora.decode_step(q, k, v, S)
    expect = np.einsum("ui,uij->uj", q, S) + np.sum(q * k, -1)[:, None] * v
    assert np.abs(o - expect).max() < 1e-12
    assert np.abs(S1 - (S + k[:, :, None] * v[:, None, :])).max() < 1e-12


def test_continuation_prefill():
    q, k, v = (x.double().numpy() for x in inputs.random_qkv(33, 1, 2, 40, 4, 4))
    O, S = ora.recurrent(q, k, v)
    O1, S1 = ora.recurrent(q[:, :, :17], k[:, :, :17], v[:, :, :17])
    O2, S2 = ora.recurrent(q[:, :, 17:], k[:, :, 17:], v[:, :, 17:], S1)
    assert np.abs(np.concatenate([O1, O2], 2) - O).max() < 1e-12
    assert np.abs(S2 - S).max() < 1e-12


def test_varlen_equals_separate_runs():
    H, d = 3, 4
    lens = [5, 0, 12, 1, 9]
    cu = np.concatenate([[0], np.cumsum(lens)])
    q, k, v = (x.double().numpy() for x in inputs.random_qkv(44, 1, H, int(cu[-1]), d, d))
    S0 = np.random.default_rng(1).standard_normal((len(lens), H, d, d))
    O, S = ora.recurrent(q, k, v, S0, cu_seqlens=cu)
    for n, L in enumerate(lens):
        a, b = cu[n], cu[n + 1]
        On, Sn = ora.recurrent(q[:, :, a:b], k[:, :, a:b], v[:, :, a:b], S0[n][None])
        if L:
            assert np.abs(O[:, :, a:b] - On).max() < 1e-12
        assert np.abs(S[n] - Sn[0]).max() < 1e-12
    assert np.array_equal(S[1], S0[1])  # empty sequence: state untouched
    Oc, Sc = ora.chunked(q, k, v, 4, S0, cu_seqlens=cu)
    assert np.abs(Oc - O).max() < 1e-12 and np.abs(Sc - S).max() < 1e-12


def test_future_independence_and_diagonal():
    T, d = 16, 5
    q, k, v = (x[0, 0].double().numpy() for x in inputs.random_qkv(55, 1, 1, T, d, d))
    O, _ = _run_recurrent_c(q, k, v, np.zeros((d, d)))
    k2, v2 = k.copy(), v.copy()
    k2[9:] = 100.0
    v2[9:] = -50.0
    O2, _ = _run_recurrent_c(q, k2, v2, np.zeros((d, d)))
    assert np.array_equal(O[:9], O2[:9])
    assert np.abs(O[0] - (q[0] @ k[0]) * v[0]).max() < 1e-14


def test_empty_sequence_is_a_noop():
    S0 = np.random.default_rng(2).standard_normal((1, 1, 3, 3))
    z = np.zeros((1, 1, 0, 3))
    O, S = ora.recurrent(z, z, z, S0)
    assert O.shape == (1, 1, 0, 3) and np.array_equal(S, S0)


def test_bf16_inputs_upcast_exactly():
    x = torch.randn(4, 8).to(torch.bfloat16)
    assert np.array_equal(ora._f64(x), x.float().double().numpy())
