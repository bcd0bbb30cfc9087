"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each case checks the oracle against something other than itself: a hand-worked
example, a closed form, a separately written textbook delta rule in the pages'
own orientation, exact-retrieval and overwrite properties, invariants, linearity.
A dropped term, a swapped decay/read order, a transposed operand or an output read
before the update fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from linear_attention_rule_b200 import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_inputs(T, H, dk, dv, seed, g_mean=3.0, unit_keys=True):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, H, dk))
    k = rng.standard_normal((T, H, dk))
    if unit_keys:
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, H, dv))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((T, H))))
    x = g_mean + rng.standard_normal((T, H, dk))
    g = -np.log1p(np.exp(-x))
    f = lambda a: a.astype(np.float32)
    return f(q), f(k), f(v), f(g), f(beta)


def test_hand_worked_2x2():
    """Exact rationals worked by hand (tests/golden/kda_hand_2x2.json)."""
    with open(os.path.join(GOLDEN, "kda_hand_2x2.json")) as fh:
        G = json.load(fh)
    alpha = np.array(G["alpha"])
    g = np.log(alpha)[:, None, :].astype(np.float32)
    k = np.array(G["k"], dtype=np.float32)[:, None, :]
    v = np.array(G["v"], dtype=np.float32)[:, None, :]
    q = np.array(G["q"], dtype=np.float32)[:, None, :]
    beta = np.array(G["beta"], dtype=np.float32)[:, None]
    out, sf = oracle.prefill(q, k, v, g, beta, G["cu_seqlens"])
    # k2 = (0.6, 0.8) and log(alpha) are rounded to fp32 on input; 1e-6 covers that.
    np.testing.assert_allclose(out[:, 0], np.array(G["expected_out"]), atol=1e-6)
    np.testing.assert_allclose(sf[0, 0], np.array(G["expected_final_state"]), atol=1e-6)


def test_beta_zero_is_pure_channel_decay():
    """beta = 0: the state only decays per key channel, S_t = Diag(exp(sum g)) S_0."""
    T, H, dk, dv = 37, 2, 8, 5
    q, k, v, g, beta = _rand_inputs(T, H, dk, dv, 1)
    beta[:] = 0
    s0 = np.random.default_rng(2).standard_normal((1, H, dk, dv))
    out, sf = oracle.prefill(q, k, v, g, beta, [0, T], s0=s0)
    a = np.cumsum(g.astype(np.float64), axis=0)  # [T, H, dk]
    for h in range(H):
        for t in range(T):
            S_t = np.exp(a[t, h])[:, None] * s0[0, h]
            np.testing.assert_allclose(out[t, h], S_t.T @ q[t, h].astype(np.float64),
                                       rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(sf[0, h], np.exp(a[-1, h])[:, None] * s0[0, h],
                                   rtol=1e-12, atol=1e-14)


def _textbook_delta_rule(q, k, v, beta):
    """The pages' DeltaNet update in the pages' own orientation: S is [dv, dk],
    retrieval is S k, S_t = S_{t-1} - beta_t (S_{t-1} k_t - v_t) k_t^T, o_t = S_t q_t."""
    T, dk = k.shape
    dv = v.shape[1]
    S = np.zeros((dv, dk))
    outs = []
    for t in range(T):
        S = S - beta[t] * np.outer(S @ k[t] - v[t], k[t])
        outs.append(S @ q[t])
    return np.array(outs), S


def test_alpha_one_is_the_delta_rule():
    """g = 0 (alpha = 1): KDA reduces to the plain delta rule (dk != dv catches transposes)."""
    T, H, dk, dv = 29, 3, 6, 4
    q, k, v, g, beta = _rand_inputs(T, H, dk, dv, 3)
    g[:] = 0
    out, sf = oracle.prefill(q, k, v, g, beta, [0, T])
    for h in range(H):
        o_ref, S_ref = _textbook_delta_rule(q[:, h].astype(np.float64), k[:, h].astype(np.float64),
                                            v[:, h].astype(np.float64), beta[:, h].astype(np.float64))
        np.testing.assert_allclose(out[:, h], o_ref, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(sf[0, h], S_ref.T, rtol=1e-11, atol=1e-12)


def test_orthonormal_keys_exact_retrieval():
    """beta = 1, alpha = 1, orthonormal keys, zero start: S^T k_i = v_i for every i, and
    o_t = sum_{i<=t} (k_i . q_t) v_i."""
    dk = dv = 16
    T = 12
    rng = np.random.default_rng(5)
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    keys = Qm[:T].astype(np.float32)           # rows orthonormal (fp32-rounded)
    k = keys[:, None, :]
    q = rng.standard_normal((T, 1, dk)).astype(np.float32)
    v = rng.standard_normal((T, 1, dv)).astype(np.float32)
    g = np.zeros((T, 1, dk), dtype=np.float32)
    beta = np.ones((T, 1), dtype=np.float32)
    out, sf = oracle.prefill(q, k, v, g, beta, [0, T])
    kk = keys.astype(np.float64)
    for i in range(T):
        np.testing.assert_allclose(sf[0, 0].T @ kk[i], v[i, 0], atol=1e-6)
    for t in range(T):
        ref = sum((kk[i] @ q[t, 0].astype(np.float64)) * v[i, 0].astype(np.float64)
                  for i in range(t + 1))
        np.testing.assert_allclose(out[t, 0], ref, atol=1e-6)


def test_same_key_overwrites_value():
    """Writing the same unit key again at beta = 1 replaces its value (the pages'
    example of correcting a stored fact)."""
    dk = dv = 8
    rng = np.random.default_rng(7)
    key = rng.standard_normal(dk)
    key /= np.linalg.norm(key)
    k = np.stack([key, key]).astype(np.float32)[:, None, :]
    v = rng.standard_normal((2, 1, dv)).astype(np.float32)
    q = k.copy()
    g = np.zeros((2, 1, dk), dtype=np.float32)
    beta = np.ones((2, 1), dtype=np.float32)
    out, sf = oracle.prefill(q, k, v, g, beta, [0, 2])
    kk = k[0, 0].astype(np.float64)
    # fp32 rounding of the key leaves |k|^2 = 1 +- 1e-7.
    np.testing.assert_allclose(sf[0, 0].T @ kk, v[1, 0], atol=1e-6)
    np.testing.assert_allclose(out[1, 0], v[1, 0], atol=1e-6)
    np.testing.assert_allclose(out[0, 0], v[0, 0], atol=1e-6)


def test_single_token_from_zero():
    """One token from a zero state: o = beta v (k . q)."""
    dk, dv, H = 7, 5, 3
    q, k, v, g, beta = _rand_inputs(1, H, dk, dv, 11)
    out, _ = oracle.prefill(q, k, v, g, beta, [0, 1])
    for h in range(H):
        ref = float(beta[0, h]) * v[0, h].astype(np.float64) * float(
            k[0, h].astype(np.float64) @ q[0, h].astype(np.float64))
        np.testing.assert_allclose(out[0, h], ref, rtol=1e-12, atol=1e-15)


def test_step_invariant_unit_keys():
    """With |k| = 1: S_t^T k_t = (1 - beta) S'^T k_t + beta v_t, where S' is the decayed
    previous state."""
    N, H, dk, dv = 3, 2, 16, 12
    rng = np.random.default_rng(13)
    state = rng.standard_normal((N, H, dk, dv))
    kk = rng.standard_normal((N, H, dk))
    kk /= np.linalg.norm(kk, axis=-1, keepdims=True)
    k = kk.astype(np.float32)
    q = rng.standard_normal((N, H, dk)).astype(np.float32)
    v = rng.standard_normal((N, H, dv)).astype(np.float32)
    g = (-np.abs(rng.standard_normal((N, H, dk))) * 0.3).astype(np.float32)
    beta = rng.uniform(0.1, 0.9, (N, H)).astype(np.float32)
    _, S1 = oracle.decode(q, k, v, g, beta, state)
    for n in range(N):
        for h in range(H):
            kd = k[n, h].astype(np.float64)
            nk2 = kd @ kd  # 1 up to the fp32 rounding of the key
            Sp = np.exp(g[n, h].astype(np.float64))[:, None] * state[n, h]
            b = float(beta[n, h])
            lhs = S1[n, h].T @ kd
            rhs = (1 - b * nk2) * (Sp.T @ kd) + b * nk2 * v[n, h]
            np.testing.assert_allclose(lhs, rhs, rtol=1e-10, atol=1e-12)
            assert abs(nk2 - 1) < 1e-6


def test_linear_in_values_and_initial_state():
    """For fixed q, k, g, beta the map (V, S_0) -> (O, S_T) is linear."""
    T, H, dk, dv = 21, 2, 8, 8
    q, k, v1, g, beta = _rand_inputs(T, H, dk, dv, 17)
    rng = np.random.default_rng(19)
    # values on a 1/64 grid keep a*v1 + b*v2 exactly representable in fp32
    v1 = (np.round(v1 * 64) / 64).astype(np.float32)
    v2 = (np.round(rng.standard_normal(v1.shape) * 64) / 64).astype(np.float32)
    s01 = rng.standard_normal((1, H, dk, dv))
    s02 = rng.standard_normal((1, H, dk, dv))
    a, b = 0.75, -1.5  # exact in fp32
    o1, f1 = oracle.prefill(q, k, v1, g, beta, [0, T], s0=s01)
    o2, f2 = oracle.prefill(q, k, v2, g, beta, [0, T], s0=s02)
    v12 = (a * v1.astype(np.float64) + b * v2.astype(np.float64)).astype(np.float32)
    assert np.array_equal(v12.astype(np.float64), a * v1.astype(np.float64) + b * v2.astype(np.float64))
    o12, f12 = oracle.prefill(q, k, v12, g, beta, [0, T], s0=a * s01 + b * s02)
    np.testing.assert_allclose(o12, a * o1 + b * o2, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(f12, a * f1 + b * f2, rtol=1e-10, atol=1e-12)


def test_varlen_equals_separate_sequences_and_continuation():
    """Packed sequences are independent; splitting a sequence and continuing from the
    final state reproduces the unsplit run (append-prefill)."""
    H, dk, dv = 2, 8, 6
    lens = [5, 0, 13, 1]
    T = sum(lens)
    q, k, v, g, beta = _rand_inputs(T, H, dk, dv, 23)
    cu = np.cumsum([0] + lens)
    out, sf = oracle.prefill(q, k, v, g, beta, cu)
    for n in range(len(lens)):
        a, b = cu[n], cu[n + 1]
        o_n, f_n = oracle.prefill(q[a:b], k[a:b], v[a:b], g[a:b], beta[a:b], [0, b - a])
        np.testing.assert_array_equal(out[a:b], o_n)
        np.testing.assert_array_equal(sf[n], f_n[0])
    # empty sequence keeps its (zero) initial state
    assert np.all(sf[1] == 0)
    # continuation: 13 tokens = 4 + 9
    a = cu[2]
    oA, fA = oracle.prefill(q[a:a + 4], k[a:a + 4], v[a:a + 4], g[a:a + 4], beta[a:a + 4], [0, 4])
    oB, fB = oracle.prefill(q[a + 4:a + 13], k[a + 4:a + 13], v[a + 4:a + 13], g[a + 4:a + 13],
                            beta[a + 4:a + 13], [0, 9], s0=fA)
    np.testing.assert_allclose(np.concatenate([oA, oB]), out[a:a + 13], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(fB, sf[2:3], rtol=1e-13, atol=1e-15)


def test_decode_chain_equals_prefill():
    """T decode steps from S_0 equal a T-token prefill from S_0."""
    T, H, dk, dv = 9, 2, 8, 8
    q, k, v, g, beta = _rand_inputs(T, H, dk, dv, 29)
    s0 = np.random.default_rng(31).standard_normal((1, H, dk, dv))
    out, sf = oracle.prefill(q, k, v, g, beta, [0, T], s0=s0)
    S = s0.copy()
    for t in range(T):
        o, S = oracle.decode(q[t:t + 1], k[t:t + 1], v[t:t + 1], g[t:t + 1], beta[t:t + 1], S)
        np.testing.assert_allclose(o[0], out[t], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(S, sf, rtol=1e-13, atol=1e-15)


def test_head_subset_matches_full_run():
    """Computing a subset of heads gives the same numbers as the full run."""
    lens = [40, 17]
    d = synthetic.make_prefill_inputs(lens, 4, 16, 16, torch.bfloat16, 3.0, 0.02, 123)
    out, sf = oracle.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"], s0=d["s0"])
    sub = synthetic.make_prefill_inputs(lens, 4, 16, 16, torch.bfloat16, 3.0, 0.02, 123, heads=[2, 3])
    for key in ("q", "k", "v", "g", "beta"):
        assert torch.equal(sub[key], d[key][:, 2:4])
    assert torch.equal(sub["s0"], d["s0"][:, 2:4])
    o2, f2 = oracle.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"],
                            s0=d["s0"][:, [1, 3]], heads=[1, 3])
    np.testing.assert_array_equal(o2, out[:, [1, 3]])
    np.testing.assert_array_equal(f2, sf[:, [1, 3]])


def test_metric_helpers():
    ref = np.ones((4, 3))
    assert oracle.rel_frobenius(ref * 1.01, ref) == pytest.approx(0.01)
    assert oracle.rel_frobenius(np.zeros(3) + 1e-3, np.zeros(3)) == pytest.approx(math.sqrt(3) * 1e-3)


def _slices_with_known_errors():
    """Outputs [T=5, H=2, dv=2] of three sequences (lengths 2, 0, 3) with reference 1
    everywhere and one perturbed element per (sequence, head) slice, so each slice's
    relative Frobenius error is delta / sqrt(2 len) (hand-computed below).  The worst
    slice is the last sequence's last head."""
    cu = [0, 2, 2, 5]
    ref = np.ones((5, 2, 2))
    out = ref.copy()
    out[0, 0, 0] += 0.02      # seq 0 head 0: 0.02 / sqrt(4) = 0.01
    out[1, 1, 1] += 0.04      # seq 0 head 1: 0.04 / 2 = 0.02
    out[3, 0, 0] += 0.06      # seq 2 head 0: 0.06 / sqrt(6) = 0.0244949
    out[4, 1, 0] -= 0.12      # seq 2 head 1: 0.12 / sqrt(6) = 0.0489898
    return cu, out, ref


def test_max_rel_frobenius_per_slice_takes_the_worst_slice():
    cu, out, ref = _slices_with_known_errors()
    worst = oracle.max_rel_frobenius_per_slice(out, ref, cu)
    assert worst == pytest.approx(0.12 / math.sqrt(6), rel=1e-12)
    # not the mean of the four slices, not the first sequence alone, not the global error
    assert worst > 1.5 * np.mean([0.01, 0.02, 0.06 / math.sqrt(6), 0.12 / math.sqrt(6)])
    assert worst > 0.02 + 1e-9
    assert abs(worst - oracle.rel_frobenius(out, ref)) > 1e-3
    # dropping the last sequence (an off-by-one on cu_seqlens) would miss the worst slice
    assert oracle.max_rel_frobenius_per_slice(out[:2], ref[:2], cu[:2]) == pytest.approx(0.02)
    # the empty sequence contributes nothing; its neighbours still count
    assert oracle.max_rel_frobenius_per_slice(out, ref, [0, 0, 2, 5]) == pytest.approx(worst)


def test_max_rel_frobenius_per_slice_absolute_branch():
    """A slice whose reference is zero is judged by its absolute error."""
    cu = [0, 1, 3]
    ref = np.ones((3, 2, 2))
    ref[1:, 1] = 0.0                 # seq 1, head 1: zero reference
    out = ref.copy()
    out[2, 1, 0] = 3e-3              # absolute error 3e-3 there
    out[0, 0, 0] += 1e-4             # seq 0 head 0: 1e-4 / sqrt(2)
    assert oracle.max_rel_frobenius_per_slice(out, ref, cu) == pytest.approx(3e-3, rel=1e-12)


def test_max_rel_frobenius_states_takes_the_worst_state():
    ref = np.ones((3, 2, 2, 2))      # [N, H, dk, dv]: every state has norm 2
    S = ref.copy()
    S[0, 0, 0, 0] += 0.01            # 0.005
    S[1, 1, 1, 0] += 0.02            # 0.01
    S[2, 1, 1, 1] -= 0.08            # 0.04: the last sequence's last head
    assert oracle.max_rel_frobenius_states(S, ref) == pytest.approx(0.04, rel=1e-12)
    assert oracle.max_rel_frobenius_states(S[:2], ref[:2]) == pytest.approx(0.01, rel=1e-12)
    Z = np.zeros((1, 1, 2, 2))
    assert oracle.max_rel_frobenius_states(Z + 2e-3, Z) == pytest.approx(4e-3, rel=1e-12)


def test_max_rel_frobenius_per_chunk_sees_one_bad_row():
    """One wrong row in a 600-token slice: the per-slice error stays small, the error of
    its own chunk (C = 64, the row's chunk 2 of 10, the last one 24 rows) does not."""
    T, C = 600, 64
    ref = np.ones((T, 1, 4))
    out = ref.copy()
    out[150, 0, :] = 0.0             # row 150 lies in chunk [128, 192)
    per_slice = oracle.max_rel_frobenius_per_slice(out, ref, [0, T])
    per_chunk = oracle.max_rel_frobenius_per_chunk(out, ref, [0, T], C)
    assert per_slice == pytest.approx(math.sqrt(4 / (4 * T)), rel=1e-12)     # 0.0408
    assert per_chunk == pytest.approx(math.sqrt(4 / (4 * C)), rel=1e-12)     # 0.125
    # chunks restart at each sequence start: the same row as the 23rd of a second
    # sequence starting at 128 falls in that sequence's first chunk [128, 192)
    assert oracle.max_rel_frobenius_per_chunk(out, ref, [0, 128, T], C) == pytest.approx(0.125)
    # the partial last chunk (rows 576..599) is compared on its own rows
    out2 = ref.copy()
    out2[590, 0, 0] = 1.48
    assert oracle.max_rel_frobenius_per_chunk(out2, ref, [0, T], C) == pytest.approx(
        0.48 / math.sqrt(4 * 24), rel=1e-12)


def test_prologue_definitions():
    """The prologue's three functions at values fixed by their definitions."""
    assert oracle.logsigmoid(np.array([0.0]))[0] == pytest.approx(-math.log(2), rel=1e-15)
    assert oracle.sigmoid(np.array([0.0]))[0] == 0.5
    # sigmoid(ln 3) = 3/4, logsigmoid(ln 3) = ln(3/4), sigmoid(-ln 3) = 1/4
    x = np.array([math.log(3.0), -math.log(3.0)])
    np.testing.assert_allclose(oracle.sigmoid(x), [0.75, 0.25], rtol=1e-15)
    np.testing.assert_allclose(oracle.logsigmoid(x), [math.log(0.75), math.log(0.25)], rtol=1e-15)
    # tails: logsigmoid(x) -> x as x -> -inf and -> -e^{-x} as x -> +inf; no overflow
    big = np.array([-1000.0, 1000.0, 40.0])
    ls = oracle.logsigmoid(big)
    assert ls[0] == -1000.0 and ls[1] == 0.0
    assert ls[2] == pytest.approx(-math.exp(-40.0), rel=1e-12)
    np.testing.assert_array_equal(oracle.sigmoid(big[:2]), [0.0, 1.0])
    # the log-decay is log(sigmoid) (a sign or a dropped log fails here)
    xs = np.linspace(-20, 20, 81)
    np.testing.assert_allclose(np.exp(oracle.logsigmoid(xs)), oracle.sigmoid(xs), rtol=1e-14)
    assert np.all(oracle.logsigmoid(xs) < 0)
    # L2 norm over the last axis with a 1e-12 clamp
    np.testing.assert_allclose(oracle.l2_normalize(np.array([3.0, 4.0])), [0.6, 0.8], rtol=1e-15)
    np.testing.assert_array_equal(oracle.l2_normalize(np.zeros((2, 3))), np.zeros((2, 3)))
    np.testing.assert_allclose(oracle.l2_normalize(np.array([1e-13, 0.0])), [0.1, 0.0], rtol=1e-12)
    m = oracle.l2_normalize(np.array([[[1.0, 0.0], [0.0, 2.0]]]))        # per row, not per tensor
    np.testing.assert_array_equal(m, [[[1.0, 0.0], [0.0, 1.0]]])


def test_prologue_applies_each_flag_alone():
    rng = np.random.default_rng(5)
    q, k = rng.standard_normal((3, 2, 4)), rng.standard_normal((3, 2, 4))
    g, b = rng.standard_normal((3, 2, 4)), rng.standard_normal((3, 2))
    q1, k1, g1, b1 = oracle.prologue(q, k, g, b, True, False, False)
    np.testing.assert_allclose(np.linalg.norm(q1, axis=-1), 1.0, rtol=1e-15)
    np.testing.assert_allclose(q1 * np.linalg.norm(q, axis=-1, keepdims=True), q, rtol=1e-14)
    np.testing.assert_array_equal(g1, g)
    np.testing.assert_array_equal(b1, b)
    _, k2, g2, b2 = oracle.prologue(q, k, g, b, False, True, True)
    np.testing.assert_array_equal(k2, k)
    np.testing.assert_allclose(g2, np.log(1.0 / (1.0 + np.exp(-g))), rtol=1e-14)
    np.testing.assert_allclose(b2, 1.0 / (1.0 + np.exp(-b)), rtol=1e-14)
