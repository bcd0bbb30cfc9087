"""The chunkwise form (oracle.chunked) against the token recurrence (kda_oracle.c).

The two are written independently; agreement to ~1e-12 pins the reconstructed chunk
algebra (cumulative decay, Q_decay / K_inv / K_restore, L, the UT transform, W, U,
the masked Q_decay K_inv^T) before any GPU code relies on it.
"""
import numpy as np
import pytest

import oracle
from oracle import chunked


def _inputs(T, H, dk, dv, seed, g_mean=3.0):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, H, dk))
    k = rng.standard_normal((T, H, dk))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, H, dv))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((T, H))))
    g = -np.log1p(np.exp(-(g_mean + rng.standard_normal((T, H, dk)))))
    f = lambda a: a.astype(np.float32)
    return f(q), f(k), f(v), f(g), f(beta)


@pytest.mark.parametrize("C", [1, 2, 4, 16, 64])
def test_chunked_equals_recurrence(C):
    H, dk, dv = 2, 16, 12
    for T in sorted({1, max(C - 1, 1), C, C + 1, 5 * C + 3}):
        q, k, v, g, beta = _inputs(T, H, dk, dv, 100 + C + T)
        s0 = 0.1 * np.random.default_rng(T).standard_normal((1, H, dk, dv))
        o_r, f_r = oracle.prefill(q, k, v, g, beta, [0, T], s0=s0)
        o_c, f_c = chunked.kda_prefill_chunked(q, k, v, g, beta, [0, T], C, s0=s0)
        assert oracle.rel_frobenius(o_c, o_r) < 1e-12, (C, T)
        assert oracle.rel_frobenius(f_c, f_r) < 1e-12, (C, T)


def test_chunked_varlen_nonzero_initial_state():
    H, dk, dv, C = 3, 8, 8, 16
    lens = [1, 16, 0, 33, 47]
    T = sum(lens)
    cu = np.cumsum([0] + lens)
    q, k, v, g, beta = _inputs(T, H, dk, dv, 7)
    s0 = 0.02 * np.random.default_rng(8).standard_normal((len(lens), H, dk, dv))
    o_r, f_r = oracle.prefill(q, k, v, g, beta, cu, s0=s0)
    o_c, f_c = chunked.kda_prefill_chunked(q, k, v, g, beta, cu, C, s0=s0)
    assert oracle.rel_frobenius(o_c, o_r) < 1e-12
    assert oracle.rel_frobenius(f_c, f_r) < 1e-12


def test_ut_transform_inverse_and_glossary_identities():
    """(I + L) INV = I; K_restore[t] = D_{j:t+1} k_t; (Q_decay K_inv^T)[j,t] =
    q_j^T D_{j:t+1} k_t for t <= j; the mask M_qk keeps the diagonal."""
    n, dk, dv = 64, 32, 8
    q, k, v, g, beta = (x[:, 0].astype(np.float64) for x in _inputs(n, 1, dk, dv, 42))
    T = chunked.chunk_tensors(q, k, v, g, beta)
    I = np.eye(n)
    np.testing.assert_allclose((I + T["L"]) @ T["INV"], I, atol=1e-13)
    np.testing.assert_allclose(T["INV"] @ (I + T["L"]), I, atol=1e-13)
    assert np.all(np.triu(T["INV"], 1) == 0)
    alpha = np.exp(g)  # [n, dk]
    for t in (0, 5, n - 1):
        D = np.prod(alpha[t + 1:], axis=0) if t + 1 < n else np.ones(dk)
        np.testing.assert_allclose(T["K_res"][t], D * k[t], rtol=1e-12)
    for j, t in ((0, 0), (10, 3), (63, 62), (40, 40)):
        D = np.prod(alpha[t + 1:j + 1], axis=0) if j > t else np.ones(dk)
        np.testing.assert_allclose(T["Aqk"][j, t], q[j] @ (D * k[t]), rtol=1e-11, atol=1e-14)
    assert T["Aqk"][3, 4] == 0 and T["Aqk"][4, 4] != 0
    np.testing.assert_allclose(T["gamma"], np.prod(alpha, axis=0), rtol=1e-12)


def test_forward_substitution_against_closed_form_2x2():
    """(I + L)^{-1} for L = [[0,0],[l,0]] is [[1,0],[-l,1]]."""
    L = np.array([[0.0, 0.0], [0.3, 0.0]])
    np.testing.assert_array_equal(chunked.forward_substitution_inverse(L),
                                  np.array([[1.0, 0.0], [-0.3, 1.0]]))


@pytest.mark.parametrize("seg", [1, 2, 3, 7])
def test_segmented_scan_equals_recurrence(seg):
    """The chunk-parallel scan (segment transitions composed, then every segment run from
    its starting state) equals the token recurrence, for varlen sequences with empty, short
    and long members and a nonzero initial state."""
    lens = [0, 1, 63, 64, 65, 700]
    T, H, dk, dv = sum(lens), 2, 8, 5
    q, k, v, g, beta = _inputs(T, H, dk, dv, 90 + seg)
    cu = np.concatenate([[0], np.cumsum(lens)])
    s0 = np.random.default_rng(91).standard_normal((len(lens), H, dk, dv))
    o_ref, f_ref = oracle.prefill(q, k, v, g, beta, cu, s0=s0)
    o, f = chunked.kda_prefill_segmented(q, k, v, g, beta, cu, 64, seg, s0=s0)
    assert oracle.rel_frobenius(o, o_ref) < 1e-12
    assert oracle.rel_frobenius(f, f_ref) < 1e-12


def test_chunk_affine_map_matches_chunk_step():
    """chunk_step is affine in S_in: S_out(S) = A S + b, with b the result from zero."""
    q, k, v, g, beta = _inputs(64, 1, 8, 5, 93)
    Tc = chunked.chunk_tensors(q[:, 0], k[:, 0], v[:, 0], g[:, 0], beta[:, 0])
    A, b = chunked.chunk_affine(Tc)
    S = np.random.default_rng(94).standard_normal((8, 5))
    _, S_out = chunked.chunk_step(S, Tc)
    _, b0 = chunked.chunk_step(np.zeros((8, 5)), Tc)
    np.testing.assert_allclose(b, b0, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(S_out, A @ S + b, rtol=1e-12, atol=1e-12)
