"""The chunk form behind the per-key-decay tensor-core prefill, checked on the CPU in float64
against the oracle's sequential recurrence.

Operation: "com.microsoft.GatedDeltaNet" (Description) with `decay` in its per-key-dimension
spelling (Inputs table, shape (..., num_heads_v, head_size_qk)), read as D_t = diag(exp(g_t))
on the key axis of the state.  Over a chunk with incoming state S0 (Dk x Dv) and, per key
dimension, the cumulative log-decay G_i = g_1 + ... + g_i inside the chunk, the recurrence
unrolls to
    A_ij = beta_i sum_d k_i[d] k_j[d] e^{G_i[d] - G_j[d]}   (j < i),     T = (I + A)^-1
    U    = T diag(beta) V - T diag(beta) (K * e^G) S0
    P_ij = sum_d q_i[d] k_j[d] e^{G_i[d] - G_j[d]}          (j <= i)
    O    = scale ((Q * e^G) S0 + P U)
    S_C  = diag(e^{G_C}) S0 + (K * e^{G_C - G})^T U
(substitute S_i = Gamma_i S0 + sum_{j<=i} Gamma_i Gamma_j^-1 k_j u_j^T, Gamma_i = diag(e^{G_i}),
into u_i = beta_i (v_i - (D_i S_{i-1})^T k_i)).  The kernel splits each decay factor between the
two operands of A and P around a reference: for a row in 16-token block I, M_I = G at the
block's eighth token; the row operand is x_i e^{G_i - M_I} and the key operand of block I is
k_j e^{M_I - G_j} for every j up to the block's end, the four key operands stacked into one
160-row tile (block I from row 8 I (I + 1)).

The tests check, in float64 and without the kernel's bf16 roundings:
* the chunk form reproduces the oracle's outputs and final state, over full and ragged chunks;
* the split products equal the direct ones;
* once every log-decay is at least -9, every split factor is at most e^72 < 2^104, and the
  bound is reached when every decay sits at the floor.
"""
import numpy as np
import pytest

import oracle

C = 64      # tokens a chunk
BLK = 16    # tokens a block
G_FLOOR = -9.0


def _case(seed, L, Dk, Dv):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((L, Dk))
    k = rng.standard_normal((L, Dk))
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((L, Dv))
    # -softplus of N(0, 4), floored at -9 as the kernel floors it
    g = np.maximum(-np.logaddexp(0.0, rng.standard_normal((L, Dk)) * 2.0), G_FLOOR)
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal(L)))
    S0 = 0.05 * rng.standard_normal((Dk, Dv))
    return q, k, v, g, beta, S0


def _chunk_form(q, k, v, g, beta, S0, scale):
    """Outputs [L, Dv] and final state [Dk, Dv] of one head by the chunk form."""
    L, Dv = v.shape
    S = S0.copy()
    out = np.zeros((L, Dv))
    for c0 in range(0, L, C):
        sl = slice(c0, min(L, c0 + C))
        n = sl.stop - sl.start
        K, Q, V, b = k[sl], q[sl], v[sl], beta[sl]
        G = np.cumsum(g[sl], axis=0)
        Kg, Qg, Kinv = K * np.exp(G), Q * np.exp(G), K * np.exp(-G)
        A = np.tril(b[:, None] * (Kg @ Kinv.T), -1)
        P = np.tril(Qg @ Kinv.T)
        T = np.linalg.inv(np.eye(n) + A)
        U = T @ (b[:, None] * V) - T @ (b[:, None] * Kg) @ S
        out[sl] = scale * (Qg @ S + P @ U)
        S = np.exp(G[-1])[:, None] * S + (K * np.exp(G[-1] - G)).T @ U
    return out, S


def _oracle(q, k, v, g, beta, S0, scale):
    L = q.shape[0]
    o, st = oracle.prefill(q[:, None], k[:, None], v[:, None], g[:, None], beta[:, None],
                           np.array([0, L], np.int32), S0.T[None, None].copy(), B=1,
                           scale=scale, decay_per_key=True)
    return o[:, 0], st[0, 0].T


def _split(x, G, I):
    """Row operands x_i e^{G_i - M_I} (rows of block I) and the key operand of block I."""
    M = G[BLK * I + 7]
    rows = slice(BLK * I, BLK * (I + 1))
    return x[rows] * np.exp(G[rows] - M), np.exp(M - G[:BLK * (I + 1)])


@pytest.mark.parametrize("L,Dk,Dv", [(64, 32, 16), (150, 32, 16), (130, 128, 8)])
def test_chunk_form_matches_the_recurrence(L, Dk, Dv):
    q, k, v, g, beta, S0 = _case(L + Dk, L, Dk, Dv)
    scale = Dk ** -0.5
    o_c, s_c = _chunk_form(q, k, v, g, beta, S0, scale)
    o_r, s_r = _oracle(q, k, v, g, beta, S0, scale)
    assert np.abs(o_c - o_r).max() <= 1e-10 * max(1.0, np.abs(o_r).max())
    assert np.abs(s_c - s_r).max() <= 1e-10 * max(1.0, np.abs(s_r).max())


def test_a_dropped_decay_term_is_caught():
    # the check above is sharp: leaving the decay out of P (one plausible slip) fails it
    q, k, v, g, beta, S0 = _case(5, 70, 16, 8)
    scale = 0.25
    o_r, _ = _oracle(q, k, v, g, beta, S0, scale)
    L = len(q)
    S, out = S0.copy(), np.zeros_like(o_r)
    for c0 in range(0, L, C):
        sl = slice(c0, min(L, c0 + C))
        n = sl.stop - sl.start
        K, Q, V, b = k[sl], q[sl], v[sl], beta[sl]
        G = np.cumsum(g[sl], axis=0)
        Kg, Kinv = K * np.exp(G), K * np.exp(-G)
        T = np.linalg.inv(np.eye(n) + np.tril(b[:, None] * (Kg @ Kinv.T), -1))
        U = T @ (b[:, None] * V) - T @ (b[:, None] * Kg) @ S
        out[sl] = scale * ((Q * np.exp(G)) @ S + np.tril(Q @ K.T) @ U)
        S = np.exp(G[-1])[:, None] * S + (K * np.exp(G[-1] - G)).T @ U
    assert np.abs(out - o_r).max() > 1e-3


def test_split_products_equal_the_direct_ones():
    q, k, v, g, beta, S0 = _case(11, C, 64, 8)
    G = np.cumsum(g, axis=0)
    D = np.exp(G[:, None, :] - G[None, :, :])            # [i, j, d]: e^{G_i - G_j}
    KK = np.einsum("id,jd,ijd->ij", k, k, D)
    QK = np.einsum("id,jd,ijd->ij", q, k, D)
    offsets = [8 * I * (I + 1) for I in range(4)]
    assert offsets == [0, 16, 48, 96] and offsets[3] + BLK * 4 == 160   # the stacked key tile
    for I in range(4):
        rk, f = _split(k, G, I)
        rq, _ = _split(q, G, I)
        kb = k[:BLK * (I + 1)] * f                         # key operand of block I
        rows = slice(BLK * I, BLK * (I + 1))
        cols = slice(0, BLK * (I + 1))
        np.testing.assert_allclose(rk @ kb.T, KK[rows, cols], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(rq @ kb.T, QK[rows, cols], rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("at_floor", [False, True])
def test_split_factors_stay_below_2_to_104(at_floor):
    rng = np.random.default_rng(21)
    Dk = 128
    g = np.full((C, Dk), G_FLOOR) if at_floor else \
        np.maximum(-np.logaddexp(0.0, 3.0 * rng.standard_normal((C, Dk))), G_FLOOR)
    G = np.cumsum(g, axis=0)
    worst = 0.0
    for I in range(4):
        M = G[BLK * I + 7]
        row = G[BLK * I:BLK * (I + 1)] - M                  # exponent of the row operand
        key = M - G[:BLK * (I + 1)]                         # exponent of the key operand
        worst = max(worst, row.max(), key.max())
        # the product a kept entry (j <= i) needs is e^{G_i - G_j} <= 1
        for i in range(BLK * I, BLK * (I + 1)):
            assert (G[i] - G[:i + 1]).max() <= 1e-12
    assert worst <= 8 * -G_FLOOR + 1e-9                     # at most 8 tokens from the reference
    assert worst * np.log2(np.e) < 104
    if at_floor:
        assert worst == pytest.approx(72.0)                 # the bound is reached
