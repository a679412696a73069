"""The algebra of the scalar-decay tensor-core prefill, checked on the CPU in float64 against the
oracle's sequential recurrence.

Operation: "com.microsoft.GatedDeltaNet" (Description), scalar decay exp(g_t) per token and
head, with the Attributes table's qk_l2_norm (epsilon 1e-12).  The kernel never scales the
q/k bytes the tensor cores read: with rk_i^2 = 1 / (k_i . k_i + eps), B = (K K^T) * e^{G_i - G_j}
the raw key products and D = diag(rk), the chunk's matrix A = diag(beta rk) B D (strictly lower)
satisfies (I + A)^-1 = D^-1 (I + A')^-1 D with A' = diag(beta rk^2) B, whose rows need only their
own norm.  Carrying U' = D U instead of U,
    T'  = (I + A')^-1,   Tb = T' diag(beta rk),   Tbg = T' diag(beta Gamma rk^2)
    U'  = Tb V - Tbg K S0
    S_C = Gamma_C S0 + (diag(e^{G_C - G}) K)^T U'
    O   = scale (diag(Gamma rq) Q S0 + P' U'),   P'_ij = rq_i (q_i . k_j) e^{G_i - G_j} (j <= i)
with Gamma = e^G and G the cumulative log-decay inside the chunk.  The tests check that this
reproduces the recurrence over full and ragged chunks, that U' is D times the U of the
normalised form, and that putting the key norms on the wrong side of A' (one plausible slip)
is caught.
"""
import numpy as np
import pytest

import oracle

C = 64
EPS = 1e-12


def _case(seed, L, Dk, Dv):
    rng = np.random.default_rng(seed)
    q = 2.0 * rng.standard_normal((L, Dk))
    k = 0.5 * rng.standard_normal((L, Dk))
    v = rng.standard_normal((L, Dv))
    g = -np.logaddexp(0.0, rng.standard_normal(L))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal(L)))
    S0 = 0.05 * rng.standard_normal((Dk, Dv))
    return q, k, v, g, beta, S0


def _row_local(q, k, v, g, beta, S0, scale, slip=False):
    """Outputs and final state by the row-local-norm chunk form, also U' and D U per chunk."""
    L, Dv = v.shape
    S = S0.copy()
    out = np.zeros((L, Dv))
    pairs = []
    for c0 in range(0, L, C):
        sl = slice(c0, min(L, c0 + C))
        n = sl.stop - sl.start
        K, Q, V, b = k[sl], q[sl], v[sl], beta[sl]
        G = np.cumsum(g[sl])
        Gam = np.exp(G)
        dec = np.exp(G[:, None] - G[None, :])
        rk2 = 1.0 / (np.sum(K * K, axis=1) + EPS)
        rk, rq = np.sqrt(rk2), 1.0 / np.sqrt(np.sum(Q * Q, axis=1) + EPS)
        Bm = np.tril((K @ K.T) * dec, -1)
        Ap = (b * rk2)[:, None] * Bm if not slip else Bm * (b * rk2)[None, :]
        Tp = np.linalg.inv(np.eye(n) + Ap)
        Tb = Tp * (b * rk)[None, :]
        Tbg = Tp * (b * Gam * rk2)[None, :]
        Up = Tb @ V - Tbg @ K @ S
        Pp = rq[:, None] * np.tril((Q @ K.T) * dec)
        out[sl] = scale * ((Gam * rq)[:, None] * (Q @ S) + Pp @ Up)
        # the normalised form's U, for the identity U' = D U
        Kh, bb = K * rk[:, None], b
        A = np.tril(bb[:, None] * (Kh @ Kh.T) * dec, -1)
        T = np.linalg.inv(np.eye(n) + A)
        U = T @ (bb[:, None] * V) - T @ (bb[:, None] * Gam[:, None] * Kh) @ S
        pairs.append((Up, rk[:, None] * U))
        S = Gam[-1] * S + (np.exp(G[-1] - G)[:, None] * K).T @ Up
    return out, S, pairs


def _oracle(q, k, v, g, beta, S0, scale):
    L = q.shape[0]
    o, st = oracle.prefill(q[:, None], k[:, None], v[:, None], g[:, None], beta[:, None],
                           np.array([0, L], np.int32), S0.T[None, None].copy(), B=1,
                           scale=scale, qk_l2norm=True)
    return o[:, 0], st[0, 0].T


@pytest.mark.parametrize("L,Dk,Dv", [(64, 32, 16), (150, 16, 8), (129, 64, 32)])
def test_row_local_norm_form_matches_the_recurrence(L, Dk, Dv):
    q, k, v, g, beta, S0 = _case(L * 3 + Dk, L, Dk, Dv)
    scale = Dk ** -0.5
    o_c, s_c, pairs = _row_local(q, k, v, g, beta, S0, scale)
    o_r, s_r = _oracle(q, k, v, g, beta, S0, scale)
    assert np.abs(o_c - o_r).max() <= 1e-10 * max(1.0, np.abs(o_r).max())
    assert np.abs(s_c - s_r).max() <= 1e-10 * max(1.0, np.abs(s_r).max())
    for Up, DU in pairs:
        np.testing.assert_allclose(Up, DU, rtol=1e-10, atol=1e-12)


def test_norms_on_the_wrong_side_are_caught():
    q, k, v, g, beta, S0 = _case(4, 100, 16, 8)
    o_c, _, _ = _row_local(q, k, v, g, beta, S0, 0.25, slip=True)
    o_r, _ = _oracle(q, k, v, g, beta, S0, 0.25)
    assert np.abs(o_c - o_r).max() > 1e-3
