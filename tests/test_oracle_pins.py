"""Pins for the float64 oracle, against things other than the oracle itself.

* the worked examples printed on "Gated DeltaNet State Update" (tests/golden);
* a brute-force restatement of that page's gamma form,
  S_t = gamma_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T, written as
  literal Dk x Dk matrix products in numpy (the oracle uses the log-space
  rank-1 form of "com.microsoft.GatedDeltaNet", so a dropped term, a wrong
  sign, a transposed state or a wrong GQA index disagrees here);
* closed forms and invariants (beta = 0, unit keys, orthonormal keys);
* the cu_seqlens clamping and empty-request rules of the op's Inputs table;
* for decode, a brute-force DeltaProduct step with the fused gate restated in
  numpy from "flashinfer.cake_gdp.cake_gated_delta_product_mtp".
No test here needs a GPU.
"""
import json
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "p1_worked_examples.json")


# ---------------------------------------------------------------- brute force
def brute_prefill(q, k, v, g, beta, lengths, init, scale, l2norm, Hq, Hv):
    """gamma form with explicit (I - beta k k^T) products; K-major state."""
    N = q.shape[0]
    Dk, Dv = q.shape[2], v.shape[2]
    B = len(lengths)
    out = np.zeros((N, Hv, Dv))
    final = np.zeros((B, Hv, Dv, Dk))
    off = 0
    for b, L in enumerate(lengths):
        for h in range(Hv):
            qh = (h * Hq) // Hv
            S = np.zeros((Dk, Dv)) if init is None else init[b, h].T.copy()
            for t in range(off, off + L):
                kt = k[t, qh].astype(np.float64)
                qt = q[t, qh].astype(np.float64)
                if l2norm:
                    kt = kt / np.sqrt(kt @ kt + 1e-12)
                    qt = qt / np.sqrt(qt @ qt + 1e-12)
                gam = np.exp(g[t, h])
                bt = beta[t, h]
                S = gam * (np.eye(Dk) - bt * np.outer(kt, kt)) @ S + bt * np.outer(kt, v[t, h])
                out[t, h] = scale * (qt @ S)
            final[b, h] = S.T
        off += L
    return out, final


def np_softplus20(x):
    x = np.asarray(x, np.float64)
    return np.where(x > 20.0, x, np.log1p(np.exp(np.minimum(x, 20.0))))


def brute_decode_row(S0_vmajor, qs, ks, vs, a, bgate, A_log, dt_bias, scale, l2):
    """One (row, head): returns per-token outputs and per-token states (V-major)."""
    S = S0_vmajor.T.copy()  # K-major
    Dk = S.shape[0]
    outs, states = [], []
    for t in range(qs.shape[0]):
        alpha = np.exp(-np.exp(A_log) * np_softplus20(a[t] + dt_bias))
        S = alpha * S
        for j in range(ks.shape[1]):
            kj = ks[t, j].astype(np.float64)
            if l2:
                kj = kj / np.sqrt(kj @ kj + 1e-6)
            bj = 1.0 / (1.0 + np.exp(-bgate[t, j]))
            S = (np.eye(Dk) - bj * np.outer(kj, kj)) @ S + bj * np.outer(kj, vs[t, j])
        qt = qs[t].astype(np.float64)
        if l2:
            qt = qt / np.sqrt(qt @ qt + 1e-6)
        outs.append(scale * (qt @ S))
        states.append(S.T.copy())
    return np.array(outs), states


# ------------------------------------------------------------ golden examples
def test_worked_examples(oracle_mod):
    ex = json.load(open(GOLDEN))["examples"]
    assert len(ex) == 3
    for e in ex:
        q = np.array(e["q"], np.float64)
        k = np.array(e["k"], np.float64)
        v = np.array(e["v"], np.float64)
        gamma = np.array(e["gamma"], np.float64)
        beta = np.array(e["beta"], np.float64)
        B, S, Dk = q.shape
        Dv = v.shape[2]
        out, fs = oracle_mod.prefill(q.reshape(B * S, 1, Dk), k.reshape(B * S, 1, Dk),
                                     v.reshape(B * S, 1, Dv), np.log(gamma).reshape(B * S, 1),
                                     beta.reshape(B * S, 1), None, None, B=B, scale=1.0)
        np.testing.assert_allclose(out.reshape(B, S, Dv), np.array(e["outputs"]), atol=1e-12)
        # V-major [B, 1, Dv, Dk] -> the page's K-major (B, Dk, Dv)
        np.testing.assert_allclose(fs[:, 0].transpose(0, 2, 1), np.array(e["final_state"]),
                                   atol=1e-12)


# ---------------------------------------------------------------- brute force
@pytest.mark.parametrize("l2norm", [False, True])
@pytest.mark.parametrize("Hq,Hv", [(1, 1), (1, 2), (2, 4), (3, 6)])
def test_prefill_matches_gamma_form(oracle_mod, l2norm, Hq, Hv):
    rng = np.random.default_rng(100 + Hq * 10 + Hv + int(l2norm))
    lengths = [5, 1, 9, 4]
    N, Dk, Dv = sum(lengths), 6, 4
    q = rng.standard_normal((N, Hq, Dk))
    k = rng.standard_normal((N, Hq, Dk))
    if not l2norm:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((N, Hv, Dv))
    g = -rng.uniform(0.0, 1.5, (N, Hv))
    beta = rng.uniform(0.0, 1.0, (N, Hv))
    init = rng.standard_normal((len(lengths), Hv, Dv, Dk))
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    scale = 0.7
    out, fs = oracle_mod.prefill(q, k, v, g, beta, cu, init, scale=scale, qk_l2norm=l2norm)
    bo, bf = brute_prefill(q, k, v, g, beta, lengths, init, scale, l2norm, Hq, Hv)
    np.testing.assert_allclose(out, bo, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(fs, bf, rtol=1e-10, atol=1e-12)


def test_uniform_packing_equals_cu_seqlens(oracle_mod):
    rng = np.random.default_rng(7)
    B, S, H, D = 3, 6, 2, 4
    q, k = rng.standard_normal((2, B * S, H, D))
    v = rng.standard_normal((B * S, H, D))
    g = -rng.uniform(0, 1, (B * S, H))
    beta = rng.uniform(0, 1, (B * S, H))
    cu = np.arange(0, B * S + 1, S, dtype=np.int32)
    o1, f1 = oracle_mod.prefill(q, k, v, g, beta, None, None, B=B, qk_l2norm=True)
    bo, bf = brute_prefill(q, k, v, g, beta, [S] * B, None, 1.0, True, H, H)
    np.testing.assert_allclose(o1, bo, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(f1, bf, rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------------- invariants
def test_beta0_gamma1_keeps_state(oracle_mod):
    rng = np.random.default_rng(11)
    N, Dk, Dv = 7, 5, 3
    q, k = rng.standard_normal((2, N, 1, Dk))
    v = rng.standard_normal((N, 1, Dv))
    init = rng.standard_normal((1, 1, Dv, Dk))
    out, fs = oracle_mod.prefill(q, k, v, np.zeros((N, 1)), np.zeros((N, 1)), None, init,
                                 B=1, scale=0.5)
    np.testing.assert_allclose(fs, init, atol=0, rtol=0)
    np.testing.assert_allclose(out[:, 0], 0.5 * q[:, 0] @ init[0, 0].T, rtol=1e-13, atol=1e-13)


def test_beta0_closed_form_decay(oracle_mod):
    rng = np.random.default_rng(12)
    N, Dk, Dv = 9, 4, 4
    q, k = rng.standard_normal((2, N, 1, Dk))
    v = rng.standard_normal((N, 1, Dv))
    g = -rng.uniform(0, 0.5, (N, 1))
    init = rng.standard_normal((1, 1, Dv, Dk))
    out, fs = oracle_mod.prefill(q, k, v, g, np.zeros((N, 1)), None, init, B=1, scale=1.0)
    np.testing.assert_allclose(fs, np.exp(g.sum()) * init, rtol=1e-12)
    cum = np.cumsum(g[:, 0])
    np.testing.assert_allclose(out[:, 0], np.exp(cum)[:, None] * (q[:, 0] @ init[0, 0].T),
                               rtol=1e-12, atol=1e-14)


def test_unit_key_beta1_retrieves_value(oracle_mod):
    """beta = 1 with a unit key makes S_t^T k_t = v_t for any gamma; with q = k the output is v."""
    rng = np.random.default_rng(13)
    N, Dk, Dv = 12, 8, 5
    k = rng.standard_normal((N, 1, Dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((N, 1, Dv))
    g = -rng.uniform(0, 2, (N, 1))
    init = rng.standard_normal((1, 1, Dv, Dk))
    out, _ = oracle_mod.prefill(k, k, v, g, np.ones((N, 1)), None, init, B=1, scale=1.0)
    np.testing.assert_allclose(out, v, rtol=1e-11, atol=1e-12)


def test_orthonormal_keys_lookup(oracle_mod):
    Dk, Dv = 6, 3
    rng = np.random.default_rng(14)
    E = np.eye(Dk)
    v = rng.standard_normal((Dk, 1, Dv))
    k = E[:, None, :]
    out, fs = oracle_mod.prefill(k, k, v, np.zeros((Dk, 1)), np.ones((Dk, 1)), None, None,
                                 B=1, scale=1.0)
    np.testing.assert_allclose(out, v, atol=1e-15)
    np.testing.assert_allclose(fs[0, 0], v[:, 0, :].T, atol=1e-15)  # V-major: [Dv, Dk]


# ---------------------------------------------------------- cu_seqlens rules
def test_cu_seqlens_clamp_and_empty(oracle_mod):
    rng = np.random.default_rng(15)
    N, H, D = 10, 1, 3
    q, k = rng.standard_normal((2, N, H, D))
    v = rng.standard_normal((N, H, D))
    g = -rng.uniform(0, 1, (N, H))
    beta = rng.uniform(0, 1, (N, H))
    init = rng.standard_normal((4, H, D, D))
    sentinel = np.full((N, H, D), 123.0)
    # request 0: [0,4); request 1: decreasing -> empty; request 2: [2, 10) clamped from 99;
    # request 3: [-5 -> 0, 0) empty
    cu = np.array([0, 4, 2, 99, -5], np.int32)
    out, fs = oracle_mod.prefill(q, k, v, g, beta, cu, init, out=sentinel, qk_l2norm=True)
    o0, f0 = brute_prefill(q[:4], k[:4], v[:4], g[:4], beta[:4], [4], init[0:1], 1.0, True, 1, 1)
    o2, f2 = brute_prefill(q[2:], k[2:], v[2:], g[2:], beta[2:], [8], init[2:3], 1.0, True, 1, 1)
    np.testing.assert_allclose(fs[0], f0[0], rtol=1e-12)
    np.testing.assert_array_equal(fs[1], init[1])       # empty request copies its state
    np.testing.assert_allclose(fs[2], f2[0], rtol=1e-12)
    np.testing.assert_array_equal(fs[3], init[3])
    np.testing.assert_allclose(out[4:], o2[2:], rtol=1e-12)


def test_split_and_resume(oracle_mod):
    rng = np.random.default_rng(16)
    N, Hq, Hv, D = 20, 1, 2, 4
    q, k = rng.standard_normal((2, N, Hq, D))
    v = rng.standard_normal((N, Hv, D))
    g = -rng.uniform(0, 1, (N, Hv))
    beta = rng.uniform(0, 1, (N, Hv))
    init = rng.standard_normal((1, Hv, D, D))
    o, f = oracle_mod.prefill(q, k, v, g, beta, None, init, B=1, qk_l2norm=True)
    n = 7
    oa, fa = oracle_mod.prefill(q[:n], k[:n], v[:n], g[:n], beta[:n], None, init, B=1,
                                qk_l2norm=True)
    ob, fb = oracle_mod.prefill(q[n:], k[n:], v[n:], g[n:], beta[n:], None, fa, B=1,
                                qk_l2norm=True)
    np.testing.assert_allclose(np.concatenate([oa, ob]), o, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(fb, f, rtol=1e-12, atol=1e-14)


# -------------------------------------------------------------------- decode
def _decode_inputs(rng, B, T, nh, H, Dk, Dv, P):
    q = rng.standard_normal((B, T, H, Dk))
    k = rng.standard_normal((B, T, nh, H, Dk))
    v = rng.standard_normal((B, T, nh, H, Dv))
    pool = rng.standard_normal((P, H, Dv, Dk)) * 0.3
    A_log = rng.uniform(-2, 1, H)
    dt_bias = rng.standard_normal(H) * 0.5
    a = rng.standard_normal((B, T, H))
    b = rng.standard_normal((B, T, nh, H))
    return q, k, v, pool, A_log, dt_bias, a, b


@pytest.mark.parametrize("nh", [1, 2, 3])
def test_decode_matches_bruteforce(oracle_mod, nh):
    rng = np.random.default_rng(20 + nh)
    B, T, H, Dk, Dv, P = 4, 3, 2, 8, 4, 12
    q, k, v, pool, A_log, dt_bias, a, b = _decode_inputs(rng, B, T, nh, H, Dk, Dv, P)
    a[0, 1, 0] = 25.0  # softplus threshold branch
    read = np.array([3, -1, 7, 0], np.int32)
    write = np.array([5, 9, -1, 0], np.int32)
    sentinel = np.full((B, T, H, Dv), -7.0)
    out, newpool = oracle_mod.decode(q, k, v, pool, read, A_log, a, dt_bias, b, write_idx=write,
                                     scale=0.4, out=sentinel)
    expect_pool = pool.copy()
    for row in range(B):
        if read[row] < 0:
            np.testing.assert_array_equal(out[row], sentinel[row])  # padding row untouched
            continue
        for h in range(H):
            o, states = brute_decode_row(pool[read[row], h], q[row, :, h], k[row, :, :, h],
                                         v[row, :, :, h], a[row, :, h], b[row, :, :, h],
                                         A_log[h], dt_bias[h], 0.4, True)
            np.testing.assert_allclose(out[row, :, h], o, rtol=1e-10, atol=1e-12)
            if write[row] >= 0:
                expect_pool[write[row], h] = states[-1]
    np.testing.assert_allclose(newpool, expect_pool, rtol=1e-10, atol=1e-12)
    # slot 9 is written by padding row 1, which must skip everything
    np.testing.assert_array_equal(newpool[9], pool[9])


def test_decode_softplus_threshold_exact(oracle_mod):
    """x > 20 takes softplus(x) = x: alpha = exp(-exp(A_log) * x) exactly."""
    B, T, nh, H, Dk, Dv = 1, 1, 1, 1, 4, 2
    q = np.zeros((B, T, H, Dk)); q[..., 0] = 1
    k = np.zeros((B, T, nh, H, Dk)); k[..., 1] = 1
    v = np.zeros((B, T, nh, H, Dv))
    pool = np.zeros((1, H, Dv, Dk)); pool[0, 0, :, 0] = [1.0, 2.0]
    b = np.full((B, T, nh, H), -1e4)    # sigmoid -> 0: no write
    out, newpool = oracle_mod.decode(q, k, v, pool, np.array([0], np.int32), np.array([0.0]),
                                     np.full((B, T, H), 20.5), np.array([0.0]), b, scale=1.0,
                                     use_qk_l2norm=False)
    alpha = np.exp(-20.5)
    np.testing.assert_allclose(out[0, 0, 0], alpha * np.array([1.0, 2.0]), rtol=1e-14)


def test_decode_deltaproduct_reductions(oracle_mod):
    rng = np.random.default_rng(30)
    B, T, H, Dk, Dv, P = 2, 2, 2, 8, 4, 4
    q, k, v, pool, A_log, dt_bias, a, b = _decode_inputs(rng, B, T, 2, H, Dk, Dv, P)
    read = np.array([0, 1], np.int32)
    # nh=2 with beta_1 = sigmoid(-1e4) = 0 equals nh=1
    b2 = b.copy()
    b2[:, :, 1] = -1e4
    o2, p2 = oracle_mod.decode(q, k, v, pool, read, A_log, a, dt_bias, b2)
    o1, p1 = oracle_mod.decode(q, k[:, :, :1], v[:, :, :1], pool, read, A_log, a, dt_bias,
                               b[:, :, :1])
    np.testing.assert_allclose(o2, o1, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(p2, p1, rtol=1e-12, atol=1e-14)
    # nh=2 with k_1 = k_0, beta = 1: the second value overwrites; with q = k the readout is v_1
    # (unit keys supplied directly: the in-kernel norm's 1e-6 epsilon would leave |k| < 1)
    k3 = k / np.linalg.norm(k, axis=-1, keepdims=True)
    k3[:, :, 1] = k3[:, :, 0]
    q3 = k3[:, :, 0].copy()
    b3 = np.full_like(b, 1e4)
    o3, _ = oracle_mod.decode(q3, k3, v, pool, read, A_log, a, dt_bias, b3, scale=1.0,
                              use_qk_l2norm=False)
    np.testing.assert_allclose(o3, v[:, :, 1], rtol=1e-9, atol=1e-11)


def test_decode_scatter_and_disable(oracle_mod):
    rng = np.random.default_rng(31)
    B, T, nh, H, Dk, Dv, P = 2, 3, 2, 1, 8, 4, 10
    q, k, v, pool, A_log, dt_bias, a, b = _decode_inputs(rng, B, T, nh, H, Dk, Dv, P)
    read = np.array([0, 1], np.int32)
    write = np.array([2, 3], np.int32)
    sc = np.array([[4, -1, 5], [6, 7, 8]], np.int32)
    out, newpool = oracle_mod.decode(q, k, v, pool, read, A_log, a, dt_bias, b, write_idx=write,
                                     scatter_idx=sc)
    expect = pool.copy()
    for row in range(B):
        o, states = brute_decode_row(pool[read[row], 0], q[row, :, 0], k[row, :, :, 0],
                                     v[row, :, :, 0], a[row, :, 0], b[row, :, :, 0], A_log[0],
                                     dt_bias[0], 1 / np.sqrt(Dk), True)
        np.testing.assert_allclose(out[row, :, 0], o, rtol=1e-10, atol=1e-12)
        for t in range(T):
            if sc[row, t] >= 0:
                expect[sc[row, t], 0] = states[t]
    # scatter given: the end write-back to write_idx is skipped
    np.testing.assert_allclose(newpool, expect, rtol=1e-10, atol=1e-12)
    np.testing.assert_array_equal(newpool[2], pool[2])
    out_d, pool_d = oracle_mod.decode(q, k, v, pool, read, A_log, a, dt_bias, b, write_idx=write,
                                      disable_state_update=True)
    np.testing.assert_array_equal(pool_d, pool)
    np.testing.assert_allclose(out_d, out, rtol=1e-12)


def test_decode_equals_prefill_with_restated_gate(oracle_mod):
    """nh = 1 decode over T tokens equals prefill with g = log(alpha), beta = sigmoid(b)."""
    rng = np.random.default_rng(32)
    B, T, H, Dk, Dv = 1, 6, 2, 8, 5
    q, k, v, pool, A_log, dt_bias, a, b = _decode_inputs(rng, B, T, 1, H, Dk, Dv, 1)
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    od, pd = oracle_mod.decode(q, k, v, pool, np.array([0], np.int32), A_log, a, dt_bias, b,
                               use_qk_l2norm=False, scale=0.3)
    g = -np.exp(A_log)[None, :] * np_softplus20(a[0] + dt_bias[None, :])
    beta = 1.0 / (1.0 + np.exp(-b[0, :, 0]))
    op, fp = oracle_mod.prefill(q[0], k[0, :, 0], v[0, :, 0], g, beta, None, pool, B=1, scale=0.3)
    np.testing.assert_allclose(od[0], op, rtol=1e-10, atol=1e-13)
    np.testing.assert_allclose(pd, fp, rtol=1e-10, atol=1e-13)


# ------------------------------------------- update rules, gate and beta activations
# "com.microsoft.GatedDeltaNet", Attributes table: update_rule keeps or drops the decay and
# the delta retrieval; gate_activation qwen maps the decay input to
# -exp(a_log) * softplus(decay + dt_bias); beta_activation sigmoid.  Pinned here against
# closed forms of the rules without retrieval (causal sums of decayed outer products),
# the gamma-form brute force with gamma = 1, and special gate values.
def _rand_case(seed, N, Dk, Dv, unit_keys=True):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((N, 1, Dk))
    k = rng.standard_normal((N, 1, Dk))
    if unit_keys:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((N, 1, Dv))
    init = rng.standard_normal((1, 1, Dv, Dk))
    return rng, q, k, v, init


def _decayed_sum_closed_form(q, k, v, G, S0k, scale):
    """out_t = scale (exp(G_t) S0^T q_t + sum_{j<=t} exp(G_t - G_j) (k_j . q_t) v_j) and the
    final state exp(G_T) S0 + sum_j exp(G_T - G_j) k_j v_j^T (K-major), as masked products."""
    N = q.shape[0]
    Q, K, V = q[:, 0], k[:, 0], v[:, 0]
    D = np.exp(G[:, None] - G[None, :]) * np.tril(np.ones((N, N)))
    out = scale * (np.exp(G)[:, None] * (Q @ S0k) + (D * (Q @ K.T)) @ V)
    fin = np.exp(G[-1]) * S0k + (np.exp(G[-1] - G)[:, None] * K).T @ V
    return out, fin


def test_rule_linear_is_causal_linear_attention(oracle_mod):
    _, q, k, v, init = _rand_case(201, 11, 6, 4, unit_keys=False)
    out, fs = oracle_mod.prefill(q, k, v, None, None, None, init, B=1, scale=0.7,
                                 update_rule="linear")
    ro, rf = _decayed_sum_closed_form(q, k, v, np.zeros(11), init[0, 0].T, 0.7)
    np.testing.assert_allclose(out[:, 0], ro, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(fs[0, 0], rf.T, rtol=1e-11, atol=1e-12)


def test_rule_gated_is_decayed_linear_attention(oracle_mod):
    rng, q, k, v, init = _rand_case(202, 13, 5, 3, unit_keys=False)
    g = -rng.uniform(0.0, 1.0, (13, 1))
    out, fs = oracle_mod.prefill(q, k, v, g, None, None, init, B=1, scale=1.3,
                                 update_rule="gated")
    ro, rf = _decayed_sum_closed_form(q, k, v, np.cumsum(g[:, 0]), init[0, 0].T, 1.3)
    np.testing.assert_allclose(out[:, 0], ro, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(fs[0, 0], rf.T, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("l2norm", [False, True])
def test_rule_delta_is_gamma_form_with_gamma_one(oracle_mod, l2norm):
    rng, q, k, v, init = _rand_case(203 + int(l2norm), 9, 6, 4, unit_keys=not l2norm)
    beta = rng.uniform(0.0, 1.0, (9, 1))
    out, fs = oracle_mod.prefill(q, k, v, None, beta, None, init, B=1, scale=0.5,
                                 qk_l2norm=l2norm, update_rule="delta")
    ro, rf = brute_prefill(q, k, v, np.zeros((9, 1)), beta, [9], init, 0.5, l2norm, 1, 1)
    np.testing.assert_allclose(out, ro, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(fs, rf, rtol=1e-11, atol=1e-12)


def test_qwen_gate_reproduces_worked_example_two(oracle_mod):
    """a_log = 0, dt_bias = 0, decay = 0 gives g = -softplus(0) = -ln 2, i.e. gamma = 0.5 on
    every token: the page's second worked example (4 stored, then halved to 2) with the first
    token's gate replaced by the same 0.5 and beta_1 = 0."""
    e = json.load(open(GOLDEN))["examples"][1]
    q = np.array(e["q"], np.float64).reshape(2, 1, 2)
    k = np.array(e["k"], np.float64).reshape(2, 1, 2)
    v = np.array(e["v"], np.float64).reshape(2, 1, 2)
    beta = np.array(e["beta"], np.float64).reshape(2, 1)
    out, fs = oracle_mod.prefill(q, k, v, np.zeros((2, 1)), beta, None, None, B=1, scale=1.0,
                                 gate_activation="qwen", a_log=np.zeros(1), dt_bias=np.zeros(1))
    # token 0: S = 0.5*0 + k(1*(4 - 0)) -> 4; token 1: S = 0.5*4, beta = 0 -> 2
    np.testing.assert_allclose(out[:, 0], np.array(e["outputs"])[0], atol=1e-12)
    np.testing.assert_allclose(fs[0, 0].T, np.array(e["final_state"])[0], atol=1e-12)


def test_qwen_gate_closed_form_decay(oracle_mod):
    """beta = 0 leaves only the decay: exp(a_log) = 2 with decay + dt_bias = 0 gives
    gamma = 2^-2 per token; decay + dt_bias = 30 lies above the softplus threshold, so with
    exp(a_log) = ln(2)/30 the gate is again exactly 0.5."""
    rng, q, k, v, init = _rand_case(205, 6, 4, 3)
    for a_log, dec, dtb, gam in [(np.log(2.0), -0.75, 0.75, 0.25), (np.log(np.log(2.0) / 30.0),
                                                                    29.0, 1.0, 0.5)]:
        out, fs = oracle_mod.prefill(q, k, v, np.full((6, 1), dec), np.zeros((6, 1)), None, init,
                                     B=1, scale=1.0, gate_activation="qwen",
                                     a_log=np.array([a_log]), dt_bias=np.array([dtb]))
        decay = gam ** np.arange(1, 7)
        np.testing.assert_allclose(out[:, 0], decay[:, None] * (q[:, 0] @ init[0, 0].T),
                                   rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(fs[0, 0], gam ** 6 * init[0, 0], rtol=1e-12, atol=1e-14)


def test_beta_sigmoid_special_values(oracle_mod):
    """sigmoid(0) = 1/2 exactly (gamma-form brute force with beta = 0.5); a large positive
    input saturates to 1 (unit key, q = k: the output is the value, the overwrite rule of the
    first worked example); a large negative one to 0 (only the decay remains)."""
    rng, q, k, v, init = _rand_case(206, 8, 5, 3)
    g = -rng.uniform(0.0, 1.0, (8, 1))
    out, fs = oracle_mod.prefill(q, k, v, g, np.zeros((8, 1)), None, init, B=1, scale=1.0,
                                 beta_activation="sigmoid")
    ro, rf = brute_prefill(q, k, v, g, np.full((8, 1), 0.5), [8], init, 1.0, False, 1, 1)
    np.testing.assert_allclose(out, ro, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(fs, rf, rtol=1e-11, atol=1e-12)
    out, _ = oracle_mod.prefill(k, k, v, g, np.full((8, 1), 60.0), None, init, B=1, scale=1.0,
                                beta_activation="sigmoid")
    np.testing.assert_allclose(out, v, rtol=1e-11, atol=1e-12)
    out, fs = oracle_mod.prefill(q, k, v, g, np.full((8, 1), -60.0), None, init, B=1, scale=1.0,
                                 beta_activation="sigmoid")
    cum = np.cumsum(g[:, 0])
    np.testing.assert_allclose(out[:, 0], np.exp(cum)[:, None] * (q[:, 0] @ init[0, 0].T),
                               rtol=1e-11, atol=1e-13)


def test_rule_inputs_are_checked(oracle_mod):
    _, q, k, v, _ = _rand_case(207, 3, 2, 2)
    z = np.zeros((3, 1))
    with pytest.raises(AssertionError):
        oracle_mod.prefill(q, k, v, z, z, None, None, B=1, update_rule="linear")
    with pytest.raises(AssertionError):
        oracle_mod.prefill(q, k, v, None, z, None, None, B=1, update_rule="gated_delta")


# ---------------------------------------------------------------- per-key-dimension decay
# "com.microsoft.GatedDeltaNet", Inputs table (`decay`, the per-key-dimension spelling
# (..., num_heads_v, head_size_qk)): the scalar exp(g_t) of the Description's recurrence is
# read as D_t = diag(exp(g_t)) on the key axis of the K-major state, in both places,
#   S_t = D_t S_{t-1} + k_t (beta_t (v_t - (D_t S_{t-1})^T k_t))^T,
# i.e. the gamma form S_t = (I - beta_t k_t k_t^T) D_t S_{t-1} + beta_t k_t v_t^T.
def brute_prefill_per_key(q, k, v, g, beta, lengths, init, scale, l2norm, Hq, Hv,
                          a_log=None, dt_bias=None):
    """The gamma form with a diagonal decay, as literal Dk x Dk matrix products (K-major)."""
    N = q.shape[0]
    Dk, Dv = q.shape[2], v.shape[2]
    out = np.zeros((N, Hv, Dv))
    final = np.zeros((len(lengths), Hv, Dv, Dk))
    off = 0
    for b, L in enumerate(lengths):
        for h in range(Hv):
            qh = (h * Hq) // Hv
            S = np.zeros((Dk, Dv)) if init is None else init[b, h].T.copy()
            for t in range(off, off + L):
                kt, qt = k[t, qh].copy(), q[t, qh].copy()
                if l2norm:
                    kt = kt / np.sqrt(kt @ kt + 1e-12)
                    qt = qt / np.sqrt(qt @ qt + 1e-12)
                lg = g[t, h]
                if a_log is not None:
                    lg = -np.exp(a_log[h]) * np_softplus20(lg + dt_bias[h])
                Dt = np.diag(np.exp(lg))
                bt = beta[t, h]
                S = (np.eye(Dk) - bt * np.outer(kt, kt)) @ Dt @ S + bt * np.outer(kt, v[t, h])
                out[t, h] = scale * (qt @ S)
            final[b, h] = S.T
        off += L
    return out, final


@pytest.mark.parametrize("l2norm", [False, True])
@pytest.mark.parametrize("Hq,Hv", [(1, 1), (1, 2), (2, 4)])
def test_per_key_decay_matches_diagonal_gamma_form(oracle_mod, l2norm, Hq, Hv):
    rng = np.random.default_rng(300 + Hq * 10 + Hv + int(l2norm))
    lengths = [6, 1, 8, 0, 3]
    N, Dk, Dv = sum(lengths), 5, 4
    q = rng.standard_normal((N, Hq, Dk))
    k = rng.standard_normal((N, Hq, Dk))
    if not l2norm:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((N, Hv, Dv))
    g = -rng.uniform(0.0, 2.0, (N, Hv, Dk))
    beta = rng.uniform(0.0, 1.0, (N, Hv))
    init = rng.standard_normal((len(lengths), Hv, Dv, Dk))
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    out, fs = oracle_mod.prefill(q, k, v, g, beta, cu, init, scale=0.8, qk_l2norm=l2norm,
                                 decay_per_key=True)
    bo, bf = brute_prefill_per_key(q, k, v, g, beta, lengths, init, 0.8, l2norm, Hq, Hv)
    np.testing.assert_allclose(out, bo, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(fs, bf, rtol=1e-10, atol=1e-12)
    # the empty request copies its state through
    np.testing.assert_array_equal(fs[3], init[3])


def test_per_key_decay_qwen_gate_and_sigmoid_beta(oracle_mod):
    """The qwen gate maps every key dimension's decay input with the head's a_log and
    dt_bias; beta_activation sigmoid as in the scalar case."""
    rng = np.random.default_rng(310)
    N, Hv, Dk, Dv = 9, 2, 4, 3
    q, k = rng.standard_normal((2, N, 1, Dk))
    v = rng.standard_normal((N, Hv, Dv))
    graw = rng.standard_normal((N, Hv, Dk))
    braw = rng.standard_normal((N, Hv))
    a_log, dtb = rng.uniform(-1, 1, Hv), rng.uniform(-1, 1, Hv)
    init = rng.standard_normal((1, Hv, Dv, Dk))
    out, fs = oracle_mod.prefill(q, k, v, graw, braw, None, init, B=1, scale=0.9,
                                 qk_l2norm=True, gate_activation="qwen", a_log=a_log,
                                 dt_bias=dtb, beta_activation="sigmoid", decay_per_key=True)
    bo, bf = brute_prefill_per_key(q, k, v, graw, 1.0 / (1.0 + np.exp(-braw)), [N], init, 0.9,
                                   True, 1, Hv, a_log=a_log, dt_bias=dtb)
    np.testing.assert_allclose(out, bo, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(fs, bf, rtol=1e-10, atol=1e-12)


def test_per_key_gated_rule_is_decayed_linear_attention(oracle_mod):
    """update_rule gated with a per-key decay: the causal sum with per-dimension decay
    ratios, out_t = scale (sum_i q_t[i] e^{G_t[i]} S0[i, :] + sum_{j<=t} (sum_i q_t[i] k_j[i]
    e^{G_t[i] - G_j[i]}) v_j), and final state diag(e^{G_T}) S0 + sum_j (k_j e^{G_T - G_j}) v_j^T,
    with G the inclusive prefix sums of g over the tokens."""
    rng, q, k, v, init = _rand_case(311, 12, 5, 3, unit_keys=False)
    g = -rng.uniform(0.0, 1.0, (12, 1, 5))
    out, fs = oracle_mod.prefill(q, k, v, g, None, None, init, B=1, scale=1.1,
                                 update_rule="gated", decay_per_key=True)
    Q, K, V, G = q[:, 0], k[:, 0], v[:, 0], np.cumsum(g[:, 0], axis=0)
    S0k = init[0, 0].T
    mask = np.tril(np.ones((12, 12)))
    scores = np.einsum("ti,ji,tji->tj", Q, K, np.exp(G[:, None, :] - G[None, :, :])) * mask
    ro = 1.1 * ((Q * np.exp(G)) @ S0k + scores @ V)
    rf = np.exp(G[-1])[:, None] * S0k + (K * np.exp(G[-1] - G)).T @ V
    np.testing.assert_allclose(out[:, 0], ro, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(fs[0, 0], rf.T, rtol=1e-10, atol=1e-12)


def test_per_key_beta0_scales_state_columns(oracle_mod):
    """beta = 0 leaves only the decay: the V-major final state's column i is the initial one
    times exp(sum_t g_t[i]), and o_t = scale S0 (e^{G_t} * q_t)."""
    rng, q, k, v, init = _rand_case(312, 7, 6, 4)
    g = -rng.uniform(0.0, 0.7, (7, 1, 6))
    out, fs = oracle_mod.prefill(q, k, v, g, np.zeros((7, 1)), None, init, B=1, scale=0.6,
                                 decay_per_key=True)
    np.testing.assert_allclose(fs[0, 0], init[0, 0] * np.exp(g[:, 0].sum(0))[None, :],
                               rtol=1e-12)
    G = np.cumsum(g[:, 0], axis=0)
    np.testing.assert_allclose(out[:, 0], 0.6 * (q[:, 0] * np.exp(G)) @ init[0, 0].T,
                               rtol=1e-12, atol=1e-14)


def test_per_key_decay_with_equal_dimensions_is_the_scalar_gate(oracle_mod):
    """A per-key decay that is the same in every key dimension is the scalar decay, whose
    oracle is pinned to the page's worked examples and its own brute force above."""
    rng = np.random.default_rng(313)
    N, Hv, Dk, Dv = 10, 2, 4, 5
    q, k = rng.standard_normal((2, N, 1, Dk))
    v = rng.standard_normal((N, Hv, Dv))
    g = -rng.uniform(0.0, 1.5, (N, Hv))
    beta = rng.uniform(0.0, 1.0, (N, Hv))
    init = rng.standard_normal((1, Hv, Dv, Dk))
    o1, f1 = oracle_mod.prefill(q, k, v, g, beta, None, init, B=1, qk_l2norm=True)
    o2, f2 = oracle_mod.prefill(q, k, v, np.repeat(g[:, :, None], Dk, axis=2), beta, None, init,
                                B=1, qk_l2norm=True, decay_per_key=True)
    np.testing.assert_allclose(o2, o1, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(f2, f1, rtol=1e-12, atol=1e-14)
