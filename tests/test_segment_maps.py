"""The algebra behind the sequence-parallel split of long requests, checked on the CPU in float64
with the oracle alone.

Operation: the recurrence of "com.microsoft.GatedDeltaNet" (Description), which treats every
value column s of the state (Dk x Dv) on its own: s <- D_t s + k_t beta_t (v_t - (D_t s) . k_t),
with D_t = exp(g_t) (or diag(exp(g_t)) in the per-key-dimension spelling).  The step is affine in
s, so a run of tokens maps the state as S_end = A S_start + B with A (Dk x Dk) independent of the
values.  The split obtains both from ordinary runs of the recurrence, in the V-major layout the
kernels keep (rows = value columns):
* from the identity (Dk rows) with v = 0 the final state is A^T;
* from zero with the real v it is B^T;
so that S_end^T = S_start^T A^T + B^T, and three segments compose exactly like one run
(segment 0 from the true state gives S1, segment 1's map gives S2 = S1 A1^T + B1^T, segment 2
runs from S2).  The option attribute chunk_size states that the result does not depend on how
the sequence is cut, which these identities make concrete.
"""
import numpy as np
import pytest

import oracle


def _case(seed, L, Dk, Dv, per_key):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((L, 1, Dk))
    k = rng.standard_normal((L, 1, Dk))
    v = rng.standard_normal((L, 1, Dv))
    gshape = (L, 1, Dk) if per_key else (L, 1)
    g = -np.logaddexp(0.0, rng.standard_normal(gshape))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((L, 1))))
    S0 = 0.1 * rng.standard_normal((1, 1, Dv, Dk))       # V-major: [B, Hv, Dv, Dk]
    return q, k, v, g, beta, S0


def _run(q, k, v, g, beta, S, per_key):
    L = q.shape[0]
    return oracle.prefill(q, k, v, g, beta, np.array([0, L], np.int32), S, B=1, scale=0.5,
                          qk_l2norm=True, decay_per_key=per_key)


def _maps(q, k, v, g, beta, per_key):
    """(A^T, B^T) of a run, V-major, from the identity run with v = 0 and the zero run."""
    Dk, Dv = q.shape[2], v.shape[2]
    eye = np.eye(Dk)[None, None]
    _, At = _run(q, k, np.zeros((q.shape[0], 1, Dk)), g, beta, eye, per_key)
    _, Bt = _run(q, k, v, g, beta, np.zeros((1, 1, Dv, Dk)), per_key)
    return At[0, 0], Bt[0, 0]


@pytest.mark.parametrize("per_key", [False, True])
def test_a_run_is_affine_in_its_start_state(per_key):
    q, k, v, g, beta, S0 = _case(3, 57, 16, 8, per_key)
    At, Bt = _maps(q, k, v, g, beta, per_key)
    _, S_end = _run(q, k, v, g, beta, S0, per_key)
    np.testing.assert_allclose(S0[0, 0] @ At + Bt, S_end[0, 0], rtol=1e-12, atol=1e-12)
    # the map does not depend on the values: a run with other values has the same A
    At2, _ = _maps(q, k, 3.0 * v + 1.0, g, beta, per_key)
    np.testing.assert_allclose(At2, At, rtol=0, atol=0)


@pytest.mark.parametrize("per_key", [False, True])
def test_three_segments_compose_like_one_run(per_key):
    # weak decays over wide keys, so that each segment's map keeps much of its start state
    L, Dk, Dv = 200, 64, 8
    q, k, v, g, beta, S0 = _case(7, L, Dk, Dv, per_key)
    g = 0.02 * g
    o_ref, S_ref = _run(q, k, v, g, beta, S0, per_key)
    cuts = [0, 67, 134, L]
    seg = [tuple(x[cuts[i]:cuts[i + 1]] for x in (q, k, v, g, beta)) for i in range(3)]
    o0, S1 = _run(*seg[0], S0, per_key)
    A1t, B1t = _maps(*seg[1], per_key)
    assert np.abs(A1t).max() > 0.1
    S2 = S1[0, 0] @ A1t + B1t                              # the compose step
    o1, S2_run = _run(*seg[1], S1, per_key)
    o2, S3 = _run(*seg[2], S2[None, None], per_key)
    np.testing.assert_allclose(S2, S2_run[0, 0], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(np.concatenate([o0, o1, o2]), o_ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(S3, S_ref, rtol=1e-11, atol=1e-12)


def test_a_wrongly_transposed_map_is_caught():
    # the identities above are sharp: composing with A instead of A^T (one plausible slip) fails
    # on a short, weakly decayed run, whose map keeps much of the start state
    q, k, v, g, beta, S0 = _case(9, 6, 8, 8, False)
    g = np.full_like(g, -0.05)
    At, Bt = _maps(q, k, v, g, beta, False)
    _, S_end = _run(q, k, v, g, beta, S0, False)
    assert np.abs(S0[0, 0] @ At.T + Bt - S_end[0, 0]).max() > 1e-3
