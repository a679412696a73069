"""The blocked solve T = (I + A)^-1 of the chunked prefill kernels, checked on the CPU in float64.

A is the strictly lower-triangular 64 x 64 matrix of a chunk (the delta rule's key products,
"com.microsoft.GatedDeltaNet", Description, unrolled over a chunk).  The kernels invert I + A by
16 x 16 blocks:
* diagonal blocks D_I = (I + A_II)^-1 by forward substitution; the per-key kernel runs it as a
  column sweep in which the finished row m is broadcast and every later row r subtracts
  A_rm times it;
* T_10 = -D_1 A_10 D_0 and T_32 = -D_3 A_32 D_2;
* the lower-left 2 x 2 of blocks: X = A_BA T_AA, then T_BA = -T_BB X, where AA are blocks 0-1
  and BB blocks 2-3.
The tests check that these steps give the inverse, and that the sweep gives each diagonal
block's inverse.
"""
import numpy as np


def _lower(seed, n=64, scale=0.4):
    rng = np.random.default_rng(seed)
    return np.tril(rng.standard_normal((n, n)) * scale, -1)


def _sweep(Ab):
    """(I + Ab)^-1 of a strictly lower block, one column at a time as the per-key kernel does."""
    n = Ab.shape[0]
    X = np.zeros((n, n))
    for c in range(n):
        x = (np.arange(n) == c).astype(float)
        for m in range(n - 1):
            y = x[m]                          # row m is final at step m
            for r in range(m + 1, n):
                x[r] -= Ab[r, m] * y
        X[:, c] = x
    return X


def _blocked_inverse(A):
    blk = lambda I, J: A[16 * I:16 * I + 16, 16 * J:16 * J + 16]
    D = [_sweep(blk(I, I)) for I in range(4)]
    T10 = -D[1] @ blk(1, 0) @ D[0]
    T32 = -D[3] @ blk(3, 2) @ D[2]
    T_AA = np.block([[D[0], np.zeros((16, 16))], [T10, D[1]]])
    T_BB = np.block([[D[2], np.zeros((16, 16))], [T32, D[3]]])
    A_BA = A[32:, :32]
    X = A_BA @ T_AA
    T_BA = -T_BB @ X
    return np.block([[T_AA, np.zeros((32, 32))], [T_BA, T_BB]])


def test_sweep_inverts_a_diagonal_block():
    Ab = _lower(1, 16, 0.6)
    np.testing.assert_allclose(_sweep(Ab), np.linalg.inv(np.eye(16) + Ab), rtol=1e-12, atol=1e-12)


def test_blocked_steps_give_the_inverse():
    for seed in range(3):
        A = _lower(seed + 10)
        T = _blocked_inverse(A)
        np.testing.assert_allclose(T @ (np.eye(64) + A), np.eye(64), atol=1e-9)
        np.testing.assert_allclose(T, np.linalg.inv(np.eye(64) + A), rtol=1e-9, atol=1e-9)


def test_a_dropped_merge_term_is_caught():
    # forgetting the T_BB factor of the merge (one plausible slip) leaves a wrong inverse
    A = _lower(5)
    T = _blocked_inverse(A)
    T_bad = T.copy()
    T_bad[32:, :32] = -(A[32:, :32] @ T[:32, :32])
    assert np.abs(T_bad - np.linalg.inv(np.eye(64) + A)).max() > 1e-2
