"""Pins for the oracle's causal conv1d with a slot-indexed window pool.

Source: "max.nn.legacy.state_space.gated_delta_conv1d_fwd" (description,
Parameters, worked example).  The checks do not restate the oracle's loop:

* the worked example's stated outcome (two ragged sequences of lengths 3 and
  2 on slots 2 and 0 of a 3-slot pool: those slots end up holding the
  sequences' last inputs, slot 1 is unchanged, the result is [5, 8]);
* numpy's library convolution of the extended sequence (window, then the
  request's inputs) against the flipped weights;
* closed forms for delta weights (identity, a pure delay of K-1 tokens that
  pulls the first outputs from the window);
* continuation: one request split over two calls on the same slot equals a
  single call, for every split point (including pieces shorter than K-1);
* write_state = False leaves the pool unchanged and gives the same outputs;
  empty requests and out-of-range slots touch nothing.
No test here needs a GPU.
"""
import numpy as np
import pytest


def _case(rng, N, conv_dim, K, max_slots, lengths, slots):
    x = rng.standard_normal((N, conv_dim))
    w = rng.standard_normal((conv_dim, K))
    pool = rng.standard_normal((max_slots, conv_dim, K - 1))
    off = np.concatenate([[0], np.cumsum(lengths)]).astype(np.uint32)
    return x, w, pool, np.asarray(slots, np.uint32), off


def test_worked_example_slots(oracle_mod):
    # the page's example: total_seq_len 5, conv_dim 8, kernel_size 4, max_slots 3,
    # slots [2, 0], offsets [0, 3, 5], float32 inputs drawn by default_rng(0) in
    # the order x, weight, state
    total, conv_dim, K, max_slots = 5, 8, 4, 3
    rng = np.random.default_rng(0)
    x = rng.standard_normal((total, conv_dim), dtype=np.float32)
    w = rng.standard_normal((conv_dim, K), dtype=np.float32)
    state = rng.standard_normal((max_slots, conv_dim, K - 1), dtype=np.float32)
    y, new = oracle_mod.conv1d(x, w, state, np.array([2, 0], np.uint32),
                               np.array([0, 3, 5], np.uint32))
    assert y.shape == (5, 8)
    np.testing.assert_array_equal(new[1], state[1])            # slot 1 unchanged
    np.testing.assert_array_equal(new[2], x[0:3].T)            # last three inputs of sequence 0
    # sequence 1 has two inputs: they are the two newest entries, behind the
    # newest entry the slot held before
    np.testing.assert_array_equal(new[0][:, 1:], x[3:5].T)
    np.testing.assert_array_equal(new[0][:, 0], state[0][:, 2])


@pytest.mark.parametrize("K", [1, 2, 4, 5])
def test_matches_library_convolution(oracle_mod, K):
    rng = np.random.default_rng(11)
    lengths = [7, 1, 0, 12, 2]
    N, conv_dim, max_slots = sum(lengths), 6, 8
    slots = [5, 0, 3, 7, 2]
    x, w, pool, si, off = _case(rng, N, conv_dim, K, max_slots, lengths, slots)
    y, new = oracle_mod.conv1d(x, w, pool, si, off)
    for b, L in enumerate(lengths):
        s = int(off[b])
        if L == 0:
            continue
        for c in range(conv_dim):
            xe = np.concatenate([pool[slots[b], c], x[s:s + L, c]])
            full = np.convolve(xe, w[c, ::-1])
            np.testing.assert_allclose(y[s:s + L, c], full[K - 1:K - 1 + L], rtol=1e-12, atol=1e-12)
            np.testing.assert_array_equal(new[slots[b], c], xe[len(xe) - (K - 1):])
    # the slots no request names keep their values; so does the empty request's
    for r in set(range(max_slots)) - {slots[b] for b, L in enumerate(lengths) if L}:
        np.testing.assert_array_equal(new[r], pool[r])


def test_delta_weights(oracle_mod):
    rng = np.random.default_rng(3)
    K, conv_dim, lengths = 4, 5, [2, 9]
    N = sum(lengths)
    x, _, pool, si, off = _case(rng, N, conv_dim, K, 4, lengths, [1, 3])
    ident = np.zeros((conv_dim, K)); ident[:, K - 1] = 1.0
    y, _ = oracle_mod.conv1d(x, ident, pool, si, off)
    np.testing.assert_array_equal(y, x)
    delay = np.zeros((conv_dim, K)); delay[:, 0] = 1.0
    y, _ = oracle_mod.conv1d(x, delay, pool, si, off)
    # request 0 (2 tokens, slot 1): both outputs come from the window
    np.testing.assert_array_equal(y[0], pool[1][:, 0])
    np.testing.assert_array_equal(y[1], pool[1][:, 1])
    # request 1 (slot 3): three outputs from the window, then x delayed by K-1
    np.testing.assert_array_equal(y[2:5], pool[3].T)
    np.testing.assert_array_equal(y[5:11], x[2:8])


@pytest.mark.parametrize("split", [0, 1, 2, 3, 5, 10])
def test_continuation_over_two_calls(oracle_mod, split):
    rng = np.random.default_rng(5)
    K, conv_dim, L = 4, 3, 10
    x, w, pool, _, _ = _case(rng, L, conv_dim, K, 2, [L], [1])
    one_y, one_pool = oracle_mod.conv1d(x, w, pool, [1], [0, L])
    y1, p1 = oracle_mod.conv1d(x[:split], w, pool, [1], [0, split])
    y2, p2 = oracle_mod.conv1d(x[split:], w, p1, [1], [0, L - split])
    np.testing.assert_allclose(np.concatenate([y1, y2]), one_y, rtol=1e-13, atol=1e-13)
    np.testing.assert_array_equal(p2, one_pool)


def test_read_only_and_skips(oracle_mod):
    rng = np.random.default_rng(9)
    K, conv_dim, lengths = 3, 4, [4, 3, 0]
    N = sum(lengths) + 2                      # two trailing rows no request covers
    x, w, pool, _, _ = _case(rng, N, conv_dim, K, 3, lengths, [0, 1, 2])
    off = np.array([0, 4, 7, 7], np.uint32)
    y_w, p_w = oracle_mod.conv1d(x, w, pool, [2, 1, 0], off)
    y_r, p_r = oracle_mod.conv1d(x, w, pool, [2, 1, 0], off, write_state=False)
    np.testing.assert_array_equal(y_r, y_w)
    np.testing.assert_array_equal(p_r, pool)
    np.testing.assert_array_equal(p_w[0], pool[0])          # empty request: slot untouched
    np.testing.assert_array_equal(y_w[7:], 0.0)            # uncovered rows keep `out`
    # a slot >= max_slots: no output and no pool access for that request
    keep = np.full((N, conv_dim), 7.0)
    y_b, p_b = oracle_mod.conv1d(x, w, pool, [2, 9, 0], off, out=keep)
    np.testing.assert_array_equal(y_b[4:7], 7.0)
    np.testing.assert_array_equal(p_b[1], pool[1])
    np.testing.assert_array_equal(y_b[:4], y_w[:4])
    # offsets beyond N are clamped to N
    y_c, _ = oracle_mod.conv1d(x[:5], w, pool, [2, 1, 0], np.array([0, 4, 9, 9], np.uint32))
    np.testing.assert_allclose(y_c[:4], y_w[:4], rtol=0, atol=0)
    np.testing.assert_allclose(y_c[4], y_w[4], rtol=0, atol=0)
