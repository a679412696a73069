"""CPU checks of the parity helpers used by the GPU tests.

The GPU parity tests apply the stated tolerance to every (request, value head) block and to
every output row, not only to the whole tensor.  These tests plant mistakes into a copy of an
oracle result (on the CPU) and check that the block and row bounds catch what a whole-tensor
norm lets through: one wrong token row among thousands, and one wrong final state among many.
"""
import numpy as np
import pytest

from _util import (TOL_BF16, assert_out_close, assert_prefill_parity, assert_states_close,
                   f64, oracle_prefill_case, rel_l2, request_ranges)


@pytest.fixture(scope="module")
def case_and_ref(oracle_mod):
    from gated_deltanet_state_gdn_b200 import workloads as W
    c = W.make_prefill(3001, [1000, 37, 0, 64], 1, 4, 32, 32, init_std=0.1, qk_l2norm=True)
    ro, rf = oracle_prefill_case(oracle_mod, c)
    # a stand-in for a correct kernel result: the reference with a relative error of 3e-3,
    # about what the tensor-core kernel measures against the oracle
    rng = np.random.default_rng(1)
    o = ro * (1 + 3e-3 * rng.standard_normal(ro.shape))
    f = rf * (1 + 3e-3 * rng.standard_normal(rf.shape))
    return c, ro, rf, o, f


def test_correct_result_passes(case_and_ref):
    c, ro, rf, o, f = case_and_ref
    assert_prefill_parity(o, f, ro, rf, request_ranges(c.cu_seqlens, c.B, c.N), TOL_BF16)


def test_one_wrong_row_is_caught(case_and_ref):
    c, ro, rf, o, f = case_and_ref
    bad = o.copy()
    bad[700, 2] = 0.1 * ro[700, 2]          # one token of one head, 90 % off
    assert rel_l2(bad, ro) <= TOL_BF16      # the whole-tensor norm does not see it
    with pytest.raises(AssertionError, match="row"):
        assert_prefill_parity(bad, f, ro, rf, request_ranges(c.cu_seqlens, c.B, c.N), TOL_BF16)


def test_tail_row_of_short_request_is_caught(case_and_ref):
    c, ro, rf, o, f = case_and_ref
    bad = o.copy()
    bad[1036, 1] = ro[1035, 1]              # the last token of the 37-token request, shifted
    with pytest.raises(AssertionError):
        assert_prefill_parity(bad, f, ro, rf, request_ranges(c.cu_seqlens, c.B, c.N), TOL_BF16)


def test_one_wrong_final_state_is_caught(case_and_ref):
    c, ro, rf, o, f = case_and_ref
    bad = f.copy()
    bad[1, 3] = 0.97 * rf[1, 3]             # one (request, head) state 3 % off
    assert rel_l2(bad, rf) <= TOL_BF16      # the whole-tensor norm does not see it
    with pytest.raises(AssertionError, match="final state request 1 head 3"):
        assert_prefill_parity(o, bad, ro, rf, request_ranges(c.cu_seqlens, c.B, c.N), TOL_BF16)


def test_decode_blocks(oracle_mod):
    from gated_deltanet_state_gdn_b200 import workloads as W
    c = W.make_decode(3002, P=96, B=40, T=2, nh=1, H=4, Dv=64, pad_frac=0.0,
                      write_mode="distinct")
    ro, rp = oracle_mod.decode(f64(c.q), f64(c.k), f64(c.v), f64(c.pool), c.read_idx.numpy(),
                               f64(c.A_log), f64(c.a), f64(c.dt_bias), f64(c.b),
                               write_idx=c.write_idx.numpy(), scale=c.scale,
                               use_qk_l2norm=c.use_qk_l2norm)
    assert_out_close(ro.copy(), ro, TOL_BF16)
    bad = ro.copy()
    bad[17, 1, 3] *= 0.7                    # one token of one (row, head), 30 % off
    assert rel_l2(bad, ro) <= TOL_BF16
    with pytest.raises(AssertionError, match="row 17 head 3"):
        assert_out_close(bad, ro, TOL_BF16)
    slots = c.write_idx.numpy()
    badp = rp.copy()
    badp[slots[5], 2, 10] = 0.0             # one state row of one (slot, head)
    with pytest.raises(AssertionError):
        assert_states_close(badp[slots], rp[slots], TOL_BF16)


def test_request_ranges_clamp():
    assert request_ranges(np.array([10, 40, 40, 60, 120, 3]), 5, 140) == \
        [(10, 40), (40, 40), (40, 60), (60, 120), (120, 120)]
    assert request_ranges(np.array([-9, 40, 30, 640]), 3, 140) == [(0, 40), (40, 40), (30, 140)]
    assert request_ranges(None, 2, 10) == [(0, 5), (5, 10)]
