"""GPU parity of the chunked prefill under its two unit schedules and unit switches.

The chunked kernel hands (request, value head) units to persistent CTAs: with
at most 32 requests by a least-loaded assignment computed on the device, with
more by dealing units in length order.  A CTA with several units hands the
state over between them at a unit's last chunk.  These cases put many units
on each CTA (empty and one-token requests between long ones), more value heads
than CTAs, and both schedules, and compare every output and final state with
the float64 oracle (relative L2 <= 2e-2, bf16 activations, per (request, head) block
and per row); no pipeline wait
may time out.
"""
import pytest
import torch

from _util import TOL_BF16, assert_prefill_parity, dev, oracle_prefill_case, request_ranges

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gdn():
    import gated_deltanet_state_gdn_b200 as g
    g.lib()
    return g


@pytest.fixture(scope="module")
def W():
    from gated_deltanet_state_gdn_b200 import workloads
    return workloads


def run_checked(gdn, c):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, fs = gdn.gdn_prefill(dev(c.q), dev(c.k), dev(c.v), dev(c.g), dev(c.beta),
                              dev(c.cu_seqlens), dev(c.initial_state), scale=c.scale,
                              qk_l2norm=c.qk_l2norm, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return out, fs


def check_all(gdn, oracle_mod, c):
    Hq, Hv, Dk, Dv = c.dims
    assert gdn.prefill_uses_chunked(c.q.dtype, Hv, Dk, Dv)
    out, fs = run_checked(gdn, c)
    ro, rf = oracle_prefill_case(oracle_mod, c)
    assert_prefill_parity(out, fs, ro, rf, request_ranges(c.cu_seqlens, c.B, c.N), TOL_BF16)


def test_least_loaded_schedule_many_units_per_cta(gdn, W, oracle_mod):
    # 20 requests x 32 heads = 640 units on at most 148 CTAs: several units per CTA, with
    # empty and one-token requests between long ones (state hand-over at each switch)
    lengths = [300, 0, 1, 65, 64, 129, 0, 200, 7, 250, 1, 0, 190, 63, 128, 2, 33, 0, 111, 5]
    c = W.make_prefill(901, lengths, 16, 32, 128, 128, init_std=0.05, qk_l2norm=True)
    check_all(gdn, oracle_mod, c)


def test_length_order_schedule_over_32_requests(gdn, W, oracle_mod):
    # 40 requests: the kernel deals units in length order instead
    lengths = [(37 * i) % 150 for i in range(40)]
    c = W.make_prefill(902, lengths, 2, 8, 128, 128, init_std=0.05, qk_l2norm=True)
    check_all(gdn, oracle_mod, c)


def test_more_heads_than_ctas(gdn, W, oracle_mod):
    # one request with 256 value heads (128 query/key heads): the least-loaded assignment
    # needs two rounds for the request's heads
    c = W.make_prefill(903, [130], 128, 256, 128, 128, init_std=0.05, qk_l2norm=True)
    check_all(gdn, oracle_mod, c)


def test_schedules_agree(gdn, W):
    # the same units under both schedules give identical bytes: 32 requests take the
    # least-loaded assignment, the same 32 requests plus one empty request the other
    lengths = [(53 * i) % 200 + 1 for i in range(32)]
    c = W.make_prefill(904, lengths, 2, 8, 128, 128, init_std=0.05, qk_l2norm=True)
    out_a, fs_a = run_checked(gdn, c)
    c2 = W.make_prefill(904, lengths, 2, 8, 128, 128, init_std=0.05, qk_l2norm=True)
    N = c2.q.shape[0]
    c2.cu_seqlens = torch.cat([c2.cu_seqlens, torch.tensor([N], dtype=torch.int32)])
    c2.initial_state = torch.cat([c2.initial_state, c2.initial_state[:1]])
    c2.B = c2.B + 1
    out_b, fs_b = run_checked(gdn, c2)
    assert torch.equal(out_a, out_b)
    assert torch.equal(fs_a, fs_b[:32])
    assert torch.equal(fs_b[32], c2.initial_state[32].cuda())
