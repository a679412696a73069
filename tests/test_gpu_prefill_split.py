"""GPU parity of the sequence-parallel prefill (gdn_prefill_ws, through the C ABI).

A long request of a call with few (request, head) units is cut into three segments: segment 0
from the true initial state; segment 1 from the identity with v = 0 and from zero, in parallel
(its affine map S -> A S + B); a composition of segment 2's start state; then segments 1 and 2
from their true start states.  Results must match the float64 oracle with the tolerance of the
unsplit path (relative L2 <= 2e-2 for bf16 activations with the fp32 state, per (request, head)
block and per row), and the unsplit chunked path with the same bound.
"""
import ctypes

import pytest
import torch

from _util import (TOL_BF16, assert_prefill_parity, dev, f64, oracle_prefill_case,
                   request_ranges)

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


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def call_ws(gdn, c, ws, ws_bytes=None, out=None, fs=None):
    """gdn_prefill_ws on case c with the workspace tensor ws; returns (status, out, final)."""
    Hq, Hv, Dk, Dv = c.dims
    q, k, v, g, b = (dev(t) for t in (c.q, c.k, c.v, c.g, c.beta))
    cu, init = dev(c.cu_seqlens), dev(c.initial_state)
    out = torch.empty((c.N, Hv, Dv), dtype=c.q.dtype, device="cuda") if out is None else out
    fs = torch.empty((c.B, Hv, Dv, Dk), dtype=torch.float32, device="cuda") if fs is None else fs
    nbytes = (ws.numel() * ws.element_size()) if ws_bytes is None else ws_bytes
    st = gdn.lib().gdn_prefill_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b), None, None,
                                  _ptr(cu), _ptr(init), _ptr(fs), _ptr(out), c.B, c.N, Hq, Hv,
                                  Dk, Dv, gdn.GDN_BF16, c.scale, int(c.qk_l2norm), 0, _ptr(ws),
                                  nbytes, None, None)
    torch.cuda.synchronize()
    return st, out, fs


@pytest.mark.parametrize("lengths,l2norm", [([1573], True), ([24 * 64], False),
                                            ([1600, 100, 0], True), ([2000, 1700], True)])
def test_split_matches_oracle_and_unsplit(gdn, W, oracle_mod, lengths, l2norm):
    """Requests of 24+ chunks are split (one per call, or all of them, or beside short and
    empty ones); every output row and final state against the oracle and against the unsplit
    call.  The workspace starts as NaN: the split wrote segment 1's start state, its A and B,
    and segment 2's start state for every head of a split request."""
    c = W.make_prefill(1400 + sum(lengths), lengths, 2, 4, 128, 128, init_std=0.05,
                       qk_l2norm=l2norm, host_norm_qk=not l2norm)
    nbytes = int(gdn.lib().gdn_prefill_workspace_size(c.B, c.N, 2, 4, 128, 128, gdn.GDN_BF16, 0))
    assert nbytes == c.B * 4 * (3 * 128 * 128 + 128 * 128) * 4
    ws = torch.full((nbytes // 4,), float("nan"), dtype=torch.float32, device="cuda")
    st, out, fs = call_ws(gdn, c, ws)
    assert st == gdn.GDN_OK
    ro, rf = oracle_prefill_case(oracle_mod, c)
    ranges = request_ranges(c.cu_seqlens, c.B, c.N)
    assert_prefill_parity(out, fs, ro, rf, ranges, TOL_BF16)
    ou, fu = gdn.gdn_prefill(dev(c.q), dev(c.k), dev(c.v), dev(c.g), dev(c.beta),
                             dev(c.cu_seqlens), dev(c.initial_state), scale=c.scale,
                             qk_l2norm=c.qk_l2norm, split=False)
    torch.cuda.synchronize()
    assert_prefill_parity(out, fs, f64(ou), f64(fu), ranges, TOL_BF16)
    per_bh = 4 * 128 * 128
    wsv = ws.view(c.B, 4, per_bh)
    for bq, L in enumerate(lengths):
        written = torch.isfinite(wsv[bq]).all().item()
        assert written == (L >= 24 * 64), (bq, L)
    if c.initial_state is not None:
        # an empty request copies its state through
        for bq, L in enumerate(lengths):
            if L == 0:
                assert torch.equal(fs[bq].cpu(), c.initial_state[bq])


def test_split_workspace_errors_and_short_calls(gdn, W):
    """A workspace smaller than the size the call needs is GDN_ERR_SHAPE, a misaligned one
    GDN_ERR_ALIGN, one that overlaps `out` GDN_ERR_ALIAS; a call that cannot split (too many
    units for the SMs, or an other rule) ignores its workspace."""
    c = W.make_prefill(1501, [1600], 2, 4, 128, 128, init_std=0.05, qk_l2norm=True)
    nbytes = int(gdn.lib().gdn_prefill_workspace_size(c.B, c.N, 2, 4, 128, 128, gdn.GDN_BF16, 0))
    assert nbytes > 0
    ws = torch.zeros(nbytes // 4 + 4, dtype=torch.float32, device="cuda")
    assert call_ws(gdn, c, ws, ws_bytes=nbytes - 16)[0] == gdn.GDN_ERR_SHAPE
    assert call_ws(gdn, c, ws[1:], ws_bytes=nbytes)[0] == gdn.GDN_ERR_ALIGN
    big = torch.zeros(c.N * 4 * 128 // 2 + nbytes // 4, dtype=torch.float32, device="cuda")
    out_alias = big[:c.N * 4 * 128 // 2].view(torch.bfloat16).view(c.N, 4, 128)
    assert call_ws(gdn, c, big, ws_bytes=nbytes, out=out_alias)[0] == gdn.GDN_ERR_ALIAS
    nsm = torch.cuda.get_device_properties(0).multi_processor_count
    many = nsm // 32 + 1   # requests x 32 heads > SMs: no split
    assert gdn.lib().gdn_prefill_workspace_size(many, 64 * many, 16, 32, 128, 128,
                                                gdn.GDN_BF16, 0) == 0
    assert gdn.lib().gdn_prefill_workspace_size(1, 4096, 16, 32, 128, 128, gdn.GDN_BF16,
                                                gdn._binding.GDN_RULE_DELTA) == 0


def test_split_long_context_all_heads_against_unsplit(gdn, W):
    """The long-context workload (B=1, S=32768, 32 heads): split and unsplit calls agree on
    every head (both are held against the oracle in test_gpu_prefill), and the split is taken
    (its workspace is written)."""
    c = W.long_prefill_case()
    nbytes = int(gdn.lib().gdn_prefill_workspace_size(1, c.N, 16, 32, 128, 128, gdn.GDN_BF16, 0))
    assert nbytes > 0
    ws = torch.full((nbytes // 4,), float("nan"), dtype=torch.float32, device="cuda")
    st, out, fs = call_ws(gdn, c, ws)
    assert st == gdn.GDN_OK
    assert torch.isfinite(ws).all()
    ou, fu = gdn.gdn_prefill(dev(c.q), dev(c.k), dev(c.v), dev(c.g), dev(c.beta),
                             dev(c.cu_seqlens), None, scale=c.scale, qk_l2norm=False,
                             split=False)
    torch.cuda.synchronize()
    assert_prefill_parity(out, fs, f64(ou), f64(fu), request_ranges(c.cu_seqlens, c.B, c.N),
                          TOL_BF16)
