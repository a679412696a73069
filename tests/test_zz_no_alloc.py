"""gdn_prefill_noalloc: the split prefill with the library's own fixed workspace.

Callers that cannot allocate device memory (a host runtime that owns all device memory in its
own pool, a C caller without a memory manager, a serving path that must never allocate) use
this entry point instead of gdn_prefill_ws: the workspace is a static device array inside
libgdn.so (8 MiB), looked up on the first call on each device.  Its results must equal those of
the existing entry point that takes a caller workspace, within the tolerance of the other
prefill tests (relative L2 <= 2e-2 for bf16 activations, per (request, head) block and per row),
on two calls in a row (the second finds the first call's contents in the array).

This file is collected last, so that a run stopping at the first failure has run every other
test; it also passes alone in a fresh process (it loads the library itself).
"""
import ctypes

import pytest
import torch

from _util import TOL_BF16, assert_prefill_parity, dev, f64, request_ranges

pytestmark = pytest.mark.gpu

MAX_BYTES = 8 << 20   # the library's static workspace


@pytest.fixture(scope="module")
def gdn():
    import gated_deltanet_state_gdn_b200 as g
    g.lib()
    return g


@pytest.fixture(scope="module")
def W():
    from gated_deltanet_state_gdn_b200 import workloads
    return workloads


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def noalloc(gdn, c, tensors):
    """One gdn_prefill_noalloc call through the C ABI; returns (status, out, final_state)."""
    Hq, Hv, Dk, Dv = c.dims
    q, k, v, g, b, cu, init = tensors
    out = torch.empty((c.N, Hv, Dv), dtype=c.q.dtype, device="cuda")
    fs = torch.empty((c.B, Hv, Dv, Dk), dtype=torch.float32, device="cuda")
    st = gdn.lib().gdn_prefill_noalloc(_p(q), _p(k), _p(v), _p(g), _p(b), None, None, _p(cu),
                                       _p(init), _p(fs), _p(out), c.B, c.N, Hq, Hv, Dk, Dv,
                                       gdn.GDN_BF16, c.scale, int(c.qk_l2norm), 0, None, None)
    torch.cuda.synchronize()
    return st, out, fs


@pytest.mark.parametrize("which", ["long", "two_requests"])
def test_noalloc_matches_workspace_entry_point(gdn, W, which):
    """The long-context workload (one request, 32 heads: the whole 8 MiB) and a two-request
    call with short and split requests, each called twice in a row without allocating; both
    calls against gdn_prefill_ws with a workspace from torch."""
    if which == "long":
        c = W.long_prefill_case()
    else:
        c = W.make_prefill(2201, [2000, 300], 2, 4, 128, 128, init_std=0.05, qk_l2norm=True)
    Hq, Hv, Dk, Dv = c.dims
    need = int(gdn.lib().gdn_prefill_workspace_size(c.B, c.N, Hq, Hv, Dk, Dv, gdn.GDN_BF16, 0))
    assert 0 < need <= MAX_BYTES
    tensors = [dev(t) for t in (c.q, c.k, c.v, c.g, c.beta, c.cu_seqlens, c.initial_state)]
    ro, rf = gdn.gdn_prefill(*tensors, num_requests=c.B, scale=c.scale, qk_l2norm=c.qk_l2norm)
    torch.cuda.synchronize()
    ranges = request_ranges(c.cu_seqlens, c.B, c.N)
    for _ in range(2):
        st, out, fs = noalloc(gdn, c, tensors)
        assert st == gdn.GDN_OK
        assert_prefill_parity(out, fs, f64(ro), f64(rf), ranges, TOL_BF16)


def test_noalloc_rejects_calls_beyond_its_workspace(gdn, W):
    """Two requests of 32 heads would need 16 MiB of split workspace: refused with
    GDN_ERR_UNSUPPORTED before anything is launched (the outputs keep their values)."""
    nsm = torch.cuda.get_device_properties(0).multi_processor_count
    assert 64 <= nsm
    c = W.make_prefill(2202, [1600, 1600], 16, 32, 128, 128, init_std=None, qk_l2norm=True)
    need = int(gdn.lib().gdn_prefill_workspace_size(c.B, c.N, 16, 32, 128, 128, gdn.GDN_BF16, 0))
    assert need > MAX_BYTES
    tensors = [dev(t) for t in (c.q, c.k, c.v, c.g, c.beta, c.cu_seqlens, c.initial_state)]
    out = torch.full((c.N, 32, 128), 5.0, dtype=torch.bfloat16, device="cuda")
    fs = torch.empty((c.B, 32, 128, 128), dtype=torch.float32, device="cuda")
    q, k, v, g, b, cu, init = tensors
    st = gdn.lib().gdn_prefill_noalloc(_p(q), _p(k), _p(v), _p(g), _p(b), None, None, _p(cu),
                                       None, _p(fs), _p(out), c.B, c.N, 16, 32, 128, 128,
                                       gdn.GDN_BF16, c.scale, 1, 0, None, None)
    torch.cuda.synchronize()
    assert st == gdn.GDN_ERR_UNSUPPORTED
    assert (out == 5.0).all()
