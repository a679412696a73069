"""The bounds-checked test build (libgdn_checked.so, compiled with GDN_CHECKS) on cases that
reach every kernel and launch form.

* No global access and no data-dependent shared-memory access leaves its buffer: the status
  word gets no GDN_DEV_BOUNDS (only the GDN_DEV_BAD_SLOT a case provokes on purpose).
* The checks change no arithmetic: outputs, final states and pools equal the product
  library's bit for bit.
* The persistent decode kernel's bounded wait, made to run out on request
  (GDN_DEV_TEST_STALL), ends with GDN_DEV_TIMEOUT after about a second, and the next call
  on the same context is correct.
* The chunked prefill kernel's abort path, forced the same way (its first q/k stage expects
  16 bytes more than arrive), ends every role through its waits' bounds, the abort flag and
  the per-chunk votes: GDN_DEV_TIMEOUT, a return within seconds, and a correct next call.
"""
import copy
import time

import numpy as np
import pytest
import torch

from _util import dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gdn():
    import gated_deltanet_state_gdn_b200 as g
    from gated_deltanet_state_gdn_b200 import build
    build.build(checked=True)   # rebuilds only when missing or older than the sources
    product = g._binding.LIB_PATH
    yield g
    g.use_library(product)


@pytest.fixture(scope="module")
def W():
    from gated_deltanet_state_gdn_b200 import workloads
    return workloads


def both(gdn, fn):
    """fn(status) through the product library, then through the checked build; returns both
    results and the checked run's status word."""
    product = gdn._binding.LIB_PATH
    r0 = fn(None)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    gdn.use_library(gdn.CHECKED_LIB_PATH)
    try:
        r1 = fn(st)
    finally:
        gdn.use_library(product)
    return r0, r1, int(st.item())


def assert_same(r0, r1):
    for a, b in zip(r0, r1):
        assert a.dtype == b.dtype and a.shape == b.shape
        assert torch.equal(a, b)


# ---------------------------------------------------------------- prefill
def prefill_fn(gdn, c):
    # the per-key spelling of the decay is read from g's rank
    def fn(st):
        o, f = gdn.gdn_prefill(dev(c.q), dev(c.k), dev(c.v), dev(c.g), dev(c.beta),
                               dev(c.cu_seqlens), dev(c.initial_state), None, None,
                               num_requests=c.B, scale=c.scale, qk_l2norm=c.qk_l2norm,
                               dev_status=st)
        torch.cuda.synchronize()
        return o.cpu(), f.cpu()
    return fn


@pytest.mark.parametrize("name,lengths,Hq,Hv,Dk,Dv,dtype,per_key", [
    ("chunked default", [70, 1, 130, 0, 64], 2, 4, 128, 128, torch.bfloat16, False),
    ("chunked head sizes", [33, 100], 2, 4, 64, 40, torch.bfloat16, False),
    ("chunked fp16", [90, 5], 2, 4, 128, 128, torch.float16, False),
    ("chunked plain-staged odd heads", [33, 70, 0, 5], 1, 2, 12, 9, torch.bfloat16, False),
    ("chunked per-key decay", [70, 1, 130, 0, 64], 2, 4, 128, 128, torch.bfloat16, True),
    ("chunked per-key decay odd heads", [33, 70, 0, 5], 1, 2, 10, 9, torch.bfloat16, True),
    ("per-token fp32", [20, 7], 1, 2, 12, 9, torch.float32, False),
    ("per-token per-key fp16", [20, 7], 1, 2, 12, 9, torch.float16, True),
])
def test_prefill_in_bounds(gdn, W, name, lengths, Hq, Hv, Dk, Dv, dtype, per_key):
    c = W.make_prefill(11 + len(name), lengths, Hq, Hv, Dk, Dv, dtype=dtype, init_std=0.02,
                       qk_l2norm=True, decay_per_key=per_key)
    chunked = gdn.prefill_uses_chunked(dtype, Hv, Dk, Dv, decay_per_key=per_key)
    assert chunked == name.startswith("chunked")
    r0, r1, st = both(gdn, prefill_fn(gdn, c))
    assert st == 0
    assert_same(r0, r1)


def test_chunked_prefill_wait_runs_out_on_request(gdn, W):
    """GDN_DEV_TEST_STALL in the status word makes the chunked kernel's first q/k stage expect
    16 bytes more than its copies deliver (one request of one chunk, four value heads: four
    CTAs).  The prep front's wait on that stage runs out; the UMMA issuers, the prep back and
    the state warpgroup end their waits on the abort flag; every group leaves through its
    per-chunk vote; the teardown drains and frees TMEM.  GDN_DEV_TIMEOUT is reported, no
    bounds bit, the call returns within seconds, and a normal call on the same context then
    matches the product library bit for bit."""
    c = W.make_prefill(77, [40], 1, 4, 128, 128, init_std=0.05, qk_l2norm=True)
    assert gdn.prefill_uses_chunked(c.q.dtype, 4, 128, 128)
    product = gdn._binding.LIB_PATH
    gdn.use_library(gdn.CHECKED_LIB_PATH)
    try:
        st = torch.full((1,), gdn.GDN_DEV_TEST_STALL, dtype=torch.int32, device="cuda")
        t0 = time.time()
        prefill_fn(gdn, c)(st)
        took = time.time() - t0
        s = int(st.item())
        assert s & gdn.GDN_DEV_TIMEOUT
        assert not s & gdn.GDN_DEV_BOUNDS
        assert took < 60
        st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
        r1 = prefill_fn(gdn, c)(st2)
        assert int(st2.item()) == 0
    finally:
        gdn.use_library(product)
    r0 = prefill_fn(gdn, c)(None)
    assert_same(r0, r1)


def test_per_key_prefill_wait_runs_out_on_request(gdn, W):
    """The per-key tensor-core kernel: GDN_DEV_TEST_STALL makes CTA 0 wait for its first W/U~
    MMA group on a barrier that nothing arrives on.  By then (1b) is in flight on its own
    barrier and, CTA 0's request having two chunks, so are the copies of the next chunk's decay
    tile.  The wait runs out, GDN_DEV_TIMEOUT is set, the CTA drains both barriers and its
    copies, frees TMEM and returns; the other CTAs finish normally.  A normal call on the same
    context then matches the product library bit for bit."""
    c = W.make_prefill(78, [40, 90], 1, 4, 128, 128, init_std=0.05, qk_l2norm=True,
                       decay_per_key=True)
    assert gdn.prefill_uses_chunked(c.q.dtype, 4, 128, 128, decay_per_key=True)
    product = gdn._binding.LIB_PATH
    gdn.use_library(gdn.CHECKED_LIB_PATH)
    try:
        st = torch.full((1,), gdn.GDN_DEV_TEST_STALL, dtype=torch.int32, device="cuda")
        t0 = time.time()
        prefill_fn(gdn, c)(st)
        took = time.time() - t0
        s = int(st.item())
        assert s & gdn.GDN_DEV_TIMEOUT
        assert not s & gdn.GDN_DEV_BOUNDS
        assert took < 60
        st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
        r1 = prefill_fn(gdn, c)(st2)
        assert int(st2.item()) == 0
    finally:
        gdn.use_library(product)
    r0 = prefill_fn(gdn, c)(None)
    assert_same(r0, r1)


# ---------------------------------------------------------------- decode
def decode_fn(gdn, c, pool_factory=None):
    def fn(st):
        pool = dev(c.pool) if pool_factory is None else pool_factory()
        o, _ = gdn.gdn_decode(dev(c.q), dev(c.k), dev(c.v), pool, dev(c.read_idx), dev(c.A_log),
                              dev(c.a), dev(c.dt_bias), dev(c.b), scale=c.scale,
                              scatter_idx=dev(c.scatter_idx), use_qk_l2norm=c.use_qk_l2norm,
                              write_idx=dev(c.write_idx), dev_status=st)
        torch.cuda.synchronize()
        return o.cpu(), pool.cpu()
    return fn


def test_decode_persistent_form_in_bounds(gdn, W):
    """Several tokens and Householder sub-steps, per-token scatter with a skipped entry, padding
    rows and a read slot beyond the pool (flagged as such, not as a bounds error)."""
    c = W.make_decode(21, P=64, B=12, T=4, nh=2, H=4, Dv=64, pad_frac=0.25, write_mode="none",
                      scatter=True)
    live = np.nonzero(c.read_idx.numpy() >= 0)[0]
    c.read_idx[int(live[0])] = 64
    c.scatter_idx[int(live[1]), 2] = -1
    r0, r1, st = both(gdn, decode_fn(gdn, c))
    assert st == gdn.GDN_DEV_BAD_SLOT
    assert_same(r0, r1)


def test_decode_per_unit_form_in_bounds(gdn, W):
    """Single-token rows filling many waves (the one-CTA-per-unit form), distinct write slots."""
    c = W.make_decode(22, P=200, B=96, T=1, nh=1, H=32, Dv=128, pad_frac=0.1,
                      write_mode="distinct")
    r0, r1, st = both(gdn, decode_fn(gdn, c))
    assert st == 0
    assert_same(r0, r1)


def test_decode_strided_pool_and_int64_slots_in_bounds(gdn, W):
    """A pool with padding between heads and slots (the check uses the strides' reach) and
    int64 slot indices."""
    c = W.make_decode(23, P=64, B=12, T=2, nh=1, H=4, Dv=128, pad_frac=0.25, write_mode="same")
    c = copy.copy(c)
    c.read_idx = c.read_idx.to(torch.int64)
    c.write_idx = c.write_idx.to(torch.int64)
    P, HV, Dv, Dk = c.pool.shape

    def strided_pool():
        big = torch.full((P, HV + 1, Dv + 4, Dk), 9.0, dtype=torch.float32, device="cuda")
        view = big[:, :HV, :Dv, :]
        view.copy_(dev(c.pool))
        return view

    r0, r1, st = both(gdn, decode_fn(gdn, c, strided_pool))
    assert st == 0
    assert_same(r0, r1)


def test_decode_wait_runs_out_on_request(gdn, W):
    """GDN_DEV_TEST_STALL in the status word makes the persistent kernel's first copy wait run
    out (16 bytes more are expected than arrive): GDN_DEV_TIMEOUT is reported, the call returns
    within seconds, and a normal call on the same context then matches the product library."""
    c = W.make_decode(41, P=16, B=2, T=2, nh=1, H=4, Dv=64, write_mode="distinct")
    product = gdn._binding.LIB_PATH
    gdn.use_library(gdn.CHECKED_LIB_PATH)
    try:
        st = torch.full((1,), gdn.GDN_DEV_TEST_STALL, dtype=torch.int32, device="cuda")
        t0 = time.time()
        decode_fn(gdn, c)(st)
        took = time.time() - t0
        s = int(st.item())
        assert s & gdn.GDN_DEV_TIMEOUT
        assert not s & gdn.GDN_DEV_BOUNDS
        assert took < 60
        st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
        r1 = decode_fn(gdn, c)(st2)
        assert int(st2.item()) == 0
    finally:
        gdn.use_library(product)
    r0 = decode_fn(gdn, c)(None)
    assert_same(r0, r1)


# ---------------------------------------------------------------- conv1d
def conv_fn(gdn, c):
    def fn(st):
        pool = dev(c.conv_state)
        y, _ = gdn.gdn_conv1d(dev(c.x), dev(c.weight), pool, dev(c.slot_idx),
                              dev(c.row_offsets), dev_status=st)
        torch.cuda.synchronize()
        return y.cpu(), pool.cpu()
    return fn


@pytest.mark.parametrize("name,lengths,conv_dim,K,slots,dtype", [
    ("staged rows", [5, 40, 1, 0, 77], 2048, 4, 8, torch.bfloat16),
    ("element path", [5, 40, 1, 77], 1001, 3, 8, torch.bfloat16),
    ("decode step", [1] * 64, 8192, 4, 128, torch.bfloat16),
    ("fp32 one tap", [9, 3], 256, 1, 4, torch.float32),
])
def test_conv1d_in_bounds(gdn, W, name, lengths, conv_dim, K, slots, dtype):
    c = W.make_conv1d(31 + len(name), lengths, conv_dim, K, slots, dtype=dtype)
    r0, r1, st = both(gdn, conv_fn(gdn, c))
    assert st == 0
    assert_same(r0, r1)
