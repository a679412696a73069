"""GPU parity of gdn_conv1d against the float64 oracle (through the C ABI).

Tolerance, from the arithmetic: the kernel sums K products in fp32 and rounds
once to the output dtype, so every element satisfies
    |y - y_ref| <= u_out |y_ref| + a_out + 8 K 2^-24 sum_j |w_j xe_j|
with u_out = 2^-8 (bf16), 2^-11 (fp16), 0 (fp32) -- twice the round-to-
nearest bound -- and a_out = 2^-24 for fp16, the spacing of its subnormals
(below 2^-14 fp16 rounding is absolute, not relative; bf16 and fp32
subnormals are far below any value here).  The window pool is a copy of input values, so every slot must
match the oracle bit for bit, and slots no request writes must keep their bytes.
"""
import numpy as np
import pytest
import torch

from _util import dev, f64

pytestmark = pytest.mark.gpu

U_OUT = {torch.bfloat16: 2.0 ** -8, torch.float16: 2.0 ** -11, torch.float32: 0.0}
A_OUT = {torch.bfloat16: 0.0, torch.float16: 2.0 ** -24, torch.float32: 0.0}


@pytest.fixture(scope="module")
def gdn():
    import gated_deltanet_state_gdn_b200 as g
    g.lib()
    return g


@pytest.fixture(scope="module")
def W():
    from gated_deltanet_state_gdn_b200 import workloads
    return workloads


def run_gpu(gdn, c, *, pool=None, out=None, write_state=True, dev_status=None):
    pool = dev(c.conv_state) if pool is None else pool
    y, _ = gdn.gdn_conv1d(dev(c.x), dev(c.weight), pool, dev(c.slot_idx), dev(c.row_offsets),
                          None if out is None else dev(out), write_state=write_state,
                          dev_status=dev_status)
    torch.cuda.synchronize()
    return y.cpu(), pool.cpu()


def run_oracle(oracle, c, *, out=None, write_state=True, pool=None):
    pool = c.conv_state if pool is None else pool
    return oracle.conv1d(f64(c.x), f64(c.weight), f64(pool), c.slot_idx.numpy(),
                         c.row_offsets.numpy(), write_state=write_state,
                         out=None if out is None else f64(out))


def magnitude(oracle, c):
    m, _ = oracle.conv1d(np.abs(f64(c.x)), np.abs(f64(c.weight)), np.abs(f64(c.conv_state)),
                         c.slot_idx.numpy(), c.row_offsets.numpy())
    return m


def check_outputs(y, ref, mag, dtype, K):
    err = np.abs(f64(y) - ref)
    bound = U_OUT[dtype] * np.abs(ref) + A_OUT[dtype] + 8 * K * 2.0 ** -24 * mag + 1e-30
    bad = err > bound
    assert not bad.any(), (f"{bad.sum()} elements out of bound; worst excess "
                           f"{(err - bound).max():.3e} at {np.unravel_index((err - bound).argmax(), err.shape)}")


def check_pool(pool, ref_pool, c):
    np.testing.assert_array_equal(f64(pool), ref_pool)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16, torch.float32])
@pytest.mark.parametrize("K", [4, 2, 8])
def test_ragged_parity(gdn, W, oracle_mod, dtype, K):
    # 3 channel tiles (the last partial) on the vector path; lengths cross chunk edges, are
    # shorter than the window, empty; rows before the first and after the last request
    # belong to none
    lengths = [1, 2, 3, 37, 200, 0, 64, 65, 7, 129]
    c = W.make_conv1d(100 + K, lengths, 2176, K, 16, dtype=dtype, lead=5, N=5 + sum(lengths) + 9)
    keep = torch.full_like(c.x, 3.0)
    y, pool = run_gpu(gdn, c, out=keep)
    ref, ref_pool = run_oracle(oracle_mod, c, out=keep)
    check_outputs(y, ref, magnitude(oracle_mod, c), dtype, K)
    check_pool(pool, ref_pool, c)
    assert (y[:5] == 3.0).all() and (y[-9:] == 3.0).all()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("K", [1, 3, 4, 5, 6, 7])
def test_element_path_and_other_widths(gdn, W, oracle_mod, dtype, K):
    # conv_dim 1001 breaks the 16-byte row rule, so the element-wise path runs
    lengths = [9, 1, 40, 2, 17]
    c = W.make_conv1d(200 + K, lengths, 1001, K, 8, dtype=dtype)
    y, pool = run_gpu(gdn, c)
    ref, ref_pool = run_oracle(oracle_mod, c)
    check_outputs(y, ref, magnitude(oracle_mod, c), dtype, K)
    check_pool(pool, ref_pool, c)


def test_long_requests_use_wide_chunks(gdn, W, oracle_mod):
    # 38303 tokens over 8 bf16 channel tiles: the host picks 128-token chunks on a 148-SM
    # device, so every chunk after a request's first takes its look-back from x.  The conv is
    # depthwise, so the oracle runs on a sample of channels (both edges of every tile).
    lengths = [38000, 3, 300]
    c = W.make_conv1d(301, lengths, 8192, 4, 4)
    y, pool = run_gpu(gdn, c)
    cols = np.concatenate([np.arange(t * 1024, t * 1024 + 8) for t in range(8)] +
                          [np.arange(t * 1024 + 1016, t * 1024 + 1024) for t in range(8)])
    sub = W.Conv1dCase(name="sample", x=c.x[:, cols].contiguous(), weight=c.weight[cols],
                       conv_state=c.conv_state[:, cols].contiguous(), slot_idx=c.slot_idx,
                       row_offsets=c.row_offsets)
    ref, ref_pool = run_oracle(oracle_mod, sub)
    check_outputs(y[:, cols], ref, magnitude(oracle_mod, sub), torch.bfloat16, 4)
    np.testing.assert_array_equal(f64(pool[:, cols]), ref_pool)


def test_full_size_ragged(gdn, W, oracle_mod):
    # the benchmarked ragged workload, every output and slot compared
    c = W.conv_ragged_case()
    y, pool = run_gpu(gdn, c)
    ref, ref_pool = run_oracle(oracle_mod, c)
    check_outputs(y, ref, magnitude(oracle_mod, c), torch.bfloat16, 4)
    check_pool(pool, ref_pool, c)


def test_full_size_decode_step(gdn, W, oracle_mod):
    c = W.conv_decode_case()
    y, pool = run_gpu(gdn, c)
    ref, ref_pool = run_oracle(oracle_mod, c)
    check_outputs(y, ref, magnitude(oracle_mod, c), torch.bfloat16, 4)
    check_pool(pool, ref_pool, c)


def test_read_only_leaves_pool(gdn, W, oracle_mod):
    c = W.make_conv1d(401, [5, 1, 70], 2048, 4, 6)
    pool = dev(c.conv_state)
    before = pool.clone()
    y, _ = run_gpu(gdn, c, pool=pool, write_state=False)
    assert torch.equal(pool, before)
    ref, _ = run_oracle(oracle_mod, c, write_state=False)
    check_outputs(y, ref, magnitude(oracle_mod, c), torch.bfloat16, 4)


def test_continuation_matches_single_call(gdn, W):
    # one request split over two calls on the same slot equals one call (property of the
    # window semantics; the split points include pieces shorter than K-1)
    c = W.make_conv1d(501, [300], 4096, 4, 3)
    y_one, p_one = run_gpu(gdn, c)
    for split in (1, 2, 150):
        pool = dev(c.conv_state)
        outs = []
        for lo, hi in ((0, split), (split, 300)):
            ci = W.Conv1dCase(name="piece", x=c.x[lo:hi].contiguous(), weight=c.weight,
                              conv_state=c.conv_state, slot_idx=c.slot_idx,
                              row_offsets=torch.tensor([0, hi - lo], dtype=torch.uint32))
            y, _ = run_gpu(gdn, ci, pool=pool)
            outs.append(y)
        assert torch.equal(torch.cat(outs), y_one)
        assert torch.equal(pool.cpu(), p_one)


def test_bad_slot_is_skipped_and_flagged(gdn, W, oracle_mod):
    c = W.make_conv1d(601, [4, 6, 3], 1024, 4, 4)
    c.slot_idx = torch.tensor([1, 9, 2], dtype=torch.uint32)   # 9 >= max_slots
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    keep = torch.full_like(c.x, -2.0)
    y, pool = run_gpu(gdn, c, out=keep, dev_status=status)
    assert int(status.item()) == gdn.GDN_DEV_BAD_SLOT
    ref, ref_pool = run_oracle(oracle_mod, c, out=keep)
    assert (y[4:10] == -2.0).all()
    check_outputs(y, ref, magnitude(oracle_mod, c), torch.bfloat16, 4)
    check_pool(pool, ref_pool, c)


def test_offsets_clamped_and_empty(gdn, W, oracle_mod):
    c = W.make_conv1d(701, [10, 10], 1024, 4, 4)
    c.row_offsets = torch.tensor([0, 10, 4000], dtype=torch.uint32)   # past N: clamped to N
    y, pool = run_gpu(gdn, c)
    ref, ref_pool = run_oracle(oracle_mod, c)
    check_outputs(y, ref, magnitude(oracle_mod, c), torch.bfloat16, 4)
    check_pool(pool, ref_pool, c)
    # every request empty: nothing written at all
    e = W.make_conv1d(702, [0, 0, 0], 1024, 4, 4, N=16)
    keep = torch.full_like(e.x, 5.0)
    pool = dev(e.conv_state)
    before = pool.clone()
    y, _ = run_gpu(gdn, e, pool=pool, out=keep)
    assert (y == 5.0).all() and torch.equal(pool, before)
