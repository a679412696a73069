"""GPU parity of gdn_decode against the float64 oracle (through the C ABI).

Tolerance: relative L2 <= 2e-2 (bf16 activations, fp32 state) on outputs and on
every written pool slot; pool slots nobody writes must stay bit-identical.
"""
import copy

import numpy as np
import pytest
import torch

from _util import TOL_BF16, assert_out_close, assert_states_close, dev, f64

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


def run_gpu(gdn, c, pool_dev=None, out=None, dev_status=None, disable=None):
    pool = dev(c.pool) if pool_dev is None else pool_dev
    o, _ = gdn.gdn_decode(dev(c.q), dev(c.k), dev(c.v), pool, dev(c.read_idx), dev(c.A_log),
                          dev(c.a), dev(c.dt_bias), dev(c.b), scale=c.scale,
                          out=None if out is None else dev(out),
                          scatter_idx=dev(c.scatter_idx),
                          disable_state_update=c.disable_state_update if disable is None
                          else disable,
                          use_qk_l2norm=c.use_qk_l2norm, write_idx=dev(c.write_idx),
                          dev_status=dev_status)
    torch.cuda.synchronize()
    return o, pool


def run_oracle(oracle_mod, c, rows=None, out=None):
    """Oracle on all rows, or on a subset `rows` through a compact pool holding only their
    read slots (returns outputs of those rows and the final per-row states)."""
    if rows is None:
        return oracle_mod.decode(f64(c.q), f64(c.k), f64(c.v), f64(c.pool), c.read_idx.numpy(),
                                 f64(c.A_log), f64(c.a), f64(c.dt_bias), f64(c.b),
                                 write_idx=None if c.write_idx is None else c.write_idx.numpy(),
                                 scatter_idx=None if c.scatter_idx is None
                                 else c.scatter_idx.numpy(),
                                 scale=c.scale, use_qk_l2norm=c.use_qk_l2norm,
                                 disable_state_update=c.disable_state_update,
                                 out=None if out is None else f64(out))
    rows = np.asarray(rows)
    reads = c.read_idx.numpy()[rows]
    assert (reads >= 0).all()
    small = f64(c.pool[torch.from_numpy(reads.astype(np.int64))])
    return oracle_mod.decode(f64(c.q[rows]), f64(c.k[rows]), f64(c.v[rows]), small,
                             np.arange(len(rows), dtype=np.int32), f64(c.A_log),
                             f64(c.a[rows]), f64(c.dt_bias), f64(c.b[rows]), scale=c.scale,
                             use_qk_l2norm=c.use_qk_l2norm)


def small_case(W, seed, **kw):
    base = dict(P=64, B=12, T=1, nh=1, H=4, Dv=128, pad_frac=0.25)
    base.update(kw)
    return W.make_decode(seed, **base)


@pytest.mark.parametrize("Dv", [64, 128])
@pytest.mark.parametrize("write_mode", ["distinct", "same", "none"])
def test_small_decode(gdn, W, oracle_mod, Dv, write_mode):
    c = small_case(W, 100 + Dv, Dv=Dv, write_mode=write_mode)
    sentinel = torch.full((12, 1, 4, Dv), -2.0, dtype=torch.bfloat16)
    o, pool = run_gpu(gdn, c, out=sentinel)
    ro, rp = run_oracle(oracle_mod, c, out=sentinel)
    assert_out_close(f64(o), ro, TOL_BF16)
    pad = (c.read_idx < 0).numpy()
    assert pad.any()
    assert torch.equal(o.cpu()[torch.from_numpy(pad)], sentinel[torch.from_numpy(pad)])
    written = set(c.read_idx[~torch.from_numpy(pad)].tolist()) if c.write_idx is None else \
        set(w for w in c.write_idx.tolist() if w >= 0)
    pc = pool.cpu()
    for s in range(c.pool.shape[0]):
        if s in written:
            assert_states_close(f64(pc[s:s + 1]), rp[s:s + 1], TOL_BF16, f"slot {s}")
        else:
            assert torch.equal(pc[s], c.pool[s]), s


@pytest.mark.parametrize("T,nh", [(2, 1), (4, 2), (3, 3), (16, 4), (1, 4)])
def test_multi_token_and_householder(gdn, W, oracle_mod, T, nh):
    c = small_case(W, 200 + 10 * T + nh, T=T, nh=nh, Dv=64, pad_frac=0.1)
    o, pool = run_gpu(gdn, c)
    ro, rp = run_oracle(oracle_mod, c)
    assert_out_close(f64(o), ro, TOL_BF16)
    assert_states_close(f64(pool.cpu()), rp, TOL_BF16)


def test_scatter_with_negative_entries(gdn, W, oracle_mod):
    c = small_case(W, 300, T=4, nh=2, Dv=64, write_mode="distinct", scatter=True, P=128)
    c.scatter_idx[0, 1] = -1
    c.scatter_idx[3, 0] = -5
    o, pool = run_gpu(gdn, c)
    ro, rp = run_oracle(oracle_mod, c)
    assert_out_close(f64(o), ro, TOL_BF16)
    pc = pool.cpu()
    sc = set(int(x) for x, r in zip(c.scatter_idx.flatten().tolist(),
                                    np.repeat(c.read_idx.numpy(), 4)) if x >= 0 and r >= 0)
    for s in range(128):
        if s in sc:
            assert_states_close(f64(pc[s:s + 1]), rp[s:s + 1], TOL_BF16, f"slot {s}")
        else:  # includes the write slots: scatter skips the end write-back
            assert torch.equal(pc[s], c.pool[s]), s


def test_disable_state_update(gdn, W, oracle_mod):
    c = small_case(W, 400, T=3, nh=2, Dv=128)
    c.disable_state_update = True
    o, pool = run_gpu(gdn, c)
    ro, _ = run_oracle(oracle_mod, c)
    assert_out_close(f64(o), ro, TOL_BF16)
    assert torch.equal(pool.cpu(), c.pool)


def test_bad_slot_sets_status_and_skips(gdn, W, oracle_mod):
    c = small_case(W, 500, pad_frac=0.0, write_mode="distinct")
    c.read_idx[2] = 1000        # beyond the pool: row skipped, flagged
    c.write_idx[5] = 64         # beyond the pool: write-back skipped, flagged
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    sentinel = torch.full((12, 1, 4, 128), 5.0, dtype=torch.bfloat16)
    o, pool = run_gpu(gdn, c, out=sentinel, dev_status=status)
    assert int(status.item()) == 1
    assert torch.equal(o[2].cpu(), sentinel[2])
    ok_rows = [r for r in range(12) if r != 2]
    ro, rp = run_oracle(oracle_mod, c, rows=ok_rows)
    assert_out_close(f64(o.cpu()[ok_rows]), ro, TOL_BF16)
    pc = pool.cpu()
    for i, r in enumerate(ok_rows):
        w = int(c.write_idx[r])
        if w < 64:
            assert_states_close(f64(pc[w:w + 1]), rp[i:i + 1], TOL_BF16, f"slot {w}")
    untouched = set(range(64)) - set(int(w) for w in c.write_idx.tolist() if w < 64)
    for s in untouched:
        if s != int(c.write_idx[2]):
            assert torch.equal(pc[s], c.pool[s])


def test_padded_pool_strides(gdn, W, oracle_mod):
    """A pool with padding between heads and slots (dense rows) is used in place."""
    c = small_case(W, 600, Dv=64, write_mode="same")
    P, HV, Dv, Dk = c.pool.shape
    big = torch.full((P, HV + 1, Dv + 4, Dk), 9.0, dtype=torch.float32, device="cuda")
    view = big[:, :HV, :Dv, :]
    view.copy_(dev(c.pool))
    assert not view.is_contiguous()
    o, _ = run_gpu(gdn, c, pool_dev=view)
    ro, rp = run_oracle(oracle_mod, c)
    assert_out_close(f64(o), ro, TOL_BF16)
    assert_states_close(f64(view.cpu()), rp, TOL_BF16)
    assert (big[:, HV] == 9.0).all() and (big[:, :, Dv:] == 9.0).all()


def test_deterministic(gdn, W):
    c = small_case(W, 700, T=4, nh=2, Dv=128, write_mode="distinct")
    outs = []
    for _ in range(3):
        o, pool = run_gpu(gdn, c)
        outs.append((o.clone(), pool.clone()))
    for o, p in outs[1:]:
        assert torch.equal(o, outs[0][0]) and torch.equal(p, outs[0][1])


# ---------------------------------------------------------------- full sizes
@pytest.mark.parametrize("write_mode", ["distinct", "same"])
def test_full_decode_pool(gdn, W, oracle_mod, write_mode):
    """Pool [1024, 32, 128, 128] (2 GiB), B=256 with 13 padding rows, write slots distinct from
    the read slots or equal to them, in the launch configuration the benchmark times: every one
    of the 243 live rows against the oracle (outputs per (row, head), written states per
    (slot, head), in batches of rows through compact pools of their read slots), every padding
    row and every slot outside the write set bit-identical."""
    c = W.decode_pool_case(write_mode=write_mode)
    pool = dev(c.pool)
    o, _ = run_gpu(gdn, c, pool_dev=pool)
    reads = c.read_idx.numpy()
    live = np.nonzero(reads >= 0)[0]
    assert len(live) == 243
    oc = o.cpu()
    for r0 in range(0, len(live), 64):
        rows = live[r0:r0 + 64]
        ro, rp = run_oracle(oracle_mod, c, rows=rows)
        assert_out_close(f64(oc[torch.from_numpy(rows)]), ro, TOL_BF16, "out")
        wr = torch.from_numpy(c.write_idx.numpy()[rows].astype(np.int64)).cuda()
        assert_states_close(f64(pool.index_select(0, wr).cpu()), rp, TOL_BF16, "write slot")
    pad = np.nonzero(reads < 0)[0]
    assert len(pad) == 13
    assert (oc[torch.from_numpy(pad)] == 0).all()
    written = set(int(w) for w in c.write_idx.tolist() if w >= 0)
    untouched = [s for s in range(1024) if s not in written]
    idx = torch.tensor(untouched, device="cuda")
    assert torch.equal(pool.index_select(0, idx).cpu(), c.pool[torch.tensor(untouched)])
    assert torch.isfinite(o.float()).all()


def test_full_mtp(gdn, W, oracle_mod):
    """B=64, T=4, nh=2, H=16, Dv=64, per-token scatter into 256 distinct slots: every output
    and every scattered slot against the oracle."""
    c = W.mtp_case()
    o, pool = run_gpu(gdn, c)
    ro, rp = run_oracle(oracle_mod, c)
    assert_out_close(f64(o), ro, TOL_BF16)
    pc = pool.cpu()
    sc = c.scatter_idx.flatten().tolist()
    assert_states_close(f64(pc[sc]), rp[sc], TOL_BF16)
    others = [s for s in range(512) if s not in set(sc)]
    assert torch.equal(pc[others], c.pool[others])


def test_int64_slot_indices(gdn, W):
    """int64 read/write slots (the page allows int32 or int64) give the same bytes as int32,
    padding rows included; an int64 slot beyond int32 range is out of the pool: skipped and
    flagged."""
    c = small_case(W, 800, T=2, nh=2, Dv=128, pad_frac=0.25, write_mode="distinct")
    o32, p32 = run_gpu(gdn, c)
    c64 = copy.copy(c)
    c64.read_idx = c.read_idx.to(torch.int64)
    c64.write_idx = c.write_idx.to(torch.int64)
    o64, p64 = run_gpu(gdn, c64)
    assert torch.equal(o32, o64) and torch.equal(p32, p64)
    big = copy.copy(c64)
    big.read_idx = c64.read_idx.clone()
    live = int((c64.read_idx >= 0).nonzero()[0])
    big.read_idx[live] = (1 << 33) + int(c64.read_idx[live])
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ob, pb = run_gpu(gdn, big, dev_status=status)
    assert int(status.item()) == gdn.GDN_DEV_BAD_SLOT
    keep = [r for r in range(c.read_idx.shape[0]) if r != live]
    assert torch.equal(ob[keep], o32[keep])


# ---------------------------------------------------------------- launch forms
def sub_case(c, rows):
    """The rows `rows` of decode case c as a case of their own (same pool)."""
    s = copy.copy(c)
    for name in ("q", "k", "v", "a", "b", "read_idx", "write_idx", "scatter_idx"):
        t = getattr(c, name)
        if t is not None:
            setattr(s, name, t[rows].contiguous())
    return s


@pytest.mark.parametrize("Dv", [64, 128])
def test_launch_forms_agree(gdn, W, oracle_mod, Dv):
    """Single-token rows that fill many waves of CTAs take the one-CTA-per-(row, head) form; the
    same rows called 8 at a time take the persistent form.  Both run the same per-unit
    arithmetic, so outputs and the pool agree bit for bit, padding rows, a read slot beyond the
    pool and a write slot beyond the pool included; sampled rows match the oracle."""
    B, P = 160, 352
    c = W.make_decode(900 + Dv, P=P, B=B, T=1, nh=1, H=32, Dv=Dv, pad_frac=0.1,
                      write_mode="distinct")
    reads = c.read_idx.numpy()
    live = np.nonzero(reads >= 0)[0]
    c.read_idx[int(live[3])] = P + 5
    c.write_idx[int(live[7])] = P + 7
    sentinel = torch.full((B, 1, 32, Dv), 3.0, dtype=torch.bfloat16)

    status_all = torch.zeros(1, dtype=torch.int32, device="cuda")
    pool_all = dev(c.pool)
    o_all, _ = run_gpu(gdn, c, pool_dev=pool_all, out=sentinel, dev_status=status_all)

    status_8 = torch.zeros(1, dtype=torch.int32, device="cuda")
    pool_8 = dev(c.pool)
    o_8 = []
    for r0 in range(0, B, 8):
        sc = sub_case(c, slice(r0, r0 + 8))
        o, _ = run_gpu(gdn, sc, pool_dev=pool_8, out=sentinel[r0:r0 + 8], dev_status=status_8)
        o_8.append(o)
    o_8 = torch.cat(o_8)
    assert int(status_all.item()) == gdn.GDN_DEV_BAD_SLOT == int(status_8.item())
    assert torch.equal(o_all, o_8)
    assert torch.equal(pool_all, pool_8)

    ok = [int(r) for r in live if r not in (live[3], live[7])]
    rows = np.sort(np.random.default_rng(1).choice(ok, 12, replace=False))
    ro, rp = run_oracle(oracle_mod, c, rows=rows)
    oc = o_all.cpu()
    assert_out_close(f64(oc[torch.from_numpy(rows)]), ro, TOL_BF16)
    for i, r in enumerate(rows):
        w = int(c.write_idx[r])
        assert_states_close(f64(pool_all[w:w + 1].cpu()), rp[i:i + 1], TOL_BF16, f"slot {w}")
    skipped = np.nonzero(c.read_idx.numpy() < 0)[0].tolist() + [int(live[3])]
    assert torch.equal(oc[skipped], sentinel[skipped])


def test_stream_form_walks_many_units(gdn, W, oracle_mod):
    """Persistent form with several (row, head) units per CTA: padding rows, a read slot beyond
    the pool and scatter entries of -1 interleaved with live units; every output and pool slot
    against the oracle."""
    B, P = 64, 200
    c = W.make_decode(950, P=P, B=B, T=2, nh=2, H=32, Dv=64, pad_frac=0.2,
                      write_mode="none", scatter=True)
    live = np.nonzero(c.read_idx.numpy() >= 0)[0]
    c.scatter_idx[int(live[0]), 1] = -1
    c.scatter_idx[int(live[5]), 0] = -1
    bad = int(live[9])
    c.read_idx[bad] = P + 1
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    sentinel = torch.full((B, 2, 32, 64), -4.0, dtype=torch.bfloat16)
    o, pool = run_gpu(gdn, c, out=sentinel, dev_status=status)
    assert int(status.item()) == gdn.GDN_DEV_BAD_SLOT
    ok = [r for r in range(B) if r != bad]
    good = sub_case(c, ok)
    ro, rp = run_oracle(oracle_mod, good, out=sentinel[ok])
    assert_out_close(f64(o.cpu()[ok]), ro, TOL_BF16)
    pc = pool.cpu()
    sc = set(int(x) for r in ok if c.read_idx[r] >= 0 for x in c.scatter_idx[r].tolist() if x >= 0)
    for s in range(P):
        if s in sc:
            assert_states_close(f64(pc[s:s + 1]), rp[s:s + 1], TOL_BF16, f"slot {s}")
        else:
            assert torch.equal(pc[s], c.pool[s]), s
    assert torch.equal(o.cpu()[bad], sentinel[bad])


@pytest.mark.parametrize("B", [12, 96])   # persistent form; one-CTA form (8 rows per lane)
def test_output_only_8_byte_aligned(gdn, W, oracle_mod, B):
    """The ABI asks for an 8-byte aligned `out`: an output that starts 8 bytes past a 16-byte
    boundary gets the same bytes as an aligned one, from both launch forms."""
    c = W.make_decode(1000 + B, P=2 * B + 16, B=B, T=1, nh=1, H=32, Dv=128, pad_frac=0.1,
                      write_mode="distinct")
    aligned, _ = run_gpu(gdn, c)
    buf = torch.full((B * 32 * 128 + 4,), 7.0, dtype=torch.bfloat16, device="cuda")
    out = buf[4:].view(B, 1, 32, 128)
    assert out.data_ptr() % 16 == 8
    pool = dev(c.pool)
    o, _ = gdn.gdn_decode(dev(c.q), dev(c.k), dev(c.v), pool, dev(c.read_idx), dev(c.A_log),
                          dev(c.a), dev(c.dt_bias), dev(c.b), scale=c.scale, out=out,
                          use_qk_l2norm=c.use_qk_l2norm, write_idx=dev(c.write_idx))
    torch.cuda.synchronize()
    live = (c.read_idx >= 0).cuda()
    assert torch.equal(o[live], aligned.cuda()[live])
    assert (buf[:4] == 7.0).all()
    rows = np.nonzero(c.read_idx.numpy() >= 0)[0][:6]
    ro, _ = run_oracle(oracle_mod, c, rows=rows)
    assert_out_close(f64(o.cpu()[torch.from_numpy(rows)]), ro, TOL_BF16)


def test_decode_equals_prefill_with_host_gate(gdn, W):
    """nh = 1 decode over 16 tokens equals the tensor-core prefill of the same tokens with
    g = -exp(A_log) softplus20(a + dt_bias) and beta = sigmoid(b) evaluated on the host; q and k
    are unit rows and both in-kernel norms are off (their epsilons differ)."""
    B, T, H, Dv = 4, 16, 4, 128
    c = W.make_decode(1200, P=8, B=B, T=T, nh=1, H=H, Dv=Dv, write_mode="none",
                      host_norm_qk=True, use_qk_l2norm=False)
    reads = c.read_idx.to(torch.int64)
    init = c.pool[reads].clone()   # the prefill's initial states, before the pool is updated
    pool = dev(c.pool)
    od, _ = gdn.gdn_decode(dev(c.q), dev(c.k), dev(c.v), pool, dev(c.read_idx), dev(c.A_log),
                           dev(c.a), dev(c.dt_bias), dev(c.b), scale=c.scale,
                           use_qk_l2norm=False)
    torch.cuda.synchronize()
    x = c.a.double() + c.dt_bias.double()[None, None, :]
    sp = torch.where(x > 20, x, torch.log1p(torch.exp(x)))
    g = (-torch.exp(c.A_log.double())[None, None, :] * sp).float().reshape(B * T, H)
    beta = torch.sigmoid(c.b[:, :, 0].double()).float().reshape(B * T, H)
    op, fp = gdn.gdn_prefill(dev(c.q.reshape(B * T, H, 128)), dev(c.k[:, :, 0].reshape(B * T, H, 128)),
                             dev(c.v[:, :, 0].reshape(B * T, H, Dv)), dev(g), dev(beta),
                             dev(torch.arange(0, B * T + 1, T, dtype=torch.int32)),
                             dev(init), scale=c.scale, qk_l2norm=False)
    torch.cuda.synchronize()
    assert gdn.prefill_uses_chunked(torch.bfloat16, H, 128, Dv)
    assert_out_close(f64(od), f64(op.reshape(B, T, H, Dv)), TOL_BF16)
    assert_states_close(f64(pool[reads.cuda()]), f64(fp), TOL_BF16)
