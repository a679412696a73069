"""GPU parity of gdn_prefill against the float64 oracle (through the C ABI).

Tolerances (relative L2): 1e-4 for fp32 activations, 2e-2 for bf16 activations
with the fp32 state, applied to the whole tensor, to every (request, value head)
block of outputs and final states, and to every output row (see
_util.assert_prefill_parity).
"""
import json
import os

import numpy as np
import pytest
import torch

from _util import (TOL_BF16, TOL_F32, assert_prefill_parity, dev, f64, oracle_prefill_case,
                   request_ranges, run_gpu_prefill)

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "p1_worked_examples.json")


@pytest.fixture(scope="module")
def gdn():
    import gated_deltanet_state_gdn_b200 as g
    g.lib()
    return g


@pytest.fixture(scope="module")
def W():
    from gated_deltanet_state_gdn_b200 import workloads
    return workloads


@pytest.mark.parametrize("sequential", [True, False])
def test_worked_examples(gdn, sequential):
    for e in json.load(open(GOLDEN))["examples"]:
        q = torch.tensor(e["q"], dtype=torch.float32)
        B, S, Dk = q.shape
        k = torch.tensor(e["k"], dtype=torch.float32)
        v = torch.tensor(e["v"], dtype=torch.float32)
        Dv = v.shape[2]
        g = torch.log(torch.tensor(e["gamma"], dtype=torch.float32)).reshape(B * S, 1)
        beta = torch.tensor(e["beta"], dtype=torch.float32).reshape(B * S, 1)
        out, fs = gdn.gdn_prefill(dev(q.reshape(B * S, 1, Dk)), dev(k.reshape(B * S, 1, Dk)),
                                  dev(v.reshape(B * S, 1, Dv)), dev(g), dev(beta),
                                  num_requests=B, scale=1.0, sequential=sequential)
        torch.cuda.synchronize()
        np.testing.assert_allclose(f64(out).reshape(B, S, Dv), np.array(e["outputs"]),
                                   atol=1e-5)
        np.testing.assert_allclose(f64(fs)[:, 0].transpose(0, 2, 1),
                                   np.array(e["final_state"]), atol=1e-5)


def test_tiny_oracle_case_fp32(gdn, W, oracle_mod):
    c = W.tiny_oracle_case()
    out, fs = run_gpu_prefill(c)
    ro, rf = oracle_prefill_case(oracle_mod, c)
    assert_prefill_parity(out, fs, ro, rf, request_ranges(c.cu_seqlens, c.B, c.N), TOL_F32)


@pytest.mark.parametrize("dtype,tol", [(torch.float32, TOL_F32), (torch.bfloat16, TOL_BF16)])
def test_odd_head_sizes_gqa(gdn, W, oracle_mod, dtype, tol):
    """The op page's example call shape: T=4, Hq=1, Hv=2, Dk=12, Dv=9, with an initial state;
    bf16 runs it on the tensor cores (plain-staged zero-padded tiles), fp32 on the per-token
    kernel."""
    assert gdn.prefill_uses_chunked(dtype, 2, 12, 9) == (dtype == torch.bfloat16)
    c = W.make_prefill(11, [4], 1, 2, 12, 9, dtype=dtype, uniform=True, init_std=0.5,
                       qk_l2norm=True)
    out, fs = run_gpu_prefill(c)
    ro, rf = oracle_prefill_case(oracle_mod, c)
    assert_prefill_parity(out, fs, ro, rf, request_ranges(c.cu_seqlens, c.B, c.N), tol)


@pytest.mark.parametrize("Dk,Dv", [(1, 1), (33, 7), (256, 256), (128, 40)])
def test_head_size_range_fp32(gdn, W, oracle_mod, Dk, Dv):
    c = W.make_prefill(12 + Dk, [3, 17, 0, 9], 2, 4, Dk, Dv, dtype=torch.float32, init_std=0.3,
                       qk_l2norm=True)
    out, fs = run_gpu_prefill(c)
    ro, rf = oracle_prefill_case(oracle_mod, c)
    assert_prefill_parity(out, fs, ro, rf, request_ranges(c.cu_seqlens, c.B, c.N), TOL_F32)


RAGGED = [1, 64, 65, 130, 0, 200, 63, 128]


@pytest.mark.parametrize("sequential", [True, False])
@pytest.mark.parametrize("l2norm", [True, False])
def test_ragged_bf16_d128(gdn, W, oracle_mod, sequential, l2norm):
    """Several 64-token chunks per request, ragged tails, an empty request, GQA 2 -> 4."""
    c = W.make_prefill(21 + int(l2norm), RAGGED, 2, 4, 128, 128, init_std=0.02,
                       qk_l2norm=l2norm, host_norm_qk=not l2norm)
    out, fs = run_gpu_prefill(c, sequential=sequential)
    ro, rf = oracle_prefill_case(oracle_mod, c)
    assert_prefill_parity(out, fs, ro, rf, request_ranges(c.cu_seqlens, c.B, c.N), TOL_BF16)
    # the empty request copies its initial state through bit for bit
    assert torch.equal(fs[4].cpu(), c.initial_state[4])


@pytest.mark.parametrize("sequential", [True, False])
def test_cu_seqlens_clamp_and_uncovered_tokens(gdn, W, oracle_mod, sequential):
    c = W.make_prefill(31, [40, 30, 40, 20, 10], 1, 4, 128, 128, init_std=0.1, qk_l2norm=True)
    N = c.N  # 140
    sentinel = torch.full((N, 4, 128), 3.0, dtype=torch.bfloat16)
    # (a) tokens 0..9 and N-20..N-1 belong to no request and keep the caller's values;
    #     request 1 is empty, request 4 is decreasing (empty)
    c.cu_seqlens = torch.tensor([10, 40, 40, 60, N - 20, 3], dtype=torch.int32)
    out, fs = run_gpu_prefill(c, sequential=sequential, out=sentinel)
    ro, rf = oracle_prefill_case(oracle_mod, c, out=f64(sentinel))
    assert_prefill_parity(out, fs, ro, rf, request_ranges(c.cu_seqlens, c.B, N), TOL_BF16)
    assert torch.equal(out[:10].cpu(), sentinel[:10])
    assert torch.equal(out[N - 20:].cpu(), sentinel[N - 20:])
    assert torch.equal(fs[1].cpu(), c.initial_state[1])
    assert torch.equal(fs[4].cpu(), c.initial_state[4])
    # (b) out-of-range entries clamp to [0, N]; request 1 decreasing -> empty
    c.cu_seqlens = torch.tensor([-9, 40, 30, N + 500], dtype=torch.int32)
    c.initial_state = c.initial_state[:3].contiguous()
    c.B = 3
    out, fs = run_gpu_prefill(c, sequential=sequential, out=sentinel)
    ro, rf = oracle_prefill_case(oracle_mod, c, out=f64(sentinel))
    keep = np.ones(N, bool)
    keep[30:40] = False  # tokens 30..39 lie in two requests: undefined outputs
    assert_prefill_parity(out, fs, ro, rf, request_ranges(c.cu_seqlens, c.B, N), TOL_BF16,
                          token_mask=keep)
    assert torch.equal(fs[1].cpu(), c.initial_state[1])


@pytest.mark.parametrize("sequential", [True, False])
def test_zero_gate_and_zero_initial_state(gdn, W, oracle_mod, sequential):
    """gamma = 0 (g = -inf) wipes the state; no initial state means zero."""
    c = W.make_prefill(41, [70, 130], 1, 4, 128, 128, init_std=None, qk_l2norm=True)
    c.g[5] = float("-inf")
    c.g[100] = float("-inf")
    c.g[101:110] = 0.0
    out, fs = run_gpu_prefill(c, sequential=sequential)
    ro, rf = oracle_prefill_case(oracle_mod, c)
    assert np.isfinite(f64(out)).all() and np.isfinite(f64(fs)).all()
    assert_prefill_parity(out, fs, ro, rf, request_ranges(c.cu_seqlens, c.B, c.N), TOL_BF16)


def test_noncontiguous_inputs_and_inputs_unchanged(gdn, W, oracle_mod):
    c = W.make_prefill(51, [33, 70], 2, 4, 128, 128, init_std=0.1, qk_l2norm=True)
    qd = dev(c.q).transpose(0, 1).contiguous().transpose(0, 1)   # same values, other strides
    assert not qd.is_contiguous()
    kd, vd, gd, bd = dev(c.k), dev(c.v), dev(c.g), dev(c.beta)
    init = dev(c.initial_state)
    snap = [t.clone() for t in (qd, kd, vd, gd, bd, init)]
    out, fs = gdn.gdn_prefill(qd, kd, vd, gd, bd, dev(c.cu_seqlens), init, scale=c.scale,
                              qk_l2norm=True)
    torch.cuda.synchronize()
    for a, b in zip(snap, (qd, kd, vd, gd, bd, init)):
        assert torch.equal(a, b)
    ro, rf = oracle_prefill_case(oracle_mod, c)
    assert_prefill_parity(out, fs, ro, rf, request_ranges(c.cu_seqlens, c.B, c.N), TOL_BF16)


@pytest.mark.parametrize("per_key", [False, True])
@pytest.mark.parametrize("sequential", [True, False])
def test_deterministic(gdn, W, sequential, per_key):
    """Three calls on the same bytes give the same bytes (a race would show as a difference):
    the scalar-decay chunked kernel, the per-key-decay chunked kernel and the per-token kernel."""
    c = W.make_prefill(61, [300, 77], 2, 4, 128, 128, init_std=0.02, qk_l2norm=True,
                       decay_per_key=per_key)
    runs = [run_gpu_prefill(c, sequential=sequential) for _ in range(3)]
    for o, f in runs[1:]:
        assert torch.equal(o, runs[0][0]) and torch.equal(f, runs[0][1])


def test_rank4_spelling(gdn, W, oracle_mod):
    c = W.make_prefill(71, [50, 50], 1, 4, 128, 128, uniform=True, init_std=0.1,
                       qk_l2norm=True)
    q4 = dev(c.q).reshape(2, 50, 1, 128)
    k4 = dev(c.k).reshape(2, 50, 1, 128)
    v4 = dev(c.v).reshape(2, 50, 4, 128)
    out, fs = gdn.gdn_prefill(q4, k4, v4, dev(c.g).reshape(2, 50, 4),
                              dev(c.beta).reshape(2, 50, 4), None, dev(c.initial_state),
                              scale=c.scale, qk_l2norm=True)
    torch.cuda.synchronize()
    ro, rf = oracle_prefill_case(oracle_mod, c)
    assert_prefill_parity(out, fs, ro, rf, request_ranges(c.cu_seqlens, c.B, c.N), TOL_BF16)


def test_chunked_path_is_selected(gdn):
    assert gdn.prefill_uses_chunked(torch.bfloat16, 4, 128, 128)
    assert gdn.prefill_uses_chunked(torch.bfloat16, 32, 128, 128)
    assert not gdn.prefill_uses_chunked(torch.bfloat16, 32, 128, 128, sequential=True)
    assert not gdn.prefill_uses_chunked(torch.float32, 32, 128, 128)
    assert gdn.prefill_uses_chunked(torch.bfloat16, 2, 128, 128)       # plain-staged gates
    assert gdn.prefill_uses_chunked(torch.bfloat16, 32, 64, 128)
    assert gdn.prefill_uses_chunked(torch.bfloat16, 32, 8, 8)
    assert gdn.prefill_uses_chunked(torch.bfloat16, 32, 60, 128)       # plain-staged rows
    assert gdn.prefill_uses_chunked(torch.bfloat16, 2, 12, 9)          # the op page's example
    assert gdn.prefill_uses_chunked(torch.float16, 3, 1, 1)
    assert not gdn.prefill_uses_chunked(torch.bfloat16, 32, 128, 136)  # wider than 128
    assert not gdn.prefill_uses_chunked(torch.bfloat16, 32, 256, 256)


@pytest.mark.parametrize("Hq,Hv,Dk,Dv", [(1, 2, 12, 9), (1, 3, 1, 1), (2, 6, 33, 7),
                                         (1, 2, 127, 100), (2, 4, 60, 128), (1, 1, 128, 128)])
def test_chunked_plain_staged_shapes(gdn, W, oracle_mod, Hq, Hv, Dk, Dv):
    """Head sizes that are not multiples of 8, and value-head counts that are not multiples of
    4, on the tensor-core kernel: their rows are copied into the zero-padded tiles by plain
    loads instead of tensor maps.  Ragged requests with an empty one, initial states, the
    in-kernel norm, tokens no request covers; every output and final state against the oracle,
    uncovered outputs untouched, no pipeline wait timed out."""
    assert gdn.prefill_uses_chunked(torch.bfloat16, Hv, Dk, Dv)
    c = W.make_prefill(700 + Dk + Dv + Hv, [70, 0, 1, 130, 64], Hq, Hv, Dk, Dv, init_std=0.1,
                       qk_l2norm=True)
    c.cu_seqlens = torch.tensor([0, 70, 70, 71, 201, c.N - 5], dtype=torch.int32)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    keep = torch.full((c.N, Hv, Dv), 7.0, dtype=torch.bfloat16)
    out, fs = gdn.gdn_prefill(dev(c.q), dev(c.k), dev(c.v), dev(c.g), dev(c.beta),
                              dev(c.cu_seqlens), dev(c.initial_state), None, dev(keep),
                              scale=c.scale, qk_l2norm=True, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ro, rf = oracle_prefill_case(oracle_mod, c, out=f64(keep))
    assert_prefill_parity(out, fs, ro, rf, request_ranges(c.cu_seqlens, c.B, c.N), TOL_BF16)
    assert torch.equal(out[c.N - 5:].cpu(), keep[c.N - 5:])
    assert torch.equal(fs[1].cpu(), c.initial_state[1])


@pytest.mark.parametrize("Dk,Dv", [(64, 64), (128, 64), (64, 128), (96, 32), (8, 8), (120, 128)])
def test_chunked_other_head_sizes(gdn, W, oracle_mod, Dk, Dv):
    """Heads narrower than 128 on the tensor-core kernel (zero-padded tiles): ragged requests
    with an empty one, initial states, the in-kernel norm; every output and final state against
    the oracle, and no pipeline wait timed out."""
    assert gdn.prefill_uses_chunked(torch.bfloat16, 4, Dk, Dv)
    c = W.make_prefill(500 + Dk + Dv, [70, 0, 1, 130, 64], 2, 4, Dk, Dv, init_std=0.1,
                       qk_l2norm=True)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    keep = torch.full((c.N, 4, Dv), 7.0, dtype=torch.bfloat16)
    out, fs = gdn.gdn_prefill(dev(c.q), dev(c.k), dev(c.v), dev(c.g), dev(c.beta),
                              dev(c.cu_seqlens), dev(c.initial_state), None, dev(keep),
                              scale=c.scale, qk_l2norm=True, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ro, rf = oracle_prefill_case(oracle_mod, c)
    assert_prefill_parity(out, fs, ro, rf, request_ranges(c.cu_seqlens, c.B, c.N), TOL_BF16)
    # the padded lanes and columns never reach memory: the final state of the empty request is
    # its initial state, byte for byte
    assert torch.equal(fs[1].cpu(), c.initial_state[1])


@pytest.mark.parametrize("lengths", [[1], [64], [65], [4096, 3, 700], [129, 0, 1, 191, 64]])
def test_chunked_equals_sequential(gdn, W, lengths):
    """The chunk form equals the token recurrence (same inputs, both GPU paths), and no
    pipeline wait of the chunked kernel ran out."""
    c = W.make_prefill(81 + len(lengths), lengths, 2, 8, 128, 128, init_std=0.05, qk_l2norm=True)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    oc, fc = gdn.gdn_prefill(dev(c.q), dev(c.k), dev(c.v), dev(c.g), dev(c.beta),
                             dev(c.cu_seqlens), dev(c.initial_state), scale=c.scale,
                             qk_l2norm=True, dev_status=status)
    os_, fs_ = run_gpu_prefill(c, sequential=True)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert_prefill_parity(oc, fc, f64(os_), f64(fs_), request_ranges(c.cu_seqlens, c.B, c.N),
                          TOL_BF16)


def test_norm_extremes_on_tensor_cores(gdn, W, oracle_mod):
    """In-kernel q/k normalisation with all-zero, tiny (x 1e-3) and large (x 100) rows.  A key
    row's norm comes from the Gram diagonal and its column scale rides in the T' tiles, so a zero
    key row puts a factor of about 1e6 on a column that only ever meets exact zeros; a zero query
    row reads out zero."""
    c = W.make_prefill(97, [150, 64, 33], 2, 4, 128, 128, init_std=0.02, qk_l2norm=True)
    assert gdn.prefill_uses_chunked(c.q.dtype, 4, 128, 128)
    k = c.k.float()
    q = c.q.float()
    idx = torch.from_numpy(np.random.default_rng(5).permutation(k.shape[0]))
    k[idx[:12]] = 0.0
    k[idx[12:24]] *= 1e-3
    k[idx[24:36]] *= 100.0
    q[idx[36:48]] = 0.0
    q[idx[48:60]] *= 1e-3
    c.k = k.to(c.k.dtype)
    c.q = q.to(c.q.dtype)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, fs = gdn.gdn_prefill(dev(c.q), dev(c.k), dev(c.v), dev(c.g), dev(c.beta),
                              dev(c.cu_seqlens), dev(c.initial_state), scale=c.scale,
                              qk_l2norm=True, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.isfinite(out.float()).all() and torch.isfinite(fs).all()
    ro, rf = oracle_prefill_case(oracle_mod, c)
    assert_prefill_parity(out, fs, ro, rf, request_ranges(c.cu_seqlens, c.B, c.N), TOL_BF16)
    assert (out[idx[36:48].cuda()] == 0).all()


# ---------------------------------------------------------------- full sizes
def test_full_ragged_prefill_all_heads(gdn, W, oracle_mod):
    """8 requests U[1,4096], Hq=16, Hv=32, D=128, in the launch configuration the benchmark
    times: every output row and final state of all 32 value heads against the oracle, per
    (request, head) block and per row."""
    c = W.ragged_prefill_case()
    out, fs = run_gpu_prefill(c)
    ro, rf = oracle_prefill_case(oracle_mod, c)
    assert_prefill_parity(out, fs, ro, rf, request_ranges(c.cu_seqlens, c.B, c.N), TOL_BF16)


def test_full_long_prefill_all_heads(gdn, W, oracle_mod):
    """B=1, S=32768 (512 chunks of state carry per head): all 32768 x 32 output rows and all
    32 final states against the oracle, per head and per row."""
    c = W.long_prefill_case()
    out, fs = run_gpu_prefill(c)
    ro, rf = oracle_prefill_case(oracle_mod, c)
    assert_prefill_parity(out, fs, ro, rf, request_ranges(c.cu_seqlens, c.B, c.N), TOL_BF16)


@pytest.mark.parametrize("n", [64, 100])
@pytest.mark.parametrize("per_key", [False, True])
def test_split_and_resume_on_tensor_cores(gdn, W, n, per_key):
    """A request run as two calls, the second starting from the first's final state, equals one
    call (split on a chunk boundary and inside a chunk), on the scalar-decay and the
    per-key-decay chunked kernels."""
    import copy
    L = 230
    c = W.make_prefill(124, [L], 2, 4, 128, 128, init_std=0.02, qk_l2norm=True,
                       decay_per_key=per_key)
    assert gdn.prefill_uses_chunked(c.q.dtype, 4, 128, 128, decay_per_key=per_key)
    o_full, f_full = run_gpu_prefill(c)
    parts, init = [], c.initial_state
    for lo, hi in ((0, n), (n, L)):
        s = copy.copy(c)
        for name in ("q", "k", "v", "g", "beta"):
            setattr(s, name, getattr(c, name)[lo:hi].contiguous())
        s.cu_seqlens = torch.tensor([0, hi - lo], dtype=torch.int32)
        s.initial_state = init
        o, f = run_gpu_prefill(s)
        parts.append(o.cpu())
        init = f.cpu()
    assert_prefill_parity(torch.cat(parts), init, f64(o_full), f64(f_full), [(0, L)],
                          TOL_BF16)


def test_gate_views_off_a_16_byte_boundary(gdn, W, oracle_mod):
    """The chunked kernel reads g and beta through tensor maps, whose base must be 16-byte
    aligned: the C ABI refuses a g that starts 4 bytes past a boundary (GDN_ERR_ALIGN, before
    any launch), and the binding copies such a view into an aligned buffer, with the same
    results as aligned inputs."""
    import ctypes
    c = W.make_prefill(131, [70, 100], 2, 4, 128, 128, init_std=0.02, qk_l2norm=True)
    buf = torch.zeros(c.g.numel() + 1, dtype=torch.float32, device="cuda")
    gv = buf[1:].view(c.g.shape)
    gv.copy_(c.g.cuda())
    bbuf = torch.zeros(c.beta.numel() + 2, dtype=torch.float32, device="cuda")
    bv = bbuf[2:].view(c.beta.shape)
    bv.copy_(c.beta.cuda())
    assert gv.data_ptr() % 16 == 4 and bv.data_ptr() % 16 == 8
    q, k, v, cu, init = dev(c.q), dev(c.k), dev(c.v), dev(c.cu_seqlens), dev(c.initial_state)
    out = torch.empty((c.N, 4, 128), dtype=torch.bfloat16, device="cuda")
    fs = torch.empty((c.B, 4, 128, 128), dtype=torch.float32, device="cuda")
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    st = gdn.lib().gdn_prefill(p(q), p(k), p(v), p(gv), p(c.beta.cuda()), None, None, p(cu),
                               p(init), p(fs), p(out), c.B, c.N, 2, 4, 128, 128, gdn.GDN_BF16,
                               c.scale, 1, 0, None, None)
    assert st == gdn.GDN_ERR_ALIGN
    out, fs = gdn.gdn_prefill(q, k, v, gv, bv, cu, init, scale=c.scale, qk_l2norm=True)
    torch.cuda.synchronize()
    ro, rf = oracle_prefill_case(oracle_mod, c)
    assert_prefill_parity(out, fs, ro, rf, request_ranges(c.cu_seqlens, c.B, c.N), TOL_BF16)
