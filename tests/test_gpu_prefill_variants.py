"""GPU parity of the gdn_prefill variants against the float64 oracle (through the C ABI):
the update rules of "com.microsoft.GatedDeltaNet" (Attributes table: linear, gated, delta,
gated_delta), its qwen gate and sigmoid beta activations, and float16 activations.

Tolerances (relative L2, over the whole tensor, every (request, value head) block and every
output row as in _util.assert_prefill_parity): 2e-2 for bf16 activations with the fp32
state (as for the default rule). For fp16 activations on the per-token kernel 2e-3: its only
rounding against the oracle is the fp16 cast of the outputs (unit roundoff 2^-11 ~ 4.9e-4) on
top of the fp32 state arithmetic. For fp16 on the tensor-core kernel 2.5e-3: every MMA operand
(q, k, v and the T, P, -W, U and state tiles) is rounded to fp16, and the bf16 bound 2e-2 is about
five bf16 unit roundoffs (2^-8), so the same five fp16 unit roundoffs give 2.5e-3.
"""
import numpy as np
import pytest
import torch

from _util import TOL_BF16, assert_prefill_parity, dev, f64, request_ranges

pytestmark = pytest.mark.gpu

TOL_F16 = 2e-3
TOL_F16_CHUNKED = 2.5e-3
RULES = {"gated_delta": (True, True), "gated": (True, False), "delta": (False, True),
         "linear": (False, False)}
LENGTHS = [1, 64, 65, 200, 0, 130]


@pytest.fixture(scope="module")
def gdn():
    import gated_deltanet_state_gdn_b200 as g
    g.lib()
    return g


@pytest.fixture(scope="module")
def W():
    from gated_deltanet_state_gdn_b200 import workloads
    return workloads


def _run_both(gdn, oracle_mod, c, g, beta, sequential, **kw):
    # the binding reads the per-key spelling from g's rank; the oracle takes it as a flag
    o, f = gdn.gdn_prefill(dev(c.q), dev(c.k), dev(c.v), dev(g), dev(beta), dev(c.cu_seqlens),
                           dev(c.initial_state), scale=c.scale, qk_l2norm=c.qk_l2norm,
                           sequential=sequential,
                           **{k: (dev(v) if torch.is_tensor(v) else v) for k, v in kw.items()
                              if k != "decay_per_key"})
    torch.cuda.synchronize()
    okw = {k: (f64(v) if torch.is_tensor(v) else v) for k, v in kw.items()}
    ro, rf = oracle_mod.prefill(f64(c.q), f64(c.k), f64(c.v), None if g is None else f64(g),
                                None if beta is None else f64(beta), c.cu_seqlens.numpy(),
                                None if c.initial_state is None else f64(c.initial_state),
                                scale=c.scale, qk_l2norm=c.qk_l2norm, **okw)
    return f64(o), f64(f), ro, rf


def _parity(c, o, f, ro, rf, tol):
    assert_prefill_parity(o, f, ro, rf, request_ranges(c.cu_seqlens, c.B, c.N), tol)


@pytest.mark.parametrize("sequential", [False, True])
@pytest.mark.parametrize("rule", list(RULES))
def test_update_rules(gdn, W, oracle_mod, rule, sequential):
    c = W.make_prefill(31, LENGTHS, 2, 4, 128, 128, init_std=0.02, qk_l2norm=True)
    has_decay, has_beta = RULES[rule]
    o, f, ro, rf = _run_both(gdn, oracle_mod, c, c.g if has_decay else None,
                             c.beta if has_beta else None, sequential, update_rule=rule)
    _parity(c, o, f, ro, rf, TOL_BF16)


@pytest.mark.parametrize("sequential", [False, True])
@pytest.mark.parametrize("rule", ["gated_delta", "gated", "delta"])
def test_qwen_gate_and_sigmoid_beta(gdn, W, oracle_mod, rule, sequential):
    """Raw decay N(0,1) through -exp(a_log) softplus(decay + dt_bias), a_log ~ U[-2,1],
    dt_bias ~ N(0,0.5); raw beta N(0,1) through the sigmoid."""
    c = W.make_prefill(32, LENGTHS, 2, 4, 128, 128, init_std=0.02, qk_l2norm=True)
    rng = np.random.default_rng(33)
    has_decay, has_beta = RULES[rule]
    decay = torch.from_numpy(rng.standard_normal(c.g.shape).astype(np.float32))
    braw = torch.from_numpy(rng.standard_normal(c.beta.shape).astype(np.float32))
    kw = {"update_rule": rule}
    if has_decay:
        kw.update(gate_activation="qwen",
                  a_log=torch.from_numpy(rng.uniform(-2, 1, 4).astype(np.float32)),
                  dt_bias=torch.from_numpy((0.5 * rng.standard_normal(4)).astype(np.float32)))
    if has_beta:
        kw["beta_activation"] = "sigmoid"
    o, f, ro, rf = _run_both(gdn, oracle_mod, c, decay if has_decay else None,
                             braw if has_beta else None, sequential, **kw)
    _parity(c, o, f, ro, rf, TOL_BF16)


@pytest.mark.parametrize("sequential", [True, False])
@pytest.mark.parametrize("Dk,Dv", [(128, 128), (64, 32)])
def test_fp16_activations(gdn, W, oracle_mod, Dk, Dv, sequential):
    """float16 q/k/v/out on the per-token kernel (fp32 arithmetic) and on the tensor-core kernel
    (fp16 operand tiles); the oracle reads the same fp16-rounded inputs."""
    assert gdn.prefill_uses_chunked(torch.float16, 4, Dk, Dv)
    c = W.make_prefill(34, LENGTHS, 2, 4, Dk, Dv, dtype=torch.float16, init_std=0.02,
                       qk_l2norm=True)
    o, f, ro, rf = _run_both(gdn, oracle_mod, c, c.g, c.beta, sequential)
    tol = TOL_F16 if sequential else TOL_F16_CHUNKED
    assert o.dtype == np.float64
    _parity(c, o, f, ro, rf, tol)


@pytest.mark.parametrize("rule", ["delta", "linear"])
def test_fp16_rules_on_tensor_cores(gdn, W, oracle_mod, rule):
    """The fp16 tensor-core kernel with the rule switches (general instantiation)."""
    has_decay, has_beta = RULES[rule]
    c = W.make_prefill(36, LENGTHS, 2, 4, 128, 128, dtype=torch.float16, init_std=0.02,
                       qk_l2norm=True)
    o, f, ro, rf = _run_both(gdn, oracle_mod, c, c.g if has_decay else None,
                             c.beta if has_beta else None, False, update_rule=rule)
    _parity(c, o, f, ro, rf, TOL_F16_CHUNKED)


def test_linear_rule_long_sequence_matches_oracle(gdn, W, oracle_mod):
    """Without decay the state is a plain causal sum; a 1000-token request keeps growing it."""
    c = W.make_prefill(35, [1000], 1, 4, 128, 128, init_std=None, qk_l2norm=True)
    o, f, ro, rf = _run_both(gdn, oracle_mod, c, None, None, False, update_rule="linear")
    _parity(c, o, f, ro, rf, TOL_BF16)


# ------------------------------------------------------- per-key-dimension decay
# "com.microsoft.GatedDeltaNet", Inputs table: `decay` spelled (..., num_heads_v,
# head_size_qk), exp(g_t) read as diag(exp(g_t)) on the key axis of the state (the oracle's
# reading, pinned in test_oracle_pins).  bf16 heads of 8 to 128 run the per-key tensor-core
# kernel (bf16 operand tiles, as the scalar-decay chunked kernel, so the same 2e-2 bound);
# fp16 (whose exponent range cannot hold the kernel's scaled operands), fp32, other head
# sizes and `sequential` run the per-token kernel (fp32 arithmetic).
TOL_BY_DTYPE = {torch.bfloat16: TOL_BF16, torch.float16: TOL_F16, torch.float32: 1e-4}


@pytest.mark.parametrize("sequential", [False, True])
@pytest.mark.parametrize("dtype,Dk,Dv,Hq,Hv", [
    (torch.bfloat16, 128, 128, 2, 4), (torch.float16, 64, 32, 1, 2), (torch.float32, 12, 9, 1, 2),
    (torch.float32, 256, 256, 1, 1), (torch.bfloat16, 160, 96, 2, 2), (torch.bfloat16, 1, 1, 1, 3),
    (torch.bfloat16, 12, 9, 1, 2), (torch.float16, 128, 128, 2, 2), (torch.bfloat16, 100, 72, 3, 6)])
def test_per_key_decay_matches_oracle(gdn, W, oracle_mod, dtype, Dk, Dv, Hq, Hv, sequential):
    tc = dtype == torch.bfloat16 and 8 <= min(Dk, Dv) and max(Dk, Dv) <= 128 and not sequential
    assert gdn.prefill_uses_chunked(dtype, Hv, Dk, Dv, sequential, decay_per_key=True) == tc
    c = W.make_prefill(41, LENGTHS, Hq, Hv, Dk, Dv, dtype=dtype, init_std=0.02,
                       qk_l2norm=True, decay_per_key=True)
    assert tuple(c.g.shape) == (c.N, Hv, Dk)
    o, f, ro, rf = _run_both(gdn, oracle_mod, c, c.g, c.beta, sequential, decay_per_key=True)
    _parity(c, o, f, ro, rf, TOL_BY_DTYPE[dtype])


@pytest.mark.parametrize("sequential", [False, True])
@pytest.mark.parametrize("rule,qwen", [("gated", False), ("gated", True), ("gated_delta", True)])
def test_per_key_decay_rules_and_gates(gdn, W, oracle_mod, rule, qwen, sequential):
    """The gated rule (no retrieval, beta = 1) and the qwen gate applied to every key
    dimension with its head's a_log and dt_bias (raw decay N(0,1)), with the sigmoid beta."""
    c = W.make_prefill(42, LENGTHS, 2, 4, 128, 64, init_std=0.02, qk_l2norm=True,
                       decay_per_key=True)
    has_decay, has_beta = RULES[rule]
    rng = np.random.default_rng(43)
    g = c.g
    kw = {"update_rule": rule, "decay_per_key": True}
    if qwen:
        g = torch.from_numpy(rng.standard_normal(c.g.shape).astype(np.float32))
        kw.update(gate_activation="qwen",
                  a_log=torch.from_numpy(rng.uniform(-2, 1, 4).astype(np.float32)),
                  dt_bias=torch.from_numpy((0.5 * rng.standard_normal(4)).astype(np.float32)))
    beta = None
    if has_beta:
        beta = torch.from_numpy(rng.standard_normal(c.beta.shape).astype(np.float32))
        kw["beta_activation"] = "sigmoid"
    o, f, ro, rf = _run_both(gdn, oracle_mod, c, g, beta, sequential, **kw)
    _parity(c, o, f, ro, rf, TOL_BF16)


def test_per_key_decay_strong_and_infinite_decays(gdn, W, oracle_mod):
    """Per-dimension decays down to -40 and -inf in some dimensions (a dimension that forgets
    at once) on the tensor-core kernel: it floors every per-dimension log-decay at -9 so that
    its scaled operands stay finite; a decay factor below e^-9 ~ 1.2e-4 then weighs the old
    column at 1.2e-4 instead of less, far inside the bf16 bound (the oracle keeps the raw g)."""
    c = W.make_prefill(46, LENGTHS, 2, 4, 128, 128, init_std=0.02, qk_l2norm=True,
                       decay_per_key=True)
    rng = np.random.default_rng(47)
    g = c.g.numpy().copy()
    strong = rng.random(g.shape) < 0.05
    g[strong] = -rng.uniform(9.0, 40.0, int(strong.sum()))
    g[:, :, 5] = -np.inf
    g[:, 1, :8] = -np.inf
    g = torch.from_numpy(g.astype(np.float32))
    assert gdn.prefill_uses_chunked(torch.bfloat16, 4, 128, 128, decay_per_key=True)
    o, f, ro, rf = _run_both(gdn, oracle_mod, c, g, c.beta, False, decay_per_key=True)
    _parity(c, o, f, ro, rf, TOL_BF16)


def test_per_key_decay_tensor_cores_match_per_token_kernel(gdn, W):
    """The two per-key kernels on the same bf16 bytes (requests of 1 to 200 tokens, an empty
    one, GQA): outputs and states agree within the bf16 bound."""
    c = W.make_prefill(48, LENGTHS, 2, 4, 128, 128, init_std=0.02, qk_l2norm=True,
                       decay_per_key=True)
    args = [dev(t) for t in (c.q, c.k, c.v, c.g, c.beta, c.cu_seqlens, c.initial_state)]
    o1, f1 = gdn.gdn_prefill(*args, scale=c.scale, qk_l2norm=True)
    o2, f2 = gdn.gdn_prefill(*args, scale=c.scale, qk_l2norm=True, sequential=True)
    torch.cuda.synchronize()
    assert_prefill_parity(f64(o1), f64(f1), f64(o2), f64(f2),
                          request_ranges(c.cu_seqlens, c.B, c.N), TOL_BF16)


def test_per_key_decay_equal_dimensions_match_scalar_gate(gdn, W):
    """The same decay in every key dimension is the scalar gate: the per-key and the scalar
    instantiations of the per-token kernel (fp32) agree to fp32 rounding."""
    c = W.make_prefill(44, LENGTHS, 2, 4, 64, 64, dtype=torch.float32, init_std=0.02,
                       qk_l2norm=True)
    gk = c.g[:, :, None].expand(-1, -1, 64).contiguous()
    args = (dev(c.q), dev(c.k), dev(c.v))
    o1, f1 = gdn.gdn_prefill(*args, dev(c.g), dev(c.beta), dev(c.cu_seqlens),
                             dev(c.initial_state), scale=c.scale, qk_l2norm=True)
    o2, f2 = gdn.gdn_prefill(*args, dev(gk), dev(c.beta), dev(c.cu_seqlens),
                             dev(c.initial_state), scale=c.scale, qk_l2norm=True)
    torch.cuda.synchronize()
    assert_prefill_parity(f64(o2), f64(f2), f64(o1), f64(f1),
                          request_ranges(c.cu_seqlens, c.B, c.N), 1e-5)


def test_per_key_tensor_cores_with_equal_dimensions_match_scalar_chunked(gdn, W, oracle_mod):
    """bf16: the per-key tensor-core kernel with the same decay in every key dimension and the
    scalar-decay chunked kernel (two different chunk factorings of one recurrence) are each
    held to the oracle of the scalar gate.  (Against each other the bound would be twice the
    bound each meets against the oracle.)"""
    c = W.make_prefill(49, LENGTHS, 2, 4, 128, 128, init_std=0.02, qk_l2norm=True)
    gk = c.g[:, :, None].expand(-1, -1, 128).contiguous()
    args = (dev(c.q), dev(c.k), dev(c.v))
    assert gdn.prefill_uses_chunked(torch.bfloat16, 4, 128, 128, decay_per_key=True)
    o1, f1 = gdn.gdn_prefill(*args, dev(c.g), dev(c.beta), dev(c.cu_seqlens),
                             dev(c.initial_state), scale=c.scale, qk_l2norm=True, split=False)
    o2, f2 = gdn.gdn_prefill(*args, dev(gk), dev(c.beta), dev(c.cu_seqlens),
                             dev(c.initial_state), scale=c.scale, qk_l2norm=True)
    torch.cuda.synchronize()
    ro, rf = oracle_mod.prefill(f64(c.q), f64(c.k), f64(c.v), f64(c.g), f64(c.beta),
                                c.cu_seqlens.numpy(), f64(c.initial_state), scale=c.scale,
                                qk_l2norm=True)
    ranges = request_ranges(c.cu_seqlens, c.B, c.N)
    assert_prefill_parity(f64(o1), f64(f1), ro, rf, ranges, TOL_BF16)
    assert_prefill_parity(f64(o2), f64(f2), ro, rf, ranges, TOL_BF16)


def test_per_key_decay_rank4_spelling(gdn, W, oracle_mod):
    """(batch, sequence, heads, dim) activations with the decay as (batch, sequence, Hv, Dk)."""
    B, S, Hq, Hv, D = 3, 70, 1, 2, 32
    c = W.make_prefill(45, [S] * B, Hq, Hv, D, D, uniform=True, init_std=0.02, qk_l2norm=True,
                       decay_per_key=True)
    o, f = gdn.gdn_prefill(dev(c.q).view(B, S, Hq, D), dev(c.k).view(B, S, Hq, D),
                           dev(c.v).view(B, S, Hv, D), dev(c.g).view(B, S, Hv, D),
                           dev(c.beta).view(B, S, Hv), None, dev(c.initial_state),
                           scale=c.scale, qk_l2norm=True)
    torch.cuda.synchronize()
    ro, rf = oracle_mod.prefill(f64(c.q), f64(c.k), f64(c.v), f64(c.g), f64(c.beta), None,
                                f64(c.initial_state), B=B, scale=c.scale, qk_l2norm=True,
                                decay_per_key=True)
    assert_prefill_parity(f64(o), f64(f), ro, rf, [(b * S, (b + 1) * S) for b in range(B)],
                          TOL_BF16)


def test_full_ragged_prefill_per_key_decay_all_heads(gdn, W, oracle_mod):
    """The ragged workload's shapes (8 requests, U[1, 4096], Hq=16, Hv=32, D=128, bf16) with a
    per-key decay -softplus(N(0,1)) in every key dimension: every head and row."""
    c = W.ragged_prefill_case(decay_per_key=True)
    o, f, ro, rf = _run_both(gdn, oracle_mod, c, c.g, c.beta, False, decay_per_key=True)
    _parity(c, o, f, ro, rf, TOL_BF16)


def test_per_key_decay_many_requests(gdn, W, oracle_mod):
    """600 requests of 0 to 40 tokens: more requests than the per-key kernel orders by length
    (it then takes them in index order), every request and head against the oracle."""
    rng = np.random.default_rng(50)
    lengths = rng.integers(0, 41, 600).tolist()
    c = W.make_prefill(51, lengths, 1, 2, 32, 16, init_std=0.02, qk_l2norm=True,
                       decay_per_key=True)
    assert gdn.prefill_uses_chunked(torch.bfloat16, 2, 32, 16, decay_per_key=True)
    o, f, ro, rf = _run_both(gdn, oracle_mod, c, c.g, c.beta, False, decay_per_key=True)
    _parity(c, o, f, ro, rf, TOL_BF16)


@pytest.mark.parametrize("sequential", [False, True])
def test_per_key_decay_without_in_kernel_norm(gdn, W, oracle_mod, sequential):
    """q and k unit-normalised on the host in fp32 before the bf16 cast, qk_l2norm off (the
    long-context workload's convention), with a per-key decay: both per-key kernels against
    the oracle."""
    c = W.make_prefill(52, LENGTHS, 2, 4, 128, 128, init_std=0.02, qk_l2norm=False,
                       host_norm_qk=True, decay_per_key=True)
    o, f, ro, rf = _run_both(gdn, oracle_mod, c, c.g, c.beta, sequential, decay_per_key=True)
    _parity(c, o, f, ro, rf, TOL_BF16)
