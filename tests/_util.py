"""Shared helpers for the parity tests (not collected: no test_ prefix)."""
import numpy as np
import torch

# Tolerances on relative L2 error (||x - ref|| / ||ref||) against the float64
# oracle: fp32 activations 1e-4, bf16 activations (fp32 state) 2e-2.
TOL_F32 = 1e-4
TOL_BF16 = 2e-2


def rel_l2(x, ref) -> float:
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.linalg.norm(ref.ravel())
    num = np.linalg.norm((x - ref).ravel())
    return float(num / den) if den > 0 else float(num)


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def dev(t, device="cuda"):
    return None if t is None else t.to(device)


def oracle_prefill_case(oracle, c, out=None):
    """Run the oracle on a workloads.PrefillCase (bf16 bytes widened exactly)."""
    return oracle.prefill(f64(c.q), f64(c.k), f64(c.v), f64(c.g), f64(c.beta),
                          None if c.cu_seqlens is None else c.cu_seqlens.numpy(),
                          None if c.initial_state is None else f64(c.initial_state),
                          B=c.B, scale=c.scale, qk_l2norm=c.qk_l2norm, out=out,
                          decay_per_key=c.g.dim() == 3)


def run_gpu_prefill(c, sequential=False, out=None):
    import gated_deltanet_state_gdn_b200 as gdn
    o, f = gdn.gdn_prefill(dev(c.q), dev(c.k), dev(c.v), dev(c.g), dev(c.beta),
                           dev(c.cu_seqlens), dev(c.initial_state), None,
                           None if out is None else dev(out), num_requests=c.B, scale=c.scale,
                           qk_l2norm=c.qk_l2norm, sequential=sequential)
    torch.cuda.synchronize()
    return o, f


def sub_case_head(c, h, token_slice=None, request_slice=None):
    """Reduce a prefill case to one value head (and its query/key head): Hq = Hv = 1.

    The GQA index floor(h * Hq / Hv) is applied here, independently of both
    implementations."""
    import copy
    Hq, Hv = c.q.shape[1], c.v.shape[1]
    qh = (h * Hq) // Hv
    s = copy.copy(c)
    s.q = c.q[:, qh:qh + 1].contiguous()
    s.k = c.k[:, qh:qh + 1].contiguous()
    s.v = c.v[:, h:h + 1].contiguous()
    s.g = c.g[:, h:h + 1].contiguous()
    s.beta = c.beta[:, h:h + 1].contiguous()
    if c.initial_state is not None:
        s.initial_state = c.initial_state[:, h:h + 1].contiguous()
    return s


# ------------------------------------------------------------ block and row parity
# The tolerance of the recurrence's statement (relative L2 <= 2e-2 for bf16 activations with
# the fp32 state, <= 1e-4 for fp32) is applied to every independent problem on its own, not
# only to the whole tensor: per (request, value head) block of outputs, per final state, and
# per output row (one token of one head), each row judged against the larger of its own
# reference norm and its block's RMS row norm, so that a row whose exact value nearly cancels
# is held to the scale of the terms that produced it.  One wrong row in an otherwise correct
# block therefore fails the row bound even when the whole-tensor norm hides it.
def request_ranges(cu_seqlens, B, N):
    """[start, end) of each request after clamping to [0, N] (empty when end <= start)."""
    if cu_seqlens is None:
        S = N // B if B else 0
        return [(b * S, (b + 1) * S) for b in range(B)]
    cu = np.clip(np.asarray(cu_seqlens, np.int64), 0, N)
    return [(int(cu[b]), int(max(cu[b], cu[b + 1]))) for b in range(B)]


ROW_BOUND_MIN_WIDTH = 8


def assert_rows_close(x, ref, tol, what=""):
    """x, ref: [rows, width] of one independent problem.  Block relative L2 <= tol, and every
    row's error <= tol * max(||ref_row||, RMS row norm of the block).

    The row bound is a relative L2 over the row, so it is applied to rows of at least
    ROW_BOUND_MIN_WIDTH elements: on a row of one or a few elements it turns into an
    elementwise relative bound, which the bf16 rounding of a single output can exceed where
    the exact value nearly cancels (all keys of a one-wide head are parallel).  Narrower heads
    are held to the block bound."""
    x = np.asarray(x, np.float64).reshape(ref.shape[0], -1)
    ref = np.asarray(ref, np.float64).reshape(ref.shape[0], -1)
    if ref.size == 0:
        return
    assert np.isfinite(x).all(), f"{what}: non-finite values"
    err = rel_l2(x, ref)
    assert err <= tol, f"{what}: block rel-L2 {err:.3e} > {tol}"
    if ref.shape[1] < ROW_BOUND_MIN_WIDTH:
        return
    rn = np.linalg.norm(ref, axis=1)
    rms = float(np.sqrt(np.mean(rn ** 2)))
    en = np.linalg.norm(x - ref, axis=1)
    lim = tol * np.maximum(rn, rms)
    bad = np.nonzero(en > lim)[0]
    if rms == 0.0:
        bad = np.nonzero(en > 0)[0]
    assert bad.size == 0, (f"{what}: {bad.size} rows above the row bound, worst row {bad[0]}: "
                           f"error {en[bad[0]]:.3e} vs limit {lim[bad[0]]:.3e}")


def assert_prefill_parity(out, fs, ro, rf, ranges, tol, heads=None, token_mask=None):
    """Whole-tensor, per (request, value head) and per-row parity of a prefill result.

    out [N, Hv, Dv] and fs [B, Hv, Dv, Dk] (torch or numpy) against the oracle's ro, rf;
    `heads` restricts the check to those value heads (ro, rf then hold only them, in order);
    `token_mask` (bool [N]) drops tokens whose outputs are undefined."""
    o = f64(out) if isinstance(out, torch.Tensor) else np.asarray(out, np.float64)
    f = f64(fs) if isinstance(fs, torch.Tensor) else np.asarray(fs, np.float64)
    if heads is not None:
        o = o[:, heads]
        f = f[:, heads]
    keep = slice(None) if token_mask is None else np.asarray(token_mask, bool)
    assert rel_l2(o[keep], ro[keep]) <= tol, f"outputs rel-L2 {rel_l2(o[keep], ro[keep]):.3e}"
    assert rel_l2(f, rf) <= tol, f"final states rel-L2 {rel_l2(f, rf):.3e}"
    Hv = o.shape[1]
    for b, (s, e) in enumerate(ranges):
        for h in range(Hv):
            hn = h if heads is None else heads[h]
            if e > s:
                rows = np.arange(s, e)
                if token_mask is not None:
                    rows = rows[np.asarray(token_mask, bool)[s:e]]
                assert_rows_close(o[rows, h], ro[rows, h], tol, f"out request {b} head {hn}")
            assert_rows_close(f[b, h], rf[b, h], tol, f"final state request {b} head {hn}")


def assert_out_close(o, ro, tol, what="out"):
    """Decode outputs [rows, T, HV, Dv]: whole tensor, then every (row, head) block of T
    tokens with the per-token row bound of assert_rows_close."""
    o = np.asarray(o, np.float64)
    ro = np.asarray(ro, np.float64)
    assert o.shape == ro.shape, (o.shape, ro.shape)
    assert rel_l2(o, ro) <= tol, f"{what}: rel-L2 {rel_l2(o, ro):.3e}"
    for b in range(o.shape[0]):
        for h in range(o.shape[2]):
            assert_rows_close(o[b, :, h, :], ro[b, :, h, :], tol, f"{what} row {b} head {h}")


def assert_states_close(p, rp, tol, what="slot"):
    """States [slots, HV, Dv, Dk]: whole tensor, then every (slot, head) state on its own with
    the per-row bound (one row = one value index dv)."""
    p = np.asarray(p, np.float64)
    rp = np.asarray(rp, np.float64)
    assert p.shape == rp.shape, (p.shape, rp.shape)
    assert rel_l2(p, rp) <= tol, f"{what}: rel-L2 {rel_l2(p, rp):.3e}"
    for s in range(p.shape[0]):
        for h in range(p.shape[1]):
            assert_rows_close(p[s, h], rp[s, h], tol, f"{what} {s} head {h}")
