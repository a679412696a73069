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
                          B=c.B, scale=c.scale, qk_l2norm=c.qk_l2norm, out=out)


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
