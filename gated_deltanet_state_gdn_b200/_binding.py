"""ctypes binding of libgdn (argument marshalling only).

Each function takes torch CUDA tensors, checks dtypes and shapes, makes
inputs contiguous, allocates outputs the caller did not pass (torch is the
allocator), and calls the C entry point of the same name on torch's current
stream.  Every step of the recurrence runs in libgdn's kernels; there is no
other path.  If libgdn.so cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgdn.so")
# test build compiled with GDN_CHECKS (bounds-checked accesses, GDN_DEV_BOUNDS)
CHECKED_LIB_PATH = os.path.join(_PKG, "libgdn_checked.so")

GDN_OK = 0
GDN_ERR_NULL = 1
GDN_ERR_SHAPE = 2
GDN_ERR_DTYPE = 3
GDN_ERR_ALIGN = 4
GDN_ERR_ALIAS = 5
GDN_ERR_UNSUPPORTED = 6
GDN_ERR_CUDA = 7

GDN_F32 = 0
GDN_BF16 = 1
GDN_F16 = 2

GDN_PREFILL_SEQUENTIAL = 1
GDN_DISABLE_STATE_UPDATE = 2
GDN_DECODE_QK_L2NORM = 4
GDN_DECODE_IDX64 = 1 << 7
GDN_RULE_GATED = 1 << 3
GDN_RULE_DELTA = 2 << 3
GDN_RULE_LINEAR = 3 << 3
GDN_GATE_QWEN = 1 << 5
GDN_BETA_SIGMOID = 1 << 6
GDN_DECAY_PER_KEY = 1 << 8

# update_rule of the op -> (flag bits, has decay input, has beta input)
UPDATE_RULES = {
    "gated_delta": (0, True, True),
    "gated": (GDN_RULE_GATED, True, False),
    "delta": (GDN_RULE_DELTA, False, True),
    "linear": (GDN_RULE_LINEAR, False, False),
}

GDN_DEV_BAD_SLOT = 1
GDN_DEV_TIMEOUT = 2
GDN_DEV_INTERNAL = 4
GDN_DEV_BOUNDS = 8            # checked builds only
GDN_DEV_TEST_STALL = 1 << 30  # checked builds only, set by the caller (decode timeout path)

EXPORTED = ("gdn_prefill", "gdn_prefill_ws", "gdn_prefill_workspace_size",
            "gdn_prefill_noalloc", "gdn_decode", "gdn_conv1d", "gdn_status_string",
            "gdn_last_error", "gdn_abi_version", "gdn_prefill_uses_chunked")

_lib = None


class GdnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        name = status_string(status)
        detail = ""
        if status == GDN_ERR_CUDA:
            detail = ": " + lib().gdn_last_error().decode()
        super().__init__(f"{where} failed with {name}{detail}")


def use_library(path: str) -> str:
    """Route the calls that follow through the library at `path` (for instance the checked test
    build CHECKED_LIB_PATH); returns the path in use before."""
    global _lib, LIB_PATH
    prev = LIB_PATH
    LIB_PATH = path
    _lib = None
    return prev


def lib():
    """Load libgdn.so (built in-tree); raise if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"libgdn.so not found at {LIB_PATH}: build it with "
                "`python -m gated_deltanet_state_gdn_b200.build` (there is no fallback path)")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, u32, f32 = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64,
                                  ctypes.c_uint32, ctypes.c_float)
        L.gdn_prefill.restype = ctypes.c_int
        L.gdn_prefill.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                  i32, i64, i32, i32, i32, i32, ctypes.c_int, f32, i32, u32,
                                  vp, vp]
        L.gdn_prefill_ws.restype = ctypes.c_int
        L.gdn_prefill_ws.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                     i32, i64, i32, i32, i32, i32, ctypes.c_int, f32, i32, u32,
                                     vp, ctypes.c_uint64, vp, vp]
        L.gdn_prefill_noalloc.restype = ctypes.c_int
        L.gdn_prefill_noalloc.argtypes = L.gdn_prefill.argtypes
        L.gdn_prefill_workspace_size.restype = ctypes.c_uint64
        L.gdn_prefill_workspace_size.argtypes = [i32, i64, i32, i32, i32, i32, ctypes.c_int, u32]
        L.gdn_decode.restype = ctypes.c_int
        L.gdn_decode.argtypes = [vp, vp, vp, vp, i32, i64, i64, vp, vp, vp,
                                 vp, vp, vp, vp, f32, vp,
                                 i32, i32, i32, i32, i32, i32, i32, u32, vp, vp]
        L.gdn_conv1d.restype = ctypes.c_int
        L.gdn_conv1d.argtypes = [vp, vp, vp, vp, vp, vp, i32, i64, i32, i32, i32, ctypes.c_int,
                                 i32, vp, vp]
        L.gdn_status_string.restype = ctypes.c_char_p
        L.gdn_status_string.argtypes = [i32]
        L.gdn_last_error.restype = ctypes.c_char_p
        L.gdn_last_error.argtypes = []
        L.gdn_abi_version.restype = i32
        L.gdn_abi_version.argtypes = []
        L.gdn_prefill_uses_chunked.restype = i32
        L.gdn_prefill_uses_chunked.argtypes = [ctypes.c_int, i32, i32, i32, u32]
        _lib = L
    return _lib


def prefill_uses_chunked(dtype: torch.dtype, Hv: int, Dk: int, Dv: int,
                         sequential: bool = False, decay_per_key: bool = False) -> bool:
    """True when gdn_prefill would run the chunked tensor-core kernel for these sizes."""
    code = {torch.bfloat16: GDN_BF16, torch.float16: GDN_F16}.get(dtype, GDN_F32)
    flags = (GDN_PREFILL_SEQUENTIAL if sequential else 0) | \
        (GDN_DECAY_PER_KEY if decay_per_key else 0)
    return bool(lib().gdn_prefill_uses_chunked(code, Hv, Dk, Dv, flags))


def status_string(status: int) -> str:
    return lib().gdn_status_string(int(status)).decode()


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check_cuda(name, t, dtype=None):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return t.contiguous()


def _align16(t):
    """A contiguous input whose data does not start on a 16-byte boundary (a view such as
    g[1:]) is copied into a fresh allocation, which the caching allocator aligns; gdn_prefill
    requires 16-byte aligned inputs."""
    if t is not None and t.data_ptr() % 16 != 0:
        t = t.clone()
    return t


def gdn_prefill(q, k, v, g, beta, cu_seqlens=None, initial_state=None, final_state=None,
                out=None, *, num_requests: Optional[int] = None, scale: Optional[float] = None,
                qk_l2norm: bool = False, sequential: bool = False, update_rule: str = "gated_delta",
                gate_activation: str = "none", a_log=None, dt_bias=None,
                beta_activation: str = "none", split: bool = True, dev_status=None, stream=None):
    """Gated DeltaNet prefill (log-space form) over ragged requests.

    q, k: [N, Hq, Dk] or [B, S, Hq, Dk]; v: [N, Hv, Dv] (same leading axes);
    activations fp32, bf16 or fp16; g, beta: [N, Hv] fp32 (g None for the rules
    without decay, beta None for those without retrieval); g may instead be
    [N, Hv, Dk] (one decay per key dimension, GDN_DECAY_PER_KEY); cu_seqlens: [B+1]
    int32 (rank-3 form) or None; initial_state: [B, Hv, Dv, Dk] fp32 or None.
    update_rule: gated_delta | gated | delta | linear; gate_activation: none |
    qwen (a_log, dt_bias: [Hv] fp32); beta_activation: none | sigmoid.
    ``scale`` None or 0 selects 1/sqrt(Dk).  With ``split`` (the default) a call that
    gdn_prefill_workspace_size says can cut long requests into parallel segments gets a
    workspace from torch's allocator and runs through gdn_prefill_ws; ``split=False`` always
    calls gdn_prefill.  Returns (out, final_state).
    """
    if update_rule not in UPDATE_RULES:
        raise ValueError(f"unknown update_rule {update_rule!r}")
    if gate_activation not in ("none", "qwen") or beta_activation not in ("none", "sigmoid"):
        raise ValueError("gate_activation must be none|qwen and beta_activation none|sigmoid")
    rule_flags, has_decay, has_beta = UPDATE_RULES[update_rule]
    if (g is not None) != has_decay or (beta is not None) != has_beta:
        raise ValueError(f"update_rule {update_rule!r} takes "
                         f"{'a' if has_decay else 'no'} decay and {'a' if has_beta else 'no'} beta")
    qwen = gate_activation == "qwen"
    if qwen != (a_log is not None and dt_bias is not None):
        raise ValueError("gate_activation 'qwen' requires a_log and dt_bias (and only it takes them)")
    # the per-key-dimension spelling of the decay has one more axis than [..., Hv]
    per_key = g is not None and g.dim() == q.dim()
    if q.dim() == 4:
        Bq, S = q.shape[0], q.shape[1]
        if cu_seqlens is not None:
            raise ValueError("cu_seqlens requires the rank-3 (total_tokens, heads, dim) form")
        num_requests = Bq
        q = q.reshape(Bq * S, *q.shape[2:])
        k = k.reshape(Bq * S, *k.shape[2:])
        v = v.reshape(Bq * S, *v.shape[2:])
        g = None if g is None else (g.reshape(Bq * S, *g.shape[2:]) if per_key
                                    else g.reshape(Bq * S, -1))
        beta = None if beta is None else beta.reshape(Bq * S, -1)
        if out is not None:
            out = out.view(Bq * S, *out.shape[2:])
    dt = {torch.bfloat16: GDN_BF16, torch.float32: GDN_F32, torch.float16: GDN_F16}.get(q.dtype)
    if dt is None:
        raise TypeError(f"unsupported activation dtype {q.dtype}")
    q = _check_cuda("q", q, q.dtype)
    k = _check_cuda("k", k, q.dtype)
    v = _check_cuda("v", v, q.dtype)
    g = _check_cuda("g", g, torch.float32)
    beta = _check_cuda("beta", beta, torch.float32)
    a_log = _check_cuda("a_log", a_log, torch.float32)
    dt_bias = _check_cuda("dt_bias", dt_bias, torch.float32)
    cu_seqlens = _check_cuda("cu_seqlens", cu_seqlens, torch.int32)
    initial_state = _check_cuda("initial_state", initial_state, torch.float32)
    q, k, v, g, beta, initial_state = map(_align16, (q, k, v, g, beta, initial_state))
    N, Hq, Dk = q.shape
    Hv, Dv = v.shape[1], v.shape[2]
    g_shape = (N, Hv, Dk) if per_key else (N, Hv)
    if k.shape != q.shape or v.shape[0] != N or (g is not None and g.shape != g_shape) or \
            (beta is not None and beta.shape != (N, Hv)):
        raise ValueError("inconsistent q/k/v/g/beta shapes")
    if qwen and (a_log.shape != (Hv,) or dt_bias.shape != (Hv,)):
        raise ValueError("a_log and dt_bias must be [Hv]")
    if cu_seqlens is not None:
        B = cu_seqlens.shape[0] - 1
    else:
        if num_requests is None:
            raise ValueError("num_requests is required without cu_seqlens")
        B = int(num_requests)
    if out is None:
        out = torch.empty((N, Hv, Dv), dtype=q.dtype, device=q.device)
    elif not out.is_contiguous() or out.dtype != q.dtype or tuple(out.shape) != (N, Hv, Dv):
        raise ValueError("out must be a contiguous [N, Hv, Dv] tensor of q's dtype")
    if final_state is None:
        final_state = torch.empty((B, Hv, Dv, Dk), dtype=torch.float32, device=q.device)
    elif not final_state.is_contiguous() or final_state.dtype != torch.float32:
        raise ValueError("final_state must be a contiguous fp32 tensor")
    if initial_state is not None and tuple(initial_state.shape) != (B, Hv, Dv, Dk):
        raise ValueError("initial_state must be [B, Hv, Dv, Dk]")
    if scale is None or scale == 0.0:
        scale = 1.0 / math.sqrt(Dk)
    flags = (GDN_PREFILL_SEQUENTIAL if sequential else 0) | rule_flags
    flags |= (GDN_GATE_QWEN if qwen else 0) | (GDN_BETA_SIGMOID if beta_activation == "sigmoid" else 0)
    flags |= GDN_DECAY_PER_KEY if per_key else 0
    ws_bytes = int(lib().gdn_prefill_workspace_size(B, N, Hq, Hv, Dk, Dv, dt, flags)) \
        if split else 0
    if ws_bytes > 0:
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
        if stream is not None:
            ws.record_stream(stream)   # released to the allocator only after the call
        st = lib().gdn_prefill_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(a_log),
                                  _ptr(dt_bias), _ptr(cu_seqlens), _ptr(initial_state),
                                  _ptr(final_state), _ptr(out), B, N, Hq, Hv, Dk, Dv, dt,
                                  float(scale), int(bool(qk_l2norm)), flags, _ptr(ws), ws_bytes,
                                  _ptr(dev_status), _stream(stream))
    else:
        st = lib().gdn_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(a_log),
                               _ptr(dt_bias), _ptr(cu_seqlens),
                               _ptr(initial_state), _ptr(final_state), _ptr(out), B, N, Hq, Hv,
                               Dk, Dv, dt, float(scale), int(bool(qk_l2norm)), flags,
                               _ptr(dev_status), _stream(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_prefill")
    return out, final_state


def gdn_decode(q, k, v, state_pool, read_idx, A_log, a, dt_bias, b, *, scale=None, out=None,
               scatter_idx=None, disable_state_update: bool = False, use_qk_l2norm: bool = True,
               write_idx=None, dev_status=None, stream=None):
    """Gated DeltaProduct decode / MTP over an fp32 pool (updated in place).

    q: [B, T, H, Dk]; k: [B, T, nh, H, Dk]; v: [B, T, nh, HV, Dv] (bf16);
    state_pool: [P, HV, Dv, Dk] fp32 with dense rows (slot/head padding allowed);
    read_idx, write_idx: [B] int32 or int64 (the same for both); scatter_idx: [B, T] int32;
    A_log, dt_bias: [HV] fp32; a: [B, T, HV]; b: [B, T, nh, HV] (bf16).
    Returns (out, state_pool).
    """
    q = _check_cuda("q", q, torch.bfloat16)
    k = _check_cuda("k", k, torch.bfloat16)
    v = _check_cuda("v", v, torch.bfloat16)
    a = _check_cuda("a", a, torch.bfloat16)
    b = _check_cuda("b", b, torch.bfloat16)
    A_log = _check_cuda("A_log", A_log, torch.float32)
    dt_bias = _check_cuda("dt_bias", dt_bias, torch.float32)
    # read/write slots: int32 or int64 (both the same); scatter slots: int32
    idx_dtype = read_idx.dtype if isinstance(read_idx, torch.Tensor) else torch.int32
    if idx_dtype not in (torch.int32, torch.int64):
        raise TypeError(f"read_idx must be int32 or int64, got {idx_dtype}")
    read_idx = _check_cuda("read_idx", read_idx, idx_dtype)
    write_idx = _check_cuda("write_idx", write_idx, idx_dtype)
    scatter_idx = _check_cuda("scatter_idx", scatter_idx, torch.int32)
    if not state_pool.is_cuda or state_pool.dtype != torch.float32 or state_pool.dim() != 4:
        raise TypeError("state_pool must be a 4-d fp32 CUDA tensor")
    P, HV, Dv, Dk = state_pool.shape
    if state_pool.stride(3) != 1 or state_pool.stride(2) != Dk:
        raise ValueError("state_pool rows must be dense")
    B, T, H, _ = q.shape
    nh = k.shape[2]
    if out is None:
        out = torch.zeros((B, T, HV, Dv), dtype=torch.bfloat16, device=q.device)
    elif (not out.is_contiguous() or out.dtype != torch.bfloat16
          or tuple(out.shape) != (B, T, HV, Dv)):
        raise ValueError("out must be a contiguous bf16 [B, T, HV, Dv] tensor")
    if scale is None:
        scale = 1.0 / math.sqrt(Dk)
    flags = (GDN_DISABLE_STATE_UPDATE if disable_state_update else 0) | \
        (GDN_DECODE_QK_L2NORM if use_qk_l2norm else 0) | \
        (GDN_DECODE_IDX64 if idx_dtype == torch.int64 else 0)
    st = lib().gdn_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(state_pool), P, state_pool.stride(0),
                          state_pool.stride(1), _ptr(read_idx), _ptr(write_idx),
                          _ptr(scatter_idx), _ptr(A_log), _ptr(a), _ptr(dt_bias), _ptr(b),
                          float(scale), _ptr(out), B, T, nh, H, HV, Dk, Dv, flags,
                          _ptr(dev_status), _stream(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_decode")
    return out, state_pool


_CONV_DTYPES = {torch.float32: GDN_F32, torch.bfloat16: GDN_BF16, torch.float16: GDN_F16}


def gdn_conv1d(x, weight, conv_state, slot_idx, row_offsets, out=None, *, write_state: bool = True,
               dev_status=None, stream=None):
    """Causal depthwise conv1d with a slot-indexed window pool (updated in place).

    x: [N, conv_dim]; weight: [conv_dim, K]; conv_state: [max_slots, conv_dim, K-1], all of
    one dtype (fp32, bf16 or fp16); slot_idx: [B] and row_offsets: [B+1], uint32 (int32
    tensors with non-negative values are accepted and reinterpreted).  ``write_state=False``
    only reads the pool.  Returns (out [N, conv_dim], conv_state).
    """
    if x.dtype not in _CONV_DTYPES:
        raise TypeError(f"x must be fp32, bf16 or fp16, got {x.dtype}")
    x = _check_cuda("x", x, x.dtype)
    weight = _check_cuda("weight", weight, x.dtype)
    if x.dim() != 2 or weight.dim() != 2 or weight.shape[0] != x.shape[1]:
        raise ValueError("x must be [N, conv_dim] and weight [conv_dim, K]")
    N, conv_dim = x.shape
    K = weight.shape[1]
    if (not isinstance(conv_state, torch.Tensor) or not conv_state.is_cuda
            or conv_state.dtype != x.dtype or conv_state.dim() != 3
            or tuple(conv_state.shape[1:]) != (conv_dim, K - 1) or not conv_state.is_contiguous()):
        raise ValueError("conv_state must be a contiguous CUDA [max_slots, conv_dim, K-1] tensor "
                         "of x's dtype")
    idx_types = (torch.uint32, torch.int32)
    if slot_idx.dtype not in idx_types or row_offsets.dtype not in idx_types:
        raise TypeError("slot_idx and row_offsets must be uint32 (or int32)")
    slot_idx = _check_cuda("slot_idx", slot_idx)
    row_offsets = _check_cuda("row_offsets", row_offsets)
    B = slot_idx.shape[0]
    if row_offsets.shape != (B + 1,):
        raise ValueError("row_offsets must have B + 1 entries")
    if out is None:
        out = torch.zeros_like(x)
    elif not out.is_contiguous() or out.dtype != x.dtype or out.shape != x.shape:
        raise ValueError("out must be a contiguous tensor shaped and typed like x")
    st = lib().gdn_conv1d(_ptr(x), _ptr(weight), _ptr(conv_state), _ptr(slot_idx),
                          _ptr(row_offsets), _ptr(out), B, N, conv_dim, K, conv_state.shape[0],
                          _CONV_DTYPES[x.dtype], int(bool(write_state)), _ptr(dev_status),
                          _stream(stream))
    if st != GDN_OK:
        raise GdnError(st, "gdn_conv1d")
    return out, conv_state
