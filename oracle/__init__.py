"""float64 CPU oracle for the Gated DeltaNet recurrence (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports, links or runs it, and it imports nothing
from the product package: callers hand it numpy arrays.

The arithmetic lives in ``gdn_oracle.c`` (plain C, float64, one token at a
time).  This module compiles it with gcc on first use and wraps its entry
points (prefill, decode, causal conv1d) with ctypes.  See ``gdn_oracle.c`` for the pages each step follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` next to its source (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        D = ctypes.POINTER(ctypes.c_double)
        I32 = ctypes.POINTER(ctypes.c_int32)
        lib.oracle_prefill.restype = None
        lib.oracle_prefill.argtypes = [
            D, D, D, D, D, I32, D, D, D,
            ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_double, ctypes.c_int, ctypes.c_int, D, D, ctypes.c_int, ctypes.c_int,
            ctypes.c_int,
        ]
        lib.oracle_decode.restype = None
        lib.oracle_decode.argtypes = [
            D, D, D, D, D, ctypes.c_int, I32, I32, I32,
            D, D, D, D, ctypes.c_double, D,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        ]
        U32 = ctypes.POINTER(ctypes.c_uint32)
        lib.oracle_conv1d.restype = None
        lib.oracle_conv1d.argtypes = [
            D, D, D, D, U32, U32, D, ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int,
        ]
        lib.oracle_max_threads.restype = ctypes.c_int
        lib.oracle_max_threads.argtypes = []
        _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def _f64(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _i32(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _dp(a):
    return None if a is None else a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _ip(a):
    return None if a is None else a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


RULES = {"gated_delta": 0, "gated": 1, "delta": 2, "linear": 3}


def prefill(q, k, v, g, beta, cu_seqlens=None, initial_state=None, *, B=None,
            scale=1.0, qk_l2norm=False, out=None, threads=None, update_rule="gated_delta",
            gate_activation="none", a_log=None, dt_bias=None, beta_activation="none",
            decay_per_key=False):
    """Sequential recurrence of the log-space form, float64.

    q, k: [N, Hq, Dk]; v: [N, Hv, Dv]; g, beta: [N, Hv] (None where the update
    rule has no decay / no retrieval); cu_seqlens: [B+1] int32 or None (uniform
    packing, needs ``B``); initial_state: [B, Hv, Dv, Dk] or None.
    update_rule: gated_delta | gated | delta | linear; gate_activation: none |
    qwen (needs a_log, dt_bias [Hv]); beta_activation: none | sigmoid.
    decay_per_key: g is [N, Hv, Dk], one log-space decay per key dimension (the op's
    per-key-dimension spelling of ``decay``; the scalar exp(g_t) becomes diag(exp(g_t))
    on the key axis of the state).
    ``out`` (optional, [N, Hv, Dv] float64) supplies the values kept for
    tokens that no request covers.
    Returns (out [N, Hv, Dv], final_state [B, Hv, Dv, Dk]) as float64.
    """
    rule = RULES[update_rule]
    has_decay, has_retr = rule in (0, 1), rule in (0, 2)
    assert (g is not None) == has_decay and (beta is not None) == has_retr
    assert gate_activation in ("none", "qwen") and beta_activation in ("none", "sigmoid")
    qwen = gate_activation == "qwen"
    assert not qwen or (has_decay and a_log is not None and dt_bias is not None)
    q, k, v = map(_f64, (q, k, v))
    g = None if g is None else _f64(g)
    beta = None if beta is None else _f64(beta)
    al = _f64(a_log) if qwen else None
    dtb = _f64(dt_bias) if qwen else None
    N, Hq, Dk = q.shape
    Hv, Dv = v.shape[1], v.shape[2]
    if cu_seqlens is not None:
        cu = _i32(cu_seqlens)
        B = cu.shape[0] - 1
    else:
        cu = None
        assert B is not None and N % B == 0
    if g is not None:
        assert g.shape == ((N, Hv, Dk) if decay_per_key else (N, Hv)), g.shape
    assert not decay_per_key or has_decay
    s0 = None if initial_state is None else _f64(initial_state)
    fs = np.zeros((B, Hv, Dv, Dk), np.float64)
    o = np.zeros((N, Hv, Dv), np.float64) if out is None else _f64(out).copy()
    nt = threads if threads is not None else max_threads()
    _load().oracle_prefill(_dp(q), _dp(k), _dp(v), _dp(g), _dp(beta), _ip(cu), _dp(s0),
                           _dp(fs), _dp(o), B, N, Hq, Hv, Dk, Dv, float(scale),
                           int(bool(qk_l2norm)), rule, _dp(al), _dp(dtb),
                           int(beta_activation == "sigmoid"), int(bool(decay_per_key)),
                           int(nt))
    return o, fs


def decode(q, k, v, pool, read_idx, A_log, a, dt_bias, b, *, write_idx=None,
           scatter_idx=None, scale=None, use_qk_l2norm=True, disable_state_update=False,
           out=None, threads=None):
    """Decode / MTP over a slot pool, float64.

    q: [B, T, H, Dk]; k: [B, T, nh, H, Dk]; v: [B, T, nh, HV, Dv];
    pool: [P, HV, Dv, Dk]; read_idx, write_idx: [B]; scatter_idx: [B, T];
    A_log, dt_bias: [HV]; a: [B, T, HV]; b: [B, T, nh, HV].
    ``scale`` None means 1/sqrt(Dk).  ``out`` supplies the values kept in
    padding rows (zeros when None).
    Returns (out [B, T, HV, Dv], new pool [P, HV, Dv, Dk]) as float64.
    """
    q, k, v = map(_f64, (q, k, v))
    Bn, T, H, Dk = q.shape
    nh = k.shape[2]
    HV, Dv = v.shape[3], v.shape[4]
    pin = _f64(pool)
    pout = pin.copy()
    P = pin.shape[0]
    if scale is None:
        scale = 1.0 / np.sqrt(Dk)
    o = np.zeros((Bn, T, HV, Dv), np.float64) if out is None else _f64(out).copy()
    ri = _i32(read_idx)
    wi = None if write_idx is None else _i32(write_idx)
    si = None if scatter_idx is None else _i32(scatter_idx)
    Al, ab, dtb, bb = map(_f64, (A_log, a, dt_bias, b))
    nt = threads if threads is not None else max_threads()
    _load().oracle_decode(_dp(q), _dp(k), _dp(v), _dp(pin), _dp(pout), P, _ip(ri), _ip(wi),
                          _ip(si), _dp(Al), _dp(ab), _dp(dtb), _dp(bb), float(scale), _dp(o),
                          Bn, T, nh, H, HV, Dk, Dv, int(bool(use_qk_l2norm)),
                          int(bool(disable_state_update)), int(nt))
    return o, pout


def conv1d(x, weight, conv_state, slot_idx, row_offsets, *, write_state=True, out=None):
    """Causal depthwise conv1d with a slot-indexed window pool, float64.

    x: [N, conv_dim]; weight: [conv_dim, K]; conv_state: [max_slots, conv_dim, K-1];
    slot_idx: [B] uint32; row_offsets: [B+1] uint32.  ``out`` supplies the values kept
    in rows no request covers (zeros when None).
    Returns (y [N, conv_dim], new conv_state) as float64; the input pool is not modified.
    """
    x = _f64(x)
    w = _f64(weight)
    pin = _f64(conv_state)
    N, conv_dim = x.shape
    K = w.shape[1]
    assert w.shape == (conv_dim, K) and K >= 1
    assert pin.ndim == 3 and pin.shape[1:] == (conv_dim, K - 1)
    si = np.ascontiguousarray(np.asarray(slot_idx, dtype=np.uint32))
    ro = np.ascontiguousarray(np.asarray(row_offsets, dtype=np.uint32))
    B = si.shape[0]
    assert ro.shape == (B + 1,)
    pout = pin.copy()
    y = np.zeros((N, conv_dim), np.float64) if out is None else _f64(out).copy()
    U32 = ctypes.POINTER(ctypes.c_uint32)
    _load().oracle_conv1d(_dp(x), _dp(w), _dp(pin), _dp(pout), si.ctypes.data_as(U32),
                          ro.ctypes.data_as(U32), _dp(y), int(B), int(N), int(conv_dim), int(K),
                          int(pin.shape[0]), int(bool(write_state)))
    return y, pout
