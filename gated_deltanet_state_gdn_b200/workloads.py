"""Seeded synthetic inputs for the Gated DeltaNet prefill and decode paths.

This module only draws numbers: it holds none of the recurrence's arithmetic
and imports neither the CUDA library nor the oracle.  The same tensors (CPU,
in their storage dtype) feed both the GPU path and the float64 oracle, so the
two always see identical bytes.

Recipes follow the workloads the pages describe: head dim 128, GQA 16 -> 32
heads, ragged cu_seqlens packing, an fp32 slot pool for decode.  Random values
are drawn with numpy ``default_rng(seed)`` in float32 and cast to bf16 with
round-to-nearest-even (torch's ``.to``).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch


def _bf16(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)


def _f32(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))


def _f16(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.float16)


def _unit_rows(x: np.ndarray) -> np.ndarray:
    """Scale each last-axis vector to unit L2 norm (input recipe, fp32)."""
    n = np.sqrt(np.sum(x.astype(np.float64) ** 2, axis=-1, keepdims=True))
    return (x / np.maximum(n, 1e-30)).astype(np.float32)


def _neg_softplus(x: np.ndarray) -> np.ndarray:
    return (-np.logaddexp(0.0, x.astype(np.float64))).astype(np.float32)


def _sigmoid(x: np.ndarray) -> np.ndarray:
    return (1.0 / (1.0 + np.exp(-x.astype(np.float64)))).astype(np.float32)


@dataclass
class PrefillCase:
    """Inputs of one gdn_prefill call (CPU tensors)."""
    name: str
    q: torch.Tensor            # [N, Hq, Dk]
    k: torch.Tensor            # [N, Hq, Dk]
    v: torch.Tensor            # [N, Hv, Dv]
    g: torch.Tensor            # [N, Hv] fp32, log-space decay
    beta: torch.Tensor         # [N, Hv] fp32
    cu_seqlens: Optional[torch.Tensor]      # [B+1] int32 or None (uniform)
    initial_state: Optional[torch.Tensor]   # [B, Hv, Dv, Dk] fp32 or None
    B: int
    scale: float
    qk_l2norm: bool
    meta: dict = field(default_factory=dict)

    @property
    def N(self) -> int:
        return self.q.shape[0]

    @property
    def dims(self):
        return self.q.shape[1], self.v.shape[1], self.q.shape[2], self.v.shape[2]


@dataclass
class DecodeCase:
    """Inputs of one gdn_decode call (CPU tensors)."""
    name: str
    q: torch.Tensor            # [B, T, H, Dk] bf16
    k: torch.Tensor            # [B, T, nh, H, Dk] bf16
    v: torch.Tensor            # [B, T, nh, HV, Dv] bf16
    pool: torch.Tensor         # [P, HV, Dv, Dk] fp32
    read_idx: torch.Tensor     # [B] int32
    write_idx: Optional[torch.Tensor]     # [B] int32 or None
    scatter_idx: Optional[torch.Tensor]   # [B, T] int32 or None
    A_log: torch.Tensor        # [HV] fp32
    a: torch.Tensor            # [B, T, HV] bf16
    dt_bias: torch.Tensor      # [HV] fp32
    b: torch.Tensor            # [B, T, nh, HV] bf16
    scale: float
    use_qk_l2norm: bool
    disable_state_update: bool = False
    meta: dict = field(default_factory=dict)


def make_prefill(seed: int, lengths, Hq: int, Hv: int, Dk: int, Dv: int, *,
                 dtype=torch.bfloat16, uniform: bool = False, init_std: Optional[float] = 0.02,
                 qk_l2norm: bool = True, host_norm_qk: bool = False, scale: Optional[float] = None,
                 gate: str = "softplus", name: str = "prefill",
                 decay_per_key: bool = False) -> PrefillCase:
    """Generic ragged prefill case.

    gate="softplus": g = -softplus(N(0,1)), beta = sigmoid(N(0,1)).
    gate="uniform":  gamma ~ U[0.8, 1] passed as g = ln(gamma), beta ~ U[0, 1].
    decay_per_key: g has one value per key dimension, [N, Hv, Dk], drawn the same way
    element by element.
    host_norm_qk: q and k are unit-normalised in fp32 before the cast.
    uniform=True: every length must be equal and cu_seqlens is None.
    """
    gshape = lambda: (N, Hv, Dk) if decay_per_key else (N, Hv)
    rng = np.random.default_rng(seed)
    lengths = [int(x) for x in lengths]
    B = len(lengths)
    N = int(sum(max(0, x) for x in lengths))
    q = rng.standard_normal((N, Hq, Dk), dtype=np.float32)
    k = rng.standard_normal((N, Hq, Dk), dtype=np.float32)
    v = rng.standard_normal((N, Hv, Dv), dtype=np.float32)
    if host_norm_qk:
        q = _unit_rows(q)
        k = _unit_rows(k)
    if gate == "softplus":
        g = _neg_softplus(rng.standard_normal(gshape(), dtype=np.float32))
        beta = _sigmoid(rng.standard_normal((N, Hv), dtype=np.float32))
    elif gate == "uniform":
        gamma = rng.uniform(0.8, 1.0, gshape())
        g = np.log(gamma).astype(np.float32)
        beta = rng.uniform(0.0, 1.0, (N, Hv)).astype(np.float32)
    else:
        raise ValueError(gate)
    init = None
    if init_std is not None:
        init = _f32(rng.standard_normal((B, Hv, Dv, Dk), dtype=np.float32) * np.float32(init_std))
    if uniform:
        assert len(set(lengths)) == 1
        cu = None
    else:
        cu = torch.from_numpy(np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32))
    conv = {torch.bfloat16: _bf16, torch.float16: _f16}.get(dtype, _f32)
    return PrefillCase(name=name, q=conv(q), k=conv(k), v=conv(v), g=_f32(g), beta=_f32(beta),
                       cu_seqlens=cu, initial_state=init, B=B,
                       scale=(1.0 / np.sqrt(Dk)) if scale is None else float(scale),
                       qk_l2norm=qk_l2norm, meta={"lengths": lengths})


def tiny_oracle_case(seed: int = 1) -> PrefillCase:
    """B=2, S=64, one head, Dk=Dv=16, fp32; unit keys; gamma ~ U[0.8,1]; beta ~ U[0,1];
    zero initial state; scale 1 (the gamma-form statement has no scale)."""
    rng = np.random.default_rng(seed)
    B, S, D = 2, 64, 16
    q = rng.standard_normal((B * S, 1, D), dtype=np.float32)
    k = _unit_rows(rng.standard_normal((B * S, 1, D), dtype=np.float32))
    v = rng.standard_normal((B * S, 1, D), dtype=np.float32)
    gamma = rng.uniform(0.8, 1.0, (B * S, 1))
    beta = rng.uniform(0.0, 1.0, (B * S, 1)).astype(np.float32)
    g = np.log(gamma).astype(np.float32)
    return PrefillCase(name="tiny_oracle_B2_S64_D16_fp32", q=_f32(q), k=_f32(k), v=_f32(v),
                       g=_f32(g), beta=_f32(beta), cu_seqlens=None, initial_state=None, B=B,
                       scale=1.0, qk_l2norm=False, meta={"S": S})


def ragged_prefill_case(seed: int = 2, n_req: int = 8, max_len: int = 4096,
                        decay_per_key: bool = False) -> PrefillCase:
    """8 requests, lengths U[1, 4096] packed by cu_seqlens; Hq=16, Hv=32, D=128, bf16,
    qk_l2_norm=1, g=-softplus(N(0,1)), beta=sigmoid(N(0,1)), initial state N(0, 0.02^2).
    decay_per_key: g is [N, 32, 128], -softplus(N(0,1)) in every key dimension."""
    rng = np.random.default_rng(seed)
    lengths = rng.integers(1, max_len + 1, n_req).tolist()
    tag = "_per_key_decay" if decay_per_key else ""
    c = make_prefill(seed + 1000, lengths, 16, 32, 128, 128, init_std=0.02, qk_l2norm=True,
                     name=f"ragged_prefill_{n_req}req_U1-{max_len}_Hq16_Hv32_D128_bf16{tag}",
                     decay_per_key=decay_per_key)
    return c


def long_prefill_case(seed: int = 3, S: int = 32768) -> PrefillCase:
    """B=1, S=32768, Hq=16, Hv=32, D=128, bf16; q/k unit-normalised on the host (norm flag off);
    zero initial state."""
    return make_prefill(seed, [S], 16, 32, 128, 128, init_std=None, qk_l2norm=False,
                        host_norm_qk=True, name=f"long_prefill_S{S}_Hq16_Hv32_D128_bf16")


def make_decode(seed: int, *, P: int, B: int, T: int, nh: int, H: int, Dv: int, Dk: int = 128,
                pad_frac: float = 0.0, write_mode: str = "distinct", scatter: bool = False,
                host_norm_qk: bool = False, use_qk_l2norm: bool = True, pool_std: float = 0.02,
                name: str = "decode") -> DecodeCase:
    """Decode/MTP case over a pool of P slots.

    write_mode: "distinct" (write slots disjoint from every read slot),
                "same" (write = read), "none" (write_idx None, i.e. = read).
    scatter: per-token scatter slots [B, T], distinct and disjoint from the read slots.
    """
    rng = np.random.default_rng(seed)
    HV = H
    perm = rng.permutation(P).astype(np.int32)
    read = perm[:B].copy()
    nxt = B
    write = None
    if write_mode == "distinct":
        write = perm[nxt:nxt + B].copy()
        nxt += B
    elif write_mode == "same":
        write = read.copy()
    sc = None
    if scatter:
        sc = perm[nxt:nxt + B * T].reshape(B, T).copy()
        nxt += B * T
    assert nxt <= P, "pool too small for distinct slots"
    n_pad = int(round(pad_frac * B))
    if n_pad:
        pad_rows = rng.choice(B, n_pad, replace=False)
        read[pad_rows] = -1
        if write is not None:
            write[pad_rows] = -1
    q = rng.standard_normal((B, T, H, Dk), dtype=np.float32)
    k = rng.standard_normal((B, T, nh, H, Dk), dtype=np.float32)
    v = rng.standard_normal((B, T, nh, HV, Dv), dtype=np.float32)
    if host_norm_qk:
        q = _unit_rows(q)
        k = _unit_rows(k)
    pool = rng.standard_normal((P, HV, Dv, Dk), dtype=np.float32)
    pool *= np.float32(pool_std)
    A_log = rng.uniform(-2.0, 1.0, HV).astype(np.float32)
    dt_bias = (rng.standard_normal(HV, dtype=np.float32) * np.float32(0.5))
    a = rng.standard_normal((B, T, HV), dtype=np.float32)
    bg = rng.standard_normal((B, T, nh, HV), dtype=np.float32)
    return DecodeCase(name=name, q=_bf16(q), k=_bf16(k), v=_bf16(v), pool=torch.from_numpy(pool),
                      read_idx=torch.from_numpy(read),
                      write_idx=None if write is None else torch.from_numpy(write),
                      scatter_idx=None if sc is None else torch.from_numpy(sc),
                      A_log=_f32(A_log), a=_bf16(a), dt_bias=_f32(dt_bias), b=_bf16(bg),
                      scale=1.0 / np.sqrt(Dk), use_qk_l2norm=use_qk_l2norm,
                      meta={"n_pad": n_pad})


def decode_pool_case(seed: int = 4, write_mode: str = "distinct") -> DecodeCase:
    """Pool [1024, 32, 128, 128] fp32 ~ N(0, 0.02); B=256, T=1, nh=1, H=HV=32; read/write slots
    from a seeded permutation; 5% padding rows (-1); use_qk_l2norm."""
    return make_decode(seed, P=1024, B=256, T=1, nh=1, H=32, Dv=128, pad_frac=0.05,
                       write_mode=write_mode, name="decode_pool_P1024_B256_H32_Dv128_T1")


def mtp_case(seed: int = 5) -> DecodeCase:
    """Pool [512, 16, 64, 128]; B=64, T=4, nh=2, H=HV=16, Dv=64; q/k unit-normalised on the host
    and use_qk_l2norm on; per-token scatter into distinct slots."""
    return make_decode(seed, P=512, B=64, T=4, nh=2, H=16, Dv=64, write_mode="none", scatter=True,
                       host_norm_qk=True, name="mtp_P512_B64_T4_nh2_H16_Dv64")


@dataclass
class Conv1dCase:
    """Inputs of one gdn_conv1d call (CPU tensors)."""
    name: str
    x: torch.Tensor            # [N, conv_dim]
    weight: torch.Tensor       # [conv_dim, K]
    conv_state: torch.Tensor   # [max_slots, conv_dim, K-1]
    slot_idx: torch.Tensor     # [B] uint32
    row_offsets: torch.Tensor  # [B+1] uint32
    meta: dict = field(default_factory=dict)

    @property
    def B(self) -> int:
        return int(self.slot_idx.shape[0])

    @property
    def N(self) -> int:
        return int(self.x.shape[0])


def make_conv1d(seed: int, lengths, conv_dim: int, K: int, max_slots: int, *,
                dtype: torch.dtype = torch.bfloat16, N: Optional[int] = None, lead: int = 0,
                name: str = "conv1d") -> Conv1dCase:
    """Ragged conv1d case: x ~ N(0, 1) (the projected q/k/v rows), weights ~ U(-1/sqrt(K),
    1/sqrt(K)) (the default init of a depthwise conv with K taps), pool ~ N(0, 1); the
    requests take distinct slots from a seeded permutation.  Requests are packed from row
    ``lead``; rows before it and after the last request (up to ``N``) belong to none."""
    rng = np.random.default_rng(seed)
    lengths = [int(L) for L in lengths]
    total = lead + sum(lengths)
    N = total if N is None else N
    assert N >= total and len(lengths) <= max_slots
    x = rng.standard_normal((N, conv_dim), dtype=np.float32)
    bound = np.float32(1.0 / np.sqrt(K))
    w = rng.uniform(-bound, bound, (conv_dim, K)).astype(np.float32)
    pool = rng.standard_normal((max_slots, conv_dim, K - 1), dtype=np.float32)
    slots = rng.permutation(max_slots)[:len(lengths)].astype(np.uint32)
    off = (lead + np.concatenate([[0], np.cumsum(lengths)])).astype(np.uint32)
    cast = {torch.bfloat16: _bf16, torch.float16: _f16, torch.float32: _f32}[dtype]
    return Conv1dCase(name=name, x=cast(x), weight=cast(w), conv_state=cast(pool),
                      slot_idx=torch.from_numpy(slots), row_offsets=torch.from_numpy(off),
                      meta={"lengths": lengths})


def conv_ragged_case(seed: int = 6, n_req: int = 8, max_len: int = 4096) -> Conv1dCase:
    """The ragged prefill's token mix (lengths U[1, 4096], the same seed draw) through the
    conv that feeds it: conv_dim = 2*16*128 + 32*128 = 8192 (q, k, v rows), K = 4, bf16,
    a pool of 64 slots."""
    rng = np.random.default_rng(2)
    lengths = rng.integers(1, max_len + 1, n_req).tolist()
    return make_conv1d(seed, lengths, 8192, 4, 64,
                       name=f"conv1d_ragged_{n_req}req_U1-{max_len}_C8192_K4_bf16")


def conv_decode_case(seed: int = 7, B: int = 256, max_slots: int = 1024) -> Conv1dCase:
    """One token for each of 256 requests (a decode step) through the conv: conv_dim 8192,
    K = 4, bf16, a pool of 1024 slots, distinct slots."""
    return make_conv1d(seed, [1] * B, 8192, 4, max_slots,
                       name=f"conv1d_decode_B{B}_P{max_slots}_C8192_K4_bf16")
