"""Seeded synthetic inputs for block-hybrid attention.

This module draws random tensors and nothing else: it holds none of the layer's arithmetic
(no feature map, no state building, no attention).  Both the float64 oracle and the CUDA
path consume what it returns, so the two sides see bit-identical inputs.

* Every draw comes from numpy's PCG64 ``default_rng`` seeded through ``SeedSequence``; each
  tensor gets its own spawned child stream, in a fixed order, so a tensor's values do not
  depend on the sizes of the tensors drawn before it.
* bf16 inputs are produced by rounding fp32 draws to bfloat16 (round to nearest, ties to
  even).  The returned arrays are float32 holding exactly bf16-representable values.
* Shapes follow the library layout: Q [T, Hq, d], K/V [T, Hkv, d] token-major with request
  r owning rows cu[r]..cu[r+1]-1; W [Hkv, d, F/2]; S [slots, Hkv, F, d]; Z [slots, Hkv, F].

Workload recipes (the serving workload they stand in for is blockwise semi-autoregressive
decoding with 32-token blocks, up to 128 concurrent requests and long prefixes; no prompt
data is used, only shapes and value distributions):
  Q, K, V ~ N(0, 1); W ~ N(0, 1/d); prefix K/V ~ N(0, 1); optional gate alpha ~ N(0, 1).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

__all__ = [
    "bf16_round",
    "bf16_bits",
    "DecodeCase",
    "decode_case",
    "tiny_case",
    "ragged_prefix_lengths",
    "random_states",
]


def bf16_round(x) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returns float32."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    b = x.view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000
    return b.astype(np.uint32).view(np.float32).reshape(x.shape)


def bf16_bits(x) -> np.ndarray:
    """The 16-bit bfloat16 encodings of already bf16-representable float32 values."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def _streams(seed: int, n: int):
    return [np.random.default_rng(s) for s in np.random.SeedSequence(seed).spawn(n)]


@dataclass
class DecodeCase:
    """One decode-step workload: an active block per request plus its committed prefix."""

    R: int
    Hq: int
    Hkv: int
    d: int
    F: int
    dtype: str                      # "bf16" or "f32": storage type of Q, K, V, W, O
    cu_blk: np.ndarray              # [R+1] int32, active-block row offsets
    cu_pre: np.ndarray              # [R+1] int64, prefix row offsets
    W: np.ndarray                   # [Hkv, d, F/2]
    Q: np.ndarray                   # [T, Hq, d]
    K: np.ndarray                   # [T, Hkv, d]
    V: np.ndarray                   # [T, Hkv, d]
    K_pre: np.ndarray               # [P_total, Hkv, d] committed prefix keys
    V_pre: np.ndarray               # [P_total, Hkv, d] committed prefix values
    alpha: np.ndarray | None = None  # [Hq] gate logits, or None for w = 1
    meta: dict = field(default_factory=dict)

    @property
    def T(self) -> int:
        return int(self.cu_blk[-1])

    @property
    def block_lens(self) -> np.ndarray:
        return np.diff(self.cu_blk)

    @property
    def prefix_lens(self) -> np.ndarray:
        return np.diff(self.cu_pre)


def _cast(x, dtype):
    return bf16_round(x) if dtype == "bf16" else np.asarray(x, dtype=np.float32)


def decode_case(R, Hq, Hkv, d, F, block_lens, prefix_lens, seed, dtype="bf16",
                with_alpha=False) -> DecodeCase:
    """Draw one decode-step workload.

    block_lens / prefix_lens: an int (same for every request) or a length-R sequence.
    Draw order (one spawned stream each): W, K_pre, V_pre, Q, K, V, alpha.
    """
    bl = np.broadcast_to(np.asarray(block_lens, dtype=np.int64), (R,))
    pl = np.broadcast_to(np.asarray(prefix_lens, dtype=np.int64), (R,))
    cu_blk = np.concatenate([[0], np.cumsum(bl)]).astype(np.int32)
    cu_pre = np.concatenate([[0], np.cumsum(pl)]).astype(np.int64)
    T, P = int(cu_blk[-1]), int(cu_pre[-1])
    rW, rKp, rVp, rQ, rK, rV, rA = _streams(seed, 7)
    Fh = F // 2
    W = _cast(rW.standard_normal((Hkv, d, Fh), dtype=np.float32) / np.float32(np.sqrt(d)), dtype)
    K_pre = _cast(rKp.standard_normal((P, Hkv, d), dtype=np.float32), dtype)
    V_pre = _cast(rVp.standard_normal((P, Hkv, d), dtype=np.float32), dtype)
    Q = _cast(rQ.standard_normal((T, Hq, d), dtype=np.float32), dtype)
    K = _cast(rK.standard_normal((T, Hkv, d), dtype=np.float32), dtype)
    V = _cast(rV.standard_normal((T, Hkv, d), dtype=np.float32), dtype)
    alpha = rA.standard_normal(Hq).astype(np.float32) if with_alpha else None
    return DecodeCase(R, Hq, Hkv, d, F, dtype, cu_blk, cu_pre, W, Q, K, V, K_pre, V_pre,
                      alpha, dict(seed=seed))


def tiny_case(seed=0, with_alpha=False) -> DecodeCase:
    """Single-head fp32 case: 1 request, d = 16, F = 32, an 8-token block and a 24-token
    (three-block) committed prefix; W ~ N(0, 1/16)."""
    return decode_case(R=1, Hq=1, Hkv=1, d=16, F=32, block_lens=8, prefix_lens=24,
                       seed=seed, dtype="f32", with_alpha=with_alpha)


def ragged_prefix_lengths(R, seed, step=32, max_len=8192) -> np.ndarray:
    """Prefix lengths uniform on {0, step, ..., max_len} (a ragged serving mix)."""
    rng = np.random.default_rng(np.random.SeedSequence(seed).spawn(1)[0])
    return step * rng.integers(0, max_len // step + 1, size=R)


def random_states(slots, Hkv, F, d, prefix_len, seed):
    """Directly drawn fp32 states of the size a prefix of `prefix_len` tokens produces.

    Z ~ prefix_len / (F/2) * U(0.5, 1.5) (positive, like a sum of simplex halves) and
    S ~ N(0, prefix_len / (F/2)^2).  Used to exercise the cross-block read in isolation.
    """
    rS, rZ = _streams(seed, 2)
    Fh = F // 2
    scale = max(prefix_len, 0) / Fh
    Z = (scale * rZ.uniform(0.5, 1.5, size=(slots, Hkv, F))).astype(np.float32)
    S = (np.sqrt(max(prefix_len, 0)) / Fh
         * rS.standard_normal((slots, Hkv, F, d), dtype=np.float32)).astype(np.float32)
    return S, Z
