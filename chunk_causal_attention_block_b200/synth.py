"""Seeded synthetic inputs for wave rounds (host side, NumPy).

This module only draws numbers; it holds none of the attention, RoPE or ring
arithmetic.  Both the CPU oracle's tests and the GPU path take their inputs
from here, and the library's device generator (``wf_synth_fill``) implements
the same definition so that full-size inputs can be drawn on the device
bit-identically.

Definition
----------
* Generator: SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom
  number generators", OOPSLA 2014) with Stafford's "Mix13" output finaliser:
  output ``i`` of a stream with state ``key`` is ``mix64(key + (i+1)*G)``,
  ``G = 0x9E3779B97F4A7C15``.
* Stream key of (seed, tensor id, tag):
  ``k0 = mix64(seed*G)``, ``k1 = mix64(k0 ^ (tensor*0xD1B54A32D192ED03))``,
  ``key = mix64(k1 ^ (tag*G))`` (tag as 64-bit two's complement; the prefill
  of the ring uses tag -1, round r uses tag r).
* Element (global chunk n, token j, head h, dim d) has flat index
  ``e = ((n*C + j)*H + h)*D + d`` and consumes outputs 3e, 3e+1, 3e+2; their
  twelve 16-bit halves u_0..u_11 give the Irwin-Hall(12) draw
  ``z = (sum(u) + 6 - 6*2^16) / 2^16`` which is exact in fp32 (|numerator| <
  2^19) and approximately N(0,1) (mean 0, variance 1 - 2^-32, tails at +-6).
* bf16 tensors hold RNE(z); the per-head key scale of the 14B-shaped round is
  ``s_h = (2^16 + 3*x_h) / 2^17`` in [0.5, 2) with x_h the low 16 bits of
  output h of the (tensor=KSCALE, tag=0) stream, applied as one fp32 multiply
  before the bf16 rounding.

The seed default 42 is the plugin's ``base_seed`` (Causal Forcing plugin page,
"Configuration" table).
"""
from __future__ import annotations

import numpy as np

GOLDEN = np.uint64(0x9E3779B97F4A7C15)
TENSOR_MUL = np.uint64(0xD1B54A32D192ED03)
M1 = np.uint64(0xBF58476D1CE4E5B9)
M2 = np.uint64(0x94D049BB133111EB)

TENSOR_Q, TENSOR_K, TENSOR_V, TENSOR_KSCALE = 1, 2, 3, 4
PREFILL_TAG = -1
DEFAULT_SEED = 42


def mix64(z):
    """Stafford Mix13 finaliser on uint64 (wrapping arithmetic)."""
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * M1
        z = (z ^ (z >> np.uint64(27))) * M2
    return z ^ (z >> np.uint64(31))


def _u64(x: int) -> np.uint64:
    return np.uint64(int(x) & 0xFFFFFFFFFFFFFFFF)


def stream_key(seed: int, tensor: int, tag: int) -> np.uint64:
    with np.errstate(over="ignore"):
        k0 = mix64(_u64(seed) * GOLDEN)
        k1 = mix64(k0 ^ (_u64(tensor) * TENSOR_MUL))
        return mix64(k1 ^ (_u64(tag) * GOLDEN))


def splitmix_outputs(key: np.uint64, idx) -> np.ndarray:
    """Outputs ``idx`` (uint64 array) of the SplitMix64 stream with state ``key``."""
    idx = np.asarray(idx, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return mix64(key + (idx + np.uint64(1)) * GOLDEN)


def irwin_hall12(key: np.uint64, e) -> np.ndarray:
    """fp32 Irwin-Hall(12) draws for flat element indices ``e`` (uint64)."""
    e = np.asarray(e, dtype=np.uint64)
    acc = np.zeros(e.shape, dtype=np.int64)
    mask = np.uint64(0xFFFF)
    with np.errstate(over="ignore"):
        base = e * np.uint64(3)
    for m in range(3):
        w = splitmix_outputs(key, base + np.uint64(m))
        for s in (0, 16, 32, 48):
            acc += ((w >> np.uint64(s)) & mask).astype(np.int64)
    num = acc + 6 - 6 * 65536
    return (num.astype(np.float32) / np.float32(65536.0)).astype(np.float32)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (b + np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def key_scales(seed: int, H: int) -> np.ndarray:
    """Per-head fp32 key scale s_h in [0.5, 2) (14B-shaped round)."""
    key = stream_key(seed, TENSOR_KSCALE, 0)
    x = (splitmix_outputs(key, np.arange(H, dtype=np.uint64)) & np.uint64(0xFFFF)).astype(np.int64)
    return ((65536 + 3 * x).astype(np.float32) / np.float32(131072.0)).astype(np.float32)


def chunk_values(seed: int, tensor: int, tag: int, n: int, C: int, H: int, D: int,
                 dtype: str = "bf16", heads=None, tokens=None, kscale: bool = False) -> np.ndarray:
    """Values of one chunk-tensor, shape [len(tokens), len(heads), D].

    ``dtype`` "bf16" returns fp32 arrays holding bf16-representable values;
    "f32" returns the raw fp32 draws.  ``heads``/``tokens`` select a subset
    (default all) so that sampled checks draw only what they need.
    """
    heads = np.arange(H) if heads is None else np.asarray(heads)
    tokens = np.arange(C) if tokens is None else np.asarray(tokens)
    j = tokens.astype(np.uint64)[:, None, None]
    h = heads.astype(np.uint64)[None, :, None]
    d = np.arange(D, dtype=np.uint64)[None, None, :]
    with np.errstate(over="ignore"):
        e = ((_u64(n) * _u64(C) + j) * _u64(H) + h) * _u64(D) + d
    z = irwin_hall12(stream_key(seed, tensor, tag), e)
    if kscale:
        s = key_scales(seed, H)[heads][None, :, None]
        z = (z * s).astype(np.float32)
    if dtype == "f32":
        return z
    if dtype != "bf16":
        raise ValueError(f"unknown dtype {dtype!r}")
    return bf16_bits_to_f32(f32_to_bf16_bits(z))


def kv_tag(n: int, n0: int, first_n0: int) -> int:
    """Tag of the K/V that chunk n holds during the round whose oldest in-round chunk is n0.

    A rollout starts with round 0 at ``n0 = first_n0`` and round r has
    ``n0 = first_n0 + r``; chunks below ``first_n0`` were written by the
    prefill (tag -1).  A chunk is re-written in every round it is in-round and
    is last in-round in the round where it is the oldest member, so in-round
    chunks carry the current round's tag and cache chunks n >= first_n0 the
    tag n - first_n0.
    """
    if n >= n0:
        return n0 - first_n0
    return n - first_n0 if n >= first_n0 else PREFILL_TAG
