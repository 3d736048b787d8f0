"""Plain fp64 CPU oracle for the step before attention: per-head RMSNorm of
the projected Q and K rows (Qwen3's QK norm), rotary position encoding, and
the append of the resulting K row (and the V row, unchanged) into the paged
pool.

TEST INFRASTRUCTURE ONLY.  Only tests, the smoke check and the benchmark's
CPU-baseline leg may import this module; the library never does.  It shares
no code with the CUDA path.

What it computes, and where the pages define it:

* Q and K each get their own RMSNorm after the projection, then RoPE encodes
  the position -- tiny-llm source reading, week 1 (the Qwen3 attention
  interface: GQA, "independent RMSNorm of Q and K after projection", RoPE);
  the course outline, chapters 1.2 (RoPE) and 1.4 (RMSNorm).
* RMSNorm, RoPE and the K/V write fused into one kernel to save memory round
  trips -- tiny-llm blog, week 2 ("fused operators: RMSNorm, RoPE ... in a
  single kernel"); tiny-llm source reading, week 2 (Fast RMSNorm and Fast
  RoPE in the M4 Pro table, and "implement or fuse RMSNorm, RoPE ...").

Readings taken where the pages are silent:
  R11 RMSNorm of a head row x (d values) with weight w (d values, one per
      element, shared by all heads): y = x / sqrt(mean(x^2) + eps) * w.
  R12 RoPE pairs element i with element i + d/2 (the "rotate half"
      convention of the Qwen3 and Llama reference code) and turns the pair by
      the angle pos * theta^(-2i/d): (a, b) -> (a cos - b sin, b cos + a sin).
  R13 the order is norm, then RoPE; V is not transformed.
  R14 the position of a row is given explicitly (R2: a decode token sits at
      kv_len - 1, chunk row i at c + i).
The oracle works in fp64 and rounds once, to nearest even, where a bf16 value
is stored.
"""
from __future__ import annotations

import numpy as np

from .paged_attention import bf16_bits_to_f64


def f64_to_bf16_bits(x) -> np.ndarray:
    """Round fp64 values to the nearest bfloat16 (ties to even), as uint16
    bit patterns.  One rounding straight from fp64 (no fp32 step).  Finite
    normal inputs in bf16's range only."""
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros(x.shape, dtype=np.uint16)
    nz = x != 0
    m, e = np.frexp(np.abs(x[nz]))            # |x| = m * 2^e, m in [0.5, 1)
    q = np.rint(m * 256.0)                     # 8 significant bits, ties to even
    v = np.ldexp(q / 256.0, e)                 # the rounded magnitude
    bits = (v.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    bits |= np.where(x[nz] < 0, np.uint16(0x8000), np.uint16(0))
    out[nz] = bits
    out[~nz] = np.where(np.signbit(x[~nz]), 0x8000, 0).astype(np.uint16)
    return out


def rms_norm(x: np.ndarray, w: np.ndarray, eps: float) -> np.ndarray:
    """R11: x [..., d] / sqrt(mean(x^2) + eps) * w [d], in fp64."""
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * w


def rope(x: np.ndarray, pos, theta: float) -> np.ndarray:
    """R12: rotate element pairs (i, i + d/2) of x [..., d] by pos * theta^(-2i/d).

    pos broadcasts against x's leading dimensions (one position per row)."""
    d = x.shape[-1]
    half = d // 2
    i = np.arange(half, dtype=np.float64)
    inv_freq = theta ** (-2.0 * i / d)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * inv_freq     # [..., d/2]
    while ang.ndim < x.ndim:
        ang = ang[..., None, :]
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., :half], x[..., half:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


def qk_norm_rope(q_bits, k_bits, positions, q_w_bits, k_w_bits, eps: float, theta: float):
    """R13: the normalised and rotated rows, in fp64.

    q_bits [T][Hq][d], k_bits [T][Hkv][d], weights [d] (bf16 bits);
    positions [T].  Returns (q [T][Hq][d], k [T][Hkv][d]) fp64."""
    pos = np.asarray(positions, dtype=np.int64)
    q = rms_norm(bf16_bits_to_f64(q_bits), bf16_bits_to_f64(q_w_bits), eps)
    k = rms_norm(bf16_bits_to_f64(k_bits), bf16_bits_to_f64(k_w_bits), eps)
    return rope(q, pos[:, None], theta), rope(k, pos[:, None], theta)


def qk_norm_rope_append(k_pool, v_pool, q_bits, k_bits, v_bits, q_w_bits, k_w_bits, positions,
                        slot_mapping, page_size: int, eps: float, theta: float):
    """The fused prologue: returns the rotated queries (fp64 [T][Hq][d]) and
    writes, for every row t with slot_mapping[t] != -1, the rotated K row
    (rounded to bf16) and the V row (its bits, unchanged) into the pools at
    that slot (slot = page * P + offset).  Pools are uint16 bf16 bit arrays
    [num_pages][Hkv][P][d], modified in place."""
    q, k = qk_norm_rope(q_bits, k_bits, positions, q_w_bits, k_w_bits, eps, theta)
    k_store = f64_to_bf16_bits(k)
    for t in range(len(slot_mapping)):
        slot = int(slot_mapping[t])
        if slot == -1:
            continue
        page, off = divmod(slot, page_size)
        k_pool[page, :, off, :] = k_store[t]
        v_pool[page, :, off, :] = v_bits[t]
    return q, k
