"""Pins for the prologue oracle (QK RMSNorm, RoPE, fused append), checked
against things other than itself.

Each check_* function takes the oracle module so that the mutation tests can
rerun it against copies with planted mistakes.  The pins:

* bf16 rounding: explicit bit patterns (ties to even) and, for random values,
  that the result is the nearer of its two bf16 neighbours;
* RMSNorm: torch.nn.functional.rms_norm (a library routine) in fp64; unit
  RMS and scale invariance;
* RoPE: for d = 2 it is multiplication by e^(i pos) in the complex plane
  (numpy complex arithmetic); on unit vectors it shows which elements pair
  and the sign of the turn; position 0 is the identity; pair norms and
  dot products under a common shift are preserved;
* the composite: torch's rms_norm followed by complex multiplication of the
  pairs (x_i + i x_{i+d/2}) by e^(i pos theta^(-2i/d));
* the fused append: V rows copied bit for bit, K rows the rounded composite,
  slot -1 skipped, other slots untouched.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle.prologue as OP
from oracle.paged_attention import bf16_bits_to_f64
from workloads import f32_to_bf16_bits


def rand_bits(rng, shape, scale=1.0):
    return f32_to_bf16_bits((scale * rng.standard_normal(shape)).astype(np.float32))


# -------------------------------------------------------------- rounding
def check_bf16_rounding(o):
    one = 1.0
    cases = {
        1.0: 0x3F80, -2.0: 0xC000, 0.0: 0x0000,
        one + 2.0 ** -8: 0x3F80,                  # tie: to the even 1.0
        one + 3 * 2.0 ** -8: 0x3F82,              # tie: to the even 1 + 2^-6
        one + 2.0 ** -8 + 2.0 ** -20: 0x3F81,     # just above the tie
        0.1: 0x3DCD, -1.0e-3: 0xBA83, 3.0e5: 0x4892,   # 3e5 = 2^18 * (1 + 18.48/128)
    }
    for x, want in cases.items():
        got = int(o.f64_to_bf16_bits(np.array([x]))[0])
        assert got == want, (x, hex(got), hex(want))
    rng = np.random.default_rng(0)
    x = rng.standard_normal(4000) * np.exp(rng.uniform(-20, 20, 4000))
    b = o.f64_to_bf16_bits(x).astype(np.int64)
    v = bf16_bits_to_f64(b.astype(np.uint16))
    # the nearer of the two neighbours (same sign, one bit pattern apart)
    up = bf16_bits_to_f64((b + 1).astype(np.uint16))
    dn = bf16_bits_to_f64((b - 1).astype(np.uint16))
    assert (np.abs(v - x) <= np.abs(up - x)).all() and (np.abs(v - x) <= np.abs(dn - x)).all()
    # bf16 values come back unchanged
    rb = rand_bits(rng, 3000, 5.0)
    assert np.array_equal(o.f64_to_bf16_bits(bf16_bits_to_f64(rb)), rb)


def test_bf16_rounding():
    check_bf16_rounding(OP)


# --------------------------------------------------------------- RMSNorm
def check_rms_norm(o):
    rng = np.random.default_rng(1)
    x = rng.standard_normal((5, 3, 64)) * 3
    w = rng.uniform(0.5, 1.5, 64)
    eps = 1e-6
    ref = F.rms_norm(torch.from_numpy(x), (64,), torch.from_numpy(w), eps).numpy()
    assert np.abs(o.rms_norm(x, w, eps) - ref).max() < 1e-12
    y = o.rms_norm(x, np.ones(64), 0.0)
    assert np.abs(np.mean(y * y, axis=-1) - 1).max() < 1e-12
    assert np.abs(o.rms_norm(7.5 * x, w, 0.0) - o.rms_norm(x, w, 0.0)).max() < 1e-12


def test_rms_norm():
    check_rms_norm(OP)


# ------------------------------------------------------------------ RoPE
def check_rope(o):
    rng = np.random.default_rng(2)
    # d = 2: one pair, frequency 1: multiplication by e^(i pos)
    x = rng.standard_normal((50, 2))
    pos = rng.integers(0, 100000, 50)
    z = (x[:, 0] + 1j * x[:, 1]) * np.exp(1j * pos.astype(np.float64))
    got = o.rope(x, pos, 10000.0)
    assert np.abs(got[:, 0] - z.real).max() < 1e-9 and np.abs(got[:, 1] - z.imag).max() < 1e-9
    # unit vectors: element i pairs with i + d/2; the first of a pair turns
    # towards the second (a -> (cos, sin)), the second away from the first
    d, theta, p = 8, 100.0, 3
    for i in range(d // 2):
        f = theta ** (-2.0 * i / d)
        e = np.zeros(d); e[i] = 1.0
        r = o.rope(e[None], np.array([p]), theta)[0]
        want = np.zeros(d); want[i] = np.cos(p * f); want[i + d // 2] = np.sin(p * f)
        assert np.abs(r - want).max() < 1e-12, i
        e = np.zeros(d); e[i + d // 2] = 1.0
        r = o.rope(e[None], np.array([p]), theta)[0]
        want = np.zeros(d); want[i] = -np.sin(p * f); want[i + d // 2] = np.cos(p * f)
        assert np.abs(r - want).max() < 1e-12, i
    # position 0 is the identity; pair norms are kept
    x = rng.standard_normal((7, 4, 128))
    assert np.array_equal(o.rope(x, np.zeros((7, 1), np.int64), 1e6), x)
    pos = rng.integers(0, 131072, (7, 1))
    y = o.rope(x, pos, 1e6)
    h = 64
    assert np.abs(np.hypot(y[..., :h], y[..., h:]) - np.hypot(x[..., :h], x[..., h:])).max() < 1e-9
    # a common shift of both positions keeps every dot product
    q, k = rng.standard_normal(128), rng.standard_normal(128)
    for m, n, s in ((5, 2, 100), (1000, 10, 7), (0, 40000, 3000)):
        a = o.rope(q[None], np.array([m]), 1e4)[0] @ o.rope(k[None], np.array([n]), 1e4)[0]
        b = o.rope(q[None], np.array([m + s]), 1e4)[0] @ o.rope(k[None], np.array([n + s]), 1e4)[0]
        assert abs(a - b) < 1e-9


def test_rope():
    check_rope(OP)


# ------------------------------------------------------------- composite
def _composite_reference(x_bits, w_bits, pos, eps, theta):
    """torch rms_norm, then each pair (x_i, x_{i+d/2}) as a complex number
    times e^(i pos theta^(-2i/d))."""
    x = torch.from_numpy(bf16_bits_to_f64(x_bits))
    d = x.shape[-1]
    y = F.rms_norm(x, (d,), torch.from_numpy(bf16_bits_to_f64(w_bits)), eps).numpy()
    h = d // 2
    z = y[..., :h] + 1j * y[..., h:]
    f = theta ** (-np.arange(0, d, 2, dtype=np.float64) / d)
    z = z * np.exp(1j * pos.astype(np.float64)[:, None, None] * f)
    return np.concatenate([z.real, z.imag], axis=-1)


def check_qk_norm_rope(o):
    rng = np.random.default_rng(3)
    T, hq, hkv, d = 6, 8, 2, 128
    q, k = rand_bits(rng, (T, hq, d), 2.0), rand_bits(rng, (T, hkv, d), 0.5)
    wq = f32_to_bf16_bits((1 + 0.2 * rng.standard_normal(d)).astype(np.float32))
    wk = f32_to_bf16_bits((1 + 0.2 * rng.standard_normal(d)).astype(np.float32))
    pos = np.array([0, 1, 17, 4095, 65536, 131071])
    eps, theta = 1e-6, 1e6
    gq, gk = o.qk_norm_rope(q, k, pos, wq, wk, eps, theta)
    assert np.abs(gq - _composite_reference(q, wq, pos, eps, theta)).max() < 1e-8
    assert np.abs(gk - _composite_reference(k, wk, pos, eps, theta)).max() < 1e-8
    # unit weights, eps 0: every row keeps RMS 1 through the rotation
    ones = f32_to_bf16_bits(np.ones(d, np.float32))
    gq, _ = o.qk_norm_rope(q, k, pos, ones, ones, 0.0, theta)
    assert np.abs(np.sqrt(np.mean(gq * gq, axis=-1)) - 1).max() < 1e-12


def test_qk_norm_rope():
    check_qk_norm_rope(OP)


def check_fused_append(o):
    rng = np.random.default_rng(4)
    T, hq, hkv, d, P = 5, 4, 2, 64, 16
    q, k, v = rand_bits(rng, (T, hq, d)), rand_bits(rng, (T, hkv, d)), rand_bits(rng, (T, hkv, d))
    wq = f32_to_bf16_bits((1 + 0.1 * rng.standard_normal(d)).astype(np.float32))
    wk = f32_to_bf16_bits((1 + 0.1 * rng.standard_normal(d)).astype(np.float32))
    pos = np.array([3, 40, 41, 7, 900])
    slots = np.array([2 * P + 3, -1, 5 * P + 15, 0, 3 * P + 1], np.int32)
    kp = np.full((6, hkv, P, d), 0x7FC0, np.uint16)
    vp = kp.copy()
    qo, ko = o.qk_norm_rope_append(kp, vp, q, k, v, wq, wk, pos, slots, P, 1e-6, 1e6)
    ref_q = _composite_reference(q, wq, pos, 1e-6, 1e6)
    ref_k = _composite_reference(k, wk, pos, 1e-6, 1e6)
    assert np.abs(qo - ref_q).max() < 1e-8 and np.abs(ko - ref_k).max() < 1e-8
    written = np.zeros((6, P), bool)
    for t, s in enumerate(slots):
        if s < 0:
            continue
        pg, off = divmod(int(s), P)
        written[pg, off] = True
        assert np.array_equal(vp[pg, :, off], v[t])
        kb = bf16_bits_to_f64(kp[pg, :, off])
        # stored K: the composite within half a bf16 step (half a step is
        # at most 2^-8 of the value, at the bottom of a binade)
        assert (np.abs(kb - ref_k[t]) <= 2.0 ** -8 * np.abs(ref_k[t])).all()
    for pg in range(6):
        for off in range(P):
            if not written[pg, off]:
                assert (kp[pg, :, off] == 0x7FC0).all() and (vp[pg, :, off] == 0x7FC0).all()


def test_fused_append():
    check_fused_append(OP)


ALL_CHECKS = [check_bf16_rounding, check_rms_norm, check_rope, check_qk_norm_rope, check_fused_append]
