"""Plant plausible mistakes in the prologue and copy-on-write oracles (on the
CPU) and check that their pins catch every one."""
import types

import numpy as np
import pytest

import oracle.prefix_pages as OX
import oracle.prologue as OP
from tests.test_oracle_pins_prefix import ALL_CHECKS as PREFIX_CHECKS
from tests.test_oracle_pins_prologue import ALL_CHECKS as PROLOGUE_CHECKS


def _rope_interleaved(x, pos, theta):
    # pairs (2i, 2i+1) instead of (i, i + d/2)
    d = x.shape[-1]
    y = x.reshape(x.shape[:-1] + (d // 2, 2))
    y = np.concatenate([y[..., 0], y[..., 1]], axis=-1)
    r = OP.__dict__["_orig_rope"](y, pos, theta)
    h = d // 2
    return np.stack([r[..., :h], r[..., h:]], axis=-1).reshape(x.shape)


def _rope_sign(x, pos, theta):
    return OP.__dict__["_orig_rope"](x, -np.asarray(pos), theta)


def _rope_freq(x, pos, theta):
    d = x.shape[-1]
    half = d // 2
    inv = theta ** (-np.arange(half, dtype=np.float64) / d)  # missing factor 2
    ang = np.asarray(pos, dtype=np.float64)[..., None] * inv
    while ang.ndim < x.ndim:
        ang = ang[..., None, :]
    a, b = x[..., :half], x[..., half:]
    return np.concatenate([a * np.cos(ang) - b * np.sin(ang), b * np.cos(ang) + a * np.sin(ang)], axis=-1)


def _rms_no_weight(x, w, eps):
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def _rms_mean_abs(x, w, eps):
    return x / (np.mean(np.abs(x), axis=-1, keepdims=True) + eps) * w


def _round_truncate(x):
    b = np.asarray(x, dtype=np.float64).astype(np.float32).view(np.uint32) >> 16
    return b.astype(np.uint16)


def _qknr_swapped(q_bits, k_bits, positions, q_w_bits, k_w_bits, eps, theta):
    # the order reversed: RoPE, then the weighted norm
    pos = np.asarray(positions, dtype=np.int64)
    f = OP.bf16_bits_to_f64
    q = OP.rms_norm(OP.rope(f(q_bits), pos[:, None], theta), f(q_w_bits), eps)
    k = OP.rms_norm(OP.rope(f(k_bits), pos[:, None], theta), f(k_w_bits), eps)
    return q, k


def _cow_copy_all_rows(k_pool, v_pool, page_table, refcount, free_pages, k_new, v_new, token_req, token_pos, P):
    used = 0
    for t in range(len(token_req)):
        r, pos = int(token_req[t]), int(token_pos[t])
        e, off = divmod(pos, P)
        if (t == 0 or int(token_req[t - 1]) != r or off == 0) and refcount[page_table[r][e]] > 1:
            fresh = int(free_pages[used]); used += 1
            page = int(page_table[r][e])
            k_pool[fresh] = k_pool[page]; v_pool[fresh] = v_pool[page]
            refcount[page] -= 1; refcount[fresh] = 1; page_table[r][e] = fresh
        page = int(page_table[r][e])
        k_pool[page, :, off] = k_new[t]; v_pool[page, :, off] = v_new[t]
    return used


def _cow_never(k_pool, v_pool, page_table, refcount, free_pages, k_new, v_new, token_req, token_pos, P):
    for t in range(len(token_req)):
        r, pos = int(token_req[t]), int(token_pos[t])
        page = int(page_table[r][pos // P])
        k_pool[page, :, pos % P] = k_new[t]; v_pool[page, :, pos % P] = v_new[t]
    return 0


def _cow_no_decrement(k_pool, v_pool, page_table, refcount, free_pages, k_new, v_new, token_req, token_pos, P):
    rc = refcount.copy()
    used = OX.__dict__["_orig_cow"](k_pool, v_pool, page_table, rc, free_pages, k_new, v_new,
                                     token_req, token_pos, P)
    changed = rc != refcount
    refcount[changed] = np.maximum(rc[changed], refcount[changed])  # shared pages keep their count
    return used


def _cow_always(k_pool, v_pool, page_table, refcount, free_pages, k_new, v_new, token_req, token_pos, P):
    rc = refcount.copy()
    rc[rc == 1] = 2  # every page treated as shared
    used = OX.__dict__["_orig_cow"](k_pool, v_pool, page_table, rc, free_pages, k_new, v_new,
                                     token_req, token_pos, P)
    refcount[:] = np.where(rc == 2, refcount, rc)
    return used


PROLOGUE = {
    "rope_interleaved_pairs": ("rope", _rope_interleaved),
    "rope_wrong_sign": ("rope", _rope_sign),
    "rope_frequency": ("rope", _rope_freq),
    "rms_weight_dropped": ("rms_norm", _rms_no_weight),
    "rms_mean_abs": ("rms_norm", _rms_mean_abs),
    "bf16_truncate": ("f64_to_bf16_bits", _round_truncate),
    "rope_before_norm": ("qk_norm_rope", _qknr_swapped),
}
PREFIX = {
    "cow_copies_whole_page": _cow_copy_all_rows,
    "cow_never": _cow_never,
    "cow_keeps_shared_count": _cow_no_decrement,
    "cow_every_page": _cow_always,
}


def _caught(checks, mod):
    caught = []
    for check in checks:
        try:
            check(mod)
        except Exception as e:  # an assertion, or a crash on a wrong index
            caught.append((check.__name__, type(e).__name__))
    return caught


@pytest.mark.parametrize("name", sorted(PROLOGUE))
def test_prologue_pins_catch_mutation(name, monkeypatch):
    attr, fn = PROLOGUE[name]
    monkeypatch.setitem(OP.__dict__, "_orig_rope", OP.rope)
    monkeypatch.setattr(OP, attr, fn)
    assert _caught(PROLOGUE_CHECKS, OP), f"no pin catches mutation {name}"


@pytest.mark.parametrize("name", sorted(PREFIX))
def test_prefix_pins_catch_mutation(name, monkeypatch):
    monkeypatch.setitem(OX.__dict__, "_orig_cow", OX.kv_append_cow)
    monkeypatch.setattr(OX, "kv_append_cow", PREFIX[name])
    assert _caught(PREFIX_CHECKS, OX), f"no pin catches mutation {name}"
