"""Plant plausible mistakes in the oracle (on the CPU) and check that the pins
catch every one: a pin suite that lets a wrong GQA mapping, a dropped scale or
an off-by-one causal mask through would not be pinning anything."""
import numpy as np
import pytest

import oracle.paged_attention as O
from tests.test_oracle_pins import ALL_CHECKS


def _softmax_unnormalised(s, v):
    m = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e @ v, (m + np.log(e.sum(-1, keepdims=True)))[..., 0]


def _softmax_lse_sign(s, v):
    if s.shape[-1] == 0:
        return np.zeros(s.shape[:-1] + (v.shape[-1],)), np.full(s.shape[:-1], -np.inf)
    m = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(-1, keepdims=True)
    return (e / l) @ v, (m - np.log(l))[..., 0]


def _combine_plain_mean(part_o, part_lse, num_splits):
    B, hq, _, d = part_o.shape
    out = np.zeros((B, hq, d))
    for r in range(B):
        out[r] = part_o[r, :, :num_splits[r]].mean(axis=1)
    return out, np.max(np.nan_to_num(part_lse, nan=-np.inf), axis=2)


def _append_shifted(k_pool, v_pool, k_new, v_new, slot_mapping, page_size):
    for t, slot in enumerate(slot_mapping):
        if slot < 0:
            continue
        page, off = divmod(int(slot), page_size)
        k_pool[page, :, (off + 1) % page_size] = k_new[t]
        v_pool[page, :, (off + 1) % page_size] = v_new[t]


MUTATIONS = {
    "gqa_modulo": ("_kv_head_of", lambda h, g: h % g),
    "page_offset_swapped": ("_page_and_offset", lambda j, p: (j % p, j // p)),
    "causal_strict": ("_visible", lambda k, q: k < q),
    "causal_off_by_one": ("_visible", lambda k, q: k <= q + 1),
    "scale_dropped": ("_scores", lambda q, k, s: q @ k.T),
    "keys_reversed": ("_scores", lambda q, k, s: s * (q @ k[::-1].T)),
    "softmax_unnormalised": ("_softmax_attend", _softmax_unnormalised),
    "lse_sign": ("_softmax_attend", _softmax_lse_sign),
    "combine_plain_mean": ("split_k_combine", _combine_plain_mean),
    "append_offset_shift": ("kv_append", _append_shifted),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_mutation(name, monkeypatch):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(O, attr, fn)
    caught = []
    for check in ALL_CHECKS:
        try:
            check(O)
        except Exception as e:  # an assertion, or a crash on a wrong index
            caught.append((check.__name__, type(e).__name__))
    assert caught, f"no pin catches mutation {name}"
