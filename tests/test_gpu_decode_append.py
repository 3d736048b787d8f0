"""Parity of the fused decode step, pkv_paged_attn_decode_append (the step's
kv_append and decode in one launch), with the CPU oracle's kv_append followed
by its decode; and bit equality of the pools it leaves with those a separate
pkv_kv_append of the same rows leaves (NaN sentinels of unused slots
included).

Cases: the decode workloads at small sizes over seeds 0-2 (tiny, Qwen3-4B
layer, page-32 fragmented, split-K long contexts), the automatic split, no
split and fixed partitions, every GQA group at d = 64 and 128, lengths at
page and partition edges (a one-key request is its new row alone), an empty
request, a repeated call, and a new row whose page id is out of range.
"""
import numpy as np
import pytest
import torch

from tests.harness import DeviceStep, OracleStep, assert_close, bf16_to_f64, dev_bf16, dev_i32
from workloads import make_workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pkv():
    import paged_kv_attention_37_b200 as m
    assert torch.cuda.is_available()
    m.pkv_device_error_flags(clear=True)
    return m


def new_rows_by_request(w):
    """k_new, v_new [len(decode_ids), Hkv, d] on the device: decode request
    i's new row (zeros for a request that appends none)."""
    dec = list(w.decode_ids)
    k = np.zeros((len(dec), w.num_kv_heads, w.head_dim), np.uint16)
    v = np.zeros_like(k)
    for i, r in enumerate(dec):
        if w.new_lens[r] == 1:
            kr, vr = w.new_rows(r)
            k[i], v[i] = kr[0], vr[0]
    return dev_bf16(k), dev_bf16(v)


def same_bits(a, b):
    return torch.equal(a.view(torch.int16), b.view(torch.int16))


def run_fused_case(pkv, w, partitions=(0,), repeat=1):
    sep = DeviceStep(pkv, w)   # separate kv_append: the pools to match
    fused = DeviceStep(pkv, w)  # same context fill, new rows not yet appended
    sep.append()
    os_ = OracleStep(w)
    os_.append()
    ref, ref_lse, sel = os_.decode()
    k_new, v_new = new_rows_by_request(w)
    dec = list(w.decode_ids)
    for part in partitions:
        for _ in range(repeat):
            lse = torch.full((len(dec), w.num_q_heads), float("nan"), device="cuda")
            out = pkv.pkv_paged_attn_decode_append(fused.q_dec, k_new, v_new, fused.k_pool, fused.v_pool,
                                                   fused.pt_dec, fused.len_dec, w.scale, partition_tokens=part,
                                                   out_lse=lse)
            assert_close(bf16_to_f64(out)[sel], ref[sel], f"{w.name} fused decode partition={part}")
            assert_close(lse.cpu().numpy().astype(np.float64)[sel], ref_lse[sel],
                         f"{w.name} fused decode lse partition={part}")
            assert same_bits(fused.k_pool, sep.k_pool) and same_bits(fused.v_pool, sep.v_pool), \
                f"{w.name} pools after the fused call, partition={part}"
    assert pkv.pkv_device_error_flags(clear=True) == 0


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_fused_tiny(pkv, seed):
    run_fused_case(pkv, make_workload("tiny_decode", seed), partitions=(0, -1, 32))


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_fused_qwen3_small(pkv, seed):
    w = make_workload("qwen3_decode", seed, B=8, len_lo=100, len_hi=1100)
    run_fused_case(pkv, w, partitions=(0, -1, 96, 512))


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_fused_page32_fragmented(pkv, seed):
    w = make_workload("frag_large", seed, B=24, median=300.0, max_len=2000)
    assert w.page_size == 32
    run_fused_case(pkv, w, partitions=(0, -1, 128))


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_fused_splitk(pkv, seed):
    w = make_workload("splitk_long", seed, lens=[4000, 8192 + 13, 20000, 33])
    run_fused_case(pkv, w, partitions=(0, 1024, -1))


def test_fused_edge_lengths(pkv):
    w = make_workload("qwen3_decode", 5, lens=[1, 2, 15, 16, 17, 31, 32, 33, 255, 256, 257])
    run_fused_case(pkv, w, partitions=(0, -1, 32, 256))


@pytest.mark.parametrize("group,d", [(1, 128), (2, 128), (4, 128), (8, 128), (1, 64), (4, 64), (8, 64)])
def test_fused_group_and_head_dim(pkv, group, d):
    w = make_workload("qwen3_decode", 7, B=5, len_lo=20, len_hi=700, num_kv_heads=4,
                      num_q_heads=4 * group, head_dim=d)
    run_fused_case(pkv, w, partitions=(0, -1, 64))


def test_fused_repeated_call(pkv):
    # the second call writes the same row again and reads it from the new rows
    w = make_workload("qwen3_decode", 9, B=6, len_lo=50, len_hi=900)
    run_fused_case(pkv, w, partitions=(0,), repeat=2)


def test_fused_empty_request(pkv):
    # kv_len 0: zero output, lse -inf, nothing appended for that request
    w = make_workload("qwen3_decode", 6, lens=[5, 40, 3])
    fused = DeviceStep(pkv, w)
    before = fused.k_pool.clone()
    k_new, v_new = new_rows_by_request(w)
    lens = dev_i32([5, 0, 3])
    lse = torch.zeros((3, w.num_q_heads), device="cuda")
    out = pkv.pkv_paged_attn_decode_append(fused.q_dec, k_new, v_new, fused.k_pool, fused.v_pool, fused.pt_dec,
                                           lens, w.scale, out_lse=lse)
    assert (bf16_to_f64(out)[1] == 0).all()
    assert torch.isneginf(lse[1]).all() and torch.isfinite(lse[[0, 2]]).all()
    changed = (fused.k_pool.view(torch.int16) != before.view(torch.int16)).any(dim=(1, 2, 3))
    pages = set(torch.nonzero(changed).flatten().tolist())
    assert pages == {int(w.page_table[0][(5 - 1) // w.page_size]), int(w.page_table[2][(3 - 1) // w.page_size])}
    assert pkv.pkv_device_error_flags(clear=True) == 0


def test_fused_bad_page_not_written(pkv):
    # a new row whose page id is out of range is neither written nor read
    # from the pool: the call raises PKV_FLAG_BAD_PAGE and leaves the pools
    w = make_workload("qwen3_decode", 10, lens=[40, 70])
    fused = DeviceStep(pkv, w)
    pt = fused.pt_dec.clone()
    pt[1, (70 - 1) // w.page_size] = w.num_pages + 3
    k_before, v_before = fused.k_pool.clone(), fused.v_pool.clone()
    k_new, v_new = new_rows_by_request(w)
    keep = [0]
    pkv.pkv_paged_attn_decode_append(fused.q_dec[keep], k_new[keep], v_new[keep], fused.k_pool, fused.v_pool,
                                     pt[keep], fused.len_dec[keep], w.scale)
    assert pkv.pkv_device_error_flags(clear=True) == 0
    k_mid, v_mid = fused.k_pool.clone(), fused.v_pool.clone()
    assert not same_bits(k_mid, k_before) and not same_bits(v_mid, v_before)  # request 0's row landed
    pkv.pkv_paged_attn_decode_append(fused.q_dec, k_new, v_new, fused.k_pool, fused.v_pool, pt, fused.len_dec,
                                     w.scale)
    assert pkv.pkv_device_error_flags(clear=True) & pkv.FLAG_BAD_PAGE
    # request 0's row was written again (the same bits); request 1's was not
    # written anywhere
    assert same_bits(fused.k_pool, k_mid) and same_bits(fused.v_pool, v_mid)
