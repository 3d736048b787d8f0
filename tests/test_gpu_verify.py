"""Parity of split-K short-chunk attention (pkv_paged_attn_verify, the verify
step of speculative decoding) through the C ABI with the CPU oracle.

The rows and their causal masking are those of chunked prefill, so the
oracle is oracle.chunked_prefill_attention; outputs must be within 1e-2 max
abs and 1e-3 mean abs.  Cases: 2-16 rows per request over contexts up to
40 000 keys, automatic and fixed partitions (including partitions shorter
than a chunk), every GQA group size at d = 64 and 128, page 32, a chunk at
context 0, one-row chunks (which must agree with decode), and rows past the
last chunk left untouched.
"""
import numpy as np
import pytest
import torch

from tests.harness import DeviceStep, OracleStep, assert_close, bf16_to_f64, dev_i32
from workloads import make_workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pkv():
    import paged_kv_attention_37_b200 as m
    assert torch.cuda.is_available()
    m.pkv_device_error_flags(clear=True)
    return m


def verify_case(pkv, w, partitions=(0,), what="verify"):
    ds, os_ = DeviceStep(pkv, w), OracleStep(w)
    ds.append()
    os_.append()
    ref, _, rows = os_.prefill()
    pre = list(w.prefill_ids)
    max_q = int(w.new_lens[pre].max())
    for part in partitions:
        out = torch.full_like(ds.q_pre, 3.0)
        pkv.pkv_paged_attn_verify(ds.q_pre, ds.cu_q, ds.ctx_pre, ds.k_pool, ds.v_pool, ds.pt_pre, w.scale,
                                  max_q, partition_tokens=part, out=out)
        assert_close(bf16_to_f64(out)[rows], ref[rows], f"{what} partition={part}")
    assert pkv.pkv_device_error_flags(clear=True) == 0
    return ds, os_


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_verify_batch(pkv, seed):
    rng = np.random.default_rng(seed)
    n = 12
    chunks = rng.integers(2, 17, n)
    ctxs = rng.integers(100, 5000, n)
    w = make_workload("mixed_prefill_decode", seed, n_prefill=n, chunks=list(chunks), ctxs=list(ctxs), n_decode=1)
    verify_case(pkv, w, partitions=(0, 64, 512, 4096))


def test_verify_long_context(pkv):
    w = make_workload("mixed_prefill_decode", 3, n_prefill=3, chunks=[8, 16, 3], ctxs=[40000, 17000, 123],
                      n_decode=1)
    verify_case(pkv, w, partitions=(0, 1024))


def test_verify_partition_inside_chunk(pkv):
    # chunks longer than a partition: rows of one chunk end in different splits
    w = make_workload("mixed_prefill_decode", 4, n_prefill=3, chunks=[150, 70, 16], ctxs=[0, 30, 200],
                      n_decode=1)
    verify_case(pkv, w, partitions=(64, 128, 0))


@pytest.mark.parametrize("group,d", [(1, 128), (2, 128), (4, 128), (8, 128), (1, 64), (4, 64), (8, 64)])
def test_verify_group_and_head_dim(pkv, group, d):
    w = make_workload("mixed_prefill_decode", 5, n_prefill=4, chunks=[4, 9, 16, 2], ctxs=[700, 2500, 64, 1],
                      n_decode=1, num_kv_heads=2, num_q_heads=2 * group, head_dim=d)
    verify_case(pkv, w, partitions=(0, 256))


def test_verify_page32(pkv):
    w = make_workload("mixed_prefill_decode", 6, n_prefill=4, chunks=[5, 12, 16, 7], ctxs=[900, 3000, 31, 0],
                      n_decode=1, page_size=32)
    verify_case(pkv, w, partitions=(0, 128))


def test_verify_one_row_matches_decode(pkv):
    # one row per request is decode: the same keys, the same query
    w = make_workload("mixed_prefill_decode", 7, n_prefill=6, chunks=[1] * 6,
                      ctxs=[99, 1000, 3000, 15, 4095, 600], n_decode=1)
    ds, _ = verify_case(pkv, w, partitions=(0, 512))
    pre = list(w.prefill_ids)
    q = ds.q_pre.view(len(pre), w.num_q_heads, w.head_dim)
    lens = dev_i32(w.kv_lens[pre])
    dec = pkv.pkv_paged_attn_decode(q, ds.k_pool, ds.v_pool, ds.pt_pre, lens, w.scale)
    ver = pkv.pkv_paged_attn_verify(ds.q_pre, ds.cu_q, ds.ctx_pre, ds.k_pool, ds.v_pool, ds.pt_pre, w.scale, 1)
    assert np.abs(bf16_to_f64(dec) - bf16_to_f64(ver.view_as(dec))).max() <= 1e-2


def test_verify_rows_past_the_chunks_untouched(pkv):
    w = make_workload("mixed_prefill_decode", 8, n_prefill=3, chunks=[4, 6, 5], ctxs=[3000, 10, 800], n_decode=1)
    ds = DeviceStep(pkv, w)
    ds.append()
    pre = list(w.prefill_ids)
    total = int(w.new_lens[pre].sum())
    q = torch.zeros((total + 5, w.num_q_heads, w.head_dim), dtype=torch.bfloat16, device="cuda")
    q[:total] = ds.q_pre
    out = torch.full_like(q, 5.0)
    pkv.pkv_paged_attn_verify(q, ds.cu_q, ds.ctx_pre, ds.k_pool, ds.v_pool, ds.pt_pre, w.scale, 6,
                              partition_tokens=512, out=out)
    assert (out[total:] == 5.0).all()
    assert pkv.pkv_device_error_flags(clear=True) == 0


def _splits_of_rows(pkv, w, ds, total_q, max_q):
    """Run the automatic verify call on an explicit workspace and return the
    splits the call gave each chunk row (the workspace's leading int32s)."""
    max_kv = ds.pt_pre.shape[1] * w.page_size
    ws = pkv.verify_workspace(total_q, w.num_q_heads, w.head_dim, max_kv, 0, ds.q_pre.device)
    out = torch.empty_like(ds.q_pre)
    pkv.pkv_paged_attn_verify(ds.q_pre, ds.cu_q, ds.ctx_pre, ds.k_pool, ds.v_pool, ds.pt_pre, w.scale, max_q,
                              partition_tokens=0, workspace=ws, out=out)
    torch.cuda.synchronize()
    return out, ws[: total_q * 4].view(torch.int32).cpu().numpy()


def test_verify_automatic_split_choice(pkv):
    # few (request, KV head) units: the automatic partition splits the long
    # requests so that the GPU's CTA slots fill; many units: no split at all
    slots = 2 * torch.cuda.get_device_properties(0).multi_processor_count
    few = make_workload("mixed_prefill_decode", 9, n_prefill=3, chunks=[4, 4, 2], ctxs=[20000, 9000, 100],
                        n_decode=1)
    assert few.num_kv_heads * 3 < slots
    many = make_workload("spec_verify", 1)
    assert many.num_kv_heads * len(many.prefill_ids) >= slots
    for w, expect_split in ((few, True), (many, False)):
        ds, os_ = DeviceStep(pkv, w), OracleStep(w)
        ds.append()
        os_.append()
        ref, _, rows = os_.prefill()
        pre = list(w.prefill_ids)
        total_q, max_q = int(w.new_lens[pre].sum()), int(w.new_lens[pre].max())
        out, splits = _splits_of_rows(pkv, w, ds, total_q, max_q)
        assert_close(bf16_to_f64(out)[rows], ref[rows], f"automatic verify ({'few' if expect_split else 'many'})")
        if expect_split:
            assert splits.max() > 1 and splits.min() >= 1
        else:
            assert (splits == 1).all()
        assert pkv.pkv_device_error_flags(clear=True) == 0
