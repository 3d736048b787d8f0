"""Parity of the single-launch mixed batch (pkv_paged_attn_mixed: prefill
chunks and decode requests pulled from one work queue by persistent CTAs)
through the C ABI with the CPU oracle.

Chunk rows follow oracle.chunked_prefill_attention and decode rows
oracle.decode_attention, within 1e-2 max abs and 1e-3 mean abs.  Cases: the
mixed workload at small sizes over seeds 0-2, every GQA group size (group 8
takes the two-kernel path) at d = 64 and 128, page 32, one part empty, a
workspace reused across calls (the queue counters return to zero), and the
full-size workload in the benchmark's configuration with sampled requests.
"""
import numpy as np
import pytest
import torch

from tests.harness import DeviceStep, OracleStep, assert_close, bf16_to_f64
from workloads import make_workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pkv():
    import paged_kv_attention_37_b200 as m
    assert torch.cuda.is_available()
    m.pkv_device_error_flags(clear=True)
    return m


def mixed_case(pkv, w, ids=None, calls=1, what="mixed"):
    ds, os_ = DeviceStep(pkv, w, host_ids=ids), OracleStep(w, ids)
    ds.append()
    os_.append()
    ref_p, _, rows = os_.prefill()
    ref_d, ref_lse, sel = os_.decode()
    pre, dec = list(w.prefill_ids), list(w.decode_ids)
    ws = pkv.mixed_workspace(len(dec), w.num_q_heads, w.head_dim, w.max_pages * w.page_size)
    for call in range(calls):
        lse = torch.full((len(dec), w.num_q_heads), float("nan"), device="cuda")
        out_p, out_d = pkv.pkv_paged_attn_mixed(ds.q_pre, ds.cu_q, ds.ctx_pre, ds.pt_pre,
                                                int(w.new_lens[pre].max()), ds.q_dec, ds.pt_dec, ds.len_dec,
                                                ds.k_pool, ds.v_pool, w.scale, workspace=ws, out_lse_dec=lse)
        assert_close(bf16_to_f64(out_p)[rows], ref_p[rows], f"{what} chunk rows, call {call}")
        assert_close(bf16_to_f64(out_d)[sel], ref_d[sel], f"{what} decode rows, call {call}")
        assert_close(lse.cpu().numpy().astype(np.float64)[sel], ref_lse[sel], f"{what} decode lse, call {call}")
    assert (ws[:16] == 0).all(), "the queue and scheduling counters are left at zero"
    assert pkv.pkv_device_error_flags(clear=True) == 0


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_mixed_small(pkv, seed):
    w = make_workload("mixed_prefill_decode", seed, n_prefill=3, chunks=[512, 100, 37], ctx_hi=1000,
                      n_decode=9, len_lo=50, len_hi=2000)
    mixed_case(pkv, w, calls=2)


@pytest.mark.parametrize("group,d", [(1, 128), (2, 128), (8, 128), (1, 64), (4, 64), (8, 64)])
def test_mixed_group_and_head_dim(pkv, group, d):
    w = make_workload("mixed_prefill_decode", 9, n_prefill=2, chunks=[150, 77], ctx_hi=400, n_decode=6,
                      len_lo=30, len_hi=1500, num_kv_heads=2, num_q_heads=2 * group, head_dim=d)
    mixed_case(pkv, w)


def test_mixed_page32(pkv):
    w = make_workload("mixed_prefill_decode", 10, n_prefill=2, chunks=[256, 90], ctx_hi=700, n_decode=5,
                      len_lo=40, len_hi=3000, page_size=32)
    mixed_case(pkv, w)


def test_mixed_long_decode_tree(pkv):
    # a decode request long enough for a multi-level merge tree next to chunks
    w = make_workload("mixed_prefill_decode", 11, n_prefill=2, chunks=[64, 200], ctxs=[3000, 10], n_decode=3,
                      len_lo=30000, len_hi=40000)
    mixed_case(pkv, w)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_mixed_full_sampled(pkv, seed):
    w = make_workload("mixed_prefill_decode", seed)
    pre = list(w.prefill_ids)
    by_ctx = sorted(pre, key=lambda r: w.ctx_lens[r])
    dec = sorted(list(w.decode_ids), key=lambda r: w.kv_lens[r])
    rng = np.random.default_rng(seed)
    ids = [by_ctx[0], by_ctx[-1], dec[0], dec[-1]] + [int(x) for x in rng.choice(dec, 3, replace=False)]
    mixed_case(pkv, w, ids=ids, calls=2, what=f"full mixed seed {seed}")
