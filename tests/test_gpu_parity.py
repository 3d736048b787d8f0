"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

kv_append must match the oracle bit for bit; attention outputs (bf16) must be
within 1e-2 max abs and 1e-3 mean abs of the oracle's fp64 result, and the
decode lse within the same bounds.  Small variants of every workload run in
full; the full-size workloads run in the launch configuration the benchmark
times, with the oracle checking a sample of requests.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.harness import (MAX_ABS, DeviceStep, OracleStep, assert_close, bf16_to_f64, dev_bf16,
                           dev_i32, host_bits)
from workloads import make_workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pkv():
    import paged_kv_attention_37_b200 as m
    assert torch.cuda.is_available()
    m.pkv_device_error_flags(clear=True)
    return m


def check_no_flags(pkv):
    flags = pkv.pkv_device_error_flags(clear=True)
    assert flags == 0, f"device error flags {flags:#x}"


def check_pool_bits(ds: DeviceStep, os_: OracleStep):
    kd, vd = host_bits(ds.k_pool), host_bits(ds.v_pool)
    used = os_.used_pages
    assert np.array_equal(kd[used], os_.k_pool), "k_pool differs from the oracle"
    assert np.array_equal(vd[used], os_.v_pool), "v_pool differs from the oracle"


def run_decode_case(pkv, w, ids=None, partitions=(0,), check_pool=True):
    ds = DeviceStep(pkv, w, host_ids=ids)
    os_ = OracleStep(w, ids)
    ds.append()
    os_.append()
    if check_pool:
        check_pool_bits(ds, os_)
    ref, ref_lse, sel = os_.decode()
    dec = list(w.decode_ids)
    for part in partitions:
        lse = torch.full((len(dec), w.num_q_heads), float("nan"), device="cuda")
        out = ds.decode(partition=part, out_lse=lse)
        got = bf16_to_f64(out)
        assert_close(got[sel], ref[sel], f"{w.name} decode partition={part}")
        assert_close(lse.cpu().numpy().astype(np.float64)[sel], ref_lse[sel],
                     f"{w.name} decode lse partition={part}")
    check_no_flags(pkv)
    return ds, os_


# ------------------------------------------------------------- kv_append
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_kv_append_bit_exact_tiny(pkv, seed):
    w = make_workload("tiny_decode", seed)
    ds = DeviceStep(pkv, w)
    os_ = OracleStep(w)
    ds.append()
    os_.append()
    check_pool_bits(ds, os_)
    # pages outside every table keep their NaN sentinel bits
    unused = np.setdiff1d(np.arange(w.num_pages), os_.used_pages)
    assert (host_bits(ds.k_pool)[unused] == 0x7FC0).all()
    check_no_flags(pkv)


def test_kv_append_skip_and_special_bits(pkv):
    P, hkv, d = 16, 2, 64
    kp = torch.zeros((6, hkv, P, d), dtype=torch.bfloat16, device="cuda")
    vp = torch.zeros_like(kp)
    rng = np.random.default_rng(0)
    k = rng.integers(0, 1 << 16, size=(5, hkv, d), dtype=np.uint16)
    k[0, 0, :4] = [0x7F81, 0x8000, 0x0001, 0xFF80]  # sNaN, -0, denormal, -inf
    v = rng.integers(0, 1 << 16, size=(5, hkv, d), dtype=np.uint16)
    slots = np.array([5 * P + 15, -1, 0, 3 * P + 7, -1], np.int32)
    pkv.pkv_kv_append(dev_bf16(k), dev_bf16(v), dev_i32(slots), kp, vp)
    ek = np.zeros((6, hkv, P, d), np.uint16)
    ev = np.zeros_like(ek)
    oracle.kv_append(ek, ev, k, v, slots, P)
    assert np.array_equal(host_bits(kp), ek) and np.array_equal(host_bits(vp), ev)
    check_no_flags(pkv)


def test_kv_append_out_of_range_slot_flags(pkv):
    kp = torch.zeros((2, 1, 16, 64), dtype=torch.bfloat16, device="cuda")
    vp = torch.zeros_like(kp)
    k = torch.ones((2, 1, 64), dtype=torch.bfloat16, device="cuda")
    pkv.pkv_kv_append(k, k, dev_i32([3, 2 * 16]), kp, vp)  # slot 32 is past the pool
    flags = pkv.pkv_device_error_flags(clear=True)
    assert flags & pkv.FLAG_BAD_SLOT
    got = host_bits(kp)
    assert (got[0, 0, 3] == 0x3F80).all() and (got.reshape(-1) != 0).sum() == 64


def test_kv_append_negative_slots(pkv):
    # -1 is padding (skipped, no flag); any other negative slot is not a slot
    # of the pool: the row is skipped and PKV_FLAG_BAD_SLOT raised
    kp = torch.zeros((2, 1, 16, 64), dtype=torch.bfloat16, device="cuda")
    vp = torch.zeros_like(kp)
    k = torch.ones((3, 1, 64), dtype=torch.bfloat16, device="cuda")
    pkv.pkv_kv_append(k, k, dev_i32([-1, 5, -1]), kp, vp)
    assert pkv.pkv_device_error_flags(clear=True) == 0
    pkv.pkv_kv_append(k, k, dev_i32([-7, 6, -2]), kp, vp)
    assert pkv.pkv_device_error_flags(clear=True) & pkv.FLAG_BAD_SLOT
    got = host_bits(kp).reshape(2 * 16, 64)
    assert (got[5] == 0x3F80).all() and (got[6] == 0x3F80).all()
    assert (np.delete(got, [5, 6], axis=0) == 0).all()


# ------------------------------------------------------------------ decode
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_decode_tiny(pkv, seed):
    run_decode_case(pkv, make_workload("tiny_decode", seed), partitions=(0, -1, 32, 64))


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_decode_qwen3_small(pkv, seed):
    w = make_workload("qwen3_decode", seed, B=8, len_lo=100, len_hi=1100)
    run_decode_case(pkv, w, partitions=(0, -1, 32, 96, 256, 512))


def test_decode_edge_lengths(pkv):
    # one key, a page boundary on either side, the last slot of a page, and
    # a length of exactly one partition
    w = make_workload("qwen3_decode", 5, lens=[1, 2, 15, 16, 17, 31, 32, 33, 255, 256, 257])
    run_decode_case(pkv, w, partitions=(0, -1, 32, 256))


def test_decode_empty_request(pkv):
    # kv_len 0 gives a zero output and lse -inf
    w = make_workload("qwen3_decode", 6, lens=[5, 40, 3])
    ds = DeviceStep(pkv, w)
    ds.append()
    lens = dev_i32([5, 0, 3])
    lse = torch.zeros((3, w.num_q_heads), device="cuda")
    out = pkv.pkv_paged_attn_decode(ds.q_dec, ds.k_pool, ds.v_pool, ds.pt_dec, lens, w.scale,
                                    out_lse=lse)
    assert (bf16_to_f64(out)[1] == 0).all()
    assert torch.isneginf(lse[1]).all() and torch.isfinite(lse[[0, 2]]).all()
    check_no_flags(pkv)


@pytest.mark.parametrize("group,d", [(1, 128), (2, 128), (8, 128), (1, 64), (2, 64), (4, 64), (8, 64)])
def test_decode_group_and_head_dim(pkv, group, d):
    w = make_workload("qwen3_decode", 7, B=5, len_lo=20, len_hi=700, num_kv_heads=4,
                      num_q_heads=4 * group, head_dim=d)
    run_decode_case(pkv, w, partitions=(0, -1, 64))


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_decode_page32_fragmented_small(pkv, seed):
    w = make_workload("frag_large", seed, B=24, median=300.0, max_len=2000)
    assert w.page_size == 32
    run_decode_case(pkv, w, partitions=(0, -1, 128))


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_decode_splitk_small(pkv, seed):
    w = make_workload("splitk_long", seed, lens=[4000, 8192 + 13, 20000, 33])
    run_decode_case(pkv, w, partitions=(0, 512, 1024, 2048, 4096, -1))


@pytest.mark.parametrize("d,L", [(128, 900), (128, 1100), (128, 8100), (128, 8400), (128, 66000),
                                 (64, 1900), (64, 2200), (64, 33000)])
def test_decode_auto_merge_tree_levels(pkv, d, L):
    # one request and one KV head: the automatic split cuts it into slices of
    # about 128 tokens.  With a fan-in of 8 (d = 128) these lengths give about
    # 7, 9, 63, 66 and 516 pieces, merge trees of one, two, two, three and four
    # levels; with 16 (d = 64), about 15, 17 and 258 pieces: one, two, three.
    w = make_workload("qwen3_decode", 31, lens=[L], num_kv_heads=1, num_q_heads=4, head_dim=d)
    run_decode_case(pkv, w, partitions=(0,))


def test_decode_reuses_workspace(pkv):
    # the scheduling counters in the workspace must return to zero each call
    w = make_workload("qwen3_decode", 8, B=6, len_lo=300, len_hi=3000)
    ds = DeviceStep(pkv, w)
    ds.append()
    ws = pkv.decode_workspace(w.B, w.num_q_heads, w.head_dim, w.max_pages * w.page_size, 0)
    first = ds.decode(partition=0, workspace=ws).clone()
    for part in (0, 256, 0):
        again = ds.decode(partition=part, workspace=ws)
        assert np.abs(bf16_to_f64(again) - bf16_to_f64(first)).max() <= MAX_ABS
    assert (ws[:8] == 0).all()
    check_no_flags(pkv)


def test_decode_workspace_survives_batch_growth(pkv):
    # a larger batch moves the workspace's later regions, so its counters land
    # where a smaller batch left split counts and partials; the library must
    # clear them before the larger call
    small = make_workload("qwen3_decode", 21, B=5, len_lo=300, len_hi=3000)
    big = make_workload("qwen3_decode", 22, B=12, len_lo=300, len_hi=3000)
    max_kv = max(small.max_pages * small.page_size, big.max_pages * big.page_size)
    ws = pkv.decode_workspace(big.B, big.num_q_heads, big.head_dim, max_kv, 0)
    ds_small, ds_big = DeviceStep(pkv, small), DeviceStep(pkv, big)
    ds_small.append()
    ds_big.append()
    ref = ds_big.decode(partition=0).clone()  # a fresh workspace of its own
    for part in (0, 512, 0):
        ds_small.decode(partition=part, workspace=ws)
    got = ds_big.decode(partition=0, workspace=ws)
    assert np.abs(bf16_to_f64(got) - bf16_to_f64(ref)).max() <= MAX_ABS
    check_no_flags(pkv)


@pytest.mark.parametrize("name,over", [
    ("tiny_decode", {}),
    ("qwen3_decode", dict(B=8, len_lo=100, len_hi=1100)),
    ("qwen3_decode", dict(lens=[1, 2, 15, 16, 17, 31, 32, 33, 255, 256, 257])),
    ("splitk_long", dict(lens=[4000, 8192 + 13, 20000, 33])),
    ("frag_large", dict(B=24, median=300.0, max_len=2000)),
    ("qwen3_decode", dict(B=5, len_lo=20, len_hi=700, num_kv_heads=4, num_q_heads=32, head_dim=64)),
])
def test_decode_metadata_ready(pkv, name, over):
    # the plan and first page-table reads run before the wait on the kernel
    # ahead (here the append, launched just before): same results
    w = make_workload(name, 13, **over)
    ds, os_ = DeviceStep(pkv, w), OracleStep(w)
    os_.append()
    ref, ref_lse, sel = os_.decode()
    dec = list(w.decode_ids)
    ws = pkv.decode_workspace(len(dec), w.num_q_heads, w.head_dim, w.max_pages * w.page_size, 0)
    for rep in range(2):
        ds.append()
        lse = torch.full((len(dec), w.num_q_heads), float("nan"), device="cuda")
        out = pkv.pkv_paged_attn_decode_flags(ds.q_dec, ds.k_pool, ds.v_pool, ds.pt_dec, ds.len_dec, w.scale,
                                              0, workspace=ws, out_lse=lse, flags=pkv.DECODE_METADATA_READY)
        assert_close(bf16_to_f64(out)[sel], ref[sel], f"{name} metadata-ready decode, call {rep}")
        assert_close(lse.cpu().numpy().astype(np.float64)[sel], ref_lse[sel], f"{name} lse, call {rep}")
    check_no_flags(pkv)


# ------------------------------------------------------- split-K combine API
@pytest.mark.parametrize("d", [64, 128])
def test_split_k_combine(pkv, d):
    rng = np.random.default_rng(d)
    B, hq, S = 5, 8, 7
    part_o = rng.standard_normal((B, hq, S, d)).astype(np.float32)
    part_lse = (3 * rng.standard_normal((B, hq, S))).astype(np.float32)
    part_lse[1, :, 2] = -np.inf           # an empty split
    part_lse[2, :, :] = -np.inf           # a request with no keys at all
    ns = np.array([7, 4, 3, 1, 0], np.int32)
    ref, ref_lse = oracle.split_k_combine(part_o.astype(np.float64), part_lse.astype(np.float64), ns)
    lse = torch.zeros((B, hq), device="cuda")
    out = pkv.pkv_split_k_combine(torch.from_numpy(part_o).cuda(), torch.from_numpy(part_lse).cuda(),
                                  dev_i32(ns), out_lse=lse)
    assert_close(bf16_to_f64(out), ref, "combine")
    got_lse = lse.cpu().numpy().astype(np.float64)
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isneginf(got_lse), ~fin)
    assert np.abs(got_lse[fin] - ref_lse[fin]).max() <= 1e-4


# ------------------------------------------------------------------ prefill
def run_prefill_case(pkv, w, ids=None):
    ds = DeviceStep(pkv, w, host_ids=ids)
    os_ = OracleStep(w, ids)
    ds.append()
    os_.append()
    check_pool_bits(ds, os_)
    ref, _, rows = os_.prefill()
    got = bf16_to_f64(ds.prefill())
    assert_close(got[rows], ref[rows], f"{w.name} prefill")
    check_no_flags(pkv)
    return ds, os_


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_prefill_mixed_small(pkv, seed):
    w = make_workload("mixed_prefill_decode", seed, n_prefill=3, chunks=[512, 100, 37], ctx_hi=1000,
                      n_decode=5, len_lo=50, len_hi=900)
    ds, os_ = run_prefill_case(pkv, w)
    ref, _, sel = os_.decode()
    assert_close(bf16_to_f64(ds.decode())[sel], ref[sel], "mixed decode part")


def test_prefill_context_edges(pkv):
    # no prior context; a context ending exactly on a 128-key tile; a chunk
    # of one row; a chunk shorter than a query tile
    w = make_workload("mixed_prefill_decode", 4, n_prefill=4, chunks=[200, 64, 1, 7],
                      ctxs=[0, 128, 300, 127], n_decode=1)
    run_prefill_case(pkv, w)


@pytest.mark.parametrize("group,d", [(1, 128), (2, 128), (8, 128), (1, 64), (4, 64), (8, 64)])
def test_prefill_group_and_head_dim(pkv, group, d):
    w = make_workload("mixed_prefill_decode", 9, n_prefill=2, chunks=[150, 77], ctx_hi=400,
                      n_decode=1, num_kv_heads=2, num_q_heads=2 * group, head_dim=d)
    run_prefill_case(pkv, w)


def test_prefill_chunk_longer_than_max_q_len(pkv):
    # the grid is sized from max_q_len: a longer chunk is refused whole (its
    # rows keep their contents) and PKV_FLAG_BAD_QUERY_ROWS is raised; the
    # other request is computed as usual
    w = make_workload("mixed_prefill_decode", 12, n_prefill=2, chunks=[300, 20], ctx_hi=200,
                      n_decode=1)
    ds = DeviceStep(pkv, w)
    os_ = OracleStep(w)
    ds.append()
    os_.append()
    ref, _, rows = os_.prefill()
    pre = list(w.prefill_ids)
    cu = w.cu_q_lens(pre)
    out = torch.full_like(ds.q_pre, 7.0)
    pkv.pkv_paged_attn_chunked_prefill(ds.q_pre, ds.cu_q, ds.ctx_pre, ds.k_pool, ds.v_pool, ds.pt_pre,
                                       w.scale, 64, out=out)
    assert pkv.pkv_device_error_flags(clear=True) & pkv.FLAG_BAD_QUERY_ROWS
    got = bf16_to_f64(out)
    long_r = int(np.argmax(np.diff(cu)))
    short_rows = np.arange(cu[1 - long_r], cu[2 - long_r])
    assert (got[cu[long_r]:cu[long_r + 1]] == 7.0).all()
    assert_close(got[short_rows], ref[short_rows], "prefill, the chunk within max_q_len")


def test_prefill_page32(pkv):
    w = make_workload("mixed_prefill_decode", 10, n_prefill=2, chunks=[256, 90], ctx_hi=700,
                      n_decode=1, page_size=32)
    run_prefill_case(pkv, w)


# --------------------------------------------- full-size workloads, sampled
def sample_ids(w, k, rng_seed=0):
    rng = np.random.default_rng(rng_seed)
    dec, pre = list(w.decode_ids), list(w.prefill_ids)
    pick = []
    if dec:
        by_len = sorted(dec, key=lambda r: w.kv_lens[r])
        pick += [by_len[0], by_len[-1]] + list(rng.choice(dec, size=min(k, len(dec)), replace=False))
    return sorted(set(int(r) for r in pick))


@pytest.mark.slow
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_full_qwen3_decode_sampled(pkv, seed):
    w = make_workload("qwen3_decode", seed)
    run_decode_case(pkv, w, ids=sample_ids(w, 6, seed), partitions=(0,))


@pytest.mark.slow
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_full_splitk_long_sampled(pkv, seed):
    w = make_workload("splitk_long", seed)
    # the shortest and the longest request (32 768 and 131 072 tokens)
    run_decode_case(pkv, w, ids=[0, 3], partitions=(0, 512, 4096))


@pytest.mark.slow
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_full_frag_large_sampled(pkv, seed):
    w = make_workload("frag_large", seed)
    run_decode_case(pkv, w, ids=sample_ids(w, 6, seed), partitions=(0,))


@pytest.mark.slow
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_full_mixed_sampled(pkv, seed):
    w = make_workload("mixed_prefill_decode", seed)
    pre = list(w.prefill_ids)
    by_ctx = sorted(pre, key=lambda r: w.ctx_lens[r])
    ids = [by_ctx[0], by_ctx[-1]] + sample_ids(w, 3, seed)
    ds, os_ = run_prefill_case(pkv, w, ids=ids)
    ref, _, sel = os_.decode()
    assert_close(bf16_to_f64(ds.decode())[sel], ref[sel], "mixed decode part")
