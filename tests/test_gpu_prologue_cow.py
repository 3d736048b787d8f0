"""Parity of the fused QK-norm + RoPE + append prologue and of copy-on-write
append on shared-prefix pages (through the C ABI) with the CPU oracle.

Prologue: the rotated queries and the stored K rows are computed values,
rounded once to bf16 on both sides (the oracle from fp64, the kernel from
fp32), so they must agree to within one bf16 step (2^-7 of the value at
most); V rows are a bit copy and must match exactly.  Attention after the
prologue must meet the attention tolerance (1e-2 max, 1e-3 mean abs).

Copy-on-write: which sharer keeps a page and which free page each request
gets depend on the order of the device's atomics, so the comparison is of
what is unique -- every request's tokens read through its table, bit for bit,
and the number of free pages taken -- and the rest is checked for validity:
reference counts equal the table entries naming each page, the pages taken
are the front of the free list, and attention through the shared tables is
bit-identical to attention through private copies of every page.
"""
import numpy as np
import pytest
import torch

import oracle
import oracle.prefix_pages as OX
import oracle.prologue as OP
from tests.harness import assert_close, bf16_to_f64, dev_bf16, dev_i32, host_bits
from workloads import f32_to_bf16_bits
from workloads.prefix import make_prefix_scenario, private_copy

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pkv():
    import paged_kv_attention_37_b200 as m
    assert torch.cuda.is_available()
    m.pkv_device_error_flags(clear=True)
    return m


def within_one_step(got, ref, what):
    """|got - ref| <= 2^-7 |ref| (one bf16 step at most), plus a hair for
    values near zero."""
    err = np.abs(got - ref)
    bound = 2.0 ** -7 * np.abs(ref) + 1e-6
    assert (err <= bound).all(), f"{what}: worst excess {np.max(err - bound):.3g}"


def rand_bits(rng, shape, scale=1.0):
    return f32_to_bf16_bits((scale * rng.standard_normal(shape)).astype(np.float32))


# ----------------------------------------------------------------- prologue
@pytest.mark.parametrize("d,hq,hkv", [(128, 32, 8), (64, 32, 8), (128, 16, 8), (64, 8, 1)])
def test_prologue_matches_oracle(pkv, d, hq, hkv):
    rng = np.random.default_rng(d + hq)
    T, P, pages = 37, 16, 40
    q, k, v = rand_bits(rng, (T, hq, d), 2.0), rand_bits(rng, (T, hkv, d), 0.7), rand_bits(rng, (T, hkv, d))
    wq = f32_to_bf16_bits((1 + 0.3 * rng.standard_normal(d)).astype(np.float32))
    wk = f32_to_bf16_bits((1 + 0.3 * rng.standard_normal(d)).astype(np.float32))
    pos = rng.integers(0, 131072, T).astype(np.int32)
    pos[:4] = [0, 1, 131071, 65535]
    slots = rng.permutation(pages * P)[:T].astype(np.int32)
    slots[5] = -1
    eps, theta = 1e-6, 1e6
    kp = torch.full((pages, hkv, P, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    vp = torch.full_like(kp, float("nan"))
    q_out = pkv.pkv_qk_norm_rope_append(dev_bf16(q), dev_bf16(k), dev_bf16(v), dev_bf16(wq), dev_bf16(wk),
                                        dev_i32(pos), dev_i32(slots), kp, vp, eps=eps, rope_theta=theta)
    ek = np.full((pages, hkv, P, d), 0x7FC0, np.uint16)
    ev = ek.copy()
    rq, rk = OP.qk_norm_rope_append(ek, ev, q, k, v, wq, wk, pos, slots, P, eps, theta)
    within_one_step(bf16_to_f64(q_out), rq, "q_out")
    gk, gv = host_bits(kp), host_bits(vp)
    assert np.array_equal(gv, ev), "V rows are a bit copy"
    written = slots[slots >= 0]
    pg, off = written // P, written % P
    within_one_step(oracle.bf16_bits_to_f64(gk[pg, :, off]),
                    rk[slots >= 0], "stored K rows")
    mask = np.ones((pages, P), bool)
    mask[pg, off] = False
    assert (gk.transpose(0, 2, 1, 3)[mask] == 0x7FC0).all(), "other slots untouched"
    assert pkv.pkv_device_error_flags(clear=True) == 0


def test_prologue_in_place_and_bad_slot(pkv):
    rng = np.random.default_rng(7)
    T, hq, hkv, d, P = 4, 8, 2, 128, 16
    q, k, v = rand_bits(rng, (T, hq, d)), rand_bits(rng, (T, hkv, d)), rand_bits(rng, (T, hkv, d))
    w = f32_to_bf16_bits(np.ones(d, np.float32))
    pos = np.array([3, 9, 100, 7], np.int32)
    slots = np.array([1, 2 * P + 3, -9, 5], np.int32)  # -9: not a slot
    kp = torch.zeros((3, hkv, P, d), dtype=torch.bfloat16, device="cuda")
    vp = torch.zeros_like(kp)
    qd = dev_bf16(q)
    out = pkv.pkv_qk_norm_rope_append(qd, dev_bf16(k), dev_bf16(v), dev_bf16(w), dev_bf16(w), dev_i32(pos),
                                      dev_i32(slots), kp, vp, q_out=qd)
    assert out.data_ptr() == qd.data_ptr()
    assert pkv.pkv_device_error_flags(clear=True) & pkv.FLAG_BAD_SLOT
    rq, _ = OP.qk_norm_rope(q, k, pos, w, w, 1e-6, 1e6)
    within_one_step(bf16_to_f64(out), rq, "q_out in place (every row, the bad slot's too)")
    gv = host_bits(vp)
    for t in (0, 1, 3):  # the rows with valid slots; the bad one wrote nothing
        a, b = divmod(int(slots[t]), P)
        assert np.array_equal(gv[a, :, b], v[t])
    assert int((gv != 0).any(axis=(1, 3)).sum()) == 3


def test_prologue_then_decode(pkv):
    # the prologue writes the new token's K/V; decode reads it with the rotated
    # query: the attention result against the oracle's prologue + attention
    from tests.harness import DeviceStep, OracleStep
    from workloads import make_workload
    w = make_workload("qwen3_decode", 3, B=6, len_lo=40, len_hi=900)
    ds, os_ = DeviceStep(pkv, w), OracleStep(w)
    rng = np.random.default_rng(11)
    dec = list(w.decode_ids)
    T = len(dec)
    q = w.batch_q(dec)
    k, v, slots = w.batch_new()
    wq = f32_to_bf16_bits((1 + 0.2 * rng.standard_normal(w.head_dim)).astype(np.float32))
    wk = f32_to_bf16_bits((1 + 0.2 * rng.standard_normal(w.head_dim)).astype(np.float32))
    pos = (w.kv_lens[dec] - 1).astype(np.int32)
    q_dev = pkv.pkv_qk_norm_rope_append(dev_bf16(q), dev_bf16(k), dev_bf16(v), dev_bf16(wq), dev_bf16(wk),
                                        dev_i32(pos), dev_i32(slots), ds.k_pool, ds.v_pool)
    out = pkv.pkv_paged_attn_decode(q_dev, ds.k_pool, ds.v_pool, ds.pt_dec, ds.len_dec, w.scale)
    # oracle: the same prologue into its compact pool (slots renumbered), then attention
    cslots = np.array([os_.cw.page_table[r][int(p) // w.page_size] * w.page_size + int(p) % w.page_size
                       for r, p in zip(dec, pos)], np.int32)
    rq, _ = OP.qk_norm_rope_append(os_.k_pool, os_.v_pool, q, k, v, wq, wk, pos, cslots, w.page_size, 1e-6, 1e6)
    q_bits = OP.f64_to_bf16_bits(rq)  # the rounded rotated queries attention reads
    got_q = host_bits(q_dev)
    ref, _ = oracle.decode_attention(got_q, os_.k_pool, os_.v_pool, os_.cw.page_table[dec],
                                     w.kv_lens[dec], w.page_size, w.scale)
    assert_close(bf16_to_f64(out), ref, "decode after the prologue")
    assert np.abs(oracle.bf16_bits_to_f64(got_q) - oracle.bf16_bits_to_f64(q_bits)).max() <= \
        2.0 ** -7 * np.abs(rq).max()
    assert pkv.pkv_device_error_flags(clear=True) == 0


# ------------------------------------------------------------ copy-on-write
def to_device(s):
    return (dev_bf16(s.k_pool), dev_bf16(s.v_pool), dev_i32(s.page_table), dev_i32(s.refcount),
            dev_i32(s.free_pages))


def logical(pool_bits, table, L, P):
    return oracle.gather_request_kv(pool_bits, table, int(L), P)


@pytest.mark.parametrize("seed,n_new,d", [(0, 1, 64), (1, 1, 128), (2, 5, 64), (3, 20, 128), (4, 3, 128)])
def test_cow_append_matches_oracle(pkv, seed, n_new, d):
    s = make_prefix_scenario(seed, groups=((37, 3, 0), (64, 2, 1), (50, 4, 2), (21, 5, 0)),
                             n_new=n_new, num_kv_heads=4, head_dim=d)
    kp, vp, table, rc, free = to_device(s)
    used = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.pkv_kv_append_cow(dev_bf16(s.k_new), dev_bf16(s.v_new), dev_i32(s.token_req), dev_i32(s.token_pos),
                          table, rc, free, used, kp, vp)
    assert pkv.pkv_device_error_flags(clear=True) == 0
    ek, ev, et, erc = s.k_pool.copy(), s.v_pool.copy(), s.page_table.copy(), s.refcount.copy()
    n_used = OX.kv_append_cow(ek, ev, et, erc, s.free_pages, s.k_new, s.v_new, s.token_req, s.token_pos,
                              s.page_size)
    gk, gv, gt, grc = host_bits(kp), host_bits(vp), table.cpu().numpy(), rc.cpu().numpy()
    assert int(used.item()) == n_used
    L = s.kv_lens
    for r in range(s.B):
        assert np.array_equal(logical(gk, gt[r], L[r], s.page_size), logical(ek, et[r], L[r], s.page_size)), r
        assert np.array_equal(logical(gv, gt[r], L[r], s.page_size), logical(ev, et[r], L[r], s.page_size)), r
    want = OX.table_refcounts(gt, L, s.page_size, s.num_pages)
    named = want > 0
    assert np.array_equal(grc[named], want[named])
    taken = set(s.free_pages[:n_used].tolist())
    assert taken <= set(gt[gt >= 0].ravel().tolist())
    assert not (set(gt[gt >= 0].ravel().tolist()) & set(s.free_pages[n_used:].tolist()))
    # attention through the shared tables == through private copies
    dec_q = torch.from_numpy(rand_bits(np.random.default_rng(seed), (s.B, 4 * s.num_kv_heads, d))
                             .view(np.int16)).view(torch.bfloat16).cuda()
    lens = dev_i32(L)
    scale = 1.0 / np.sqrt(d)
    shared_out = pkv.pkv_paged_attn_decode(dec_q, kp, vp, table, lens, scale)
    pk, pv, pt = private_copy(s)
    O_pk, O_pv = pk.copy(), pv.copy()
    from tests.test_oracle_pins_prefix import slots_from_tables
    oracle.kv_append(O_pk, O_pv, s.k_new, s.v_new, slots_from_tables(pt, s.token_req, s.token_pos, s.page_size),
                     s.page_size)
    priv_out = pkv.pkv_paged_attn_decode(dec_q, dev_bf16(O_pk), dev_bf16(O_pv), dev_i32(pt), lens, scale)
    assert torch.equal(shared_out, priv_out), "sharing pages must not change attention"
    assert pkv.pkv_device_error_flags(clear=True) == 0


def test_cow_free_list_exhausted(pkv):
    s = make_prefix_scenario(3, groups=((21, 4, 0),), n_new=1, spare_pages=0)
    kp, vp, table, rc, free = to_device(s)
    used = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.pkv_kv_append_cow(dev_bf16(s.k_new), dev_bf16(s.v_new), dev_i32(s.token_req), dev_i32(s.token_pos),
                          table, rc, free[:1], used, kp, vp)
    assert pkv.pkv_device_error_flags(clear=True) & pkv.FLAG_NO_FREE_PAGE
    gt = table.cpu().numpy()
    e = 21 // s.page_size
    # one request got the free page, one kept the shared page, two lost the entry
    assert sorted(int(x == -1) for x in gt[:4, e]) == [0, 0, 1, 1]
