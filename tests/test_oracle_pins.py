"""Pins for the CPU oracle, checked against things other than itself.

Each check_* function takes the oracle module so that test_oracle_mutations
can rerun it against copies of the oracle with planted mistakes.  The pins:

* the page-table walk and kv_append follow the page's own page-table example
  (tiny-llm source reading, "Paged KV Cache") and the slot definition, with
  explicit expected positions;
* attention equals PyTorch's scaled_dot_product_attention (an independent
  library routine) on the same rows laid out contiguously, for decode (GQA)
  and for a causal chunk at a context offset;
* hand-derived worked examples (tests/golden/*.json);
* closed forms, invariance under page permutation and page size, causal
  perturbation, and the split-K/combine identity.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle.paged_attention as O
from workloads import f32_to_bf16_bits

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def load_golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def bits(x):
    return f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def rand_bits(rng, shape, scale=1.0):
    return bits(scale * rng.standard_normal(shape).astype(np.float32))


def f64(b):
    return O.bf16_bits_to_f64(b)


NAN16 = np.uint16(0x7FC0)


def build_pool(o, rows_k, rows_v, tables, num_pages, page_size):
    """Place each request's contiguous rows into a NaN pool via the oracle's
    kv_append, using slots written out from the table definition."""
    hkv, d = rows_k[0].shape[1], rows_k[0].shape[2]
    kp = np.full((num_pages, hkv, page_size, d), NAN16, np.uint16)
    vp = kp.copy()
    for rk, rv, table in zip(rows_k, rows_v, tables):
        slots = [table[j // page_size] * page_size + j % page_size for j in range(len(rk))]
        o.kv_append(kp, vp, rk, rv, np.array(slots, np.int32), page_size)
    return kp, vp


def table_array(tables, width=None):
    width = width or max(len(t) for t in tables)
    out = np.full((len(tables), width), -1, np.int32)
    for i, t in enumerate(tables):
        out[i, :len(t)] = t
    return out


def random_tables(rng, lens, page_size, num_pages):
    perm = rng.permutation(num_pages)
    tables, at = [], 0
    for L in lens:
        n = -(-L // page_size)
        tables.append(list(perm[at:at + n]))
        at += n
    return tables


def sdpa(q, k, v, scale, causal=False):
    """torch SDPA in fp64: q [Hq][Lq][d], k/v [Hkv][Lk][d] -> [Hq][Lq][d]."""
    tq, tk, tv = (torch.from_numpy(np.ascontiguousarray(a))[None] for a in (q, k, v))
    o = F.scaled_dot_product_attention(tq, tk, tv, scale=scale, is_causal=causal,
                                       enable_gqa=True)
    return o[0].numpy()


# ------------------------------------------------------- page-table walk
def check_gather_page_example(o):
    ex = load_golden("page_table_example.json")
    P = 4
    pool = np.full((ex["pool_pages"], 1, P, 1), NAN16, np.uint16)
    for p in range(ex["pool_pages"]):
        for r in range(P):
            pool[p, 0, r, 0] = 100 * p + r
    got = o.gather_request_kv(pool, ex["tables"]["A"], 10, P)[:, 0, 0]
    assert got.tolist() == [700, 701, 702, 703, 200, 201, 202, 203, 1100, 1101]
    got = o.gather_request_kv(pool, ex["tables"]["B"], 5, P)[:, 0, 0]
    assert got.tolist() == [400, 401, 402, 403, 900]


def check_kv_append_slots(o):
    P, hkv, d = 4, 2, 3
    kp = np.full((12, hkv, P, d), 0x1234, np.uint16)
    vp = np.full((12, hkv, P, d), 0x4321, np.uint16)
    # slot = page * P + offset: 7*4+3 -> page 7 row 3; 2*4+0 -> page 2 row 0; 11*4+1
    slots = np.array([31, -1, 8, 45], np.int32)
    kn = np.arange(4 * hkv * d, dtype=np.uint16).reshape(4, hkv, d) + 1
    # bit patterns that any float conversion would alter: sNaN, -0, denormal
    kn[0, 0, 0], kn[2, 1, 2], kn[3, 0, 1] = 0x7F81, 0x8000, 0x0001
    vn = kn + 1000
    o.kv_append(kp, vp, kn, vn, slots, P)
    assert (kp[7, :, 3] == kn[0]).all() and (vp[7, :, 3] == vn[0]).all()
    assert (kp[2, :, 0] == kn[2]).all() and (vp[2, :, 0] == vn[2]).all()
    assert (kp[11, :, 1] == kn[3]).all() and (vp[11, :, 1] == vn[3]).all()
    touched = np.zeros((12, P), bool)
    touched[7, 3] = touched[2, 0] = touched[11, 1] = True
    assert (kp.transpose(0, 2, 1, 3)[~touched] == 0x1234).all()
    assert (vp.transpose(0, 2, 1, 3)[~touched] == 0x4321).all()


def test_gather_page_example():
    check_gather_page_example(O)


def test_kv_append_slots():
    check_kv_append_slots(O)


# --------------------------------------------------- library equivalence
def check_decode_vs_sdpa(o, seed=0):
    rng = np.random.default_rng(seed)
    hq, hkv, d, P = 8, 2, 16, 4
    lens = [1, 5, 13, 32]
    rows_k = [rand_bits(rng, (L, hkv, d)) for L in lens]
    rows_v = [rand_bits(rng, (L, hkv, d)) for L in lens]
    tables = random_tables(rng, lens, P, 40)
    kp, vp = build_pool(o, rows_k, rows_v, tables, 40, P)
    q = rand_bits(rng, (len(lens), hq, d))
    scale = 1 / math.sqrt(d)
    out, lse = o.decode_attention(q, kp, vp, table_array(tables), np.array(lens), P, scale)
    for r, L in enumerate(lens):
        ref = sdpa(f64(q[r])[:, None, :], f64(rows_k[r]).transpose(1, 0, 2),
                   f64(rows_v[r]).transpose(1, 0, 2), scale)[:, 0, :]
        np.testing.assert_allclose(out[r], ref, rtol=0, atol=1e-12)
        # the lse is the log of the softmax denominator
        s = np.einsum("hgd,lhd->hgl", f64(q[r]).reshape(hkv, hq // hkv, d), f64(rows_k[r])) * scale
        from scipy.special import logsumexp
        np.testing.assert_allclose(lse[r], logsumexp(s, axis=-1).reshape(hq), atol=1e-12)


def check_prefill_vs_sdpa(o, seed=0):
    rng = np.random.default_rng(seed)
    hq, hkv, d, P = 4, 2, 8, 4
    ctx = [0, 5, 9]
    chunk = [6, 3, 7]
    lens = [c + n for c, n in zip(ctx, chunk)]
    rows_k = [rand_bits(rng, (L, hkv, d)) for L in lens]
    rows_v = [rand_bits(rng, (L, hkv, d)) for L in lens]
    tables = random_tables(rng, lens, P, 24)
    kp, vp = build_pool(o, rows_k, rows_v, tables, 24, P)
    q = rand_bits(rng, (sum(chunk), hq, d))
    cu = np.concatenate([[0], np.cumsum(chunk)])
    scale = 0.3
    out, lse = o.chunked_prefill_attention(q, cu, np.array(ctx), kp, vp, table_array(tables), P, scale)
    for r in range(len(ctx)):
        L = lens[r]
        # full causal attention over all L positions; the chunk is its last rows
        qfull = np.zeros((hq, L, d))
        qfull[:, ctx[r]:, :] = f64(q[cu[r]:cu[r + 1]]).transpose(1, 0, 2)
        ref = sdpa(qfull, f64(rows_k[r]).transpose(1, 0, 2), f64(rows_v[r]).transpose(1, 0, 2),
                   scale, causal=True)[:, ctx[r]:, :].transpose(1, 0, 2)
        np.testing.assert_allclose(out[cu[r]:cu[r + 1]], ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_decode_vs_sdpa(seed):
    check_decode_vs_sdpa(O, seed)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_prefill_vs_sdpa(seed):
    check_prefill_vs_sdpa(O, seed)


# --------------------------------------------------------- worked examples
def check_two_key_example(o):
    ex = load_golden("two_key_example.json")
    scale = math.log(ex["scale_is_ln"])
    k, v = bits(ex["k"])[:, None, :], bits(ex["v"])[:, None, :]
    kp, vp = build_pool(o, [k], [v], [[0, 1]], 2, 1)
    q = bits([[ex["q"]]])
    out, lse = o.decode_attention(q, kp, vp, np.array([[0, 1]]), np.array([2]), 1, scale)
    np.testing.assert_allclose(out[0, 0], ex["expected_out"], rtol=0, atol=1e-14)
    assert abs(lse[0, 0] - math.log(ex["expected_lse_is_ln"])) < 1e-14
    sk = ex["split_k"]
    po = np.array(sk["part_o"])[None, None]
    pl = np.log(np.array(sk["part_lse_is_ln"]))[None, None]
    o2, l2 = o.split_k_combine(po, pl, np.array([2]))
    np.testing.assert_allclose(o2[0, 0], ex["expected_out"], rtol=0, atol=1e-14)
    assert abs(l2[0, 0] - math.log(ex["expected_lse_is_ln"])) < 1e-14
    # and the oracle's own partials of this example are those hand values
    pO, pL, ns = o.decode_partials(q, kp, vp, np.array([[0, 1]]), np.array([2]), 1, scale, 1)
    np.testing.assert_allclose(pO[0, 0], sk["part_o"], atol=1e-14)
    np.testing.assert_allclose(pL[0, 0], np.log(sk["part_lse_is_ln"]), atol=1e-14)


def check_causal_chunk_example(o):
    ex = load_golden("causal_chunk_example.json")
    k, v = bits(ex["k"])[:, None, :], bits(ex["v"])[:, None, :]
    kp, vp = build_pool(o, [k], [v], [[2, 0, 1]], 3, 1)
    q = bits(ex["q_rows"])[:, None, :]
    out, lse = o.chunked_prefill_attention(q, np.array([0, 2]), np.array([ex["ctx"]]), kp, vp,
                                           np.array([[2, 0, 1]]), 1, 1.0)
    np.testing.assert_allclose(out[:, 0], ex["expected_out"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse[:, 0], np.log(ex["expected_lse_is_ln"]), atol=1e-14)


def test_two_key_example():
    check_two_key_example(O)


def test_causal_chunk_example():
    check_causal_chunk_example(O)


# ---------------------------------------------------------- invariances
def _decode_case(o, rng, tables, lens, num_pages, P, rows_k, rows_v, q, scale=0.25):
    kp, vp = build_pool(o, rows_k, rows_v, tables, num_pages, P)
    return o.decode_attention(q, kp, vp, table_array(tables), np.array(lens), P, scale)


def check_page_permutation(o):
    """Page example tables vs. an identity assignment: bit-identical output."""
    ex = load_golden("page_table_example.json")
    rng = np.random.default_rng(7)
    P, hkv, d, hq = 16, 2, 8, 4
    lens = [40, 20]  # A uses 3 pages, B uses 2
    rows_k = [rand_bits(rng, (L, hkv, d)) for L in lens]
    rows_v = [rand_bits(rng, (L, hkv, d)) for L in lens]
    q = rand_bits(rng, (2, hq, d))
    a = _decode_case(o, rng, [ex["tables"]["A"], ex["tables"]["B"]], lens, 12, P, rows_k, rows_v, q)
    b = _decode_case(o, rng, [[0, 1, 2], [3, 4]], lens, 12, P, rows_k, rows_v, q)
    c = _decode_case(o, rng, random_tables(rng, lens, P, 12), lens, 12, P, rows_k, rows_v, q)
    for x in (b, c):
        assert np.array_equal(a[0], x[0]) and np.array_equal(a[1], x[1])
    assert np.isfinite(a[0]).all()  # NaN pages outside the tables were never read


def check_page_size_invariance(o):
    rng = np.random.default_rng(3)
    hkv, d, hq = 2, 8, 4
    lens = [1, 17, 64, 65]
    rows_k = [rand_bits(rng, (L, hkv, d)) for L in lens]
    rows_v = [rand_bits(rng, (L, hkv, d)) for L in lens]
    q = rand_bits(rng, (len(lens), hq, d))
    results = []
    for P in (1, 2, 16, 32, 64):
        n = sum(-(-L // P) for L in lens) + 3
        results.append(_decode_case(o, rng, random_tables(rng, lens, P, n), lens, n, P, rows_k, rows_v, q))
    for x in results[1:]:
        assert np.array_equal(results[0][0], x[0])


def test_page_permutation():
    check_page_permutation(O)


def test_page_size_invariance():
    check_page_size_invariance(O)


# ------------------------------------------------------------ causality
def check_causal_perturbation(o):
    rng = np.random.default_rng(11)
    hq, hkv, d, P = 4, 2, 8, 4
    c, n = 6, 5
    L = c + n
    rk, rv = rand_bits(rng, (L, hkv, d)), rand_bits(rng, (L, hkv, d))
    q = rand_bits(rng, (n, hq, d))
    cu = np.array([0, n])
    base = o.chunked_prefill_attention(q, cu, [c], *build_pool(o, [rk], [rv], [[0, 1, 2]], 3, P),
                                       np.array([[0, 1, 2]]), P, 0.5)[0]
    for p in range(c, L - 1):  # perturb every key after position p
        k2, v2 = rk.copy(), rv.copy()
        k2[p + 1:] = rand_bits(rng, k2[p + 1:].shape)
        v2[p + 1:] = rand_bits(rng, v2[p + 1:].shape)
        got = o.chunked_prefill_attention(q, cu, [c], *build_pool(o, [k2], [v2], [[0, 1, 2]], 3, P),
                                          np.array([[0, 1, 2]]), P, 0.5)[0]
        i = p - c
        assert np.array_equal(got[:i + 1], base[:i + 1])
        assert not np.array_equal(got[i + 1:], base[i + 1:])
    # prefill row i equals a decode over the first c+i+1 keys
    kp, vp = build_pool(o, [rk], [rv], [[0, 1, 2]], 3, P)
    for i in range(n):
        dec = o.decode_attention(q[i:i + 1], kp, vp, np.array([[0, 1, 2]]), [c + i + 1], P, 0.5)[0]
        np.testing.assert_allclose(dec[0], base[i], rtol=0, atol=1e-15)


def test_causal_perturbation():
    check_causal_perturbation(O)


# --------------------------------------------------------- closed forms
def check_closed_forms(o):
    rng = np.random.default_rng(5)
    hq, hkv, d, P = 6, 3, 8, 4
    L = 23
    tables = [[5, 1, 3, 0, 2, 4]]
    q = rand_bits(rng, (1, hq, d))
    rk = rand_bits(rng, (L, hkv, d))
    # all V rows equal to one row v -> output is v exactly
    v_row = rand_bits(rng, (1, hkv, d))
    out, _ = _decode_case(o, rng, tables, [L], 6, P, [rk], [np.repeat(v_row, L, 0)], q)
    for h in range(hq):
        assert np.allclose(out[0, h], f64(v_row[0, h // 2]), rtol=0, atol=1e-15)
    # L = 1 -> output is V[0]
    rv = rand_bits(rng, (L, hkv, d))
    out, lse = _decode_case(o, rng, tables, [1], 6, P, [rk[:1]], [rv[:1]], q)
    for h in range(hq):
        assert np.array_equal(out[0, h], f64(rv[0, h // 2]))
    # q = 0 -> the plain mean of the V rows, lse = log L
    out, lse = _decode_case(o, rng, tables, [L], 6, P, [rk], [rv], np.zeros_like(q))
    for h in range(hq):
        np.testing.assert_allclose(out[0, h], f64(rv[:, h // 2]).mean(0), atol=1e-14)
    np.testing.assert_allclose(lse[0], math.log(L), atol=1e-14)
    # identical K rows -> the mean of V, for any q
    out, _ = _decode_case(o, rng, tables, [L], 6, P, [np.repeat(rk[:1], L, 0)], [rv], q)
    for h in range(hq):
        np.testing.assert_allclose(out[0, h], f64(rv[:, h // 2]).mean(0), atol=1e-14)
    # query heads of one group with identical q give identical outputs
    q2 = q.copy()
    q2[0, 1] = q2[0, 0]
    out, _ = _decode_case(o, rng, tables, [L], 6, P, [rk], [rv], q2)
    assert np.array_equal(out[0, 0], out[0, 1])
    # softmax weights sum to one: V = 1 gives exactly 1
    ones = np.full((L, hkv, d), bits(1.0), np.uint16)
    out, _ = _decode_case(o, rng, tables, [L], 6, P, [rk], [ones], q)
    assert np.abs(out - 1.0).max() < 1e-15
    # a request with no keys: zero output, lse -inf (reading R7)
    out, lse = _decode_case(o, rng, tables, [0], 6, P, [rk[:0]], [rv[:0]], q)
    assert (out == 0).all() and np.isneginf(lse).all()


def test_closed_forms():
    check_closed_forms(O)


# ---------------------------------------------------------- split / combine
def check_split_identity(o):
    rng = np.random.default_rng(9)
    hq, hkv, d, P = 4, 2, 8, 4
    lens = [1, 7, 33, 64, 100]
    rows_k = [rand_bits(rng, (L, hkv, d)) for L in lens]
    rows_v = [rand_bits(rng, (L, hkv, d)) for L in lens]
    tables = random_tables(rng, lens, P, 60)
    kp, vp = build_pool(o, rows_k, rows_v, tables, 60, P)
    q = rand_bits(rng, (len(lens), hq, d))
    T = table_array(tables)
    full, full_lse = o.decode_attention(q, kp, vp, T, lens, P, 0.35)
    for part in (1, 4, 8, 12, 32, 128):
        po, pl, ns = o.decode_partials(q, kp, vp, T, lens, P, 0.35, part)
        assert ns.tolist() == [-(-L // part) for L in lens]
        out, lse = o.split_k_combine(po, pl, ns)
        np.testing.assert_allclose(out, full, rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse, full_lse, rtol=0, atol=1e-13)
    # an empty split (lse = -inf) carries no weight
    po, pl, ns = o.decode_partials(q, kp, vp, T, lens, P, 0.35, 32)
    po2 = np.concatenate([po, np.full_like(po[:, :, :1], np.nan)], axis=2)
    pl2 = np.concatenate([pl, np.full_like(pl[:, :, :1], np.nan)], axis=2)
    for r, n in enumerate(ns):
        po2[r, :, n], pl2[r, :, n] = 123.0, -np.inf
    out, _ = o.split_k_combine(po2, pl2, ns + 1)
    np.testing.assert_allclose(out, full, rtol=0, atol=1e-13)


def test_split_identity():
    check_split_identity(O)


ALL_CHECKS = [
    check_gather_page_example, check_kv_append_slots, check_decode_vs_sdpa,
    check_prefill_vs_sdpa, check_two_key_example, check_causal_chunk_example,
    check_page_permutation, check_page_size_invariance, check_causal_perturbation,
    check_closed_forms, check_split_identity,
]
