"""Pins for the copy-on-write append oracle (shared-prefix pages), checked
against things other than itself.

Each check_* function takes the oracle module so that the mutation tests can
rerun it against copies with planted mistakes.  The pins:

* with no page shared, it is the plain kv_append with slots read off the
  tables (itself pinned by the page's page-table example);
* a hand-worked fork: two requests sharing a partly filled page, one appends;
* copy-on-write is invisible: the tokens every request sees through its
  table after the append equal those of the same append made on private
  copies of every page (plain kv_append), and a request that did not append
  sees exactly what it saw before;
* reference counts afterwards equal the number of table entries naming each
  page; pages are taken from the front of the free list; when every sharer
  of a page appends, the last one writes in place.
"""
import numpy as np
import pytest

import oracle.paged_attention as O
import oracle.prefix_pages as OX
from workloads.prefix import make_prefix_scenario, private_copy


def logical(kp, table_row, n, P):
    return O.gather_request_kv(kp, table_row, n, P)


def slots_from_tables(table, token_req, token_pos, P):
    return np.array([table[r, p // P] * P + p % P for r, p in zip(token_req, token_pos)], np.int32)


def run(o, s):
    kp, vp, table, rc = s.k_pool.copy(), s.v_pool.copy(), s.page_table.copy(), s.refcount.copy()
    used = o.kv_append_cow(kp, vp, table, rc, s.free_pages, s.k_new, s.v_new, s.token_req,
                           s.token_pos, s.page_size)
    return kp, vp, table, rc, used


def check_no_sharing_is_plain_append(o):
    s = make_prefix_scenario(5, groups=((37, 1, 0), (20, 1, 1), (64, 1, 0)), n_new=3)
    assert (s.refcount <= 1).all()
    kp, vp, table, rc, used = run(o, s)
    assert used == 0 and np.array_equal(table, s.page_table)
    ek, ev = s.k_pool.copy(), s.v_pool.copy()
    O.kv_append(ek, ev, s.k_new, s.v_new, slots_from_tables(s.page_table, s.token_req, s.token_pos,
                                                             s.page_size), s.page_size)
    assert np.array_equal(kp, ek) and np.array_equal(vp, ev)


def test_no_sharing_is_plain_append():
    check_no_sharing_is_plain_append(OX)


def check_hand_fork(o):
    # page 5 holds 2 valid rows shared by requests 0 and 1 (count 2), and a
    # stale row 3 left by an earlier owner; request 0 appends its token at
    # position 2; free list [9, 2].  Expected: page 9 gets rows 0..1 of page
    # 5 and the new row 2, and nothing at row 3 (rows past the shared prefix
    # are not copied); request 0's entry -> 9; counts: page 5 -> 1, page 9 ->
    # 1; page 5 and request 1 untouched.
    P, hkv, d = 4, 1, 2
    kp = np.full((10, hkv, P, d), 0x7FC0, np.uint16)
    vp = kp.copy()
    kp[5, 0, :2] = [[1, 2], [3, 4]]
    vp[5, 0, :2] = [[7, 8], [9, 10]]
    kp[5, 0, 3] = [99, 99]
    vp[5, 0, 3] = [98, 98]
    table = np.array([[5, -1], [5, -1]], np.int32)
    rc = np.zeros(10, np.int32)
    rc[5] = 2
    used = o.kv_append_cow(kp, vp, table, rc, np.array([9, 2], np.int32),
                           np.array([[[21, 22]]], np.uint16), np.array([[[31, 32]]], np.uint16),
                           np.array([0], np.int32), np.array([2], np.int32), P)
    nan = 0x7FC0
    assert used == 1
    assert table.tolist() == [[9, -1], [5, -1]]
    assert rc[5] == 1 and rc[9] == 1 and rc[2] == 0
    assert kp[9, 0].tolist() == [[1, 2], [3, 4], [21, 22], [nan, nan]]
    assert vp[9, 0].tolist() == [[7, 8], [9, 10], [31, 32], [nan, nan]]
    assert kp[5, 0].tolist() == [[1, 2], [3, 4], [nan, nan], [99, 99]]
    assert (kp[2] == nan).all()


def test_hand_fork():
    check_hand_fork(OX)


def check_cow_is_invisible(o):
    for seed in range(4):
        for n_new in (1, 5, 20):
            s = make_prefix_scenario(seed, n_new=n_new)
            assert (s.refcount > 1).any()
            kp, vp, table, rc, used = run(o, s)
            # private copies of everything, plain append
            pk, pv, pt = private_copy(s)
            O.kv_append(pk, pv, s.k_new, s.v_new,
                        slots_from_tables(pt, s.token_req, s.token_pos, s.page_size), s.page_size)
            L = s.kv_lens
            for r in range(s.B):
                assert np.array_equal(logical(kp, table[r], L[r], s.page_size),
                                      logical(pk, pt[r], L[r], s.page_size)), (seed, n_new, r)
                assert np.array_equal(logical(vp, table[r], L[r], s.page_size),
                                      logical(pv, pt[r], L[r], s.page_size)), (seed, n_new, r)
            # counts match the tables; the free pages taken are the list's front
            want = OX.table_refcounts(table, L, s.page_size, s.num_pages)
            named = want > 0
            assert np.array_equal(rc[named], want[named])
            taken = set(s.free_pages[:used].tolist())
            assert all(rc[p] == 1 for p in taken)
            assert not (set(table[table >= 0].ravel().tolist()) & set(s.free_pages[used:].tolist()))


def test_cow_is_invisible():
    check_cow_is_invisible(OX)


def check_bystanders_unchanged(o):
    s = make_prefix_scenario(7, groups=((45, 3, 0), (30, 2, 1)), n_new=2)
    # only requests 0 and 3 append this time
    keep = np.isin(s.token_req, [0, 3])
    kp, vp, table, rc = s.k_pool.copy(), s.v_pool.copy(), s.page_table.copy(), s.refcount.copy()
    o.kv_append_cow(kp, vp, table, rc, s.free_pages, s.k_new[keep], s.v_new[keep],
                    s.token_req[keep], s.token_pos[keep], s.page_size)
    for r in range(s.B):
        if r in (0, 3):
            continue
        n = int(s.ctx_lens[r])
        assert np.array_equal(table[r], s.page_table[r])
        assert np.array_equal(logical(kp, table[r], n, s.page_size),
                              logical(s.k_pool, s.page_table[r], n, s.page_size))


def test_bystanders_unchanged():
    check_bystanders_unchanged(OX)


def check_last_sharer_writes_in_place(o):
    # one group of 3 just-forked requests sharing a partly filled page: the
    # first two take copies, the third (the page's last sharer) writes in place
    s = make_prefix_scenario(9, groups=((21, 3, 0),), n_new=1)
    shared = s.page_table[0, 21 // s.page_size]
    assert s.refcount[shared] == 3
    kp, vp, table, rc, used = run(o, s)
    assert used == 2 and rc[shared] == 1
    assert sum(int(table[r, 21 // s.page_size] == shared) for r in range(3)) == 1


def test_last_sharer_writes_in_place():
    check_last_sharer_writes_in_place(OX)


def test_free_list_exhaustion_raises():
    s = make_prefix_scenario(3, groups=((21, 4, 0),), n_new=1, spare_pages=0)
    with pytest.raises(ValueError):
        OX.kv_append_cow(s.k_pool.copy(), s.v_pool.copy(), s.page_table.copy(), s.refcount.copy(),
                         s.free_pages[:1], s.k_new, s.v_new, s.token_req, s.token_pos, s.page_size)


ALL_CHECKS = [check_no_sharing_is_plain_append, check_hand_fork, check_cow_is_invisible,
              check_bystanders_unchanged, check_last_sharer_writes_in_place]
