"""Plain CPU oracle for appending new K/V rows to page tables that share
pages (a common prompt prefix), with copy-on-write.

TEST INFRASTRUCTURE ONLY.  Only tests and the smoke check may import this
module; the library never does.  It shares no code with the CUDA path.

What it computes, and where the pages define it: mini-vllm advanced series
design, section 4, Phase C, adv05 "Radix Attention + Copy-on-Write" (a KV
cache organised for automatic prefix reuse, with copy-on-write, compared with
the main series' hash + ref_count scheme).  Several requests' page tables name
the same physical pages for their common prefix; each page carries the count
of table entries that name it.  Attention reads through the tables, so
sharing changes nothing there.  Writing is where sharing matters: a request
that appends into a page another request also names must not change the
other's view.

Readings taken where the pages are silent:
  R15 the only page a request can append into while it is shared is the page
      holding its first new token; later new tokens fill pages the cache
      manager handed out fresh.  The check is made for the page of the
      request's first new token of the call and for every page a new token
      starts (offset 0).
  R16 when such a page's count is above 1, the request takes the next page of
      a free list given with the call, copies into it the rows of the page
      that precede its first new token (rows 0 .. offset-1, every KV head,
      K and V), points its table entry at it, sets its count to 1 and lowers
      the shared page's count by one.  The last request still naming a page
      writes into it in place.
  R17 new tokens of a request come in increasing positions, the tokens of one
      request contiguous in the call.
"""
from __future__ import annotations

import numpy as np


def kv_append_cow(k_pool, v_pool, page_table, refcount, free_pages, k_new, v_new, token_req,
                  token_pos, page_size: int) -> int:
    """Append row t of k_new/v_new ([T][Hkv][d] bf16 bits) at position
    token_pos[t] of request token_req[t], copying shared pages first (R15-R17).

    page_table [B][max_pages] int32, refcount [num_pages] int32 and the pools
    are modified in place.  Returns how many pages of free_pages were taken
    (always a prefix of the list).  Raises when the free list runs out."""
    used = 0
    for t in range(len(token_req)):
        r, pos = int(token_req[t]), int(token_pos[t])
        entry, off = divmod(pos, page_size)
        first_of_request = t == 0 or int(token_req[t - 1]) != r
        if first_of_request or off == 0:
            page = int(page_table[r][entry])
            if refcount[page] > 1:
                if used >= len(free_pages):
                    raise ValueError("free page list exhausted")
                fresh = int(free_pages[used])
                used += 1
                k_pool[fresh, :, :off, :] = k_pool[page, :, :off, :]
                v_pool[fresh, :, :off, :] = v_pool[page, :, :off, :]
                refcount[page] -= 1
                refcount[fresh] = 1
                page_table[r][entry] = fresh
        page = int(page_table[r][entry])
        k_pool[page, :, off, :] = k_new[t]
        v_pool[page, :, off, :] = v_new[t]
    return used


def table_refcounts(page_table, lengths, page_size: int, num_pages: int) -> np.ndarray:
    """How many table entries name each page, over the entries that hold the
    first lengths[r] tokens of each request r."""
    rc = np.zeros(num_pages, dtype=np.int64)
    for r, L in enumerate(lengths):
        for e in range(-(-int(L) // page_size)):
            rc[int(page_table[r][e])] += 1
    return rc
