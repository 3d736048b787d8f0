"""Seeded shared-prefix scenarios: page tables that name the same pool pages
for a common prompt prefix, with per-page reference counts and a free list.

This module only builds inputs (the state a prefix-caching page manager
would hand to the append step); it holds none of the attention or
copy-on-write arithmetic.

A scenario has groups of requests that fork from one prompt prefix of Lg
tokens (mini-vllm advanced series design, adv05: automatic prefix reuse with
copy-on-write; the main series keeps a hash and a ref_count per block):
  * the pages wholly inside the prefix are shared by every request of the
    group;
  * a "just forked" request (parallel sampling, beam search) has no token of
    its own yet: it also shares the prefix's partly filled last page, so its
    first append lands in a shared page;
  * a request that already has its own continuation holds a private copy of
    that partly filled page, followed by private pages.
Each request then appends n_new rows at positions ctx .. ctx + n_new - 1.
Pages that those rows open (offset 0 past the request's last page) are taken
from the free list up front, as the page manager would; the rest of the free
list is what the copy-on-write append may take.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from . import f32_to_bf16_bits

NAN16 = np.uint16(0x7FC0)


@dataclass
class PrefixScenario:
    page_size: int
    num_kv_heads: int
    head_dim: int
    k_pool: np.ndarray      # uint16 [num_pages][Hkv][P][d]
    v_pool: np.ndarray
    page_table: np.ndarray  # int32 [B][max_pages], -1 unused
    refcount: np.ndarray    # int32 [num_pages]: table entries naming each page
    free_pages: np.ndarray  # int32 [n_free]
    ctx_lens: np.ndarray    # int32 [B]: tokens before this step
    token_req: np.ndarray   # int32 [T]
    token_pos: np.ndarray   # int32 [T]
    k_new: np.ndarray       # uint16 [T][Hkv][d]
    v_new: np.ndarray
    group_of: np.ndarray    # int32 [B]

    @property
    def B(self) -> int:
        return int(self.page_table.shape[0])

    @property
    def num_pages(self) -> int:
        return int(self.k_pool.shape[0])

    @property
    def kv_lens(self) -> np.ndarray:
        n = np.bincount(self.token_req, minlength=self.B)
        return (self.ctx_lens + n).astype(np.int32)


def _rows(rng, n, hkv, d):
    return f32_to_bf16_bits(rng.standard_normal((n, hkv, d)).astype(np.float32))


def make_prefix_scenario(seed: int, groups=((37, 3, 0), (64, 2, 1), (50, 4, 2)), page_size=16,
                         num_kv_heads=2, head_dim=64, n_new=1, spare_pages=8) -> PrefixScenario:
    """groups: (prefix length, requests, of which already continued) per group.

    Already-continued requests hold a private continuation of 1..2*P tokens."""
    rng = np.random.Generator(np.random.PCG64([seed, 0xFEED]))
    P, hkv, d = page_size, num_kv_heads, head_dim
    # plan every request's page count to size the pool
    plan = []  # (group, prefix len, private len)
    for gi, (Lg, n_req, n_cont) in enumerate(groups):
        for j in range(n_req):
            own = int(rng.integers(1, 2 * P + 1)) if j < n_cont else 0
            plan.append((gi, Lg, own))
    B = len(plan)
    max_len = max(Lg + own + n_new for _, Lg, own in plan)
    max_pages = -(-max_len // P)
    need = sum(-(-Lg // P) for Lg, _, _ in groups) + sum(-(-(Lg + own + n_new) // P) for _, Lg, own in plan)
    num_pages = need + spare_pages
    order = [int(x) for x in rng.permutation(num_pages)]
    take = order.pop
    kp = np.full((num_pages, hkv, P, d), NAN16, np.uint16)
    vp = kp.copy()
    table = np.full((B, max_pages), -1, np.int32)
    ctx = np.zeros(B, np.int32)
    group_pages = []
    for gi, (Lg, _, _) in enumerate(groups):
        pages = [take() for _ in range(-(-Lg // P))]
        k, v = _rows(rng, Lg, hkv, d), _rows(rng, Lg, hkv, d)
        for pos in range(Lg):
            kp[pages[pos // P], :, pos % P] = k[pos]
            vp[pages[pos // P], :, pos % P] = v[pos]
        group_pages.append(pages)
    for r, (gi, Lg, own) in enumerate(plan):
        pages = list(group_pages[gi])
        full = Lg // P
        if own > 0 and Lg % P:
            # a private copy of the prefix's partly filled page
            mine = take()
            kp[mine, :, :Lg % P] = kp[pages[full], :, :Lg % P]
            vp[mine, :, :Lg % P] = vp[pages[full], :, :Lg % P]
            pages[full] = mine
        L = Lg + own
        while len(pages) < -(-L // P):
            pages.append(take())
        if own:
            k, v = _rows(rng, own, hkv, d), _rows(rng, own, hkv, d)
            for i, pos in enumerate(range(Lg, L)):
                kp[pages[pos // P], :, pos % P] = k[i]
                vp[pages[pos // P], :, pos % P] = v[i]
        table[r, :len(pages)] = pages
        ctx[r] = L
    # pages opened by this step's rows come from the free list up front
    for r in range(B):
        L = int(ctx[r])
        for e in range(-(-L // P), -(-(L + n_new) // P)):
            table[r, e] = take()
    rc = np.zeros(num_pages, np.int32)
    for r in range(B):
        for e in range(-(-(int(ctx[r]) + n_new) // P)):
            rc[table[r, e]] += 1
    token_req = np.repeat(np.arange(B, dtype=np.int32), n_new)
    token_pos = np.concatenate([np.arange(int(ctx[r]), int(ctx[r]) + n_new) for r in range(B)]).astype(np.int32)
    T = len(token_req)
    return PrefixScenario(P, hkv, d, kp, vp, table, rc, np.array(order[::-1], np.int32), ctx,
                          token_req, token_pos, _rows(rng, T, hkv, d), _rows(rng, T, hkv, d),
                          np.array([g for g, _, _ in plan], np.int32))


def private_copy(s: PrefixScenario):
    """The same logical contents with no page shared: every request gets its
    own copy of each page it names (pages renumbered; pool grown).  Returns
    (k_pool, v_pool, page_table) with each request's pages private."""
    B, P = s.B, s.page_size
    counts = [int(np.sum(s.page_table[r] >= 0)) for r in range(B)]
    n = sum(counts)
    kp = np.full((n,) + s.k_pool.shape[1:], NAN16, np.uint16)
    vp = kp.copy()
    table = np.full_like(s.page_table, -1)
    at = 0
    for r in range(B):
        for e in range(counts[r]):
            kp[at] = s.k_pool[s.page_table[r, e]]
            vp[at] = s.v_pool[s.page_table[r, e]]
            table[r, e] = at
            at += 1
    return kp, vp, table
