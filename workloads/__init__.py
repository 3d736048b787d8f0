"""Seeded synthetic workloads for paged KV attention.

This module only builds inputs: request lengths, page tables drawn from a
shared page pool, slot numbers for the rows each step appends, and the bf16
Q/K/V rows themselves.  It holds none of the attention arithmetic, and it is
the one module that both the CUDA path's tests/bench and the CPU oracle use.

Shapes follow the workloads the pages describe:
  * "tiny_decode"          - 4 requests, lengths {7,33,64,100}, 16/8 heads,
                              d=128, page 16, 64-page pool (tiny-llm's Qwen3
                              GQA shape at toy size).
  * "qwen3_decode"         - Qwen3-4B decode layer: 64 slots, 32/8 heads,
                              d=128, page 16, lengths U[128,4096], K rows
                              RMS-normalised (Qwen3 applies QK-norm before
                              attention).
  * "mixed_prefill_decode" - 8 requests prefilling 512-token chunks at prior
                              offsets U[0,8192] plus 56 decode requests with
                              lengths U[256,4096] in one batch.
  * "splitk_long"          - Llama-3.2-1B shapes (32/8 heads, d=64), 4 long
                              contexts 32k..128k, the flash-decoding case.
  * "spec_verify"          - speculative-decoding verify: 64 requests of
                              the Qwen3-4B layer, 4 query rows each (3 draft
                              tokens + the last accepted one) at the end of
                              contexts U[128,4096].
  * "frag_large"           - 256 requests, lognormal lengths (median 1536,
                              sigma 0.8, clipped [16,16384]), page 32, page
                              tables produced by an alloc/free trace over a
                              LIFO free list so they are non-monotonic.

Pages: tiny-llm's source-reading page ("Paged KV Cache") describes a shared
pool of fixed-size pages handed out on demand and returned when a request
finishes, with a per-request page table (its example: A -> 7,2,11; B -> 4,9).
That is what the page tables here model.

Values: every bf16 row is drawn per request from numpy's PCG64 seeded with
(seed, request, stream), so any subset of requests can be regenerated on the
host without generating the rest.  ``fill_device_*`` helpers draw the bulk of a
large pool directly on the GPU for timing runs.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

BF16_NAN = np.uint16(0x7FC0)

CONFIG_NAMES = (
    "tiny_decode",
    "qwen3_decode",
    "mixed_prefill_decode",
    "splitk_long",
    "frag_large",
)

# stream ids for the per-request generators
_S_CTX_K, _S_CTX_V, _S_NEW_K, _S_NEW_V, _S_Q = 1, 2, 3, 4, 5


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (round-to-nearest-even) and return the bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    out = rounded.astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        out[nan] = BF16_NAN
    return out


def _rms_normalise(x: np.ndarray) -> np.ndarray:
    """Scale each length-d row (last axis) to unit root-mean-square, in fp32."""
    ms = np.mean(x.astype(np.float32) ** 2, axis=-1, keepdims=True)
    return (x / np.sqrt(ms)).astype(np.float32)


@dataclass
class Workload:
    """One batch of one layer: page pool geometry, page tables and lengths.

    For request r:
      ctx_lens[r]  tokens already in the pool before this step,
      new_lens[r]  tokens this step appends (1 for a decode request, the chunk
                   length for a prefill request),
      kv_lens[r] = ctx_lens[r] + new_lens[r], the keys the step attends to.
    Decode requests put their one query at position kv_lens[r]-1; a prefill
    request's chunk occupies positions ctx_lens[r] .. kv_lens[r]-1.
    """

    name: str
    seed: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    page_size: int
    num_pages: int
    page_table: np.ndarray  # int32 [B, max_pages], -1 where unused
    ctx_lens: np.ndarray  # int32 [B]
    new_lens: np.ndarray  # int32 [B]
    is_prefill: np.ndarray  # bool [B]
    k_rms_norm: bool = False
    notes: dict = field(default_factory=dict)

    # ----------------------------------------------------------- geometry
    @property
    def B(self) -> int:
        return int(self.page_table.shape[0])

    @property
    def max_pages(self) -> int:
        return int(self.page_table.shape[1])

    @property
    def kv_lens(self) -> np.ndarray:
        return (self.ctx_lens + self.new_lens).astype(np.int32)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    @property
    def decode_ids(self) -> np.ndarray:
        return np.nonzero(~self.is_prefill)[0]

    @property
    def prefill_ids(self) -> np.ndarray:
        return np.nonzero(self.is_prefill)[0]

    def kv_bytes_read(self, ids=None) -> int:
        """Algorithmic K+V bytes attention reads for the given requests."""
        ids = np.arange(self.B) if ids is None else np.asarray(ids)
        toks = int(self.kv_lens[ids].astype(np.int64).sum())
        return toks * 2 * self.num_kv_heads * self.head_dim * 2

    def pool_shape(self):
        return (self.num_pages, self.num_kv_heads, self.page_size, self.head_dim)

    # ------------------------------------------------------------- slots
    def slots(self, r: int, start: int, stop: int) -> np.ndarray:
        """Pool slot numbers (page*P + offset) of positions [start, stop) of r.

        This is the caller-side bookkeeping a scheduler does when it hands
        kv_append its slot mapping (tiny-llm's TinyLlmBatch / page table).
        """
        pos = np.arange(start, stop, dtype=np.int64)
        pages = self.page_table[r, pos // self.page_size].astype(np.int64)
        assert (pages >= 0).all(), "position beyond the request's pages"
        return (pages * self.page_size + pos % self.page_size).astype(np.int32)

    def ctx_slots(self, ids=None) -> np.ndarray:
        ids = range(self.B) if ids is None else ids
        parts = [self.slots(r, 0, int(self.ctx_lens[r])) for r in ids]
        return np.concatenate(parts) if parts else np.zeros(0, np.int32)

    def new_slots(self, ids=None) -> np.ndarray:
        ids = range(self.B) if ids is None else ids
        parts = [self.slots(r, int(self.ctx_lens[r]), int(self.kv_lens[r])) for r in ids]
        return np.concatenate(parts) if parts else np.zeros(0, np.int32)

    # ------------------------------------------------------------ values
    def _rng(self, r: int, stream: int) -> np.random.Generator:
        return np.random.Generator(np.random.PCG64([self.seed, int(r), stream]))

    def _rows(self, r: int, stream: int, n: int, heads: int, is_key: bool) -> np.ndarray:
        x = self._rng(r, stream).standard_normal((n, heads, self.head_dim), dtype=np.float32)
        if is_key and self.k_rms_norm:
            x = _rms_normalise(x)
        return f32_to_bf16_bits(x)

    def ctx_rows(self, r: int):
        """bf16 bits of K and V for positions [0, ctx_lens[r]) of request r."""
        n = int(self.ctx_lens[r])
        return (self._rows(r, _S_CTX_K, n, self.num_kv_heads, True),
                self._rows(r, _S_CTX_V, n, self.num_kv_heads, False))

    def new_rows(self, r: int):
        """bf16 bits of the K and V rows request r appends this step."""
        n = int(self.new_lens[r])
        return (self._rows(r, _S_NEW_K, n, self.num_kv_heads, True),
                self._rows(r, _S_NEW_V, n, self.num_kv_heads, False))

    def q_rows(self, r: int) -> np.ndarray:
        """bf16 bits of request r's query rows [new_lens[r], Hq, d]."""
        return self._rows(r, _S_Q, int(self.new_lens[r]), self.num_q_heads, False)

    # ------------------------------------------------ batched host views
    def batch_new(self, ids=None):
        """Concatenated new K/V rows and their slots for the given requests."""
        ids = list(range(self.B)) if ids is None else list(ids)
        ks, vs = zip(*[self.new_rows(r) for r in ids]) if ids else ((), ())
        shape = (0, self.num_kv_heads, self.head_dim)
        k = np.concatenate(ks) if ids else np.zeros(shape, np.uint16)
        v = np.concatenate(vs) if ids else np.zeros(shape, np.uint16)
        return k, v, self.new_slots(ids)

    def batch_ctx(self, ids=None):
        ids = list(range(self.B)) if ids is None else list(ids)
        ks, vs = zip(*[self.ctx_rows(r) for r in ids]) if ids else ((), ())
        shape = (0, self.num_kv_heads, self.head_dim)
        k = np.concatenate(ks) if ids else np.zeros(shape, np.uint16)
        v = np.concatenate(vs) if ids else np.zeros(shape, np.uint16)
        return k, v, self.ctx_slots(ids)

    def batch_q(self, ids):
        """Queries of the given requests, concatenated [sum new_lens, Hq, d]."""
        ids = list(ids)
        if not ids:
            return np.zeros((0, self.num_q_heads, self.head_dim), np.uint16)
        return np.concatenate([self.q_rows(r) for r in ids])

    def cu_q_lens(self, ids) -> np.ndarray:
        ids = list(ids)
        return np.concatenate([[0], np.cumsum(self.new_lens[ids])]).astype(np.int32)

    def empty_pool(self) -> np.ndarray:
        """A pool of NaN bf16: slots nobody wrote stay NaN so a stray read shows."""
        return np.full(self.pool_shape(), BF16_NAN, dtype=np.uint16)

    def describe(self) -> dict:
        return {
            "workload": self.name,
            "batch": self.B,
            "num_q_heads": self.num_q_heads,
            "num_kv_heads": self.num_kv_heads,
            "head_dim": self.head_dim,
            "page_size": self.page_size,
            "num_pages": self.num_pages,
            "kv_tokens": int(self.kv_lens.astype(np.int64).sum()),
            "prefill_requests": int(self.is_prefill.sum()),
            "prefill_rows": int(self.new_lens[self.is_prefill].sum()),
            "seed": self.seed,
        }


# ---------------------------------------------------------------- builders
def _permuted_tables(rng, kv_lens, page_size, num_pages, max_pages=None):
    """Give each request its pages from one random permutation of the pool."""
    need = [(int(L) + page_size - 1) // page_size for L in kv_lens]
    if max_pages is None:
        max_pages = max(need) if need else 1
    assert sum(need) <= num_pages
    perm = rng.permutation(num_pages).astype(np.int32)
    table = np.full((len(kv_lens), max(max_pages, 1)), -1, dtype=np.int32)
    at = 0
    for r, n in enumerate(need):
        table[r, :n] = perm[at:at + n]
        at += n
    return table


def _trace_tables(rng, lens_a, lens_b_fn, page_size, free_frac=0.3):
    """Page tables from an allocation trace over a LIFO free list.

    Phase 1 grows every request one page at a time, choosing the request at
    random each step.  Phase 2 frees a random ``free_frac`` of the requests
    (their pages go back on top of the free stack).  Phase 3 gives the freed
    requests fresh lengths and grows them again in random order.  Pages come
    back in a scrambled, non-monotonic order, as in a pool that has served a
    while.  Returns (table, final_lens, num_pages).
    """
    B = len(lens_a)
    need_a = np.array([(int(L) + page_size - 1) // page_size for L in lens_a])
    freed = np.sort(rng.choice(B, size=int(round(free_frac * B)), replace=False))
    lens = np.array(lens_a, dtype=np.int64)
    lens[freed] = lens_b_fn(len(freed))
    need_b = np.array([(int(L) + page_size - 1) // page_size for L in lens])
    peak = max(int(need_a.sum()), int(need_b.sum()))
    num_pages = int(math.ceil(1.25 * peak))
    free = list(range(num_pages - 1, -1, -1))  # pop() hands out 0, 1, 2, ...
    pages = [[] for _ in range(B)]

    def grow(ids, need):
        want = {int(r): int(need[r]) for r in ids}
        pending = [r for r in want for _ in range(want[r])]
        order = rng.permutation(len(pending))
        for i in order:
            pages[pending[i]].append(free.pop())

    grow(range(B), need_a)
    for r in rng.permutation(freed):
        while pages[r]:
            free.append(pages[r].pop())
    grow(freed, need_b)
    max_pages = max(len(p) for p in pages)
    table = np.full((B, max_pages), -1, dtype=np.int32)
    for r, p in enumerate(pages):
        table[r, :len(p)] = p
    return table, lens.astype(np.int32), num_pages


def make_workload(name: str, seed: int = 0, **over) -> Workload:
    """Build one of the named workloads; keyword overrides shrink it for tests.

    Recognised overrides: B (batch), len_lo/len_hi (uniform lengths),
    lens (explicit kv lengths), n_prefill/chunk/chunks/ctx_hi/ctxs/n_decode
    (mixed batch),
    median (lognormal median), max_len, page_size, num_q_heads, num_kv_heads,
    head_dim.
    """
    rng = np.random.Generator(np.random.PCG64([seed, 0xC0FFEE]))
    if name == "tiny_decode":
        Hq, Hkv, D, P = over.get("num_q_heads", 16), over.get("num_kv_heads", 8), over.get("head_dim", 128), over.get("page_size", 16)
        kv = np.array(over.get("lens", [7, 33, 64, 100]), dtype=np.int32)
        num_pages = over.get("num_pages", 64)
        table = _permuted_tables(rng, kv, P, num_pages)
        return Workload(name, seed, Hq, Hkv, D, P, num_pages, table,
                        kv - 1, np.ones_like(kv), np.zeros(len(kv), bool))
    if name == "qwen3_decode":
        Hq, Hkv, D, P = over.get("num_q_heads", 32), over.get("num_kv_heads", 8), over.get("head_dim", 128), over.get("page_size", 16)
        B = over.get("B", 64)
        kv = over.get("lens")
        if kv is None:
            kv = rng.integers(over.get("len_lo", 128), over.get("len_hi", 4096), size=B, endpoint=True)
        kv = np.asarray(kv, dtype=np.int32)
        need = int(sum((int(L) + P - 1) // P for L in kv))
        num_pages = int(math.ceil(1.25 * need))
        table = _permuted_tables(rng, kv, P, num_pages)
        return Workload(name, seed, Hq, Hkv, D, P, num_pages, table,
                        kv - 1, np.ones_like(kv), np.zeros(len(kv), bool), k_rms_norm=True)
    if name == "mixed_prefill_decode":
        Hq, Hkv, D, P = over.get("num_q_heads", 32), over.get("num_kv_heads", 8), over.get("head_dim", 128), over.get("page_size", 16)
        n_pre, chunk = over.get("n_prefill", 8), over.get("chunk", 512)
        n_dec = over.get("n_decode", 56)
        ctx_pre = rng.integers(0, over.get("ctx_hi", 8192), size=n_pre, endpoint=True)
        if "ctxs" in over:
            ctx_pre = np.asarray(over["ctxs"], dtype=np.int64)
        chunks = np.asarray(over.get("chunks", [chunk] * n_pre), dtype=np.int64)
        kv_dec = rng.integers(over.get("len_lo", 256), over.get("len_hi", 4096), size=n_dec, endpoint=True)
        ctx = np.concatenate([ctx_pre, kv_dec - 1]).astype(np.int32)
        new = np.concatenate([chunks, np.ones(n_dec, np.int64)]).astype(np.int32)
        kv = ctx + new
        need = int(sum((int(L) + P - 1) // P for L in kv))
        num_pages = int(math.ceil(1.25 * need))
        table = _permuted_tables(rng, kv, P, num_pages)
        is_pre = np.concatenate([np.ones(n_pre, bool), np.zeros(n_dec, bool)])
        return Workload(name, seed, Hq, Hkv, D, P, num_pages, table, ctx, new, is_pre)
    if name == "splitk_long":
        Hq, Hkv, D, P = over.get("num_q_heads", 32), over.get("num_kv_heads", 8), over.get("head_dim", 64), over.get("page_size", 16)
        kv = np.asarray(over.get("lens", [32768, 65536, 98304, 131072]), dtype=np.int32)
        need = int(sum((int(L) + P - 1) // P for L in kv))
        num_pages = int(math.ceil(1.25 * need))
        max_pages = over.get("max_pages", (int(kv.max()) + P - 1) // P)
        table = _permuted_tables(rng, kv, P, num_pages, max_pages)
        return Workload(name, seed, Hq, Hkv, D, P, num_pages, table,
                        kv - 1, np.ones_like(kv), np.zeros(len(kv), bool))
    if name == "frag_large":
        Hq, Hkv, D, P = over.get("num_q_heads", 32), over.get("num_kv_heads", 8), over.get("head_dim", 128), over.get("page_size", 32)
        B = over.get("B", 256)
        med, sig = over.get("median", 1536.0), over.get("sigma", 0.8)
        lo, hi = over.get("min_len", 16), over.get("max_len", 16384)

        def draw(n):
            z = rng.standard_normal(n)
            return np.clip(np.round(np.exp(np.log(med) + sig * z)), lo, hi).astype(np.int64)

        table, kv, num_pages = _trace_tables(rng, draw(B), draw, P)
        return Workload(name, seed, Hq, Hkv, D, P, num_pages, table,
                        kv - 1, np.ones_like(kv), np.zeros(len(kv), bool),
                        notes={"trace": "grow-all / free 30% / regrow, LIFO free list"})
    if name == "spec_verify":
        # every request verifies q_len tokens (draft tokens plus the last
        # accepted one) over its context: chunk rows at kv_len - q_len ..
        # kv_len - 1
        Hq, Hkv, D, P = over.get("num_q_heads", 32), over.get("num_kv_heads", 8), over.get("head_dim", 128), over.get("page_size", 16)
        B, q_len = over.get("B", 64), over.get("q_len", 4)
        kv = rng.integers(over.get("len_lo", 128), over.get("len_hi", 4096), size=B, endpoint=True).astype(np.int32)
        need = int(sum((int(L) + P - 1) // P for L in kv))
        num_pages = int(math.ceil(1.25 * need))
        table = _permuted_tables(rng, kv, P, num_pages)
        new = np.full(B, q_len, np.int32)
        return Workload(name, seed, Hq, Hkv, D, P, num_pages, table, kv - new, new, np.ones(B, bool),
                        k_rms_norm=True, notes={"attention": "verify"})
    raise ValueError(f"unknown workload {name!r}; known: {CONFIG_NAMES}")
