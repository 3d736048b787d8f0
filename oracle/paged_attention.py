"""Plain fp64 CPU oracle for attention on a paged KV cache.

TEST INFRASTRUCTURE ONLY.  Only tests, the smoke check and the benchmark's
CPU-baseline leg may import this module; the library never does.  It shares no
code with the CUDA path: it is written from the definitions on the pages and
from the mathematics of softmax attention, slowly and in full precision.

What it computes, and where the pages define it:

* Page pool and page tables -- tiny-llm source reading, section "Paged KV
  Cache": K/V live in a shared pool of fixed-size pages; each request keeps a
  page table listing its pages in logical order (the page's example: request A
  -> pages 7, 2, 11; B -> 4, 9); attention reads the discrete pages through
  the table instead of a concatenated KV tensor ("direct paged attention").
* kv_append -- the same section: pages are handed out on demand and the new
  K/V rows of a step are written into them.  A slot number names one row of
  the pool: slot = page * P + offset.  Slot -1 means "skip" (a padding row).
* GQA -- tiny-llm source reading, week 1 ("Query heads and KV heads differ in
  number"), and the tiny-llm course outline (chapter 1.3, grouped-query
  attention): G = Hq / Hkv query heads share one KV head.
* Causal mask -- tiny-llm source reading, week 1 (the attention interface
  includes the causal mask); chunked prefill at a context offset -- the same
  page, section "Chunked Prefill".
* Softmax attention and its log-sum-exp -- the attention tiny-vllm derives
  from scratch (tiny-vllm article, "From Safetensors to PagedAttention");
  the online softmax there reaches this same result, so the oracle computes
  the plain definition softmax(scale * q K^T) V with no online rescaling.
* Split-K -- mini-vllm advanced series design, section 4, Phase B, adv04
  "Flash-Decoding": a long context is cut along the KV length into
  partitions whose partial results are then combined.

Readings taken where the pages are silent:
  R1  query head h uses KV head h // G (contiguous groups);
  R2  a decode request's kv_len counts the token appended this step, whose
      query sits at position kv_len - 1; a prefill chunk of n rows after c
      context tokens occupies positions c .. c+n-1;
  R3  pool layout [num_pages][Hkv][P][d], separate K and V pools;
  R4  scale is passed in (1/sqrt(d) for every workload here);
  R5  split-K combine: M = max_s lse_s, w_s = exp(lse_s - M),
      o = sum_s w_s o_s / sum_s w_s, lse = M + log(sum_s w_s);
  R6  key j is visible to the query at position p iff j <= p;
  R7  a request with no keys yields a zero output and lse = -inf.

Every function is pinned by tests that do not re-type these formulas: a
library attention routine on contiguous tensors, closed forms, invariances
under page permutation and page size, causal perturbation, a hand-worked
two-key example, and the split/combine identity.
"""
from __future__ import annotations

import numpy as np


# ------------------------------------------------------------------ values
def bf16_bits_to_f64(bits) -> np.ndarray:
    """Decode bfloat16 bit patterns (uint16) to float64, exactly."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ------------------------------------------------------- small named steps
def _kv_head_of(h: int, group: int) -> int:
    """R1: query head h reads KV head h // G."""
    return h // group


def _page_and_offset(j: int, page_size: int):
    """Logical token j of a request lives in table entry j // P, row j % P."""
    return j // page_size, j % page_size


def _visible(key_pos: np.ndarray, query_pos: int) -> np.ndarray:
    """R6: causal visibility, diagonal included."""
    return key_pos <= query_pos


def _scores(queries: np.ndarray, keys: np.ndarray, scale: float) -> np.ndarray:
    """Scaled dot products: queries [..., d] against key rows [L][d] -> [..., L]."""
    return scale * (queries @ keys.T)


def _softmax_attend(s: np.ndarray, v: np.ndarray):
    """softmax over the last axis of scores s, applied to rows v.

    s: [..., L] scaled scores (fp64); v: [L, d].  Returns (o [..., d], lse).
    """
    if s.shape[-1] == 0:  # R7
        return (np.zeros(s.shape[:-1] + (v.shape[-1],)),
                np.full(s.shape[:-1], -np.inf))
    m = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - m)
    l = np.sum(e, axis=-1, keepdims=True)
    o = (e / l) @ v
    lse = (m + np.log(l))[..., 0]
    return o, lse


# -------------------------------------------------------------- kv_append
def kv_append(k_pool, v_pool, k_new, v_new, slot_mapping, page_size: int) -> None:
    """Write row t of k_new/v_new (all KV heads) into pool slot slot_mapping[t].

    Pools are uint16 bf16 bit arrays [num_pages][Hkv][P][d], modified in
    place; k_new/v_new are [T][Hkv][d].  Slot -1 skips the row.  A pure bit
    copy: no value is converted.
    """
    for t in range(len(slot_mapping)):
        slot = int(slot_mapping[t])
        if slot < 0:
            continue
        page, off = divmod(slot, page_size)
        k_pool[page, :, off, :] = k_new[t]
        v_pool[page, :, off, :] = v_new[t]


# --------------------------------------------------------- page-table walk
def gather_request_kv(pool, page_table_row, n_tokens: int, page_size: int) -> np.ndarray:
    """Direct paged read: the first n_tokens rows of one request, in order.

    Walks the request's page table and copies each page's rows out of the
    pool.  Returns bf16 bits [n_tokens][Hkv][d].
    """
    hkv, d = pool.shape[1], pool.shape[3]
    rows = np.empty((n_tokens, hkv, d), dtype=pool.dtype)
    for j in range(n_tokens):
        entry, off = _page_and_offset(j, page_size)
        page = int(page_table_row[entry])
        rows[j] = pool[page, :, off, :]
    return rows


# ---------------------------------------------------------------- decode
def decode_attention(q, k_pool, v_pool, page_table, kv_lens, page_size: int,
                     scale: float, ids=None, token_range=None):
    """q_len = 1 attention of each request over its whole paged context.

    q: bf16 bits [B][Hq][d]; kv_lens[r] keys per request (R2).  ids limits
    the work to some requests (others are left NaN).  token_range(r) may
    return (t0, t1) to restrict the keys to [t0, t1) -- one split-K
    partition.  Returns out fp64 [B][Hq][d] and lse fp64 [B][Hq] (natural
    log of the softmax denominator of the scaled scores).
    """
    q = np.asarray(q)
    B, hq, d = q.shape
    hkv = k_pool.shape[1]
    group = hq // hkv
    out = np.full((B, hq, d), np.nan)
    lse = np.full((B, hq), np.nan)
    for r in (range(B) if ids is None else ids):
        L = int(kv_lens[r])
        t0, t1 = (0, L) if token_range is None else token_range(r)
        K = bf16_bits_to_f64(gather_request_kv(k_pool, page_table[r], L, page_size))[t0:t1]
        V = bf16_bits_to_f64(gather_request_kv(v_pool, page_table[r], L, page_size))[t0:t1]
        qf = bf16_bits_to_f64(q[r])
        for h in range(hq):
            g = _kv_head_of(h, group)
            s = _scores(qf[h], K[:, g, :], scale)
            out[r, h], lse[r, h] = _softmax_attend(s, V[:, g, :])
    return out, lse


# --------------------------------------------------------------- split-K
def decode_partials(q, k_pool, v_pool, page_table, kv_lens, page_size: int,
                    scale: float, partition: int, ids=None):
    """Split-K partial results: split s of request r covers keys
    [s*partition, min((s+1)*partition, L)).  Each partial is normalised within
    its split and carries that split's lse.

    Returns part_o [B][Hq][S][d], part_lse [B][Hq][S], num_splits [B] with
    S = max over requests of ceil(L / partition); unused splits are NaN.
    """
    B, hq, d = np.asarray(q).shape
    kv_lens = np.asarray(kv_lens)
    num_splits = np.array([-(-int(L) // partition) for L in kv_lens], dtype=np.int32)
    S = max(1, int(num_splits.max(initial=0)))
    part_o = np.full((B, hq, S, d), np.nan)
    part_lse = np.full((B, hq, S), np.nan)
    for s in range(S):
        sel = [r for r in (range(B) if ids is None else ids) if s < num_splits[r]]
        if not sel:
            continue
        o, l = decode_attention(
            q, k_pool, v_pool, page_table, kv_lens, page_size, scale, ids=sel,
            token_range=lambda r: (s * partition, min((s + 1) * partition, int(kv_lens[r]))))
        part_o[sel, :, s] = o[sel]
        part_lse[sel, :, s] = l[sel]
    return part_o, part_lse, num_splits


def split_k_combine(part_o, part_lse, num_splits):
    """R5: merge split-K partials by their log-sum-exp weights.

    Splits whose lse is -inf (no keys) get weight zero; a request whose every
    split is empty gets a zero output and lse -inf.
    """
    B, hq, _, d = part_o.shape
    out = np.zeros((B, hq, d))
    lse = np.full((B, hq), -np.inf)
    for r in range(B):
        n = int(num_splits[r])
        for h in range(hq):
            ls = part_lse[r, h, :n]
            if n == 0 or not np.isfinite(ls).any():
                continue
            M = np.max(ls)
            w = np.exp(ls - M)
            out[r, h] = (w[:, None] * part_o[r, h, :n]).sum(axis=0) / w.sum()
            lse[r, h] = M + np.log(w.sum())
    return out, lse


# -------------------------------------------------------- chunked prefill
def chunked_prefill_attention(q, cu_q_lens, ctx_offsets, k_pool, v_pool,
                              page_table, page_size: int, scale: float,
                              ids=None):
    """Causal attention of each request's prompt chunk over its paged keys.

    Request r owns query rows cu_q_lens[r] .. cu_q_lens[r+1]-1 of q
    ([T][Hq][d] bf16 bits); row i sits at position ctx_offsets[r] + i (R2)
    and sees keys 0 .. ctx_offsets[r] + i (R6).  The chunk's own K/V rows
    are expected in the pool already (appended before attention).
    Returns out fp64 [T][Hq][d] and lse fp64 [T][Hq]; rows of requests not
    in ids stay NaN.
    """
    q = np.asarray(q)
    T, hq, d = q.shape
    hkv = k_pool.shape[1]
    group = hq // hkv
    out = np.full((T, hq, d), np.nan)
    lse = np.full((T, hq), np.nan)
    B = len(cu_q_lens) - 1
    for r in (range(B) if ids is None else ids):
        a, b = int(cu_q_lens[r]), int(cu_q_lens[r + 1])
        c = int(ctx_offsets[r])
        n_keys = c + (b - a)
        K = bf16_bits_to_f64(gather_request_kv(k_pool, page_table[r], n_keys, page_size))
        V = bf16_bits_to_f64(gather_request_kv(v_pool, page_table[r], n_keys, page_size))
        key_pos = np.arange(n_keys)
        # visible[i, j]: key j is visible to chunk row i (position c + i)
        visible = np.stack([_visible(key_pos, c + i) for i in range(b - a)]) \
            if b > a else np.zeros((0, n_keys), bool)
        for h in range(hq):
            g = _kv_head_of(h, group)
            Qh = bf16_bits_to_f64(q[a:b, h, :])           # [n][d]
            s = _scores(Qh, K[:, g, :], scale)             # [n][n_keys]
            # a hidden key gets score -inf, i.e. softmax weight exactly 0
            s = np.where(visible, s, -np.inf)
            out[a:b, h], lse[a:b, h] = _softmax_attend(s, V[:, g, :])
    return out, lse
