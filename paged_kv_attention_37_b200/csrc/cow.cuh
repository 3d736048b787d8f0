// cow.cuh -- appending new K/V rows to page tables that share pages (a
// common prompt prefix), with copy-on-write, on the device.
//
// Source: mini-vllm advanced series design, section 4, Phase C, adv05
// "Radix Attention + Copy-on-Write" (automatic prefix reuse of the KV cache
// with copy-on-write; the main series keeps a hash and a ref_count per
// block); tiny-llm source reading, "Paged KV Cache" (pages handed out on
// demand).
//
// Several requests' tables may name the same pool page; page_refcount[p]
// counts the table entries that do.  A request may append into a shared page
// only at its first new token (later tokens open pages the page manager
// handed out fresh); that page, and every page a new token opens at offset
// 0, is settled first:
//   prepare kernel, one warp per new token (the settling ones act): the
//     warp's lane 0 takes one reference off the page (atomicSub).  If it was
//     the last reference the request owns the page alone: the reference is
//     put back and the rows go in place.  Otherwise it pops the next page of
//     the caller's free list (atomicAdd on *free_used), the warp copies rows
//     0 .. offset-1 of every KV head, K and V, into it (only the rows before
//     the first new token: rows past it may hold stale data or, in this very
//     call, the in-place rows of the page's last sharer), the table entry is
//     pointed at the copy and its count set to 1.
//   append kernel (a programmatic dependent: it waits for the prepare grid),
//     one thread per 16-byte chunk of a new row: slot = table[r][pos / P] * P
//     + pos % P read from the settled table, then the bit copy of kv_append.
// Which sharer writes in place and which free page a request gets depend on
// the order of the atomics; what each request reads through its table does
// not.
#pragma once

#include "ptx.cuh"

namespace pkv {
namespace cow {

constexpr int kPrepWarps = 8;

struct Params {
  const uint4* k_new;           // [T][Hkv][D] bf16, as 16-byte chunks
  const uint4* v_new;
  const int32_t* token_req;     // [T]
  const int32_t* token_pos;     // [T]
  int32_t* page_table;          // [B][max_pages], updated in place
  int32_t* refcount;            // [num_pages], updated in place
  const int32_t* free_pages;    // [num_free]
  int32_t* free_used;           // pages taken from free_pages so far
  uint4* k_pool;                // [num_pages][Hkv][P][D]
  uint4* v_pool;
  int32_t T, B, max_pages, num_free, num_pages, Hkv, P;
};

// Row r's settled entry for this token, or -1 (and a flag) when the token's
// request or position lies outside the tables.
__device__ __forceinline__ int32_t* entry_of(const Params& p, int r, int pos) {
  if (static_cast<unsigned>(r) >= static_cast<unsigned>(p.B) || pos < 0 ||
      pos / p.P >= p.max_pages)
    return nullptr;
  return p.page_table + static_cast<size_t>(r) * p.max_pages + pos / p.P;
}

template <int D>
__global__ void __launch_bounds__(kPrepWarps * 32) prepare_kernel(const Params p) {
  constexpr int kChunks = D / 8;  // 16-byte chunks per row
  pdl_wait();
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kPrepWarps + (threadIdx.x >> 5);
  if (t >= p.T) return;
  const int r = p.token_req[t], pos = p.token_pos[t];
  const int off = pos % p.P;
  const bool settles = t == 0 || p.token_req[t - 1] != r || off == 0;
  if (!settles) return;
  int32_t* ent = entry_of(p, r, pos);
  if (ent == nullptr) {
    if (lane == 0) raise_flag(PKV_FLAG_BAD_LENGTH);
    return;
  }
  int page = 0, fresh = -1;
  if (lane == 0) {
    page = *ent;
    if (static_cast<unsigned>(page) >= static_cast<unsigned>(p.num_pages)) {
      raise_flag(PKV_FLAG_BAD_PAGE);
      page = -1;
    } else if (atomicSub(p.refcount + page, 1) == 1) {
      atomicAdd(p.refcount + page, 1);  // the only reference: write in place
    } else {
      const int idx = atomicAdd(p.free_used, 1);
      if (idx < p.num_free) {
        fresh = p.free_pages[idx];
        if (static_cast<unsigned>(fresh) >= static_cast<unsigned>(p.num_pages)) {
          raise_flag(PKV_FLAG_BAD_PAGE);
          fresh = -2;
        }
      } else {
        fresh = -2;
      }
      if (fresh == -2) {
        // no private page to be had: the request loses this entry (-1, so
        // its rows are skipped), having given up its reference
        raise_flag(PKV_FLAG_NO_FREE_PAGE);
        *ent = -1;
      }
    }
  }
  fresh = __shfl_sync(0xffffffffu, fresh, 0);
  page = __shfl_sync(0xffffffffu, page, 0);
  if (fresh < 0) return;
  // copy rows [0, off) of every KV head of both pools into the fresh page
  const int n = off * kChunks;  // chunks per (page, head) to copy
  for (int h = 0; h < p.Hkv; ++h) {
    const size_t src = (static_cast<size_t>(page) * p.Hkv + h) * p.P * kChunks;
    const size_t dst = (static_cast<size_t>(fresh) * p.Hkv + h) * p.P * kChunks;
    for (int i = lane; i < n; i += 32) {
      p.k_pool[dst + i] = p.k_pool[src + i];
      p.v_pool[dst + i] = p.v_pool[src + i];
    }
  }
  if (lane == 0) {
    p.refcount[fresh] = 1;
    *ent = fresh;
  }
}

template <int D>
__global__ void __launch_bounds__(256) append_kernel(const Params p) {
  constexpr int kChunks = D / 8;
  pdl_wait();  // the prepare grid has settled every table entry
  pdl_launch_dependents();
  const int64_t total = static_cast<int64_t>(p.T) * p.Hkv * kChunks;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(idx % kChunks);
    const int64_t row = idx / kChunks;
    const int h = static_cast<int>(row % p.Hkv);
    const int t = static_cast<int>(row / p.Hkv);
    const int r = __ldg(p.token_req + t), pos = __ldg(p.token_pos + t);
    const int32_t* ent = entry_of(p, r, pos);
    if (ent == nullptr) continue;  // flagged by the prepare kernel
    const int page = *ent;
    if (static_cast<unsigned>(page) >= static_cast<unsigned>(p.num_pages)) {
      if (page != -1 && c == 0 && h == 0) raise_flag(PKV_FLAG_BAD_PAGE);
      continue;
    }
    const size_t dst = ((static_cast<size_t>(page) * p.Hkv + h) * p.P + pos % p.P) * kChunks + c;
    p.k_pool[dst] = __ldg(p.k_new + idx);
    p.v_pool[dst] = __ldg(p.v_new + idx);
  }
}

}  // namespace cow
}  // namespace pkv
