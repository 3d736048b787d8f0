// kv_append.cuh -- scatter this step's new K/V rows into pool pages through
// the slot mapping (tiny-llm source reading, "Paged KV Cache": pages are
// handed out on demand and new rows are written into them).
#pragma once

#include "ptx.cuh"

namespace pkv {

// One thread moves one 16-byte chunk of one (token, KV head) row of both
// pools.  Source rows are [T][Hkv][D] and contiguous, so consecutive threads
// read consecutive 16-byte chunks; each destination row is D*2 contiguous
// bytes of the pool.  A pure bit copy.
template <int D>
__global__ void __launch_bounds__(256) kv_append_kernel(const uint4* __restrict__ k_new,
                                                        const uint4* __restrict__ v_new,
                                                        const int32_t* __restrict__ slots,
                                                        int32_t T, uint4* __restrict__ k_pool,
                                                        uint4* __restrict__ v_pool,
                                                        int32_t num_kv_heads, int32_t page_size,
                                                        int64_t num_slots) {
  constexpr int kChunks = D / 8;  // 16-byte chunks per row
  // the attention kernel that usually follows may be scheduled now; it waits
  // for this grid to complete before reading the pool
  pdl_launch_dependents();
  const int64_t total = static_cast<int64_t>(T) * num_kv_heads * kChunks;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(idx % kChunks);
    const int64_t row = idx / kChunks;
    const int h = static_cast<int>(row % num_kv_heads);
    const int64_t t = row / num_kv_heads;
    const int32_t slot = __ldg(slots + t);
    if (slot == -1) continue;  // padding row
    if (slot < 0 || slot >= num_slots) {  // not a slot of this pool: skipped, flagged
      if (c == 0 && h == 0) raise_flag(PKV_FLAG_BAD_SLOT);
      continue;
    }
    const int64_t page = slot / page_size;
    const int64_t off = slot - page * page_size;
    const int64_t dst = ((page * num_kv_heads + h) * page_size + off) * kChunks + c;
    const uint4 kv = __ldg(k_new + idx);
    const uint4 vv = __ldg(v_new + idx);
    k_pool[dst] = kv;
    v_pool[dst] = vv;
  }
}

}  // namespace pkv
