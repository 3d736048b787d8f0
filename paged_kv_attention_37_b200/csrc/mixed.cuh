// mixed.cuh -- one persistent launch for a continuous batch that mixes
// prefill chunks and decode requests: CTAs pull work units from one queue,
// the chunks' query tiles first (heaviest request first), then decode
// slices, so CTAs that finish their chunk work early stream decode KV while
// the last chunk tiles are still running.
//
// Sources: tiny-llm source reading, "Continuous Batching" (prefill and
// decode requests handled in the same round) and "Chunked Prefill" (bounded
// chunks interleaved with decode work).
//
// Geometry: two CTAs per SM (the chunk kernel's shape: 6 warps, about half an
// SM's shared memory, 256 TMEM columns); a decode unit is kDecodeWarps warp
// slices of the automatic split, since that many decode warps fit the same
// shared memory (the sixth warp only takes part in the unit's barrier).
// The queue counter and the count of CTAs done live in the decode
// workspace; the last CTA out sets both back to zero.  Nothing waits on
// another CTA.
#pragma once

#include "decode.cuh"
#include "prefill.cuh"

namespace pkv {
namespace mixed {

constexpr int kDecodeWarps = 5;

struct Params {
  prefill::Params pre;
  decode::Params dec;
  int32_t pre_units;  // chunk work units (the standalone chunk launch's CTAs)
  int32_t dec_units;  // decode units of kDecodeWarps slices
  uint32_t* queue;    // [0] next unit, [1] CTAs done
};

template <int D, int G>
__global__ void __launch_bounds__(prefill::kThreads, 2)
    mixed_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                 const __grid_constant__ CUtensorMap vmap, const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ int unit_s;
  // launched as a programmatic dependent: the pools (appended just before)
  // and every input are read after the kernel ahead has completed
  pdl_wait();
  pdl_launch_dependents();
  // the queue hands out every chunk unit before any decode unit: a CTA runs
  // chunk units until it draws a decode unit, then decode units until the
  // queue is empty
  auto pull = [&]() {
    if (threadIdx.x == 0) unit_s = static_cast<int>(atomicAdd(p.queue, 1u));
    __syncthreads();
    const int u = unit_s;
    // shared memory the last unit wrote with ordinary stores may next be
    // written by TMA (the async proxy)
    fence_proxy_async_smem();
    __syncthreads();  // unit_s is rewritten by the next pull
    return u;
  };
  int u = pull();
  for (; u < p.pre_units; u = pull())
    prefill::prefill_body<D, G, prefill::kKeyTile, false>(&qmap, &kmap, &vmap, p.pre, u, smem_raw);
  for (; u < p.pre_units + p.dec_units; u = pull())
    decode::decode_body<D, G, 2, true>(p.dec, u - p.pre_units, p.dec_units, kDecodeWarps, smem_raw);
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(p.queue + 1, 1u) == gridDim.x - 1) {
      p.queue[0] = 0;
      p.queue[1] = 0;
      __threadfence();
    }
  }
}

}  // namespace mixed
}  // namespace pkv
