// decode.cuh -- paged attention for q_len = 1 (paged FlashAttention,
// decode) with split-K over the KV length (flash-decoding), and the
// log-sum-exp combine of split partials.
//
// Sources: tiny-llm source reading, "Paged KV Cache" (attention reads the
// discrete pages named by the page table; paging and the online softmax fused
// in one kernel, no score matrix stored); tiny-vllm article, "From
// Safetensors to PagedAttention" (FlashAttention-style online softmax);
// mini-vllm advanced series design, section 4 Phase B adv04 (split-K over a
// long KV sequence).
//
// Work unit ("item"): one (request r, KV head g, split s); it covers tokens
// [s*part, min((s+1)*part, L_r)) and produces the outputs of all G query
// heads of the group, so every K/V byte is read from HBM once and used G
// times.  Items whose length is a whole partition are handed out first, the
// shorter remainders last (largest-first order), from an atomic counter in
// the workspace (dynamic load balancing over ragged lengths).
//
// Every warp is independent: it takes an item, walks its page-table entries
// (32 per warp-wide load), and keeps NS-1 chunks in flight in its own ring of
// NS shared-memory stages of 8 KB: a chunk is 2048/d tokens (16 at d=128, 32
// at d=64), fetched as TMA tensor boxes of 16 token rows -- K 128-byte
// swizzled, V plain -- each box one page or half of a 32-token page,
// completing on the stage's mbarrier, issued by lane 0 ahead of the chunk
// being computed.  There is no cross-warp synchronisation after the planning
// step, and the small per-warp footprint keeps 10-12 warps resident per SM.
//
// Inside a chunk every lane scores 64 elements of one token: at d=128 lanes
// t and t+16 share token t (one half of d each, one shuffle adds them), at
// d=64 lane t owns token t.  Scores use q as broadcast fp32 pairs from
// shared memory (the halves padded onto different banks), k read from the
// swizzled block without bank conflicts, and packed fp32x2 FMAs.  The online softmax keeps a warp-uniform
// running max and per-lane partial sums.  For P.V lane l owns output columns
// [l*D/32, (l+1)*D/32) of every head.  At the item's end the warp writes
// bf16 output (single-split request) or an fp32 partial and its lse.
#pragma once

#include "ptx.cuh"

namespace pkv {
namespace decode {

constexpr int kBoxRows = 16;     // token rows per copy unit (a page, or half of one)
#ifndef PKV_DECODE_CPASYNC
#define PKV_DECODE_CPASYNC 1
#endif
// Stage fills: 16-byte cp.async copies issued by all 32 lanes (completion
// tracked per thread with commit/wait groups), or TMA issued by lane 0.
constexpr bool kCpAsync = PKV_DECODE_CPASYNC != 0;
template <int D>
struct Chunk {
  static constexpr int kLanesPerToken = D / 64;        // each lane scores 64 elements
  static constexpr int kTokens = 32 / kLanesPerToken;  // tokens per pipeline stage
  static constexpr int kBoxes = kTokens / kBoxRows;    // TMA boxes per stage (per K half)
};
constexpr int kItemSlots = 8;    // per-warp ring of item descriptors
constexpr int kMinAutoPartition = 256;
constexpr int kMaxAutoPartition = 8192;
constexpr int kAutoItemsPerWarp = 3;  // auto split: each warp's share >= 3 partitions

constexpr int kPartitionQuantum = 32;  // split lengths are multiples of this
constexpr float kLazyRescale = 8.0f;  // log2 units: move the running max when it grows > 2^8
constexpr int kFirst = 1;  // first chunk of an item
constexpr int kLast = 2;   // last chunk of an item

struct Params {
  const uint16_t* q;          // bf16 [B][Hq][D]
  const uint16_t* k_pool;     // bf16 [num_pages][Hkv][P][D]
  const uint16_t* v_pool;     // bf16 [num_pages][Hkv][P][D]
  const int32_t* page_table;  // [B][max_pages]
  const int32_t* kv_lens;     // [B]
  uint16_t* out;              // bf16 [B][Hq][D]
  float* out_lse;             // [B][Hq] or null
  float* part_o;              // [B][Hq][S_max][D]
  float* part_lse;            // [B][Hq][S_max]
  int32_t* num_splits;        // [B]
  uint32_t* counters;         // [0] next item, [1] finished warps
  int32_t B, Hq, Hkv, P, max_pages, num_pages, S_max, partition;
  float scale_log2;           // softmax scale * log2(e)
};

struct ChunkInfo {
  int32_t slot, ntok, flags, qslot;
};
struct ItemInfo {
  int32_t r, g, s, nsplit;
};

// Shared memory: one block per warp (the warp count W is chosen at launch
// from the shared-memory budget), then the plan shared by the CTA.
template <int D, int G, int NS>
struct Layout {
  static constexpr int kTok = Chunk<D>::kTokens;
  // K: [kTok rows][D/64 parts][128 B], 128-byte swizzled per 128-byte line
  static constexpr int kKBytes = kTok * D * 2;
  static constexpr int kVBytes = kTok * D * 2;  // [kTok rows][D] bf16
  static constexpr int kStageBytes = kKBytes + kVBytes;
  // scaled query pairs, fp32 [D/64 parts][32 pairs][G][2]; each part starts
  // 16 bytes past a 128-byte multiple so the half-warps' broadcast reads land
  // on different banks
  static constexpr int kQHalfBytes = 32 * G * 8 + 16;
  static constexpr int kQInOff = NS * kStageBytes;              // bf16 [NS][G][D] staged queries
  static constexpr int kQfOff = kQInOff + NS * G * D * 2;
  static constexpr int kPbOff = kQfOff + (D / 64) * kQHalfBytes;  // fp32 [kTok][G][2] (p, p) pairs
  static constexpr int kBarOff = kPbOff + kTok * G * 8;         // NS mbarriers
  static constexpr int kFifoOff = kBarOff + NS * 8;             // NS ChunkInfo
  static constexpr int kItemOff = kFifoOff + NS * 16;           // kItemSlots ItemInfo
  static constexpr int kWarpBytes = (kItemOff + kItemSlots * 16 + 1023) / 1024 * 1024;
  // after the W warp blocks: misc[4], lens[B], prefF[B+1], prefR[B+1]
  static size_t plan_bytes(int B) { return 16 + (3 * static_cast<size_t>(B) + 2) * 4; }
  static size_t bytes(int W, int B) { return static_cast<size_t>(W) * kWarpBytes + plan_bytes(B) + 1024; }
};

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// largest r in [0, n) with pref[r] <= x (pref non-decreasing, pref[n] > x)
__device__ __forceinline__ int upper_index(const int32_t* pref, int n, int x) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pref[mid] <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

template <int D, int G, int NS, int MAXW>
__global__ void __launch_bounds__(MAXW * 32, 1) partition_kernel(const __grid_constant__ CUtensorMap kmap,
                                                                 const __grid_constant__ CUtensorMap vmap,
                                                                 const Params p) {
  using LY = Layout<D, G, NS>;
  constexpr int kTok = Chunk<D>::kTokens, kLPT = Chunk<D>::kLanesPerToken;
  const int W = blockDim.x >> 5;
  const int log2P = 31 - __clz(p.P);  // P is a power of two
  constexpr int DPL = D / 32;  // P.V output columns per lane
  static_assert(DPL == 2 || DPL == 4, "head_dim 64 or 128");
  static_assert(NS >= 2, "at least two stages per warp");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int32_t* misc = reinterpret_cast<int32_t*>(smem + W * LY::kWarpBytes);
  int32_t* lens = misc + 4;
  int32_t* prefF = lens + p.B;
  int32_t* prefR = prefF + p.B + 1;

  uint8_t* wb = smem + warp * LY::kWarpBytes;
  const uint32_t wbase = smem_addr(wb);
  auto full_bar = [&](int i) { return wbase + LY::kBarOff + 8u * i; };
  ChunkInfo* fifo = reinterpret_cast<ChunkInfo*>(wb + LY::kFifoOff);
  ItemInfo* items = reinterpret_cast<ItemInfo*>(wb + LY::kItemOff);
  float* qf = reinterpret_cast<float*>(wb + LY::kQfOff);
  float* pb = reinterpret_cast<float*>(wb + LY::kPbOff);

  if (lane == 0) {
    for (int i = 0; i < NS; ++i) mbar_init(full_bar(i), 1);
    fence_barrier_init();
  }
  if (threadIdx.x == 0) {
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&vmap);
  }

  // ---- plan (warp 0): clamp lengths, pick the partition, count the items:
  // whole-partition items first (prefF), then one remainder item per
  // (request, KV head) whose length is not a multiple of the partition
  // (prefR; an empty request also gets one, to write its zero output).
  if (warp == 0) {
    const int maxL = p.max_pages * p.P;
    long long tot = 0;
    bool bad = false;
    for (int r = lane; r < p.B; r += 32) {
      int L = p.kv_lens[r];
      if (L < 0 || L > maxL) {
        bad = true;
        L = L < 0 ? 0 : maxL;
      }
      lens[r] = L;
      tot += L;
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0 && blockIdx.x == 0) raise_flag(PKV_FLAG_BAD_LENGTH);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
    int part;
    if (p.partition > 0) {
      part = p.partition;
    } else if (p.partition < 0) {
      part = ((maxL > 0 ? maxL : 1) + kPartitionQuantum - 1) / kPartitionQuantum * kPartitionQuantum;
    } else {
      const long long warps = static_cast<long long>(gridDim.x) * W;
      const long long share = tot * p.Hkv / (warps * kAutoItemsPerWarp);
      part = kMaxAutoPartition;
      while (part > kMinAutoPartition && part > share) part >>= 1;
    }
    __syncwarp();
    int runF = 0, runR = 0;
    for (int base = 0; base < p.B; base += 32) {
      const int r = base + lane;
      int nf = 0, nr = 0;
      if (r < p.B) {
        const int L = lens[r];
        nf = (L / part) * p.Hkv;
        nr = (L % part != 0 || L == 0) ? p.Hkv : 0;
        if (blockIdx.x == 0) p.num_splits[r] = L == 0 ? 1 : (L + part - 1) / part;
      }
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int yf = __shfl_up_sync(0xffffffffu, nf, o);
        const int yr = __shfl_up_sync(0xffffffffu, nr, o);
        if (lane >= o) {
          nf += yf;
          nr += yr;
        }
      }
      if (r < p.B) {
        prefF[r + 1] = runF + nf;
        prefR[r + 1] = runR + nr;
      }
      runF += __shfl_sync(0xffffffffu, nf, 31);
      runR += __shfl_sync(0xffffffffu, nr, 31);
    }
    if (lane == 0) {
      prefF[0] = 0;
      prefR[0] = 0;
      misc[0] = part;
      misc[1] = runF;
      misc[2] = runR;
    }
  }
  __syncthreads();
  const int part = misc[0], nF = misc[1], total = misc[1] + misc[2];

  // ================= issue side: item cursor, lane 0 issues TMA =================
  bool more = true, active = false;
  int it_r = 0, it_g = 0, it_t0 = 0, it_ntok = 0, it_nch = 0, it_k = 0, it_slot = 0, it_qslot = 0;
  int fetched = 0, pid_base = 0, pid_cur = -1, pid_next = -1, it_npg = 0;
  const int32_t* ptab = p.page_table;

  auto fetch = [&]() {
    int idx = 0;
    if (lane == 0) idx = static_cast<int>(atomicAdd(p.counters, 1u));
    idx = __shfl_sync(0xffffffffu, idx, 0);
    if (idx >= total) {
      more = false;
      return;
    }
    int r, g, s, t0, ntok;
    if (idx < nF) {
      r = upper_index(prefF, p.B, idx);
      const int local = idx - prefF[r];
      s = local / p.Hkv;
      g = local - s * p.Hkv;
      t0 = s * part;
      ntok = part;
    } else {
      const int j = idx - nF;
      r = upper_index(prefR, p.B, j);
      g = j - prefR[r];
      s = lens[r] / part;
      t0 = s * part;
      ntok = lens[r] - t0;
    }
    const int L = lens[r];
    it_r = r;
    it_g = g;
    it_t0 = t0;
    it_ntok = ntok;
    it_nch = (ntok + kTok - 1) / kTok;
    it_k = 0;
    it_slot = fetched % kItemSlots;
    it_qslot = fetched % NS;
    ++fetched;
    if (lane == 0) items[it_slot] = ItemInfo{r, g, s, L == 0 ? 1 : (L + part - 1) / part};
    it_npg = (ntok + p.P - 1) >> log2P;
    ptab = p.page_table + static_cast<size_t>(r) * p.max_pages + (t0 >> log2P);
    pid_base = 0;
    pid_cur = lane < it_npg ? __ldg(ptab + lane) : -1;
    pid_next = 32 + lane < it_npg ? __ldg(ptab + 32 + lane) : -1;
    active = true;
  };

  // Issue the next chunk of the current (or next) item into stage n % NS.
  auto issue = [&](int n) -> bool {
    if (!active) {
      if (!more) return false;
      fetch();
      if (!active) return false;
    }
    const int stage = n % NS;
    const int tok0 = it_k * kTok;  // relative to the item's first token (a page start)
    const int ntok = it_nch == 0 ? 0 : min(kTok, it_ntok - tok0);
    const int flags = (it_k == 0 ? kFirst : 0) | (it_k + 1 >= it_nch ? kLast : 0);
    const int nbox = (ntok + kBoxRows - 1) / kBoxRows;
    // each 16-row box lies inside one page: page-table entry (tok >> log2P),
    // first row (tok & (P-1))
    int pages[Chunk<D>::kBoxes];
#pragma unroll
    for (int b = 0; b < Chunk<D>::kBoxes; ++b) {
      pages[b] = -1;
      if (b < nbox) {
        const int pi = (tok0 + b * kBoxRows) >> log2P;
        while (pi >= pid_base + 32) {
          pid_base += 32;
          pid_cur = pid_next;
          pid_next = pid_base + 32 + lane < it_npg ? __ldg(ptab + pid_base + 32 + lane) : -1;
        }
        pages[b] = __shfl_sync(0xffffffffu, pid_cur, pi & 31);
      }
    }
    if constexpr (kCpAsync) {
      // all lanes copy 16-byte pieces; K goes to its swizzled position
      if (lane == 0) fifo[stage] = ChunkInfo{it_slot, ntok, flags, it_qslot};
      if (ntok > 0) {
        const uint32_t st = wbase + stage * LY::kStageBytes;
#pragma unroll
        for (int b = 0; b < Chunk<D>::kBoxes; ++b) {
          if (b >= nbox) break;
          int page = pages[b];
          if (static_cast<unsigned>(page) >= static_cast<unsigned>(p.num_pages)) {
            if (lane == 0) raise_flag(PKV_FLAG_BAD_PAGE);  // read page 0: wrong values, no stray access
            page = 0;
          }
          const size_t row0 = (static_cast<size_t>(page) * p.Hkv + it_g) * p.P + ((tok0 + b * kBoxRows) & (p.P - 1));
          const uint8_t* ksrc = reinterpret_cast<const uint8_t*>(p.k_pool + row0 * D);
          const uint8_t* vsrc = reinterpret_cast<const uint8_t*>(p.v_pool + row0 * D);
          constexpr int kPieces = kBoxRows * D / 8;  // 16-byte pieces per 16-row box
#pragma unroll
          for (int i = lane; i < kPieces; i += 32) {
            const int t = i / (D / 8), c16 = i % (D / 8);
            const int line = (b * kBoxRows + t) * (D / 64) + (c16 >> 3);
            cp_async16(st + line * 128 + (((c16 & 7) ^ (line & 7)) << 4), ksrc + i * 16);
            cp_async16(st + LY::kKBytes + ((b * kBoxRows + t) * D + c16 * 8) * 2, vsrc + i * 16);
          }
        }
        if (it_k == 0) {
          const uint8_t* qsrc = reinterpret_cast<const uint8_t*>(
              p.q + (static_cast<size_t>(it_r) * p.Hq + static_cast<size_t>(it_g) * G) * D);
          const uint32_t qdst = wbase + LY::kQInOff + it_qslot * (G * D * 2);
#pragma unroll
          for (int i = lane; i < G * D * 2 / 16; i += 32) cp_async16(qdst + i * 16, qsrc + i * 16);
        }
      }
    } else if (lane == 0) {
      fifo[stage] = ChunkInfo{it_slot, ntok, flags, it_qslot};
      if (ntok > 0) {
        const bool with_q = it_k == 0;
        const uint32_t bytes = static_cast<uint32_t>(nbox * kBoxRows * D * 2 * 2) +
                               (with_q ? static_cast<uint32_t>(G * D * 2) : 0u);
        const uint32_t st = wbase + stage * LY::kStageBytes;
        mbar_arrive_expect_tx(full_bar(stage), bytes);
#pragma unroll
        for (int b = 0; b < Chunk<D>::kBoxes; ++b) {
          if (b >= nbox) break;
          int page = pages[b];
          if (static_cast<unsigned>(page) >= static_cast<unsigned>(p.num_pages)) {
            raise_flag(PKV_FLAG_BAD_PAGE);  // read page 0 instead: wrong values, no stray access
            page = 0;
          }
          const int row = page * p.Hkv + it_g;
          const int r0 = (tok0 + b * kBoxRows) & (p.P - 1);
          // K: one tensor box = 16 token rows x all D/64 parts, swizzled;
          // V: the same 16 rows are one contiguous run of the pool
          tma_load_4d(st + b * (kBoxRows * D * 2), &kmap, 0, 0, r0, row, full_bar(stage));
          bulk_load(st + LY::kKBytes + b * (kBoxRows * D * 2),
                    p.v_pool + (static_cast<size_t>(row) * p.P + r0) * D, kBoxRows * D * 2,
                    full_bar(stage));
        }
        if (with_q)
          bulk_load(wbase + LY::kQInOff + it_qslot * (G * D * 2),
                    p.q + (static_cast<size_t>(it_r) * p.Hq + static_cast<size_t>(it_g) * G) * D,
                    G * D * 2, full_bar(stage));
      } else {
        mbar_arrive(full_bar(stage));
      }
    }
    __syncwarp();
    if (++it_k >= max(1, it_nch)) active = false;
    return true;
  };

  // ================================ compute side ================================
  // token of this lane, and which 64-element part of d it scores
  const int tl = kLPT == 2 ? (lane & 15) : lane, hh = kLPT == 2 ? (lane >> 4) : 0;
  float2 o2[G][DPL / 2];
  float m[G], l[G];
  // Every issue attempt commits one cp.async group (possibly empty), so the
  // group of chunk n is complete once at most NS-2 newer groups are pending.
  int issued = 0;
  for (int i = 0; i < NS - 1; ++i) {
    const bool ok = issued == i && issue(issued);
    if constexpr (kCpAsync) cp_async_commit();
    if (ok) ++issued;
  }
  int n = 0;
  for (; n < issued; ++n) {
    const int stage = n % NS;
    if constexpr (kCpAsync) {
      cp_async_wait<NS - 2>();
      __syncwarp();
    } else {
      if (!mbar_wait(full_bar(stage), (n / NS) & 1)) break;
    }
    const ChunkInfo ci = fifo[stage];
    const int ntok = ci.ntok;
    if (ci.flags & kFirst) {
#pragma unroll
      for (int g = 0; g < G; ++g) {
        m[g] = -INFINITY;
        l[g] = 0.f;
#pragma unroll
        for (int e = 0; e < DPL / 2; ++e) o2[g][e] = make_float2(0.f, 0.f);
      }
      if (ntok > 0) {
        // staged bf16 query rows [G][D] -> fp32 pairs [part][32][G][2],
        // times scale*log2(e)
        const uint32_t* qin = reinterpret_cast<const uint32_t*>(wb + LY::kQInOff + ci.qslot * (G * D * 2));
        for (int i = lane; i < G * D / 2; i += 32) {
          const int g = i / (D / 2), pp = i - g * (D / 2);
          const int half = pp >> 5, ppl = pp & 31;
          const uint32_t x = qin[i];
          *reinterpret_cast<float2*>(reinterpret_cast<uint8_t*>(qf) + half * LY::kQHalfBytes + (ppl * G + g) * 8) =
              make_float2(bf16lo(x) * p.scale_log2, bf16hi(x) * p.scale_log2);
        }
      }
    }
    // keep NS-1 chunks in flight: refill the stage chunk n-1 used
    __syncwarp();
    if constexpr (!kCpAsync) fence_proxy_async_smem();
    {
      const bool ok = issue(issued);
      if constexpr (kCpAsync) cp_async_commit();
      if (ok) ++issued;
    }

    if (ntok > 0) {
      const uint8_t* stp = wb + stage * LY::kStageBytes;
      // ---- scores: each lane takes 64 elements (one 128-byte K row) of its token
      float2 acc[G];
#pragma unroll
      for (int g = 0; g < G; ++g) acc[g] = make_float2(0.f, 0.f);
      // this lane's 128-byte line of K: token tl, part hh; its swizzle phase
      // is the line index mod 8
      const int kline = tl * (D / 64) + hh;
      const uint8_t* krow = stp + kline * 128;
      const uint32_t swz = static_cast<uint32_t>(kline & 7) << 4;
      const uint8_t* qh = reinterpret_cast<const uint8_t*>(qf) + hh * LY::kQHalfBytes;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 kk = *reinterpret_cast<const uint4*>(krow + ((c << 4) ^ swz));
        const uint32_t kw[4] = {kk.x, kk.y, kk.z, kk.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 k2 = make_float2(bf16lo(kw[j]), bf16hi(kw[j]));
          const int ppl = c * 4 + j;
          if constexpr (G == 1) {
            const float2 q2 = *reinterpret_cast<const float2*>(qh + ppl * 8);
            acc[0] = __ffma2_rn(q2, k2, acc[0]);
          } else {
#pragma unroll
            for (int g = 0; g < G; g += 2) {
              const float4 q4 = *reinterpret_cast<const float4*>(qh + (ppl * G + g) * 8);
              acc[g] = __ffma2_rn(make_float2(q4.x, q4.y), k2, acc[g]);
              acc[g + 1] = __ffma2_rn(make_float2(q4.z, q4.w), k2, acc[g + 1]);
            }
          }
        }
      }
      // ---- online softmax, log2 domain; hidden tokens get -inf -> weight 0.
      // The running max m is only moved (and o, l rescaled) when some score
      // exceeds it by more than 2^8 -- in practice on an item's first chunk.
      // Between moves the exponentials are taken against the stale max, so
      // p <= 2^8; the final normalisation by l uses the same m, so the
      // result is the same softmax.
      float sv[G];
      bool grow = false;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float x = acc[g].x + acc[g].y;
        if constexpr (kLPT == 2) x += __shfl_xor_sync(0xffffffffu, x, 16);
        sv[g] = tl < ntok ? x : -INFINITY;
        grow |= sv[g] > m[g] + kLazyRescale;
      }
      if (__any_sync(0xffffffffu, grow)) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
          float mx = sv[g];
#pragma unroll
          for (int o = kTok / 2; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
          const float mn = fmaxf(m[g], mx);
          const float alpha = fast_exp2(m[g] - mn);
          l[g] *= alpha;
          const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
          for (int e = 0; e < DPL / 2; ++e) o2[g][e] = __fmul2_rn(o2[g][e], a2);
          m[g] = mn;
        }
      }
      float pvs[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        pvs[g] = fast_exp2(sv[g] - m[g]);
        if (hh == 0) l[g] += pvs[g];
      }
      if (hh == 0) {
        if constexpr (G == 1) {
          *reinterpret_cast<float2*>(pb + tl * 2) = make_float2(pvs[0], pvs[0]);
        } else {
#pragma unroll
          for (int g = 0; g < G; g += 2)
            *reinterpret_cast<float4*>(pb + (tl * G + g) * 2) = make_float4(pvs[g], pvs[g], pvs[g + 1], pvs[g + 1]);
        }
      }
      __syncwarp();
      // ---- P.V: lane owns DPL output columns of every head
      const uint8_t* vb = stp + LY::kKBytes + lane * DPL * 2;
      auto pv_token = [&](int t) {
        float2 pg[G];
        if constexpr (G == 1) {
          pg[0] = *reinterpret_cast<const float2*>(pb + t * 2);
        } else {
#pragma unroll
          for (int g = 0; g < G; g += 2) {
            const float4 x = *reinterpret_cast<const float4*>(pb + (t * G + g) * 2);
            pg[g] = make_float2(x.x, x.y);
            pg[g + 1] = make_float2(x.z, x.w);
          }
        }
        if constexpr (DPL == 4) {
          const uint2 x = *reinterpret_cast<const uint2*>(vb + t * D * 2);
          const float2 v01 = make_float2(bf16lo(x.x), bf16hi(x.x));
          const float2 v23 = make_float2(bf16lo(x.y), bf16hi(x.y));
#pragma unroll
          for (int g = 0; g < G; ++g) {
            o2[g][0] = __ffma2_rn(pg[g], v01, o2[g][0]);
            o2[g][1] = __ffma2_rn(pg[g], v23, o2[g][1]);
          }
        } else {
          const uint32_t x = *reinterpret_cast<const uint32_t*>(vb + t * D * 2);
          const float2 v01 = make_float2(bf16lo(x), bf16hi(x));
#pragma unroll
          for (int g = 0; g < G; ++g) o2[g][0] = __ffma2_rn(pg[g], v01, o2[g][0]);
        }
      };
      if (ntok == kTok) {  // full chunk: fully unrolled, constant offsets
#pragma unroll
        for (int t = 0; t < kTok; ++t) pv_token(t);
      } else {
#pragma unroll 1
        for (int t = 0; t < ntok; ++t) pv_token(t);
      }
    }

    if (ci.flags & kLast) {
      // ---- item done: normalise and write bf16 output or an fp32 partial
      const ItemInfo it = items[ci.slot];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float ls = warp_sum(l[g]);
        const float inv = ls > 0.f ? 1.f / ls : 0.f;
        const float lse = ls > 0.f ? (m[g] + __log2f(ls)) * 0.69314718055994531f : -INFINITY;
        const size_t row = static_cast<size_t>(it.r) * p.Hq + it.g * G + g;
        if (it.nsplit == 1) {
          uint16_t* dst = p.out + row * D + lane * DPL;
          if constexpr (DPL == 4) {
            *reinterpret_cast<uint2*>(dst) =
                make_uint2(pack_bf16x2(o2[g][0].x * inv, o2[g][0].y * inv),
                           pack_bf16x2(o2[g][1].x * inv, o2[g][1].y * inv));
          } else {
            *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(o2[g][0].x * inv, o2[g][0].y * inv);
          }
          if (p.out_lse != nullptr && lane == 0) p.out_lse[row] = lse;
        } else {
          const size_t prow = row * p.S_max + it.s;
          float* dst = p.part_o + prow * D + lane * DPL;
          if constexpr (DPL == 4) {
            *reinterpret_cast<float4*>(dst) = make_float4(o2[g][0].x * inv, o2[g][0].y * inv,
                                                          o2[g][1].x * inv, o2[g][1].y * inv);
          } else {
            *reinterpret_cast<float2*>(dst) = make_float2(o2[g][0].x * inv, o2[g][0].y * inv);
          }
          if (lane == 0) p.part_lse[prow] = lse;
        }
      }
    }
  }
  if (n < issued) {
    // a wait gave up: give copies still in flight a bounded chance to land
    for (int k = n + 1; k < issued; ++k) mbar_wait(full_bar(k % NS), (k / NS) & 1);
  }
  if (lane == 0) {
    __threadfence();
    if (atomicAdd(&p.counters[1], 1u) == gridDim.x * W - 1) {
      p.counters[0] = 0;
      p.counters[1] = 0;
      __threadfence();
    }
  }
}

// Merge split partials.  One CTA per (request, query head) row; its warps
// stride over the splits (four splits' loads in flight per warp), each lane
// owning D/32 columns, and the per-warp sums meet in shared memory.
// skip_single: requests with one split were written by the partition kernel.
constexpr int kCombineMaxWarps = 8;

template <int D>
__global__ void __launch_bounds__(32 * kCombineMaxWarps) combine_kernel(
    const float* __restrict__ part_o, const float* __restrict__ part_lse,
    const int32_t* __restrict__ num_splits, int32_t B, int32_t Hq, int32_t S_max,
    uint16_t* __restrict__ out, float* __restrict__ out_lse, int skip_single) {
  constexpr int DPL = D / 32;
  constexpr float kLog2e = 1.4426950408889634f;
  __shared__ float red_m[kCombineMaxWarps], red_den[kCombineMaxWarps];
  __shared__ __align__(16) float red_acc[kCombineMaxWarps][D];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const long long row = blockIdx.x;
  const int r = static_cast<int>(row / Hq);
  int n = num_splits[r];
  if (skip_single && n <= 1) return;
  n = max(0, min(n, S_max));
  const float* ls = part_lse + row * S_max;
  float M = -INFINITY;
  for (int s = threadIdx.x; s < n; s += blockDim.x) M = fmaxf(M, ls[s]);
  M = warp_max(M);
  if (lane == 0) red_m[warp] = M;
  __syncthreads();
  M = red_m[0];
  for (int w = 1; w < nw; ++w) M = fmaxf(M, red_m[w]);
  float acc[DPL], den = 0.f;
#pragma unroll
  for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
  if (M != -INFINITY) {
    const float* po = part_o + row * S_max * D + lane * DPL;
    auto load = [&](int s, float (&v)[DPL]) {
      if constexpr (DPL == 4) {
        const float4 x = *reinterpret_cast<const float4*>(po + static_cast<size_t>(s) * D);
        v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
      } else {
        const float2 x = *reinterpret_cast<const float2*>(po + static_cast<size_t>(s) * D);
        v[0] = x.x; v[1] = x.y;
      }
    };
    int s = warp;
    for (; s + 3 * nw < n; s += 4 * nw) {
      float v[4][DPL], lv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        lv[u] = ls[s + u * nw];
        load(s + u * nw, v[u]);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float w = fast_exp2((lv[u] - M) * kLog2e);
        den += w;
#pragma unroll
        for (int e = 0; e < DPL; ++e) acc[e] = fmaf(w, v[u][e], acc[e]);
      }
    }
    for (; s < n; s += nw) {
      float v[DPL];
      load(s, v);
      const float w = fast_exp2((ls[s] - M) * kLog2e);
      den += w;
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[e] = fmaf(w, v[e], acc[e]);
    }
  }
#pragma unroll
  for (int e = 0; e < DPL; ++e) red_acc[warp][lane * DPL + e] = acc[e];
  if (lane == 0) red_den[warp] = den;
  __syncthreads();
  if (warp != 0) return;
  for (int w = 1; w < nw; ++w) {
    den += red_den[w];
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[e] += red_acc[w][lane * DPL + e];
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  uint16_t* dst = out + row * D + lane * DPL;
  if constexpr (DPL == 4) {
    *reinterpret_cast<uint2*>(dst) =
        make_uint2(pack_bf16x2(acc[0] * inv, acc[1] * inv), pack_bf16x2(acc[2] * inv, acc[3] * inv));
  } else {
    *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  }
  if (out_lse != nullptr && lane == 0) out_lse[row] = den > 0.f ? M + logf(den) : -INFINITY;
}

}  // namespace decode
}  // namespace pkv
