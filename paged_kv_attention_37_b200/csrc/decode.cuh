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
// Work unit ("item"): one (request r, KV head g, split s) triple; it covers
// tokens [s*part, min((s+1)*part, L_r)) and produces the outputs of all G
// query heads of the group, so every K/V byte is read from HBM once and used
// G times.  A persistent grid takes items from an atomic counter in the
// workspace (dynamic load balancing over ragged lengths).
//
// CTA layout: warp 0 is the producer, warps 1..4 are consumers.
//   producer: walks the item's page-table entries (32 at a time, loaded by
//     the whole warp), and for each 32-token chunk issues TMA tensor loads of
//     the K block (128-byte swizzle) and V block of every page in the chunk
//     into one ring stage, completing on that stage's mbarrier;
//   consumers: chunk k of an item goes to consumer k % 4; a consumer keeps
//     its own online-softmax state (running max m, per-lane partial sum l,
//     output accumulator o) for the G heads; at the item's end the four
//     states are merged through shared memory and written out: bf16 output
//     when the request has one split, else an fp32 partial plus its lse.
// Inside a chunk, lane t owns token t for the scores (q . k_t for G heads,
// q read as broadcast fp32 from shared memory, k_t read from the swizzled
// block without bank conflicts), and lane l owns output columns
// [l*D/32, (l+1)*D/32) for P.V.
#pragma once

#include "ptx.cuh"

namespace pkv {
namespace decode {

constexpr int kChunk = 32;       // tokens per pipeline stage
constexpr int kConsumers = 4;    // consumer warps per CTA
constexpr int kThreads = 32 * (kConsumers + 1);
constexpr int kItemSlots = 8;    // ring of in-flight item descriptors
constexpr int kMinAutoPartition = 256;
constexpr int kMaxAutoPartition = 8192;
constexpr int kAutoItemsPerCta = 4;  // auto split: a CTA's share of work >= 4 partitions

constexpr int kFlagLast = 1;  // this consumer's last stage of the item
constexpr int kFlagDone = 2;  // no more items
constexpr int kFlagQ = 4;     // stage also carries the item's G query rows

struct Params {
  const uint16_t* q;          // bf16 [B][Hq][D]
  const int32_t* page_table;  // [B][max_pages]
  const int32_t* kv_lens;     // [B]
  uint16_t* out;              // bf16 [B][Hq][D]
  float* out_lse;             // [B][Hq] or null
  float* part_o;              // [B][Hq][S_max][D]
  float* part_lse;            // [B][Hq][S_max]
  int32_t* num_splits;        // [B]
  uint32_t* counters;         // [0] next item, [1] finished CTAs
  int32_t B, Hq, Hkv, P, max_pages, num_pages, S_max, partition;
  float scale_log2;           // softmax scale * log2(e)
};

struct StageInfo {
  int32_t slot, ntok, flags, pad;
};
struct ItemInfo {
  int32_t r, g, s, nsplit;
};

template <int D, int G, int STAGES>
struct Layout {
  static constexpr int kKBytes = kChunk * D * 2;  // [D/64][32 rows][128 B], swizzled
  static constexpr int kVBytes = kChunk * D * 2;  // [32 rows][D] bf16
  static constexpr int kQBytes = G * D * 2;       // [G][D] bf16
  static constexpr int kStageBytes = (kKBytes + kVBytes + kQBytes + 1023) / 1024 * 1024;
  static constexpr int kQfOff = STAGES * kStageBytes;                 // fp32 [NC][G][D]
  static constexpr int kPbufOff = kQfOff + kConsumers * G * D * 4;    // fp32 [NC][32][G]
  static constexpr int kMergeEntry = G * D + ((2 * G + 3) / 4) * 4;  // floats: o[G][D], m[G], l[G]
  static constexpr int kMergeOff = kPbufOff + kConsumers * kChunk * G * 4;
  static constexpr int kBarOff = kMergeOff + 2 * kConsumers * kMergeEntry * 4;
  static constexpr int kInfoOff = kBarOff + (2 * STAGES + 2) * 8;
  static constexpr int kItemOff = kInfoOff + STAGES * 16;
  static constexpr int kMiscOff = kItemOff + kItemSlots * 16;
  static constexpr int kLensOff = kMiscOff + 16;  // int32 lens[B], prefix[B+1]
  static size_t bytes(int B) { return kLensOff + static_cast<size_t>(2 * B + 1) * 4 + 1024; }
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

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

template <int D, int G, int STAGES>
__global__ void __launch_bounds__(kThreads, 2) partition_kernel(const __grid_constant__ CUtensorMap kmap,
                                                             const __grid_constant__ CUtensorMap vmap,
                                                             const Params p) {
  using LY = Layout<D, G, STAGES>;
  constexpr int DPL = D / 32;  // output columns per lane
  static_assert(DPL == 2 || DPL == 4, "head_dim 64 or 128");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_addr(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  auto full_bar = [&](int i) { return sbase + LY::kBarOff + 8u * i; };
  auto empty_bar = [&](int i) { return sbase + LY::kBarOff + 8u * (STAGES + i); };
  auto merge_bar = [&](int b) { return sbase + LY::kBarOff + 8u * (2 * STAGES + b); };
  StageInfo* info = reinterpret_cast<StageInfo*>(smem + LY::kInfoOff);
  ItemInfo* items = reinterpret_cast<ItemInfo*>(smem + LY::kItemOff);
  int32_t* misc = reinterpret_cast<int32_t*>(smem + LY::kMiscOff);
  int32_t* lens = reinterpret_cast<int32_t*>(smem + LY::kLensOff);
  int32_t* prefix = lens + p.B;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(full_bar(i), 1);
      mbar_init(empty_bar(i), 1);
    }
    mbar_init(merge_bar(0), kConsumers);
    mbar_init(merge_bar(1), kConsumers);
    fence_barrier_init();
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&vmap);
  }

  // ---- plan: clamp lengths, pick the partition, prefix-count the items
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
      part = ((maxL > 0 ? maxL : 1) + kChunk - 1) / kChunk * kChunk;
    } else {
      const long long share = tot * p.Hkv / (static_cast<long long>(gridDim.x) * kAutoItemsPerCta);
      part = kMaxAutoPartition;
      while (part > kMinAutoPartition && part > share) part >>= 1;
    }
    __syncwarp();
    int running = 0;
    for (int base = 0; base < p.B; base += 32) {
      const int r = base + lane;
      int ns = 0;
      if (r < p.B) {
        const int L = lens[r];
        ns = L == 0 ? 1 : (L + part - 1) / part;
        if (blockIdx.x == 0) p.num_splits[r] = ns;
      }
      int v = ns * p.Hkv;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += y;
      }
      if (r < p.B) prefix[r + 1] = running + v;
      running += __shfl_sync(0xffffffffu, v, 31);
    }
    if (lane == 0) {
      prefix[0] = 0;
      misc[0] = part;
      misc[1] = running;
    }
  }
  __syncthreads();

  if (warp == 0) {
    // =========================== producer ===========================
    const int part = misc[0], total_items = misc[1];
    int seq = 0, item_count = 0;
    bool ok = true;
    while (ok) {
      int item = 0;
      if (lane == 0) item = static_cast<int>(atomicAdd(&p.counters[0], 1u));
      item = __shfl_sync(0xffffffffu, item, 0);
      if (item >= total_items) break;
      int lo = 0, hi = p.B - 1;  // request r with prefix[r] <= item < prefix[r+1]
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (prefix[mid] <= item) lo = mid; else hi = mid - 1;
      }
      const int r = lo;
      const int local = item - prefix[r];
      const int s = local / p.Hkv, g = local - s * p.Hkv;
      const int L = lens[r];
      const int nsplit = L == 0 ? 1 : (L + part - 1) / part;
      const int t0 = s * part, t1 = min(L, t0 + part);
      const int ntok_item = max(0, t1 - t0);
      const int nch = (ntok_item + kChunk - 1) / kChunk;
      const int nst = max(1, (nch + kConsumers - 1) / kConsumers) * kConsumers;
      const int slot = item_count % kItemSlots;
      ++item_count;
      if (lane == 0) items[slot] = ItemInfo{r, g, s, nsplit};

      // page ids of this item, 32 entries per warp-wide load
      const int npg = (ntok_item + p.P - 1) / p.P;
      const int32_t* ptab = p.page_table + static_cast<size_t>(r) * p.max_pages + t0 / p.P;
      int base = 0;
      int pid_cur = lane < npg ? __ldg(ptab + lane) : -1;
      int pid_next = 32 + lane < npg ? __ldg(ptab + 32 + lane) : -1;
      const uint16_t* qsrc = p.q + (static_cast<size_t>(r) * p.Hq + static_cast<size_t>(g) * G) * D;

      for (int k = 0; k < nst; ++k) {
        const int stage = seq % STAGES;
        if (seq >= STAGES && !mbar_wait(empty_bar(stage), ((seq / STAGES) - 1) & 1)) {
          ok = false;
          break;
        }
        int flags = (k >= nst - kConsumers) ? kFlagLast : 0;
        const uint32_t st = sbase + stage * LY::kStageBytes;
        if (k < nch) {
          const int tok0 = k * kChunk;  // relative to t0
          const int ntok = min(kChunk, ntok_item - tok0);
          const bool with_q = k < kConsumers;
          if (with_q) flags |= kFlagQ;
          const int npc = (ntok + p.P - 1) / p.P;  // pages touched by this chunk
          int pids[kChunk / 16];
#pragma unroll
          for (int j = 0; j < kChunk / 16; ++j) {
            pids[j] = -1;
            if (j < npc) {
              const int pi = tok0 / p.P + j;
              while (pi >= base + 32) {
                base += 32;
                pid_cur = pid_next;
                pid_next = base + 32 + lane < npg ? __ldg(ptab + base + 32 + lane) : -1;
              }
              pids[j] = __shfl_sync(0xffffffffu, pid_cur, pi & 31);
            }
          }
          if (lane == 0) {
            info[stage] = StageInfo{slot, ntok, flags, 0};
            const uint32_t bytes = static_cast<uint32_t>(npc * p.P * D * 2 * 2) +
                                   (with_q ? static_cast<uint32_t>(LY::kQBytes) : 0u);
            mbar_arrive_expect_tx(full_bar(stage), bytes);
#pragma unroll
            for (int j = 0; j < kChunk / 16; ++j) {
              if (j >= npc) break;
              const int page = pids[j];
              if (static_cast<unsigned>(page) >= static_cast<unsigned>(p.num_pages))
                raise_flag(PKV_FLAG_BAD_PAGE);  // TMA reads zeros out of bounds
              const int row = page * p.Hkv + g;
#pragma unroll
              for (int h = 0; h < D / 64; ++h)
                tma_load_3d(st + h * (kChunk * 128) + j * p.P * 128, &kmap, 64 * h, 0, row,
                            full_bar(stage));
              tma_load_3d(st + LY::kKBytes + j * p.P * D * 2, &vmap, 0, 0, row, full_bar(stage));
            }
            if (with_q) bulk_load(st + LY::kKBytes + LY::kVBytes, qsrc, LY::kQBytes, full_bar(stage));
          }
        } else if (lane == 0) {
          info[stage] = StageInfo{slot, 0, flags, 0};
          mbar_arrive(full_bar(stage));
        }
        __syncwarp();
        ++seq;
      }
    }
    if (ok) {
      for (int c = 0; c < kConsumers; ++c) {
        const int stage = seq % STAGES;
        if (seq >= STAGES && !mbar_wait(empty_bar(stage), ((seq / STAGES) - 1) & 1)) break;
        if (lane == 0) {
          info[stage] = StageInfo{0, 0, kFlagDone, 0};
          mbar_arrive(full_bar(stage));
        }
        __syncwarp();
        ++seq;
      }
    } else {
      // give copies already issued a bounded chance to land before exiting
      for (int i = 0; i < STAGES && i < seq; ++i) {
        const int sq = seq - 1 - i;
        mbar_wait(full_bar(sq % STAGES), (sq / STAGES) & 1);
      }
    }
    if (lane == 0) {
      __threadfence();
      if (atomicAdd(&p.counters[1], 1u) == gridDim.x - 1) {
        p.counters[0] = 0;
        p.counters[1] = 0;
        __threadfence();
      }
    }
    return;
  }

  // ============================= consumers =============================
  const int cw = warp - 1;
  float* qf = reinterpret_cast<float*>(smem + LY::kQfOff) + cw * G * D;
  float* pb = reinterpret_cast<float*>(smem + LY::kPbufOff) + cw * kChunk * G;
  float* merge_base = reinterpret_cast<float*>(smem + LY::kMergeOff);
  const uint32_t swz = static_cast<uint32_t>(lane & 7) << 4;

  float o[G][DPL], m[G], l[G];
  int seq = cw, cur_slot = -1, merged = 0;
  while (true) {
    const int stage = seq % STAGES;
    if (!mbar_wait(full_bar(stage), (seq / STAGES) & 1)) break;
    const StageInfo inf = info[stage];
    if (inf.flags & kFlagDone) break;
    const uint8_t* stp = smem + stage * LY::kStageBytes;
    if (inf.slot != cur_slot) {
      cur_slot = inf.slot;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        m[g] = -INFINITY;
        l[g] = 0.f;
#pragma unroll
        for (int e = 0; e < DPL; ++e) o[g][e] = 0.f;
      }
    }
    if (inf.flags & kFlagQ) {
      // query rows of the group -> fp32, pre-multiplied by scale*log2(e)
      const uint16_t* qb = reinterpret_cast<const uint16_t*>(stp + LY::kKBytes + LY::kVBytes);
      for (int i = lane * 2; i < G * D; i += 64) {
        const uint32_t x = *reinterpret_cast<const uint32_t*>(qb + i);
        qf[i] = bf16lo(x) * p.scale_log2;
        qf[i + 1] = bf16hi(x) * p.scale_log2;
      }
      __syncwarp();
    }
    const int ntok = inf.ntok;
    if (ntok > 0) {
      // ---- scores: lane t <- token t
      float acc[G];
#pragma unroll
      for (int g = 0; g < G; ++g) acc[g] = 0.f;
      const uint8_t* krow = stp + lane * 128;
#pragma unroll
      for (int h = 0; h < D / 64; ++h) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 kk =
              *reinterpret_cast<const uint4*>(krow + h * (kChunk * 128) + ((c << 4) ^ swz));
          const float k0 = bf16lo(kk.x), k1 = bf16hi(kk.x), k2 = bf16lo(kk.y), k3 = bf16hi(kk.y);
          const float k4 = bf16lo(kk.z), k5 = bf16hi(kk.z), k6 = bf16lo(kk.w), k7 = bf16hi(kk.w);
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float4 qa = *reinterpret_cast<const float4*>(qf + g * D + h * 64 + c * 8);
            const float4 qc = *reinterpret_cast<const float4*>(qf + g * D + h * 64 + c * 8 + 4);
            float a = acc[g];
            a = fmaf(qa.x, k0, a);
            a = fmaf(qa.y, k1, a);
            a = fmaf(qa.z, k2, a);
            a = fmaf(qa.w, k3, a);
            a = fmaf(qc.x, k4, a);
            a = fmaf(qc.y, k5, a);
            a = fmaf(qc.z, k6, a);
            a = fmaf(qc.w, k7, a);
            acc[g] = a;
          }
        }
      }
      // ---- online softmax (log2 domain; hidden tokens get -inf -> weight 0)
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float sv = lane < ntok ? acc[g] : -INFINITY;
        const float mn = fmaxf(m[g], warp_max(sv));
        const float alpha = fast_exp2(m[g] - mn);
        const float pv = fast_exp2(sv - mn);
        l[g] = fmaf(l[g], alpha, pv);
#pragma unroll
        for (int e = 0; e < DPL; ++e) o[g][e] *= alpha;
        m[g] = mn;
        pb[lane * G + g] = pv;
      }
      __syncwarp();
      // ---- P.V: lane owns DPL output columns
      const uint8_t* vb = stp + LY::kKBytes + lane * DPL * 2;
#pragma unroll 4
      for (int t = 0; t < ntok; ++t) {
        float pg[G];
        if constexpr (G % 4 == 0) {
#pragma unroll
          for (int g = 0; g < G; g += 4) {
            const float4 x = *reinterpret_cast<const float4*>(pb + t * G + g);
            pg[g] = x.x; pg[g + 1] = x.y; pg[g + 2] = x.z; pg[g + 3] = x.w;
          }
        } else {
#pragma unroll
          for (int g = 0; g < G; ++g) pg[g] = pb[t * G + g];
        }
        float v[DPL];
        if constexpr (DPL == 4) {
          const uint2 x = *reinterpret_cast<const uint2*>(vb + t * D * 2);
          v[0] = bf16lo(x.x); v[1] = bf16hi(x.x); v[2] = bf16lo(x.y); v[3] = bf16hi(x.y);
        } else {
          const uint32_t x = *reinterpret_cast<const uint32_t*>(vb + t * D * 2);
          v[0] = bf16lo(x); v[1] = bf16hi(x);
        }
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
          for (int e = 0; e < DPL; ++e) o[g][e] = fmaf(pg[g], v[e], o[g][e]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty_bar(stage));

    if (inf.flags & kFlagLast) {
      // ---- merge the four consumers' states of this item
      const ItemInfo it = items[inf.slot];
      const int b = merged & 1;
      const uint32_t phase = (merged >> 1) & 1;
      ++merged;
      float* mine = merge_base + (b * kConsumers + cw) * LY::kMergeEntry;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float ls = warp_sum(l[g]);
        if constexpr (DPL == 4) {
          *reinterpret_cast<float4*>(mine + g * D + lane * 4) =
              make_float4(o[g][0], o[g][1], o[g][2], o[g][3]);
        } else {
          *reinterpret_cast<float2*>(mine + g * D + lane * 2) = make_float2(o[g][0], o[g][1]);
        }
        if (lane == 0) {
          mine[G * D + g] = m[g];
          mine[G * D + G + g] = ls;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(merge_bar(b));
      if (!mbar_wait(merge_bar(b), phase)) break;
      const float* all = merge_base + b * kConsumers * LY::kMergeEntry;
      for (int g = cw; g < G; g += kConsumers) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumers; ++w) M = fmaxf(M, all[w * LY::kMergeEntry + G * D + g]);
        float den = 0.f, num[DPL];
#pragma unroll
        for (int e = 0; e < DPL; ++e) num[e] = 0.f;
        if (M != -INFINITY) {
#pragma unroll
          for (int w = 0; w < kConsumers; ++w) {
            const float* ew = all + w * LY::kMergeEntry;
            const float f = fast_exp2(ew[G * D + g] - M);
            den = fmaf(f, ew[G * D + G + g], den);
#pragma unroll
            for (int e = 0; e < DPL; ++e) num[e] = fmaf(f, ew[g * D + lane * DPL + e], num[e]);
          }
        }
        const float inv = den > 0.f ? 1.f / den : 0.f;
        const float lse = den > 0.f ? (M + __log2f(den)) * 0.69314718055994531f : -INFINITY;
        const int hq = it.g * G + g;
        const size_t row = static_cast<size_t>(it.r) * p.Hq + hq;
        if (it.nsplit == 1) {
          uint16_t* dst = p.out + row * D + lane * DPL;
          if constexpr (DPL == 4) {
            *reinterpret_cast<uint2*>(dst) =
                make_uint2(pack_bf16x2(num[0] * inv, num[1] * inv), pack_bf16x2(num[2] * inv, num[3] * inv));
          } else {
            *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(num[0] * inv, num[1] * inv);
          }
          if (p.out_lse != nullptr && lane == 0) p.out_lse[row] = lse;
        } else {
          const size_t prow = row * p.S_max + it.s;
          float* dst = p.part_o + prow * D + lane * DPL;
          if constexpr (DPL == 4) {
            *reinterpret_cast<float4*>(dst) =
                make_float4(num[0] * inv, num[1] * inv, num[2] * inv, num[3] * inv);
          } else {
            *reinterpret_cast<float2*>(dst) = make_float2(num[0] * inv, num[1] * inv);
          }
          if (lane == 0) p.part_lse[prow] = lse;
        }
      }
    }
    seq += kConsumers;
  }
}

// Merge split partials.  One warp per (request, query head); lane owns D/32
// columns.  skip_single: requests with one split were written by the
// partition kernel already.
template <int D>
__global__ void __launch_bounds__(128) combine_kernel(const float* __restrict__ part_o,
                                                      const float* __restrict__ part_lse,
                                                      const int32_t* __restrict__ num_splits,
                                                      int32_t B, int32_t Hq, int32_t S_max,
                                                      uint16_t* __restrict__ out,
                                                      float* __restrict__ out_lse,
                                                      int skip_single) {
  constexpr int DPL = D / 32;
  constexpr float kLog2e = 1.4426950408889634f;
  const int lane = threadIdx.x & 31;
  const long long idx = static_cast<long long>(blockIdx.x) * 4 + (threadIdx.x >> 5);
  if (idx >= static_cast<long long>(B) * Hq) return;
  const int r = static_cast<int>(idx / Hq);
  int n = num_splits[r];
  if (skip_single && n <= 1) return;
  n = max(0, min(n, S_max));
  const float* ls = part_lse + idx * S_max;
  float M = -INFINITY;
  for (int s = lane; s < n; s += 32) M = fmaxf(M, ls[s]);
  M = warp_max(M);
  float acc[DPL], den = 0.f;
#pragma unroll
  for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
  if (M != -INFINITY) {
    const float* po = part_o + idx * S_max * D + lane * DPL;
#pragma unroll 4
    for (int s = 0; s < n; ++s) {
      const float w = fast_exp2((ls[s] - M) * kLog2e);
      den += w;
      if constexpr (DPL == 4) {
        const float4 x = *reinterpret_cast<const float4*>(po + static_cast<size_t>(s) * D);
        acc[0] = fmaf(w, x.x, acc[0]); acc[1] = fmaf(w, x.y, acc[1]);
        acc[2] = fmaf(w, x.z, acc[2]); acc[3] = fmaf(w, x.w, acc[3]);
      } else {
        const float2 x = *reinterpret_cast<const float2*>(po + static_cast<size_t>(s) * D);
        acc[0] = fmaf(w, x.x, acc[0]); acc[1] = fmaf(w, x.y, acc[1]);
      }
    }
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  uint16_t* dst = out + idx * D + lane * DPL;
  if constexpr (DPL == 4) {
    *reinterpret_cast<uint2*>(dst) =
        make_uint2(pack_bf16x2(acc[0] * inv, acc[1] * inv), pack_bf16x2(acc[2] * inv, acc[3] * inv));
  } else {
    *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  }
  if (out_lse != nullptr && lane == 0) out_lse[idx] = den > 0.f ? M + logf(den) : -INFINITY;
}

}  // namespace decode
}  // namespace pkv
