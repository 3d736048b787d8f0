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
// Work unit ("item"): a token range of one (request r, KV head g); it
// produces the outputs of all G query heads of the group, so every K/V byte
// is read from HBM once and used G times.  Two schedules:
//   automatic split (partition_tokens == 0): each group is padded to whole
//   32-token quanta, led by kGroupCost empty quanta that stand for its fixed
//   per-piece cost, and the groups are laid end to end; warp w takes the
//   w-th of Weff equal slices (to one quantum; at least kMinShare tokens) of
//   that line, so every warp has the same work and all finish together.
//   A slice may
//   end inside a group and the next one continue it: such a group's pieces
//   are split-K partials, merged inside the kernel by a tree of merges of
//   at most kMergeFanIn partials, each done by the warp that completes the
//   node's last child.
//   fixed partition: items are (r, g, split s) of the given length; whole
//   partitions are handed out first and the shorter remainders last, from an
//   atomic counter in the workspace (dynamic balancing over ragged lengths),
//   and combine_kernel merges the partials.
//
// Every warp is independent: it takes an item, walks its page-table entries
// (32 per warp-wide load), and keeps NS-1 chunks in flight in its own ring of
// NS shared-memory stages of 8 KB: a chunk is 2048/d tokens (16 at d=128, 32
// at d=64), K rows then V rows, each 16-row piece one page or half of a
// 32-token page and contiguous in the pool.  Stages are filled with 16-byte
// cp.async copies from all lanes (or bulk copies issued by one lane).  There
// is no cross-warp synchronisation after the planning step.
//
// Scores: T lanes share one token (T = 8, or 16 at d=128 with G=8), each
// holding E = d/T elements of it, so a warp covers 32/T tokens per step.  The
// query rows live in registers (fp32, times scale*log2(e)): each lane keeps
// its E elements of all G heads.  A score is a dot product over the T lanes
// of a group: a butterfly reduce-scatter leaves each lane with the full score
// of one head (G partial sums in, one out, no value sent twice; the heads are
// held in a lane-dependent order so the exchange needs no selects).  K is
// read from shared memory once, with 16-byte loads that cover whole 128-byte
// lines per quarter warp.  The weights go through a small per-warp buffer;
// for P.V lane l owns output elements [l*d/32, (l+1)*d/32) of every head and
// walks the chunk's V rows.  The online softmax keeps a warp-uniform running
// max per head that only moves when a score exceeds it by more than 2^8 (in
// practice on an item's first chunk).
#pragma once

#include "ptx.cuh"

namespace pkv {
namespace decode {

#ifndef PKV_DECODE_CHUNK_BYTES
#define PKV_DECODE_CHUNK_BYTES 8192
#endif
#ifndef PKV_DECODE_CPASYNC
#define PKV_DECODE_CPASYNC 1
#endif
// Stage fills: 16-byte cp.async copies issued by all 32 lanes (completion
// tracked per thread with commit/wait groups), or bulk copies issued by lane
// 0 that complete on the stage's mbarrier.
constexpr bool kCpAsync = PKV_DECODE_CPASYNC != 0;
template <int D>
struct Chunk {
  // tokens per pipeline stage: PKV_DECODE_CHUNK_BYTES of K+V (16 at d=128
  // and 8 KB)
  static constexpr int kTokens = PKV_DECODE_CHUNK_BYTES / (4 * D);
  // token rows per copy unit: one page of 16, half of a 32-token page, or a
  // part of either; each unit is one contiguous run of the pool
  static constexpr int kBoxRows = kTokens < 16 ? kTokens : 16;
  static constexpr int kBoxes = kTokens / kBoxRows;    // copy units per stage (per K or V)
  static_assert(kTokens >= 8 && 32 % kTokens == 0, "chunks tile a 32-token quantum");
};
constexpr int kItemSlots = 8;    // per-warp ring of item descriptors
// Merge-tree nodes above the first level whose first-level child this warp
// completed, climbed after the warp's slice (a slice holds at most two
// pieces of split groups: its first and its last).
constexpr int kClimbSlots = 2;
// Automatic split (partition_tokens == 0): the padded token-heads of the
// batch are cut into one equal slice per warp, at least kMinShare tokens, so
// every warp streams the same number of bytes and all finish together.
constexpr int kMinShare = 128;

constexpr int kPartitionQuantum = 32;  // split lengths are multiples of this
// Each group enters the balanced slicing with this many extra quanta ahead of
// its tokens, which hold no tokens: they stand for the fixed cost of starting
// and ending a piece of a group (page-table fetch, output or partial write,
// and the merge that the warp holding a group's first piece usually does).
#ifndef PKV_DECODE_GROUP_COST
#define PKV_DECODE_GROUP_COST 2
#endif
constexpr int kGroupCost = PKV_DECODE_GROUP_COST;
// Automatic split: the pieces of a (request, KV head) group are merged inside
// the partition kernel by a tree whose nodes merge at most kMergeFanIn
// partials.  Level 0 holds the n pieces; level k+1 has ceil(n_k / fan-in)
// nodes, node j merging children [j*fan-in, (j+1)*fan-in) of level k; the
// single top node writes the output.  The warp whose increment completes a
// node's child count merges it, so no warp waits and no second kernel runs.
// Partial slots of a row: the pieces, then each inner level below the top.
// The fan-in keeps one head's children at 4 KB (8 partials of 128 fp32 or
// 16 of 64), so four heads' fit a warp's two 8 KB stage buffers at once.
template <int D>
constexpr int kMergeFanIn = D == 64 ? 16 : 8;

__host__ __device__ constexpr int merge_tree_slots(int n, int fan_in) {
  int total = n;
  while (n > fan_in) {
    n = (n + fan_in - 1) / fan_in;
    total += n;
  }
  return total;
}
// merge nodes of that tree (the top one included): one counter each
__host__ __device__ constexpr int merge_tree_nodes(int n, int fan_in) {
  int total = 0;
  while (n > 1) {
    n = (n + fan_in - 1) / fan_in;
    total += n;
  }
  return total;
}
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
  uint32_t* group_done;       // [B*Hkv][merge_nodes] finished children per merge node (automatic split)
  int32_t B, Hq, Hkv, P, max_pages, num_pages, S_max, partition, merge_nodes;
  float scale_log2;           // softmax scale * log2(e)
  int32_t meta_ready;         // the kernel ahead writes neither kv_lens nor page_table
  // the step's new rows, one per request ([B][Hkv][D] bf16), or null: row r
  // is the key/value of position kv_lens[r] - 1, written to its pool slot by
  // the warp that streams that position just before it streams it
  const uint16_t* k_new;
  const uint16_t* v_new;
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
  static constexpr int kKBytes = kTok * D * 2;   // K rows [kTok][D] bf16
  static constexpr int kVBytes = kTok * D * 2;   // V rows [kTok][D] bf16
  static constexpr int kStageBytes = kKBytes + kVBytes;
  static constexpr int kQInOff = NS * kStageBytes;              // bf16 [NS][G][D] staged queries
  static constexpr int kPbOff = kQInOff + NS * G * D * 2;       // fp32 [kTok][G][2] (p, p) pairs
  static constexpr int kBarOff = kPbOff + kTok * G * 8;         // NS mbarriers
  static constexpr int kFifoOff = kBarOff + NS * 8;             // NS ChunkInfo
  static constexpr int kItemOff = kFifoOff + NS * 16;           // kItemSlots ItemInfo
  static constexpr int kClimbOff = kItemOff + kItemSlots * 16;  // kClimbSlots ItemInfo
  static constexpr int kWarpBytes = (kClimbOff + kClimbSlots * 16 + 127) / 128 * 128;
  // after the W warp blocks: misc[4], lens[B], prefF[B+1], prefR[B+1]
  static size_t plan_bytes(int B) { return 16 + (3 * static_cast<size_t>(B) + 2) * 4; }
  static size_t bytes(int W, int B) { return static_cast<size_t>(W) * kWarpBytes + plan_bytes(B) + 128; }
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

__host__ __device__ constexpr int ilog2(int x) { return x <= 1 ? 0 : 1 + ilog2(x >> 1); }

// Butterfly reduce-scatter of G per-head partial sums over the T lanes of a
// token group (lanes [T*k, T*k+T)), then an all-reduce over the group bits
// left over.  The caller orders the partial sums per lane as
// v[j] = head h ^ (G-1-j), h = (lane & (T-1)) >> (log2 T - log2 G): at every
// level the first half of v is what the partner keeps, so each lane sends
// v[0..half) and adds what it receives to v[half..G) -- no selects.  On
// return the result is the full sum of head h.
template <int G, int T>
__device__ __forceinline__ float reduce_scatter_heads(float (&v)[G]) {
  constexpr int LG = ilog2(G), LT = ilog2(T);
  static_assert(LG <= LT, "more heads than lanes per token");
#pragma unroll
  for (int lv = 0; lv < LG; ++lv) {
    const int off = T >> (lv + 1);   // partner distance
    const int half = G >> (lv + 1);  // values kept after this level
#pragma unroll
    for (int k = 0; k < half; ++k) v[k] = v[k + half] + __shfl_xor_sync(0xffffffffu, v[k], off);
  }
#pragma unroll
  for (int off = T >> (LG + 1); off > 0; off >>= 1) v[0] += __shfl_xor_sync(0xffffffffu, v[0], off);
  return v[0];
}

// Merge partial slots [base, base + cnt) of the G query heads of one
// (request, KV head) group: o = sum_s w_s o_s / sum_s w_s with
// w_s = exp(lse_s - max lse) (the split-K rule of combine_kernel), into the
// bf16 output (kToOut) or into partial slot dst (normalised o and its lse,
// for the next level of the tree).  One warp, after its slice: the partials
// (other warps wrote them during this launch) are copied through L2 into the
// warp's idle stage buffers, as many heads' at once as fit, so a merge costs
// one memory round trip per batch of heads; lane l then owns elements
// [l*D/32, (l+1)*D/32).  cnt <= kMergeFanIn<D>.
template <int D, int G, int NS, bool kToOut>
__device__ __forceinline__ void merge_staged(const Params& p, int r, int g, int base, int cnt, int dst, int lane,
                                             uint32_t sbase, const float* sbuf) {
  constexpr int FI = kMergeFanIn<D>;
  constexpr int DPL = D / 32;
  constexpr int kPieces = D * 4 / 16;  // 16-byte pieces of one partial row: 32 or 16
  constexpr int kRows = 32 / kPieces;  // rows one warp-wide copy covers
  constexpr int kFit = NS * Layout<D, G, NS>::kStageBytes / (FI * D * 4);
  static_assert(kFit >= 1, "one head's partials fit the stage buffers");
  constexpr int HB = kFit < G ? kFit : G;  // heads per batch
  constexpr float kLog2e = 1.4426950408889634f;
  const size_t row0 = static_cast<size_t>(r) * p.Hq + static_cast<size_t>(g) * G;
  float ls[G];
#pragma unroll
  for (int h = 0; h < G; ++h)
    ls[h] = lane < cnt ? __ldcg(p.part_lse + (row0 + h) * p.S_max + base + lane) : -INFINITY;
#pragma unroll
  for (int h0 = 0; h0 < G; h0 += HB) {
    const int c = lane % kPieces;
#pragma unroll
    for (int hb = 0; hb < HB; ++hb) {
      const float* src = p.part_o + ((row0 + h0 + hb) * p.S_max + base) * D + c * 4;
      for (int sp = lane / kPieces; sp < cnt; sp += kRows)
        cp_async16(sbase + static_cast<uint32_t>(((hb * FI + sp) * D + c * 4) * 4), src + static_cast<size_t>(sp) * D);
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncwarp();
#pragma unroll
    for (int hb = 0; hb < HB; ++hb) {
      const int h = h0 + hb;
      const float lh = ls[h];
      const float M = warp_max(lh);
      const float w = M == -INFINITY ? 0.f : fast_exp2((lh - M) * kLog2e);
      const float den = warp_sum(w);
      float acc[DPL];
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
#pragma unroll
      for (int sp = 0; sp < FI; ++sp) {
        const float ws = __shfl_sync(0xffffffffu, w, sp);
        if (sp < cnt) {
          const float* x = sbuf + (hb * FI + sp) * D + lane * DPL;
#pragma unroll
          for (int e = 0; e < DPL; ++e) acc[e] = fmaf(ws, x[e], acc[e]);
        }
      }
      const float inv = den > 0.f ? 1.f / den : 0.f;
      const float lse = den > 0.f ? M + logf(den) : -INFINITY;
      if constexpr (kToOut) {
        uint16_t* o = p.out + (row0 + h) * D + lane * DPL;
        if constexpr (DPL == 4) {
          *reinterpret_cast<uint2*>(o) =
              make_uint2(pack_bf16x2(acc[0] * inv, acc[1] * inv), pack_bf16x2(acc[2] * inv, acc[3] * inv));
        } else {
          *reinterpret_cast<uint32_t*>(o) = pack_bf16x2(acc[0] * inv, acc[1] * inv);
        }
        if (p.out_lse != nullptr && lane == 0) p.out_lse[row0 + h] = lse;
      } else {
        const size_t prow = (row0 + h) * p.S_max + dst;
        float* o = p.part_o + prow * D + lane * DPL;
        if constexpr (DPL == 4) {
          *reinterpret_cast<float4*>(o) = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
        } else {
          *reinterpret_cast<float2*>(o) = make_float2(acc[0] * inv, acc[1] * inv);
        }
        if (lane == 0) p.part_lse[prow] = lse;
      }
    }
    __syncwarp();  // the next batch overwrites the stage buffers
  }
}

// The same merge of a group's nsplit <= kMergeFanIn<D> pieces (slots
// [0, nsplit)) into the output, inside the streaming loop, where the stage
// buffers are busy: the partials come through registers, one head's batch of
// loads at a time (more heads per batch spill the loop's registers), so it
// costs about one memory round trip per head.
template <int D, int G>
__device__ __forceinline__ void merge_regs(const Params& p, int r, int g, int nsplit, int lane) {
  constexpr int DPL = D / 32;
  constexpr int HB = 1;  // heads per batch of loads
  constexpr float kLog2e = 1.4426950408889634f;
  const size_t row0 = static_cast<size_t>(r) * p.Hq + static_cast<size_t>(g) * G;
  float ls[G];
#pragma unroll
  for (int h = 0; h < G; ++h)
    ls[h] = lane < nsplit ? __ldcg(p.part_lse + (row0 + h) * p.S_max + lane) : -INFINITY;
#pragma unroll
  for (int h0 = 0; h0 < G; h0 += HB) {
    float v[HB][kMergeFanIn<D>][DPL];
#pragma unroll
    for (int hb = 0; hb < HB; ++hb) {
      const float* po = p.part_o + (row0 + h0 + hb) * p.S_max * D + lane * DPL;
#pragma unroll
      for (int s = 0; s < kMergeFanIn<D>; ++s) {
        if (s < nsplit) {
          if constexpr (DPL == 4) {
            const float4 x = __ldcg(reinterpret_cast<const float4*>(po + static_cast<size_t>(s) * D));
            v[hb][s][0] = x.x; v[hb][s][1] = x.y; v[hb][s][2] = x.z; v[hb][s][3] = x.w;
          } else {
            const float2 x = __ldcg(reinterpret_cast<const float2*>(po + static_cast<size_t>(s) * D));
            v[hb][s][0] = x.x; v[hb][s][1] = x.y;
          }
        }
      }
    }
#pragma unroll
    for (int hb = 0; hb < HB; ++hb) {
      const int h = h0 + hb;
      const float M = warp_max(ls[h]);
      const float w = M == -INFINITY ? 0.f : fast_exp2((ls[h] - M) * kLog2e);
      const float den = warp_sum(w);
      float acc[DPL];
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
#pragma unroll
      for (int s = 0; s < kMergeFanIn<D>; ++s) {
        const float ws = __shfl_sync(0xffffffffu, w, s);
        if (s < nsplit) {
#pragma unroll
          for (int e = 0; e < DPL; ++e) acc[e] = fmaf(ws, v[hb][s][e], acc[e]);
        }
      }
      const float inv = den > 0.f ? 1.f / den : 0.f;
      uint16_t* dst = p.out + (row0 + h) * D + lane * DPL;
      if constexpr (DPL == 4) {
        *reinterpret_cast<uint2*>(dst) =
            make_uint2(pack_bf16x2(acc[0] * inv, acc[1] * inv), pack_bf16x2(acc[2] * inv, acc[3] * inv));
      } else {
        *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(acc[0] * inv, acc[1] * inv);
      }
      if (p.out_lse != nullptr && lane == 0) p.out_lse[row0 + h] = den > 0.f ? M + logf(den) : -INFINITY;
    }
  }
}

// The body of the decode kernel, for CTA number `cta` of `ncta` CTAs that
// share the batch, with W decode warps; warps of the CTA past W (when the
// CTA has more, as in the mixed kernel) only take part in its barrier.
// `smem` is the CTA's dynamic shared memory.  kLean: 8 elements of d per
// lane in the score phase even where 16 would fit, which frees the
// registers of half the query rows (for kernels that hold other work).
// kAppend: the launch takes each request's new row from p.k_new / p.v_new
// and writes it to the pool (a separate instantiation, so plain decode keeps
// its code unchanged).
template <int D, int G, int NS, bool kLean = false, bool kAppend = false>
__device__ __forceinline__ void decode_body(const Params& p, int cta, int ncta, int W, uint8_t* smem) {
  using LY = Layout<D, G, NS>;
  constexpr int kFI = kMergeFanIn<D>;  // merge-tree fan-in
  using CK = Chunk<D>;
  constexpr int kTok = CK::kTokens;
  // score phase: E elements of d per lane (16 at d=128 unless G=8, whose
  // doubled query registers would not fit; else 8), T lanes per token
  constexpr int E = (D == 128 && G <= 4 && !kLean) ? 16 : 8;
  constexpr int T = D / E, TPS = 32 / T, STEPS = kTok / TPS;
  constexpr int LG = ilog2(G), LT = ilog2(T);
  constexpr int DPL = D / 32;  // P.V output elements per lane
  const int log2P = 31 - __clz(p.P);  // P is a power of two
  static_assert((T == 8 || T == 16) && (D == 64 || D == 128), "head_dim 64 or 128");
  static_assert(NS >= 2, "at least two stages per warp");
  // launched as a programmatic dependent: nothing global is read before the
  // kernel ahead of it on the stream (usually the append) has completed --
  // except, when the caller vouches that the kernel ahead writes neither the
  // lengths nor the page table (meta_ready) and the split is automatic (the
  // plan then reads no workspace counter), the plan and each warp's first
  // page-table fetch, which so overlap the tail of that kernel
  const bool early = p.meta_ready != 0 && p.partition == 0;
  if (!early) pdl_wait();

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
  ItemInfo* climb = reinterpret_cast<ItemInfo*>(wb + LY::kClimbOff);
  if (warp < W && lane < kClimbSlots) climb[lane].r = -1;
  float* pb = reinterpret_cast<float*>(wb + LY::kPbOff);

  if constexpr (!kCpAsync) {
    if (warp < W && lane == 0) {
      for (int i = 0; i < NS; ++i) mbar_init(full_bar(i), 1);
      fence_barrier_init();
    }
  }

  // ---- plan (warp 0).  Automatic split: every (request, KV head) group is
  // padded to whole 32-token quanta (an empty request to one, so its zero
  // output is written) plus kGroupCost empty leading quanta; prefF[r] is the
  // first quantum of request r's groups
  // in the concatenation, and warp w takes quanta [w*share, (w+1)*share).
  // Fixed partition: whole-partition items first (prefF), then one remainder
  // item per (request, KV head) whose length is not a multiple of the
  // partition (prefR; an empty request also gets one).
  const bool balanced = p.partition == 0;
  if (warp == 0) {
    const int maxL = p.max_pages * p.P;
    bool bad = false;
    for (int r = lane; r < p.B; r += 32) {
      int L = p.kv_lens[r];
      if (L < 0 || L > maxL) {
        bad = true;
        L = L < 0 ? 0 : maxL;
      }
      lens[r] = L;
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0 && cta == 0) raise_flag(PKV_FLAG_BAD_LENGTH);
    int part = 0;
    if (p.partition > 0) {
      part = p.partition;
    } else if (p.partition < 0) {
      part = ((maxL > 0 ? maxL : 1) + kPartitionQuantum - 1) / kPartitionQuantum * kPartitionQuantum;
    }
    __syncwarp();
    int runF = 0, runR = 0;
    if (balanced) {
      for (int base = 0; base < p.B; base += 32) {
        const int r = base + lane;
        int nq = 0;
        if (r < p.B) nq = (max(1, (lens[r] + kPartitionQuantum - 1) / kPartitionQuantum) + kGroupCost) * p.Hkv;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, nq, o);
          if (lane >= o) nq += y;
        }
        if (r < p.B) prefF[r + 1] = runF + nq;
        runF += __shfl_sync(0xffffffffu, nq, 31);
      }
      // slices of floor(Q/Weff) or one quantum more, at least kMinShare tokens
      const int weff = static_cast<int>(
          min(static_cast<long long>(ncta) * W, max(1ll, static_cast<long long>(runF) / (kMinShare / kPartitionQuantum))));
      if (lane == 0) {
        prefF[0] = 0;
        misc[0] = weff;  // warps with a slice
        misc[1] = runF;  // total quanta
        misc[2] = 0;
      }
    }
    for (int base = 0; base < p.B && !balanced; base += 32) {
      const int r = base + lane;
      int nf = 0, nr = 0;
      if (r < p.B) {
        const int L = lens[r];
        nf = (L / part) * p.Hkv;
        nr = (L % part != 0 || L == 0) ? p.Hkv : 0;
        if (cta == 0) p.num_splits[r] = L == 0 ? 1 : (L + part - 1) / part;
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
    if (lane == 0 && !balanced) {
      prefF[0] = 0;
      prefR[0] = 0;
      misc[0] = part;
      misc[1] = runF;
      misc[2] = runR;
    }
  }
  __syncthreads();
  // let a dependent launch (the combine kernel) be scheduled now; it waits
  // for this whole grid to finish before reading anything
  pdl_launch_dependents();
  if (warp >= W) return;
  // misc[0] holds one value with two readings: under a fixed partition its
  // length in tokens (part), under the automatic split the number of warps
  // that get a slice (weff)
  const int part = misc[0], weff = part;
  const int nF = misc[1], total = misc[1] + misc[2];
  // automatic split: warp w < Weff takes quanta [floor(w*Q/Weff),
  // floor((w+1)*Q/Weff)) of the Q = nF quanta; the slice holding quantum x
  // is floor(((x+1)*Weff - 1) / Q)
  const int wid = cta * W + warp;
  auto slice_start = [&](int w) { return static_cast<int>(static_cast<long long>(w) * nF / weff); };
  auto slice_of = [&](int x) { return static_cast<int>((static_cast<long long>(x + 1) * weff - 1) / nF); };
  int bq = balanced && wid < weff ? slice_start(wid) : 0;
  const int bq_end = balanced && wid < weff ? slice_start(wid + 1) : 0;

  // ================= issue side: item cursor, lane 0 issues TMA =================
  bool more = true, active = false;
  int it_r = 0, it_g = 0, it_t0 = 0, it_ntok = 0, it_nch = 0, it_k = 0, it_slot = 0, it_qslot = 0;
  int fetched = 0, pid_base = 0, pid_cur = -1, pid_next = -1, it_npg = 0;
  const int32_t* ptab = p.page_table;

  auto fetch = [&]() {
    int r, g, s, t0, ntok, nsplit;
    if (balanced) {
      // next piece of this warp's slice: the rest of the group at bq; a
      // piece that holds only a group's cost quanta is no item
      int first, iend;
      for (;;) {
        if (bq >= bq_end) {
          more = false;
          return;
        }
        r = upper_index(prefF, p.B, bq);
        const int gq = (prefF[r + 1] - prefF[r]) / p.Hkv;  // quanta per group of request r
        g = (bq - prefF[r]) / gq;
        const int gstart = prefF[r] + g * gq;
        first = gstart + kGroupCost;  // the group's first token quantum
        iend = min(gstart + gq, bq_end);
        if (iend > first) {
          nsplit = slice_of(gstart + gq - 1) - slice_of(first) + 1;
          break;
        }
        bq = iend;
      }
      t0 = (max(bq, first) - first) * kPartitionQuantum;
      ntok = max(0, min((iend - first) * kPartitionQuantum, lens[r]) - t0);
      s = wid - slice_of(first);
      bq = iend;
    } else {
    int idx = 0;
    if (lane == 0) idx = static_cast<int>(atomicAdd(p.counters, 1u));
    idx = __shfl_sync(0xffffffffu, idx, 0);
    if (idx >= total) {
      more = false;
      return;
    }
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
    nsplit = lens[r] == 0 ? 1 : (lens[r] + part - 1) / part;
    }
    it_r = r;
    it_g = g;
    it_t0 = t0;
    it_ntok = ntok;
    it_nch = (ntok + kTok - 1) / kTok;
    it_k = 0;
    it_slot = fetched % kItemSlots;
    it_qslot = fetched % NS;
    ++fetched;
    if (lane == 0) items[it_slot] = ItemInfo{r, g, s, nsplit};
    it_npg = (ntok + p.P - 1) >> log2P;
    ptab = p.page_table + static_cast<size_t>(r) * p.max_pages + (t0 >> log2P);
    pid_base = 0;
    pid_cur = lane < it_npg ? __ldg(ptab + lane) : -1;
    pid_next = 32 + lane < it_npg ? __ldg(ptab + 32 + lane) : -1;
    active = true;
    if (balanced && bq < bq_end && lane == 0) {
      // the next item of the slice is known: pull its first page-table line
      // into L1 now, so starting it does not wait on the page table
      const int r2 = upper_index(prefF, p.B, bq);
      const int gq2 = (prefF[r2 + 1] - prefF[r2]) / p.Hkv;
      const int g2 = (bq - prefF[r2]) / gq2;
      const int t2 = max(0, bq - prefF[r2] - g2 * gq2 - kGroupCost) * kPartitionQuantum;
      prefetch_l1(p.page_table + static_cast<size_t>(r2) * p.max_pages + (t2 >> log2P));
    }
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
    const int nbox = (ntok + CK::kBoxRows - 1) / CK::kBoxRows;
    // each 16-row piece lies inside one page: page-table entry (tok >> log2P),
    // first row (tok & (P-1)); out-of-range page ids read page 0 instead
    // (wrong values, no stray access) and raise PKV_FLAG_BAD_PAGE
    size_t rows[CK::kBoxes];
    uint32_t bad_boxes = 0;  // boxes whose page id was out of range (read from page 0)
#pragma unroll
    for (int b = 0; b < CK::kBoxes; ++b) {
      rows[b] = 0;
      if (b < nbox) {
        const int pi = (tok0 + b * CK::kBoxRows) >> log2P;
        while (pi >= pid_base + 32) {
          pid_base += 32;
          pid_cur = pid_next;
          pid_next = pid_base + 32 + lane < it_npg ? __ldg(ptab + pid_base + 32 + lane) : -1;
        }
        int page = __shfl_sync(0xffffffffu, pid_cur, pi & 31);
        if (static_cast<unsigned>(page) >= static_cast<unsigned>(p.num_pages)) {
          if (lane == 0) raise_flag(PKV_FLAG_BAD_PAGE);
          page = 0;
          bad_boxes |= 1u << b;
        }
        rows[b] = (static_cast<size_t>(page) * p.Hkv + it_g) * p.P + ((tok0 + b * CK::kBoxRows) & (p.P - 1));
      }
    }
    const uint32_t st = wbase + stage * LY::kStageBytes;
    const uint16_t* qsrc = p.q + (static_cast<size_t>(it_r) * p.Hq + static_cast<size_t>(it_g) * G) * D;
    const uint32_t qdst = wbase + LY::kQInOff + it_qslot * (G * D * 2);
    if (lane == 0) fifo[stage] = ChunkInfo{it_slot, ntok, flags, it_qslot};
    if constexpr (kCpAsync) {
      if (ntok > 0) {
        constexpr int kPieces = CK::kBoxRows * D / 8;  // 16-byte pieces per 16-row piece
        // the chunk that ends the request holds position kv_lens[r] - 1: with
        // the step's new rows given, the warp first writes that row to its
        // pool slot (one 16-byte piece per lane, K then V), makes the stores
        // visible device-wide and then streams the chunk as usual; no other
        // warp of the launch reads that slot.  A bad page id or an
        // out-of-range length (both flagged) writes nothing.
        if constexpr (kAppend) {
          if ((flags & kLast) && it_t0 + it_ntok == lens[it_r]) {
            const int last = ntok - 1, bl = last / CK::kBoxRows;
            if (((bad_boxes >> bl) & 1u) == 0 && __ldg(p.kv_lens + it_r) == lens[it_r] && lane < D / 4) {
              const bool is_v = lane >= D / 8;
              const int piece = is_v ? lane - D / 8 : lane;
              const size_t nrow = (static_cast<size_t>(it_r) * p.Hkv + it_g) * D + piece * 8;
              size_t row_bl = 0;  // rows[bl], selected without indexing the array at run time
#pragma unroll
              for (int b = 0; b < CK::kBoxes; ++b)
                if (b == bl) row_bl = rows[b];
              const size_t prow = (row_bl + last % CK::kBoxRows) * D + piece * 8;
              const uint4 val = *reinterpret_cast<const uint4*>((is_v ? p.v_new : p.k_new) + nrow);
              *reinterpret_cast<uint4*>(const_cast<uint16_t*>(is_v ? p.v_pool : p.k_pool) + prow) = val;
              __threadfence();
            }
            __syncwarp();
          }
        }
#pragma unroll
        for (int b = 0; b < CK::kBoxes; ++b) {
          if (b >= nbox) break;
          const uint8_t* ksrc = reinterpret_cast<const uint8_t*>(p.k_pool + rows[b] * D);
          const uint8_t* vsrc = reinterpret_cast<const uint8_t*>(p.v_pool + rows[b] * D);
#pragma unroll
          for (int i = lane; i < kPieces; i += 32) {
            cp_async16(st + b * (CK::kBoxRows * D * 2) + i * 16, ksrc + i * 16);
            cp_async16(st + LY::kKBytes + b * (CK::kBoxRows * D * 2) + i * 16, vsrc + i * 16);
          }
        }
        if (it_k == 0) {
#pragma unroll
          for (int i = lane; i < G * D * 2 / 16; i += 32)
            cp_async16(qdst + i * 16, reinterpret_cast<const uint8_t*>(qsrc) + i * 16);
        }
      }
    } else if (lane == 0) {
      if (ntok > 0) {
        const bool with_q = it_k == 0;
        const uint32_t bytes = static_cast<uint32_t>(nbox * CK::kBoxRows * D * 2 * 2) +
                               (with_q ? static_cast<uint32_t>(G * D * 2) : 0u);
        mbar_arrive_expect_tx(full_bar(stage), bytes);
#pragma unroll
        for (int b = 0; b < CK::kBoxes; ++b) {
          if (b >= nbox) break;
          bulk_load(st + b * (CK::kBoxRows * D * 2), p.k_pool + rows[b] * D, CK::kBoxRows * D * 2, full_bar(stage));
          bulk_load(st + LY::kKBytes + b * (CK::kBoxRows * D * 2), p.v_pool + rows[b] * D, CK::kBoxRows * D * 2,
                    full_bar(stage));
        }
        if (with_q) bulk_load(qdst, qsrc, G * D * 2, full_bar(stage));
      } else {
        mbar_arrive(full_bar(stage));
      }
    }
    __syncwarp();
    if (++it_k >= max(1, it_nch)) active = false;
    return true;
  };

  if (early) {
    if (more && !active) fetch();
    pdl_wait();  // the queries, the pools and the workspace come after the kernel ahead
  }
  // ================================ compute side ================================
  // Score phase: token group tg (token tg of each step); this lane holds E
  // elements of d as E/8 pieces of 8, piece j at elements [8*(T*j + ei), +8).
  // Its query registers hold the G heads in the order perm[j] = h ^ (G-1-j),
  // h being the head it ends up with, so the reduce-scatter needs no selects.
  const int tg = lane / T, ei = lane & (T - 1);
  const int hl = ei >> (LT - LG);  // the head whose score this lane holds
  float2 qv[G][E / 2];             // query * scale*log2(e), permuted heads
  // P.V phase: lane owns output elements [lane*DPL, (lane+1)*DPL) of every head
  float2 o2[G][DPL / 2];
  float m[G];                      // running max per head (log2 units), warp-uniform
  float m_lane = -INFINITY;        // m[hl]
  float l_lane = 0.f;              // sum of this lane's weights (head hl, its token group)
#pragma unroll
  for (int g = 0; g < G; ++g) m[g] = -INFINITY;
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
#pragma unroll
        for (int e = 0; e < DPL / 2; ++e) o2[g][e] = make_float2(0.f, 0.f);
      }
      m_lane = -INFINITY;
      l_lane = 0.f;
      if (ntok > 0) {
        const uint8_t* qin = wb + LY::kQInOff + ci.qslot * (G * D * 2) + ei * 16;
#pragma unroll
        for (int jj = 0; jj < G; ++jj) {
          const int head = hl ^ (G - 1 - jj);
#pragma unroll
          for (int j = 0; j < E / 8; ++j) {
            const uint4 x = *reinterpret_cast<const uint4*>(qin + head * D * 2 + j * T * 16);
            qv[jj][j * 4 + 0] = make_float2(bf16lo(x.x) * p.scale_log2, bf16hi(x.x) * p.scale_log2);
            qv[jj][j * 4 + 1] = make_float2(bf16lo(x.y) * p.scale_log2, bf16hi(x.y) * p.scale_log2);
            qv[jj][j * 4 + 2] = make_float2(bf16lo(x.z) * p.scale_log2, bf16hi(x.z) * p.scale_log2);
            qv[jj][j * 4 + 3] = make_float2(bf16lo(x.w) * p.scale_log2, bf16hi(x.w) * p.scale_log2);
          }
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
      const uint8_t* krow = stp + tg * D * 2 + ei * 16;  // piece 0 of this lane's token, step 0
      // ---- scores of every step: lane holds head hl of token step*TPS + tg
      float sc[STEPS];
#pragma unroll
      for (int s = 0; s < STEPS; ++s) {
        float2 acc[G];
#pragma unroll
        for (int j = 0; j < E / 8; ++j) {
          const uint4 kk = *reinterpret_cast<const uint4*>(krow + s * TPS * D * 2 + j * T * 16);
          const float2 k0 = make_float2(bf16lo(kk.x), bf16hi(kk.x));
          const float2 k1 = make_float2(bf16lo(kk.y), bf16hi(kk.y));
          const float2 k2 = make_float2(bf16lo(kk.z), bf16hi(kk.z));
          const float2 k3 = make_float2(bf16lo(kk.w), bf16hi(kk.w));
#pragma unroll
          for (int jj = 0; jj < G; ++jj) {
            float2 a = j == 0 ? __fmul2_rn(qv[jj][0], k0) : __ffma2_rn(qv[jj][j * 4], k0, acc[jj]);
            a = __ffma2_rn(qv[jj][j * 4 + 1], k1, a);
            a = __ffma2_rn(qv[jj][j * 4 + 2], k2, a);
            acc[jj] = __ffma2_rn(qv[jj][j * 4 + 3], k3, a);
          }
        }
        float part[G];
#pragma unroll
        for (int jj = 0; jj < G; ++jj) part[jj] = acc[jj].x + acc[jj].y;
        sc[s] = reduce_scatter_heads<G, T>(part);
      }
      if (ntok < kTok) {
#pragma unroll
        for (int s = 0; s < STEPS; ++s)
          if (s * TPS + tg >= ntok) sc[s] = -INFINITY;
      }
      // ---- online softmax (log2 domain).  The running max moves only when a
      // score exceeds it by more than 2^8; between moves the weights are taken
      // against the stale max (so p <= 2^8) and the final division by l uses
      // the same max, so the result is the same softmax.
      bool grow = false;
#pragma unroll
      for (int s = 0; s < STEPS; ++s) grow |= sc[s] > m_lane + kLazyRescale;
      if (__any_sync(0xffffffffu, grow)) {
        float mx = sc[0];
#pragma unroll
        for (int s = 1; s < STEPS; ++s) mx = fmaxf(mx, sc[s]);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float mg = warp_max(hl == g ? mx : -INFINITY);
          const float mn = fmaxf(m[g], mg);
          const float alpha = mn == -INFINITY ? 1.f : fast_exp2(m[g] - mn);
          m[g] = mn;
          const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
          for (int e = 0; e < DPL / 2; ++e) o2[g][e] = __fmul2_rn(o2[g][e], a2);
          if (hl == g) {
            l_lane *= alpha;
            m_lane = mn;
          }
        }
      }
      // weights -> per-warp buffer as (p, p) pairs [token][head]
#pragma unroll
      for (int s = 0; s < STEPS; ++s) {
        const float pw = fast_exp2(sc[s] - m_lane);
        l_lane += pw;
        *reinterpret_cast<float2*>(pb + ((s * TPS + tg) * G + hl) * 2) = make_float2(pw, pw);
      }
      __syncwarp();
      // ---- P.V: lane accumulates its DPL elements of every head over the chunk
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
      } else {             // rows past ntok may hold anything: never read
#pragma unroll 1
        for (int t = 0; t < ntok; ++t) pv_token(t);
      }
      __syncwarp();  // pb is rewritten by the next chunk
    }

    if (ci.flags & kLast) {
      // ---- item done: total weight per head, normalise, and write bf16
      // output (single-split request) or an fp32 partial and its lse
      const ItemInfo it = items[ci.slot];
#pragma unroll
      for (int off = T; off < 32; off <<= 1) l_lane += __shfl_xor_sync(0xffffffffu, l_lane, off);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float ls = __shfl_sync(0xffffffffu, l_lane, g << (LT - LG));  // total weight of head g
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
      if (balanced && it.nsplit > 1) {
        // count this piece in its first-level merge node; the warp that
        // completes the node merges it: now when it is the tree's top, else
        // after its slice.  Lane 0's release add publishes every lane's
        // partial stores (they precede it through the warp barrier).
        __syncwarp();
        const int jp = it.s / kFI;
        uint32_t* c = p.group_done + (static_cast<size_t>(it.r) * p.Hkv + it.g) * p.merge_nodes + jp;
        uint32_t done = 0;
        if (lane == 0) done = atomic_add_release_gpu(c, 1u);
        done = __shfl_sync(0xffffffffu, done, 0);
        if (done == static_cast<uint32_t>(min(kFI, it.nsplit - jp * kFI) - 1)) {
          __threadfence();
          if (lane == 0) *c = 0;  // ready for the next launch
          if (it.nsplit <= kFI) {
            merge_regs<D, G>(p, it.r, it.g, it.nsplit, lane);  // a one-level tree: done now
          } else if (lane == 0) {
            climb[climb[0].r < 0 ? 0 : 1] = ItemInfo{it.r, it.g, jp, it.nsplit};
          }
        }
      }
    }
  }
  if constexpr (!kCpAsync) {
    if (n < issued) {
      // a wait gave up: give copies still in flight a bounded chance to land
      for (int k = n + 1; k < issued; ++k) mbar_wait(full_bar(k % NS), (k / NS) & 1);
    }
  } else {
    cp_async_wait<0>();
  }
  // merge the first-level tree nodes this warp completed, then climb: node
  // (level k, index j) of a group cut into n pieces merges children slots
  // off_{k-1} + [j*fan-in, (j+1)*fan-in) into slot off_k + j (off_0 = 0,
  // off_{k+1} = off_k + n_k) or, at the top, into the output, and counts its
  // finished children in counter off_k - n + j
  __syncwarp();
#pragma unroll 1
  for (int e = 0; e < kClimbSlots; ++e) {
    const ItemInfo cl = climb[e];
    if (cl.r < 0) continue;
    __threadfence();  // acquire: lane 0 saw the node's last child arrive
    const int n = cl.nsplit;
    uint32_t* ctr = p.group_done + (static_cast<size_t>(cl.r) * p.Hkv + cl.g) * p.merge_nodes;
    int j = cl.s, nprev = n, offprev = 0, nk = (n + kFI - 1) / kFI, offk = n;
    for (;;) {
      const int c0 = j * kFI, cnt = min(kFI, nprev - c0);
      if (nk == 1) {
        merge_staged<D, G, NS, true>(p, cl.r, cl.g, offprev + c0, cnt, 0, lane, wbase, reinterpret_cast<const float*>(wb));
        break;
      }
      merge_staged<D, G, NS, false>(p, cl.r, cl.g, offprev + c0, cnt, offk + j, lane, wbase,
                                   reinterpret_cast<const float*>(wb));
      const int jp = j / kFI;
      uint32_t* c = ctr + (offk + nk - n + jp);
      __syncwarp();
      uint32_t done = 0;
      if (lane == 0) done = atomic_add_release_gpu(c, 1u);
      done = __shfl_sync(0xffffffffu, done, 0);
      if (done != static_cast<uint32_t>(min(kFI, nk - jp * kFI) - 1)) break;
      __threadfence();
      if (lane == 0) *c = 0;  // ready for the next launch
      nprev = nk;
      offprev = offk;
      offk += nk;
      nk = (nk + kFI - 1) / kFI;
      j = jp;
    }
  }
  if (lane == 0) {
    __threadfence();
    if (atomicAdd(&p.counters[1], 1u) == static_cast<uint32_t>(ncta * W - 1)) {
      p.counters[0] = 0;
      p.counters[1] = 0;
      __threadfence();
    }
  }
}

template <int D, int G, int NS, int MAXW, bool APPEND = false>
__global__ void __launch_bounds__(MAXW * 32, 1) partition_kernel(const Params p) {
  extern __shared__ __align__(128) uint8_t smem[];
  decode_body<D, G, NS, false, APPEND>(p, blockIdx.x, gridDim.x, blockDim.x >> 5, smem);
}

// Merge split partials.  One CTA per (request, query head) row; its warps
// stride over the splits (four splits' loads in flight per warp), each lane
// owning D/32 columns, and the per-warp sums meet in shared memory.
// num_splits[row / Hq] is the row's split count; rows with at most
// skip_below splits are left alone (a fixed-partition decode writes the
// unsplit rows itself).
constexpr int kCombineMaxWarps = 8;

template <int D>
__global__ void __launch_bounds__(32 * kCombineMaxWarps) combine_kernel(
    const float* __restrict__ part_o, const float* __restrict__ part_lse,
    const int32_t* __restrict__ num_splits, int32_t Hq, int32_t S_max,
    uint16_t* __restrict__ out, float* __restrict__ out_lse, int skip_below) {
  constexpr int DPL = D / 32;
  constexpr float kLog2e = 1.4426950408889634f;
  __shared__ float red_m[kCombineMaxWarps], red_den[kCombineMaxWarps];
  __shared__ __align__(16) float red_acc[kCombineMaxWarps][D];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const long long row = blockIdx.x;
  // launched as a programmatic dependent of the partition kernel: wait for
  // that grid to complete (a no-op when launched normally)
  pdl_wait();
  int n = num_splits[row / Hq];
  if (n <= skip_below) return;
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
