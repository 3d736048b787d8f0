// prefill.cuh -- causal attention of prompt chunks at per-request context
// offsets, reading K/V from the paged pool, on 5th-generation tensor cores
// (tcgen05.mma, accumulators in tensor memory).
//
// Sources: tiny-llm source reading, "Chunked Prefill" (bounded prompt chunks
// batched with decode work) and "Paged KV Cache" (keys read through the page
// table; paging fused with the online softmax, no score matrix in memory);
// tiny-vllm article, "From Safetensors to PagedAttention" (online softmax).
//
// Tile: one CTA computes 128 query rows = 128/G consecutive chunk positions
// x the G query heads of one KV head (GQA packing: each K/V tile in shared
// memory serves all G heads).  Keys stream in tiles of BN (64: 4 pages of 16
// or 2 of 32), gathered page by page with TMA into 128-byte-swizzled tiles.
//   S = Q K^T   : M=128, N=BN, K=d  -> TMEM (two buffers, double-buffered)
//   softmax     : one thread per TMEM lane (= one query row), log2 domain,
//                 lazy rescale of O only when the running max grows by > 2^8
//   O += P V    : M=128, N=d, K=BN; P (bf16) written back into tensor memory
//                 over the S columns it came from and read by the MMA from
//                 there (A operand in TMEM); V is an MN-major operand
//                 straight from its tile
// With BN=64 a CTA needs ~96 KB of shared memory and 256 TMEM columns, so
// two CTAs share an SM and one CTA's softmax overlaps the other's MMAs.
// Warp roles: warp 0 TMA producer, warp 1 TMEM owner + MMA issuer (one
// thread), warps 2..5 softmax and epilogue.
#pragma once

#include "ptx.cuh"

namespace pkv {
namespace prefill {

constexpr int kM = 128;  // query rows per CTA
constexpr int kThreads = 192;        // TMA warp, MMA warp, 4 softmax warps (chunk units of the mixed kernel)
constexpr int kThreadsAlone = 224;   // the standalone kernel: S and P.V issued by two warps
// What the launcher needs to know: query rows (positions x group heads) per
// CTA, keys per K/V tile (split partitions are multiples of it), and the
// dynamic shared memory of a CTA.
constexpr int kRowsPerCta = kM;
constexpr int kKeyTile = 64;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale when the max grows by > 256x

struct Params {
  const int32_t* cu_q_lens;    // [B+1]
  const int32_t* ctx_offsets;  // [B]
  const int32_t* page_table;   // [B][max_pages]
  uint16_t* out;               // bf16 [total_q][Hq][D]
  int32_t B, Hq, Hkv, P, max_pages, num_pages, total_q;
  int32_t qtiles;  // query tiles per request in the grid (ceil(max_q_len / rows per tile))
  float scale_log2;
  // split-K over the keys (short chunks over long contexts): a CTA takes the
  // keys [s*partition, (s+1)*partition) of its request and, when the request
  // has more than one split, writes a partial normalised within the split and
  // its lse for the combine kernel.  partition = 0: no split (splits = 1).
  int32_t partition;    // keys per split, a multiple of the key tile
  int32_t splits;       // splits per request in the grid
  float* part_o;        // [total_q][Hq][splits][D]
  float* part_lse;      // [total_q][Hq][splits]
  int32_t* num_splits;  // [total_q]: splits of each chunk row's request
};


template <int D, int BN>
struct Layout {
  static constexpr int kQHalf = kM * 128;               // one 64-column half of the Q or P tile
  static constexpr int kKVHalf = BN * 128;              // one 64-column half of a K or V tile
  static constexpr int kQOff = 0;                       // [D/64][128 rows][128 B]
  static constexpr int kKVTile = (D / 64) * kKVHalf;    // [D/64][BN rows][128 B]
  static constexpr int kKOff = kQOff + (D / 64) * kQHalf;  // 2 stages
  static constexpr int kVOff = kKOff + 2 * kKVTile;
  static constexpr int kBarOff = kVOff + 2 * kKVTile;   // P lives in TMEM, over its S columns
  static constexpr int kTmemCols = 2 * BN + D <= 256 ? 256 : 512;  // S0, S1, O
  static constexpr int kColS0 = 0, kColS1 = BN, kColO = 2 * BN;
  // barriers: q, kfull[2], kempty[2], vfull[2], vempty[2], sfull[2], pfull[2], pvdone[2], final
  static constexpr int kNumBars = 16;
  static constexpr int kTmemSlotOff = kBarOff + kNumBars * 8;
  static constexpr size_t kBytes = kTmemSlotOff + 16;  // the base is 1024-byte aligned
};

template <int D>
constexpr size_t smem_bytes();

enum Bar { kQ = 0, kKFull = 1, kKEmpty = 3, kVFull = 5, kVEmpty = 7, kSFull = 9, kPFull = 11,
           kPVDone = 13, kFinal = 15 };

// Rows of a chunk and keys its last row sees: the CTAs' weight ranking key.
__device__ __forceinline__ long long chunk_weight(const Params& p, int r) {
  const int q0 = p.cu_q_lens[r], q1 = p.cu_q_lens[r + 1], c = p.ctx_offsets[r];
  return (q1 >= q0 && c >= 0) ? static_cast<long long>(q1 - q0) * (c + q1 - q0) : 0;
}

// The request that comes rank-th when the requests are ordered by decreasing
// work (rows x keys of the last row, ties by index).  CTAs take the chunks
// heaviest request first, so the longest-running CTAs start early instead of
// being left alone at the end.  The CTA's threads stage one weight each in
// shared memory and each ranks its own request against the staged ones;
// batches larger than the CTA keep their own order.  Every thread of the
// CTA calls it.
constexpr int kRankMax = 192;  // = the chunk kernel's threads
__device__ __forceinline__ int request_by_weight(const Params& p, int rank) {
  __shared__ long long wt[kRankMax];
  __shared__ int chosen;
  if (p.B > kRankMax || p.B > static_cast<int>(blockDim.x)) return rank;
  const int c = threadIdx.x;
  if (c < p.B) wt[c] = chunk_weight(p, c);
  if (c == 0) chosen = rank;
  __syncthreads();
  if (c < p.B) {
    const long long wc = wt[c];
    int k = 0;
    for (int o = 0; o < p.B; ++o) k += (wt[o] > wc) || (wt[o] == wc && o < c);
    if (k == rank) chosen = c;
  }
  __syncthreads();
  const int r = chosen;
  __syncthreads();  // wt and chosen are reused by the next call
  return r;
}

// The body of the chunk kernel for work unit `unit` (what a CTA of the
// standalone launch does for blockIdx.x = unit), on the CTA's dynamic shared
// memory `smem_raw`.  The caller has waited for the kernel ahead.  kOnce: the
// CTA runs one unit and gives up its TMEM allocation permit after it
// allocates; a persistent CTA (one allocation per unit) keeps it.
// kTwoIssuers: warp 1 issues the S MMAs and warp 2 the P.V MMAs (softmax
// warps 3..6); else warp 1 issues both (softmax warps 2..5).  One thread
// issues tcgen05.mma at a bounded rate, so two issuers per CTA keep the
// tensor pipe busier.
template <int D, int G, int BN, bool kOnce = true, bool kTwoIssuers = false>
__device__ __forceinline__ void prefill_body(const CUtensorMap* qmap_p, const CUtensorMap* kmap_p,
                                             const CUtensorMap* vmap_p, const Params& p, int unit,
                                             uint8_t* smem_raw) {
  using LY = Layout<D, BN>;
  constexpr int kN = BN;        // keys per tile
  constexpr int kTmemCols = LY::kTmemCols;
  constexpr int kColS0 = LY::kColS0, kColS1 = LY::kColS1, kColO = LY::kColO;
  constexpr int QPOS = kM / G;  // chunk positions per tile
  constexpr uint32_t kIdescS = idesc_bf16_f32(kM, kN, false, false);
  constexpr uint32_t kIdescPV = idesc_bf16_f32(kM, D, false, true);
  // ---- which tile: the query tiles of one (request, KV head) are
  // adjacent, heaviest (last) first, so the CTAs that read the same keys run
  // together and share them through L2; requests by decreasing work; the
  // splits of one query tile adjacent
  const int split = unit % p.splits;
  const int bx = unit / p.splits;
  const int qt_rev = bx % p.qtiles;
  const int g = (bx / p.qtiles) % p.Hkv;
  const int r = request_by_weight(p, bx / p.qtiles / p.Hkv);
  const int q0 = p.cu_q_lens[r], q1 = p.cu_q_lens[r + 1];
  const int n_r = q1 - q0;
  if (q0 < 0 || n_r < 0 || q1 > p.total_q) {
    if (g == 0 && qt_rev == 0 && threadIdx.x == 0) raise_flag(PKV_FLAG_BAD_QUERY_ROWS);
    return;
  }
  const int n_qt = (n_r + QPOS - 1) / QPOS;
  if (n_qt > p.qtiles) {
    // a chunk longer than the max_q_len the grid was sized for: refused whole
    if (g == 0 && qt_rev == 0 && threadIdx.x == 0) raise_flag(PKV_FLAG_BAD_QUERY_ROWS);
    return;
  }
  if (qt_rev >= n_qt) return;
  const int qt = n_qt - 1 - qt_rev;
  const int c = p.ctx_offsets[r];
  if (c < 0 || static_cast<long long>(c) + n_r > static_cast<long long>(p.max_pages) * p.P) {
    if (g == 0 && qt_rev == 0 && threadIdx.x == 0) raise_flag(PKV_FLAG_BAD_LENGTH);
    return;
  }
  const int pos_lo = c + qt * QPOS;                      // smallest query position in the tile
  const int rows_valid = min(QPOS, n_r - qt * QPOS);     // chunk positions present
  const int kv_end = pos_lo + rows_valid;                // keys 0 .. kv_end-1 are used
  // this CTA's key tiles [j0, j0 + nt): all of them, or its split's
  const bool split_mode = p.partition > 0;
  const int req_splits = split_mode ? (c + n_r + p.partition - 1) / p.partition : 1;
  if (split >= req_splits) return;
  const int j0 = split_mode ? split * (p.partition / kN) : 0;
  const int j1 = split_mode ? min((kv_end + kN - 1) / kN, j0 + p.partition / kN) : (kv_end + kN - 1) / kN;
  const int nt = max(0, j1 - j0);                        // key tiles of this CTA
  const bool to_partial = req_splits > 1;

  // 128-byte swizzle atoms need 1024-byte alignment; the declaration asks
  // for it, and a misaligned base (never expected) is refused, not used
  uint8_t* smem = smem_raw;
  const uint32_t sbase = smem_addr(smem);
  if (sbase & 1023u) {
    if (threadIdx.x == 0) raise_flag(PKV_FLAG_INTERNAL);
    return;
  }
  auto bar = [&](int i) { return sbase + LY::kBarOff + 8u * i; };
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + LY::kTmemSlotOff);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(bar(kQ), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(kKFull + i), 1);
      mbar_init(bar(kKEmpty + i), 1);
      mbar_init(bar(kVFull + i), 1);
      mbar_init(bar(kVEmpty + i), 1);
      mbar_init(bar(kSFull + i), 1);
      mbar_init(bar(kPFull + i), 128);
      mbar_init(bar(kPVDone + i), 1);
    }
    mbar_init(bar(kFinal), kTwoIssuers ? 2 : 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    if constexpr (kOnce)
      tmem_alloc(smem_addr(smem + LY::kTmemSlotOff), kTmemCols);
    else
      tmem_alloc_again(smem_addr(smem + LY::kTmemSlotOff), kTmemCols);
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  const uint32_t sQ = sbase + LY::kQOff;
  auto sK = [&](int b) { return sbase + LY::kKOff + b * LY::kKVTile; };
  auto sV = [&](int b) { return sbase + LY::kVOff + b * LY::kKVTile; };

  if (warp == 0) {
    // ============================ TMA producer ============================
    const int32_t* ptab = p.page_table + static_cast<size_t>(r) * p.max_pages;
    if (lane == 0) {
      prefetch_tensormap(qmap_p);
      prefetch_tensormap(kmap_p);
      prefetch_tensormap(vmap_p);
      mbar_arrive_expect_tx(bar(kQ), kM * D * 2);
#pragma unroll
      for (int h = 0; h < D / 64; ++h)
        tma_load_3d(sQ + h * LY::kQHalf, qmap_p, 64 * h, g * G, q0 + qt * QPOS, bar(kQ));
    }
    // K of tile j only waits for its stage (freed when S of tile j-2 is
    // done); V trails one tile behind, since P.V of a tile runs after its
    // softmax.  Coupling the two would make every S wait for an earlier P.V.
    // page ids of tile j: the request's page-table entries are read 32 at a
    // time, the next 32 already in flight, so no TMA issue waits on them
    const int total_pages = (kv_end + p.P - 1) / p.P;
    int pid_base = (j0 * kN / p.P) & ~31;  // the 32-entry window of the first page
    int pid_cur = pid_base + lane < total_pages ? __ldg(ptab + pid_base + lane) : -1;
    int pid_next = pid_base + 32 + lane < total_pages ? __ldg(ptab + pid_base + 32 + lane) : -1;
    auto tile_pages = [&](int jl) {  // jl: the CTA's local tile index
      const int j = j0 + jl;
      const int first = j * kN / p.P;
      const int npg = (min(kN, kv_end - j * kN) + p.P - 1) / p.P;
      while (first >= pid_base + 32) {
        pid_base += 32;
        pid_cur = pid_next;
        pid_next = pid_base + 32 + lane < total_pages ? __ldg(ptab + pid_base + 32 + lane) : -1;
      }
      // a tile's pages never straddle a 32-entry window: kN/P divides 32
      const int src = (first - pid_base) + (lane < npg ? lane : 0);
      const int pid = __shfl_sync(0xffffffffu, pid_cur, src & 31);
      return make_int2(npg, lane < npg ? pid : -1);
    };
    auto issue_tile = [&](int j, int2 pg, int which) {  // which: 0 = K, 1 = V
      const int b = j & 1;
      const uint32_t full = bar((which ? kVFull : kKFull) + b);
      const CUtensorMap* map = which ? vmap_p : kmap_p;
      const uint32_t dst = which ? sV(b) : sK(b);
      if (lane == 0) mbar_arrive_expect_tx(full, static_cast<uint32_t>(pg.x * p.P * D * 2));
      __syncwarp();
      // one box per lane, lane -> (page pi, 64-column half h): a TMA issue
      // occupies its thread for ~130 cycles, so boxes issued by one lane go
      // out one after another while boxes of different lanes go out together
      constexpr int H = D / 64;
      const int pi = lane / H, h = lane % H;
      const int page = __shfl_sync(0xffffffffu, pg.y, pi & 31);
      if (pi < pg.x) {
        if (which == 0 && h == 0 && static_cast<unsigned>(page) >= static_cast<unsigned>(p.num_pages))
          raise_flag(PKV_FLAG_BAD_PAGE);  // TMA reads zeros out of bounds
        tma_load_3d(dst + h * LY::kKVHalf + pi * p.P * 128, map, 64 * h, 0, page * p.Hkv + g, full);
      }
    };
    bool ok = true;
    int2 pg_prev = make_int2(0, -1);
    for (int j = 0; j <= nt && ok; ++j) {
      int2 pg = make_int2(0, -1);
      if (j < nt) {
        pg = tile_pages(j);
        if (j >= 2 && !(ok = mbar_wait(bar(kKEmpty + (j & 1)), ((j >> 1) - 1) & 1))) break;
        issue_tile(j, pg, 0);
      }
      if (j >= 1) {
        const int jv = j - 1;
        if (jv >= 2 && !(ok = mbar_wait(bar(kVEmpty + (jv & 1)), ((jv >> 1) - 1) & 1))) break;
        issue_tile(jv, pg_prev, 1);
      }
      pg_prev = pg;
      __syncwarp();
    }
  } else if (kTwoIssuers && (warp == 1 || warp == 2)) {
    // ======================== MMA issuers (S / P.V) ========================
    // warp 1: S of tile j once K(j) is in and the buffer's P.V(j-2) is done;
    // warp 2: P.V of tile i once P(i) and V(i) are in
    bool ok = mbar_wait(bar(kQ), 0);
    if (warp == 1) {
      for (int j = 0; j < nt && ok; ++j) {
        const int b = j & 1;
        ok = (j < 2 || mbar_wait(bar(kPVDone + b), ((j - 2) >> 1) & 1)) && mbar_wait(bar(kKFull + b), (j >> 1) & 1);
        if (!ok) break;
        tc_fence_after_sync();
        if (lane == 0) {
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint64_t a = smem_desc_sw128(sQ + (ks >> 2) * LY::kQHalf + (ks & 3) * 32, 16, 1024);
            const uint64_t bdesc = smem_desc_sw128(sK(b) + (ks >> 2) * LY::kKVHalf + (ks & 3) * 32, 16, 1024);
            tc_mma_ss(tmem + (b ? kColS1 : kColS0), a, bdesc, kIdescS, ks > 0);
          }
          tc_commit(bar(kSFull + b));
          tc_commit(bar(kKEmpty + b));
        }
        __syncwarp();
      }
    } else {
      for (int i = 0; i < nt && ok; ++i) {
        const int b = i & 1;
        ok = mbar_wait(bar(kPFull + b), (i >> 1) & 1) && mbar_wait(bar(kVFull + b), (i >> 1) & 1);
        if (!ok) break;
        tc_fence_after_sync();
        if (lane == 0) {
#pragma unroll
          for (int ks = 0; ks < kN / 16; ++ks) {
            const uint32_t a = tmem + (b ? kColS1 : kColS0) + ks * 8;
            const uint64_t bdesc = smem_desc_sw128(sV(b) + ks * 16 * 128, LY::kKVHalf, 1024);
            tc_mma_ts(tmem + kColO, a, bdesc, kIdescPV, i > 0 || ks > 0);
          }
          tc_commit(bar(kPVDone + b));
          tc_commit(bar(kVEmpty + b));
        }
        __syncwarp();
      }
    }
    if (lane == 0) tc_commit(bar(kFinal));
    __syncwarp();
  } else if (warp == 1) {
    // ============================ MMA issuer =============================
    // Two streams of MMAs: S of tile j (needs K(j) and a free S buffer) and
    // P.V of tile j (needs P(j) and V(j)).  The issuer takes whichever is
    // ready, P.V first, so a late K tile never holds up a P.V the softmax
    // warps are waiting for.  S of tile j+2 reuses the buffer of tile j as
    // soon as the softmax warps have read S(j).
    bool ok = mbar_wait(bar(kQ), 0);
    auto do_pv = [&](int i) {
      const int b = i & 1;
      tc_fence_after_sync();
      if (lane == 0) {
#pragma unroll
        for (int ks = 0; ks < kN / 16; ++ks) {
          // A = P(i) from TMEM: 16 bf16 per row = 8 columns of its S buffer
          const uint32_t a = tmem + (b ? kColS1 : kColS0) + ks * 8;
          const uint64_t bdesc = smem_desc_sw128(sV(b) + ks * 16 * 128, LY::kKVHalf, 1024);
          tc_mma_ts(tmem + kColO, a, bdesc, kIdescPV, i > 0 || ks > 0);
        }
        tc_commit(bar(kPVDone + b));
        tc_commit(bar(kVEmpty + b));
      }
      __syncwarp();
    };
    auto do_s = [&](int j) {
      const int b = j & 1;
      tc_fence_after_sync();
      if (lane == 0) {
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t a = smem_desc_sw128(sQ + (ks >> 2) * LY::kQHalf + (ks & 3) * 32, 16, 1024);
          const uint64_t bdesc = smem_desc_sw128(sK(b) + (ks >> 2) * LY::kKVHalf + (ks & 3) * 32, 16, 1024);
          tc_mma_ss(tmem + (b ? kColS1 : kColS0), a, bdesc, kIdescS, ks > 0);
        }
        tc_commit(bar(kSFull + b));
        tc_commit(bar(kKEmpty + b));
      }
      __syncwarp();
    };
    for (int j = 0; j < 2 && j < nt && ok; ++j) {
      ok = mbar_wait(bar(kKFull + (j & 1)), (j >> 1) & 1);
      if (ok) do_s(j);
    }
    int ns = 2, npv = 0;
    uint64_t t_idle = global_timer_ns();
    while (ok && npv < nt) {
      int act = 0;  // 1: P.V(npv), 2: S(ns); decided by lane 0 for the whole warp
      if (lane == 0) {
        if (mbar_try_wait(bar(kPFull + (npv & 1)), (npv >> 1) & 1) &&
            mbar_try_wait(bar(kVFull + (npv & 1)), (npv >> 1) & 1))
          act = 1;
        else if (ns < nt && mbar_try_wait(bar(kPVDone + (ns & 1)), ((ns - 2) >> 1) & 1) &&
                 mbar_try_wait(bar(kKFull + (ns & 1)), (ns >> 1) & 1))
          act = 2;  // S(ns) overwrites the buffer whose P fed PV(ns-2): wait for it
      }
      act = __shfl_sync(0xffffffffu, act, 0);
      if (act == 1) {
        do_pv(npv++);
        t_idle = global_timer_ns();
      } else if (act == 2) {
        do_s(ns++);
        t_idle = global_timer_ns();
      } else if (global_timer_ns() - t_idle > kWaitLimitNs) {
        if (lane == 0) raise_flag(PKV_FLAG_WAIT_TIMEOUT);
        ok = false;
      }
    }
    if (lane == 0) tc_commit(bar(kFinal));
    __syncwarp();
  } else {
    // ========================= softmax / epilogue ========================
    const int quad = warp & 3;             // TMEM lane quadrant this warp may access
    const int sw = warp - (kTwoIssuers ? 3 : 2);  // 0..3 within the softmax warps (ragged-tile zeroing)
    const int row = quad * 32 + lane;      // query row of this thread
    const int pos_local = row / G, hh = row % G;
    const int qpos = pos_lo + pos_local;   // absolute position
    const bool row_valid = pos_local < rows_valid;
    // a warp whose 32 rows all lie past the chunk (short chunks, the last
    // tile of a chunk) computes no softmax: it waits for S (so it never runs
    // ahead into the next phase), zeroes its share of a ragged V tile and
    // counts itself done with P; its rows' P and O are never read out
    const bool warp_idle = quad * 32 >= rows_valid * G;
    const uint32_t trow = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const float sl2 = p.scale_log2;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nt; ++j) {
      const int b = j & 1;
      if (!mbar_wait(bar(kSFull + b), (j >> 1) & 1)) { ok = false; break; }
      const int key0 = (j0 + j) * kN;
      if (!warp_idle) {
      tc_fence_after_sync();
      // raw scores of this row; hidden keys -> -inf (scale > 0, so the max
      // of raw scores gives the max of scaled ones)
      float s[kN];
      {
        uint32_t v[kN / 32][32];
#pragma unroll
        for (int cc = 0; cc < kN / 32; ++cc) tmem_ld_32x32b_x32(trow + (b ? kColS1 : kColS0) + cc * 32, v[cc]);
        tmem_wait_ld();
#pragma unroll
        for (int cc = 0; cc < kN / 32; ++cc)
#pragma unroll
          for (int e = 0; e < 32; ++e) s[cc * 32 + e] = __uint_as_float(v[cc][e]);
      }
      if (key0 + kN - 1 > pos_lo || key0 + kN > kv_end) {  // diagonal or ragged tile
#pragma unroll
        for (int e = 0; e < kN; ++e) {
          const int key = key0 + e;
          if (key > qpos || key >= kv_end) s[e] = -INFINITY;
        }
      }
      float mx = -INFINITY;
#pragma unroll
      for (int e = 0; e < kN; ++e) mx = fmaxf(mx, s[e]);
      const float mc = fmaxf(m, mx * sl2);
      const bool need = mc > m + kRescaleThreshold;
      float alpha = 1.f;
      if (need) {
        alpha = fast_exp2(m - mc);
        m = mc;
      }
      // p = 2^(s*scale*log2e - m): one FMA and one exp2 per element.  A row
      // that has seen no visible key yet (possible inside a later split) keeps
      // m = -inf; its weights are then 2^-inf = 0, never 2^(-inf + inf).
      const float msub = m == -INFINITY ? 0.f : m;
      uint32_t pk[kN / 2];
      float2 rs = make_float2(0.f, 0.f);
#pragma unroll
      for (int e = 0; e < kN; e += 2) {
        const float a0 = fast_exp2(fmaf(s[e], sl2, -msub)), a1 = fast_exp2(fmaf(s[e + 1], sl2, -msub));
        rs = __fadd2_rn(rs, make_float2(a0, a1));
        pk[e / 2] = pack_bf16x2(a0, a1);
      }
      l = fmaf(l, alpha, rs.x + rs.y);
      if (j >= 1 && __any_sync(0xffffffffu, need)) {
        // O is rescaled only after PV of the previous tile is done
        if (!mbar_wait(bar(kPVDone + ((j - 1) & 1)), ((j - 1) >> 1) & 1)) { ok = false; break; }
        tc_fence_after_sync();
        {
#pragma unroll 1
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(trow + kColO + cc * 32, v);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
            tmem_st_32x32b_x32(trow + kColO + cc * 32, v);
          }
          tmem_wait_st();
        }
      }
      // P row -> TMEM over this tile's S columns (read above), the K-major
      // A operand of the PV MMA: two bf16 per 32-bit column
#pragma unroll
      for (int cc = 0; cc < kN / 64; ++cc) {
        uint32_t w[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) w[e] = pk[cc * 32 + e];
        tmem_st_32x32b_x32(trow + (b ? kColS1 : kColS0) + cc * 32, w);
      }
      tmem_wait_st();
      }  // !warp_idle
      if (key0 + kN > kv_end) {
        // ragged last tile: V rows past kv_end were not loaded (or hold
        // unused slots); zero them so 0 * garbage cannot reach O
        if (!mbar_wait(bar(kVFull + b), (j >> 1) & 1)) { ok = false; break; }
        const int first = kv_end - key0;
        const int nbytes = (kN - first) * 128;
        for (int h = 0; h < D / 64; ++h) {
          uint8_t* vz = smem + LY::kVOff + b * LY::kKVTile + h * LY::kKVHalf + first * 128;
          for (int off = (sw * 32 + lane) * 16; off < nbytes; off += kM * 16)
            *reinterpret_cast<uint4*>(vz + off) = make_uint4(0, 0, 0, 0);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before_sync();
      mbar_arrive(bar(kPFull + b));
    }
    const bool have_o = ok && !warp_idle && nt >= 1 && mbar_wait(bar(kPVDone + ((nt - 1) & 1)), ((nt - 1) >> 1) & 1);
    const size_t qrow = static_cast<size_t>(q0 + qt * QPOS + pos_local);  // this thread's chunk row
    if (split_mode && split == 0 && g == 0 && hh == 0 && row_valid) p.num_splits[qrow] = req_splits;
    if (have_o) tc_fence_after_sync();
    const float inv = l > 0.f ? 1.f / l : 0.f;
    if (to_partial && !warp_idle && (have_o || (ok && nt == 0))) {
      // a partial normalised within this split (zero, lse -inf, when the
      // split holds none of the tile's keys), for the combine kernel
      const size_t prow = (qrow * p.Hq + g * G + hh) * p.splits + split;
      float* dst = p.part_o + prow * D;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t v[32];
        if (have_o) {
          tmem_ld_32x32b_x32(trow + kColO + cc * 32, v);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = 0u;
        }
        if (row_valid) {
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(dst + cc * 32 + e) =
                make_float4(__uint_as_float(v[e]) * inv, __uint_as_float(v[e + 1]) * inv,
                            __uint_as_float(v[e + 2]) * inv, __uint_as_float(v[e + 3]) * inv);
        }
      }
      if (row_valid) p.part_lse[prow] = l > 0.f ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
    } else if (!to_partial && have_o) {
      uint16_t* dst = p.out + (qrow * p.Hq + g * G + hh) * D;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(trow + kColO + cc * 32, v);
        tmem_wait_ld();
        if (row_valid) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(v[e]) * inv, __uint_as_float(v[e + 1]) * inv);
            w.y = pack_bf16x2(__uint_as_float(v[e + 2]) * inv, __uint_as_float(v[e + 3]) * inv);
            w.z = pack_bf16x2(__uint_as_float(v[e + 4]) * inv, __uint_as_float(v[e + 5]) * inv);
            w.w = pack_bf16x2(__uint_as_float(v[e + 6]) * inv, __uint_as_float(v[e + 7]) * inv);
            *reinterpret_cast<uint4*>(dst + cc * 32 + e) = w;
          }
        }
      }
    }
  }

  // ---- teardown: every tcgen05 op done before TMEM is released
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    mbar_wait(bar(kFinal), 0);
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, int G, int BN>
__global__ void __launch_bounds__(kThreadsAlone, BN == 64 ? 2 : 1)
    prefill_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                   const __grid_constant__ CUtensorMap vmap, const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // launched as a programmatic dependent (see pdl_wait): nothing global is
  // read before the kernel ahead of it has completed
  pdl_wait();
  pdl_launch_dependents();
  prefill_body<D, G, BN, true, true>(&qmap, &kmap, &vmap, p, blockIdx.x, smem_raw);
}

template <int D>
constexpr size_t smem_bytes() {
  return Layout<D, kKeyTile>::kBytes;  // about half an SM: two CTAs share one
}

}  // namespace prefill
}  // namespace pkv
