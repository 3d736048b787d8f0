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
// memory serves all G heads).  Keys stream in tiles of 128 (8 pages of 16, or
// 4 of 32), gathered page by page with TMA into 128-byte-swizzled tiles.
//   S = Q K^T   : M=128, N=128, K=d  -> TMEM (two buffers, double-buffered)
//   softmax     : one thread per TMEM lane (= one query row), log2 domain,
//                 lazy rescale of O only when the running max grows by > 2^8
//   O += P V    : M=128, N=d, K=128; P (bf16) staged in shared memory,
//                 V used as an MN-major operand straight from its tile
// Warp roles: warp 0 TMA producer, warp 1 TMEM owner + MMA issuer (one
// thread), warps 2..5 softmax and epilogue.
#pragma once

#include "ptx.cuh"

namespace pkv {
namespace prefill {

constexpr int kM = 128;  // query rows per CTA
constexpr int kN = 128;  // keys per tile
constexpr int kThreads = 192;
constexpr int kTmemCols = 512;
constexpr int kColS0 = 0, kColS1 = 128, kColO = 256;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale when the max grows by > 256x

struct Params {
  const int32_t* cu_q_lens;    // [B+1]
  const int32_t* ctx_offsets;  // [B]
  const int32_t* page_table;   // [B][max_pages]
  uint16_t* out;               // bf16 [total_q][Hq][D]
  int32_t B, Hq, Hkv, P, max_pages, num_pages, total_q;
  float scale_log2;
};

template <int D>
struct Layout {
  static constexpr int kHalf = kM * 128;            // one 64-column half of a 128-row tile
  static constexpr int kQOff = 0;                   // [D/64][128 rows][128 B]
  static constexpr int kTileBytes = (D / 64) * kHalf;
  static constexpr int kKOff = kQOff + kTileBytes;  // 2 stages
  static constexpr int kVOff = kKOff + 2 * kTileBytes;
  static constexpr int kPOff = kVOff + 2 * kTileBytes;  // [2 halves][128 rows][128 B]
  static constexpr int kBarOff = kPOff + 2 * kHalf;
  // barriers: q, kfull[2], kempty[2], vfull[2], vempty[2], sfull[2], pfull, pvdone, final
  static constexpr int kNumBars = 14;
  static constexpr int kTmemSlotOff = kBarOff + kNumBars * 8;
  static constexpr size_t kBytes = kTmemSlotOff + 16 + 1024;
};

enum Bar { kQ = 0, kKFull = 1, kKEmpty = 3, kVFull = 5, kVEmpty = 7, kSFull = 9, kPFull = 11,
           kPVDone = 12, kFinal = 13 };

template <int D, int G>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                   const __grid_constant__ CUtensorMap vmap, const Params p) {
  using LY = Layout<D>;
  constexpr int QPOS = kM / G;  // chunk positions per tile
  constexpr uint32_t kIdescS = idesc_bf16_f32(kM, kN, false, false);
  constexpr uint32_t kIdescPV = idesc_bf16_f32(kM, D, false, true);

  // ---- which tile: heaviest (last) q-tiles of every request first
  const int r = blockIdx.x % p.B;
  const int rest = blockIdx.x / p.B;
  const int g = rest % p.Hkv;
  const int qt_rev = rest / p.Hkv;
  const int q0 = p.cu_q_lens[r], q1 = p.cu_q_lens[r + 1];
  const int n_r = q1 - q0;
  if (q0 < 0 || n_r < 0 || q1 > p.total_q) {
    if (g == 0 && qt_rev == 0 && threadIdx.x == 0) raise_flag(PKV_FLAG_BAD_QUERY_ROWS);
    return;
  }
  const int n_qt = (n_r + QPOS - 1) / QPOS;
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
  const int nt = (kv_end + kN - 1) / kN;                 // key tiles

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_addr(smem);
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
    }
    mbar_init(bar(kPFull), 128);
    mbar_init(bar(kPVDone), 1);
    mbar_init(bar(kFinal), 1);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(smem_addr(smem + LY::kTmemSlotOff), kTmemCols);
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  const uint32_t sQ = sbase + LY::kQOff;
  auto sK = [&](int b) { return sbase + LY::kKOff + b * LY::kTileBytes; };
  auto sV = [&](int b) { return sbase + LY::kVOff + b * LY::kTileBytes; };
  const uint32_t sP = sbase + LY::kPOff;

  if (warp == 0) {
    // ============================ TMA producer ============================
    const int32_t* ptab = p.page_table + static_cast<size_t>(r) * p.max_pages;
    if (lane == 0) {
      prefetch_tensormap(&qmap);
      prefetch_tensormap(&kmap);
      prefetch_tensormap(&vmap);
      mbar_arrive_expect_tx(bar(kQ), kM * D * 2);
#pragma unroll
      for (int h = 0; h < D / 64; ++h)
        tma_load_3d(sQ + h * LY::kHalf, &qmap, 64 * h, g * G, q0 + qt * QPOS, bar(kQ));
    }
    bool ok = true;
    for (int j = 0; j < nt && ok; ++j) {
      const int b = j & 1;
      const int key0 = j * kN;
      const int nkeys = min(kN, kv_end - key0);
      const int npg = (nkeys + p.P - 1) / p.P;
      const int pid = lane < npg ? __ldg(ptab + key0 / p.P + lane) : -1;
      if (j >= 2) {
        ok = mbar_wait(bar(kKEmpty + b), ((j >> 1) - 1) & 1);
        if (ok) ok = mbar_wait(bar(kVEmpty + b), ((j >> 1) - 1) & 1);
        if (!ok) break;
      }
      if (lane == 0) {
        mbar_arrive_expect_tx(bar(kKFull + b), static_cast<uint32_t>(npg * p.P * D * 2));
      }
      for (int pi = 0; pi < npg; ++pi) {
        const int page = __shfl_sync(0xffffffffu, pid, pi);
        if (lane == 0) {
          if (static_cast<unsigned>(page) >= static_cast<unsigned>(p.num_pages)) raise_flag(PKV_FLAG_BAD_PAGE);
          const int row = page * p.Hkv + g;
#pragma unroll
          for (int h = 0; h < D / 64; ++h)
            tma_load_3d(sK(b) + h * LY::kHalf + pi * p.P * 128, &kmap, 64 * h, 0, row, bar(kKFull + b));
        }
      }
      if (lane == 0) {
        mbar_arrive_expect_tx(bar(kVFull + b), static_cast<uint32_t>(npg * p.P * D * 2));
      }
      for (int pi = 0; pi < npg; ++pi) {
        const int page = __shfl_sync(0xffffffffu, pid, pi);
        if (lane == 0) {
          const int row = page * p.Hkv + g;
#pragma unroll
          for (int h = 0; h < D / 64; ++h)
            tma_load_3d(sV(b) + h * LY::kHalf + pi * p.P * 128, &vmap, 64 * h, 0, row, bar(kVFull + b));
        }
      }
      __syncwarp();
    }
  } else if (warp == 1) {
    // ============================ MMA issuer =============================
    bool ok = mbar_wait(bar(kQ), 0);
    auto issue_pv = [&](int i) -> bool {
      const int b = i & 1;
      if (!mbar_wait(bar(kPFull), i & 1)) return false;
      if (!mbar_wait(bar(kVFull + b), (i >> 1) & 1)) return false;
      tc_fence_after_sync();
      if (lane == 0) {
#pragma unroll
        for (int ks = 0; ks < kN / 16; ++ks) {
          const uint64_t a = smem_desc_sw128(sP + (ks >> 2) * LY::kHalf + (ks & 3) * 32, 16, 1024);
          const uint64_t bdesc = smem_desc_sw128(sV(b) + ks * 16 * 128, LY::kHalf, 1024);
          tc_mma_ss(tmem + kColO, a, bdesc, kIdescPV, i > 0 || ks > 0);
        }
        tc_commit(bar(kPVDone));
        tc_commit(bar(kVEmpty + b));
      }
      __syncwarp();
      return true;
    };
    for (int j = 0; j < nt && ok; ++j) {
      const int b = j & 1;
      ok = mbar_wait(bar(kKFull + b), (j >> 1) & 1);
      if (!ok) break;
      tc_fence_after_sync();
      if (lane == 0) {
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t a = smem_desc_sw128(sQ + (ks >> 2) * LY::kHalf + (ks & 3) * 32, 16, 1024);
          const uint64_t bdesc = smem_desc_sw128(sK(b) + (ks >> 2) * LY::kHalf + (ks & 3) * 32, 16, 1024);
          tc_mma_ss(tmem + (b ? kColS1 : kColS0), a, bdesc, kIdescS, ks > 0);
        }
        tc_commit(bar(kSFull + b));
        tc_commit(bar(kKEmpty + b));
      }
      __syncwarp();
      if (j >= 1) ok = issue_pv(j - 1);
    }
    if (ok && nt >= 1) ok = issue_pv(nt - 1);
    if (lane == 0) tc_commit(bar(kFinal));
    __syncwarp();
  } else {
    // ========================= softmax / epilogue ========================
    const int quad = warp & 3;             // TMEM lane quadrant this warp may access
    const int row = quad * 32 + lane;      // query row of this thread
    const int pos_local = row / G, hh = row % G;
    const int qpos = pos_lo + pos_local;   // absolute position
    const bool row_valid = pos_local < rows_valid;
    const uint32_t trow = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const float sl2 = p.scale_log2;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nt; ++j) {
      const int b = j & 1;
      if (!mbar_wait(bar(kSFull + b), (j >> 1) & 1)) { ok = false; break; }
      tc_fence_after_sync();
      float s[kN];
      {
        uint32_t v[kN / 32][32];
#pragma unroll
        for (int cc = 0; cc < kN / 32; ++cc) tmem_ld_32x32b_x32(trow + (b ? kColS1 : kColS0) + cc * 32, v[cc]);
        tmem_wait_ld();
#pragma unroll
        for (int cc = 0; cc < kN / 32; ++cc)
#pragma unroll
          for (int e = 0; e < 32; ++e) s[cc * 32 + e] = __uint_as_float(v[cc][e]) * sl2;
      }
      const int key0 = j * kN;
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
      const float mc = fmaxf(m, mx);
      const bool need = mc > m + kRescaleThreshold;
      float alpha = 1.f;
      if (need) {
        alpha = fast_exp2(m - mc);
        m = mc;
      }
      uint32_t pk[kN / 2];
      float rowsum = 0.f;
#pragma unroll
      for (int e = 0; e < kN; e += 2) {
        const float a0 = fast_exp2(s[e] - m), a1 = fast_exp2(s[e + 1] - m);
        rowsum += a0 + a1;
        pk[e / 2] = pack_bf16x2(a0, a1);
      }
      l = fmaf(l, alpha, rowsum);
      if (j >= 1) {
        // PV of the previous tile must be done: P is single-buffered and O
        // may need rescaling.
        if (!mbar_wait(bar(kPVDone), (j - 1) & 1)) { ok = false; break; }
        tc_fence_after_sync();
        if (__any_sync(0xffffffffu, need)) {
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
      // P row -> shared memory, 128-byte swizzle (K-major A operand)
      uint8_t* prow = smem + LY::kPOff + row * 128;
#pragma unroll
      for (int ch = 0; ch < kN / 8; ++ch) {
        const int half = ch >> 3, c16 = ch & 7;
        *reinterpret_cast<uint4*>(prow + half * LY::kHalf + ((c16 ^ (row & 7)) << 4)) =
            make_uint4(pk[ch * 4], pk[ch * 4 + 1], pk[ch * 4 + 2], pk[ch * 4 + 3]);
      }
      if (key0 + kN > kv_end) {
        // ragged last tile: V rows past kv_end were not loaded (or hold
        // unused slots); zero them so 0 * garbage cannot reach O
        if (!mbar_wait(bar(kVFull + b), (j >> 1) & 1)) { ok = false; break; }
        const int first = kv_end - key0;
        const int nbytes = (kN - first) * 128;
        for (int h = 0; h < D / 64; ++h) {
          uint8_t* vz = smem + LY::kVOff + b * LY::kTileBytes + h * LY::kHalf + first * 128;
          for (int off = (row) * 16; off < nbytes; off += kM * 16)
            *reinterpret_cast<uint4*>(vz + off) = make_uint4(0, 0, 0, 0);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before_sync();
      mbar_arrive(bar(kPFull));
    }
    if (ok && nt >= 1 && mbar_wait(bar(kPVDone), (nt - 1) & 1)) {
      tc_fence_after_sync();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      uint16_t* dst = p.out + (static_cast<size_t>(q0 + qt * QPOS + pos_local) * p.Hq + g * G + hh) * D;
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

}  // namespace prefill
}  // namespace pkv
