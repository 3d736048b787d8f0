// prologue.cuh -- the step before attention, fused into one kernel: the
// separate RMSNorm of each projected Q and K head row (Qwen3's QK norm),
// rotary position encoding of both, and the write of the new K row (and the
// unchanged V row) into the paged pool.
//
// Sources: tiny-llm source reading, week 1 (Qwen3 attention: Q and K each get
// their own RMSNorm after projection, RoPE encodes the position) and week 2
// (Fast RMSNorm, Fast RoPE; "implement or fuse RMSNorm, RoPE ..."); tiny-llm
// blog, week 2 (RMSNorm and RoPE fused into a single kernel to save memory
// round trips); "Paged KV Cache" for the pool write.
//
// RMSNorm of a head row x with weight w: x / sqrt(mean(x^2) + eps) * w.
// RoPE pairs element i with element i + d/2 and turns the pair by the angle
// pos * theta^(-2i/d).  Work is fp32 from the bf16 inputs, rounded once to
// bf16; the angles are formed in fp64 (pos * inv_freq reaches ~1e5 rad at
// long contexts, where an fp32 product is off by ~1e-2 rad).
//
// One CTA per token.  Its first d/2 threads fill a table of the token's
// cos/sin per pair in shared memory; then each warp takes head rows: the Hq
// query rows (normalised, rotated, written to q_out), the Hkv key rows
// (normalised, rotated, written to the pool slot) and the Hkv value rows
// (copied to the pool slot).  Lane l holds elements [l*d/32, (l+1)*d/32); the
// partner of element i sits in lane l ^ 16.
#pragma once

#include "ptx.cuh"

namespace pkv {
namespace prologue {

constexpr int kWarps = 8;

struct Params {
  const uint16_t* q;          // [T][Hq][D]
  const uint16_t* k;          // [T][Hkv][D]
  const uint16_t* v;          // [T][Hkv][D]
  const uint16_t* q_w;        // [D]
  const uint16_t* k_w;        // [D]
  const int32_t* positions;   // [T]
  const int32_t* slots;       // [T]
  uint16_t* q_out;            // [T][Hq][D]
  uint16_t* k_pool;           // [num_pages][Hkv][P][D]
  uint16_t* v_pool;
  int32_t T, Hq, Hkv, P;
  int64_t num_slots;
  float eps;
  double log2_theta;
};

template <int N>
struct Vec;  // N bf16 values as one load
template <>
struct Vec<2> { using T = uint32_t; };
template <>
struct Vec<4> { using T = uint2; };

__device__ __forceinline__ void unpack(uint32_t x, float& a, float& b) {
  a = __uint_as_float(x << 16);
  b = __uint_as_float(x & 0xFFFF0000u);
}

template <int D>
__global__ void __launch_bounds__(kWarps * 32) qk_norm_rope_append_kernel(const Params p) {
  constexpr int EPL = D / 32;  // elements per lane
  using V = typename Vec<EPL>::T;
  __shared__ float cs[D / 2], sn[D / 2];
  // the new rows may come from the kernel ahead (a projection): wait for it
  pdl_wait();
  pdl_launch_dependents();
  const int t = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pos = p.positions[t];
  if (threadIdx.x < D / 2) {
    const int i = threadIdx.x;
    // theta^(-2i/d) and the angle in fp64, then its sine and cosine
    const double inv_freq = exp2(-2.0 * i / D * p.log2_theta);
    double s, c;
    sincos(static_cast<double>(pos) * inv_freq, &s, &c);
    cs[i] = static_cast<float>(c);
    sn[i] = static_cast<float>(s);
  }
  __syncthreads();
  const int32_t slot = p.slots[t];
  const bool write_kv = slot != -1;
  if (write_kv && (slot < 0 || slot >= p.num_slots)) {
    if (threadIdx.x == 0) raise_flag(PKV_FLAG_BAD_SLOT);
  }
  const bool slot_ok = slot >= 0 && slot < p.num_slots;
  const int64_t page = slot_ok ? slot / p.P : 0, off = slot_ok ? slot - page * p.P : 0;
  // this lane's weights and rotation coefficients
  const int i0 = (lane & 15) * EPL;  // pair index of this lane's first element
  const bool second = lane >= 16;    // holds elements i + d/2
  float c[EPL], s[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) {
    c[e] = cs[i0 + e];
    s[e] = second ? sn[i0 + e] : -sn[i0 + e];
  }
  const int rows = p.Hq + 2 * p.Hkv;
  for (int row = warp; row < rows; row += kWarps) {
    if (row >= p.Hq + p.Hkv) {
      // a V row: copied as it is
      if (!slot_ok) continue;
      const int h = row - p.Hq - p.Hkv;
      const V x = *reinterpret_cast<const V*>(p.v + (static_cast<size_t>(t) * p.Hkv + h) * D + lane * EPL);
      *reinterpret_cast<V*>(p.v_pool + ((page * p.Hkv + h) * p.P + off) * D + lane * EPL) = x;
      continue;
    }
    const bool is_q = row < p.Hq;
    if (!is_q && !slot_ok) continue;
    const int h = is_q ? row : row - p.Hq;
    const uint16_t* src = is_q ? p.q + (static_cast<size_t>(t) * p.Hq + h) * D
                               : p.k + (static_cast<size_t>(t) * p.Hkv + h) * D;
    const uint16_t* wsrc = is_q ? p.q_w : p.k_w;
    float x[EPL], w[EPL];
    {
      const V xv = *reinterpret_cast<const V*>(src + lane * EPL);
      const V wv = *reinterpret_cast<const V*>(wsrc + lane * EPL);
      if constexpr (EPL == 4) {
        unpack(xv.x, x[0], x[1]);
        unpack(xv.y, x[2], x[3]);
        unpack(wv.x, w[0], w[1]);
        unpack(wv.y, w[2], w[3]);
      } else {
        unpack(xv, x[0], x[1]);
        unpack(wv, w[0], w[1]);
      }
    }
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) ss = fmaf(x[e], x[e], ss);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv_rms = rsqrtf(ss / D + p.eps);
    float y[EPL], partner[EPL], out[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) y[e] = x[e] * inv_rms * w[e];
#pragma unroll
    for (int e = 0; e < EPL; ++e) partner[e] = __shfl_xor_sync(0xffffffffu, y[e], 16);
    // first of a pair: a cos - b sin; second: b cos + a sin
#pragma unroll
    for (int e = 0; e < EPL; ++e) out[e] = fmaf(y[e], c[e], partner[e] * s[e]);
    uint16_t* dst = is_q ? p.q_out + (static_cast<size_t>(t) * p.Hq + h) * D
                         : p.k_pool + ((page * p.Hkv + h) * p.P + off) * D;
    if constexpr (EPL == 4) {
      *reinterpret_cast<uint2*>(dst + lane * EPL) =
          make_uint2(pack_bf16x2(out[0], out[1]), pack_bf16x2(out[2], out[3]));
    } else {
      *reinterpret_cast<uint32_t*>(dst + lane * EPL) = pack_bf16x2(out[0], out[1]);
    }
  }
}

}  // namespace prologue
}  // namespace pkv
