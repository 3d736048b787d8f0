// pkv_api.cu -- the C ABI declared in include/pkv.h: argument checks on the
// host, TMA tensor maps, kernel selection by (head_dim, group size), and
// launches.  The library allocates nothing and never synchronises the device
// (pkv_device_error_flags excepted, as documented).
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>
#include <unordered_map>

#include "cow.cuh"
#include "decode.cuh"
#include "kv_append.cuh"
#include "mixed.cuh"
#include "prefill.cuh"
#include "prologue.cuh"

namespace {


struct DeviceInfo {
  int sm_count = 0;
  int major = 0, minor = 0;
  bool valid = false;
};

constexpr int kMaxDevices = 64;
DeviceInfo g_devices[kMaxDevices];
std::mutex g_mutex;

int current_device(DeviceInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PKV_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceInfo& d = g_devices[dev];
  if (!d.valid) {
    if (cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return PKV_ERR_CUDA;
    d.valid = true;
  }
  *out = d;
  return (d.major == 10 && d.minor == 0) ? PKV_OK : PKV_ERR_DEVICE;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 3-D bf16 tensor map: dims[0] innermost (elements), strides in bytes of
// dims 1 and 2.
int make_map(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
             uint64_t stride1, uint64_t stride2, uint32_t b0, uint32_t b1, uint32_t b2,
             bool swizzle128) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return PKV_ERR_TENSOR_MAP;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {stride1, stride2};
  const cuuint32_t box[3] = {b0, b1, b2};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PKV_OK : PKV_ERR_TENSOR_MAP;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_pool(const pkv_pool_desc& pool) {
  if (pool.num_pages <= 0 || pool.num_kv_heads <= 0) return PKV_ERR_BAD_SHAPE;
  if (pool.head_dim != 64 && pool.head_dim != 128) return PKV_ERR_UNSUPPORTED;
  if (pool.page_size != 16 && pool.page_size != 32) return PKV_ERR_UNSUPPORTED;
  // TMA row coordinate is page * Hkv + head, an int32
  if (static_cast<long long>(pool.num_pages) * pool.num_kv_heads >= (1ll << 31)) return PKV_ERR_BAD_SHAPE;
  return PKV_OK;
}

int check_heads(int32_t num_q_heads, const pkv_pool_desc& pool, int* group) {
  if (num_q_heads <= 0 || num_q_heads % pool.num_kv_heads != 0) return PKV_ERR_BAD_SHAPE;
  const int g = num_q_heads / pool.num_kv_heads;
  if (g != 1 && g != 2 && g != 4 && g != 8) return PKV_ERR_UNSUPPORTED;
  *group = g;
  return PKV_OK;
}

int launch_status() { return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA; }

// Launch as a programmatic dependent of the previous kernel on the stream:
// the kernel starts early and waits (pdl_wait) before its first global read,
// so its launch latency overlaps the tail of the kernel ahead of it.
template <typename... KArgs, typename... Args>
int launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
               Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) != cudaSuccess) return PKV_ERR_CUDA;
  return launch_status();
}

// warps per combine CTA: about one per eight splits, a power of two in [1, 8]
int combine_warps(int32_t max_splits) {
  int w = 1;
  while (w < pkv::decode::kCombineMaxWarps && w * 8 < max_splits) w <<= 1;
  return w;
}

// after_decode: the combine follows the partition kernel on the stream and is
// launched as its programmatic dependent (the partition kernel signals at its
// start, the combine waits for the partition grid's completion before its
// first read), so the combine's launch overlaps the partition kernel instead
// of following its last CTA.
template <int D>
int launch_combine(const float* part_o, const float* part_lse, const int32_t* num_splits, int32_t B,
                   int32_t Hq, int32_t S, uint16_t* out, float* out_lse,
                   int skip_below, bool after_decode, cudaStream_t stream) {
  const long long rows = static_cast<long long>(B) * Hq;
  if (rows > 0x7FFFFFFFll) return PKV_ERR_BAD_SHAPE;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(rows));
  cfg.blockDim = dim3(32 * combine_warps(S));
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = after_decode ? 1 : 0;
  if (cudaLaunchKernelEx(&cfg, pkv::decode::combine_kernel<D>, part_o, part_lse, num_splits, Hq, S,
                         out, out_lse, skip_below) != cudaSuccess)
    return PKV_ERR_CUDA;
  return launch_status();
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Partial slots per (request, query head): a fixed partition gives
// ceil(len / partition) splits; the automatic split gives a group of padded
// length Lp at most ceil(Lp / kMinShare) + 1 (slices are >= kMinShare tokens,
// and the group's first and last slice may be partial).
int32_t max_splits_for(int32_t max_kv_len, int32_t partition_tokens) {
  if (partition_tokens < 0) return 1;
  const int32_t len = std::max<int32_t>(max_kv_len, 1);
  if (partition_tokens == 0) return (len + pkv::decode::kMinShare - 1) / pkv::decode::kMinShare + 1;
  return (len + partition_tokens - 1) / partition_tokens;
}

// Partial slots per (request, query head) row and merge-tree counters per
// (request, KV head): the automatic split keeps its pieces and the inner
// levels of the merge tree in the row; a fixed partition keeps its splits.
struct SplitSlots {
  int32_t slots = 1, nodes = 0;
};

SplitSlots split_slots(int32_t max_kv_len, int32_t partition_tokens, int32_t head_dim) {
  SplitSlots ss;
  const int32_t pieces = max_splits_for(max_kv_len, partition_tokens);
  const int fan_in = head_dim == 64 ? pkv::decode::kMergeFanIn<64> : pkv::decode::kMergeFanIn<128>;
  ss.slots = partition_tokens == 0 ? pkv::decode::merge_tree_slots(pieces, fan_in) : pieces;
  ss.nodes = partition_tokens == 0 ? pkv::decode::merge_tree_nodes(pieces, fan_in) : 0;
  return ss;
}

// Workspace: [counters | group_done | num_splits | part_lse | part_o].  The
// first two regions must be zero before the first call; every call that
// completes leaves them zero (zero_bytes covers them).
struct WorkspaceLayout {
  size_t counters = 0, group_done = 0, num_splits = 0, part_lse = 0, part_o = 0, total = 0, zero_bytes = 0;
};

WorkspaceLayout workspace_layout(int32_t B, int32_t Hq, int32_t D, SplitSlots ss) {
  WorkspaceLayout w;
  const size_t groups = static_cast<size_t>(B) * Hq;  // Hq bounds the KV heads
  const int32_t S = ss.slots;
  w.counters = 0;
  w.group_done = 256;
  w.num_splits = w.group_done + align256(groups * std::max<int32_t>(ss.nodes, 1) * 4);
  w.zero_bytes = w.num_splits;
  w.part_lse = w.num_splits + align256(static_cast<size_t>(B) * 4);
  w.part_o = w.part_lse + align256(static_cast<size_t>(B) * Hq * S * 4);
  w.total = w.part_o + align256(static_cast<size_t>(B) * Hq * S * D * 4);
  return w;
}

// Leading bytes of each workspace known to be zero when its last call ended
// (the counters of that call's layout; calls that complete leave them zero).
// A call whose counters reach further -- a larger batch moves the later
// regions, whose old contents then sit where the new counters go -- first
// clears the difference on its stream.  Keyed by workspace address; an
// address seen for the first time is cleared over its whole counter region.
std::unordered_map<const void*, size_t> g_ws_zero;
constexpr size_t kMaxTrackedWorkspaces = 4096;

int prepare_workspace(void* ws, size_t need, cudaStream_t stream) {
  std::lock_guard<std::mutex> lock(g_mutex);
  auto it = g_ws_zero.find(ws);
  const size_t have = it == g_ws_zero.end() ? 0 : it->second;
  if (need > have &&
      cudaMemsetAsync(static_cast<uint8_t*>(ws) + have, 0, need - have, stream) != cudaSuccess)
    return PKV_ERR_CUDA;
  if (it == g_ws_zero.end() && g_ws_zero.size() >= kMaxTrackedWorkspaces) g_ws_zero.clear();
  g_ws_zero[ws] = need;
  return PKV_OK;
}

// Record that the first `bytes` of workspace ws are zero (the caller has
// just cleared them on the stream the next call uses).
void mark_workspace_zero(void* ws, size_t bytes) {
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_ws_zero.find(ws) == g_ws_zero.end() && g_ws_zero.size() >= kMaxTrackedWorkspaces) g_ws_zero.clear();
  g_ws_zero[ws] = bytes;
}

// ------------------------------------------------------------ decode launch
template <int D, int G>
int launch_decode(const pkv::decode::Params& prm, int sm_count, cudaStream_t stream) {
#ifndef PKV_DECODE_NS128
#define PKV_DECODE_NS128 2
#endif
#ifndef PKV_DECODE_NS64
#define PKV_DECODE_NS64 2
#endif
#ifndef PKV_DECODE_MAXW128
#define PKV_DECODE_MAXW128 12
#endif
#ifndef PKV_DECODE_MAXW64
#define PKV_DECODE_MAXW64 12
#endif
  constexpr int NS = D == 128 ? PKV_DECODE_NS128 : PKV_DECODE_NS64;        // stages per warp
  // warps per CTA; at G=8 the query and output registers double, so fewer
  // warps keep every thread's registers unspilled
  constexpr int kMaxWD = D == 128 ? PKV_DECODE_MAXW128 : PKV_DECODE_MAXW64;
  constexpr int kMaxW = G == 8 ? (kMaxWD < 8 ? kMaxWD : 8) : kMaxWD;
  using LY = pkv::decode::Layout<D, G, NS>;
  // with the step's new rows: the instantiation that appends them
  auto kernel = prm.k_new != nullptr ? pkv::decode::partition_kernel<D, G, NS, kMaxW, true>
                                     : pkv::decode::partition_kernel<D, G, NS, kMaxW, false>;
  constexpr size_t kBudget = 227 * 1024;
  const size_t fixed = LY::bytes(0, prm.B);
  if (fixed + LY::kWarpBytes > kBudget) return PKV_ERR_BAD_SHAPE;  // batch too large for the plan
  const int W = static_cast<int>(std::min<size_t>(kMaxW, (kBudget - fixed) / LY::kWarpBytes));
  const size_t smem = LY::bytes(W, prm.B);
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return PKV_ERR_CUDA;
  if (launch_pdl(kernel, dim3(sm_count), dim3(W * 32), smem, stream, prm) != PKV_OK) return PKV_ERR_CUDA;
  if (prm.partition < 0) return PKV_OK;  // every request is one split
  if (prm.partition == 0) return PKV_OK;  // automatic split: merged by the partition kernel's tree
  return launch_combine<D>(prm.part_o, prm.part_lse, prm.num_splits, prm.B, prm.Hq, prm.S_max,
                           prm.out, prm.out_lse, 1, true, stream);
}

template <int D>
int dispatch_decode_group(int group, const pkv::decode::Params& prm, int sm_count, cudaStream_t stream) {
  switch (group) {
    case 1: return launch_decode<D, 1>(prm, sm_count, stream);
    case 2: return launch_decode<D, 2>(prm, sm_count, stream);
    case 4: return launch_decode<D, 4>(prm, sm_count, stream);
    case 8: return launch_decode<D, 8>(prm, sm_count, stream);
  }
  return PKV_ERR_UNSUPPORTED;
}

// ----------------------------------------------------------- prefill launch
template <int D, int G>
int launch_prefill(const pkv::prefill::Params& prm, const CUtensorMap& qmap, const CUtensorMap& kmap,
                   const CUtensorMap& vmap, int32_t max_q_len, cudaStream_t stream) {
  auto kernel = pkv::prefill::prefill_kernel<D, G, pkv::prefill::kKeyTile>;
  const size_t smem = pkv::prefill::smem_bytes<D>();
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return PKV_ERR_CUDA;
  constexpr int QPOS = pkv::prefill::kRowsPerCta / G;  // chunk positions per CTA
  const long long tiles = (static_cast<long long>(max_q_len) + QPOS - 1) / QPOS;
  const long long blocks = tiles * prm.Hkv * prm.B * prm.splits;
  if (blocks == 0) return PKV_OK;
  if (blocks > 0x7FFFFFFFll) return PKV_ERR_BAD_SHAPE;
  pkv::prefill::Params args = prm;
  args.qtiles = static_cast<int32_t>(tiles);
  return launch_pdl(kernel, dim3(static_cast<unsigned>(blocks)), dim3(pkv::prefill::kThreadsAlone), smem, stream, qmap,
                    kmap, vmap, args);
}

template <int D>
int dispatch_prefill_group(int group, const pkv::prefill::Params& prm, const CUtensorMap& qmap,
                           const CUtensorMap& kmap, const CUtensorMap& vmap, int32_t max_q_len,
                           cudaStream_t stream) {
  switch (group) {
    case 1: return launch_prefill<D, 1>(prm, qmap, kmap, vmap, max_q_len, stream);
    case 2: return launch_prefill<D, 2>(prm, qmap, kmap, vmap, max_q_len, stream);
    case 4: return launch_prefill<D, 4>(prm, qmap, kmap, vmap, max_q_len, stream);
    case 8: return launch_prefill<D, 8>(prm, qmap, kmap, vmap, max_q_len, stream);
  }
  return PKV_ERR_UNSUPPORTED;
}

// Split-K chunk attention (short chunks over long contexts).  The workspace
// size depends on the longest context and the partition only, so it can be
// computed without device data.
constexpr int kPrefillBN = pkv::prefill::kKeyTile;

// The smallest partition the automatic choice takes: the workspace of an
// automatic call is sized for it.
constexpr int32_t kVerifyMinPartition = 512;

int32_t round_up_tile(long long keys) {
  return static_cast<int32_t>((std::max<long long>(keys, 1) + kPrefillBN - 1) / kPrefillBN * kPrefillBN);
}

// Keys per split of a verify call.  Automatic: no split while the (request,
// KV head, query tile) units already give every CTA slot of the GPU (two per
// SM) its own unit -- splitting then only adds partial writes and CTA start-up
// per split -- else enough splits of the longest request to fill the slots,
// none shorter than kVerifyMinPartition keys.
int32_t verify_partition(int32_t max_kv_len, int32_t partition_tokens, long long units, long long slots) {
  if (partition_tokens > 0) return partition_tokens;
  const int32_t whole = round_up_tile(max_kv_len);
  if (units >= slots) return whole;
  const long long splits = (slots + std::max<long long>(units, 1) - 1) / std::max<long long>(units, 1);
  const int32_t part = round_up_tile((static_cast<long long>(max_kv_len) + splits - 1) / splits);
  return std::min(whole, std::max(kVerifyMinPartition, part));
}

struct VerifyLayout {
  int32_t partition = 0, splits = 1;
  size_t num_splits = 0, part_lse = 0, part_o = 0, total = 0;
};

// The workspace layout for splits of `partition` keys (> 0).
VerifyLayout verify_layout(int32_t total_q, int32_t Hq, int32_t D, int32_t max_kv_len, int32_t partition) {
  VerifyLayout v;
  v.partition = partition;
  v.splits = std::max<int32_t>(1, (max_kv_len + v.partition - 1) / v.partition);
  const size_t rows = static_cast<size_t>(total_q) * Hq;
  v.num_splits = 0;
  v.part_lse = align256(static_cast<size_t>(total_q) * 4);
  v.part_o = v.part_lse + align256(rows * v.splits * 4);
  v.total = v.part_o + align256(rows * v.splits * D * 4);
  return v;
}

// A checked chunk launch: the kernel's parameters, the three tensor maps and
// the GQA group.
struct PrefillLaunch {
  pkv::prefill::Params prm;
  CUtensorMap qmap, kmap, vmap;
  int group = 0;
};

// Host-side checks of a chunk call and its parameters (no split).  Returns
// PKV_OK, kNothingToDo for an empty call (after the shape checks), or an
// error status.
constexpr int kNothingToDo = 1;

int build_prefill(const void* q, const int32_t* cu_q_lens, int32_t batch, int32_t num_q_heads, int32_t total_q,
                  int32_t max_q_len, const int32_t* ctx_offsets, const void* k_pool, const void* v_pool,
                  const pkv_pool_desc& pool, const int32_t* page_table, int32_t max_pages, float scale, void* out,
                  PrefillLaunch* pl) {
  if (batch < 0 || total_q < 0 || max_q_len < 0 || max_pages <= 0) return PKV_ERR_BAD_SHAPE;
  int st = check_pool(pool);
  if (st != PKV_OK) return st;
  if ((st = check_heads(num_q_heads, pool, &pl->group)) != PKV_OK) return st;
  if (!std::isfinite(scale) || !(scale > 0.f)) return PKV_ERR_BAD_SHAPE;
  if (static_cast<long long>(max_pages) * pool.page_size > (1ll << 30)) return PKV_ERR_BAD_SHAPE;
  if (batch == 0 || total_q == 0 || max_q_len == 0) return kNothingToDo;
  if (!q || !cu_q_lens || !ctx_offsets || !k_pool || !v_pool || !page_table || !out)
    return PKV_ERR_NULL_POINTER;
  if (!aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(out))
    return PKV_ERR_MISALIGNED;
  const int qpos = pkv::prefill::kRowsPerCta / pl->group;
  pkv::prefill::Params& prm = pl->prm;
  prm.cu_q_lens = cu_q_lens;
  prm.ctx_offsets = ctx_offsets;
  prm.page_table = page_table;
  prm.out = static_cast<uint16_t*>(out);
  prm.B = batch;
  prm.Hq = num_q_heads;
  prm.Hkv = pool.num_kv_heads;
  prm.P = pool.page_size;
  prm.max_pages = max_pages;
  prm.num_pages = pool.num_pages;
  prm.total_q = total_q;
  prm.qtiles = static_cast<int32_t>((static_cast<long long>(max_q_len) + qpos - 1) / qpos);
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.partition = 0;
  prm.splits = 1;
  prm.part_o = nullptr;
  prm.part_lse = nullptr;
  prm.num_splits = nullptr;
  return PKV_OK;
}

// The TMA maps of a checked chunk launch (after every argument check: the
// driver's encoder is the first call that can fail for reasons of its own).
int make_prefill_maps(const void* q, const void* k_pool, const void* v_pool, const pkv_pool_desc& pool,
                      int32_t num_q_heads, int32_t total_q, PrefillLaunch* pl) {
  const int D = pool.head_dim;
  const uint64_t rows = static_cast<uint64_t>(pool.num_pages) * pool.num_kv_heads;
  const int qpos = pkv::prefill::kRowsPerCta / pl->group;
  int st;
  if ((st = make_map(&pl->qmap, q, D, num_q_heads, total_q, D * 2ull, static_cast<uint64_t>(num_q_heads) * D * 2,
                     64, pl->group, qpos, true)) != PKV_OK)
    return st;
  if ((st = make_map(&pl->kmap, k_pool, D, pool.page_size, rows, D * 2ull, pool.page_size * D * 2ull, 64,
                     pool.page_size, 1, true)) != PKV_OK)
    return st;
  return make_map(&pl->vmap, v_pool, D, pool.page_size, rows, D * 2ull, pool.page_size * D * 2ull, 64,
                  pool.page_size, 1, true);
}

// Chunked prefill (split_tokens = 0) or its split-K form (split_tokens =
// the partition, -1 = automatic; workspace as verify_layout).
int run_prefill(const void* q, const int32_t* cu_q_lens, int32_t batch, int32_t num_q_heads, int32_t total_q,
                int32_t max_q_len, const int32_t* ctx_offsets, const void* k_pool, const void* v_pool,
                const pkv_pool_desc& pool, const int32_t* page_table, int32_t max_pages, float scale,
                int32_t split_tokens, void* workspace, size_t workspace_bytes, void* out, cudaStream_t s) {
  PrefillLaunch pl;
  int st = build_prefill(q, cu_q_lens, batch, num_q_heads, total_q, max_q_len, ctx_offsets, k_pool, v_pool, pool,
                         page_table, max_pages, scale, out, &pl);
  if (st == kNothingToDo) return PKV_OK;
  if (st != PKV_OK) return st;
  VerifyLayout vl;
  if (split_tokens != 0) {
    // the workspace an automatic call needs is sized for its smallest partition
    const int32_t max_kv = max_pages * pool.page_size;
    const VerifyLayout worst = verify_layout(total_q, num_q_heads, pool.head_dim, max_kv,
                                             split_tokens < 0 ? std::min(kVerifyMinPartition, round_up_tile(max_kv))
                                                              : split_tokens);
    if (workspace == nullptr || workspace_bytes < worst.total) return PKV_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return PKV_ERR_MISALIGNED;
  }
  DeviceInfo dev;
  if ((st = current_device(&dev)) != PKV_OK) return st;
  if (split_tokens != 0) {
    const long long units = static_cast<long long>(pl.prm.qtiles) * pool.num_kv_heads * batch;
    vl = verify_layout(total_q, num_q_heads, pool.head_dim, max_pages * pool.page_size,
                       verify_partition(max_pages * pool.page_size, split_tokens < 0 ? 0 : split_tokens, units,
                                        2ll * dev.sm_count));
  }
  if ((st = make_prefill_maps(q, k_pool, v_pool, pool, num_q_heads, total_q, &pl)) != PKV_OK) return st;
  const int D = pool.head_dim;
  pkv::prefill::Params& prm = pl.prm;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (split_tokens != 0) {
    prm.partition = vl.partition;
    prm.splits = vl.splits;
    prm.num_splits = reinterpret_cast<int32_t*>(ws + vl.num_splits);
    prm.part_lse = reinterpret_cast<float*>(ws + vl.part_lse);
    prm.part_o = reinterpret_cast<float*>(ws + vl.part_o);
    // rows the kernel does not reach (past cu_q_lens[batch]) must read as
    // "one split" to the combine, which then leaves them alone
    if (cudaMemsetAsync(prm.num_splits, 0, static_cast<size_t>(total_q) * 4, s) != cudaSuccess) return PKV_ERR_CUDA;
  }
  st = D == 128 ? dispatch_prefill_group<128>(pl.group, prm, pl.qmap, pl.kmap, pl.vmap, max_q_len, s)
                : dispatch_prefill_group<64>(pl.group, prm, pl.qmap, pl.kmap, pl.vmap, max_q_len, s);
  if (st != PKV_OK || split_tokens == 0 || prm.splits == 1) return st;
  // merge the rows whose request was split (rows of single-split requests
  // were written by the kernel itself; with one split for every request
  // there is nothing to merge and no combine launch)
  if (D == 128)
    return launch_combine<128>(prm.part_o, prm.part_lse, prm.num_splits, total_q, num_q_heads, prm.splits,
                               prm.out, nullptr, 1, true, s);
  return launch_combine<64>(prm.part_o, prm.part_lse, prm.num_splits, total_q, num_q_heads, prm.splits,
                            prm.out, nullptr, 1, true, s);
}

// Host-side checks shared by both decode entry points, and the split and
// workspace layout the call implies.  Returns PKV_OK for an empty batch
// before the pointer checks (nothing will be launched).
struct DecodePlan {
  int group = 0;
  SplitSlots ss;
  WorkspaceLayout wl;
};

int check_decode(const void* q, int32_t batch, int32_t num_q_heads, const void* k_pool, const void* v_pool,
                 const pkv_pool_desc& pool, const int32_t* page_table, int32_t max_pages,
                 const int32_t* kv_lens, float scale, int32_t partition_tokens, const void* out,
                 DecodePlan* dp) {
  if (batch < 0 || max_pages <= 0) return PKV_ERR_BAD_SHAPE;
  int st = check_pool(pool);
  if (st != PKV_OK) return st;
  if ((st = check_heads(num_q_heads, pool, &dp->group)) != PKV_OK) return st;
  if (partition_tokens > 0 &&
      (partition_tokens % pkv::decode::kPartitionQuantum != 0 || partition_tokens > 65536))
    return PKV_ERR_BAD_SHAPE;
  if (partition_tokens < -1) return PKV_ERR_BAD_SHAPE;
  if (static_cast<long long>(max_pages) * pool.page_size > (1ll << 30)) return PKV_ERR_BAD_SHAPE;
  if (!std::isfinite(scale)) return PKV_ERR_BAD_SHAPE;
  const int32_t max_kv = max_pages * pool.page_size;
  // the automatic split counts the batch's token-heads in 32-token quanta (int32)
  if (partition_tokens == 0 &&
      static_cast<long long>(batch) * pool.num_kv_heads * (max_kv / pkv::decode::kPartitionQuantum + 1) >=
          (1ll << 31))
    return PKV_ERR_BAD_SHAPE;
  dp->ss = split_slots(max_kv, partition_tokens, pool.head_dim);
  dp->wl = workspace_layout(batch, num_q_heads, pool.head_dim, dp->ss);
  if (batch == 0) return PKV_OK;
  if (!q || !k_pool || !v_pool || !page_table || !kv_lens || !out) return PKV_ERR_NULL_POINTER;
  if (!aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(out))
    return PKV_ERR_MISALIGNED;
  return PKV_OK;
}

// The decode kernel's parameters for a checked call on workspace ws (at
// least dp.wl.total bytes, 256-byte aligned).
pkv::decode::Params fill_decode(const void* q, int32_t batch, int32_t num_q_heads, const void* k_pool,
                                const void* v_pool, const pkv_pool_desc& pool, const int32_t* page_table,
                                int32_t max_pages, const int32_t* kv_lens, float scale, int32_t partition_tokens,
                                const DecodePlan& dp, void* workspace, void* out, float* out_lse, uint32_t flags) {
  const WorkspaceLayout& wl = dp.wl;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  pkv::decode::Params prm;
  prm.q = static_cast<const uint16_t*>(q);
  prm.k_pool = static_cast<const uint16_t*>(k_pool);
  prm.v_pool = static_cast<const uint16_t*>(v_pool);
  prm.page_table = page_table;
  prm.kv_lens = kv_lens;
  prm.out = static_cast<uint16_t*>(out);
  prm.out_lse = out_lse;
  prm.part_o = reinterpret_cast<float*>(ws + wl.part_o);
  prm.part_lse = reinterpret_cast<float*>(ws + wl.part_lse);
  prm.num_splits = reinterpret_cast<int32_t*>(ws + wl.num_splits);
  prm.counters = reinterpret_cast<uint32_t*>(ws + wl.counters);
  prm.group_done = reinterpret_cast<uint32_t*>(ws + wl.group_done);
  prm.B = batch;
  prm.Hq = num_q_heads;
  prm.Hkv = pool.num_kv_heads;
  prm.P = pool.page_size;
  prm.max_pages = max_pages;
  prm.num_pages = pool.num_pages;
  prm.S_max = dp.ss.slots;
  prm.partition = partition_tokens;
  prm.merge_nodes = dp.ss.nodes;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.meta_ready = (flags & PKV_DECODE_METADATA_READY) ? 1 : 0;
  prm.k_new = nullptr;
  prm.v_new = nullptr;
  return prm;
}

// Launch a checked decode call on workspace ws (at least dp.wl.total bytes,
// 256-byte aligned); k_new / v_new: the step's new rows to append and attend
// to (one per request), or null.
int run_decode(const void* q, int32_t batch, int32_t num_q_heads, const void* k_pool, const void* v_pool,
               const pkv_pool_desc& pool, const int32_t* page_table, int32_t max_pages,
               const int32_t* kv_lens, float scale, int32_t partition_tokens, const DecodePlan& dp,
               void* workspace, void* out, float* out_lse, uint32_t flags, cudaStream_t s,
               const void* k_new = nullptr, const void* v_new = nullptr) {
  DeviceInfo dev;
  int st;
  if ((st = current_device(&dev)) != PKV_OK) return st;
  pkv::decode::Params prm = fill_decode(q, batch, num_q_heads, k_pool, v_pool, pool, page_table, max_pages, kv_lens,
                                        scale, partition_tokens, dp, workspace, out, out_lse, flags);
  prm.k_new = static_cast<const uint16_t*>(k_new);
  prm.v_new = static_cast<const uint16_t*>(v_new);
  if ((st = prepare_workspace(workspace, dp.wl.zero_bytes, s)) != PKV_OK) return st;
  if (pool.head_dim == 128) return dispatch_decode_group<128>(dp.group, prm, dev.sm_count, s);
  return dispatch_decode_group<64>(dp.group, prm, dev.sm_count, s);
}

// One persistent launch of a mixed batch (chunks and decode requests):
// returns kNothingToDo when this group size or shared-memory footprint does
// not allow two CTAs per SM, and the caller runs the two kernels instead.
template <int D, int G>
int launch_mixed(const PrefillLaunch& pl, const pkv::decode::Params& dprm, uint32_t* queue, int sm_count,
                 cudaStream_t s) {
  if constexpr (G > 4) {
    return kNothingToDo;  // the decode body at G = 8 needs more registers than two CTAs per SM leave
  } else {
    using DL = pkv::decode::Layout<D, G, 2>;
    const size_t smem = std::max<size_t>(pkv::prefill::smem_bytes<D>(), DL::bytes(pkv::mixed::kDecodeWarps, dprm.B));
    auto kernel = pkv::mixed::mixed_kernel<D, G>;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
        cudaSuccess)
      return PKV_ERR_CUDA;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, pkv::prefill::kThreads, smem) != cudaSuccess)
      return PKV_ERR_CUDA;
    if (per_sm < 2) return kNothingToDo;
    pkv::mixed::Params mp;
    mp.pre = pl.prm;
    mp.dec = dprm;
    const long long units = static_cast<long long>(pl.prm.qtiles) * pl.prm.Hkv * pl.prm.B;
    if (units > 0x3FFFFFFFll) return PKV_ERR_BAD_SHAPE;
    mp.pre_units = static_cast<int32_t>(units);
    mp.dec_units = 2 * sm_count;
    mp.queue = queue;
    return launch_pdl(kernel, dim3(2 * sm_count), dim3(pkv::prefill::kThreads), smem, s, pl.qmap, pl.kmap, pl.vmap,
                      mp);
  }
}

template <int D>
int dispatch_mixed_group(const PrefillLaunch& pl, const pkv::decode::Params& dprm, uint32_t* queue, int sm_count,
                         cudaStream_t s) {
  switch (pl.group) {
    case 1: return launch_mixed<D, 1>(pl, dprm, queue, sm_count, s);
    case 2: return launch_mixed<D, 2>(pl, dprm, queue, sm_count, s);
    case 4: return launch_mixed<D, 4>(pl, dprm, queue, sm_count, s);
    case 8: return launch_mixed<D, 8>(pl, dprm, queue, sm_count, s);
  }
  return PKV_ERR_UNSUPPORTED;
}

}  // namespace

extern "C" {

const char* pkv_status_string(int status) {
  switch (status) {
    case PKV_OK: return "ok";
    case PKV_ERR_NULL_POINTER: return "null pointer argument";
    case PKV_ERR_BAD_SHAPE: return "invalid shape or size";
    case PKV_ERR_UNSUPPORTED: return "unsupported head_dim, page_size or GQA group size";
    case PKV_ERR_MISALIGNED: return "tensor pointer not 16-byte aligned";
    case PKV_ERR_WORKSPACE: return "workspace missing or too small";
    case PKV_ERR_CUDA: return "CUDA launch or runtime error";
    case PKV_ERR_DEVICE: return "current device is not sm_100 (B200)";
    case PKV_ERR_TENSOR_MAP: return "TMA tensor map rejected by the driver";
  }
  return "unknown status";
}

int pkv_kv_append(const void* k_new, const void* v_new, const int32_t* slot_mapping,
                  int32_t num_tokens, void* k_pool, void* v_pool, pkv_pool_desc pool,
                  pkv_stream_t stream) {
  if (num_tokens < 0) return PKV_ERR_BAD_SHAPE;
  int st = check_pool(pool);
  if (st != PKV_OK) return st;
  if (num_tokens == 0) return PKV_OK;
  if (!k_new || !v_new || !slot_mapping || !k_pool || !v_pool) return PKV_ERR_NULL_POINTER;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_pool) || !aligned16(v_pool))
    return PKV_ERR_MISALIGNED;
  DeviceInfo dev;
  if ((st = current_device(&dev)) != PKV_OK) return st;
  const long long chunks = static_cast<long long>(num_tokens) * pool.num_kv_heads * (pool.head_dim / 8);
  const int threads = 256;
  const long long want = (chunks + threads - 1) / threads;
  const int blocks = static_cast<int>(std::min<long long>(want, static_cast<long long>(dev.sm_count) * 16));
  const int64_t num_slots = static_cast<int64_t>(pool.num_pages) * pool.page_size;
  auto s = reinterpret_cast<cudaStream_t>(stream);
  if (pool.head_dim == 128)
    pkv::kv_append_kernel<128><<<blocks, threads, 0, s>>>(
        static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new), slot_mapping, num_tokens,
        static_cast<uint4*>(k_pool), static_cast<uint4*>(v_pool), pool.num_kv_heads, pool.page_size, num_slots);
  else
    pkv::kv_append_kernel<64><<<blocks, threads, 0, s>>>(
        static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new), slot_mapping, num_tokens,
        static_cast<uint4*>(k_pool), static_cast<uint4*>(v_pool), pool.num_kv_heads, pool.page_size, num_slots);
  return launch_status();
}

size_t pkv_decode_workspace_bytes(int32_t batch, int32_t num_q_heads, int32_t head_dim,
                                  int32_t max_kv_len, int32_t partition_tokens) {
  if (batch < 0 || num_q_heads < 0 || head_dim < 0 || max_kv_len < 0) return 0;
  return workspace_layout(batch, num_q_heads, head_dim, split_slots(max_kv_len, partition_tokens, head_dim)).total;
}

int pkv_paged_attn_decode(const void* q, int32_t batch, int32_t num_q_heads, const void* k_pool,
                          const void* v_pool, pkv_pool_desc pool, const int32_t* page_table,
                          int32_t max_pages, const int32_t* kv_lens, float scale,
                          int32_t partition_tokens, void* workspace, size_t workspace_bytes,
                          void* out, float* out_lse, pkv_stream_t stream) {
  return pkv_paged_attn_decode_flags(q, batch, num_q_heads, k_pool, v_pool, pool, page_table, max_pages, kv_lens,
                                     scale, partition_tokens, workspace, workspace_bytes, out, out_lse, 0u, stream);
}

int pkv_paged_attn_decode_flags(const void* q, int32_t batch, int32_t num_q_heads, const void* k_pool,
                                const void* v_pool, pkv_pool_desc pool, const int32_t* page_table,
                                int32_t max_pages, const int32_t* kv_lens, float scale,
                                int32_t partition_tokens, void* workspace, size_t workspace_bytes, void* out,
                                float* out_lse, uint32_t flags, pkv_stream_t stream) {
  if ((flags & ~static_cast<uint32_t>(PKV_DECODE_METADATA_READY)) != 0) return PKV_ERR_BAD_SHAPE;
  DecodePlan dp;
  const int st = check_decode(q, batch, num_q_heads, k_pool, v_pool, pool, page_table, max_pages, kv_lens,
                              scale, partition_tokens, out, &dp);
  if (st != PKV_OK || batch == 0) return st;
  if (workspace == nullptr || workspace_bytes < dp.wl.total) return PKV_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return PKV_ERR_MISALIGNED;
  return run_decode(q, batch, num_q_heads, k_pool, v_pool, pool, page_table, max_pages, kv_lens, scale,
                    partition_tokens, dp, workspace, out, out_lse, flags, reinterpret_cast<cudaStream_t>(stream));
}

int pkv_paged_attn_decode_append(const void* q, const void* k_new, const void* v_new, int32_t batch,
                                 int32_t num_q_heads, void* k_pool, void* v_pool, pkv_pool_desc pool,
                                 const int32_t* page_table, int32_t max_pages, const int32_t* kv_lens, float scale,
                                 int32_t partition_tokens, void* workspace, size_t workspace_bytes, void* out,
                                 float* out_lse, uint32_t flags, pkv_stream_t stream) {
  if ((flags & ~static_cast<uint32_t>(PKV_DECODE_METADATA_READY)) != 0) return PKV_ERR_BAD_SHAPE;
  DecodePlan dp;
  const int st = check_decode(q, batch, num_q_heads, k_pool, v_pool, pool, page_table, max_pages, kv_lens,
                              scale, partition_tokens, out, &dp);
  if (st != PKV_OK || batch == 0) return st;
  if (!k_new || !v_new) return PKV_ERR_NULL_POINTER;
  if (!aligned16(k_new) || !aligned16(v_new)) return PKV_ERR_MISALIGNED;
  if (!pkv::decode::kCpAsync) return PKV_ERR_UNSUPPORTED;  // the bulk-copy build streams rows it cannot swap
  if (workspace == nullptr || workspace_bytes < dp.wl.total) return PKV_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return PKV_ERR_MISALIGNED;
  return run_decode(q, batch, num_q_heads, k_pool, v_pool, pool, page_table, max_pages, kv_lens, scale,
                    partition_tokens, dp, workspace, out, out_lse, flags, reinterpret_cast<cudaStream_t>(stream),
                    k_new, v_new);
}

int pkv_split_k_combine(const float* part_o, const float* part_lse, const int32_t* num_splits,
                        int32_t batch, int32_t num_q_heads, int32_t head_dim, int32_t max_splits,
                        void* out, float* out_lse, pkv_stream_t stream) {
  if (batch < 0 || num_q_heads <= 0 || max_splits <= 0) return PKV_ERR_BAD_SHAPE;
  if (head_dim != 64 && head_dim != 128) return PKV_ERR_UNSUPPORTED;
  if (batch == 0) return PKV_OK;
  if (!part_o || !part_lse || !num_splits || !out) return PKV_ERR_NULL_POINTER;
  if (!aligned16(part_o) || !aligned16(out)) return PKV_ERR_MISALIGNED;
  DeviceInfo dev;
  int st;
  if ((st = current_device(&dev)) != PKV_OK) return st;
  auto s = reinterpret_cast<cudaStream_t>(stream);
  if (head_dim == 128)
    return launch_combine<128>(part_o, part_lse, num_splits, batch, num_q_heads, max_splits,
                               static_cast<uint16_t*>(out), out_lse, -1, false, s);
  return launch_combine<64>(part_o, part_lse, num_splits, batch, num_q_heads, max_splits,
                            static_cast<uint16_t*>(out), out_lse, -1, false, s);
}

int pkv_paged_attn_chunked_prefill(const void* q, const int32_t* cu_q_lens, int32_t batch,
                                   int32_t num_q_heads, int32_t total_q, int32_t max_q_len,
                                   const int32_t* ctx_offsets, const void* k_pool, const void* v_pool,
                                   pkv_pool_desc pool, const int32_t* page_table, int32_t max_pages,
                                   float scale, void* out, pkv_stream_t stream) {
  return run_prefill(q, cu_q_lens, batch, num_q_heads, total_q, max_q_len, ctx_offsets, k_pool, v_pool, pool,
                     page_table, max_pages, scale, 0, nullptr, 0, out, reinterpret_cast<cudaStream_t>(stream));
}

size_t pkv_verify_workspace_bytes(int32_t total_q, int32_t num_q_heads, int32_t head_dim, int32_t max_kv_len,
                                  int32_t partition_tokens) {
  if (total_q < 0 || num_q_heads < 0 || head_dim < 0 || max_kv_len < 0 || partition_tokens < 0) return 0;
  return verify_layout(total_q, num_q_heads, head_dim, max_kv_len,
                       partition_tokens > 0 ? partition_tokens
                                            : std::min(kVerifyMinPartition, round_up_tile(max_kv_len)))
      .total;
}

int pkv_paged_attn_verify(const void* q, const int32_t* cu_q_lens, int32_t batch, int32_t num_q_heads,
                          int32_t total_q, int32_t max_q_len, const int32_t* ctx_offsets, const void* k_pool,
                          const void* v_pool, pkv_pool_desc pool, const int32_t* page_table, int32_t max_pages,
                          float scale, int32_t partition_tokens, void* workspace, size_t workspace_bytes,
                          void* out, pkv_stream_t stream) {
  if (partition_tokens < 0 || (partition_tokens > 0 && partition_tokens % kPrefillBN != 0) ||
      partition_tokens > (1 << 20))
    return PKV_ERR_BAD_SHAPE;
  return run_prefill(q, cu_q_lens, batch, num_q_heads, total_q, max_q_len, ctx_offsets, k_pool, v_pool, pool,
                     page_table, max_pages, scale, partition_tokens == 0 ? -1 : partition_tokens, workspace,
                     workspace_bytes, out, reinterpret_cast<cudaStream_t>(stream));
}

size_t pkv_mixed_workspace_bytes(int32_t batch_dec, int32_t num_q_heads, int32_t head_dim, int32_t max_kv_len) {
  return pkv_decode_workspace_bytes(std::max<int32_t>(batch_dec, 1), num_q_heads, head_dim, max_kv_len, 0);
}

int pkv_paged_attn_mixed(const void* q_pre, const int32_t* cu_q_lens, int32_t batch_pre, int32_t total_q,
                         int32_t max_q_len, const int32_t* ctx_offsets, const int32_t* page_table_pre,
                         int32_t max_pages_pre, const void* q_dec, int32_t batch_dec,
                         const int32_t* page_table_dec, int32_t max_pages_dec, const int32_t* kv_lens,
                         int32_t num_q_heads, const void* k_pool, const void* v_pool, pkv_pool_desc pool,
                         float scale, void* workspace, size_t workspace_bytes, void* out_pre, void* out_dec,
                         float* out_lse_dec, pkv_stream_t stream) {
  PrefillLaunch pl;
  const int stp = build_prefill(q_pre, cu_q_lens, batch_pre, num_q_heads, total_q, max_q_len, ctx_offsets, k_pool,
                                v_pool, pool, page_table_pre, max_pages_pre, scale, out_pre, &pl);
  if (stp < 0) return stp;
  DecodePlan dp;
  int st = check_decode(q_dec, batch_dec, num_q_heads, k_pool, v_pool, pool, page_table_dec, max_pages_dec, kv_lens,
                        scale, 0, out_dec, &dp);
  if (st != PKV_OK) return st;
  const bool has_pre = stp == PKV_OK, has_dec = batch_dec > 0;
  if (has_dec) {
    if (workspace == nullptr || workspace_bytes < dp.wl.total) return PKV_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return PKV_ERR_MISALIGNED;
  }
  if (!has_pre && !has_dec) return PKV_OK;
  DeviceInfo dev;
  if ((st = current_device(&dev)) != PKV_OK) return st;
  if (has_pre && (st = make_prefill_maps(q_pre, k_pool, v_pool, pool, num_q_heads, total_q, &pl)) != PKV_OK)
    return st;
  auto s = reinterpret_cast<cudaStream_t>(stream);
  const int D = pool.head_dim;
  if (!has_dec)
    return D == 128 ? dispatch_prefill_group<128>(pl.group, pl.prm, pl.qmap, pl.kmap, pl.vmap, max_q_len, s)
                    : dispatch_prefill_group<64>(pl.group, pl.prm, pl.qmap, pl.kmap, pl.vmap, max_q_len, s);
  const pkv::decode::Params dprm = fill_decode(q_dec, batch_dec, num_q_heads, k_pool, v_pool, pool, page_table_dec,
                                               max_pages_dec, kv_lens, scale, 0, dp, workspace, out_dec,
                                               out_lse_dec, 0u);
  if ((st = prepare_workspace(workspace, dp.wl.zero_bytes, s)) != PKV_OK) return st;
  if (has_pre) {
    // the queue counters sit after the decode kernel's two in the workspace's
    // counter block, which every completed call leaves zero
    uint32_t* queue = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(workspace) + dp.wl.counters) + 2;
    st = D == 128 ? dispatch_mixed_group<128>(pl, dprm, queue, dev.sm_count, s)
                  : dispatch_mixed_group<64>(pl, dprm, queue, dev.sm_count, s);
    if (st != kNothingToDo) return st;
    // this batch runs as two kernels
    st = D == 128 ? dispatch_prefill_group<128>(pl.group, pl.prm, pl.qmap, pl.kmap, pl.vmap, max_q_len, s)
                  : dispatch_prefill_group<64>(pl.group, pl.prm, pl.qmap, pl.kmap, pl.vmap, max_q_len, s);
    if (st != PKV_OK) return st;
  }
  if (D == 128) return dispatch_decode_group<128>(dp.group, dprm, dev.sm_count, s);
  return dispatch_decode_group<64>(dp.group, dprm, dev.sm_count, s);
}

int pkv_qk_norm_rope_append(const void* q, const void* k, const void* v, int32_t num_tokens,
                            int32_t num_q_heads, const void* q_norm_weight, const void* k_norm_weight,
                            const int32_t* positions, const int32_t* slot_mapping, float eps,
                            float rope_theta, void* q_out, void* k_pool, void* v_pool, pkv_pool_desc pool,
                            pkv_stream_t stream) {
  if (num_tokens < 0) return PKV_ERR_BAD_SHAPE;
  int st = check_pool(pool);
  if (st != PKV_OK) return st;
  int group = 0;
  if ((st = check_heads(num_q_heads, pool, &group)) != PKV_OK) return st;
  if (!std::isfinite(eps) || eps < 0.f || !std::isfinite(rope_theta) || !(rope_theta > 1.f))
    return PKV_ERR_BAD_SHAPE;
  if (num_tokens == 0) return PKV_OK;
  if (!q || !k || !v || !q_norm_weight || !k_norm_weight || !positions || !slot_mapping || !q_out ||
      !k_pool || !v_pool)
    return PKV_ERR_NULL_POINTER;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(q_norm_weight) ||
      !aligned16(k_norm_weight) || !aligned16(q_out) || !aligned16(k_pool) || !aligned16(v_pool))
    return PKV_ERR_MISALIGNED;
  DeviceInfo dev;
  if ((st = current_device(&dev)) != PKV_OK) return st;
  pkv::prologue::Params prm;
  prm.q = static_cast<const uint16_t*>(q);
  prm.k = static_cast<const uint16_t*>(k);
  prm.v = static_cast<const uint16_t*>(v);
  prm.q_w = static_cast<const uint16_t*>(q_norm_weight);
  prm.k_w = static_cast<const uint16_t*>(k_norm_weight);
  prm.positions = positions;
  prm.slots = slot_mapping;
  prm.q_out = static_cast<uint16_t*>(q_out);
  prm.k_pool = static_cast<uint16_t*>(k_pool);
  prm.v_pool = static_cast<uint16_t*>(v_pool);
  prm.T = num_tokens;
  prm.Hq = num_q_heads;
  prm.Hkv = pool.num_kv_heads;
  prm.P = pool.page_size;
  prm.num_slots = static_cast<int64_t>(pool.num_pages) * pool.page_size;
  prm.eps = eps;
  prm.log2_theta = std::log2(static_cast<double>(rope_theta));
  auto s = reinterpret_cast<cudaStream_t>(stream);
  const dim3 grid(static_cast<unsigned>(num_tokens)), block(32 * pkv::prologue::kWarps);
  if (pool.head_dim == 128) return launch_pdl(pkv::prologue::qk_norm_rope_append_kernel<128>, grid, block, 0, s, prm);
  return launch_pdl(pkv::prologue::qk_norm_rope_append_kernel<64>, grid, block, 0, s, prm);
}

int pkv_kv_append_cow(const void* k_new, const void* v_new, const int32_t* token_req, const int32_t* token_pos,
                      int32_t num_tokens, int32_t* page_table, int32_t batch, int32_t max_pages,
                      int32_t* page_refcount, const int32_t* free_pages, int32_t num_free, int32_t* free_used,
                      void* k_pool, void* v_pool, pkv_pool_desc pool, pkv_stream_t stream) {
  if (num_tokens < 0 || batch < 0 || max_pages <= 0 || num_free < 0) return PKV_ERR_BAD_SHAPE;
  int st = check_pool(pool);
  if (st != PKV_OK) return st;
  if (static_cast<long long>(max_pages) * pool.page_size > (1ll << 30)) return PKV_ERR_BAD_SHAPE;
  if (num_tokens == 0) return PKV_OK;
  if (!k_new || !v_new || !token_req || !token_pos || !page_table || !page_refcount || !free_used ||
      !k_pool || !v_pool || (num_free > 0 && !free_pages))
    return PKV_ERR_NULL_POINTER;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_pool) || !aligned16(v_pool))
    return PKV_ERR_MISALIGNED;
  DeviceInfo dev;
  if ((st = current_device(&dev)) != PKV_OK) return st;
  pkv::cow::Params prm;
  prm.k_new = static_cast<const uint4*>(k_new);
  prm.v_new = static_cast<const uint4*>(v_new);
  prm.token_req = token_req;
  prm.token_pos = token_pos;
  prm.page_table = page_table;
  prm.refcount = page_refcount;
  prm.free_pages = free_pages;
  prm.free_used = free_used;
  prm.k_pool = static_cast<uint4*>(k_pool);
  prm.v_pool = static_cast<uint4*>(v_pool);
  prm.T = num_tokens;
  prm.B = batch;
  prm.max_pages = max_pages;
  prm.num_free = num_free;
  prm.num_pages = pool.num_pages;
  prm.Hkv = pool.num_kv_heads;
  prm.P = pool.page_size;
  auto s = reinterpret_cast<cudaStream_t>(stream);
  const dim3 pgrid(static_cast<unsigned>((num_tokens + pkv::cow::kPrepWarps - 1) / pkv::cow::kPrepWarps));
  const dim3 pblock(32 * pkv::cow::kPrepWarps);
  const long long chunks = static_cast<long long>(num_tokens) * pool.num_kv_heads * (pool.head_dim / 8);
  const unsigned ablocks = static_cast<unsigned>(std::min<long long>((chunks + 255) / 256, dev.sm_count * 16ll));
  if (pool.head_dim == 128) {
    if ((st = launch_pdl(pkv::cow::prepare_kernel<128>, pgrid, pblock, 0, s, prm)) != PKV_OK) return st;
    return launch_pdl(pkv::cow::append_kernel<128>, dim3(ablocks), dim3(256), 0, s, prm);
  }
  if ((st = launch_pdl(pkv::cow::prepare_kernel<64>, pgrid, pblock, 0, s, prm)) != PKV_OK) return st;
  return launch_pdl(pkv::cow::append_kernel<64>, dim3(ablocks), dim3(256), 0, s, prm);
}

int pkv_device_error_flags(uint32_t* flags, int clear) {
  if (flags == nullptr) return PKV_ERR_NULL_POINTER;
  if (cudaDeviceSynchronize() != cudaSuccess) return PKV_ERR_CUDA;
  uint32_t v = 0;
  if (cudaMemcpyFromSymbol(&v, pkv::g_error_flags, sizeof(v)) != cudaSuccess) return PKV_ERR_CUDA;
  *flags = v;
  if (clear) {
    const uint32_t zero = 0;
    if (cudaMemcpyToSymbol(pkv::g_error_flags, &zero, sizeof(zero)) != cudaSuccess) return PKV_ERR_CUDA;
  }
  return PKV_OK;
}

}  // extern "C"

// ===========================================================================
// Decode with built-in scratch: pkv_paged_attn_decode_static
//
// Some callers cannot allocate device memory at the moment they run decode:
// code that runs inside another allocator's callbacks (where allocating would
// re-enter it), plugins whose host framework hands out only the input and
// output buffers and owns every other allocation, and processes that must not
// grow their device footprint once serving has started.  This entry point
// keeps the split-K scratch of pkv_paged_attn_decode (the per-split partials
// and the two work-scheduling counters) in one fixed array compiled into the
// library instead of in a caller-provided workspace, and allocates nothing.
// ===========================================================================

namespace {
// Size of the built-in scratch.  Every GPU that loads this library holds this
// much device memory for it until the process exits.
constexpr size_t kStaticScratchBytes = size_t{32} << 20;  // 32 MiB
}  // namespace

static __device__ __align__(256) uint8_t g_static_decode_scratch[kStaticScratchBytes];

namespace {
// Device address of g_static_decode_scratch, looked up once per device.  In
// host code the array's name only stands in for the symbol; kernels must be
// given the address the runtime reports for the current device.
void* g_static_scratch_addr[kMaxDevices] = {};

int static_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PKV_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_static_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_decode_scratch) != cudaSuccess || p == nullptr)
      return PKV_ERR_CUDA;
    g_static_scratch_addr[dev] = p;
  }
  *out = g_static_scratch_addr[dev];
  return PKV_OK;
}
}  // namespace

extern "C" int pkv_paged_attn_decode_static(const void* q, int32_t batch, int32_t num_q_heads,
                                            const void* k_pool, const void* v_pool,
                                            pkv_pool_desc pool, const int32_t* page_table,
                                            int32_t max_pages, const int32_t* kv_lens, float scale,
                                            int32_t partition_tokens, void* out, float* out_lse,
                                            pkv_stream_t stream) {
  // every argument check of pkv_paged_attn_decode comes first, so that a
  // refused call leaves the scratch untouched
  DecodePlan dp;
  int st = check_decode(q, batch, num_q_heads, k_pool, v_pool, pool, page_table, max_pages, kv_lens, scale,
                        partition_tokens, out, &dp);
  if (st != PKV_OK) return st;
  if (dp.wl.total > kStaticScratchBytes) return PKV_ERR_WORKSPACE;  // beyond the built-in 32 MiB
  if (batch == 0) return PKV_OK;
  void* scratch = nullptr;
  if ((st = static_scratch(&scratch)) != PKV_OK) return st;
  // The array keeps whatever the previous call left; the scheduling and
  // per-group split counters at its start must be zero when the decode
  // kernel begins.  Having cleared them here, record them as clear so the
  // shared launch path does not clear them a second time.
  auto s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(scratch, 0, dp.wl.zero_bytes, s) != cudaSuccess) return PKV_ERR_CUDA;
  mark_workspace_zero(scratch, dp.wl.zero_bytes);
  return run_decode(q, batch, num_q_heads, k_pool, v_pool, pool, page_table, max_pages, kv_lens, scale,
                    partition_tokens, dp, scratch, out, out_lse, 0u, s);
}
