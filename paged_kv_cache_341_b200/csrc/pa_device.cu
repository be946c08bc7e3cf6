// Device entry points of libpagedattn.so (declared in include/pa.h): argument
// checks, launch configuration, TMA tensor maps, and the device error word.
// All kernels live in this one translation unit.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdlib>
#include <mutex>
#include <string>

#include "cache_ops.cuh"
#include "decode.cuh"
#include "prefix.cuh"
#include "prefix_tc.cuh"
#include "prefix_tc2.cuh"
#include "pa.h"
#include "pa_common.h"

#include "launch_decode.cuh"

namespace {

// Split of the shared prefix into slices of this many tokens: the units of
// work of the prefix kernels (and the partial slots of each query row); fixed
// so that the workspace size is a function of the arguments alone.
constexpr int kPrefixSplitTokens = 512;

int prefix_splits(int prefix_len) { return (prefix_len + kPrefixSplitTokens - 1) / kPrefixSplitTokens; }

struct PrefixArgs {
  const int32_t* prefix_blocks;
  int prefix_len;
};

// Prefix kernel: the SM-pair tcgen05 kernel by default (head_dim 128, where
// clusters of two fit; else the one-SM tcgen05 kernel); PA_PREFIX_PATH=umma
// picks the one-SM kernel and PA_PREFIX_PATH=mma the mma.sync kernel (same
// results within rounding, kept for comparison).
enum class PrefixPath { kUmma, kPair, kMma };
thread_local int g_last_prefix_kernel = 0;     // pa_debug_last_prefix_kernel
PrefixPath prefix_path() {
  const char* v = std::getenv("PA_PREFIX_PATH");
  if (v && std::string(v) == "mma") return PrefixPath::kMma;
  if (v && std::string(v) == "umma") return PrefixPath::kUmma;
  return PrefixPath::kPair;
}

// Queries [S][Hq][D] as a 4-D map (64 elements, D / 64 panels, Hq heads, S
// sequences) with 128-byte swizzle, box (64, 1, G, 128 / G): one box is the
// query-tile panel of 128 rows s * G + g of one head group.
template <typename T>
pa_status make_query_map(CUtensorMap* map, const void* q, int S, int Hq, int D, int G) {
  auto encode = tensor_map_encoder();
  if (!encode) return pa::fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t dims[4] = {64, static_cast<cuuint64_t>(D / 64), static_cast<cuuint64_t>(Hq),
                              static_cast<cuuint64_t>(S)};
  const cuuint64_t strides[3] = {128, static_cast<cuuint64_t>(D) * sizeof(T),
                                 static_cast<cuuint64_t>(Hq) * D * sizeof(T)};
  const cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(G), static_cast<cuuint32_t>(pa::kUmmaRows / G)};
  const cuuint32_t elem_strides[4] = {1, 1, 1, 1};
  CUresult r = encode(map, map_type<T>(), 4, const_cast<void*>(q), dims, strides, box, elem_strides,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return pa::fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled (queries) failed (" + std::to_string(r) + ")");
  return PA_OK;
}

template <typename T, int D, int G>
pa_status launch_prefix_umma(const DecodeArgs& a, const PrefixArgs& pf, const DeviceInfo& dev) {
  int stages = 2;
  const int forced_st = env_int("PA_PREFIX_STAGES");
  if (forced_st >= 2 && forced_st <= 8) stages = forced_st;
  while (stages >= 2 && pa::prefix_umma_smem_bytes<D>(stages) > static_cast<size_t>(dev.smem_optin)) --stages;
  if (stages < 2) return pa::fail(PA_ERR_UNSUPPORTED, "shared prefix: stage does not fit in shared memory");
  const size_t smem = pa::prefix_umma_smem_bytes<D>(stages);
  auto kern = pa::prefix_umma_kernel<T, D, G>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(prefix umma)");
  CUtensorMap tm_k, tm_v;
  const long long rows = static_cast<long long>(a.num_blocks) * a.BS;
  const int box_rows = a.BS < pa::kChunkTokens ? a.BS : pa::kChunkTokens;
  pa_status st = make_cache_map<T>(&tm_k, a.k_cache, D, a.Hkv, rows, 1, true, box_rows);
  if (st != PA_OK) return st;
  st = make_cache_map<T>(&tm_v, a.v_cache, D, a.Hkv, rows, 1, true, box_rows);
  if (st != PA_OK) return st;
  CUtensorMap tm_q;
  st = make_query_map<T>(&tm_q, a.q, a.S, a.Hq, D, G);
  if (st != PA_OK) return st;
  const int np = a.total_parts;
  const size_t acc_elems = static_cast<size_t>(a.S) * a.Hq * np * D;
  char* ws = static_cast<char*>(a.workspace);
  const size_t list_bytes = units_bytes(a.S, a.Hq, max_parts(a.max_blocks, a.BS, a.P));
  pa::PrefixParams prm;
  prm.q = a.q;
  prm.prefix_blocks = pf.prefix_blocks;
  prm.part_acc = reinterpret_cast<float*>(ws + kSchedBytes + list_bytes);
  prm.part_ml = reinterpret_cast<float2*>(prm.part_acc + acc_elems);
  prm.num_seqs = a.S;
  prm.num_q_heads = a.Hq;
  prm.num_kv_heads = a.Hkv;
  prm.block_size = a.BS;
  prm.num_blocks = a.num_blocks;
  prm.prefix_len = pf.prefix_len;
  prm.split_tokens = kPrefixSplitTokens;
  prm.max_parts = np;
  prm.stages = stages;
  prm.stage_bytes = static_cast<uint32_t>(pa::kUmmaTile * D * sizeof(T));
  prm.qk_scale = a.scale * 1.4426950408889634f;
  // persistent grid: one CTA per SM (it holds all the tensor memory), each
  // taking a contiguous share of the (query-tile pair, KV head, slice) units
  constexpr int kCtaRows = pa::kUmmaTiles * pa::kUmmaRows;
  prm.row_pairs = (a.S * G + kCtaRows - 1) / kCtaRows;
  prm.num_splits = prefix_splits(pf.prefix_len);
  prm.num_units = static_cast<long long>(prm.row_pairs) * a.Hkv * prm.num_splits;
  const int grid = prm.num_units < dev.sms ? static_cast<int>(prm.num_units) : dev.sms;
  kern<<<grid, pa::kUmmaThreads, smem, a.stream>>>(tm_k, tm_v, tm_q, prm);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "prefix_umma_kernel launch");
  g_last_prefix_kernel = 2;
  return PA_OK;
}

// The SM-pair kernel (head_dim 128): clusters of two CTAs, as many as can be
// resident at once.  Returns PA_ERR_UNSUPPORTED without launching when no
// cluster of two fits, and the caller falls back to the one-SM kernel.
template <typename T, int G>
pa_status launch_prefix_pair(const DecodeArgs& a, const PrefixArgs& pf, const DeviceInfo& dev) {
  constexpr int D = 128;
  int stages = 4;
  const int forced_st = env_int("PA_PREFIX_STAGES");
  if (forced_st >= 2 && forced_st <= 8) stages = forced_st;
  while (stages >= 2 && pa::prefix_pair_smem_bytes<D>(stages) > static_cast<size_t>(dev.smem_optin)) --stages;
  if (stages < 2) return PA_ERR_UNSUPPORTED;
  const size_t smem = pa::prefix_pair_smem_bytes<D>(stages);
  auto kern = pa::prefix_pair_kernel<T, G>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(prefix pair)");
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(pa::kPairThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = a.stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // resident clusters of two for this kernel and size, once per device
  static std::mutex mu;
  static int max_clusters[64][9] = {};
  int dev_id = 0;
  e = cudaGetDevice(&dev_id);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  int resident = 0;
  {
    std::lock_guard<std::mutex> lock(mu);
    int& slot = max_clusters[dev_id < 64 ? dev_id : 63][stages];
    if (slot == 0) {
      cfg.gridDim = dim3(2 * (dev.sms / 2));
      int n = 0;
      e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
      if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveClusters(prefix pair)");
      slot = n > 0 ? n : -1;
    }
    resident = slot;
  }
  if (resident <= 0) return PA_ERR_UNSUPPORTED;

  CUtensorMap tm_k, tm_v;
  const long long rows = static_cast<long long>(a.num_blocks) * a.BS;
  const int box_rows = a.BS < pa::kChunkTokens ? a.BS : pa::kChunkTokens;
  pa_status st = make_cache_map<T>(&tm_k, a.k_cache, D, a.Hkv, rows, 1, true, box_rows);
  if (st != PA_OK) return st;
  st = make_cache_map<T>(&tm_v, a.v_cache, D, a.Hkv, rows, 1, true, box_rows);
  if (st != PA_OK) return st;
  CUtensorMap tm_q;
  st = make_query_map<T>(&tm_q, a.q, a.S, a.Hq, D, G);
  if (st != PA_OK) return st;
  const int np = a.total_parts;
  const size_t acc_elems = static_cast<size_t>(a.S) * a.Hq * np * D;
  char* ws = static_cast<char*>(a.workspace);
  const size_t list_bytes = units_bytes(a.S, a.Hq, max_parts(a.max_blocks, a.BS, a.P));
  pa::PrefixParams prm;
  prm.q = a.q;
  prm.prefix_blocks = pf.prefix_blocks;
  prm.part_acc = reinterpret_cast<float*>(ws + kSchedBytes + list_bytes);
  prm.part_ml = reinterpret_cast<float2*>(prm.part_acc + acc_elems);
  prm.num_seqs = a.S;
  prm.num_q_heads = a.Hq;
  prm.num_kv_heads = a.Hkv;
  prm.block_size = a.BS;
  prm.num_blocks = a.num_blocks;
  prm.prefix_len = pf.prefix_len;
  prm.split_tokens = kPrefixSplitTokens;
  prm.max_parts = np;
  prm.stages = stages;
  prm.stage_bytes = static_cast<uint32_t>(pa::kUmmaTile * D * sizeof(T) / 2);
  prm.qk_scale = a.scale * 1.4426950408889634f;
  prm.row_pairs = (a.S * G + pa::kPairRows - 1) / pa::kPairRows;
  prm.num_splits = prefix_splits(pf.prefix_len);
  prm.num_units = static_cast<long long>(prm.row_pairs) * a.Hkv * prm.num_splits;
  // a multiple of the pairs per head, so that the clusters that read the same
  // (head, slice) for different pairs are at the same offset of their shares
  int clusters = resident;
  if (prm.row_pairs <= clusters) clusters = clusters / prm.row_pairs * prm.row_pairs;
  if (prm.num_units < clusters) clusters = static_cast<int>(prm.num_units);
  cfg.gridDim = dim3(2 * clusters);
  e = cudaLaunchKernelEx(&cfg, kern, tm_k, tm_v, tm_q, prm);
  if (e != cudaSuccess) return cuda_fail(e, "prefix_pair_kernel launch");
  g_last_prefix_kernel = 1;
  return PA_OK;
}

template <typename T, int D, int G>
pa_status launch_prefix(const DecodeArgs& a, const PrefixArgs& pf) {
  DeviceInfo dev;
  pa_status st = device_info(&dev);
  if (st != PA_OK) return st;
  const PrefixPath path = prefix_path();
  if constexpr (D == 128) {
    if (path == PrefixPath::kPair) {
      st = launch_prefix_pair<T, G>(a, pf, dev);
      if (st != PA_ERR_UNSUPPORTED) return st;
    }
  }
  if (path != PrefixPath::kMma) return launch_prefix_umma<T, D, G>(a, pf, dev);
  const size_t stage_bytes = static_cast<size_t>(pa::kPrefixTile) * D * sizeof(T);
  int stages = 3;
  const int forced_st = env_int("PA_PREFIX_STAGES");
  if (forced_st >= 2 && forced_st <= 8) stages = forced_st;
  while (stages >= 2 && pa::prefix_smem_bytes(stages, stage_bytes) > static_cast<size_t>(dev.smem_optin)) --stages;
  if (stages < 2) return pa::fail(PA_ERR_UNSUPPORTED, "shared prefix: stage does not fit in shared memory");
  const size_t smem = pa::prefix_smem_bytes(stages, stage_bytes);
  auto kern = pa::prefix_attention_kernel<T, D, G>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(prefix)");

  CUtensorMap tm_k, tm_v;
  const long long rows = static_cast<long long>(a.num_blocks) * a.BS;
  const int box_rows = a.BS < pa::kChunkTokens ? a.BS : pa::kChunkTokens;
  st = make_cache_map<T>(&tm_k, a.k_cache, D, a.Hkv, rows, 1, true, box_rows);
  if (st != PA_OK) return st;
  st = make_cache_map<T>(&tm_v, a.v_cache, D, a.Hkv, rows, 1, true, box_rows);
  if (st != PA_OK) return st;

  const int np = a.total_parts;
  const size_t acc_elems = static_cast<size_t>(a.S) * a.Hq * np * D;
  char* ws = static_cast<char*>(a.workspace);
  const size_t list_bytes = units_bytes(a.S, a.Hq, max_parts(a.max_blocks, a.BS, a.P));
  pa::PrefixParams prm;
  prm.q = a.q;
  prm.prefix_blocks = pf.prefix_blocks;
  prm.part_acc = reinterpret_cast<float*>(ws + kSchedBytes + list_bytes);
  prm.part_ml = reinterpret_cast<float2*>(prm.part_acc + acc_elems);
  prm.num_seqs = a.S;
  prm.num_q_heads = a.Hq;
  prm.num_kv_heads = a.Hkv;
  prm.block_size = a.BS;
  prm.num_blocks = a.num_blocks;
  prm.prefix_len = pf.prefix_len;
  prm.split_tokens = kPrefixSplitTokens;
  prm.max_parts = np;
  prm.stages = stages;
  prm.stage_bytes = static_cast<uint32_t>(stage_bytes);
  prm.qk_scale = a.scale * 1.4426950408889634f;
  const dim3 grid((a.S * G + pa::kPrefixRows - 1) / pa::kPrefixRows, a.Hkv, prefix_splits(pf.prefix_len));
  kern<<<grid, (pa::kPrefixWarps + 1) * 32, smem, a.stream>>>(tm_k, tm_v, prm);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "prefix_attention_kernel launch");
  g_last_prefix_kernel = 3;
  return PA_OK;
}

template <typename T, int D>
pa_status dispatch_prefix_group(const DecodeArgs& a, const PrefixArgs& pf) {
  switch (a.Hq / a.Hkv) {
    case 1: return launch_prefix<T, D, 1>(a, pf);
    case 2: return launch_prefix<T, D, 2>(a, pf);
    case 4: return launch_prefix<T, D, 4>(a, pf);
    case 8: return launch_prefix<T, D, 8>(a, pf);
    default: return pa::fail(PA_ERR_UNSUPPORTED, "shared prefix: Hq/Hkv must be 1, 2, 4 or 8");
  }
}

template <typename T>
pa_status dispatch_prefix(const DecodeArgs& a, const PrefixArgs& pf) {
  switch (a.D) {
    case 64: return dispatch_prefix_group<T, 64>(a, pf);
    case 128: return dispatch_prefix_group<T, 128>(a, pf);
    default: return pa::fail(PA_ERR_UNSUPPORTED, "shared prefix: head_dim must be 64 or 128");
  }
}

// The driver context current on this thread (nullptr before the thread's
// first runtime call binds one).
CUcontext current_context() {
  using Fn = CUresult (*)(CUcontext*);
  static Fn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<Fn>(p);
  });
  CUcontext c = nullptr;
  if (fn && fn(&c) != CUDA_SUCCESS) c = nullptr;
  return c;
}

// The shared-prefix call's side stream on each device (created on first use,
// highest priority) and the events of its fork and join.  They belong to the
// context they were made in: another context on the device (after a device
// reset, or one the caller bound) gets its own.
struct SideStream {
  cudaStream_t stream = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  CUcontext ctx = nullptr;
  std::mutex mu;              // its creation, and one call's fork, launches and join at a time
};

// The current device's side stream, returned with its mutex held in *hold
// (creation, or re-creation for another context, happens under it too).
pa_status side_stream(SideStream** out, std::unique_lock<std::mutex>* hold) {
  static SideStream cache[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev >= 64) return pa::fail(PA_ERR_UNSUPPORTED, "shared prefix: device index above 63");
  SideStream& s = cache[dev];
  std::unique_lock<std::mutex> lock(s.mu);
  const CUcontext ctx = current_context();
  if (!s.stream || (ctx && s.ctx && ctx != s.ctx)) {
    // (the handles of a context that is gone are dropped, not destroyed)
    int least = 0, greatest = 0;
    s.stream = nullptr;
    e = cudaDeviceGetStreamPriorityRange(&least, &greatest);
    if (e == cudaSuccess) e = cudaStreamCreateWithPriority(&s.stream, cudaStreamNonBlocking, greatest);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&s.fork, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&s.join, cudaEventDisableTiming);
    if (e != cudaSuccess) {
      s.stream = nullptr;
      return cuda_fail(e, "shared prefix: side stream and events");
    }
    s.ctx = current_context();
  }
  *out = &s;
  *hold = std::move(lock);
  return PA_OK;
}

}  // namespace

extern "C" {

pa_status pa_append_kv(const void* k_new, const void* v_new, const int64_t* slot_mapping, int32_t num_tokens,
                       void* k_cache, void* v_cache, int32_t num_blocks, int32_t block_size, int32_t num_kv_heads,
                       int32_t head_dim, pa_dtype dtype, void* stream) {
  if (!dtype_ok(dtype)) return pa::fail(PA_ERR_INVALID, "pa_append_kv: bad dtype");
  if (num_tokens < 0 || num_blocks < 0 || block_size <= 0 || num_kv_heads <= 0 || head_dim <= 0)
    return pa::fail(PA_ERR_INVALID, "pa_append_kv: bad sizes");
  const size_t row_bytes = static_cast<size_t>(num_kv_heads) * head_dim * elem_bytes(dtype);
  if (row_bytes % 16 != 0) return pa::fail(PA_ERR_UNSUPPORTED, "pa_append_kv: row bytes must be a multiple of 16");
  if (num_tokens == 0) return pa::ok();
  if (!k_new || !v_new || !slot_mapping || !k_cache || !v_cache)
    return pa::fail(PA_ERR_INVALID, "pa_append_kv: null pointer");
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache))
    return pa::fail(PA_ERR_INVALID, "pa_append_kv: pointers must be 16-byte aligned");
  const int row_vecs = static_cast<int>(row_bytes / 16);
  const int threads = row_vecs >= 256 ? 256 : ((row_vecs + 31) / 32) * 32;
  dim3 grid(num_tokens, 2);
  pa::append_kernel<<<grid, threads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new), slot_mapping, static_cast<uint4*>(k_cache),
      static_cast<uint4*>(v_cache), static_cast<int64_t>(num_blocks) * block_size, row_vecs);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "append_kernel launch");
  return pa::ok();
}

pa_status pa_copy_blocks(void* k_cache, void* v_cache, const int32_t* pairs, int32_t num_pairs, int32_t num_blocks,
                         int32_t block_size, int32_t num_kv_heads, int32_t head_dim, pa_dtype dtype, void* stream) {
  if (!dtype_ok(dtype)) return pa::fail(PA_ERR_INVALID, "pa_copy_blocks: bad dtype");
  if (num_pairs < 0 || num_blocks < 0 || block_size <= 0 || num_kv_heads <= 0 || head_dim <= 0)
    return pa::fail(PA_ERR_INVALID, "pa_copy_blocks: bad sizes");
  const size_t block_bytes = static_cast<size_t>(block_size) * num_kv_heads * head_dim * elem_bytes(dtype);
  if (block_bytes % 16 != 0) return pa::fail(PA_ERR_UNSUPPORTED, "pa_copy_blocks: block bytes must be a multiple of 16");
  if (num_pairs == 0) return pa::ok();
  if (!k_cache || !v_cache || !pairs) return pa::fail(PA_ERR_INVALID, "pa_copy_blocks: null pointer");
  if (!aligned16(k_cache) || !aligned16(v_cache))
    return pa::fail(PA_ERR_INVALID, "pa_copy_blocks: pointers must be 16-byte aligned");
  const int block_vecs = static_cast<int>(block_bytes / 16);
  dim3 grid(num_pairs, 2, (block_vecs + pa::kCopySliceVecs - 1) / pa::kCopySliceVecs);
  pa::copy_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), pairs, num_blocks, block_vecs);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "copy_kernel launch");
  return pa::ok();
}

pa_status pa_update_block_tables(int32_t* block_tables, int32_t num_rows, int32_t table_stride,
                                 const int32_t* updates, int32_t num_updates, int32_t* context_lens,
                                 const int32_t* new_lens, int32_t num_lens, void* stream) {
  if (num_rows < 0 || table_stride <= 0 || num_updates < 0 || num_lens < 0 || num_lens > num_rows)
    return pa::fail(PA_ERR_INVALID, "pa_update_block_tables: bad sizes");
  if (!context_lens) num_lens = 0;
  const int n = num_updates > num_lens ? num_updates : num_lens;
  if (n == 0) return pa::ok();
  if ((num_updates > 0 && (!block_tables || !updates)) || (num_lens > 0 && !new_lens))
    return pa::fail(PA_ERR_INVALID, "pa_update_block_tables: null pointer");
  const int threads = 256;
  pa::table_update_kernel<<<(n + threads - 1) / threads, threads, 0, static_cast<cudaStream_t>(stream)>>>(
      block_tables, num_rows, table_stride, updates, num_updates, num_lens ? context_lens : nullptr, new_lens,
      num_lens);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "table_update_kernel launch");
  return pa::ok();
}

pa_status pa_read_stream(const void* buf, size_t bytes, uint32_t* sink, void* stream) {
  if (bytes % 16 != 0) return pa::fail(PA_ERR_INVALID, "pa_read_stream: bytes must be a multiple of 16");
  if (bytes == 0) return pa::ok();
  if (!buf || !sink || !aligned16(buf)) return pa::fail(PA_ERR_INVALID, "pa_read_stream: null or misaligned buffer");
  DeviceInfo di;
  pa_status st = device_info(&di);
  if (st != PA_OK) return st;
  pa::read_stream_kernel<<<di.sms * 4, 512, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(buf), static_cast<int64_t>(bytes / 16), sink);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "read_stream_kernel launch");
  return pa::ok();
}

size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_q_heads, int32_t head_dim, int32_t max_blocks_per_seq,
                                int32_t block_size, int32_t partition_size) {
  if (num_seqs <= 0 || num_q_heads <= 0 || head_dim <= 0 || max_blocks_per_seq <= 0 || block_size <= 0 ||
      partition_size < 0)
    return 0;
  const size_t np = static_cast<size_t>(max_parts(max_blocks_per_seq, block_size, partition_size));
  const size_t list = units_bytes(num_seqs, num_q_heads, np);
  if (partition_size == 0) return kSchedBytes + list;
  return kSchedBytes + list + static_cast<size_t>(num_seqs) * num_q_heads * np * (static_cast<size_t>(head_dim) * 4 + 8);
}

pa_status pa_decode_attention(const void* q, const void* k_cache, const void* v_cache, int32_t num_blocks,
                              const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* context_lens,
                              int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                              int32_t block_size, float scale, int32_t partition_size, void* workspace,
                              size_t workspace_bytes, void* out, pa_dtype dtype, void* stream) {
  if (!dtype_ok(dtype)) return pa::fail(PA_ERR_INVALID, "pa_decode_attention: bad dtype");
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0)
    return pa::fail(PA_ERR_INVALID, "pa_decode_attention: need Hq a positive multiple of Hkv");
  if (num_blocks <= 0 || max_blocks_per_seq <= 0 || block_size <= 0)
    return pa::fail(PA_ERR_INVALID, "pa_decode_attention: bad pool sizes");
  if (block_size != 8 && block_size % pa::kChunkTokens != 0)
    return pa::fail(PA_ERR_UNSUPPORTED, "pa_decode_attention: block_size must be 8 or a multiple of 16");
  if (static_cast<long long>(num_blocks) * block_size >= (1ll << 31) ||
      static_cast<long long>(max_blocks_per_seq) * block_size >= (1ll << 31))
    return pa::fail(PA_ERR_INVALID, "pa_decode_attention: pool or table too large for 32-bit token indices");
  if (partition_size < 0 ||
      (partition_size > 0 && (partition_size % block_size != 0 || partition_size % pa::kChunkTokens != 0)))
    return pa::fail(PA_ERR_INVALID,
                    "pa_decode_attention: partition_size must be 0 or a multiple of block_size and of 16");
  if (!(scale == scale) || scale > 3.0e38f || scale < -3.0e38f)
    return pa::fail(PA_ERR_INVALID, "pa_decode_attention: scale must be finite");
  if (num_seqs == 0) return pa::ok();
  if (!q || !k_cache || !v_cache || !block_tables || !context_lens || !out)
    return pa::fail(PA_ERR_INVALID, "pa_decode_attention: null pointer");
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out))
    return pa::fail(PA_ERR_INVALID, "pa_decode_attention: q, caches and out must be 16-byte aligned");
  if (partition_size > 0 || workspace) {
    const size_t need = pa_decode_workspace_size(num_seqs, num_q_heads, head_dim, max_blocks_per_seq, block_size,
                                                 partition_size);
    if (!workspace || workspace_bytes < need || !aligned16(workspace))
      return pa::fail(PA_ERR_INVALID, "pa_decode_attention: workspace missing, too small (need " +
                                          std::to_string(need) + " bytes) or misaligned");
  }
  DecodeArgs a{q,        k_cache,      v_cache,     num_blocks, block_tables, max_blocks_per_seq,
               context_lens, num_seqs, num_q_heads, num_kv_heads, head_dim,  block_size,
               scale,    partition_size, workspace, out,         dtype,        static_cast<cudaStream_t>(stream)};
  switch (dtype) {
    case PA_F32: return dispatch_dim<float>(a);
    case PA_F16: return dispatch_dim<__half>(a);
    case PA_BF16: return dispatch_dim<__nv_bfloat16>(a);
  }
  return pa::fail(PA_ERR_INVALID, "pa_decode_attention: bad dtype");
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Workspace for pa_decode_attention_static: one fixed device array per GPU,
// alive until the process exits, so that call never allocates.
static __device__ __align__(256) unsigned char g_static_workspace[PA_STATIC_WORKSPACE_BYTES];

namespace {

// Device address of g_static_workspace in the current device's context.  In
// host code the symbol is only a stand-in, not a device address, and the
// address belongs to a context (it changes after cudaDeviceReset, and differs
// under another driver context), so it is looked up on every call rather than
// cached: the lookup allocates nothing.  The first lookup in a context loads
// the library's device code into it.
pa_status static_workspace(void** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_static_workspace);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static workspace)");
  *out = p;
  return PA_OK;
}

}  // namespace

extern "C" {

pa_status pa_decode_attention_static(const void* q, const void* k_cache, const void* v_cache, int32_t num_blocks,
                                     const int32_t* block_tables, int32_t max_blocks_per_seq,
                                     const int32_t* context_lens, int32_t num_seqs, int32_t num_q_heads,
                                     int32_t num_kv_heads, int32_t head_dim, int32_t block_size, float scale,
                                     int32_t partition_size, void* out, pa_dtype dtype, void* stream) {
  const size_t need = pa_decode_workspace_size(num_seqs, num_q_heads, head_dim, max_blocks_per_seq, block_size,
                                               partition_size);
  if (need > PA_STATIC_WORKSPACE_BYTES)
    return pa::fail(PA_ERR_INVALID, "pa_decode_attention_static: these sizes need " + std::to_string(need) +
                                        " bytes of workspace, more than the static " +
                                        std::to_string(PA_STATIC_WORKSPACE_BYTES) +
                                        "; use pa_decode_attention with a caller-allocated workspace");
  void* ws = nullptr;
  if (need > 0) {
    pa_status st = static_workspace(&ws);
    if (st != PA_OK) return st;
  }
  return pa_decode_attention(q, k_cache, v_cache, num_blocks, block_tables, max_blocks_per_seq, context_lens,
                             num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, scale, partition_size, ws,
                             ws ? PA_STATIC_WORKSPACE_BYTES : 0, out, dtype, stream);
}

size_t pa_shared_prefix_workspace_size(int32_t num_seqs, int32_t num_q_heads, int32_t head_dim, int32_t prefix_len,
                                       int32_t max_suffix_blocks, int32_t block_size, int32_t partition_size) {
  if (num_seqs <= 0 || num_q_heads <= 0 || head_dim <= 0 || prefix_len < 0 || max_suffix_blocks <= 0 ||
      block_size <= 0 || partition_size < 0)
    return 0;
  const size_t suffix_parts = static_cast<size_t>(max_parts(max_suffix_blocks, block_size, partition_size));
  const size_t np = static_cast<size_t>(prefix_splits(prefix_len)) + suffix_parts;
  return kSchedBytes + units_bytes(num_seqs, num_q_heads, suffix_parts) +
         static_cast<size_t>(num_seqs) * num_q_heads * np * (static_cast<size_t>(head_dim) * 4 + 8);
}

pa_status pa_decode_attention_shared_prefix(const void* q, const void* k_cache, const void* v_cache,
                                            int32_t num_blocks, const int32_t* prefix_blocks, int32_t prefix_len,
                                            const int32_t* suffix_tables, int32_t suffix_table_stride,
                                            int32_t max_suffix_blocks, const int32_t* suffix_lens, int32_t num_seqs,
                                            int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                            int32_t block_size, float scale, int32_t partition_size,
                                            void* workspace, size_t workspace_bytes, void* out, pa_dtype dtype,
                                            void* stream) {
  if (dtype != PA_F16 && dtype != PA_BF16)
    return pa::fail(PA_ERR_UNSUPPORTED, "shared prefix: the tensor-core path takes f16/bf16 caches");
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0)
    return pa::fail(PA_ERR_INVALID, "shared prefix: need Hq a positive multiple of Hkv");
  if (num_blocks <= 0 || max_suffix_blocks <= 0 || block_size <= 0 || suffix_table_stride < max_suffix_blocks)
    return pa::fail(PA_ERR_INVALID, "shared prefix: bad pool or table sizes");
  if (block_size != 8 && block_size % pa::kChunkTokens != 0)
    return pa::fail(PA_ERR_UNSUPPORTED, "shared prefix: block_size must be 8 or a multiple of 16");
  if (prefix_len < 0 || prefix_len % block_size != 0 || prefix_len % pa::kChunkTokens != 0)
    return pa::fail(PA_ERR_INVALID, "shared prefix: prefix_len must be a multiple of block_size and of 16");
  if (static_cast<long long>(num_blocks) * block_size >= (1ll << 31) ||
      static_cast<long long>(max_suffix_blocks) * block_size >= (1ll << 31))
    return pa::fail(PA_ERR_INVALID, "shared prefix: pool or table too large for 32-bit token indices");
  if (partition_size < 0 ||
      (partition_size > 0 && (partition_size % block_size != 0 || partition_size % pa::kChunkTokens != 0)))
    return pa::fail(PA_ERR_INVALID, "shared prefix: partition_size must be 0 or a multiple of block_size and 16");
  if (!(scale == scale) || scale > 3.0e38f || scale < -3.0e38f)
    return pa::fail(PA_ERR_INVALID, "shared prefix: scale must be finite");
  if (num_seqs == 0) return pa::ok();
  if (!q || !k_cache || !v_cache || !suffix_tables || !suffix_lens || !out || (prefix_len > 0 && !prefix_blocks))
    return pa::fail(PA_ERR_INVALID, "shared prefix: null pointer");
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out))
    return pa::fail(PA_ERR_INVALID, "shared prefix: q, caches and out must be 16-byte aligned");
  if (prefix_len == 0)
    return pa_decode_attention(q, k_cache, v_cache, num_blocks, suffix_tables, max_suffix_blocks, suffix_lens,
                               num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, scale, partition_size,
                               workspace, workspace_bytes, out, dtype, stream);
  const size_t need = pa_shared_prefix_workspace_size(num_seqs, num_q_heads, head_dim, prefix_len, max_suffix_blocks,
                                                      block_size, partition_size);
  if (!workspace || workspace_bytes < need || !aligned16(workspace))
    return pa::fail(PA_ERR_INVALID, "shared prefix: workspace missing, too small (need " + std::to_string(need) +
                                        " bytes) or misaligned");
  DecodeArgs a{q,        k_cache,      v_cache,     num_blocks, suffix_tables, max_suffix_blocks,
               suffix_lens, num_seqs,  num_q_heads, num_kv_heads, head_dim,  block_size,
               scale,    partition_size, workspace, out,          dtype,       static_cast<cudaStream_t>(stream)};
  a.table_stride = suffix_table_stride;
  a.part_offset = prefix_splits(prefix_len);
  a.total_parts = a.part_offset + max_parts(max_suffix_blocks, block_size, partition_size);
  const PrefixArgs pf{prefix_blocks, prefix_len};
  if (env_int("PA_PREFIX_SERIAL")) {
    // everything on the caller's stream, one kernel after the other
    pa_status st = dtype == PA_F16 ? dispatch_prefix<__half>(a, pf) : dispatch_prefix<__nv_bfloat16>(a, pf);
    if (st != PA_OK) return st;
    st = dtype == PA_F16 ? dispatch_dim<__half>(a) : dispatch_dim<__nv_bfloat16>(a);
    return st == PA_OK ? pa::ok() : st;
  }
  // The prefix kernel on a side stream forked from the caller's; the
  // suffixes' planner and decode on the caller's stream meanwhile; the merge
  // after both (the side stream joins before it).  The two halves share no
  // data until the merge, so they may run in either order or together.
  SideStream* ss = nullptr;
  std::unique_lock<std::mutex> lock;
  pa_status st = side_stream(&ss, &lock);
  if (st != PA_OK) return st;
  cudaError_t e = cudaEventRecord(ss->fork, a.stream);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(ss->stream, ss->fork, 0);
  if (e != cudaSuccess) return cuda_fail(e, "shared prefix: fork to the side stream");
  DecodeArgs ap = a;
  ap.stream = ss->stream;
  st = dtype == PA_F16 ? dispatch_prefix<__half>(ap, pf) : dispatch_prefix<__nv_bfloat16>(ap, pf);
  if (st != PA_OK) return st;
  e = cudaEventRecord(ss->join, ss->stream);
  if (e != cudaSuccess) return cuda_fail(e, "shared prefix: join event");
  a.merge_after = ss->join;
  st = dtype == PA_F16 ? dispatch_dim<__half>(a) : dispatch_dim<__nv_bfloat16>(a);
  return st == PA_OK ? pa::ok() : st;
}

int pa_debug_last_prefix_kernel(void) { return g_last_prefix_kernel; }

pa_status pa_debug_decode_stall(int64_t wait_limit_ns) {
  if (wait_limit_ns != 0 && (wait_limit_ns < 1000 || wait_limit_ns > static_cast<int64_t>(pa::kWaitLimitNs)))
    return pa::fail(PA_ERR_INVALID, "pa_debug_decode_stall: wait_limit_ns must be 0 or in [1e3, 2e9]");
  g_decode_stall_ns.store(wait_limit_ns, std::memory_order_relaxed);
  return pa::ok();
}

pa_status pa_device_error(int32_t* code_out, int32_t reset) {
  if (!code_out) return pa::fail(PA_ERR_INVALID, "pa_device_error: code_out is NULL");
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, pa::g_device_error, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyFromSymbol");
  if (reset) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(pa::g_device_error, &zero, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyToSymbol");
  }
  *code_out = v;
  return pa::ok();
}

}  // extern "C"
