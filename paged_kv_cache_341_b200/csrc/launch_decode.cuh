// Host-side launch of the decode kernels (included by pa_device.cu only):
// argument bundle, TMA tensor maps over the paged cache, the planner /
// decode / merge launch sequence, and dispatch over head_dim and group size.
// Kept apart from the other launchers so that a digest of this file, the
// kernels and their PTX helpers identifies exactly the decode path.
#ifndef PAGEDATTN_LAUNCH_DECODE_CUH
#define PAGEDATTN_LAUNCH_DECODE_CUH

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <mutex>
#include <string>

#include "decode.cuh"
#include "pa.h"
#include "pa_common.h"

namespace {


size_t elem_bytes(pa_dtype d) { return d == PA_F32 ? 4 : 2; }
bool dtype_ok(int d) { return d == PA_F32 || d == PA_F16 || d == PA_BF16; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

pa_status cuda_fail(cudaError_t e, const char* what) {
  return pa::fail(PA_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
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

struct DeviceInfo {
  int sms = 0;
  int smem_optin = 0;
};

pa_status device_info(DeviceInfo* out) {
  static std::mutex mu;
  static DeviceInfo cache[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  std::lock_guard<std::mutex> lock(mu);
  if (dev < 64 && cache[dev].sms > 0) {
    *out = cache[dev];
    return PA_OK;
  }
  DeviceInfo d;
  e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
  if (dev < 64) cache[dev] = d;
  *out = d;
  return PA_OK;
}

// Test hook of pa_debug_decode_stall: 0 = off (every normal call); otherwise
// the wait bound in nanoseconds, and every decode CTA withholds its first
// stage so that its consumers' bounded wait runs out.
std::atomic<long long> g_decode_stall_ns{0};

// Optional tuning overrides (no effect on results): KV heads per CTA tile and
// pipeline depth of the decode kernel.
int env_int(const char* name) {
  const char* v = std::getenv(name);
  return v ? std::atoi(v) : 0;
}

struct DecodeArgs {
  const void* q;
  const void* k_cache;
  const void* v_cache;
  int num_blocks;
  const int32_t* block_tables;
  int max_blocks;
  const int32_t* context_lens;
  int S, Hq, Hkv, D, BS;
  float scale;
  int P;
  void* workspace;
  void* out;
  pa_dtype dtype;
  cudaStream_t stream;
  // shared-prefix mode (pa_decode_attention_shared_prefix); plain calls leave the defaults
  int table_stride = 0;          // 0: rows of block_tables are max_blocks apart
  int part_offset = 0;           // partials before partition 0 (prefix splits)
  int total_parts = 0;           // 0: ceil(max_blocks*block_size/P), else the partial row stride
  cudaEvent_t merge_after = nullptr;  // the merge also waits for this event (the prefix kernel's side stream)
};

constexpr size_t kSchedBytes = 256;   // unit counter and unit count at the head of the workspace

size_t round256(size_t n) { return (n + 255) / 256 * 256; }

// Planned unit list: at most S * n_tiles * parts units (n_tiles <= Hkv <= Hq).
size_t units_bytes(long long S, long long Hq, long long parts) {
  return round256(static_cast<size_t>(S) * Hq * parts * sizeof(int4));
}

int max_parts(int max_blocks, int block_size, int P) {
  if (P <= 0) return 1;
  const long long cap = static_cast<long long>(max_blocks) * block_size;
  return static_cast<int>((cap + P - 1) / P);
}

template <typename T>
CUtensorMapDataType map_type();
template <>
CUtensorMapDataType map_type<float>() { return CU_TENSOR_MAP_DATA_TYPE_FLOAT32; }
template <>
CUtensorMapDataType map_type<__half>() { return CU_TENSOR_MAP_DATA_TYPE_FLOAT16; }
template <>
CUtensorMapDataType map_type<__nv_bfloat16>() { return CU_TENSOR_MAP_DATA_TYPE_BFLOAT16; }

// Tensor map over one cache viewed as [num_blocks*block_size][Hkv][D].
// Plain: boxes of 16 tokens x `tile_heads` heads x D.  Swizzled (tensor-core
// consumer): the row viewed as Hkv*D/64 column blocks of 128 bytes, boxes of
// 16 tokens x one column block, stored 128B-swizzled in shared memory.
template <typename T>
pa_status make_cache_map(CUtensorMap* map, const void* base, int D, int Hkv, long long rows, int tile_heads,
                         bool swizzled, int box_rows) {
  auto encode = tensor_map_encoder();
  if (!encode) return pa::fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t row_bytes = static_cast<cuuint64_t>(Hkv) * D * sizeof(T);
  const cuuint32_t elem_strides[3] = {1, 1, 1};
  CUresult r;
  if (swizzled) {
    const cuuint64_t box_elems = pa::kSwizzleBytes / sizeof(T);
    const cuuint64_t dims[3] = {box_elems, static_cast<cuuint64_t>(Hkv) * D / box_elems,
                                static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(pa::kSwizzleBytes), row_bytes};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(box_elems), 1, static_cast<cuuint32_t>(box_rows)};
    r = encode(map, map_type<T>(), 3, const_cast<void*>(base), dims, strides, box, elem_strides,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  } else {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(Hkv),
                                static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * sizeof(T), row_bytes};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(D), static_cast<cuuint32_t>(tile_heads),
                               static_cast<cuuint32_t>(box_rows)};
    r = encode(map, map_type<T>(), 3, const_cast<void*>(base), dims, strides, box, elem_strides,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  }
  if (r != CUDA_SUCCESS) return pa::fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled failed (" + std::to_string(r) + ")");
  return PA_OK;
}

// Consumer used for 16-bit caches: tensor cores unless PA_DECODE_PATH=alu
// (the CUDA-core consumer, kept for float32 caches and for comparisons).
bool use_tensor_cores() {
  const char* v = std::getenv("PA_DECODE_PATH");
  return !(v && std::string(v) == "alu");
}

template <typename T, int D, int G>
pa_status launch_decode(const DecodeArgs& a) {
  DeviceInfo dev;
  pa_status st = device_info(&dev);
  if (st != PA_OK) return st;

  // Launch shape, chosen by measurement on B200 (sweep over 1/2/4/8 KV heads
  // per CTA x 2..6 stages on the four large workloads): one KV head per CTA
  // and a 2- or 3-deep ring, i.e. small CTAs, eight per SM, whose independent
  // producers keep HBM busy, beat fewer, wider CTAs by up to 25%.
  int ht = 1;
  // 3 stages for groups up to 4; 2 for 8 query heads per KV head, whose
  // consumer spends longer on each stage (70B-shaped call: 5,569 -> 5,653 GB/s,
  // while the Llama shapes lose 2 % with 2)
  int stages = G >= 8 ? 2 : 3;
  const int forced_ht = env_int("PA_DECODE_TILE_HEADS");
  if (forced_ht > 0 && forced_ht <= pa::kMaxTileHeads && a.Hkv % forced_ht == 0) ht = forced_ht;
  const int forced_st = env_int("PA_DECODE_STAGES");
  if (forced_st >= 2 && forced_st <= 8) stages = forced_st;

  const size_t tile_bytes = static_cast<size_t>(pa::kChunkTokens) * ht * D * sizeof(T);
  const size_t q_bytes = static_cast<size_t>(ht) * G * D * sizeof(T);
  while (stages >= 2 && pa::pipeline_smem_bytes(stages, tile_bytes, q_bytes) > static_cast<size_t>(dev.smem_optin))
    --stages;
  if (stages < 2) return pa::fail(PA_ERR_UNSUPPORTED, "pa_decode_attention: stage does not fit in shared memory");
  const size_t smem = pa::pipeline_smem_bytes(stages, tile_bytes, q_bytes);

  bool mma = false;
  void (*kern)(const CUtensorMap, const CUtensorMap, const pa::DecodeParams) = pa::decode_kernel<T, D, G>;
  if constexpr (sizeof(T) == 2) {
    if (use_tensor_cores()) {
      kern = pa::decode_mma_kernel<T, D, G>;
      mma = true;
    }
  }
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(decode)");
  const int threads = (ht + 1) * 32;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem);
  if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
  if (per_sm < 1) return pa::fail(PA_ERR_UNSUPPORTED, "pa_decode_attention: kernel does not fit on an SM");

  const int n_tiles = a.Hkv / ht;
  const int np = a.total_parts > 0 ? a.total_parts : max_parts(a.max_blocks, a.BS, a.P);
  const bool partials = a.P > 0 || a.part_offset > 0;
  const long long units_bound = static_cast<long long>(a.S) * n_tiles * np;
  const long long slots = static_cast<long long>(dev.sms) * per_sm;
  const int grid = static_cast<int>(units_bound < slots ? units_bound : slots);

  CUtensorMap tm_k, tm_v;
  const long long rows = static_cast<long long>(a.num_blocks) * a.BS;
  const int box_rows = a.BS < pa::kChunkTokens ? a.BS : pa::kChunkTokens;
  st = make_cache_map<T>(&tm_k, a.k_cache, D, a.Hkv, rows, ht, mma, box_rows);
  if (st != PA_OK) return st;
  st = make_cache_map<T>(&tm_v, a.v_cache, D, a.Hkv, rows, ht, mma, box_rows);
  if (st != PA_OK) return st;

  pa::DecodeParams prm;
  prm.q = a.q;
  prm.block_tables = a.block_tables;
  prm.context_lens = a.context_lens;
  prm.out = a.out;
  // workspace: [unit counter + count, 256 B][unit list][partial outputs][partial (m, l)]
  const size_t acc_elems = static_cast<size_t>(a.S) * a.Hq * np * D;
  char* ws = static_cast<char*>(a.workspace);
  const size_t list_bytes = units_bytes(a.S, a.Hq, max_parts(a.max_blocks, a.BS, a.P));
  prm.sched = ws ? reinterpret_cast<int*>(ws) : nullptr;
  prm.units = ws ? reinterpret_cast<const int4*>(ws + kSchedBytes) : nullptr;
  prm.part_acc = partials ? reinterpret_cast<float*>(ws + kSchedBytes + list_bytes) : nullptr;
  prm.part_ml = partials ? reinterpret_cast<float2*>(prm.part_acc + acc_elems) : nullptr;
  prm.table_stride = a.table_stride > 0 ? a.table_stride : a.max_blocks;
  prm.part_offset = a.part_offset;
  prm.force_partials = a.part_offset > 0 ? 1 : 0;
  prm.num_seqs = a.S;
  prm.num_q_heads = a.Hq;
  prm.num_kv_heads = a.Hkv;
  prm.max_blocks = a.max_blocks;
  prm.block_size = a.BS;
  prm.num_blocks = a.num_blocks;
  prm.partition_size = a.P;
  prm.max_parts = np;
  prm.tile_heads = ht;
  prm.num_tiles = n_tiles;
  prm.stages = stages;
  prm.tile_bytes = static_cast<uint32_t>(tile_bytes);
  prm.q_bytes = static_cast<uint32_t>(q_bytes);
  prm.qk_scale = a.scale * 1.4426950408889634f;
  const long long stall_ns = g_decode_stall_ns.load(std::memory_order_relaxed);
  prm.wait_limit_ns = stall_ns > 0 ? static_cast<uint64_t>(stall_ns) : pa::kWaitLimitNs;
  prm.withhold_first = stall_ns > 0 ? 1 : 0;

  if (prm.units) {
    // planner (one CTA), then the decode grid as its programmatic dependent
    pa::PlanParams pp;
    pp.context_lens = a.context_lens;
    pp.units = reinterpret_cast<int4*>(ws + kSchedBytes);
    pp.header = prm.sched;
    pp.num_seqs = a.S;
    pp.partition_size = a.P;
    pp.num_tiles = n_tiles;
    pp.cap = a.max_blocks * a.BS;
    pp.num_ctas = grid;
    pp.balance = env_int("PA_DECODE_NO_BALANCE") ? 0 : 1;
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t pcfg = {};
    pcfg.gridDim = dim3(1);
    pcfg.stream = a.stream;
    pcfg.attrs = pdl;
    pcfg.numAttrs = 1;
    if (a.S <= pa::kPlanSmallSeqs) {
      pcfg.blockDim = dim3(32);
      e = cudaLaunchKernelEx(&pcfg, pa::plan_small_kernel, pp);
    } else {
      pcfg.blockDim = dim3(pa::kPlanThreads);
      e = cudaLaunchKernelEx(&pcfg, pa::plan_kernel, pp);
    }
    if (e != cudaSuccess) return cuda_fail(e, "plan_kernel launch");
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = a.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, tm_k, tm_v, prm);
  } else {
    kern<<<grid, threads, smem, a.stream>>>(tm_k, tm_v, prm);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) return cuda_fail(e, "decode_kernel launch");

  if (partials) {
    pa::ReduceParams rp;
    rp.context_lens = a.context_lens;
    rp.part_acc = prm.part_acc;
    rp.part_ml = prm.part_ml;
    rp.out = a.out;
    rp.num_seqs = a.S;
    rp.num_q_heads = a.Hq;
    rp.partition_size = a.P;
    rp.max_parts = np;
    rp.cap = a.max_blocks * a.BS;
    rp.part_offset = a.part_offset;
    // warps per head from the partitions that hold tokens: with a shared
    // prefix, only a few of the prefix slots of a row are written (one per
    // run of slices a prefix CTA accumulated), the rest are skipped
    rp.warps_per_head = pa::reduce_warps_per_head(a.part_offset > 0 ? np - a.part_offset + 2 : np);
    const int heads_per_cta = pa::kReduceWarps / rp.warps_per_head;
    // programmatic dependent launch: resident early, waits for the decode grid
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((a.Hq + heads_per_cta - 1) / heads_per_cta, a.S);
    cfg.blockDim = dim3(pa::kReduceWarps * 32);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = a.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (a.merge_after) {
      // the join with the side stream: an ordinary launch after the event
      e = cudaStreamWaitEvent(a.stream, a.merge_after, 0);
      if (e != cudaSuccess) return cuda_fail(e, "cudaStreamWaitEvent(merge after the prefix kernel)");
      cfg.numAttrs = 0;
    }
    // six rows a warp in flight where a head has more than 16 partitions (one
    // round of loads for up to 48 partitions; 64 registers, so a 70B-shaped
    // merge of 512 CTAs is one wave), four otherwise (48 registers)
    if (rp.warps_per_head >= 4) {
      e = cudaLaunchKernelEx(&cfg, pa::reduce_kernel<T, D, 6>, rp);
    } else {
      e = cudaLaunchKernelEx(&cfg, pa::reduce_kernel<T, D, 4>, rp);
    }
    if (e != cudaSuccess) return cuda_fail(e, "reduce_kernel launch");
  }

  return pa::ok();
}

template <typename T, int D>
pa_status dispatch_group(const DecodeArgs& a) {
  switch (a.Hq / a.Hkv) {
    case 1: return launch_decode<T, D, 1>(a);
    case 2: return launch_decode<T, D, 2>(a);
    case 4: return launch_decode<T, D, 4>(a);
    case 8: return launch_decode<T, D, 8>(a);
    default: return pa::fail(PA_ERR_UNSUPPORTED, "pa_decode_attention: Hq/Hkv must be 1, 2, 4 or 8");
  }
}

template <typename T>
pa_status dispatch_dim(const DecodeArgs& a) {
  switch (a.D) {
    case 64: return dispatch_group<T, 64>(a);
    case 128: return dispatch_group<T, 128>(a);
    default: return pa::fail(PA_ERR_UNSUPPORTED, "pa_decode_attention: head_dim must be 64 or 128");
  }
}

}  // namespace

#endif
