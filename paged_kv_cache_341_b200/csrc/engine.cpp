// Step executor (pa_engine_*): one whole decode step of a batch, from host
// buffers to host buffers, issued by a single call.
//
// A decode step of the paged cache is: reserve one slot per sequence on the
// host (a fresh block at offset 0, a private copy of a shared partly filled
// block -- "PagedAttention Explained: Managing KV Cache Efficiently",
// sections "Implementing a Simplified Paged KV Cache" and "Shared Prefix
// Caching"; "Master Paged Attention for LLM Inference", "How Paged Attention
// Works", steps 3-4), copy the shared blocks, write the new token's K/V into
// its slot, and attend over each sequence's blocks through its table.  The
// engine strings those calls together around the copies a serving loop needs,
// so the host side of a step is one C call instead of a dozen:
//
//   upload stream   : q, k_new, v_new (caller's page-locked host buffers) and
//                     one metadata block (slots, lengths, changed table
//                     entries, copy pairs) -> device slot b = step % 2
//   compute stream  : waits for the upload; table/length update, block copies,
//                     append, attention (planner, decode, merge)
//   download stream : waits for the compute; out -> caller's host buffer
//
// Two device slots let step i+1's upload run while step i computes and step
// i's download run while step i+1 computes.  Before reusing slot b the host
// waits for the download of step i-2, so when pa_engine_step(i) returns,
// the output of step i-2 is in host memory.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <string>
#include <vector>

#include "pa.h"
#include "pa_common.h"
#include "pool_internal.h"

namespace {

constexpr int kSlots = 2;

size_t round256(size_t n) { return (n + 255) / 256 * 256; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

pa_status cuda_fail(cudaError_t e, const char* what) {
  return pa::fail(PA_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

}  // namespace

struct pa_engine {
  pa_pool* pool = nullptr;
  int32_t* h_tables = nullptr;  // caller's host tables [S][MB]
  int32_t* h_lens = nullptr;    // caller's host lengths [S]
  int32_t S = 0, MB = 0;
  int32_t* d_tables = nullptr;  // caller's device tables [S][MB]
  int32_t* d_lens = nullptr;    // caller's device lengths [S]
  void* k_cache = nullptr;
  void* v_cache = nullptr;
  int32_t Hq = 0, Hkv = 0, D = 0, part = 0;
  pa_dtype dtype = PA_BF16;
  int device = -1;
  cudaStream_t compute = nullptr, up = nullptr, down = nullptr;
  size_t q_row = 0, kv_row = 0;
  unsigned char* dev_base = nullptr;
  unsigned char* host_base = nullptr;
  void* dq[kSlots] = {};
  void* dk[kSlots] = {};
  void* dv[kSlots] = {};
  void* dout[kSlots] = {};
  unsigned char* hmeta[kSlots] = {};
  unsigned char* dmeta[kSlots] = {};
  size_t meta_bytes = 0;
  void* ws = nullptr;
  size_t ws_bytes = 0;
  cudaEvent_t in_ready[kSlots] = {};
  cudaEvent_t comp_done[kSlots] = {};
  cudaEvent_t out_read[kSlots] = {};
  bool used[kSlots] = {false, false};
  int64_t steps = 0;

  // metadata block of one slot: slots int64 [S] | lengths int32 [S] |
  // updates int32 [S][3] | pairs int32 [S][2]
  size_t off_lens() const { return 8 * static_cast<size_t>(S); }
  size_t off_upd() const { return 12 * static_cast<size_t>(S); }
  size_t off_pairs() const { return 24 * static_cast<size_t>(S); }

  void release() {
    for (int b = 0; b < kSlots; ++b) {
      if (in_ready[b]) cudaEventDestroy(in_ready[b]);
      if (comp_done[b]) cudaEventDestroy(comp_done[b]);
      if (out_read[b]) cudaEventDestroy(out_read[b]);
    }
    if (up) cudaStreamDestroy(up);
    if (down) cudaStreamDestroy(down);
    if (dev_base) cudaFree(dev_base);
    if (host_base) cudaFreeHost(host_base);
  }
};

extern "C" {

pa_status pa_engine_create(pa_pool* pool, int32_t* host_tables, int32_t* host_lens, int32_t num_seqs,
                           int32_t max_blocks_per_seq, int32_t* device_tables, int32_t* device_lens,
                           void* k_cache, void* v_cache, int32_t num_q_heads, int32_t num_kv_heads,
                           int32_t head_dim, pa_dtype dtype, int32_t partition_size, void* stream,
                           pa_engine** engine_out) {
  if (!engine_out) return pa::fail(PA_ERR_INVALID, "pa_engine_create: engine_out is null");
  *engine_out = nullptr;
  if (!pool || !host_tables || !host_lens || !device_tables || !device_lens || !k_cache || !v_cache)
    return pa::fail(PA_ERR_INVALID, "pa_engine_create: null pointer");
  if (num_seqs <= 0 || max_blocks_per_seq <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
      num_q_heads % num_kv_heads != 0)
    return pa::fail(PA_ERR_INVALID, "pa_engine_create: bad sizes");
  if (dtype != PA_F32 && dtype != PA_F16 && dtype != PA_BF16)
    return pa::fail(PA_ERR_INVALID, "pa_engine_create: bad dtype");
  if (!aligned16(k_cache) || !aligned16(v_cache))
    return pa::fail(PA_ERR_INVALID, "pa_engine_create: caches must be 16-byte aligned");
  const size_t ws_bytes = pa_decode_workspace_size(num_seqs, num_q_heads, head_dim, max_blocks_per_seq,
                                                   pool->block_size, partition_size);
  if (ws_bytes == 0 || (partition_size > 0 && partition_size % pool->block_size != 0))
    return pa::fail(PA_ERR_INVALID, "pa_engine_create: bad partition size");

  pa_engine* e = new pa_engine();
  e->pool = pool;
  e->h_tables = host_tables;
  e->h_lens = host_lens;
  e->S = num_seqs;
  e->MB = max_blocks_per_seq;
  e->d_tables = device_tables;
  e->d_lens = device_lens;
  e->k_cache = k_cache;
  e->v_cache = v_cache;
  e->Hq = num_q_heads;
  e->Hkv = num_kv_heads;
  e->D = head_dim;
  e->dtype = dtype;
  e->part = partition_size;
  e->compute = static_cast<cudaStream_t>(stream);
  const size_t es = dtype == PA_F32 ? 4 : 2;
  e->q_row = static_cast<size_t>(num_q_heads) * head_dim * es;
  e->kv_row = static_cast<size_t>(num_kv_heads) * head_dim * es;
  e->meta_bytes = 32 * static_cast<size_t>(num_seqs);
  e->ws_bytes = ws_bytes;

  const size_t q_bytes = round256(e->q_row * num_seqs);
  const size_t kv_bytes = round256(e->kv_row * num_seqs);
  const size_t meta = round256(e->meta_bytes);
  const size_t per_slot = 2 * q_bytes + 2 * kv_bytes + meta;   // q, out, k_new, v_new, metadata
  cudaError_t err = cudaGetDevice(&e->device);
  if (err == cudaSuccess) err = cudaMalloc(&e->dev_base, kSlots * per_slot + round256(ws_bytes));
  if (err == cudaSuccess) err = cudaHostAlloc(&e->host_base, kSlots * meta, cudaHostAllocDefault);
  if (err == cudaSuccess) err = cudaStreamCreateWithFlags(&e->up, cudaStreamNonBlocking);
  if (err == cudaSuccess) err = cudaStreamCreateWithFlags(&e->down, cudaStreamNonBlocking);
  for (int b = 0; b < kSlots && err == cudaSuccess; ++b) {
    err = cudaEventCreateWithFlags(&e->in_ready[b], cudaEventDisableTiming);
    if (err == cudaSuccess) err = cudaEventCreateWithFlags(&e->comp_done[b], cudaEventDisableTiming);
    if (err == cudaSuccess) err = cudaEventCreateWithFlags(&e->out_read[b], cudaEventDisableTiming);
  }
  if (err != cudaSuccess) {
    e->release();
    delete e;
    return cuda_fail(err, "pa_engine_create");
  }
  unsigned char* p = e->dev_base;
  for (int b = 0; b < kSlots; ++b) {
    e->dq[b] = p;
    p += q_bytes;
    e->dout[b] = p;
    p += q_bytes;
    e->dk[b] = p;
    p += kv_bytes;
    e->dv[b] = p;
    p += kv_bytes;
    e->dmeta[b] = p;
    p += meta;
    e->hmeta[b] = e->host_base + b * meta;
  }
  e->ws = p;
  *engine_out = e;
  return pa::ok();
}

void pa_engine_destroy(pa_engine* e) {
  if (!e) return;
  // nothing the engine issued may still be running when its buffers go
  cudaStreamSynchronize(e->up);
  cudaStreamSynchronize(e->compute);
  cudaStreamSynchronize(e->down);
  e->release();
  delete e;
}

pa_status pa_engine_step(pa_engine* e, int32_t row0, int32_t num_rows, const void* q, const void* k_new,
                         const void* v_new, void* out, float scale, int64_t* slots_out, int32_t* pairs_out,
                         int32_t* num_pairs_out) {
  if (!e) return pa::fail(PA_ERR_INVALID, "pa_engine_step: null engine");
  if (row0 < 0 || num_rows < 0 || static_cast<int64_t>(row0) + num_rows > e->S)
    return pa::fail(PA_ERR_INVALID, "pa_engine_step: rows outside the engine's batch");
  if (!(scale == scale) || scale > 3.0e38f || scale < -3.0e38f)
    return pa::fail(PA_ERR_INVALID, "pa_engine_step: scale must be finite");
  if (num_pairs_out) *num_pairs_out = 0;
  if (num_rows == 0) return pa::ok();
  if (!q || !k_new || !v_new || !out) return pa::fail(PA_ERR_INVALID, "pa_engine_step: null buffer");
  int dev = -1;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return cuda_fail(err, "pa_engine_step: cudaGetDevice");
  if (dev != e->device) return pa::fail(PA_ERR_INVALID, "pa_engine_step: engine was created on another device");

  const int b = static_cast<int>(e->steps & 1);
  if (e->used[b]) {
    // step i-2's output has reached the host, so its device buffers and its
    // host metadata block are free again
    err = cudaEventSynchronize(e->out_read[b]);
    if (err != cudaSuccess) return cuda_fail(err, "pa_engine_step: wait for step i-2");
  }
  const int32_t bs = e->pool->block_size;
  const int32_t MB = e->MB;
  int32_t* tables = e->h_tables + static_cast<int64_t>(row0) * MB;
  int32_t* lens = e->h_lens + row0;
  unsigned char* hm = e->hmeta[b];
  int64_t* slots = reinterpret_cast<int64_t*>(hm);
  int32_t* h_lens_meta = reinterpret_cast<int32_t*>(hm + e->off_lens());
  int32_t* upd = reinterpret_cast<int32_t*>(hm + e->off_upd());
  int32_t* pairs = reinterpret_cast<int32_t*>(hm + e->off_pairs());
  int32_t npairs = 0, nupd = 0;
  // all or nothing: on failure the pool, tables and lengths are unchanged;
  // the table entries the reservation wrote go to the device tables below
  pa_status st = pa_reserve_slots_with_updates(e->pool, tables, MB, lens, num_rows, row0, slots, pairs, &npairs,
                                               upd, &nupd);
  if (st != PA_OK) return st;
  std::memcpy(h_lens_meta, e->h_lens, sizeof(int32_t) * e->S);

  unsigned char* dm = e->dmeta[b];
  const size_t qb = e->q_row * num_rows, kvb = e->kv_row * num_rows;
  err = cudaMemcpyAsync(e->dq[b], q, qb, cudaMemcpyHostToDevice, e->up);
  if (err == cudaSuccess) err = cudaMemcpyAsync(e->dk[b], k_new, kvb, cudaMemcpyHostToDevice, e->up);
  if (err == cudaSuccess) err = cudaMemcpyAsync(e->dv[b], v_new, kvb, cudaMemcpyHostToDevice, e->up);
  if (err == cudaSuccess) err = cudaMemcpyAsync(dm, hm, e->meta_bytes, cudaMemcpyHostToDevice, e->up);
  if (err == cudaSuccess) err = cudaEventRecord(e->in_ready[b], e->up);
  if (err == cudaSuccess) err = cudaStreamWaitEvent(e->compute, e->in_ready[b], 0);
  if (err != cudaSuccess) return cuda_fail(err, "pa_engine_step: upload");

  const int32_t nb = e->pool->num_blocks;
  st = pa_update_block_tables(e->d_tables, e->S, MB, reinterpret_cast<const int32_t*>(dm + e->off_upd()), nupd,
                              e->d_lens, reinterpret_cast<const int32_t*>(dm + e->off_lens()), e->S, e->compute);
  if (st == PA_OK && npairs > 0)
    st = pa_copy_blocks(e->k_cache, e->v_cache, reinterpret_cast<const int32_t*>(dm + e->off_pairs()), npairs, nb,
                        bs, e->Hkv, e->D, e->dtype, e->compute);
  if (st == PA_OK)
    st = pa_append_kv(e->dk[b], e->dv[b], reinterpret_cast<const int64_t*>(dm), num_rows, e->k_cache, e->v_cache,
                      nb, bs, e->Hkv, e->D, e->dtype, e->compute);
  if (st == PA_OK)
    st = pa_decode_attention(e->dq[b], e->k_cache, e->v_cache, nb, e->d_tables + static_cast<int64_t>(row0) * MB, MB,
                             e->d_lens + row0, num_rows, e->Hq, e->Hkv, e->D, bs, scale, e->part, e->ws, e->ws_bytes,
                             e->dout[b], e->dtype, e->compute);
  if (st != PA_OK) return st;

  err = cudaEventRecord(e->comp_done[b], e->compute);
  if (err == cudaSuccess) err = cudaStreamWaitEvent(e->down, e->comp_done[b], 0);
  if (err == cudaSuccess) err = cudaMemcpyAsync(out, e->dout[b], qb, cudaMemcpyDeviceToHost, e->down);
  if (err == cudaSuccess) err = cudaEventRecord(e->out_read[b], e->down);
  if (err != cudaSuccess) return cuda_fail(err, "pa_engine_step: download");
  e->used[b] = true;
  ++e->steps;
  if (slots_out) std::memcpy(slots_out, slots, sizeof(int64_t) * num_rows);
  if (pairs_out && npairs) std::memcpy(pairs_out, pairs, sizeof(int32_t) * 2 * npairs);
  if (num_pairs_out) *num_pairs_out = npairs;
  return pa::ok();
}

pa_status pa_engine_join(pa_engine* e) {
  if (!e) return pa::fail(PA_ERR_INVALID, "pa_engine_join: null engine");
  for (int b = 0; b < kSlots; ++b) {
    if (!e->used[b]) continue;
    cudaError_t err = cudaStreamWaitEvent(e->compute, e->out_read[b], 0);
    if (err != cudaSuccess) return cuda_fail(err, "pa_engine_join");
  }
  return pa::ok();
}

pa_status pa_engine_synchronize(pa_engine* e) {
  if (!e) return pa::fail(PA_ERR_INVALID, "pa_engine_synchronize: null engine");
  cudaError_t err = cudaStreamSynchronize(e->up);
  if (err == cudaSuccess) err = cudaStreamSynchronize(e->compute);
  if (err == cudaSuccess) err = cudaStreamSynchronize(e->down);
  if (err != cudaSuccess) return cuda_fail(err, "pa_engine_synchronize");
  return pa::ok();
}

}  // extern "C"
