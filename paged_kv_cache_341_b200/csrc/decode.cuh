// Paged single-query decode attention for sm_100a.
//
// What it computes (include/pa.h, pa_decode_attention): for each sequence s
// and query head h, softmax(q . K^T * scale) V over the sequence's tokens,
// where token j's K/V row sits in block block_tables[s][j / block_size] --
// the kernel walks the block table rather than gathering the blocks
// ("PagedAttention Explained: Managing KV Cache Efficiently", section
// "Block Tables and Non-Contiguous Storage").
//
// Design (HBM-bound: every K/V byte is read exactly once):
//
// * Work unit = (sequence, partition of `partition_size` tokens, tile of HT
//   KV heads).  plan_kernel lists the units -- every full partition in
//   sequence order, then every remainder partition (or, without partitions,
//   every whole sequence) longest first -- and the persistent grid takes them
//   from an atomic counter in that order, so the small units come last and
//   the SMs finish together.  The decode kernel is a programmatic dependent of
//   the planner: its CTAs start while the plan is written and wait for it.
//   Without a workspace the units are walked from the lengths and dealt
//   round-robin instead.
// * One producer warp streams each unit as chunks of 16 tokens, each chunk
//   taken straight from the physical block the block table names, by TMA tile
//   loads into a ring of shared-memory stages guarded by full/empty mbarriers.
//   The table slice sits in the producer's registers (32 entries per warp
//   load); the unit's HT*G query rows come in by one bulk copy into a double
//   buffer.
// * Consumer warp j owns KV head j of the tile and all G = Hq/Hkv query heads
//   that share it, so every K/V element loaded serves G query heads.  Two
//   consumers exist:
//   - decode_kernel (CUDA cores; float32 caches): lanes form groups of L
//     lanes per token, each lane holding E = D/L elements of the G query rows
//     as float32 pairs; dot products finish with log2(L) xor-shuffles, and
//     each group keeps its own online-softmax state, merged at unit end.
//   - decode_mma_kernel (tensor cores, mma.sync m16n8k16; 16-bit caches):
//     S^T = K Q^T with the 16 tokens of a chunk as rows and the query heads
//     as 8 columns, then O^T += V^T P^T with D as rows; K/V tiles arrive
//     128-byte swizzled so ldmatrix reads them without bank conflicts, and P
//     is transposed in registers with movmatrix.  Accumulation is float32; P
//     is rounded to the cache's 16-bit type for the second product, and the
//     softmax denominator sums the same rounded weights.
// * Online softmax keeps a reference max m, moved only when a score exceeds
//   it by more than kTau = 8 (base-2 units): exp2(score - m) stays <= 256 and
//   the final division by l cancels the choice of m exactly, so accumulator
//   rescaling is rare.
// * With partitions, each unit writes its (m, l, unnormalised output) in
//   float32 and reduce_kernel merges them; it is launched as a programmatic
//   dependent of the decode kernel, so its CTAs are resident before the
//   decode grid drains and start the moment its writes are visible.
//   Sequences that fit in one partition are written out directly.  (Merging
//   inside the decode kernel -- the last partition of a head merges -- was
//   measured 8 % slower: the merging warp stalls its CTA's pipeline.)
#ifndef PAGEDATTN_DECODE_CUH
#define PAGEDATTN_DECODE_CUH

#include <cuda.h>
#include <cstdint>

#include "dtype.cuh"
#include "ptx.cuh"

namespace pa {

constexpr int kChunkTokens = 16;      // tokens per pipeline stage
constexpr float kTau = 8.0f;          // allowed growth of a score over the reference max (base 2)
constexpr int kMaxTileHeads = 8;      // KV heads per CTA tile (consumer warps)
constexpr int kSwizzleBytes = 128;    // TMA swizzle span of the tensor-core path
constexpr int kSmemAlign = 1024;      // alignment of the stage ring (swizzle atom)

struct DecodeParams {
  const void* q;                 // [S][Hq][D]
  const int32_t* block_tables;   // [S][MB]
  const int32_t* context_lens;   // [S]
  void* out;                     // [S][Hq][D]
  float* part_acc;               // [S][Hq][NP][D]   (partitioned mode)
  float2* part_ml;               // [S][Hq][NP]      (m in base-2 units, l)
  int* sched;                    // [0] unit counter, [1] planned units, [2] CTAs that take units (plan_kernel)
  const int4* units;             // planned unit list {seq, part, tile, len}, or null: walk the sequences
  int table_stride;              // elements between rows of block_tables (>= max_blocks)
  int part_offset;               // partial index of partition 0 (shared-prefix mode)
  int force_partials;            // write partials even for single-partition sequences
  int num_seqs, num_q_heads, num_kv_heads;
  int max_blocks, block_size, num_blocks;
  int partition_size;            // 0 = whole context in one unit
  int max_parts;                 // NP
  int tile_heads;                // HT
  int num_tiles;                 // Hkv / HT
  int stages;
  uint32_t tile_bytes;           // bytes of one K (or V) stage tile
  uint32_t q_bytes;              // bytes of one unit's query rows
  float qk_scale;                // scale * log2(e)
  uint64_t wait_limit_ns;        // bound of every pipeline wait (kWaitLimitNs unless a test shortens it)
  int withhold_first;            // test hook, 0 in every normal call: see pa_debug_decode_stall
};

struct StageMeta {
  int seq, part, tile, ntok, flags, nparts, qslot, pad;
};
constexpr int kFirst = 1, kLast = 2;

__device__ __forceinline__ int parts_of(int len, int psize) {
  return (psize > 0 && len > 0) ? (len + psize - 1) / psize : 1;
}

// Bytes of dynamic shared memory the pipeline layout needs.
__host__ __device__ constexpr size_t pipeline_smem_bytes(int stages, size_t tile_bytes, size_t q_bytes) {
  return kSmemAlign + stages * (2 * tile_bytes + sizeof(StageMeta) + 2 * sizeof(uint64_t)) + 2 * q_bytes +
         4 * sizeof(uint64_t) + 16;
}

// Shared-memory layout of both kernels: K ring, V ring, query double buffer,
// stage metadata, barriers, abort flag.  The rings start 1 KB aligned.
template <typename T, int D, int G>
struct Pipeline {
  T* s_k;
  T* s_v;
  T* s_q;
  StageMeta* meta;
  uint64_t* full;
  uint64_t* empty;
  uint64_t* q_full;
  uint64_t* q_empty;
  volatile int* abort_flag;
  int stages, ht, tile_elems;

  __device__ __forceinline__ Pipeline(unsigned char* raw, const DecodeParams& prm) {
    const uintptr_t base =
        (reinterpret_cast<uintptr_t>(raw) + kSmemAlign - 1) & ~static_cast<uintptr_t>(kSmemAlign - 1);
    ht = prm.tile_heads;
    stages = prm.stages;
    tile_elems = kChunkTokens * ht * D;
    s_k = reinterpret_cast<T*>(base);
    s_v = s_k + stages * tile_elems;
    s_q = s_v + stages * tile_elems;
    meta = reinterpret_cast<StageMeta*>(s_q + 2 * ht * G * D);
    full = reinterpret_cast<uint64_t*>(meta + stages);
    empty = full + stages;
    q_full = empty + stages;
    q_empty = q_full + 2;
    abort_flag = reinterpret_cast<volatile int*>(q_empty + 2);
  }

  __device__ __forceinline__ void init() {
    for (int i = 0; i < stages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], ht);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], ht);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
};

// Producer warp: walks this CTA's units and fills the stage ring.
// kSwizzled: one TMA box of 16 tokens x 128 bytes (128B-swizzled) per
// (head, 128-byte column block of D) -- the layout the tensor-core consumer
// reads; otherwise one box of 16 tokens x HT heads x D per K and per V tile.
template <typename T, int D, int G, bool kSwizzled>
__device__ __forceinline__ void run_producer(Pipeline<T, D, G>& pl, const DecodeParams& prm,
                                             const CUtensorMap* tm_k, const CUtensorMap* tm_v, int lane) {
  constexpr int kHalves = D * static_cast<int>(sizeof(T)) / kSwizzleBytes;
  constexpr int kBoxElems = kSwizzleBytes / static_cast<int>(sizeof(T));
  if (lane == 0) {
    prefetch_tensormap(tm_k);
    prefetch_tensormap(tm_v);
  }
  const uint64_t policy = policy_evict_first();
  const int S = prm.num_seqs;
  const int MB = prm.max_blocks;
  const int BS = prm.block_size;
  const int cap = MB * BS;
  const int P = prm.partition_size;
  const int n_tiles = prm.num_tiles;
  const int HT = pl.ht;
  const int stages = pl.stages;

  // Units come in two passes over the sequences: pass 0 holds every full
  // partition (the whole sequence when P == 0), pass 1 every remainder
  // partition (and the single unit of an empty sequence).  A window of 32
  // sequences is walked at a time: lane i holds sequence win_s0 + i.
  int pass = 0;
  int win_s0 = 0, win_base = 0;
  int my_len = 0, my_units = 0, my_incl = 0, win_total = 0;
  auto load_window = [&]() {
    const int s = win_s0 + lane;
    my_len = 0;
    my_units = 0;
    if (s < S) {
      int len = prm.context_lens[s];
      if (len > cap || len < 0) {
        if (pass == 0) set_device_error(DEVERR_BAD_LENGTH);
        len = len < 0 ? 0 : cap;
      }
      my_len = len;
      int n;
      if (P == 0) {
        n = pass == 0 ? 1 : 0;
      } else if (pass == 0) {
        n = len / P;
      } else {
        n = (len % P != 0 || len == 0) ? 1 : 0;
      }
      my_units = n * n_tiles;
    }
    my_incl = my_units;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, my_incl, off);
      if (lane >= off) my_incl += v;
    }
    win_total = __shfl_sync(0xffffffffu, my_incl, 31);
  };
  if (prm.units == nullptr) load_window();

  int stage = 0;
  uint32_t phase = 0;
  int units_done = 0;
  long long armed = 0;               // stages armed so far (for the drain at exit)
  int q_issued = 0;                  // query copies issued so far
  int tw_seq = -1, tw_base = -1, tw_val = 0;
  bool ok = true;

  // Planned order: claim the next unit index and fetch its descriptor one
  // unit ahead (lane 0), so both round trips overlap the current unit.  The
  // plan lists (sequence, partition) entries; unit c is KV-head tile c % n_tiles
  // of entry c / n_tiles, so the tiles of one partition are taken together.
  const bool planned = prm.units != nullptr;
  int total_units = 0;
  int4 next_desc = make_int4(-1, 0, 0, 0);
  auto claim = [&]() {
    int4 d = make_int4(-1, 0, 0, 0);
    if (lane == 0) {
      const int c = atomicAdd(prm.sched, 1);
      if (c < total_units) {
        const int e = c / n_tiles;
        d = __ldcg(prm.units + e);
        d.z = c - e * n_tiles;
      }
    }
    return d;
  };
  if (planned) {
    wait_prerequisite_grids();                       // the plan is complete and visible
    // CTAs beyond the planner's working grid take no units
    if (lane == 0) total_units = static_cast<int>(blockIdx.x) < __ldcg(prm.sched + 2) ? __ldcg(prm.sched + 1) : 0;
    total_units = __shfl_sync(0xffffffffu, total_units, 0);
    if (total_units > 0) next_desc = claim();
  }
  int rr = blockIdx.x;

  while (ok) {
    int seq, len, part, tile;
    if (planned) {
      const int4 d = make_int4(__shfl_sync(0xffffffffu, next_desc.x, 0), __shfl_sync(0xffffffffu, next_desc.y, 0),
                               __shfl_sync(0xffffffffu, next_desc.z, 0), __shfl_sync(0xffffffffu, next_desc.w, 0));
      if (d.x < 0) break;
      next_desc = claim();
      seq = d.x;
      part = d.y;
      tile = d.z;
      len = d.w;
    } else {
      const int u = rr;
      rr += gridDim.x;
      bool exhausted = false;
      while (u >= win_base + win_total) {
        win_base += win_total;
        win_s0 += 32;
        if (win_s0 >= S) {
          if (pass == 1) {
            exhausted = true;
            break;
          }
          pass = 1;
          win_s0 = 0;
        }
        load_window();
      }
      if (exhausted) break;
      const unsigned hit = __ballot_sync(0xffffffffu, win_base + my_incl > u);
      const int hl = __ffs(hit) - 1;
      seq = win_s0 + hl;
      len = __shfl_sync(0xffffffffu, my_len, hl);
      const int excl = __shfl_sync(0xffffffffu, my_incl - my_units, hl);
      const int r = u - (win_base + excl);
      if (pass == 0) {
        part = r / n_tiles;
        tile = r - part * n_tiles;
      } else {
        part = len / P;
        tile = r;
      }
    }
    const int nparts = parts_of(len, P);
    const int tok_begin = P > 0 ? part * P : 0;
    const int tok_end = P > 0 ? min(len, tok_begin + P) : len;
    const int nchunks = max(1, (tok_end - tok_begin + kChunkTokens - 1) / kChunkTokens);
    const int qslot = units_done & 1;

    // Query rows of this unit: [HT*G][D] contiguous in q.
    if (!__all_sync(0xffffffffu,
                    mbar_wait(&pl.q_empty[qslot], ((units_done >> 1) & 1) ^ 1, pl.abort_flag, prm.wait_limit_ns))) {
      ok = false;
      break;
    }
    ++q_issued;
    if (lane == 0) {
      const char* src = static_cast<const char*>(prm.q) +
                        (static_cast<size_t>(seq) * prm.num_q_heads + static_cast<size_t>(tile) * HT * G) * D *
                            sizeof(T);
      mbar_arrive_expect_tx(&pl.q_full[qslot], prm.q_bytes);
      bulk_load(pl.s_q + qslot * HT * G * D, src, prm.q_bytes, &pl.q_full[qslot]);
    }

    for (int c = 0; c < nchunks; ++c) {
      const int tok = tok_begin + c * kChunkTokens;
      const int ntok = max(0, min(kChunkTokens, tok_end - tok));
      // A chunk is one 16-row piece of one block, or, with 8-token blocks,
      // two 8-row pieces of two logically consecutive blocks.
      const int piece_rows = BS < kChunkTokens ? BS : kChunkTokens;
      const int npieces = kChunkTokens / piece_rows;
      int rows[2] = {0, 0};
      int loaded = 0;
      for (int pc = 0; pc < npieces; ++pc) {
        const int t0 = tok + pc * piece_rows;
        if (t0 >= tok_end) break;
        const int blk = t0 / BS;
        const int within = t0 - blk * BS;
        const int wb = blk & ~31;
        if (seq != tw_seq || wb != tw_base) {
          tw_seq = seq;
          tw_base = wb;
          const int idx = wb + lane;
          tw_val = idx < MB ? prm.block_tables[static_cast<size_t>(seq) * prm.table_stride + idx] : 0;
        }
        int phys = __shfl_sync(0xffffffffu, tw_val, blk - wb);
        if (phys < 0 || phys >= prm.num_blocks) {
          if (lane == 0) set_device_error(DEVERR_BAD_BLOCK_ID);
          phys = 0;
        }
        rows[pc] = phys * BS + within;
        loaded = pc + 1;
      }
      if (!__all_sync(0xffffffffu, mbar_wait(&pl.empty[stage], phase ^ 1, pl.abort_flag, prm.wait_limit_ns))) {
        ok = false;
        break;
      }
      // test hook: the first arming of the CTA is never made, so the consumers'
      // wait for it runs out (never set in a normal call)
      const bool withhold = prm.withhold_first && armed == 0;
      if (lane == 0 && !withhold) {
        StageMeta m;
        m.seq = seq;
        m.part = part;
        m.tile = tile;
        m.ntok = ntok;
        m.flags = (c == 0 ? kFirst : 0) | (c == nchunks - 1 ? kLast : 0);
        m.nparts = nparts;
        m.qslot = qslot;
        m.pad = 0;
        pl.meta[stage] = m;
        if (loaded > 0) {
          mbar_arrive_expect_tx(&pl.full[stage], 2 * prm.tile_bytes / npieces * loaded);
        } else {
          mbar_arrive(&pl.full[stage]);
        }
      }
      __syncwarp();
      if (loaded > 0 && !withhold) {
        T* dk = pl.s_k + stage * pl.tile_elems;
        T* dv = pl.s_v + stage * pl.tile_elems;
        if constexpr (kSwizzled) {
          // lanes split the loaded pieces' K and V boxes, one per (head, column block)
          const int nbox = HT * kHalves;
          for (int b = lane; b < loaded * 2 * nbox; b += 32) {
            const int pc = b / (2 * nbox);
            const int r = b - pc * 2 * nbox;
            const int kv = r >= nbox ? 1 : 0;
            const int hb = r - kv * nbox;                 // head-in-tile * kHalves + column block
            T* dst = (kv ? dv : dk) + hb * kChunkTokens * kBoxElems + pc * piece_rows * kBoxElems;
            tma_load_3d(dst, kv ? tm_v : tm_k, &pl.full[stage], 0, tile * HT * kHalves + hb, rows[pc], policy);
          }
        } else {
          if (lane < 2 * loaded) {
            const int pc = lane >> 1;
            const int kv = lane & 1;
            T* dst = (kv ? dv : dk) + pc * piece_rows * HT * D;
            tma_load_3d(dst, kv ? tm_v : tm_k, &pl.full[stage], 0, tile * HT, rows[pc], policy);
          }
        }
      }
      ++armed;
      if (++stage == stages) {
        stage = 0;
        phase ^= 1;
      }
    }
    ++units_done;
  }

  if (ok) {
    // End-of-work marker for the consumers.
    if (__all_sync(0xffffffffu, mbar_wait(&pl.empty[stage], phase ^ 1, pl.abort_flag, prm.wait_limit_ns))) {
      if (lane == 0 && !(prm.withhold_first && armed == 0)) {
        pl.meta[stage].seq = -1;
        mbar_arrive(&pl.full[stage]);
      }
      __syncwarp();
      // the marker is an arming of this stage too: the drain below walks
      // back from the newest arming of every stage
      ++armed;
      if (++stage == stages) {
        stage = 0;
        phase ^= 1;
      }
    }
  }
  // Drain: every tile or query copy issued must have landed before exit.
  if (lane == 0) {
    int st = stage, ph = phase;
    const long long back = armed < stages ? armed : stages;
    for (long long k = 0; k < back; ++k) {
      if (--st < 0) {
        st = stages - 1;
        ph ^= 1;
      }
      mbar_wait_drain(&pl.full[st], ph, prm.wait_limit_ns);
    }
    for (int k = 1; k <= 2 && k <= q_issued; ++k) {
      const int un = q_issued - k;
      mbar_wait_drain(&pl.q_full[un & 1], (un >> 1) & 1, prm.wait_limit_ns);
    }
  }
  __syncwarp();
}

// ===========================================================================
// CUDA-core consumer
// ===========================================================================

// Lanes per token for a head size / group size: enough that the per-lane
// q + accumulator registers (2*G*D/L floats) stay at or below 128.
template <int D, int G>
struct Lanes {
  static constexpr int L = (D * G / 64 > 8) ? D * G / 64 : 8;
  static_assert(L <= 32 && (32 % L) == 0, "unsupported head_dim / group size");
};

template <typename T, int D, int G>
// 8 consumer warps + 1 producer: three warps share one SM sub-partition, whose
// 16K-register file caps a thread at 168 registers.
__global__ void __launch_bounds__((kMaxTileHeads + 1) * 32, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const DecodeParams prm) {
  constexpr int L = Lanes<D, G>::L;       // lanes per token
  constexpr int NG = 32 / L;              // tokens in flight per warp
  constexpr int E = D / L;                // elements per lane
  constexpr int EPC = Chunk<T>::kElems;   // elements per 16-byte chunk
  constexpr int NCH = E / EPC;            // chunks per lane
  static_assert(NCH >= 1 && E % EPC == 0, "lane slice must be whole 16-byte chunks");

  extern __shared__ __align__(1024) unsigned char smem[];
  Pipeline<T, D, G> pl(smem, prm);
  const int HT = pl.ht;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) pl.init();
  __syncthreads();
  allow_dependent_launch();

  if (warp == HT) {
    run_producer<T, D, G, false>(pl, prm, &tm_k, &tm_v, lane);
    return;
  }

  const int j = warp;                 // KV head within the tile
  const int grp = lane / L;           // token group
  const int li = lane % L;            // lane within the group

  float2 qv[G][E / 2];
  float2 acc[G][E / 2];
  float m[G], l[G];

  int stage = 0;
  uint32_t phase = 0;
  int units_done = 0;

  while (true) {
    if (!__all_sync(0xffffffffu, mbar_wait(&pl.full[stage], phase, pl.abort_flag, prm.wait_limit_ns))) return;
    const StageMeta mt = pl.meta[stage];
    if (mt.seq < 0) return;

    if (mt.flags & kFirst) {
      if (!__all_sync(0xffffffffu,
                      mbar_wait(&pl.q_full[mt.qslot], (units_done >> 1) & 1, pl.abort_flag, prm.wait_limit_ns)))
        return;
      const T* qrow = pl.s_q + mt.qslot * HT * G * D + j * G * D;
#pragma unroll
      for (int g = 0; g < G; ++g) {
#pragma unroll
        for (int k = 0; k < NCH; ++k) {
          Chunk<T>::load(qrow + g * D + (li + k * L) * EPC, &qv[g][k * EPC / 2]);
        }
#pragma unroll
        for (int e = 0; e < E / 2; ++e) fmul2(qv[g][e], make_float2(prm.qk_scale, prm.qk_scale));
        m[g] = -INFINITY;
        l[g] = 0.f;
#pragma unroll
        for (int e = 0; e < E / 2; ++e) acc[g][e] = make_float2(0.f, 0.f);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&pl.q_empty[mt.qslot]);
    }

    if (mt.ntok > 0) {
      const T* kt = pl.s_k + stage * pl.tile_elems + j * D;
      const T* vt = pl.s_v + stage * pl.tile_elems + j * D;
      const int npass = (mt.ntok + NG - 1) / NG;
#pragma unroll 1
      for (int pass = 0; pass < npass; ++pass) {
        const int t = pass * NG + grp;
        const bool valid = t < mt.ntok;
        const T* krow = kt + t * HT * D;
        float2 kf[E / 2];
#pragma unroll
        for (int k = 0; k < NCH; ++k) Chunk<T>::load(krow + (li + k * L) * EPC, &kf[k * EPC / 2]);
        float dot[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
          float2 d2 = make_float2(0.f, 0.f);
#pragma unroll
          for (int e = 0; e < E / 2; ++e) ffma2(d2, qv[g][e], kf[e]);
          dot[g] = d2.x + d2.y;
        }
#pragma unroll
        for (int off = L / 2; off >= 1; off >>= 1) {
#pragma unroll
          for (int g = 0; g < G; ++g) dot[g] += __shfl_xor_sync(0xffffffffu, dot[g], off);
        }
        if (valid) {
          const T* vrow = vt + t * HT * D;
          float2 vf[E / 2];
#pragma unroll
          for (int k = 0; k < NCH; ++k) Chunk<T>::load(vrow + (li + k * L) * EPC, &vf[k * EPC / 2]);
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float sc = dot[g];
            if (sc > m[g] + kTau) {
              const float f = exp2_approx(m[g] - sc);
              l[g] *= f;
#pragma unroll
              for (int e = 0; e < E / 2; ++e) fmul2(acc[g][e], make_float2(f, f));
              m[g] = sc;
            }
            const float p = exp2_approx(sc - m[g]);
            l[g] += p;
#pragma unroll
            for (int e = 0; e < E / 2; ++e) ffma2(acc[g][e], make_float2(p, p), vf[e]);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&pl.empty[stage]);
    if (++stage == pl.stages) {
      stage = 0;
      phase ^= 1;
    }

    if (mt.flags & kLast) {
      // Merge the token groups of this warp (xor over the group bits).
#pragma unroll
      for (int off = L; off < 32; off <<= 1) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float mo = __shfl_xor_sync(0xffffffffu, m[g], off);
          const float lo = __shfl_xor_sync(0xffffffffu, l[g], off);
          const float mx = fmaxf(m[g], mo);
          const float ref = (mx == -INFINITY) ? 0.f : mx;
          const float fa = exp2_approx(m[g] - ref);
          const float fb = exp2_approx(mo - ref);
          l[g] = l[g] * fa + lo * fb;
#pragma unroll
          for (int e = 0; e < E / 2; ++e) {
            float2 o;
            o.x = __shfl_xor_sync(0xffffffffu, acc[g][e].x, off);
            o.y = __shfl_xor_sync(0xffffffffu, acc[g][e].y, off);
            fmul2(acc[g][e], make_float2(fa, fa));
            ffma2(acc[g][e], make_float2(fb, fb), o);
          }
          m[g] = mx;
        }
      }
      // Every group now holds the merged state; group `grp` writes heads g = grp (mod NG).
      const int hq0 = (mt.tile * HT + j) * G;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        if (g % NG != grp) continue;
        const int hq = hq0 + g;
        if (mt.nparts == 1 && !prm.force_partials) {
          const float inv = l[g] > 0.f ? 1.0f / l[g] : 0.f;
          T* orow = static_cast<T*>(prm.out) + (static_cast<size_t>(mt.seq) * prm.num_q_heads + hq) * D;
#pragma unroll
          for (int k = 0; k < NCH; ++k) {
            float2 o[EPC / 2];
#pragma unroll
            for (int e = 0; e < EPC / 2; ++e) {
              o[e] = acc[g][k * EPC / 2 + e];
              fmul2(o[e], make_float2(inv, inv));
            }
            Chunk<T>::store(orow + (li + k * L) * EPC, o);
          }
        } else {
          const size_t pidx =
              (static_cast<size_t>(mt.seq) * prm.num_q_heads + hq) * prm.max_parts + prm.part_offset + mt.part;
          float* prow = prm.part_acc + pidx * D;
#pragma unroll
          for (int k = 0; k < NCH; ++k) {
            float4* dst = reinterpret_cast<float4*>(prow + (li + k * L) * EPC);
#pragma unroll
            for (int e = 0; e < EPC / 4; ++e) {
              const float2 a = acc[g][k * EPC / 2 + 2 * e];
              const float2 b = acc[g][k * EPC / 2 + 2 * e + 1];
              dst[e] = make_float4(a.x, a.y, b.x, b.y);
            }
          }
          if (li == 0) prm.part_ml[pidx] = make_float2(m[g], l[g]);
        }
      }
      ++units_done;
    }
  }
}

// ===========================================================================
// Tensor-core consumer (16-bit caches)
// ===========================================================================

template <typename T>
struct MmaType;
template <>
struct MmaType<__nv_bfloat16> {
  __device__ __forceinline__ static void mma(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
  // (lo, hi) -> packed pair, rounded to nearest even
  __device__ __forceinline__ static uint32_t pack(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
  }
  __device__ __forceinline__ static float2 unpack(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
  }
};
template <>
struct MmaType<__half> {
  __device__ __forceinline__ static void mma(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
  __device__ __forceinline__ static uint32_t pack(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
  }
  __device__ __forceinline__ static float2 unpack(uint32_t w) {
    return __half22float2(*reinterpret_cast<const __half2*>(&w));
  }
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                              uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// Transpose of an 8x8 16-bit matrix held one row pair per thread.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// Byte offset, inside one 16-token x 128-byte swizzled box, of 16-byte chunk
// `chunk` of token row `tok` (128B swizzle: chunk ^= row mod 8).
__device__ __forceinline__ uint32_t swz(int tok, int chunk) {
  return static_cast<uint32_t>(tok * kSwizzleBytes + ((chunk ^ (tok & 7)) << 4));
}

// 128 registers: eight 64-thread CTAs (the default launch shape) fill the
// register file exactly.
template <typename T, int D, int G>
__global__ void __maxnreg__(128)
    decode_mma_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                      const DecodeParams prm) {
  static_assert(sizeof(T) == 2, "tensor-core consumer takes 16-bit caches");
  static_assert(G >= 1 && G <= 8, "query heads per KV head must fit the 8 MMA columns");
  constexpr int kHalves = D * 2 / kSwizzleBytes;            // 64-element column blocks
  constexpr int kBoxBytes = kChunkTokens * kSwizzleBytes;   // one swizzled box (2 KB)
  constexpr int KSTEPS = D / 16;                            // k-steps of S^T = K Q^T
  constexpr int MTILES = D / 16;                            // m-tiles of O^T = V^T P^T
  using M = MmaType<T>;

  extern __shared__ __align__(1024) unsigned char smem[];
  Pipeline<T, D, G> pl(smem, prm);
  const int HT = pl.ht;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) pl.init();
  __syncthreads();
  allow_dependent_launch();

  if (warp == HT) {
    run_producer<T, D, G, true>(pl, prm, &tm_k, &tm_v, lane);
    return;
  }

  const int j = warp;              // KV head within the tile
  const int gq = lane >> 2;        // fragment row group
  const int tq = lane & 3;         // fragment column pair
  const int h0 = 2 * tq;           // this thread's two query-head columns h0, h0 + 1

  // ldmatrix row addresses.  QK (A = K, rows = tokens): matrix i = lane/8
  // covers tokens 8*(i%2).., column chunk i/2.  PV (A = V^T through .trans):
  // matrix i covers tokens 8*(i/2).., column chunk i%2.
  const int qk_tok = (lane & 7) + ((lane >> 3) & 1) * 8;
  const int qk_chk = lane >> 4;
  const int pv_tok = (lane & 7) + (lane >> 4) * 8;
  const int pv_chk = (lane >> 3) & 1;

  uint32_t qf[KSTEPS][2];          // B fragments of Q^T (query heads as the 8 columns)
  float o[MTILES][4];              // O^T accumulators: rows D, columns heads
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

  const uint32_t s_k0 = smem_addr(pl.s_k) + j * kHalves * kBoxBytes;
  const uint32_t s_v0 = smem_addr(pl.s_v) + j * kHalves * kBoxBytes;
  const uint32_t tile_bytes = prm.tile_bytes;

  int stage = 0;
  uint32_t phase = 0;
  int units_done = 0;

  while (true) {
    if (!__all_sync(0xffffffffu, mbar_wait(&pl.full[stage], phase, pl.abort_flag, prm.wait_limit_ns))) return;
    const StageMeta mt = pl.meta[stage];
    if (mt.seq < 0) return;

    if (mt.flags & kFirst) {
      if (!__all_sync(0xffffffffu,
                      mbar_wait(&pl.q_full[mt.qslot], (units_done >> 1) & 1, pl.abort_flag, prm.wait_limit_ns)))
        return;
      const T* qbase = pl.s_q + mt.qslot * HT * G * D + j * G * D;
#pragma unroll
      for (int kk = 0; kk < KSTEPS; ++kk) {
        if (gq < G) {
          const uint32_t* row = reinterpret_cast<const uint32_t*>(qbase + gq * D + kk * 16);
          qf[kk][0] = row[tq];
          qf[kk][1] = row[tq + 4];
        } else {
          qf[kk][0] = 0u;
          qf[kk][1] = 0u;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&pl.q_empty[mt.qslot]);
#pragma unroll
      for (int i = 0; i < MTILES; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
      m0 = m1 = -INFINITY;
      l0 = l1 = 0.f;
    }

    if (mt.ntok > 0) {
      const uint32_t kb = s_k0 + stage * tile_bytes;
      const uint32_t vb = s_v0 + stage * tile_bytes;
      // S^T[16 tokens][8 heads] = K Q^T
      float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int kk = 0; kk < KSTEPS; ++kk) {
        const int blk = (kk * 16) / 64;
        const int chunk = ((kk * 16) % 64) / 8 + qk_chk;
        uint32_t a0, a1, a2, a3;
        ldsm_x4(kb + blk * kBoxBytes + swz(qk_tok, chunk), a0, a1, a2, a3);
        M::mma(s, a0, a1, a2, a3, qf[kk][0], qf[kk][1]);
      }
      // scores in base-2 units; tokens gq, gq+8 beyond the chunk are masked
      const bool v_lo = gq < mt.ntok;
      const bool v_hi = gq + 8 < mt.ntok;
      const float x0 = v_lo ? s[0] * prm.qk_scale : -INFINITY;
      const float x1 = v_lo ? s[1] * prm.qk_scale : -INFINITY;
      const float x2 = v_hi ? s[2] * prm.qk_scale : -INFINITY;
      const float x3 = v_hi ? s[3] * prm.qk_scale : -INFINITY;
      const bool over = (x0 > m0 + kTau) | (x2 > m0 + kTau) | (x1 > m1 + kTau) | (x3 > m1 + kTau);
      if (__any_sync(0xffffffffu, over)) {
        // column maxima over the chunk's 16 tokens (the 8 lanes sharing tq)
        float c0 = fmaxf(x0, x2), c1 = fmaxf(x1, x3);
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
          c0 = fmaxf(c0, __shfl_xor_sync(0xffffffffu, c0, off));
          c1 = fmaxf(c1, __shfl_xor_sync(0xffffffffu, c1, off));
        }
        const float n0 = c0 > m0 + kTau ? c0 : m0;
        const float n1 = c1 > m1 + kTau ? c1 : m1;
        const float f0 = exp2_approx(m0 - n0);
        const float f1 = exp2_approx(m1 - n1);
        l0 *= f0;
        l1 *= f1;
#pragma unroll
        for (int i = 0; i < MTILES; ++i) {
          o[i][0] *= f0;
          o[i][1] *= f1;
          o[i][2] *= f0;
          o[i][3] *= f1;
        }
        m0 = n0;
        m1 = n1;
      }
      // P^T rounded to the 16-bit type; the denominator sums the same rounded values
      const uint32_t p_lo = M::pack(exp2_approx(x0 - m0), exp2_approx(x1 - m1));   // token gq
      const uint32_t p_hi = M::pack(exp2_approx(x2 - m0), exp2_approx(x3 - m1));   // token gq + 8
      const float2 r_lo = M::unpack(p_lo), r_hi = M::unpack(p_hi);
      l0 += r_lo.x + r_hi.x;
      l1 += r_lo.y + r_hi.y;
      const uint32_t b0 = movmatrix_trans(p_lo);     // P^T tokens 0-7 as B (k = tokens, n = heads)
      const uint32_t b1 = movmatrix_trans(p_hi);     // P^T tokens 8-15
      // rows of V beyond the chunk may hold anything: zero them in the fragments
      uint32_t mlo = 0xffffffffu, mhi = 0xffffffffu;
      if (mt.ntok < kChunkTokens) {
        mlo = (2 * tq < mt.ntok ? 0x0000ffffu : 0u) | (2 * tq + 1 < mt.ntok ? 0xffff0000u : 0u);
        mhi = (2 * tq + 8 < mt.ntok ? 0x0000ffffu : 0u) | (2 * tq + 9 < mt.ntok ? 0xffff0000u : 0u);
      }
      // O^T[D][heads] += V^T P^T
#pragma unroll
      for (int i = 0; i < MTILES; ++i) {
        const int blk = (i * 16) / 64;
        const int chunk = ((i * 16) % 64) / 8 + pv_chk;
        uint32_t a0, a1, a2, a3;
        ldsm_x4_trans(vb + blk * kBoxBytes + swz(pv_tok, chunk), a0, a1, a2, a3);
        M::mma(o[i], a0 & mlo, a1 & mlo, a2 & mhi, a3 & mhi, b0, b1);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&pl.empty[stage]);
    if (++stage == pl.stages) {
      stage = 0;
      phase ^= 1;
    }

    if (mt.flags & kLast) {
      // full column sums of l over the 8 row groups
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, off);
        l1 += __shfl_xor_sync(0xffffffffu, l1, off);
      }
      const int hq0 = (mt.tile * HT + j) * G;
      const bool w0 = h0 < G, w1 = h0 + 1 < G;
      if (mt.nparts == 1 && !prm.force_partials) {
        const float i0 = l0 > 0.f ? 1.0f / l0 : 0.f;
        const float i1 = l1 > 0.f ? 1.0f / l1 : 0.f;
        T* r0 = static_cast<T*>(prm.out) + (static_cast<size_t>(mt.seq) * prm.num_q_heads + hq0 + h0) * D;
        T* r1 = r0 + D;
#pragma unroll
        for (int i = 0; i < MTILES; ++i) {
          const int d = i * 16 + gq;
          if (w0) {
            r0[d] = static_cast<T>(o[i][0] * i0);
            r0[d + 8] = static_cast<T>(o[i][2] * i0);
          }
          if (w1) {
            r1[d] = static_cast<T>(o[i][1] * i1);
            r1[d + 8] = static_cast<T>(o[i][3] * i1);
          }
        }
      } else {
        const size_t p0 =
            (static_cast<size_t>(mt.seq) * prm.num_q_heads + hq0 + h0) * prm.max_parts + prm.part_offset + mt.part;
        const size_t p1 = p0 + prm.max_parts;
        float* r0 = prm.part_acc + p0 * D;
        float* r1 = prm.part_acc + p1 * D;
#pragma unroll
        for (int i = 0; i < MTILES; ++i) {
          const int d = i * 16 + gq;
          if (w0) {
            r0[d] = o[i][0];
            r0[d + 8] = o[i][2];
          }
          if (w1) {
            r1[d] = o[i][1];
            r1[d + 8] = o[i][3];
          }
        }
        if (gq == 0) {
          if (w0) prm.part_ml[p0] = make_float2(m0, l0);
          if (w1) prm.part_ml[p1] = make_float2(m1, l1);
        }
      }
      ++units_done;
    }
  }
}

// ===========================================================================
// Planner: the decode kernel's work list, one entry {seq, part, -, len} per
// (sequence, partition); the decode grid expands each entry into its
// n_tiles KV-head tiles, taken one after another (they read the same
// blocks).  Full partitions first, in sequence order; then the remainder
// partitions -- or, without partitions, the whole sequences -- by decreasing
// length (counting sort on 16-token chunks), so the smallest units are taken
// last.  One CTA; also zeroes the unit counter and stores the unit count.
//
// It is launched as a programmatic dependent of the kernel before it on the
// stream and lets the decode grid launch at once (its CTAs set up and then
// wait for the planner), but it writes nothing before its own
// griddepcontrol.wait has returned, and trusts no length read before it.
// That wait matters twice over: the kernel before may be the previous call's
// decode grid, still claiming units from the same workspace (resetting the
// counter under it would hand it this call's units), or it may be the kernel
// that wrote the lengths.  For up to 4096 sequences the plan is worked out
// ahead of the wait from the lengths as they stand, then the lengths are read
// again after it and the plan is redone if any changed; larger batches wait
// first.
// ===========================================================================
struct PlanParams {
  const int32_t* context_lens;
  int4* units;                   // entries {seq, part, 0, len}, one per (sequence, partition)
  int* header;                   // [0] unit counter (zeroed), [1] unit count (entries x num_tiles),
                                 // [2] decode CTAs that take units
  int num_seqs, partition_size, num_tiles, cap;
  int num_ctas;                  // CTAs of the decode grid
  int balance;                   // size the working grid to whole waves of the largest unit
};

constexpr int kPlanThreads = 1024;
constexpr int kPlanBuckets = 4096;     // remainder sizes in 16-token chunks; longer ones share the last

// Exclusive prefix sum over the CTA; *total receives the sum.  All threads call it.
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += t;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    int w = lane < nw ? warp_sums[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, w, off);
      if (lane >= off) w += t;
    }
    if (lane < nw) warp_sums[lane] = w;       // inclusive warp totals
  }
  __syncthreads();
  const int before = warp > 0 ? warp_sums[warp - 1] : 0;
  *total = warp_sums[(blockDim.x >> 5) - 1];
  __syncthreads();
  return before + incl - v;
}

// Working grid for the decode kernel (written to header[2]): with units of
// equal size u, dynamic claiming by A CTAs ends after ceil(U / A) rounds,
// while HBM is shared by whichever CTAs are still busy: a last round that
// only some CTAs reach runs at the same per-CTA rate and wastes the rest.  So
// take k = ceil(U_eff / CTAs) rounds and A = ceil(U_eff / k) CTAs, U_eff =
// work / largest unit, keeping at least 7/8 of the grid busy (HBM stays
// saturated).  Only when the smaller remainder units are too few to fill
// that last round (fewer than one per CTA); otherwise they already do.
__device__ __forceinline__ int plan_working_grid(const PlanParams& prm, int rem_entries, int work_chunks,
                                                 int largest_chunks) {
  const int nt = prm.num_tiles;
  if (!prm.balance || static_cast<long long>(rem_entries) * nt >= prm.num_ctas) return prm.num_ctas;
  const long long work = static_cast<long long>(work_chunks) * nt;
  const long long ueff = (work + largest_chunks - 1) / largest_chunks;
  const long long k = (ueff + prm.num_ctas - 1) / prm.num_ctas;
  long long a = k > 0 ? (ueff + k - 1) / k : prm.num_ctas;
  const int floor_ctas = prm.num_ctas - prm.num_ctas / 8;
  a = a < floor_ctas ? floor_ctas : (a > prm.num_ctas ? prm.num_ctas : a);
  return static_cast<int>(a);
}

constexpr int kPlanSpecRounds = 4;     // batches of up to 4 x 1024 sequences are planned ahead of the wait

__global__ void __launch_bounds__(kPlanThreads) plan_kernel(const PlanParams prm) {
  __shared__ int bucket[kPlanBuckets];
  __shared__ int warp_sums[32];
  __shared__ int s_work, s_umax;
  allow_dependent_launch();                    // the decode grid may launch; it waits for this one
  const int tid = threadIdx.x;
  const int S = prm.num_seqs, P = prm.partition_size, nt = prm.num_tiles;
  const int rounds = (S + kPlanThreads - 1) / kPlanThreads;
  // lengths through L2 (never a line cached in L1 before the wait)
  auto load_len = [&](int s) {
    int len = __ldcg(prm.context_lens + s);
    return len < 0 ? 0 : (len > prm.cap ? prm.cap : len);
  };
  auto rem_bucket = [&](int len) {               // -1: no remainder unit
    int rem;
    if (P > 0) {
      if (len % P == 0 && len > 0) return -1;
      rem = len % P;
    } else {
      rem = len;
    }
    const int chunks = (rem + kChunkTokens - 1) / kChunkTokens;
    return chunks < kPlanBuckets ? chunks : kPlanBuckets - 1;
  };
  const int full_chunks = P / kChunkTokens;
  auto rem_chunks = [&](int len, int b) {
    return b >= 0 ? max(1, ((P > 0 ? len % P : len) + kChunkTokens - 1) / kChunkTokens) : 0;
  };
  // Bucket starts, largest remainders first: start[b] = written + sum_{b' > b}
  // count[b'] (each bucket counter becomes the cursor of its bucket).  Returns
  // the number of remainder entries.
  auto bucket_starts = [&](int written) {
    constexpr int PER = kPlanBuckets / kPlanThreads;
    int local[PER];
    int sum = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      local[i] = bucket[kPlanBuckets - 1 - (tid * PER + i)];   // reversed order
      sum += local[i];
    }
    int tot;
    const int off = block_exclusive_scan(sum, warp_sums, &tot);
    int run = off;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      bucket[kPlanBuckets - 1 - (tid * PER + i)] = written + run;
      run += local[i];
    }
    return tot;
  };
  auto reset = [&]() {
    for (int b = tid; b < kPlanBuckets; b += kPlanThreads) bucket[b] = 0;
    if (tid == 0) {
      s_work = 0;
      s_umax = 1;
    }
    __syncthreads();
  };

  if (rounds > kPlanSpecRounds) {
    // Large batch: wait for the kernel before first, then plan and write in
    // one sweep per 1024 sequences.
    wait_prerequisite_grids();
    reset();
    int written = 0, my_work = 0, my_umax = 0;
    for (int base = 0; base < S; base += kPlanThreads) {
      const int s = base + tid;
      int len = 0, nfull = 0;
      if (s < S) {
        len = load_len(s);
        nfull = P > 0 ? len / P : 0;
        const int b = rem_bucket(len);
        if (b >= 0) atomicAdd(&bucket[b], 1);
        my_work += nfull * full_chunks + rem_chunks(len, b);
        my_umax = max(my_umax, max(nfull > 0 ? full_chunks : 0, rem_chunks(len, b)));
      }
      int round_total;
      const int off = block_exclusive_scan(nfull, warp_sums, &round_total);
      for (int p = 0; p < nfull; ++p) prm.units[written + off + p] = make_int4(s, p, 0, len);
      written += round_total;
    }
    const int tot = bucket_starts(written);
    atomicAdd(&s_work, my_work);
    atomicMax(&s_umax, my_umax);
    __syncthreads();
    if (tid == 0) {
      prm.header[0] = 0;
      prm.header[1] = (written + tot) * nt;
      prm.header[2] = plan_working_grid(prm, tot, s_work, s_umax);
    }
    for (int s = tid; s < S; s += kPlanThreads) {
      const int len = load_len(s);
      const int b = rem_bucket(len);
      if (b < 0) continue;
      const int pos = atomicAdd(&bucket[b], 1);
      prm.units[pos] = make_int4(s, P > 0 ? len / P : 0, 0, len);
    }
    return;
  }

  // Up to 4096 sequences: the whole plan is worked out in registers from
  // lengths read before the kernel before has finished (that kernel may be an
  // append, which writes no length, or anything else on the stream); after
  // griddepcontrol.wait the lengths are read again, and if any changed the
  // plan is worked out once more.  Nothing is written before the wait.
  int len[kPlanSpecRounds], base_off[kPlanSpecRounds], pos[kPlanSpecRounds];
  int written = 0, tot = 0;
  bool waited = false;
  for (int attempt = 0; attempt < 2; ++attempt) {
    reset();
    written = 0;
    int my_work = 0, my_umax = 0;
#pragma unroll
    for (int r = 0; r < kPlanSpecRounds; ++r) {
      if (r >= rounds) break;
      const int s = r * kPlanThreads + tid;
      int nfull = 0;
      len[r] = 0;
      if (s < S) {
        len[r] = load_len(s);
        nfull = P > 0 ? len[r] / P : 0;
        const int b = rem_bucket(len[r]);
        if (b >= 0) atomicAdd(&bucket[b], 1);
        my_work += nfull * full_chunks + rem_chunks(len[r], b);
        my_umax = max(my_umax, max(nfull > 0 ? full_chunks : 0, rem_chunks(len[r], b)));
      }
      int round_total;
      base_off[r] = written + block_exclusive_scan(nfull, warp_sums, &round_total);
      written += round_total;
    }
    tot = bucket_starts(written);
    atomicAdd(&s_work, my_work);
    atomicMax(&s_umax, my_umax);
    __syncthreads();
#pragma unroll
    for (int r = 0; r < kPlanSpecRounds; ++r) {
      if (r >= rounds) break;
      const int s = r * kPlanThreads + tid;
      const int b = s < S ? rem_bucket(len[r]) : -1;
      pos[r] = b >= 0 ? atomicAdd(&bucket[b], 1) : -1;
    }
    if (waited) break;
    wait_prerequisite_grids();                 // the kernel before has finished and its writes are visible
    waited = true;
    bool changed = false;
#pragma unroll
    for (int r = 0; r < kPlanSpecRounds; ++r) {
      if (r >= rounds) break;
      const int s = r * kPlanThreads + tid;
      if (s < S && load_len(s) != len[r]) changed = true;
    }
    if (!__syncthreads_or(changed)) break;
  }
  if (tid == 0) {
    prm.header[0] = 0;
    prm.header[1] = (written + tot) * nt;
    prm.header[2] = plan_working_grid(prm, tot, s_work, s_umax);
  }
#pragma unroll
  for (int r = 0; r < kPlanSpecRounds; ++r) {
    if (r >= rounds) break;
    const int s = r * kPlanThreads + tid;
    if (s >= S) continue;
    const int nfull = P > 0 ? len[r] / P : 0;
    for (int p = 0; p < nfull; ++p) prm.units[base_off[r] + p] = make_int4(s, p, 0, len[r]);
    if (pos[r] >= 0) prm.units[pos[r]] = make_int4(s, P > 0 ? len[r] / P : 0, 0, len[r]);
  }
}

// The planner for batches of at most 32 sequences: the same list as
// plan_kernel (full partitions in sequence order, then one remainder entry
// per sequence, larger remainders first) worked out by one warp with
// shuffles, so the decode grid waits for one warp's loads and stores rather
// than a 1,024-thread block's scans.  Same speculative protocol: the plan is
// worked out from lengths read before griddepcontrol.wait, the lengths are
// read again after it, and the plan is redone if any changed; nothing is
// written before the wait.
constexpr int kPlanSmallSeqs = 32;

__global__ void __launch_bounds__(32) plan_small_kernel(const PlanParams prm) {
  allow_dependent_launch();                    // the decode grid may launch; it waits for this one
  const int lane = threadIdx.x;
  const int S = prm.num_seqs, P = prm.partition_size, nt = prm.num_tiles;
  const bool mine = lane < S;
  auto load_len = [&]() {
    int len = mine ? __ldcg(prm.context_lens + lane) : 0;
    return len < 0 ? 0 : (len > prm.cap ? prm.cap : len);
  };
  const int full_chunks = P / kChunkTokens;
  int len = 0, nfull = 0, base = 0, written = 0, pos = -1, tot = 0, work = 0, umax = 1;
  bool waited = false;
  for (int attempt = 0; attempt < 2; ++attempt) {
    len = load_len();
    nfull = P > 0 ? len / P : 0;
    // remainder bucket (16-token chunks, largest last bucket shared), -1 if none
    int key = -1, rc = 0;
    if (mine && !(P > 0 && len > 0 && len % P == 0)) {
      const int rem = P > 0 ? len % P : len;
      const int chunks = (rem + kChunkTokens - 1) / kChunkTokens;
      key = chunks < kPlanBuckets ? chunks : kPlanBuckets - 1;
      rc = chunks > 1 ? chunks : 1;
    }
    // full entries: exclusive scan of nfull over the lanes
    int incl = nfull;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += t;
    }
    base = incl - nfull;
    written = __shfl_sync(0xffffffffu, incl, 31);
    // remainder position: after every entry with a larger bucket, or the same bucket and a lower lane
    int rank = 0;
    for (int j = 0; j < 32; ++j) {
      const int kj = __shfl_sync(0xffffffffu, key, j);
      rank += (kj >= 0 && (kj > key || (kj == key && j < lane))) ? 1 : 0;
    }
    tot = __popc(__ballot_sync(0xffffffffu, key >= 0));
    pos = key >= 0 ? written + rank : -1;
    int w = nfull * full_chunks + rc;
    int um = max(nfull > 0 ? full_chunks : 0, rc);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
      w += __shfl_xor_sync(0xffffffffu, w, off);
      um = max(um, __shfl_xor_sync(0xffffffffu, um, off));
    }
    work = w;
    umax = um > 0 ? um : 1;
    if (waited) break;
    wait_prerequisite_grids();                 // the kernel before has finished and its writes are visible
    waited = true;
    if (!__any_sync(0xffffffffu, load_len() != len)) break;
  }
  if (lane == 0) {
    prm.header[0] = 0;
    prm.header[1] = (written + tot) * nt;
    prm.header[2] = plan_working_grid(prm, tot, work, umax);
  }
  if (mine) {
    for (int p = 0; p < nfull; ++p) prm.units[base + p] = make_int4(lane, p, 0, len);
    if (pos >= 0) prm.units[pos] = make_int4(lane, nfull, 0, len);
  }
}

// ===========================================================================
// Merge of per-partition partials: M = max m_p, w_p = 2^(m_p - M),
// out = sum_p w_p acc_p / sum_p w_p l_p.  A CTA of 8 warps covers 8 / W query
// heads of one sequence with W warps per head (W from the partition count the
// workspace allows: 1 up to 16 partitions, up to 8 for 33 or more); the W warps
// of a head each take every W-th partition, 4 or 6 rows at a time loaded
// together with the (m, l) pairs (one round of loads up to 6 W partitions;
// with shared-prefix slots the pairs first, and only the non-empty rows), and
// sum their parts through shared memory.  Sequences that fit one partition were
// written by the decode kernel and are skipped.  Launched as a programmatic
// dependent of the decode kernel: it reads nothing before griddepcontrol.wait
// has returned, i.e. before that grid (and so everything before it on the
// stream) has finished and its writes are visible.
// ===========================================================================
struct ReduceParams {
  const int32_t* context_lens;
  const float* part_acc;
  const float2* part_ml;
  void* out;
  int num_seqs, num_q_heads, partition_size, max_parts, cap;
  int part_offset;               // partials before partition 0 (shared-prefix splits); 0 otherwise
  int warps_per_head;            // 1, 2, 4 or 8
};

constexpr int kReduceWarps = 8;

// Warps per (sequence, head) for a partition count: one up to 16 partitions
// (8 heads per CTA: fewer, fuller CTAs; a Llama-3-shaped merge, mostly one or
// two partitions per sequence, measured 1 % faster than with two warps), then
// about eight partitions per warp.
__host__ __device__ constexpr int reduce_warps_per_head(int max_parts) {
  return max_parts <= 16 ? 1 : (max_parts <= 32 ? 4 : 8);
}

template <typename T, int D, int ROWS>
__global__ void __launch_bounds__(kReduceWarps * 32) reduce_kernel(const ReduceParams prm) {
  constexpr int PER = D / 32;                // contiguous elements per lane
  static_assert(PER % 2 == 0, "head_dim must be a multiple of 64");
  __shared__ float2 s_sum[kReduceWarps][D / 2];
  const int s = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wph = prm.warps_per_head;
  const int hq = blockIdx.x * (kReduceWarps / wph) + warp / wph;
  const int sub = warp & (wph - 1);
  const bool active = hq < prm.num_q_heads;
  const size_t base = (static_cast<size_t>(s) * prm.num_q_heads + (active ? hq : 0)) * prm.max_parts;
  const bool dense = prm.part_offset == 0;   // every slot below np holds a partition
  auto clamp_len = [&](int v) { return v < 0 ? 0 : (v > prm.cap ? prm.cap : v); };
  // the length as it stands (through L2) before the wait: only a guess, as
  // the kernel before the planner may still be writing it; checked below
  const int len_guess = dense ? clamp_len(__ldcg(prm.context_lens + s)) : 0;
  wait_prerequisite_grids();                 // the decode grid (and all before it) is done and visible
  // Dense calls: the first round of this warp's rows (sub, sub + wph, ...)
  // below the guessed partition count, their m and the first 64 (m, l) pairs
  // are loaded together with the length; if the length read after the wait
  // differs, the round is loaded again.
  constexpr int kMergeRows = ROWS;          // 6 for long contexts, 4 otherwise (registers: CTAs per SM)
  float2 v[kMergeRows][PER / 2];
  float mk[kMergeRows];
  float2 sw0 = make_float2(-INFINITY, 0.f), sw1 = make_float2(-INFINITY, 0.f);
  const int np_guess = parts_of(len_guess, prm.partition_size);
  auto load_round = [&](int npg) {
#pragma unroll
    for (int u = 0; u < kMergeRows; ++u) {
      const int pp = sub + wph * u;
      mk[u] = -INFINITY;
      if (pp < npg) {
        const float2* src = reinterpret_cast<const float2*>(prm.part_acc + (base + pp) * D + lane * PER);
#pragma unroll
        for (int e = 0; e < PER / 2; ++e) v[u][e] = src[e];
        mk[u] = prm.part_ml[base + pp].x;
      }
    }
    sw0 = lane < npg ? prm.part_ml[base + lane] : make_float2(-INFINITY, 0.f);
    sw1 = lane + 32 < npg ? prm.part_ml[base + lane + 32] : make_float2(-INFINITY, 0.f);
  };
  if (dense && active && np_guess > 1) load_round(np_guess);
  const int len = clamp_len(prm.context_lens[s]);
  const int np = prm.part_offset + parts_of(len, prm.partition_size);
  if (dense && np <= 1) return;              // the same for the whole CTA
  if (dense && active && np != np_guess) load_round(np);
  float2 o[PER / 2];
#pragma unroll
  for (int e = 0; e < PER / 2; ++e) o[e] = make_float2(0.f, 0.f);
  float mx = -INFINITY, lsum = 0.f;
  if (active && dense) {
    // M and L in one sweep of the (m, l) pairs (each lane keeps a running
    // maximum and a sum rescaled to it, and the lanes' pairs are merged the
    // same way); then this warp's rows, kMergeRows at a time (one round of
    // loads for a head with up to kMergeRows * wph partitions)
    auto take = [&](float2 ml) {
      if (ml.x > mx) {
        lsum = lsum * exp2_approx(mx - ml.x) + ml.y;     // exp2(-inf) = 0 on the first pair
        mx = ml.x;
      } else if (ml.x != -INFINITY) {
        lsum += ml.y * exp2_approx(ml.x - mx);
      }
    };
    take(sw0);                               // -inf past np
    take(sw1);
    for (int p = lane + 64; p < np; p += 32) take(prm.part_ml[base + p]);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
      const float mo = __shfl_xor_sync(0xffffffffu, mx, off);
      const float lo = __shfl_xor_sync(0xffffffffu, lsum, off);
      const float mn = fmaxf(mx, mo);
      lsum = (mx == -INFINITY ? 0.f : lsum * exp2_approx(mx - mn)) +
             (mo == -INFINITY ? 0.f : lo * exp2_approx(mo - mn));
      mx = mn;
    }
    if (mx == -INFINITY) mx = 0.f;          // no partition saw a token: all weights are 0
    const int K = np > sub ? (np - sub + wph - 1) / wph : 0;
    for (int k0 = 0; k0 < K; k0 += kMergeRows) {
      if (k0 > 0) {
#pragma unroll
        for (int u = 0; u < kMergeRows; ++u) {
          const int pp = sub + wph * (k0 + u);
          mk[u] = -INFINITY;
          if (k0 + u < K) {
            const float2* src = reinterpret_cast<const float2*>(prm.part_acc + (base + pp) * D + lane * PER);
#pragma unroll
            for (int e = 0; e < PER / 2; ++e) v[u][e] = src[e];
            mk[u] = prm.part_ml[base + pp].x;
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kMergeRows; ++u) {
        if (k0 + u < K && mk[u] != -INFINITY) {
          const float wu = exp2_approx(mk[u] - mx);
#pragma unroll
          for (int e = 0; e < PER / 2; ++e) ffma2(o[e], make_float2(wu, wu), v[u][e]);
        }
      }
    }
  } else if (active) {
    // Shared-prefix slots, most of them empty (m = -inf, left so by the
    // prefix kernel's segments): the (m, l) sweep first, then only the rows
    // of slots that hold tokens, found by a ballot.  Every warp of the head
    // computes M and L in one sweep as above; the pairs of the first 64 slots
    // stay in registers, so the rows of all their non-empty slots are loaded
    // in one round after the sweep.
    const float2 ml0 = lane < np ? prm.part_ml[base + lane] : make_float2(-INFINITY, 0.f);
    const float2 ml1 = lane + 32 < np ? prm.part_ml[base + lane + 32] : make_float2(-INFINITY, 0.f);
    auto take = [&](float2 ml) {
      if (ml.x > mx) {
        lsum = lsum * exp2_approx(mx - ml.x) + ml.y;     // exp2(-inf) = 0 on the first pair
        mx = ml.x;
      } else if (ml.x != -INFINITY) {
        lsum += ml.y * exp2_approx(ml.x - mx);
      }
    };
    take(ml0);
    take(ml1);
    for (int p = lane + 64; p < np; p += 32) take(prm.part_ml[base + p]);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
      const float mo = __shfl_xor_sync(0xffffffffu, mx, off);
      const float lo = __shfl_xor_sync(0xffffffffu, lsum, off);
      const float mn = fmaxf(mx, mo);
      lsum = (mx == -INFINITY ? 0.f : lsum * exp2_approx(mx - mn)) + (mo == -INFINITY ? 0.f : lo * exp2_approx(mo - mn));
      mx = mn;
    }
    if (mx == -INFINITY) mx = 0.f;          // no partition saw a token: all weights are 0
    // this warp's partitions sub, sub + wph, ... that hold tokens, four rows
    // in flight.  A partition with m = -inf holds none (a slot the
    // shared-prefix kernel left empty): it is found from a ballot over the
    // (m, l) pairs and its row is never read.
    const unsigned share = wph == 1 ? 0xffffffffu
                                    : (wph == 2 ? 0x55555555u : (wph == 4 ? 0x11111111u : 0x01010101u)) << sub;
    // slots 0..63: bit b of todo[c] is slot 32 c + b
    unsigned todo[2] = {__ballot_sync(0xffffffffu, ml0.x != -INFINITY) & share,
                        __ballot_sync(0xffffffffu, ml1.x != -INFINITY) & share};
    while (todo[0] | todo[1]) {
      int pk[4];
      int n = 0;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = todo[0] ? 0 : 1;
        pk[u] = -1;
        if (todo[c]) {
          pk[u] = 32 * c + __ffs(todo[c]) - 1;
          todo[c] &= todo[c] - 1;
          ++n;
        }
      }
      float2 v[4][PER / 2];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (u < n) {
          const float2* src = reinterpret_cast<const float2*>(prm.part_acc + (base + pk[u]) * D + lane * PER);
#pragma unroll
          for (int e = 0; e < PER / 2; ++e) v[u][e] = src[e];
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (u < n) {
          const float m0 = __shfl_sync(0xffffffffu, ml0.x, pk[u] & 31);
          const float m1 = __shfl_sync(0xffffffffu, ml1.x, pk[u] & 31);
          const float wu = exp2_approx((pk[u] < 32 ? m0 : m1) - mx);
#pragma unroll
          for (int e = 0; e < PER / 2; ++e) ffma2(o[e], make_float2(wu, wu), v[u][e]);
        }
      }
    }
    for (int p0 = 64; p0 < np; p0 += 32) {
      const int pl = p0 + lane;
      const float ml_x = pl < np ? prm.part_ml[base + pl].x : -INFINITY;
      unsigned rest = __ballot_sync(0xffffffffu, ml_x != -INFINITY) & share;
      while (rest) {
        int pk[4];
        int n = 0;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          pk[u] = rest ? __ffs(rest) - 1 : -1;
          if (rest) {
            rest &= rest - 1;
            ++n;
          }
        }
        float2 v[4][PER / 2];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (u < n) {
            const float2* src = reinterpret_cast<const float2*>(prm.part_acc + (base + p0 + pk[u]) * D + lane * PER);
#pragma unroll
            for (int e = 0; e < PER / 2; ++e) v[u][e] = src[e];
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (u < n) {
            const float wu = exp2_approx(__shfl_sync(0xffffffffu, ml_x, pk[u]) - mx);
#pragma unroll
            for (int e = 0; e < PER / 2; ++e) ffma2(o[e], make_float2(wu, wu), v[u][e]);
          }
        }
      }
    }
  }
  if (wph > 1) {
#pragma unroll
    for (int e = 0; e < PER / 2; ++e) s_sum[warp][lane * (PER / 2) + e] = o[e];
    __syncthreads();
    if (sub == 0) {
      for (int k = 1; k < wph; ++k) {
#pragma unroll
        for (int e = 0; e < PER / 2; ++e) fadd2(o[e], s_sum[warp + k][lane * (PER / 2) + e]);
      }
    }
  }
  if (!active || sub != 0) return;
  const float inv = lsum > 0.f ? 1.0f / lsum : 0.f;
  T* dst = static_cast<T*>(prm.out) + (static_cast<size_t>(s) * prm.num_q_heads + hq) * D + lane * PER;
#pragma unroll
  for (int e = 0; e < PER / 2; ++e) {
    fmul2(o[e], make_float2(inv, inv));
    if constexpr (sizeof(T) == 4) {
      reinterpret_cast<float2*>(dst)[e] = o[e];
    } else {
      reinterpret_cast<uint32_t*>(dst)[e] = Chunk<T>::narrow(o[e]);
    }
  }
}

}  // namespace pa

#endif
