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
//   KV heads).  Units are numbered sequence-major and dealt to a persistent
//   grid (one or two CTAs per SM) in round-robin order, so neighbouring CTAs
//   read neighbouring head tiles of the same blocks at about the same time.
// * One producer warp streams each unit as chunks of 16 tokens.  A chunk is
//   one TMA tile load per K and per V (box = 16 tokens x HT heads x D), taken
//   straight from the physical block that the block table names; the table
//   slice is held in the producer's registers, 32 entries per warp load.  The
//   unit's HT*G query rows come in by one bulk copy into a double buffer.
//   Stages are guarded by full/empty mbarriers.
// * Consumer warp j handles KV head j of the tile for all G = Hq/Hkv query
//   heads that share it, so each K/V element loaded serves G heads.  Lanes
//   form groups of L lanes per token (L*E = D; each lane holds E elements of
//   q for all G heads, as float32 pairs); a group's dot products finish with
//   log2(L) xor-shuffles.  Every group keeps its own online-softmax state
//   (reference max m, sum l, unnormalised output), merged across groups at the
//   end of the unit, so the token loop has no cross-group traffic.
// * The reference max is only moved when a score exceeds it by more than
//   kTau = 8 (base-2 units): exp2(score - m) then stays <= 256, and the final
//   division by l cancels the choice of m exactly, so rescaling of the
//   accumulators is rare.
// * With partitions, each unit writes its (m, l, unnormalised output) in
//   float32 and a second kernel merges them; sequences that fit in one
//   partition are written out directly.
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

struct DecodeParams {
  const void* q;                 // [S][Hq][D]
  const int32_t* block_tables;   // [S][MB]
  const int32_t* context_lens;   // [S]
  void* out;                     // [S][Hq][D]
  float* part_acc;               // [S][Hq][NP][D]   (partitioned mode)
  float2* part_ml;               // [S][Hq][NP]      (m in base-2 units, l)
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
};

struct StageMeta {
  int seq, part, tile, ntok, flags, nparts, qslot, pad;
};
constexpr int kFirst = 1, kLast = 2;

// Lanes per token for a head size / group size: enough that the per-lane
// q + accumulator registers (2*G*D/L floats) stay at or below 128.
template <int D, int G>
struct Lanes {
  static constexpr int L = (D * G / 64 > 8) ? D * G / 64 : 8;
  static_assert(L <= 32 && (32 % L) == 0, "unsupported head_dim / group size");
};

__device__ __forceinline__ int parts_of(int len, int psize) {
  return (psize > 0 && len > 0) ? (len + psize - 1) / psize : 1;
}

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
  const int HT = prm.tile_heads;
  const int stages = prm.stages;
  const int tile_elems = kChunkTokens * HT * D;
  T* s_k = reinterpret_cast<T*>(smem);
  T* s_v = s_k + stages * tile_elems;
  T* s_q = s_v + stages * tile_elems;                       // 2 x [HT*G][D]
  StageMeta* meta = reinterpret_cast<StageMeta*>(s_q + 2 * HT * G * D);
  uint64_t* full = reinterpret_cast<uint64_t*>(meta + stages);
  uint64_t* empty = full + stages;
  uint64_t* q_full = empty + stages;
  uint64_t* q_empty = q_full + 2;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(q_empty + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < stages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], HT);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], HT);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == HT) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
    }
    const uint64_t policy = policy_evict_first();
    const int S = prm.num_seqs;
    const int MB = prm.max_blocks;
    const int BS = prm.block_size;
    const int cap = MB * BS;
    const int P = prm.partition_size;
    const int n_tiles = prm.num_tiles;

    // Window of 32 sequences: lane i holds sequence win_s0 + i.
    int win_s0 = 0, win_base = 0;
    int my_len = 0, my_units = 0, my_incl = 0, win_total = 0;
    auto load_window = [&]() {
      const int s = win_s0 + lane;
      my_len = 0;
      my_units = 0;
      if (s < S) {
        int len = prm.context_lens[s];
        if (len > cap || len < 0) {
          set_device_error(DEVERR_BAD_LENGTH);
          len = len < 0 ? 0 : cap;
        }
        my_len = len;
        my_units = parts_of(len, P) * n_tiles;
      }
      my_incl = my_units;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, my_incl, off);
        if (lane >= off) my_incl += v;
      }
      win_total = __shfl_sync(0xffffffffu, my_incl, 31);
    };
    load_window();

    int stage = 0;
    uint32_t phase = 0;
    int units_done = 0;
    long long armed = 0;               // stages armed so far (for the drain at exit)
    int q_issued = 0;                  // query copies issued so far
    int tw_seq = -1, tw_base = -1, tw_val = 0;
    bool ok = true;

    for (int u = blockIdx.x; ok; u += gridDim.x) {
      bool exhausted = false;
      while (u >= win_base + win_total) {
        win_base += win_total;
        win_s0 += 32;
        if (win_s0 >= S) {
          exhausted = true;
          break;
        }
        load_window();
      }
      if (exhausted) break;
      const unsigned hit = __ballot_sync(0xffffffffu, win_base + my_incl > u);
      const int hl = __ffs(hit) - 1;
      const int seq = win_s0 + hl;
      const int len = __shfl_sync(0xffffffffu, my_len, hl);
      const int excl = __shfl_sync(0xffffffffu, my_incl - my_units, hl);
      const int r = u - (win_base + excl);
      const int part = r / n_tiles;
      const int tile = r - part * n_tiles;
      const int nparts = parts_of(len, P);
      const int tok_begin = P > 0 ? part * P : 0;
      const int tok_end = P > 0 ? min(len, tok_begin + P) : len;
      const int nchunks = max(1, (tok_end - tok_begin + kChunkTokens - 1) / kChunkTokens);
      const int qslot = units_done & 1;

      // Query rows of this unit: [HT*G][D] contiguous in q.
      if (!__all_sync(0xffffffffu, mbar_wait(&q_empty[qslot], ((units_done >> 1) & 1) ^ 1, abort_flag))) {
        ok = false;
        break;
      }
      ++q_issued;
      if (lane == 0) {
        const char* src = static_cast<const char*>(prm.q) +
                          (static_cast<size_t>(seq) * prm.num_q_heads + static_cast<size_t>(tile) * HT * G) * D *
                              sizeof(T);
        mbar_arrive_expect_tx(&q_full[qslot], prm.q_bytes);
        bulk_load(s_q + qslot * HT * G * D, src, prm.q_bytes, &q_full[qslot]);
      }

      for (int c = 0; c < nchunks; ++c) {
        const int tok = tok_begin + c * kChunkTokens;
        const int ntok = max(0, min(kChunkTokens, tok_end - tok));
        int phys = 0, within = 0;
        if (ntok > 0) {
          const int blk = tok / BS;
          within = tok - blk * BS;
          const int wb = blk & ~31;
          if (seq != tw_seq || wb != tw_base) {
            tw_seq = seq;
            tw_base = wb;
            const int idx = wb + lane;
            tw_val = idx < MB ? prm.block_tables[static_cast<size_t>(seq) * MB + idx] : 0;
          }
          phys = __shfl_sync(0xffffffffu, tw_val, blk - wb);
          if (phys < 0 || phys >= prm.num_blocks) {
            if (lane == 0) set_device_error(DEVERR_BAD_BLOCK_ID);
            phys = 0;
          }
        }
        if (!__all_sync(0xffffffffu, mbar_wait(&empty[stage], phase ^ 1, abort_flag))) {
          ok = false;
          break;
        }
        if (lane == 0) {
          StageMeta m;
          m.seq = seq;
          m.part = part;
          m.tile = tile;
          m.ntok = ntok;
          m.flags = (c == 0 ? kFirst : 0) | (c == nchunks - 1 ? kLast : 0);
          m.nparts = nparts;
          m.qslot = qslot;
          m.pad = 0;
          meta[stage] = m;
          if (ntok > 0) {
            mbar_arrive_expect_tx(&full[stage], 2 * prm.tile_bytes);
            const int row = phys * BS + within;
            tma_load_3d(s_k + stage * tile_elems, &tm_k, &full[stage], 0, tile * HT, row, policy);
            tma_load_3d(s_v + stage * tile_elems, &tm_v, &full[stage], 0, tile * HT, row, policy);
          } else {
            mbar_arrive(&full[stage]);
          }
        }
        __syncwarp();
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
      if (__all_sync(0xffffffffu, mbar_wait(&empty[stage], phase ^ 1, abort_flag))) {
        if (lane == 0) {
          meta[stage].seq = -1;
          mbar_arrive(&full[stage]);
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
        mbar_wait_drain(&full[st], ph);
      }
      for (int k = 1; k <= 2 && k <= q_issued; ++k) {
        const int un = q_issued - k;
        mbar_wait_drain(&q_full[un & 1], (un >> 1) & 1);
      }
    }
    __syncwarp();
    return;
  }

  // -------------------------------------------------------------- consumers
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
    if (!__all_sync(0xffffffffu, mbar_wait(&full[stage], phase, abort_flag))) return;
    const StageMeta mt = meta[stage];
    if (mt.seq < 0) return;

    if (mt.flags & kFirst) {
      if (!__all_sync(0xffffffffu, mbar_wait(&q_full[mt.qslot], (units_done >> 1) & 1, abort_flag))) return;
      const T* qrow = s_q + mt.qslot * HT * G * D + j * G * D;
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
      if (lane == 0) mbar_arrive(&q_empty[mt.qslot]);
    }

    if (mt.ntok > 0) {
      const T* kt = s_k + stage * tile_elems + j * D;
      const T* vt = s_v + stage * tile_elems + j * D;
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
    if (lane == 0) mbar_arrive(&empty[stage]);
    if (++stage == stages) {
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
        if (mt.nparts == 1) {
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
          const size_t pidx = (static_cast<size_t>(mt.seq) * prm.num_q_heads + hq) * prm.max_parts + mt.part;
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

// Merge of per-partition partials: M = max m_p, w_p = 2^(m_p - M),
// out = sum_p w_p acc_p / sum_p w_p l_p.  One CTA per sequence; sequences
// that fit one partition were written by decode_kernel and are skipped.
struct ReduceParams {
  const int32_t* context_lens;
  const float* part_acc;
  const float2* part_ml;
  void* out;
  int num_seqs, num_q_heads, partition_size, max_parts, cap;
};

template <typename T, int D>
__global__ void __launch_bounds__(256) reduce_kernel(const ReduceParams prm) {
  constexpr int PER = D / 32;                // contiguous elements per lane
  static_assert(PER % 2 == 0, "head_dim must be a multiple of 64");
  const int s = blockIdx.x;
  int len = prm.context_lens[s];
  len = len < 0 ? 0 : (len > prm.cap ? prm.cap : len);
  const int np = parts_of(len, prm.partition_size);
  if (np <= 1) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  for (int hq = warp; hq < prm.num_q_heads; hq += nwarps) {
    const size_t base = (static_cast<size_t>(s) * prm.num_q_heads + hq) * prm.max_parts;
    float mx = -INFINITY;
    for (int p = lane; p < np; p += 32) mx = fmaxf(mx, prm.part_ml[base + p].x);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    float lsum = 0.f;
    for (int p = lane; p < np; p += 32) {
      const float2 ml = prm.part_ml[base + p];
      lsum += ml.y * exp2_approx(ml.x - mx);
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, off);
    float2 o[PER / 2];
#pragma unroll
    for (int e = 0; e < PER / 2; ++e) o[e] = make_float2(0.f, 0.f);
    for (int p = 0; p < np; ++p) {
      const float w = exp2_approx(prm.part_ml[base + p].x - mx);
      const float2* src = reinterpret_cast<const float2*>(prm.part_acc + (base + p) * D + lane * PER);
#pragma unroll
      for (int e = 0; e < PER / 2; ++e) ffma2(o[e], make_float2(w, w), src[e]);
    }
    const float inv = 1.0f / lsum;
    T* dst = static_cast<T*>(prm.out) + (static_cast<size_t>(s) * prm.num_q_heads + hq) * D + lane * PER;
#pragma unroll
    for (int e = 0; e < PER / 2; ++e) {
      fmul2(o[e], make_float2(inv, inv));
      if constexpr (sizeof(T) == 4) {
        reinterpret_cast<float2*>(dst)[e] = o[e];
      } else if constexpr (Chunk<T>::kElems == 8 && sizeof(T) == 2) {
        const uint32_t w = Chunk<T>::narrow(o[e]);
        reinterpret_cast<uint32_t*>(dst)[e] = w;
      }
    }
  }
}

}  // namespace pa

#endif
