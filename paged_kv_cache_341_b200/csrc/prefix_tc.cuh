// Shared-prefix ("cascade") decode, prefix half, on the fifth-generation
// tensor cores (tcgen05 + tensor memory), sm_100a.
//
// Same contract as prefix_attention_kernel: for one KV head h, up to two
// tiles of 128 query rows (of the S*G rows that use head h) and one slice of
// the shared prefix tokens, the online-softmax partial (m, l, unnormalised
// output) of attention over that slice.  Attention over the shared prefix is
// one dense product per KV head once the rows of every sequence are stacked
// ("Paged Attention", aidolsgroup.com, "Example"; prefixes shared
// copy-on-write, agentechip.com "Shared Prefix Caching"), which is what the
// tensor cores are for.
//
// Roles (320 threads):
//   warp 0     TMA producer: 64-token K and V tiles of the prefix, straight
//              from the paged cache through the block list (read once into
//              registers), into two rings of `stages` 128-byte-swizzled tiles
//              ([D/64 panels][64 tok][128 B]); each tile serves both query tiles.
//   warp 1     allocates all 512 tensor-memory columns; lane 0 issues the
//              MMAs.  Query tile g owns columns 256g..256g+255: S (0..63), Q
//              (64.., D/2 columns, two 16-bit values each) and O (128..).
//              Token tile t of query tile g:
//                S_g(t)  = Q_g K_t^T  (M 128, N 64, K = D; A = Q from tensor
//                                      memory, B = K from shared memory)
//                O_g    += P_g(t) V_t (M 128, N = D, K 64; A = P from tensor
//                                      memory where S_g(t) was)
//              issued as PV_0(t), S_0(t+1), PV_1(t), S_1(t+1): while one query
//              tile's softmax runs, the tensor core works for the other.
//              Keeping Q in tensor memory means the only shared-memory
//              operands are the K and V tiles themselves (2 KB per S step, 4 KB
//              per PV step), which shared memory feeds at the full MMA rate;
//              with Q read from shared memory as well, each S step waits on
//              operand reads.
//   warps 2-9  softmax of query tile (warp - 2) / 4; one query row per thread
//              (tensor-memory lane).  First each thread writes its query row
//              into tensor memory (tcgen05.st).  Per token tile: the 64 scores
//              in registers, their maximum, the decode kernel's threshold rule
//              for the reference maximum (it moves only when a scaled score
//              passes it by 2^8; O is then rescaled in tensor memory),
//              P = 2^(s*scale*log2(e) - m) rounded to the cache's 16-bit type
//              and stored over S as the A operand of PV; l sums the rounded
//              weights.
// Products issued by one thread run in issue order, and a commit arrives only
// once everything issued before it has completed.  So S_g(t+1) may overwrite
// P_g(t) as soon as PV_g(t) is issued, and when S_g(t) is reported ready,
// PV_g(t-1) has completed and O may be rescaled.  Every wait is bounded in
// time; on a timeout all roles fall through to the end, the MMA issuer waits
// for its own products, and the tensor memory is released before the CTA
// exits.
#ifndef PAGEDATTN_PREFIX_TC_CUH
#define PAGEDATTN_PREFIX_TC_CUH

#include <cuda.h>
#include <cstdint>
#include <type_traits>

#include "decode.cuh"
#include "prefix.cuh"
#include "tcgen05.cuh"

namespace pa {

// max / min of three float32 values (one instruction on sm_100a).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float fmin3(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

constexpr int kUmmaRows = 128;        // query rows per tile (MMA M)
constexpr int kUmmaTiles = 2;         // query tiles per CTA
constexpr int kUmmaTile = 64;         // prefix tokens per stage (MMA N of S, K of PV)
constexpr int kUmmaThreads = 64 + kUmmaTiles * 128;   // producer, MMA, softmax groups
constexpr uint32_t kUmmaTmemCols = 512;
constexpr uint32_t kUmmaGroupCols = 256;              // per query tile: S 0..63, Q 64..127, O 128..255
constexpr uint32_t kSCol = 0, kQCol = 64, kOCol = 128;
constexpr int kGroupBars = 4;                         // mbarriers per query tile
constexpr int kMaxSliceBlocks = 128;                  // block ids of one prefix slice held by the producer
// At least half of an SM's shared memory, so that one CTA holds the SM (and
// all of its tensor memory) whatever the head size.
constexpr size_t kUmmaMinSmem = 120 * 1024;

template <int D>
__host__ __device__ constexpr size_t prefix_umma_layout_bytes(int stages) {
  return kSmemAlign + 2 * static_cast<size_t>(stages) * (D / 64) * kUmmaTile * 128      // K and V rings
         + (4 * static_cast<size_t>(stages) + kGroupBars * kUmmaTiles + 1) * sizeof(uint64_t) + 16;
}

template <int D>
__host__ __device__ constexpr size_t prefix_umma_smem_bytes(int stages) {
  return prefix_umma_layout_bytes<D>(stages) < kUmmaMinSmem ? kUmmaMinSmem : prefix_umma_layout_bytes<D>(stages);
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kUmmaThreads, 1)
    prefix_umma_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                       const PrefixParams prm) {
  static_assert(sizeof(T) == 2, "tensor-core path takes 16-bit caches");
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  constexpr int kHalves = D / 64;                        // 128-byte panels per row
  constexpr uint32_t kPanel = kUmmaTile * 128;           // one panel of a K/V tile (8 KB)
  constexpr uint32_t kTileBytes = kHalves * kPanel;      // K (or V) bytes per stage
  constexpr int kS = kUmmaTile;                          // scores per row and tile
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  using M = MmaType<T>;

  extern __shared__ __align__(1024) unsigned char smem[];
  const uintptr_t base =
      (reinterpret_cast<uintptr_t>(smem) + kSmemAlign - 1) & ~static_cast<uintptr_t>(kSmemAlign - 1);
  const int stages = prm.stages;
  unsigned char* s_k = reinterpret_cast<unsigned char*>(base);
  unsigned char* s_v = s_k + static_cast<size_t>(stages) * kTileBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_v + static_cast<size_t>(stages) * kTileBytes);
  uint64_t* k_full = bars;
  uint64_t* k_empty = k_full + stages;
  uint64_t* v_full = k_empty + stages;
  uint64_t* v_empty = v_full + stages;
  // per query tile g: s_full (S ready), p_full (P ready, O rescaled),
  // o_done (the last PV), q_full (Q written into tensor memory)
  uint64_t* grp = v_empty + stages;
  auto s_full = [&](int g) { return grp + kGroupBars * g; };
  auto p_full = [&](int g) { return grp + kGroupBars * g + 1; };
  auto o_done = [&](int g) { return grp + kGroupBars * g + 2; };
  auto q_full = [&](int g) { return grp + kGroupBars * g + 3; };
  uint64_t* drain = grp + kGroupBars * kUmmaTiles;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const int split = blockIdx.z;
  const int tok_lo = split * prm.split_tokens;
  const int tok_hi = min(prm.prefix_len, tok_lo + prm.split_tokens);
  const int ntiles = tok_hi > tok_lo ? (tok_hi - tok_lo + kUmmaTile - 1) / kUmmaTile : 0;
  const int rows_total = prm.num_seqs * G;
  const int row0 = blockIdx.x * (kUmmaTiles * kUmmaRows);
  // query tiles of this CTA that hold at least one row
  const int ngroups = min(kUmmaTiles, (rows_total - row0 + kUmmaRows - 1) / kUmmaRows);

  if (threadIdx.x == 0) {
    for (int i = 0; i < stages; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    // softmax-side barriers take one arrival per warp (elected lane after __syncwarp)
    for (int g = 0; g < kUmmaTiles; ++g) {
      mbar_init(s_full(g), 1);
      mbar_init(p_full(g), 4);
      mbar_init(o_done(g), 1);
      mbar_init(q_full(g), 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_slot, kUmmaTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
    }
    const uint64_t policy = policy_evict_last();
    const int BS = prm.block_size;
    const int piece_rows = BS < kChunkTokens ? BS : kChunkTokens;
    // the slice's block ids, read once: lane i holds entries i, i + 32, ...
    // (a slice of split_tokens <= 1024 tokens spans at most 128 blocks of 8)
    const int blk_lo = tok_lo / BS;
    const int nblk = tok_hi > tok_lo ? (tok_hi - 1) / BS - blk_lo + 1 : 0;
    int ids[kMaxSliceBlocks / 32];
#pragma unroll
    for (int k = 0; k < kMaxSliceBlocks / 32; ++k) {
      const int b = lane + 32 * k;
      ids[k] = b < nblk ? prm.prefix_blocks[blk_lo + b] : 0;
    }
    int kst = 0, vst = 0;
    uint32_t kph = 0, vph = 0;
    int k_armed = 0, v_armed = 0;     // tiles whose K (V) copies were issued
    for (int t = 0; t < ntiles; ++t) {
      const int tok0 = tok_lo + t * kUmmaTile;
      const int ntok = min(kUmmaTile, tok_hi - tok0);
      const int npieces = ntok / piece_rows;     // <= 8
      // one box per lane: piece pc = lane / kHalves, panel hf = lane % kHalves
      const int nbox = npieces * kHalves;        // <= 16
      const int pc = lane / kHalves;
      const int hf = lane - pc * kHalves;
      const int tk = tok0 + (lane < nbox ? pc : 0) * piece_rows;
      const int bl = tk / BS - blk_lo;           // entry of this lane's piece in the slice
      int phys = 0;
#pragma unroll
      for (int k = 0; k < kMaxSliceBlocks / 32; ++k) {
        const int v = __shfl_sync(0xffffffffu, ids[k], bl & 31);
        if ((bl >> 5) == k) phys = v;
      }
      int row = 0;
      if (lane < nbox) {
        if (phys < 0 || phys >= prm.num_blocks) {
          set_device_error(DEVERR_BAD_BLOCK_ID);
          phys = 0;
        }
        row = phys * BS + (tk - (bl + blk_lo) * BS);
      }
      const uint32_t tx = static_cast<uint32_t>(nbox) * piece_rows * 128;
      // K tile
      if (!__all_sync(0xffffffffu, mbar_wait(&k_empty[kst], kph ^ 1, abort_flag))) break;
      if (lane == 0) mbar_arrive_expect_tx(&k_full[kst], tx);
      __syncwarp();
      if (lane < nbox)
        tma_load_3d(s_k + static_cast<size_t>(kst) * kTileBytes + hf * kPanel + pc * piece_rows * 128, &tm_k,
                    &k_full[kst], 0, h * kHalves + hf, row, policy);
      ++k_armed;
      if (++kst == stages) {
        kst = 0;
        kph ^= 1;
      }
      // V tile; rows past the end of a short last tile are zeroed so that
      // P = 0 there never meets stale bits
      if (!__all_sync(0xffffffffu, mbar_wait(&v_empty[vst], vph ^ 1, abort_flag))) break;
      unsigned char* vdst = s_v + static_cast<size_t>(vst) * kTileBytes;
      if (ntok < kUmmaTile) {
        const int chunks = (kUmmaTile - ntok) * 8;     // 16-byte chunks per panel
        for (int i = lane; i < kHalves * chunks; i += 32) {
          const int p = i / chunks, c = i - p * chunks;
          *reinterpret_cast<uint4*>(vdst + p * kPanel + ntok * 128 + c * 16) = make_uint4(0, 0, 0, 0);
        }
        tc::fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_expect_tx(&v_full[vst], tx);
      __syncwarp();
      if (lane < nbox)
        tma_load_3d(vdst + hf * kPanel + pc * piece_rows * 128, &tm_v, &v_full[vst], 0, h * kHalves + hf, row,
                    policy);
      ++v_armed;
      if (++vst == stages) {
        vst = 0;
        vph ^= 1;
      }
    }
    // copies still in flight must land before the CTA may exit
    if (lane == 0) {
      int st = kst;
      uint32_t ph = kph;
      for (int k = 0; k < min(k_armed, stages); ++k) {
        if (--st < 0) {
          st = stages - 1;
          ph ^= 1;
        }
        mbar_wait_drain(&k_full[st], ph);
      }
      st = vst;
      ph = vph;
      for (int k = 0; k < min(v_armed, stages); ++k) {
        if (--st < 0) {
          st = stages - 1;
          ph ^= 1;
        }
        mbar_wait_drain(&v_full[st], ph);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = tc::idesc_f16<kBf16>(kUmmaRows, kUmmaTile, false, false);
      constexpr uint32_t idesc_o = tc::idesc_f16<kBf16>(kUmmaRows, D, false, true);
      // descriptors of the operand bases; an operand at byte offset x from a
      // base is the base descriptor plus x >> 4 (start-address field, no carry
      // below 256 KB of shared memory)
      const uint64_t k_desc = tc::smem_desc_sw128(smem_addr(s_k), 16, 1024);
      const uint64_t v_desc = tc::smem_desc_sw128(smem_addr(s_v), kPanel, 1024);
      bool ok = true;
      for (int g = 0; g < ngroups && ok; ++g) ok = mbar_wait(q_full(g), 0, abort_flag);
      tc::fence_after_sync();
      int kst = 0, vst = 0;
      uint32_t kph = 0, vph = 0;
      // S_g = Q_g K^T (Q in tensor memory, 8 columns per K = 16 step)
      auto issue_s = [&](int g, int ks) {
        const uint64_t kb = k_desc + ((ks * kTileBytes) >> 4);
        const uint32_t col = tmem + g * kUmmaGroupCols;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          tc::mma_f16_ts(col + kSCol, col + kQCol + kk * 8, kb + (((kk >> 2) * kPanel + (kk & 3) * 32) >> 4),
                         idesc_s, kk > 0);
        tc::commit(s_full(g));
      };
      // O_g += P_g V; P in the first 32 columns of S, two 16-bit values per column
      auto issue_pv = [&](int g, int vs, bool first) {
        const uint64_t vb = v_desc + ((vs * kTileBytes) >> 4);
        const uint32_t col = tmem + g * kUmmaGroupCols;
#pragma unroll
        for (int kk = 0; kk < kUmmaTile / 16; ++kk)
          tc::mma_f16_ts(col + kOCol, col + kSCol + kk * 8, vb + ((kk * 16 * 128) >> 4), idesc_o, !first || kk > 0);
      };
      if (ok && ntiles > 0) {
        ok = mbar_wait(&k_full[kst], kph, abort_flag);
        if (ok) {
          tc::fence_after_sync();
          for (int g = 0; g < ngroups; ++g) issue_s(g, kst);
          tc::commit(&k_empty[kst]);
          if (++kst == stages) {
            kst = 0;
            kph ^= 1;
          }
        }
      }
      for (int t = 0; ok && t < ntiles; ++t) {
        const bool more = t + 1 < ntiles;
        if (!mbar_wait(&v_full[vst], vph, abort_flag)) {
          ok = false;
          break;
        }
        for (int g = 0; g < ngroups; ++g) {
          // P_g(t) written (and O rescaled if the maximum moved)
          if (!mbar_wait(p_full(g), t & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          issue_pv(g, vst, t == 0);
          if (more) {
            if (g == 0) {
              if (!mbar_wait(&k_full[kst], kph, abort_flag)) {
                ok = false;
                break;
              }
              tc::fence_after_sync();
            }
            issue_s(g, kst);                         // overwrites P_g(t) after PV_g(t) in issue order
          }
        }
        if (!ok) break;
        tc::commit(&v_empty[vst]);
        if (++vst == stages) {
          vst = 0;
          vph ^= 1;
        }
        if (more) {
          tc::commit(&k_empty[kst]);
          if (++kst == stages) {
            kst = 0;
            kph ^= 1;
          }
        }
      }
      for (int g = 0; g < ngroups; ++g) tc::commit(o_done(g));
      // every product issued above completes before the tensor memory goes
      tc::commit(drain);
      mbar_wait_drain(drain, 0);
    }
    __syncwarp();
  } else if ((warp - 2) / 4 < ngroups) {
    // ------------------------------------------------------------- softmax
    const int g = (warp - 2) / 4;                              // query tile of this group
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;                       // tensor-memory lane = query row in the tile
    const uint32_t t_lane = tmem + g * kUmmaGroupCols + (static_cast<uint32_t>(quarter * 32) << 16);
    const int gr = row0 + g * kUmmaRows + row;
    const bool valid = gr < rows_total;
    const int s_idx = valid ? gr / G : 0;
    const int g_idx = valid ? gr - s_idx * G : 0;
    const float qk = prm.qk_scale;
    const float pad = qk >= 0.f ? -INFINITY : INFINITY;
    const float2 qk2 = make_float2(qk, qk);
    float m = -INFINITY, l = 0.f;

    // this thread's query row into tensor memory (zeros past the batch):
    // element 2c in the low half of column kQCol + c
    {
      const uint4* src = reinterpret_cast<const uint4*>(static_cast<const T*>(prm.q) +
                                                        (static_cast<size_t>(s_idx) * prm.num_q_heads + h * G + g_idx) * D);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t qr[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint4 v = valid ? __ldg(src + c * 8 + i) : make_uint4(0, 0, 0, 0);
          qr[4 * i] = v.x;
          qr[4 * i + 1] = v.y;
          qr[4 * i + 2] = v.z;
          qr[4 * i + 3] = v.w;
        }
        tc::tmem_st32(t_lane + kQCol + c * 32, qr);
      }
      tc::tmem_wait_st();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_full(g));
    }

    bool ok = true;
    for (int t = 0; t < ntiles; ++t) {
      const int ntok = min(kUmmaTile, tok_hi - (tok_lo + t * kUmmaTile));
      const bool full = ntok == kUmmaTile;
      if (!__all_sync(0xffffffffu, mbar_wait(s_full(g), t & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      uint32_t cur[kS];
      tc::tmem_ld32_at<0>(t_lane + kSCol, cur);
      tc::tmem_ld32_at<32>(t_lane + kSCol + 32, cur);
      tc::tmem_wait_ld();
      if (!full) {
#pragma unroll
        for (int j = 0; j < kS; ++j) cur[j] = j < ntok ? cur[j] : __float_as_uint(pad);
      }
      // maximum (minimum for a negative scale) of the raw scores: four
      // chains of three-input max over the 64 scores
      float cm[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) cm[i] = __uint_as_float(cur[i]);
      float ext;
      if (qk >= 0.f) {
#pragma unroll
        for (int j = 4; j < kS - 4; j += 8)
#pragma unroll
          for (int k = 0; k < 4; ++k) cm[k] = fmax3(cm[k], __uint_as_float(cur[j + k]), __uint_as_float(cur[j + 4 + k]));
#pragma unroll
        for (int k = 0; k < 4; ++k) cm[k] = fmaxf(cm[k], __uint_as_float(cur[kS - 4 + k]));
        ext = fmax3(fmaxf(cm[0], cm[1]), cm[2], cm[3]);
      } else {
#pragma unroll
        for (int j = 4; j < kS - 4; j += 8)
#pragma unroll
          for (int k = 0; k < 4; ++k) cm[k] = fmin3(cm[k], __uint_as_float(cur[j + k]), __uint_as_float(cur[j + 4 + k]));
#pragma unroll
        for (int k = 0; k < 4; ++k) cm[k] = fminf(cm[k], __uint_as_float(cur[kS - 4 + k]));
        ext = fmin3(fminf(cm[0], cm[1]), cm[2], cm[3]);
      }
      const float c = ext * qk;
      if (__any_sync(0xffffffffu, c > m + kTau)) {
        const float mn = c > m + kTau ? c : m;
        const float f = mn != m ? exp2_approx(m - mn) : 1.f;     // 0 when m was -inf
        if (t >= 1) {
          // O holds PV(0..t-1), all completed (S(t) was issued after PV(t-1));
          // PV(t) waits for this tile's P
#pragma unroll 1
          for (int ob = 0; ob < D / 16; ++ob) {
            uint32_t o[16];
            tc::tmem_ld16(t_lane + kOCol + ob * 16, o);
            tc::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * f);
            tc::tmem_st16(t_lane + kOCol + ob * 16, o);
          }
        }
        l *= f;
        m = mn;
      }
      // P = 2^(s * qk - m), rounded to T, two per column over this tile's S;
      // the row sum takes the rounded values.  Three sweeps per half of the
      // scores (exponents, exponentials, packing), so the 32 exponentials are
      // independent and stream through the MUFU.
      const float2 nm2 = make_float2(-m, -m);
      float2 ls[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t* x = cur + half * 32;           // the scores become exponents, then weights, in place
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float2 e = nm2;
          ffma2(e, make_float2(__uint_as_float(x[2 * i]), __uint_as_float(x[2 * i + 1])), qk2);
          x[2 * i] = __float_as_uint(e.x);
          x[2 * i + 1] = __float_as_uint(e.y);
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) x[j] = __float_as_uint(exp2_approx(__uint_as_float(x[j])));
        if (!full) {
#pragma unroll
          for (int j = 0; j < 32; ++j) x[j] = half * 32 + j < ntok ? x[j] : 0u;
        }
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          w[i] = M::pack(__uint_as_float(x[2 * i]), __uint_as_float(x[2 * i + 1]));
          fadd2(ls[i & 1], M::unpack(w[i]));
        }
        tc::tmem_st16(t_lane + kSCol + half * 16, w);
      }
      tc::tmem_wait_st();
      l += (ls[0].x + ls[1].x) + (ls[0].y + ls[1].y);
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full(g));
    }
    if (ok && ntiles > 0 && !__all_sync(0xffffffffu, mbar_wait(o_done(g), 0, abort_flag))) ok = false;
    tc::fence_after_sync();
    const size_t pi = (static_cast<size_t>(s_idx) * prm.num_q_heads + h * G + g_idx) * prm.max_parts + split;
    float* dst = prm.part_acc + pi * D;
#pragma unroll
    for (int cb = 0; cb < D / 32; ++cb) {
      uint32_t o[32];
      if (ok && ntiles > 0) {
        tc::tmem_ld32(t_lane + kOCol + cb * 32, o);
        tc::tmem_wait_ld();
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) o[j] = 0u;
      }
      if (valid && ok) {
#pragma unroll
        for (int j = 0; j < 32; j += 4)
          *reinterpret_cast<float4*>(dst + cb * 32 + j) =
              make_float4(__uint_as_float(o[j]), __uint_as_float(o[j + 1]), __uint_as_float(o[j + 2]),
                          __uint_as_float(o[j + 3]));
      }
    }
    if (valid && ok) prm.part_ml[pi] = make_float2(m, l);
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kUmmaTmemCols);
  }
}

}  // namespace pa

#endif
