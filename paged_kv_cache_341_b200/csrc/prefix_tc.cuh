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
//              from the paged cache through the block list, into two rings
//              of `stages` 128-byte-swizzled tiles ([D/64 panels][64 tok][128 B]);
//              each tile serves both query tiles.
//   warp 1     allocates all 512 tensor-memory columns; lane 0 issues the
//              MMAs, for query tile g (columns 256g..256g+255):
//                S_gb = Q_g K_t^T   (M 128, N 64, K = D; b = t % 2, columns 64b)
//                O_g += P_gt V_t    (M 128, N = D, K 64; columns 128..)
//              and tracks their completion with tcgen05.commit.
//   warps 2-5  softmax of query tile 0, warps 6-9 of query tile 1; one query
//              row per thread (tensor-memory lane): load S, online max with
//              the decode kernel's threshold rule (rescale only when a score
//              passes the reference by 2^8, then O is rescaled in tensor
//              memory), P = 2^(x - m) rounded to the cache's 16-bit type and
//              written to shared memory as the A operand of the next product;
//              l sums the rounded weights.
// While one softmax group works, the tensor core runs the other group's
// products and the next S; P_t V_t follows as soon as P_t is written.  Q is
// loaded once per CTA by the softmax threads (rows beyond the batch are
// zero; a second tile with no rows at all is skipped).  Every wait is bounded in time;
// on a timeout all roles fall through to the end, the MMA issuer waits for
// its own products, and the tensor memory is released before the CTA exits.
#ifndef PAGEDATTN_PREFIX_TC_CUH
#define PAGEDATTN_PREFIX_TC_CUH

#include <cuda.h>
#include <cstdint>
#include <type_traits>

#include "decode.cuh"
#include "prefix.cuh"
#include "tcgen05.cuh"

namespace pa {

// d += a on a pair of float32 lanes (one instruction on sm_100a).
__device__ __forceinline__ void fadd2(float2& d, const float2 a) {
  asm("{\n\t.reg .b64 rd, ra;\n\t"
      "mov.b64 ra, {%2, %3};\n\t"
      "mov.b64 rd, {%0, %1};\n\t"
      "add.rn.f32x2 rd, rd, ra;\n\t"
      "mov.b64 {%0, %1}, rd;\n\t}"
      : "+f"(d.x), "+f"(d.y)
      : "f"(a.x), "f"(a.y));
}

constexpr int kUmmaRows = 128;        // query rows per tile (MMA M)
constexpr int kUmmaTiles = 2;         // query tiles per CTA
constexpr int kUmmaTile = 64;         // prefix tokens per stage (MMA N of S, K of O)
constexpr int kUmmaThreads = 64 + kUmmaTiles * 128;   // producer, MMA, softmax groups
constexpr uint32_t kUmmaTmemCols = 512;

template <int D>
__host__ __device__ constexpr size_t prefix_umma_smem_bytes(int stages) {
  return kSmemAlign + kUmmaTiles * static_cast<size_t>(D / 64) * kUmmaRows * 128   // Q panels
         + 2 * kUmmaTiles * static_cast<size_t>(kUmmaRows) * 128                    // P, two per tile
         + 2 * static_cast<size_t>(stages) * (D / 64) * kUmmaTile * 128              // K and V rings
         + (4 * static_cast<size_t>(stages) + 9 * kUmmaTiles + 1) * sizeof(uint64_t) + 16;
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
  constexpr uint32_t kQPanel = kUmmaRows * 128;          // one panel of Q (16 KB)
  constexpr uint32_t kQBytes = kHalves * kQPanel;        // one query tile
  constexpr uint32_t kPBytes = kUmmaRows * 128;          // one P tile
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  using M = MmaType<T>;

  extern __shared__ __align__(1024) unsigned char smem[];
  const uintptr_t base =
      (reinterpret_cast<uintptr_t>(smem) + kSmemAlign - 1) & ~static_cast<uintptr_t>(kSmemAlign - 1);
  const int stages = prm.stages;
  unsigned char* s_q = reinterpret_cast<unsigned char*>(base);          // [tile][panel][128 rows][128 B]
  unsigned char* s_p = s_q + kUmmaTiles * kQBytes;                       // [tile][2][128 rows][128 B]
  unsigned char* s_k = s_p + 2 * kUmmaTiles * kPBytes;
  unsigned char* s_v = s_k + static_cast<size_t>(stages) * kTileBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_v + static_cast<size_t>(stages) * kTileBytes);
  uint64_t* k_full = bars;
  uint64_t* k_empty = k_full + stages;
  uint64_t* v_full = k_empty + stages;
  uint64_t* v_empty = v_full + stages;
  // per query tile g, 9 barriers at grp + 9g: s_full[2], s_free[2], p_full[2],
  // pv_done[2] (buffer b = tile index % 2), q_full
  uint64_t* grp = v_empty + stages;
  auto s_full = [&](int g, int b) { return grp + 9 * g + b; };
  auto s_free = [&](int g, int b) { return grp + 9 * g + 2 + b; };
  auto p_full = [&](int g, int b) { return grp + 9 * g + 4 + b; };
  auto pv_done = [&](int g, int b) { return grp + 9 * g + 6 + b; };
  auto q_full = [&](int g) { return grp + 9 * g + 8; };
  uint64_t* drain = grp + 9 * kUmmaTiles;
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
    for (int g = 0; g < kUmmaTiles; ++g) {
      // softmax-side barriers take one arrival per warp (elected lane after __syncwarp)
      for (int b = 0; b < 2; ++b) {
        mbar_init(s_full(g, b), 1);
        mbar_init(s_free(g, b), 4);
        mbar_init(p_full(g, b), 4);
        mbar_init(pv_done(g, b), 1);
      }
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
    int kst = 0, vst = 0;
    uint32_t kph = 0, vph = 0;
    int k_armed = 0, v_armed = 0;     // tiles whose K (V) copies were issued
    for (int t = 0; t < ntiles; ++t) {
      const int tok0 = tok_lo + t * kUmmaTile;
      const int ntok = min(kUmmaTile, tok_hi - tok0);
      const int npieces = ntok / piece_rows;
      int row = 0;                      // lane i < npieces: cache row of piece i
      if (lane < npieces) {
        const int tk = tok0 + lane * piece_rows;
        const int blk = tk / BS;
        int phys = prm.prefix_blocks[blk];
        if (phys < 0 || phys >= prm.num_blocks) {
          set_device_error(DEVERR_BAD_BLOCK_ID);
          phys = 0;
        }
        row = phys * BS + (tk - blk * BS);
      }
      const int nbox = npieces * kHalves;        // <= 16
      const int pc = lane / kHalves;
      const int hf = lane - pc * kHalves;
      const int prow = __shfl_sync(0xffffffffu, row, pc);
      const uint32_t tx = static_cast<uint32_t>(nbox) * piece_rows * 128;
      // K tile
      if (!__all_sync(0xffffffffu, mbar_wait(&k_empty[kst], kph ^ 1, abort_flag))) break;
      if (lane == 0) mbar_arrive_expect_tx(&k_full[kst], tx);
      __syncwarp();
      if (lane < nbox)
        tma_load_3d(s_k + static_cast<size_t>(kst) * kTileBytes + hf * kPanel + pc * piece_rows * 128, &tm_k,
                    &k_full[kst], 0, h * kHalves + hf, prow, policy);
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
        tma_load_3d(vdst + hf * kPanel + pc * piece_rows * 128, &tm_v, &v_full[vst], 0, h * kHalves + hf, prow,
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
      const uint64_t q_desc = tc::smem_desc_sw128(smem_addr(s_q), 16, 1024);
      const uint64_t p_desc = tc::smem_desc_sw128(smem_addr(s_p), 16, 1024);
      const uint64_t k_desc = tc::smem_desc_sw128(smem_addr(s_k), 16, 1024);
      const uint64_t v_desc = tc::smem_desc_sw128(smem_addr(s_v), kPanel, 1024);
      int kst = 0, vst = 0;
      uint32_t kph = 0, vph = 0;
      bool ok = true;
      for (int g = 0; g < ngroups && ok; ++g) ok = mbar_wait(q_full(g), 0, abort_flag);
      tc::fence_after_sync();
      auto pv = [&](int j) -> bool {
        if (!mbar_wait(&v_full[vst], vph, abort_flag)) return false;
        const uint64_t vb = v_desc + ((vst * kTileBytes) >> 4);
        for (int g = 0; g < ngroups; ++g) {
          if (!mbar_wait(p_full(g, j & 1), (j >> 1) & 1, abort_flag)) return false;
          tc::fence_after_sync();
          const uint64_t pb = p_desc + (((2 * g + (j & 1)) * kPBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < kUmmaTile / 16; ++kk)
            tc::mma_f16_ss(tmem + g * 256 + 128, pb + ((kk * 32) >> 4), vb + ((kk * 16 * 128) >> 4), idesc_o,
                           j > 0 || kk > 0);
          tc::commit(pv_done(g, j & 1));
        }
        tc::commit(&v_empty[vst]);
        if (++vst == stages) {
          vst = 0;
          vph ^= 1;
        }
        return true;
      };
      for (int t = 0; ok && t < ntiles; ++t) {
        const int sb = t & 1;
        if (!mbar_wait(&k_full[kst], kph, abort_flag)) {
          ok = false;
          break;
        }
        const uint64_t kb = k_desc + ((kst * kTileBytes) >> 4);
        for (int g = 0; g < ngroups && ok; ++g) {
          if (t >= 2 && !mbar_wait(s_free(g, sb), ((t - 2) >> 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          const uint64_t qb = q_desc + ((g * kQBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            tc::mma_f16_ss(tmem + g * 256 + sb * kUmmaTile, qb + (((kk >> 2) * kQPanel + (kk & 3) * 32) >> 4),
                           kb + (((kk >> 2) * kPanel + (kk & 3) * 32) >> 4), idesc_s, kk > 0);
          tc::commit(s_full(g, sb));
        }
        if (!ok) break;
        tc::commit(&k_empty[kst]);
        if (++kst == stages) {
          kst = 0;
          kph ^= 1;
        }
        if (t >= 1) ok = pv(t - 1);
      }
      if (ok && ntiles > 0) ok = pv(ntiles - 1);
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
    const uint32_t t_lane = tmem + g * 256 + (static_cast<uint32_t>(quarter * 32) << 16);
    unsigned char* q_tile = s_q + g * kQBytes;
    unsigned char* p_tiles = s_p + 2 * g * kPBytes;              // two P buffers of this group
    const int gr = row0 + g * kUmmaRows + row;
    const bool valid = gr < rows_total;
    const int s_idx = valid ? gr / G : 0;
    const int g_idx = valid ? gr - s_idx * G : 0;
    {
      const uint4* src = reinterpret_cast<const uint4*>(static_cast<const T*>(prm.q) +
                                                         (static_cast<size_t>(s_idx) * prm.num_q_heads + h * G + g_idx) * D);
#pragma unroll
      for (int c = 0; c < D / 8; ++c) {
        const uint4 v = valid ? src[c] : make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(q_tile + (c >> 3) * kQPanel + row * 128 + (((c & 7) ^ (row & 7)) << 4)) = v;
      }
      tc::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_full(g));
    }
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int t = 0; t < ntiles; ++t) {
      const int sb = t & 1;
      const int ntok = min(kUmmaTile, tok_hi - (tok_lo + t * kUmmaTile));
      if (!__all_sync(0xffffffffu, mbar_wait(s_full(g, sb), (t >> 1) & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      uint32_t sr[2][32];
      tc::tmem_ld32(t_lane + sb * kUmmaTile, sr[0]);
      tc::tmem_ld32(t_lane + sb * kUmmaTile + 32, sr[1]);
      tc::tmem_wait_ld();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free(g, sb));
      // raw scores; the scaled maximum is max(s) * qk for qk >= 0 and
      // min(s) * qk otherwise (rounding is monotonic, so this equals the
      // maximum of the rounded products); columns past a short last tile
      // never win and get weight 0
      const float qk = prm.qk_scale;
      const bool full = ntok == kUmmaTile;
      float sv[kUmmaTile];
#pragma unroll
      for (int j = 0; j < kUmmaTile; ++j) sv[j] = __uint_as_float(sr[j >> 5][j & 31]);
      const float pad = qk >= 0.f ? -INFINITY : INFINITY;
      if (!full) {
#pragma unroll
        for (int j = 0; j < kUmmaTile; ++j) sv[j] = j < ntok ? sv[j] : pad;
      }
      float cm[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) cm[i] = sv[i];
      if (qk >= 0.f) {
#pragma unroll
        for (int j = 8; j < kUmmaTile; ++j) cm[j & 7] = fmaxf(cm[j & 7], sv[j]);
#pragma unroll
        for (int i = 0; i < 4; ++i) cm[i] = fmaxf(cm[i], cm[i + 4]);
        cm[0] = fmaxf(fmaxf(cm[0], cm[1]), fmaxf(cm[2], cm[3]));
      } else {
#pragma unroll
        for (int j = 8; j < kUmmaTile; ++j) cm[j & 7] = fminf(cm[j & 7], sv[j]);
#pragma unroll
        for (int i = 0; i < 4; ++i) cm[i] = fminf(cm[i], cm[i + 4]);
        cm[0] = fminf(fminf(cm[0], cm[1]), fminf(cm[2], cm[3]));
      }
      const float c = cm[0] * qk;
      const float mn = c > m + kTau ? c : m;
      // P row: 2^(s*qk - m) with one packed FMA per pair, rounded to T; the
      // row sum of the rounded weights with packed adds in 4 chains
      uint32_t w[kUmmaTile / 2];
      float2 ls[4];
      const float2 qk2 = make_float2(qk, qk);
      const float2 nm2 = make_float2(-mn, -mn);
#pragma unroll
      for (int k = 0; k < 4; ++k) ls[k] = make_float2(0.f, 0.f);
#pragma unroll
      for (int i = 0; i < kUmmaTile / 2; ++i) {
        float2 e = nm2;
        ffma2(e, make_float2(sv[2 * i], sv[2 * i + 1]), qk2);
        float p0 = exp2_approx(e.x), p1 = exp2_approx(e.y);
        if (!full) {
          p0 = 2 * i < ntok ? p0 : 0.f;
          p1 = 2 * i + 1 < ntok ? p1 : 0.f;
        }
        w[i] = M::pack(p0, p1);
        fadd2(ls[i & 3], M::unpack(w[i]));
      }
      const float lsum = (ls[0].x + ls[1].x) + (ls[2].x + ls[3].x) + ((ls[0].y + ls[1].y) + (ls[2].y + ls[3].y));
      // P buffer t % 2 was last read by PV(t-2)
      if (t >= 2 && !__all_sync(0xffffffffu, mbar_wait(pv_done(g, sb), ((t - 2) >> 1) & 1, abort_flag))) {
        ok = false;
        break;
      }
      float f = 1.f;
      if (t >= 1 && __any_sync(0xffffffffu, mn != m)) {
        // the reference maximum moved: once PV(t-1) has landed, O (in tensor
        // memory) follows; PV(t) is issued only after P(t) below
        if (!__all_sync(0xffffffffu, mbar_wait(pv_done(g, sb ^ 1), ((t - 1) >> 1) & 1, abort_flag))) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        f = mn != m ? exp2_approx(m - mn) : 1.f;
#pragma unroll
        for (int cb = 0; cb < D / 32; ++cb) {
          uint32_t o[32];
          tc::tmem_ld32(t_lane + 128 + cb * 32, o);
          tc::tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * f);
          tc::tmem_st32(t_lane + 128 + cb * 32, o);
        }
        tc::tmem_wait_st();
      }
      m = mn;
      l = l * f + lsum;
      unsigned char* prow_ptr = p_tiles + sb * kPBytes + row * 128;
#pragma unroll
      for (int ch = 0; ch < 8; ++ch)
        *reinterpret_cast<uint4*>(prow_ptr + ((ch ^ (row & 7)) << 4)) =
            make_uint4(w[ch * 4], w[ch * 4 + 1], w[ch * 4 + 2], w[ch * 4 + 3]);
      tc::fence_proxy_async_smem();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full(g, sb));
    }
    // the last product's completion (tracked by its buffer's barrier) implies all earlier ones
    if (ok && ntiles > 0 &&
        !__all_sync(0xffffffffu, mbar_wait(pv_done(g, (ntiles - 1) & 1), ((ntiles - 1) >> 1) & 1, abort_flag)))
      ok = false;
    tc::fence_after_sync();
    const size_t pi = (static_cast<size_t>(s_idx) * prm.num_q_heads + h * G + g_idx) * prm.max_parts + split;
    float* dst = prm.part_acc + pi * D;
#pragma unroll
    for (int cb = 0; cb < D / 32; ++cb) {
      uint32_t o[32];
      if (ok && ntiles > 0) {
        tc::tmem_ld32(t_lane + 128 + cb * 32, o);
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
