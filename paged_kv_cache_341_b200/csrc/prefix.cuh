// Shared-prefix ("cascade") decode, prefix half, for sm_100a.
//
// When every sequence of a batch starts with the same prefix blocks (the
// shared system prompt of "Paged Attention" on aidolsgroup.com, section
// "Example"; shared prefixes referenced copy-on-write, agentechip.com
// "Shared Prefix Caching"), attention over the prefix is one dense product
// per KV head: all S*G query rows that use KV head h against the same prefix
// K/V.  This kernel computes, for one tile of 64 of those rows and one slice of
// the prefix tokens, the online-softmax partial (m, l, unnormalised output)
// with the tensor cores, so each prefix K/V tile is loaded once per 64 query
// rows instead of once per sequence.  The per-sequence suffixes go through
// decode_mma_kernel (partials only) and reduce_kernel merges everything, so
// the result is attention over prefix ++ suffix, the same as the plain call.
//
// Layout per CTA: 1 producer warp (TMA) + 4 consumer warps of 16 query rows.
// A stage holds 64 prefix tokens of one KV head, K and V, as 128B-swizzled
// boxes of 16 (or 8) rows x 128 bytes; ldmatrix reads them conflict-free.
// Per warp and stage: S = Q K^T (8 token n-tiles x D/16 k-steps of
// mma.sync.m16n8k16), online softmax per row with the same reference-max rule
// as the decode kernel, P rounded to the 16-bit type (denominator sums the
// rounded weights), O += P V (4 token k-steps x D/8 column n-tiles).
#ifndef PAGEDATTN_PREFIX_CUH
#define PAGEDATTN_PREFIX_CUH

#include <cuda.h>
#include <cstdint>

#include "decode.cuh"

namespace pa {

constexpr int kPrefixTile = 64;      // prefix tokens per stage
constexpr int kPrefixWarps = 4;      // consumer warps, 16 query rows each
constexpr int kPrefixRows = 16 * kPrefixWarps;

struct PrefixParams {
  const void* q;                 // [S][Hq][D]
  const int32_t* prefix_blocks;  // [prefix_len / block_size]
  float* part_acc;               // [S][Hq][max_parts][D]
  float2* part_ml;               // [S][Hq][max_parts]
  int num_seqs, num_q_heads, num_kv_heads;
  int block_size, num_blocks;
  int prefix_len;                // tokens, a multiple of 16
  int split_tokens;              // prefix tokens per split (multiple of kPrefixTile)
  int max_parts;                 // row stride of the partial arrays
  int row_pairs;                 // tensor-core kernel: query-tile pairs per KV head
  int num_splits;                // tensor-core kernel: prefix slices
  long long num_units;           // tensor-core kernel: row_pairs x num_kv_heads x slices
  int stages;
  uint32_t stage_bytes;          // K (or V) bytes of one stage
  float qk_scale;                // scale * log2(e)
};

__host__ __device__ constexpr size_t prefix_smem_bytes(int stages, size_t stage_bytes) {
  return kSmemAlign + 2 * static_cast<size_t>(stages) * stage_bytes + 2 * stages * sizeof(uint64_t) + 16;
}

template <typename T, int D, int G>
__global__ void __launch_bounds__((kPrefixWarps + 1) * 32, 2)
    prefix_attention_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                            const PrefixParams prm) {
  static_assert(sizeof(T) == 2, "tensor-core path takes 16-bit caches");
  constexpr int kHalves = D * 2 / kSwizzleBytes;            // 128-byte column blocks per row
  constexpr int kBoxBytes = kChunkTokens * kSwizzleBytes;   // 16 rows x 128 B
  constexpr int KSTEPS = D / 16;                            // k-steps of S = Q K^T
  constexpr int DTILES = D / 8;                             // n-tiles of O = P V
  constexpr int NT = kPrefixTile / 8;                       // token n-tiles per stage
  using M = MmaType<T>;

  extern __shared__ __align__(1024) unsigned char smem[];
  const uintptr_t base =
      (reinterpret_cast<uintptr_t>(smem) + kSmemAlign - 1) & ~static_cast<uintptr_t>(kSmemAlign - 1);
  const int stages = prm.stages;
  unsigned char* s_k = reinterpret_cast<unsigned char*>(base);
  unsigned char* s_v = s_k + static_cast<size_t>(stages) * prm.stage_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(s_v + static_cast<size_t>(stages) * prm.stage_bytes);
  uint64_t* empty = full + stages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + stages);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int h = blockIdx.y;                                  // KV head
  const int split = blockIdx.z;
  const int tok_lo = split * prm.split_tokens;
  const int tok_hi = min(prm.prefix_len, tok_lo + prm.split_tokens);
  const int ntiles = tok_hi > tok_lo ? (tok_hi - tok_lo + kPrefixTile - 1) / kPrefixTile : 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < stages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kPrefixWarps);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kPrefixWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
    }
    const uint64_t policy = policy_evict_last();
    const int BS = prm.block_size;
    const int piece_rows = BS < kChunkTokens ? BS : kChunkTokens;
    int stage = 0;
    uint32_t phase = 0;
    int armed = 0;
    for (int t = 0; t < ntiles; ++t) {
      const int tok0 = tok_lo + t * kPrefixTile;
      const int ntok = min(kPrefixTile, tok_hi - tok0);
      const int npieces = ntok / piece_rows;
      // lane i < npieces: row of piece i in the cache
      int row = 0;
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
      if (!__all_sync(0xffffffffu, mbar_wait(&empty[stage], phase ^ 1, abort_flag))) break;
      if (lane == 0) mbar_arrive_expect_tx(&full[stage], 2u * npieces * kHalves * piece_rows * kSwizzleBytes);
      __syncwarp();
      unsigned char* dk = s_k + static_cast<size_t>(stage) * prm.stage_bytes;
      unsigned char* dv = s_v + static_cast<size_t>(stage) * prm.stage_bytes;
      // one box per lane: (K or V, piece, column block); at most 32 boxes per stage
      const int nbox = npieces * kHalves;
      const bool act = lane < 2 * nbox;
      const int kv = lane >= nbox ? 1 : 0;
      const int r = act ? lane - kv * nbox : 0;
      const int pc = r / kHalves;
      const int hf = r - pc * kHalves;
      const int prow = __shfl_sync(0xffffffffu, row, pc);
      if (act) {
        // 16-token group of the piece, column block hf, sub-piece offset inside the 2 KB box
        const int grp = (pc * piece_rows) / kChunkTokens;
        const int sub = (pc * piece_rows) % kChunkTokens;
        unsigned char* dst = (kv ? dv : dk) + (grp * kHalves + hf) * kBoxBytes + sub * kSwizzleBytes;
        tma_load_3d(dst, kv ? &tm_v : &tm_k, &full[stage], 0, h * kHalves + hf, prow, policy);
      }
      ++armed;
      if (++stage == stages) {
        stage = 0;
        phase ^= 1;
      }
    }
    if (lane == 0) {
      int st = stage, ph = phase;
      const int back = armed < stages ? armed : stages;
      for (int k = 0; k < back; ++k) {
        if (--st < 0) {
          st = stages - 1;
          ph ^= 1;
        }
        mbar_wait_drain(&full[st], ph);
      }
    }
    __syncwarp();
    return;
  }

  // -------------------------------------------------------------- consumers
  const int gq = lane >> 2;
  const int tq = lane & 3;
  const int rows_total = prm.num_seqs * G;
  // query rows of this warp: r0 = tile base + 16*warp + gq, r1 = r0 + 8
  const int r0 = blockIdx.x * kPrefixRows + warp * 16 + gq;
  const int r1 = r0 + 8;
  auto qrow = [&](int r) -> const T* {
    const int s = r / G, g = r - (r / G) * G;
    return static_cast<const T*>(prm.q) + (static_cast<size_t>(s) * prm.num_q_heads + h * G + g) * D;
  };
  // A fragments of Q (rows r0, r1; columns 16kk + 2tq (+1), +8)
  uint32_t qa[KSTEPS][4];
  {
    const uint32_t* q0 = r0 < rows_total ? reinterpret_cast<const uint32_t*>(qrow(r0)) : nullptr;
    const uint32_t* q1 = r1 < rows_total ? reinterpret_cast<const uint32_t*>(qrow(r1)) : nullptr;
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
      qa[kk][0] = q0 ? q0[kk * 8 + tq] : 0u;
      qa[kk][1] = q1 ? q1[kk * 8 + tq] : 0u;
      qa[kk][2] = q0 ? q0[kk * 8 + tq + 4] : 0u;
      qa[kk][3] = q1 ? q1[kk * 8 + tq + 4] : 0u;
    }
  }
  float o[DTILES][4];
#pragma unroll
  for (int i = 0; i < DTILES; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

  // ldmatrix lane roles.  K (B operand of S = Q K^T, rows = tokens):
  // x4 matrix i = lane/8 covers tokens 8*nt + lane%8, column chunk c0 + i.
  // V (B operand of O = P V, through .trans): matrix i covers tokens
  // 16*j + 8*(i%2) + lane%8, column chunk 2*dp + i/2.
  const int k_tok = lane & 7;
  const int k_chk = lane >> 3;
  const int v_tok = (lane & 7) + ((lane >> 3) & 1) * 8;
  const int v_chk = lane >> 4;

  int stage = 0;
  uint32_t phase = 0;
  for (int t = 0; t < ntiles; ++t) {
    const int ntok = min(kPrefixTile, tok_hi - (tok_lo + t * kPrefixTile));
    if (!__all_sync(0xffffffffu, mbar_wait(&full[stage], phase, abort_flag))) return;
    const uint32_t kb = smem_addr(s_k + static_cast<size_t>(stage) * prm.stage_bytes);
    const uint32_t vb = smem_addr(s_v + static_cast<size_t>(stage) * prm.stage_bytes);
    const int nt_valid = ntok / 8;       // ntok is a multiple of 16

    // S[16 rows][64 tokens] = Q K^T
    float s[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
      if (nt < nt_valid) {
        const int grp = nt >> 1;                 // 16-token group
        const int trow = (nt & 1) * 8 + k_tok;   // row inside the group's boxes
#pragma unroll
        for (int kp = 0; kp < KSTEPS / 2; ++kp) {
          // k-steps 2kp, 2kp+1 = column chunks 4kp .. 4kp+3 (one 128-byte block holds 8)
          const int chunk = 4 * kp + k_chk;
          const int hf = chunk >> 3;
          uint32_t b0, b1, b2, b3;
          ldsm_x4(kb + (grp * kHalves + hf) * kBoxBytes + swz(trow, chunk & 7), b0, b1, b2, b3);
          M::mma(s[nt], qa[2 * kp][0], qa[2 * kp][1], qa[2 * kp][2], qa[2 * kp][3], b0, b1);
          M::mma(s[nt], qa[2 * kp + 1][0], qa[2 * kp + 1][1], qa[2 * kp + 1][2], qa[2 * kp + 1][3], b2, b3);
        }
      }
    }
    // online softmax per row (rows r0: s[.][0..1], r1: s[.][2..3])
    float x[NT][4];
    float c0 = -INFINITY, c1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const bool v = nt < nt_valid;
      x[nt][0] = v ? s[nt][0] * prm.qk_scale : -INFINITY;
      x[nt][1] = v ? s[nt][1] * prm.qk_scale : -INFINITY;
      x[nt][2] = v ? s[nt][2] * prm.qk_scale : -INFINITY;
      x[nt][3] = v ? s[nt][3] * prm.qk_scale : -INFINITY;
      c0 = fmaxf(c0, fmaxf(x[nt][0], x[nt][1]));
      c1 = fmaxf(c1, fmaxf(x[nt][2], x[nt][3]));
    }
    c0 = fmaxf(c0, __shfl_xor_sync(0xffffffffu, c0, 1));
    c0 = fmaxf(c0, __shfl_xor_sync(0xffffffffu, c0, 2));
    c1 = fmaxf(c1, __shfl_xor_sync(0xffffffffu, c1, 1));
    c1 = fmaxf(c1, __shfl_xor_sync(0xffffffffu, c1, 2));
    if (__any_sync(0xffffffffu, (c0 > m0 + kTau) | (c1 > m1 + kTau))) {
      const float n0 = c0 > m0 + kTau ? c0 : m0;
      const float n1 = c1 > m1 + kTau ? c1 : m1;
      const float f0 = exp2_approx(m0 - n0);
      const float f1 = exp2_approx(m1 - n1);
      l0 *= f0;
      l1 *= f1;
#pragma unroll
      for (int i = 0; i < DTILES; ++i) {
        o[i][0] *= f0;
        o[i][1] *= f0;
        o[i][2] *= f1;
        o[i][3] *= f1;
      }
      m0 = n0;
      m1 = n1;
    }
    // P as A fragments of O = P V (k-step j = tokens 16j..16j+15 = n-tiles 2j, 2j+1)
    uint32_t pa_[NT / 2][4];
#pragma unroll
    for (int j = 0; j < NT / 2; ++j) {
      pa_[j][0] = M::pack(exp2_approx(x[2 * j][0] - m0), exp2_approx(x[2 * j][1] - m0));
      pa_[j][1] = M::pack(exp2_approx(x[2 * j][2] - m1), exp2_approx(x[2 * j][3] - m1));
      pa_[j][2] = M::pack(exp2_approx(x[2 * j + 1][0] - m0), exp2_approx(x[2 * j + 1][1] - m0));
      pa_[j][3] = M::pack(exp2_approx(x[2 * j + 1][2] - m1), exp2_approx(x[2 * j + 1][3] - m1));
      const float2 a = M::unpack(pa_[j][0]), b = M::unpack(pa_[j][1]);
      const float2 c = M::unpack(pa_[j][2]), d = M::unpack(pa_[j][3]);
      l0 += a.x + a.y + c.x + c.y;
      l1 += b.x + b.y + d.x + d.y;
    }
    // O[16 rows][D] += P V
#pragma unroll
    for (int j = 0; j < NT / 2; ++j) {
      if (2 * j < nt_valid) {
#pragma unroll
        for (int dp = 0; dp < DTILES / 2; ++dp) {
          // column chunks 2dp, 2dp+1 = n-tiles 2dp, 2dp+1
          const int chunk = 2 * dp + v_chk;
          const int hf = chunk >> 3;
          uint32_t b0, b1, b2, b3;
          ldsm_x4_trans(vb + (j * kHalves + hf) * kBoxBytes + swz(v_tok, chunk & 7), b0, b1, b2, b3);
          M::mma(o[2 * dp], pa_[j][0], pa_[j][1], pa_[j][2], pa_[j][3], b0, b1);
          M::mma(o[2 * dp + 1], pa_[j][0], pa_[j][1], pa_[j][2], pa_[j][3], b2, b3);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[stage]);
    if (++stage == stages) {
      stage = 0;
      phase ^= 1;
    }
  }

  // row sums over the quad, then the partial of this split for rows r0, r1
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  auto part_index = [&](int r) -> size_t {
    const int s = r / G, g = r - (r / G) * G;
    return (static_cast<size_t>(s) * prm.num_q_heads + h * G + g) * prm.max_parts + split;
  };
  if (r0 < rows_total) {
    const size_t pi = part_index(r0);
    float* dst = prm.part_acc + pi * D;
#pragma unroll
    for (int i = 0; i < DTILES; ++i)
      *reinterpret_cast<float2*>(dst + i * 8 + 2 * tq) = make_float2(o[i][0], o[i][1]);
    if (tq == 0) prm.part_ml[pi] = make_float2(m0, l0);
  }
  if (r1 < rows_total) {
    const size_t pi = part_index(r1);
    float* dst = prm.part_acc + pi * D;
#pragma unroll
    for (int i = 0; i < DTILES; ++i)
      *reinterpret_cast<float2*>(dst + i * 8 + 2 * tq) = make_float2(o[i][2], o[i][3]);
    if (tq == 0) prm.part_ml[pi] = make_float2(m1, l1);
  }
}

}  // namespace pa

#endif
