// Shared-prefix ("cascade") decode, prefix half, on the tensor cores of an
// SM pair (tcgen05 cta_group::2, clusters of two CTAs), sm_100a, D = 128.
//
// Same contract as prefix_umma_kernel (the one-SM form in prefix_tc.cuh, used
// for head_dim 64, when no cluster of two fits, or with PA_PREFIX_PATH=umma;
// this kernel is the default for head_dim 128): attention over the shared
// prefix is one dense product per KV head once the rows of every sequence are
// stacked ("Paged Attention", aidolsgroup.com, "Example"; prefixes shared
// copy-on-write, agentechip.com "Shared Prefix Caching").  What the pair
// changes is where the K/V tiles live: the two CTAs of a cluster take two
// query tiles of the same KV head (rows 256 xp .. 256 xp + 255), and one
// thread of the even CTA issues each product for both, M = 256:
//   S(t) = Q K_t^T   each CTA's A is its own 128 query rows; B (K_t) is split
//                    by N: CTA r holds tokens 64 r .. 64 r + 63 of the tile
//   O   += P(t) V_t  A = P from each CTA's own tensor memory; B (V_t) is split
//                    by N: CTA r holds head dimensions 64 r .. 64 r + 63
// so each SM loads half of every K/V tile (16 KB of K, 16 KB of V) where the
// one-SM form loads all of it for 128 rows, and each SM's tensor core still
// works on a full M 128 x N 128 tile.
//
// Tensor memory (per SM): score buffers S_0, S_1 (columns 0..255) and
// accumulators O_0, O_1 (256..511).  Token tile t, counted over the CTA's
// whole share, goes to S_{t mod 2} and PV(t) accumulates into O_{t mod 2}.
// The softmax is two groups of eight warps: group g takes the tiles with
// t mod 2 = g with its own reference maximum and sum, so that one group's
// exponentials overlap the other group's tensor-memory loads, maximum
// exchange and stores.  In a group two threads share a query row (a
// tensor-memory lane): half h takes scores 64 h .. 64 h + 63, 32 at a time,
// and the two exchange their maxima through shared memory.  The reference
// maximum moves only when a scaled score passes it by 2^8 (the decode
// kernel's rule); then the thread rescales its half of O_g once the group's
// previous PV has completed.  Weights rounded to the cache's 16-bit type go
// over the thread's own scores (tokens 64 h + 32 c + 2j, + 2j + 1 in column
// 64 h + 32 c + j) as the A operand of PV; the row sums take the weights
// before rounding.  At the end of a segment all four threads of a row
// exchange (m, l) and each writes a quarter of the partial,
// 2^(m_0 - M) O_0 + 2^(m_1 - M) O_1 with M = max(m_0, m_1).
//
// K and V halves of a stage share one "full" barrier (both producers arrive
// with their bytes; in the even CTA the relay passes on both of the odd CTA's)
// and one "empty" barrier, committed after the stage's PV, which is also how
// the softmax learns that PV(t) has completed (the empty phase of tile t's
// stage): per tile the issuing thread, which sets the period, waits twice
// (K and V, the weights) and commits twice (S ready, stage free).
//
// Measured on the 200-sequence, 30,720-token shared-prefix step (B200), with
// every kernel on one stream: a cascade call of 0.2189 ms against 0.2221 ms
// with a separate "PV done" commit; with that commit, 0.2182 against 0.2245 ms
// for the one-SM kernel on one box, and 0.2243 ms with separate K and V
// barriers too (one softmax group of sixteen warps over both score buffers:
// 0.231 against 0.225 ms).  Clock stamps per tile show each group busy
// ~2.2K of its ~4.5K-cycle period (loads and maximum ~440, exchange ~300,
// exponentials and stores ~1.3K) and the issuing thread spending ~1.3K cycles
// per tile in the sixteen M 256 x N 128 x K 16 products (about 80-87 cycles
// each, whether the pipe was idle or not) and the rest waiting for weights,
// V and K or committing; a second issuing warp for the S products was
// measured slower (0.228 against 0.224 ms on its box).  Stamps of %globaltimer
// and clock64 per CTA put the SM clock over the kernel at ~1.75 GHz (the
// step draws 965-990 W of the 1 kW limit), the first S product 4.9 us after
// launch, and the CTAs' last tiles between 138 and 160 us (per-unit times
// differ by +-7 % between clusters).  The work split (stream-K shares of (query-tile
// pair, KV head, 512-token slice) units, segments accumulated into one
// partial each) is that of the one-SM form.
//
// Roles per CTA (608 threads): warp 0 loads this CTA's query tile of each
// segment and its K halves, warp 2 its V halves (one TMA box per lane and
// block piece; boxes past the prefix read the tensor map's zero fill);
// warp 1 holds the pair's tensor memory (cta_group::2 allocation in both
// CTAs); in the even CTA its lane 0 issues the products, in the odd CTA it
// relays the completion of that CTA's own copies (which arrive on its own
// barriers, so that it can wait for them before it exits) to the even CTA's
// barriers; warps 3-18 are the softmax.  The even CTA's "full" barriers take
// its own producer's arrival (with its bytes) and the relay; "P ready" (one
// per score buffer) takes one arrival per warp of that buffer's softmax group
// in both CTAs and "O read out" one per softmax warp of both CTAs; every completion
// of products (S ready, stage and query buffers free) is committed
// to the same barrier in both CTAs.  Every wait is bounded in time; both CTAs
// meet at a cluster barrier before the tensor memory is released and before
// either exits, so no copy or product still touches a CTA that has gone.
#ifndef PAGEDATTN_PREFIX_TC2_CUH
#define PAGEDATTN_PREFIX_TC2_CUH

#include <cuda.h>
#include <cstdint>
#include <type_traits>

#include "pair.cuh"
#include "prefix_tc.cuh"

namespace pa {

constexpr int kPairRowThreads = 4;                                   // softmax threads per query row
constexpr int kPairGroupRowThreads = kPairRowThreads / 2;            // per softmax group
constexpr int kPairHalfScores = kUmmaTile / kPairGroupRowThreads;    // scores per thread and token tile (64)
constexpr int kPairSoftmaxWarps = 4 * kPairRowThreads;               // four lane quarters
constexpr int kPairGroupWarps = kPairSoftmaxWarps / 2;               // softmax warps per tile parity
constexpr int kPairSoftmaxWarp0 = 3;                                  // first softmax warp
constexpr int kPairThreads = 32 * (kPairSoftmaxWarp0 + kPairSoftmaxWarps);  // 608
constexpr uint32_t kPairSBufCols = 128;                               // score buffer b at columns 128 b
constexpr uint32_t kPairOCol = 256;                                   // O_b at columns 256 + 128 b ..
constexpr int kPairRows = 2 * kUmmaRows;                              // query rows per cluster

template <int D>
__host__ __device__ constexpr size_t prefix_pair_layout_bytes(int stages) {
  return kSmemAlign + 2 * static_cast<size_t>(D / 64) * kUmmaRows * 128     // two query tiles
         + 2 * static_cast<size_t>(stages) * (D / 64) * kUmmaTile * 64       // K and V halves
         + 2 * 2 * kUmmaRows * kPairGroupRowThreads * sizeof(float)             // maxima [group][parity]
         + 2 * kUmmaRows * kPairRowThreads * sizeof(float2)                    // (m, l) [segment parity]
         + (4 * static_cast<size_t>(stages) + 29) * sizeof(uint64_t) + 16;   // barriers, slots
}

template <int D>
__host__ __device__ constexpr size_t prefix_pair_smem_bytes(int stages) {
  return prefix_pair_layout_bytes<D>(stages) < kUmmaMinSmem ? kUmmaMinSmem : prefix_pair_layout_bytes<D>(stages);
}

// A unit is one slice of split_tokens prefix tokens for one query-tile pair
// xp (rows 256 xp ..) and one KV head h, numbered slice-fastest within a run,
// run = xp * num_kv_heads + h: the units and segments of the one-SM kernel,
// whose two query tiles are here the two CTAs' tiles.
template <int G>
__device__ __forceinline__ PrefixSegment prefix_pair_segment(int u, int u_end, const PrefixParams& prm) {
  return prefix_segment<G>(u, u_end, prm);
}

template <typename T, int G>
__global__ void __launch_bounds__(kPairThreads, 1)
    prefix_pair_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ CUtensorMap tm_q, const PrefixParams prm) {
  constexpr int D = 128;
  static_assert(sizeof(T) == 2, "tensor-core path takes 16-bit caches");
  constexpr int kHalves = D / 64;                        // 128-byte panels per row
  constexpr uint32_t kKPanel = (kUmmaTile / 2) * 128;    // one panel of a K half (64 tokens, 8 KB)
  constexpr uint32_t kKHalf = kHalves * kKPanel;         // K half per stage (16 KB)
  constexpr uint32_t kVHalf = kUmmaTile * 128;           // V half per stage: one panel of 128 tokens (16 KB)
  constexpr uint32_t kQPanel = kUmmaRows * 128;          // one panel of Q (16 KB)
  constexpr uint32_t kQBytes = kHalves * kQPanel;        // one query tile
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  constexpr unsigned kFull = 0xffffffffu;
  constexpr uint16_t kBoth = 0x3;
  using M = MmaType<T>;

  extern __shared__ __align__(1024) unsigned char smem[];
  const uintptr_t base =
      (reinterpret_cast<uintptr_t>(smem) + kSmemAlign - 1) & ~static_cast<uintptr_t>(kSmemAlign - 1);
  const int stages = prm.stages;
  unsigned char* s_q = reinterpret_cast<unsigned char*>(base);          // [2][panel][128 rows][128 B]
  unsigned char* s_k = s_q + 2 * kQBytes;                                // [stage][panel][64 tok][128 B]
  unsigned char* s_v = s_k + static_cast<size_t>(stages) * kKHalf;      // [stage][128 tok][128 B]
  float* x_max = reinterpret_cast<float*>(s_v + static_cast<size_t>(stages) * kVHalf);   // [g][par][row][half]
  float2* s_ml = reinterpret_cast<float2*>(x_max + 2 * 2 * kUmmaRows * kPairGroupRowThreads);  // [sb][row][4]
  // K and V of a stage share one "full" and one "empty" barrier
  uint64_t* k_full = reinterpret_cast<uint64_t*>(s_ml + 2 * kUmmaRows * kPairRowThreads);
  uint64_t* k_empty = k_full + stages;
  uint64_t* v_full = k_full;
  uint64_t* v_empty = k_empty;
  uint64_t* s_full = k_empty + 3 * stages;     // [2]
  uint64_t* p_full = s_full + 2;           // [2] (even CTA: both CTAs' softmax warps)
  // PV(t) completion is the "empty" phase of tile t's stage
  uint64_t* q_full = p_full + 4;           // [2]
  uint64_t* q_empty = q_full + 2;          // [2]
  uint64_t* o_free = q_empty + 2;          // (even CTA: both CTAs' softmax warps)
  uint64_t* drain = o_free + 1;
  uint64_t* xq = drain + 1;                // [group][lane quarter]
  uint64_t* sq = xq + 2 * 4;               // [segment parity][lane quarter]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sq + 2 * 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = pair::cta_rank();
  const bool lead = rank == 0;
  const int rows_total = prm.num_seqs * G;
  const int cluster = blockIdx.x >> 1, clusters = gridDim.x >> 1;
  const int u_begin = static_cast<int>(static_cast<long long>(cluster) * prm.num_units / clusters);
  const int u_end = static_cast<int>(static_cast<long long>(cluster + 1) * prm.num_units / clusters);

  if (threadIdx.x == 0) {
    // even CTA: own two producers + the odd CTA's relay of each
    const uint32_t full_count = lead ? 2 : 1;
    for (int i = 0; i < stages; ++i) {
      mbar_init(&k_full[i], 2 * full_count);
      mbar_init(&k_empty[i], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 2 * kPairGroupWarps);
      mbar_init(&q_full[b], full_count);
      mbar_init(&q_empty[b], 1);
    }
    mbar_init(o_free, 2 * kPairSoftmaxWarps);
    mbar_init(drain, 1);
    for (int i = 0; i < 2 * 4; ++i) {
      mbar_init(&xq[i], kPairGroupRowThreads);
      mbar_init(&sq[i], kPairRowThreads);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc_pair(tmem_slot, kUmmaTmemCols);
    tc::tmem_relinquish_pair();
  }
  tc::fence_before_sync();
  pair::cluster_sync();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  const int BS = prm.block_size;
  const int piece_rows = BS < kChunkTokens ? BS : kChunkTokens;
  const int oob_row = prm.num_blocks * BS;        // a box starting here reads zeros

  if (warp == 0 || warp == 2) {
    // -------------------------------------------------------- producers
    const bool kq = warp == 0;                    // K halves and query tiles; else V halves
    if (lane == 0) prefetch_tensormap(kq ? &tm_k : &tm_v);
    if (kq && lane == 0) prefetch_tensormap(&tm_q);
    const uint64_t policy = policy_evict_last();
    uint64_t* full = kq ? k_full : v_full;
    uint64_t* empty = kq ? k_empty : v_empty;
    const uint32_t half_bytes = kq ? kKHalf : kVHalf;
    int st = 0;
    uint32_t ph = 0;
    int armed = 0, q_armed = 0;
    bool ok = true;
    // the query tile of segment i into buffer i mod 2 once the products of
    // segment i - 2 have read it
    auto load_q = [&](const PrefixSegment& J, int i) {
      const int b = i & 1;
      if (!__all_sync(kFull, mbar_wait(&q_empty[b], ((i >> 1) & 1) ^ 1, abort_flag))) return false;
      if (lane == 0) {
        mbar_arrive_expect_tx(&q_full[b], kQBytes);
        const int x = J.row0 / kUmmaRows + static_cast<int>(rank);
        for (int hf = 0; hf < kHalves; ++hf)
          tma_load_4d(s_q + b * kQBytes + hf * kQPanel, &tm_q, &q_full[b], 0, hf, J.h * G, x * kUmmaRows / G);
      }
      __syncwarp();
      ++q_armed;
      return true;
    };
    PrefixSegment I{};
    if (u_begin < u_end) {
      I = prefix_pair_segment<G>(u_begin, u_end, prm);
      if (kq) ok = load_q(I, 0);
    }
    for (int i = 0, u = u_begin; ok && u < u_end; ++i) {
      const bool has_next = I.end < u_end;
      PrefixSegment J{};
      if (has_next) J = prefix_pair_segment<G>(I.end, u_end, prm);
      bool q_next = !(kq && has_next);
      for (int t = 0; t < I.ntiles; ++t) {
        const int tok0 = I.tok_lo + t * kUmmaTile;
        // K: tokens 64 rank .. of the tile, both panels (lane = piece * 2 + panel);
        // V: all 128 tokens, panel `rank` (lane = piece)
        const int first = kq ? tok0 + 64 * static_cast<int>(rank) : tok0;
        const int pieces = (kq ? kUmmaTile / 2 : kUmmaTile) / piece_rows;   // <= 16
        const int nbox = kq ? pieces * kHalves : pieces;                    // <= 16
        const int pc = kq ? lane / kHalves : lane;
        const int hf = kq ? lane - pc * kHalves : static_cast<int>(rank);
        int row = oob_row;
        if (lane < nbox) {
          const int tk = first + pc * piece_rows;
          if (tk < I.tok_hi) {
            int phys = __ldg(prm.prefix_blocks + tk / BS);
            if (phys < 0 || phys >= prm.num_blocks) {
              set_device_error(DEVERR_BAD_BLOCK_ID);
              phys = 0;
            }
            row = phys * BS + (tk - (tk / BS) * BS);
          }
        }
        if (!__all_sync(kFull, mbar_wait(&empty[st], ph ^ 1, abort_flag))) {
          ok = false;
          break;
        }
        if (lane == 0) mbar_arrive_expect_tx(&full[st], half_bytes);
        __syncwarp();
        if (lane < nbox) {
          unsigned char* dst = kq ? s_k + static_cast<size_t>(st) * kKHalf + hf * kKPanel + pc * piece_rows * 128
                                  : s_v + static_cast<size_t>(st) * kVHalf + pc * piece_rows * 128;
          tma_load_3d(dst, kq ? &tm_k : &tm_v, &full[st], 0, I.h * kHalves + hf, row, policy);
        }
        ++armed;
        if (++st == stages) {
          st = 0;
          ph ^= 1;
        }
        if (!q_next && t == min(1, I.ntiles - 1)) {
          q_next = true;
          if (!load_q(J, i + 1)) {
            ok = false;
            break;
          }
        }
      }
      if (ok && !q_next) ok = load_q(J, i + 1);
      u = I.end;
      I = J;
    }
    // this CTA's copies still in flight land before it may leave
    if (lane == 0) {
      int s2 = st;
      uint32_t p2 = ph;
      for (int k = 0; k < min(armed, stages); ++k) {
        if (--s2 < 0) {
          s2 = stages - 1;
          p2 ^= 1;
        }
        mbar_wait_drain(&full[s2], p2);
      }
      for (int k = 0; k < min(q_armed, 2); ++k) {
        const int i = q_armed - 1 - k;
        mbar_wait_drain(&q_full[i & 1], (i >> 1) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 1 && !lead) {
    // ------------------------------------------------- relay (odd CTA)
    // The odd CTA's copies complete on its own barriers; each completed phase
    // is passed on to the same barrier of the even CTA, in the order the
    // producers issue them.
    if (lane == 0) {
      const uint32_t lk = pair::map_shared(k_full, 0), lv = pair::map_shared(v_full, 0);
      const uint32_t lq = pair::map_shared(q_full, 0);
      int kst = 0, vst = 0;
      uint32_t kph = 0, vph = 0;
      bool ok = true;
      auto relay_q = [&](int i) {
        if (!mbar_wait(&q_full[i & 1], (i >> 1) & 1, abort_flag)) return false;
        pair::arrive_cluster(lq + (i & 1) * 8);
        return true;
      };
      PrefixSegment I{};
      if (u_begin < u_end) {
        I = prefix_pair_segment<G>(u_begin, u_end, prm);
        ok = relay_q(0);
      }
      for (int i = 0, u = u_begin; ok && u < u_end; ++i) {
        const bool has_next = I.end < u_end;
        PrefixSegment J{};
        if (has_next) J = prefix_pair_segment<G>(I.end, u_end, prm);
        bool q_next = !has_next;
        for (int t = 0; ok && t < I.ntiles; ++t) {
          if (!mbar_wait(&k_full[kst], kph, abort_flag)) {
            ok = false;
            break;
          }
          pair::arrive_cluster(lk + kst * 8);
          if (++kst == stages) {
            kst = 0;
            kph ^= 1;
          }
          if (!mbar_wait(&v_full[vst], vph, abort_flag)) {
            ok = false;
            break;
          }
          pair::arrive_cluster(lv + vst * 8);
          if (++vst == stages) {
            vst = 0;
            vph ^= 1;
          }
          if (!q_next && t == min(1, I.ntiles - 1)) {
            q_next = true;
            ok = relay_q(i + 1);
          }
        }
        if (ok && !q_next) ok = relay_q(i + 1);
        u = I.end;
        I = J;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ----------------------------------------- MMA issuer (even CTA)
    if (lane == 0) {
      constexpr uint32_t idesc_s = tc::idesc_f16<kBf16>(kPairRows, kUmmaTile, false, false);
      constexpr uint32_t idesc_o = tc::idesc_f16<kBf16>(kPairRows, D, false, true);
      const uint64_t q_desc = tc::smem_desc_sw128(smem_addr(s_q), 16, 1024);
      const uint64_t k_desc = tc::smem_desc_sw128(smem_addr(s_k), 16, 1024);
      const uint64_t v_desc = tc::smem_desc_sw128(smem_addr(s_v), kVHalf, 1024);
      bool ok = true;
      int kst = 0, vst = 0;
      uint32_t kph = 0, vph = 0;
      int tau_s = 0, tau_p = 0;
      auto issue_s = [&](int qb) {
        if (!mbar_wait(&k_full[kst], kph, abort_flag)) return false;
        tc::fence_after_sync();
        const uint64_t kb = k_desc + ((kst * kKHalf) >> 4);
        const uint64_t qbd = q_desc + ((qb * kQBytes) >> 4);
        const uint32_t d = tmem + static_cast<uint32_t>(tau_s & 1) * kPairSBufCols;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          tc::mma_pair_ss(d, qbd + (((kk >> 2) * kQPanel + (kk & 3) * 32) >> 4),
                          kb + (((kk >> 2) * kKPanel + (kk & 3) * 32) >> 4), idesc_s, kk > 0);
        tc::commit_pair(&s_full[tau_s & 1], kBoth);
        if (++kst == stages) {
          kst = 0;
          kph ^= 1;
        }
        ++tau_s;
        return true;
      };
      auto issue_pv = [&](bool first) {
        const uint64_t vb = v_desc + ((vst * kVHalf) >> 4);
        const uint32_t a = tmem + static_cast<uint32_t>(tau_p & 1) * kPairSBufCols;
        const uint32_t o = tmem + kPairOCol + static_cast<uint32_t>(tau_p & 1) * D;
#pragma unroll
        for (int kk = 0; kk < kUmmaTile / 16; ++kk)
          tc::mma_pair_ts(o, a + 32 * (kk >> 1) + 8 * (kk & 1), vb + ((kk * 16 * 128) >> 4), idesc_o,
                          !first || kk > 0);
        tc::commit_pair(&v_empty[vst], kBoth);
        if (++vst == stages) {
          vst = 0;
          vph ^= 1;
        }
        ++tau_p;
      };
      int items = 0;
      for (int u = u_begin; ok && u < u_end; ++items) {
        const PrefixSegment I = prefix_pair_segment<G>(u, u_end, prm);
        u = I.end;
        const int qb = items & 1;
        if (!mbar_wait(&q_full[qb], (items >> 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        const int n = I.ntiles;
        for (int j = 0; ok && j < min(2, n); ++j) ok = issue_s(qb);
        if (!ok) break;
        if (n <= 2) tc::commit_pair(&q_empty[qb], kBoth);
        for (int j = 0; j < n; ++j) {
          // V of this tile landed with its K, which S waited for
          if (!mbar_wait(&p_full[tau_p & 1], (tau_p >> 1) & 1, abort_flag) ||
              (j == 0 && items > 0 && !mbar_wait(o_free, (items - 1) & 1, abort_flag))) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          issue_pv(j < 2);
          if (j + 2 < n) {
            if (!issue_s(qb)) {
              ok = false;
              break;
            }
            if (j + 3 == n) tc::commit_pair(&q_empty[qb], kBoth);
          }
        }
      }
      tc::commit_pair(drain, 0x1);
      mbar_wait_drain(drain, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------- softmax
    // Two groups of eight warps: group g takes the token tiles with tau mod 2
    // = g (score buffer S_g, accumulator O_g) with its own reference maximum
    // and sum, so one group's exponentials overlap the other's loads,
    // exchanges and stores.  In a group two threads share a query row: half h
    // takes scores 64 h .. 64 h + 63, 32 at a time.
    const int sw = warp - kPairSoftmaxWarp0;
    const int g = sw / kPairGroupWarps;                        // tile parity
    const int half = (sw >> 2) & 1;                            // scores 64 half ..
    const int quarter = warp & 3;                              // tensor-memory lane quarter
    const int row = quarter * 32 + lane;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint32_t s_col = t_lane + static_cast<uint32_t>(g) * kPairSBufCols + half * kPairHalfScores;
    const uint32_t og_col = t_lane + kPairOCol + static_cast<uint32_t>(g) * D + half * (D / 2);   // own half of O_g
    const int cq = g * kPairGroupRowThreads + half;            // O columns 32 cq .. of the partial
    const float qk = prm.qk_scale;
    const float pad = qk >= 0.f ? -INFINITY : INFINITY;
    const float2 qk2 = make_float2(qk, qk);
    const uint32_t lead_p_full = pair::map_shared(&p_full[g], 0);
    const uint32_t lead_o_free = pair::map_shared(o_free, 0);
    // raw scores, chunk c of this half (columns 32 c ..), nq of them valid
    auto load_chunk = [&](uint32_t (&x)[32], int c, int nq) {
      tc::tmem_ld32(s_col + 32 * c, x);
      tc::tmem_wait_ld();
      if (nq < 32) {
#pragma unroll
        for (int j = 0; j < 32; ++j) x[j] = j < nq ? x[j] : __float_as_uint(pad);
      }
    };
    // largest (smallest, for a negative scale) raw score of x
    auto chunk_ext = [&](const uint32_t (&x)[32]) {
      float cm[4] = {__uint_as_float(x[0]), __uint_as_float(x[1]), __uint_as_float(x[2]), __uint_as_float(x[3])};
      if (qk >= 0.f) {
#pragma unroll
        for (int j = 4; j < 28; j += 8)
#pragma unroll
          for (int i = 0; i < 4; ++i) cm[i] = fmax3(cm[i], __uint_as_float(x[j + i]), __uint_as_float(x[j + 4 + i]));
#pragma unroll
        for (int i = 0; i < 4; ++i) cm[i] = fmaxf(cm[i], __uint_as_float(x[28 + i]));
        return fmaxf(fmax3(cm[0], cm[1], cm[2]), cm[3]);
      }
#pragma unroll
      for (int j = 4; j < 28; j += 8)
#pragma unroll
        for (int i = 0; i < 4; ++i) cm[i] = fmin3(cm[i], __uint_as_float(x[j + i]), __uint_as_float(x[j + 4 + i]));
#pragma unroll
      for (int i = 0; i < 4; ++i) cm[i] = fminf(cm[i], __uint_as_float(x[28 + i]));
      return fminf(fmin3(cm[0], cm[1], cm[2]), cm[3]);
    };
    // P = 2^(s * qk - m_ref) of the 32 scores in x rounded to T, two per
    // column, into columns 32 c .. 32 c + 15 of this half (over the chunk's
    // own scores); their sum before rounding into ls.  Of every 16
    // exponentials kPolyExp are taken by the FMA-pipe polynomial; scores past
    // the end of the tile get weight 0.
    auto weights_store = [&](uint32_t (&x)[32], float m_ref, int nq, int c, float2 (&ls)[2]) {
      const float2 nm2 = make_float2(-m_ref, -m_ref);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float2 e = nm2;
        ffma2(e, make_float2(__uint_as_float(x[2 * i]), __uint_as_float(x[2 * i + 1])), qk2);
        x[2 * i] = __float_as_uint(e.x);
        x[2 * i + 1] = __float_as_uint(e.y);
      }
#pragma unroll
      for (int b = 0; b < 2; ++b) {
#pragma unroll
        for (int j = 0; j < 16 - kPolyExp; ++j)
          x[16 * b + j] = __float_as_uint(exp2_approx(__uint_as_float(x[16 * b + j])));
#pragma unroll
        for (int j = 16 - kPolyExp; j < 16; j += 2) {
          const float2 y = exp2_poly2(make_float2(__uint_as_float(x[16 * b + j]), __uint_as_float(x[16 * b + j + 1])));
          x[16 * b + j] = __float_as_uint(y.x);
          x[16 * b + j + 1] = __float_as_uint(y.y);
        }
      }
      if (nq < 32) {
#pragma unroll
        for (int j = 0; j < 32; ++j) x[j] = j < nq ? x[j] : 0u;
      }
      uint32_t w[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float2 e = make_float2(__uint_as_float(x[2 * i]), __uint_as_float(x[2 * i + 1]));
        w[i] = M::pack(e.x, e.y);
        fadd2(ls[i & 1], e);
      }
      tc::tmem_st16(s_col + 32 * c, w);
    };
    int tau = 0, items = 0;
    bool ok = true;
    for (int u = u_begin; ok && u < u_end; ++items) {
      const PrefixSegment I = prefix_pair_segment<G>(u, u_end, prm);
      u = I.end;
      const int tau0 = tau;
      tau += I.ntiles;
      const int gr = I.row0 + static_cast<int>(rank) * kUmmaRows + row;
      const bool valid = gr < rows_total;
      const int s_idx = valid ? gr / G : 0;
      const int g_idx = valid ? gr - s_idx * G : 0;
      float m = -INFINITY, l = 0.f;
      const int t_first = (g - tau0) & 1;                      // this group's first tile of the segment
      for (int t = t_first; t < I.ntiles; t += 2) {
        const int tt = tau0 + t;
        const uint32_t ph = (tt >> 1) & 1;                     // this group's tile count parity
        const int ntok = min(kUmmaTile, I.tok_hi - (I.tok_lo + t * kUmmaTile));
        const int nh = min(kPairHalfScores, max(0, ntok - half * kPairHalfScores));
        const int nq0 = min(32, nh), nq1 = max(0, nh - 32);
        if (!__all_sync(kFull, mbar_wait(&s_full[g], ph, abort_flag))) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        uint32_t x[32];
        load_chunk(x, 0, nq0);
        const float e0 = chunk_ext(x);
        load_chunk(x, 1, nq1);                                 // x holds chunk 1 from here
        const float e1 = chunk_ext(x);
        const float ext = qk >= 0.f ? fmaxf(e0, e1) : fminf(e0, e1);
        const float c_own = nh > 0 ? ext * qk : -INFINITY;
        float* slot = x_max + ((g * 2 + static_cast<int>(ph)) * kUmmaRows + row) * kPairGroupRowThreads;
        slot[half] = c_own;
        __syncwarp();
        if (lane == 0) mbar_arrive(&xq[g * 4 + quarter]);
        if (!__all_sync(kFull, mbar_wait(&xq[g * 4 + quarter], ph, abort_flag))) {
          ok = false;
          break;
        }
        const float c = fmaxf(c_own, slot[half ^ 1]);
        const bool need = c > m + kTau;
        if (__any_sync(kFull, need)) {
          const float mn = need ? c : m;
          const float f = mn != m ? exp2_approx(m - mn) : 1.f;     // 0 when m was -inf
          if (t >= 2) {
            // O_g holds the group's earlier products of the segment once
            // PV(tt - 2) has completed; this thread's half of O_g
            if (!__all_sync(kFull, mbar_wait(&k_empty[(tt - 2) % stages], ((tt - 2) / stages) & 1, abort_flag))) {
              ok = false;
              break;
            }
            tc::fence_after_sync();
#pragma unroll 1
            for (int ob = 0; ob < 4; ++ob) {
              uint32_t o[16];
              tc::tmem_ld16(og_col + ob * 16, o);
              tc::tmem_wait_ld();
#pragma unroll
              for (int j = 0; j < 16; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * f);
              tc::tmem_st16(og_col + ob * 16, o);
            }
          }
          l *= f;
          m = mn;
        }
        // chunk 1 from the registers first (its weights overwrite only its own
        // scores), then chunk 0 again from tensor memory
        float2 ls[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        weights_store(x, m, nq1, 1, ls);
        load_chunk(x, 0, nq0);
        weights_store(x, m, nq0, 0, ls);
        tc::tmem_wait_st();
        l += (ls[0].x + ls[1].x) + (ls[0].y + ls[1].y);
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) {
          if (lead) mbar_arrive(&p_full[g]);
          else pair::arrive_cluster(lead_p_full);
        }
      }
      if (!ok) break;
      if (I.ntiles > 0) {
        // the segment's last product has completed: O_0 and O_1 are final
        if (!__all_sync(kFull, mbar_wait(&k_empty[(tau - 1) % stages], ((tau - 1) / stages) & 1, abort_flag))) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
      }
      // the row's (m, l) of both groups: O = 2^(m_0 - M) O_0 + 2^(m_1 - M) O_1
      const int sb = items & 1;
      float2* ml = s_ml + (sb * kUmmaRows + row) * kPairRowThreads;
      ml[cq] = make_float2(m, l);
      __syncwarp();
      if (lane == 0) mbar_arrive(&sq[sb * 4 + quarter]);
      if (!__all_sync(kFull, mbar_wait(&sq[sb * 4 + quarter], (items >> 1) & 1, abort_flag))) {
        ok = false;
        break;
      }
      const float4 a01 = *reinterpret_cast<const float4*>(ml);
      const float4 a23 = *reinterpret_cast<const float4*>(ml + 2);
      const bool has0 = I.ntiles > ((0 - tau0) & 1), has1 = I.ntiles > ((1 - tau0) & 1);
      const float m0 = a01.x, l0 = a01.y + a01.w, m1 = a23.x, l1 = a23.y + a23.w;
      const float mx = fmaxf(has0 ? m0 : -INFINITY, has1 ? m1 : -INFINITY);
      const float f0 = has0 ? exp2_approx(m0 - mx) : 0.f;
      const float f1 = has1 ? exp2_approx(m1 - mx) : 0.f;
      const size_t pi = (static_cast<size_t>(s_idx) * prm.num_q_heads + I.h * G + g_idx) * prm.max_parts + I.split0;
      float* dst = prm.part_acc + pi * D + cq * 32;
      const uint32_t o0_col = t_lane + kPairOCol + cq * 32, o1_col = o0_col + D;
#pragma unroll 1
      for (int ob = 0; ob < 2; ++ob) {
        uint32_t a0[16], a1[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) a0[j] = a1[j] = 0u;
        if (has0) tc::tmem_ld16(o0_col + ob * 16, a0);
        if (has1) tc::tmem_ld16(o1_col + ob * 16, a1);
        tc::tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j)
          a0[j] = __float_as_uint(f0 * __uint_as_float(a0[j]) + f1 * __uint_as_float(a1[j]));
        if (valid) {
#pragma unroll
          for (int j = 0; j < 16; j += 4)
            *reinterpret_cast<float4*>(dst + ob * 16 + j) = make_float4(
                __uint_as_float(a0[j]), __uint_as_float(a0[j + 1]), __uint_as_float(a0[j + 2]), __uint_as_float(a0[j + 3]));
        }
      }
      if (valid && cq == 0) {
        prm.part_ml[pi] = make_float2(mx, f0 * l0 + f1 * l1);
        for (int sp = 1; sp < I.split1 - I.split0; ++sp) prm.part_ml[pi + sp] = make_float2(-INFINITY, 0.f);
      }
      // O_0 and O_1 have been read out: the next segment's first products may overwrite them
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        if (lead) mbar_arrive(o_free);
        else pair::arrive_cluster(lead_o_free);
      }
    }
  }

  // both CTAs: every product has completed (the even CTA's issuer drained
  // them) and every copy has landed before the tensor memory goes
  tc::fence_before_sync();
  __syncthreads();
  pair::cluster_sync();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc_pair(tmem, kUmmaTmemCols);
  }
}

}  // namespace pa

#endif
