// Shared-prefix ("cascade") decode, prefix half, on the fifth-generation
// tensor cores (tcgen05 + tensor memory), sm_100a: the one-SM form, used for
// head_dim 64, where no cluster of two CTAs fits, and with
// PA_PREFIX_PATH=umma (the SM-pair form in prefix_tc2.cuh is the default).
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
// Roles (576 threads):
//   warp 0     TMA producer: both query tiles once (a 4-D box over q), then
//              128-token K and V tiles of the prefix, straight from the paged
//              cache through the block list (read once into registers), into
//              two rings of `stages` 128-byte-swizzled tiles
//              ([D/64 panels][128 tok][128 B]); each tile serves both query
//              tiles.
//   warp 1     allocates all 512 tensor-memory columns; lane 0 issues the
//              MMAs.  Query tile g owns columns 256g..256g+255: S (0..127)
//              and O (128..).  Token tile t of query tile g:
//                S_g(t)  = Q_g K_t^T  (M 128, N 128, K = D; both from shared memory)
//                O_g    += P_g(t) V_t (M 128, N = D, K 128; P read from tensor
//                                      memory over the scores: tokens 0..63 in
//                                      S columns 0..31, 64..127 in 64..95)
//              issued as PV_0(t), S_0(t+1), PV_1(t), S_1(t+1): while one query
//              tile's softmax runs, the tensor core works for the other.
//              Every MMA here is 64 cycles of tensor work (M 128, N 128,
//              K 16); narrower tiles (N 64) were measured to take about as
//              long per instruction, i.e. twice as long per token.
//   warps 2-17 softmax, eight warps per query tile, two threads per query row
//              (tensor-memory lane): thread half 0 takes scores 0..63 of a
//              token tile, half 1 scores 64..127.  Per token tile: the
//              maximum of each half, exchanged through shared memory between
//              the two threads of a row; the decode kernel's threshold rule
//              for the reference maximum (it moves only when a scaled score
//              passes it by 2^8; each thread then rescales its half of O in
//              tensor memory); P = 2^(s*scale*log2(e) - m) rounded to the
//              cache's 16-bit type and stored over S as the A operand of PV;
//              each thread sums its rounded weights, and the two sums of a
//              row are added at the end.  Four warps per SM sub-partition
//              share the MUFU and the other pipes, which one warp alone
//              cannot keep busy (its instructions issue in order).
// Products issued by one thread run in issue order, and a commit arrives only
// once everything issued before it has completed.  So S_g(t+1) may overwrite
// P_g(t) as soon as PV_g(t) is issued, and when S_g(t) is reported ready,
// PV_g(t-1) has completed and O may be rescaled.  Q is loaded once per CTA
// (rows beyond the batch are zero; a second tile with no rows at all is
// skipped).  Every wait is bounded in time; on a timeout all roles fall
// through to the end, the MMA issuer waits for its own products, and the
// tensor memory is released before the CTA exits.
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

// 4-D tile load global -> shared through a tensor map, completing on `bar`.
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1, int c2,
                                            int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_addr(bar))
      : "memory");
}

constexpr int kUmmaRows = 128;        // query rows per tile (MMA M)
constexpr int kUmmaTiles = 2;         // query tiles per CTA
constexpr int kUmmaTile = 128;        // prefix tokens per stage (MMA N of S, K of PV)
constexpr int kSoftmaxWarps = 8;                      // per query tile: two threads per row
constexpr int kUmmaThreads = 64 + kUmmaTiles * kSoftmaxWarps * 32;   // producer, MMA, softmax groups
constexpr uint32_t kUmmaTmemCols = 512;
constexpr uint32_t kUmmaGroupCols = 256;              // per query tile: S 0..127, O 128..255
constexpr uint32_t kSCol = 0, kOCol = 128;
constexpr int kGroupBars = 5;                         // mbarriers per query tile
#ifndef PA_PREFIX_POLY_EXP
#define PA_PREFIX_POLY_EXP 2
#endif
// Of every 16 exponentials of the softmax, this many are evaluated on the FMA
// pipe (exp2_poly2) and the rest by the MUFU, whose one instruction per 8
// cycles per SM sub-partition is otherwise the softmax's bound.
constexpr int kPolyExp = PA_PREFIX_POLY_EXP;
static_assert(kPolyExp % 2 == 0 && kPolyExp >= 0 && kPolyExp <= 16, "pairs of exponentials");

// 2^x for a pair of float32 values on the FMA pipe (no MUFU), by Cody-Waite
// range reduction and a polynomial: x = n + f with n = round(x) and
// |f| <= 1/2 (rounding through the float32 addition of 1.5 * 2^23), 2^f from
// the degree-3 polynomial of least maximum relative error on [-1/2, 1/2]
// (Remez exchange; relative error 7.5e-5, below half a unit in the last place
// of bf16 and f16 weights), and 2^n added to the exponent field.  Inputs are
// clamped to >= -125, so the result is a normal float32 (2^x below that is
// returned as about 2^-125, which no weight of a row with a finite maximum
// can tell from zero); inputs here are <= 8 (the threshold rule).
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  constexpr float kShift = 12582912.0f;                  // 1.5 * 2^23
  constexpr float c0 = 0.99992807f, c1 = 0.69326099f, c2 = 0.24261112f, c3 = 0.05517167f;
  x.x = fmaxf(x.x, -125.f);
  x.y = fmaxf(x.y, -125.f);
  float2 t = x;
  fadd2(t, make_float2(kShift, kShift));                 // n in the low mantissa bits
  float2 r = t;
  fadd2(r, make_float2(-kShift, -kShift));               // n as a float, exactly
  float2 f = x;
  ffma2(f, r, make_float2(-1.f, -1.f));                  // f = x - n
  float2 p = make_float2(c2, c2);
  ffma2(p, f, make_float2(c3, c3));                      // c2 + c3 f
  float2 p1 = make_float2(c1, c1);
  ffma2(p1, f, p);                                       // c1 + f (c2 + c3 f)
  float2 p0 = make_float2(c0, c0);
  ffma2(p0, f, p1);                                      // c0 + f (...)
  const int nx = __float_as_int(t.x) - __float_as_int(kShift);
  const int ny = __float_as_int(t.y) - __float_as_int(kShift);
  return make_float2(__int_as_float(__float_as_int(p0.x) + (nx << 23)),
                     __int_as_float(__float_as_int(p0.y) + (ny << 23)));
}
// At least half of an SM's shared memory, so that one CTA holds the SM (and
// all of its tensor memory) whatever the head size.
constexpr size_t kUmmaMinSmem = 120 * 1024;

template <int D>
__host__ __device__ constexpr size_t prefix_umma_layout_bytes(int stages) {
  return kSmemAlign + kUmmaTiles * static_cast<size_t>(D / 64) * kUmmaRows * 128         // Q panels
         + 2 * static_cast<size_t>(stages) * (D / 64) * kUmmaTile * 128                 // K and V rings
         + (4 * static_cast<size_t>(stages) + kGroupBars * kUmmaTiles + 1 + kUmmaTiles * 4 * 3 + 1) * sizeof(uint64_t)
         + kUmmaTiles * 2 * 3 * kUmmaRows * sizeof(float);
}

template <int D>
__host__ __device__ constexpr size_t prefix_umma_smem_bytes(int stages) {
  return prefix_umma_layout_bytes<D>(stages) < kUmmaMinSmem ? kUmmaMinSmem : prefix_umma_layout_bytes<D>(stages);
}

// Work of the persistent grid.  A unit is one slice of split_tokens prefix
// tokens for one query-tile pair xb (rows 256 xb ..) and one KV head h;
// units are numbered slice-fastest within a run, run = xb * num_kv_heads + h.
// With the query-tile pairs outermost, equal shares put the CTAs that need the
// same (head, slice) for different query tiles at the same slice at the same
// time whenever the grid is a multiple of the number of pairs (148 CTAs and 4
// pairs here), so each K/V tile comes from DRAM once and from L2 after.
// Each CTA takes a contiguous share of units (stream-K style), and a segment
// is the part of its share that lies in one run: consecutive slices of the
// same query tiles and head, accumulated into one partial (m, l, O) that goes
// to the slot of the segment's first slice; the other slots of the segment
// get (m, l) = (-inf, 0) and are skipped by the merge.
struct PrefixSegment {
  int h, split0, split1, tok_lo, tok_hi, ntiles, row0, ngroups;
  int end;                       // first unit after the segment
};

template <int G>
__device__ __forceinline__ PrefixSegment prefix_segment(int u, int u_end, const PrefixParams& prm) {
  PrefixSegment Sg;
  const int ns = prm.num_splits;
  const int run = u / ns;
  Sg.split0 = u - run * ns;
  Sg.end = min(u_end, (run + 1) * ns);
  Sg.split1 = Sg.split0 + (Sg.end - u);
  const int xb = run / prm.num_kv_heads;
  Sg.h = run - xb * prm.num_kv_heads;
  Sg.tok_lo = Sg.split0 * prm.split_tokens;
  Sg.tok_hi = min(prm.prefix_len, Sg.split1 * prm.split_tokens);
  Sg.ntiles = Sg.tok_hi > Sg.tok_lo ? (Sg.tok_hi - Sg.tok_lo + kUmmaTile - 1) / kUmmaTile : 0;
  Sg.row0 = xb * (kUmmaTiles * kUmmaRows);
  Sg.ngroups = min(kUmmaTiles, (prm.num_seqs * G - Sg.row0 + kUmmaRows - 1) / kUmmaRows);
  return Sg;
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kUmmaThreads, 1)
    prefix_umma_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ CUtensorMap tm_q, const PrefixParams prm) {
  static_assert(sizeof(T) == 2, "tensor-core path takes 16-bit caches");
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  constexpr int kHalves = D / 64;                        // 128-byte panels per row
  constexpr uint32_t kPanel = kUmmaTile * 128;           // one panel of a K/V tile (16 KB)
  constexpr uint32_t kTileBytes = kHalves * kPanel;      // K (or V) bytes per stage
  constexpr uint32_t kQPanel = kUmmaRows * 128;          // one panel of Q (16 KB)
  constexpr uint32_t kQBytes = kHalves * kQPanel;        // one query tile
  constexpr int kH = 64;                                 // scores per half tile
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  using M = MmaType<T>;

  extern __shared__ __align__(1024) unsigned char smem[];
  const uintptr_t base =
      (reinterpret_cast<uintptr_t>(smem) + kSmemAlign - 1) & ~static_cast<uintptr_t>(kSmemAlign - 1);
  const int stages = prm.stages;
  unsigned char* s_q = reinterpret_cast<unsigned char*>(base);          // [tile][panel][128 rows][128 B]
  unsigned char* s_k = s_q + kUmmaTiles * kQBytes;
  unsigned char* s_v = s_k + static_cast<size_t>(stages) * kTileBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_v + static_cast<size_t>(stages) * kTileBytes);
  uint64_t* k_full = bars;
  uint64_t* k_empty = k_full + stages;
  uint64_t* v_full = k_empty + stages;
  uint64_t* v_empty = v_full + stages;
  // per query tile g: s_full (S ready), p_full (P ready, O rescaled), o_done
  // (an item's last PV), o_free (the softmax has read O out), q_full (Q landed)
  uint64_t* grp = v_empty + stages;
  auto s_full = [&](int g) { return grp + kGroupBars * g; };
  auto p_full = [&](int g) { return grp + kGroupBars * g + 1; };
  auto o_done = [&](int g) { return grp + kGroupBars * g + 2; };
  auto o_free = [&](int g) { return grp + kGroupBars * g + 3; };
  auto q_full = [&](int g) { return grp + kGroupBars * g + 4; };
  uint64_t* drain = grp + kGroupBars * kUmmaTiles;
  // the two threads of a row exchange their halves' maxima (per query tile,
  // lane quarter and token-tile parity) and, at the end of an item, their sums
  uint64_t* pair_bars = drain + 1;                      // [tile][quarter][parity]
  uint64_t* sum_bars = pair_bars + kUmmaTiles * 4 * 2;  // [tile][quarter]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sum_bars + kUmmaTiles * 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // row maxima of the two score halves, [tile][half][tile parity][row], then sums [tile][half][row]
  float* s_xmax = reinterpret_cast<float*>(sum_bars + kUmmaTiles * 4 + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rows_total = prm.num_seqs * G;
  // this CTA's share of the units
  const int u_begin = static_cast<int>(static_cast<long long>(blockIdx.x) * prm.num_units / gridDim.x);
  const int u_end = static_cast<int>(static_cast<long long>(blockIdx.x + 1) * prm.num_units / gridDim.x);

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
      mbar_init(p_full(g), kSoftmaxWarps);
      mbar_init(o_done(g), 1);
      mbar_init(o_free(g), kSoftmaxWarps);
      mbar_init(q_full(g), 1);
    }
    mbar_init(drain, 1);
    for (int i = 0; i < kUmmaTiles * 4 * 3; ++i) mbar_init(&pair_bars[i], 2);   // pair and sum barriers
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
    bool ok = true;
    for (int u = u_begin; ok && u < u_end;) {
      const PrefixSegment I = prefix_segment<G>(u, u_end, prm);
      u = I.end;
      // the block id of this lane's piece of each tile, read one tile ahead
      auto piece_block = [&](int t) {
        const int tok0 = I.tok_lo + t * kUmmaTile;
        const int ntok = min(kUmmaTile, I.tok_hi - tok0);
        const int pc = lane / kHalves;
        return pc * piece_rows < ntok ? __ldg(prm.prefix_blocks + (tok0 + pc * piece_rows) / BS) : 0;
      };
      int next_phys = I.ntiles > 0 ? piece_block(0) : 0;
      for (int t = 0; t < I.ntiles; ++t) {
        const int tok0 = I.tok_lo + t * kUmmaTile;
        const int ntok = min(kUmmaTile, I.tok_hi - tok0);
        const int npieces = ntok / piece_rows;     // <= 16
        // one box per lane: piece pc = lane / kHalves, panel hf = lane % kHalves
        const int nbox = npieces * kHalves;        // <= 32
        const int pc = lane / kHalves;
        const int hf = lane - pc * kHalves;
        int phys = next_phys;
        if (t + 1 < I.ntiles) next_phys = piece_block(t + 1);
        int row = 0;
        if (lane < nbox) {
          if (phys < 0 || phys >= prm.num_blocks) {
            set_device_error(DEVERR_BAD_BLOCK_ID);
            phys = 0;
          }
          const int tk = tok0 + pc * piece_rows;
          row = phys * BS + (tk - (tk / BS) * BS);
        }
        const uint32_t tx = static_cast<uint32_t>(nbox) * piece_rows * 128;
        // K tile
        if (!__all_sync(0xffffffffu, mbar_wait(&k_empty[kst], kph ^ 1, abort_flag))) {
          ok = false;
          break;
        }
        if (lane == 0) mbar_arrive_expect_tx(&k_full[kst], tx);
        __syncwarp();
        if (lane < nbox)
          tma_load_3d(s_k + static_cast<size_t>(kst) * kTileBytes + hf * kPanel + pc * piece_rows * 128, &tm_k,
                      &k_full[kst], 0, I.h * kHalves + hf, row, policy);
        ++k_armed;
        if (++kst == stages) {
          kst = 0;
          kph ^= 1;
        }
        // V tile; rows past the end of a short last tile are zeroed so that
        // P = 0 there never meets stale bits
        if (!__all_sync(0xffffffffu, mbar_wait(&v_empty[vst], vph ^ 1, abort_flag))) {
          ok = false;
          break;
        }
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
          tma_load_3d(vdst + hf * kPanel + pc * piece_rows * 128, &tm_v, &v_full[vst], 0, I.h * kHalves + hf, row,
                      policy);
        ++v_armed;
        if (++vst == stages) {
          vst = 0;
          vph ^= 1;
        }
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
      const uint64_t k_desc = tc::smem_desc_sw128(smem_addr(s_k), 16, 1024);
      const uint64_t v_desc = tc::smem_desc_sw128(smem_addr(s_v), kPanel, 1024);
      bool ok = true;
      int kst = 0, vst = 0;
      uint32_t kph = 0, vph = 0;
      int items_g[kUmmaTiles] = {0, 0};          // items each query tile has taken so far
      int tiles_g[kUmmaTiles] = {0, 0};          // token tiles each query tile has taken so far
      // S_g = Q_g K^T into columns 256g..256g+127
      auto issue_s = [&](int g, int ks) {
        const uint64_t kb = k_desc + ((ks * kTileBytes) >> 4);
        const uint64_t qb = q_desc + ((g * kQBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          tc::mma_f16_ss(tmem + g * kUmmaGroupCols + kSCol, qb + (((kk >> 2) * kQPanel + (kk & 3) * 32) >> 4),
                         kb + (((kk >> 2) * kPanel + (kk & 3) * 32) >> 4), idesc_s, kk > 0);
        tc::commit(s_full(g));
      };
      // O_g += P_g V; P two 16-bit values per column, tokens 0..63 in S
      // columns 0..31 and tokens 64..127 in S columns 64..95 (each softmax
      // thread writes its weights over its own half of the scores)
      auto issue_pv = [&](int g, int vs, bool first) {
        const uint64_t vb = v_desc + ((vs * kTileBytes) >> 4);
        const uint32_t col = tmem + g * kUmmaGroupCols;
#pragma unroll
        for (int kk = 0; kk < kUmmaTile / 16; ++kk)
          tc::mma_f16_ts(col + kOCol, col + kSCol + kk * 8 + (kk >= 4 ? 32 : 0), vb + ((kk * 16 * 128) >> 4), idesc_o,
                         !first || kk > 0);
      };
      for (int u = u_begin; ok && u < u_end;) {
        const PrefixSegment I = prefix_segment<G>(u, u_end, prm);
        u = I.end;
        for (int g = 0; g < I.ngroups && ok; ++g) ok = mbar_wait(q_full(g), items_g[g] & 1, abort_flag);
        if (!ok) break;
        tc::fence_after_sync();
        if (I.ntiles > 0) {
          if (!mbar_wait(&k_full[kst], kph, abort_flag)) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          for (int g = 0; g < I.ngroups; ++g) issue_s(g, kst);
          tc::commit(&k_empty[kst]);
          if (++kst == stages) {
            kst = 0;
            kph ^= 1;
          }
        }
        for (int t = 0; ok && t < I.ntiles; ++t) {
          const bool more = t + 1 < I.ntiles;
          if (!mbar_wait(&v_full[vst], vph, abort_flag) || (more && !mbar_wait(&k_full[kst], kph, abort_flag))) {
            ok = false;
            break;
          }
          for (int g = 0; g < I.ngroups; ++g) {
            // P_g(t) written (and O rescaled if the maximum moved); before the
            // first product of an item, the previous item's O read out
            if (!mbar_wait(p_full(g), tiles_g[g] & 1, abort_flag) ||
                (t == 0 && items_g[g] > 0 && !mbar_wait(o_free(g), (items_g[g] - 1) & 1, abort_flag))) {
              ok = false;
              break;
            }
            ++tiles_g[g];
            tc::fence_after_sync();
            issue_pv(g, vst, t == 0);
            if (more) issue_s(g, kst);                // overwrites P_g(t) after PV_g(t) in issue order
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
        if (!ok) break;
        for (int g = 0; g < I.ngroups; ++g) {
          tc::commit(o_done(g));
          ++items_g[g];
        }
      }
      // every product issued above completes before the tensor memory goes
      tc::commit(drain);
      mbar_wait_drain(drain, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------- softmax
    const int g = (warp - 2) / kSoftmaxWarps;                  // query tile of this group
    const int half = ((warp - 2) % kSoftmaxWarps) / 4;         // scores 64 * half .. 64 * half + 63
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;                       // tensor-memory lane = query row in the tile
    const uint32_t t_lane = tmem + g * kUmmaGroupCols + (static_cast<uint32_t>(quarter * 32) << 16);
    const bool leader = (warp - 2) % kSoftmaxWarps == 0 && lane == 0;   // loads this group's query tiles
    const float qk = prm.qk_scale;
    const float pad = qk >= 0.f ? -INFINITY : INFINITY;
    const float2 qk2 = make_float2(qk, qk);
    // the two warps holding this lane quarter's rows meet at these barriers
    // (one arrival per warp; waits bounded like every other)
    uint64_t* pair_bar = pair_bars + (g * 4 + quarter) * 2;   // + tile parity
    uint64_t* sum_bar = sum_bars + g * 4 + quarter;
    float* x_max = s_xmax + (g * 2 + half) * 2 * kUmmaRows;              // [tile parity][row], own half
    const float* y_max = s_xmax + (g * 2 + (half ^ 1)) * 2 * kUmmaRows;  // the other half
    float* s_sum = s_xmax + kUmmaTiles * 2 * 2 * kUmmaRows;              // [tile][half][row]
    // the first unit, from `u` on, of a segment in which this query tile takes
    // part (u_end if none)
    auto next_segment = [&](int u) {
      while (u < u_end) {
        const PrefixSegment J = prefix_segment<G>(u, u_end, prm);
        if (g < J.ngroups) return u;
        u = J.end;
      }
      return u_end;
    };
    // the query tile g of the segment starting at unit u into shared memory:
    // the box (64 elements, G heads, 128 / G sequences) of q viewed as
    // [S][Hq][D / 64 panels][64]; rows past the batch read as zeros
    auto load_q = [&](int u) {
      const PrefixSegment J = prefix_segment<G>(u, u_end, prm);
      mbar_arrive_expect_tx(q_full(g), kQBytes);
      for (int hf = 0; hf < kHalves; ++hf)
        tma_load_4d(s_q + g * kQBytes + hf * kQPanel, &tm_q, q_full(g), 0, hf, J.h * G, (J.row0 + g * kUmmaRows) / G);
    };
    const int first = next_segment(u_begin);
    if (leader) {
      prefetch_tensormap(&tm_q);
      if (first < u_end) load_q(first);
    }
    int tiles = 0;                               // token tiles this query tile has taken so far
    int items = 0;                               // segments this query tile has taken so far
    bool ok = true;
    for (int u = first; ok && u < u_end;) {
      const PrefixSegment I = prefix_segment<G>(u, u_end, prm);
      u = next_segment(I.end);
      const int gr = I.row0 + g * kUmmaRows + row;
      const bool valid = gr < rows_total;
      const int s_idx = valid ? gr / G : 0;
      const int g_idx = valid ? gr - s_idx * G : 0;
      float m = -INFINITY, l = 0.f;
      for (int t = 0; t < I.ntiles; ++t, ++tiles) {
        const int ntok = min(kUmmaTile, I.tok_hi - (I.tok_lo + t * kUmmaTile));
        const int nh = min(kH, max(0, ntok - half * kH));         // valid scores in this half
        if (!__all_sync(0xffffffffu, mbar_wait(s_full(g), tiles & 1, abort_flag))) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        // the segment's last S has completed, so its query tile may be replaced
        if (t == I.ntiles - 1 && leader && u < u_end) load_q(u);
        const uint32_t s_col = t_lane + kSCol + half * kH;
        // maximum (minimum for a negative scale) of this half's raw scores, 32 at a time
        float ext = pad;
#pragma unroll
        for (int q32 = 0; q32 < 2; ++q32) {
          uint32_t x[32];
          tc::tmem_ld32(s_col + q32 * 32, x);
          tc::tmem_wait_ld();
          if (nh < kH) {
#pragma unroll
            for (int j = 0; j < 32; ++j) x[j] = q32 * 32 + j < nh ? x[j] : __float_as_uint(pad);
          }
          float cm[4] = {__uint_as_float(x[0]), __uint_as_float(x[1]), __uint_as_float(x[2]), __uint_as_float(x[3])};
          if (qk >= 0.f) {
#pragma unroll
            for (int j = 4; j < 28; j += 8)
#pragma unroll
              for (int k = 0; k < 4; ++k) cm[k] = fmax3(cm[k], __uint_as_float(x[j + k]), __uint_as_float(x[j + 4 + k]));
#pragma unroll
            for (int k = 0; k < 4; ++k) cm[k] = fmaxf(cm[k], __uint_as_float(x[28 + k]));
            ext = fmax3(ext, fmax3(cm[0], cm[1], cm[2]), cm[3]);
          } else {
#pragma unroll
            for (int j = 4; j < 28; j += 8)
#pragma unroll
              for (int k = 0; k < 4; ++k) cm[k] = fmin3(cm[k], __uint_as_float(x[j + k]), __uint_as_float(x[j + 4 + k]));
#pragma unroll
            for (int k = 0; k < 4; ++k) cm[k] = fminf(cm[k], __uint_as_float(x[28 + k]));
            ext = fmin3(ext, fmin3(cm[0], cm[1], cm[2]), cm[3]);
          }
        }
        // the row's scaled maximum: this half's and the other thread's
        const float c_own = nh > 0 ? ext * qk : -INFINITY;
        x_max[(tiles & 1) * kUmmaRows + row] = c_own;
        __syncwarp();
        if (lane == 0) mbar_arrive(&pair_bar[tiles & 1]);
        if (!__all_sync(0xffffffffu, mbar_wait(&pair_bar[tiles & 1], (tiles >> 1) & 1, abort_flag))) {
          ok = false;
          break;
        }
        const float c = fmaxf(c_own, y_max[(tiles & 1) * kUmmaRows + row]);
        if (__any_sync(0xffffffffu, c > m + kTau)) {
          const float mn = c > m + kTau ? c : m;
          const float f = mn != m ? exp2_approx(m - mn) : 1.f;     // 0 when m was -inf
          if (t >= 1) {
            // O holds PV(0..t-1) of this item, all completed (S(t) was issued
            // after PV(t-1)); PV(t) waits for this tile's P.  This thread's half of O.
#pragma unroll 1
            for (int ob = 0; ob < D / 32; ++ob) {
              uint32_t o[16];
              tc::tmem_ld16(t_lane + kOCol + half * (D / 2) + ob * 16, o);
              tc::tmem_wait_ld();
#pragma unroll
              for (int j = 0; j < 16; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * f);
              tc::tmem_st16(t_lane + kOCol + half * (D / 2) + ob * 16, o);
            }
          }
          l *= f;
          m = mn;
        }
        // P = 2^(s * qk - m), rounded to T, two per column: tokens 64 * half + j
        // go to column 64 * half + j / 2, i.e. over this thread's own scores
        // already read (the other thread's columns are never touched).  Of
        // every 16 exponentials, kPolyExp are taken by the FMA-pipe polynomial.
        const float2 nm2 = make_float2(-m, -m);
        float2 ls[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int q32 = 0; q32 < 2; ++q32) {
          uint32_t x[32];
          tc::tmem_ld32(s_col + q32 * 32, x);
          tc::tmem_wait_ld();
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
              const float2 y =
                  exp2_poly2(make_float2(__uint_as_float(x[16 * b + j]), __uint_as_float(x[16 * b + j + 1])));
              x[16 * b + j] = __float_as_uint(y.x);
              x[16 * b + j + 1] = __float_as_uint(y.y);
            }
          }
          if (nh < kH) {
#pragma unroll
            for (int j = 0; j < 32; ++j) x[j] = q32 * 32 + j < nh ? x[j] : 0u;
          }
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            w[i] = M::pack(__uint_as_float(x[2 * i]), __uint_as_float(x[2 * i + 1]));
            fadd2(ls[i & 1], M::unpack(w[i]));
          }
          tc::tmem_st16(t_lane + kSCol + half * kH + q32 * 16, w);
        }
        tc::tmem_wait_st();
        l += (ls[0].x + ls[1].x) + (ls[0].y + ls[1].y);
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full(g));
      }
      if (!ok) break;
      if (I.ntiles > 0 && !__all_sync(0xffffffffu, mbar_wait(o_done(g), items & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      // the row sum: this half's and the other thread's
      s_sum[(g * 2 + half) * kUmmaRows + row] = l;
      __syncwarp();
      if (lane == 0) mbar_arrive(sum_bar);
      if (!__all_sync(0xffffffffu, mbar_wait(sum_bar, items & 1, abort_flag))) {
        ok = false;
        break;
      }
      const float l_row = l + s_sum[(g * 2 + (half ^ 1)) * kUmmaRows + row];
      const size_t pi = (static_cast<size_t>(s_idx) * prm.num_q_heads + I.h * G + g_idx) * prm.max_parts + I.split0;
      float* dst = prm.part_acc + pi * D + half * (D / 2);
#pragma unroll
      for (int cb = 0; cb < D / 64; ++cb) {
        uint32_t o[32];
        if (I.ntiles > 0) {
          tc::tmem_ld32(t_lane + kOCol + half * (D / 2) + cb * 32, o);
          tc::tmem_wait_ld();
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] = 0u;
        }
        if (valid) {
#pragma unroll
          for (int j = 0; j < 32; j += 4)
            *reinterpret_cast<float4*>(dst + cb * 32 + j) =
                make_float4(__uint_as_float(o[j]), __uint_as_float(o[j + 1]), __uint_as_float(o[j + 2]),
                            __uint_as_float(o[j + 3]));
        }
      }
      if (valid && half == 0) {
        prm.part_ml[pi] = make_float2(m, l_row);
        for (int sp = 1; sp < I.split1 - I.split0; ++sp) prm.part_ml[pi + sp] = make_float2(-INFINITY, 0.f);
      }
      // O has been read out: the next item's first product may overwrite it
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_free(g));
      ++items;
    }
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
