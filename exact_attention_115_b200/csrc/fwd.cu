// Forward attention kernel for sm_100a.
//
// FlashAttention1 post (CSDN), section "具体算法", and the FlashAttention
// V1/V2 study notes (51CTO), sections "Thread Block Level 并行" and "算法的改进":
// the query rows are cut into tiles, one group of tiles per CTA; the K/V
// sequence streams through shared memory tile by tile; each row keeps a
// running maximum m, a running denominator ℓ and an unnormalised output
// accumulator that is rescaled when m grows; O and the row logsumexp L are
// written once at the end.  Causal: K/V tiles wholly above the diagonal are
// never loaded, and only tiles that cross the diagonal (or the ragged end of
// K) are masked.  The notes' instruction-level section: the softmax uses
// exp2 with scale·log2(e) folded into one FFMA per score.
//
// B200 design (not the pages'): a CTA owns one or two 128-row Q tiles
// (fwd_tiles_for: one for 16-bit types, except two for d = 128 without a
// bias or dropout when a query tile sees 24 or more K/V tiles of 128 keys
// on average, 48 under the causal mask; two for fp32).  With two tiles (NT = 2) it ping-pongs them over 128-key K/V tiles
// so the tensor core works on one tile while the softmax warps work on the
// other.  With one tile (NT = 3) the K/V tiles have 64 keys and the score
// tile is double-buffered in TMEM, so the scores of K/V tile j + 1 are
// computed while the softmax of tile j runs; two such CTAs share an SM.
// Against one tile over 128-key K/V tiles with a single score buffer (the
// design it replaced) causal B8 H16 N2048 d128 went 168.1 -> 159.1 us, and
// with dropout p = 0.1 257.3 -> 227.0 us.  Roles per CTA (128 threads per
// tile + 128):
//   warpgroup t (warps 4t..4t+3)  softmax + correction + epilogue of Q tile t
//                                 (thread = row), 200 registers
//   last warpgroup: warp 4·TILES issues the tcgen05 MMAs (one thread) and
//                   owns TMEM, the next warp is the TMA producer, the rest idle
// TMEM: S[tiles] | O[tiles] (256 or 512 columns), or S0 | S1 | O (64, 64 and
// d columns) with double-buffered scores, at d = 64 followed by 16 columns
// of row sums of the rounded P (a P · ones product; see FwdTraits::ONES).  P overwrites S in place
// (bf16 pairs or tf32) and is read by the P·V MMA straight from TMEM.  The
// running max is only moved when it grows by more than kRescaleThreshold
// (log2 units), so the O accumulator is rescaled rarely; the result is exact
// either way because O and ℓ always share the same reference maximum.
// O is written through the tile's Q buffer (free once the tile's products
// are done) with TMA tensor stores.
#define FA_SITE_BASE 10000
#include <algorithm>

#include "common.cuh"
#include "dropout.cuh"
#include "launch.h"

namespace fa {

namespace {

#ifndef FA_RESCALE_THRESHOLD
#define FA_RESCALE_THRESHOLD 8.0f
#endif
constexpr float kRescaleThreshold = FA_RESCALE_THRESHOLD;  // log2 units: P entries stay <= 2^8

// Kernel shape of the dropout and fp32 variants: 3 (one Q tile over 64-key
// K/V tiles) for 16-bit types, 2 (two Q tiles over 128-key K/V tiles) for
// fp32; the plain 16-bit d = 128 kernels come in both (fwd_tiles_for), the
// bias variants in shape 3.
constexpr int fwd_tiles(bool tf32, int d) { return (void)d, tf32 ? 2 : 3; }

// NT: 1 or 2 Q tiles of 128 rows per CTA over K/V tiles of 128 keys, or 3:
// one Q tile over K/V tiles of 64 keys with its score tile double-buffered
// in TMEM (S0 | S1 | O = 64 + 64 + d columns), so that the next score tile
// is computed while the softmax of the current one runs.
template <typename T, int D, int NT = fwd_tiles(ElemTraits<T>::tf32, D), bool BIAS = false>
struct FwdTraits {
  static constexpr int ES = sizeof(T);
  static constexpr int BN = NT == 3 ? 64 : 128;  // keys of a K/V tile
  static constexpr int SBUF = NT == 3 ? 2 : 1;   // score buffers per Q tile
  static constexpr int AW = 128 / ES;            // elements per 128-byte swizzled row
  static constexpr int DC = D / AW;              // 128-byte column blocks in a row
  static constexpr int CHUNK = 128 * 128;        // bytes of one column block of a Q (or O) tile
  static constexpr int TILE = 128 * D * ES;      // bytes of one 128-row Q (or O) tile
  static constexpr int KV_CHUNK = BN * 128;      // bytes of one column block of a K/V tile
  static constexpr int KV_TILE = BN * D * ES;    // bytes of one K/V tile
  static constexpr int KSTEP = 32 / ES;          // K extent of one MMA instruction
  // 128-row Q tiles per CTA.  With one tile a CTA needs 256 TMEM columns and
  // under half of shared memory, so two CTAs share an SM: one's softmax runs
  // while the other's products run, and one's set-up and epilogue overlap the
  // other's main loop, at the price of loading each K/V tile twice per SM.
  // With two tiles the CTA ping-pongs its own tiles over one K/V stream.
  // Which count is faster depends on how many K/V tiles a query tile sees
  // (measurements at fwd_tiles_for).
  static constexpr int TILES = NT == 2 ? 2 : 1;
  static constexpr int CTAS_PER_SM = TILES == 1 ? 2 : 1;
  // The bias variants stage each K/V step's [128 rows × BN keys] bias tile
  // of every Q tile in shared memory: 128-byte-swizzled blocks of 64 keys,
  // so that a thread's row reads are free of bank conflicts.  They are built
  // in the one-tile form only: with the four K/V slots below it measured
  // faster than two tiles with 128-key bias tiles at every length.
  static constexpr int BIAS_TILE = BIAS ? 128 * BN * ES : 0;
  static constexpr int SMEM_BUDGET = TILES == 1 ? (BIAS ? 112 : 110) * 1024 : 200 * 1024;  // tiles, per CTA
  static constexpr int NS_RAW = (SMEM_BUDGET - TILES * (TILE + BIAS_TILE)) / KV_TILE;
  static constexpr int NS = NS_RAW > 8 ? 8 : NS_RAW;  // K/V ring slots
  static constexpr int OFF_BIAS = TILES * TILE + NS * KV_TILE;
  // d = 64, one tile: the row sums of P as rounded for the P·V product come
  // from the tensor core, P · ones[64 keys × 16] into 16 TMEM columns after
  // O, with the B operand a constant [16 × 64] K-major tile of ones.
  static constexpr bool ONES = SBUF == 2 && D == 64;
  static constexpr int ONES_TILE = ONES ? 16 * 128 : 0;
  static constexpr int OFF_ONES = OFF_BIAS + TILES * BIAS_TILE;
  static constexpr int SMEM_BAR = OFF_ONES + ONES_TILE;  // the tiles' extent
  // Dynamic shared memory a CTA may take with two per SM: 228 KB, less
  // 1 KB the system reserves per CTA, halved.
  static constexpr int SMEM_2CTA = (228 * 1024 - 2 * 1024) / 2;
  // The barriers (256 bytes) go after the tiles, plus up to 1 KB of slack to
  // align the tiles to 1024 bytes.  With one tile, a bias and d = 128 (Q,
  // four K/V slots and the bias tile: 112 KB) that is 256 bytes too many for
  // two CTAs per SM; there (TIGHT) the barriers take the alignment gap when
  // it is 256 bytes or more, and follow the tiles otherwise (the gap is then
  // under 256 bytes, so they still end within the 1 KB of slack).
  static constexpr bool TIGHT = TILES == 1 && SMEM_BAR + 256 + 1024 > SMEM_2CTA;
  static constexpr int SMEM_BYTES = SMEM_BAR + (TIGHT ? 0 : 256) + 1024;
  static constexpr int THREADS = 128 * TILES + 128;
  static constexpr int TMEM_COLS = TILES == 1 ? 256 : 512;  // S[TILES] | O[TILES], or S0 | S1 | O
  static constexpr int COL_O = TILES * SBUF * BN;            // first O column
  static constexpr int COL_R = COL_O + TILES * D;            // ONES: the row sums (16 columns)
  static constexpr int MMA_WARP = 4 * TILES;                // then the TMA producer
  static constexpr int PRODUCER_WARP = MMA_WARP + 1;
  // setmaxnreg split of the registers a CTA launches with (65536 / CTAS_PER_SM)
  static constexpr int REGS_SOFTMAX = TILES == 1 ? 200 : 200;  // per thread, softmax warpgroups
  static constexpr int REGS_OTHER = TILES == 1 ? 56 : 80;      // per thread, the last warpgroup
  static constexpr uint32_t IDESC_QK = make_idesc(ElemTraits<T>::fmt, 128, BN, 0, 0);
  static constexpr uint32_t IDESC_PV =
      make_idesc(ElemTraits<T>::fmt, 128, D, 0, ElemTraits<T>::tf32 ? 0 : 1);
  static constexpr uint32_t IDESC_R = make_idesc(ElemTraits<T>::fmt, 128, 16, 0, 0);
  static_assert(NS >= 2 * SBUF, "K/V slots for the products in flight");
  static_assert(TILES == 2 || SMEM_BYTES <= SMEM_2CTA, "two one-tile CTAs per SM");
  static_assert(!BIAS || TILES == 1, "the bias variants are one-tile kernels (fwd_tiles_for)");
  static_assert(NT == 2 || NT == 3, "two Q tiles, or one over 64-key K/V tiles");
  static_assert(NT != 3 || !ElemTraits<T>::tf32, "64-key tiles: 16-bit types");
  static_assert(COL_O + TILES * D + (ONES ? 32 : 0) <= TMEM_COLS, "TMEM budget");
  static_assert(D % AW == 0, "head dim must fill whole swizzle rows");
};


struct FwdBarriers {
  uint64_t bias_full[2];   // BIAS: tile t's bias tile for the current K/V step has landed
  uint64_t bias_empty[2];  // BIAS: tile t's softmax warps have copied it out
  uint64_t q_full[2];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_full[2];
  uint64_t kv_full[8];
  uint64_t kv_empty[8];
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(FwdBarriers) <= 256, "barriers must fit the 256 bytes reserved for them");

__device__ __forceinline__ float round_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

// One pair in every emu_period(TILES) evaluates 2^x on the FMA pipe
// (exp2_pair<true>) instead of the special-function unit, to balance the two
// pipes; 0 = none.  Measured (d = 128 bf16 forward, interleaved A/B, periods
// 4, 5, 6, 8 and none): the one-tile kernel is fastest with none (causal
// N = 2048: 175.4 us with 1 in 4, 165.3 us with none), the two-tile kernel
// with 1 in 5 (non-causal N = 8192: 961.5 us with 1 in 4, 945.0 with 1 in 5,
// 1056.8 with none).
constexpr int emu_period(int tiles) { return tiles == 1 ? 0 : 5; }

// 2^x for a pair of floats: on the special-function unit, or (EMU) on the
// FMA/ALU pipes (exp2_pair_fma in common.cuh).
template <bool EMU>
__device__ __forceinline__ float2 exp2_pair(uint64_t x2) {
  const float2 x = upk2(x2);
  if constexpr (!EMU)
    return make_float2(ex2(x.x), ex2(x.y));
  else
    return exp2_pair_fma<false>(x);
}

// fp32 inputs (TF32 tensor-core products).  The tensor core reads only the
// top 19 bits of each fp32 operand, i.e. it truncates; to keep the products
// unbiased every operand is rounded to nearest TF32 first, so the producer
// warp stages fp32 tiles itself instead of with TMA.  Rows past N are zero.
//
// K-major copy of rows [row0, row0+128) of a [N, D] fp32 matrix: row r,
// element n at column block n/32 (blocks 128*128 bytes apart), 128-byte
// swizzled rows.
template <int D>
__device__ __forceinline__ void stage_rows_tf32(const float* X, int bh, int N, int row0,
                                                uint8_t* dst, int lane) {
  const float* Xh = X + size_t(bh) * N * D;
  for (int idx = lane; idx < 128 * (D / 4); idx += 32) {
    const int r = idx / (D / 4), n4 = (idx % (D / 4)) * 4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (row0 + r < N) v = *reinterpret_cast<const float4*>(Xh + size_t(row0 + r) * D + n4);
    v = make_float4(round_tf32(v.x), round_tf32(v.y), round_tf32(v.z), round_tf32(v.w));
    const uint32_t byte = (n4 & 31) * 4;
    const uint32_t o = (n4 >> 5) * (128 * 128) + r * 128 + (((byte >> 4) ^ (r & 7)) << 4);
    *reinterpret_cast<float4*>(dst + o) = v;
  }
}

// V transposed for the P·V product: row n = d index, the 128 keys along the
// row (32 keys per 128-byte column block, blocks D*128 bytes apart).
template <int D>
__device__ __forceinline__ void stage_v_transposed_tf32(const float* V, int bh, int Nk, int key0,
                                                        uint8_t* dst, int lane) {
  const float* Vh = V + size_t(bh) * Nk * D;
  for (int idx = lane; idx < 128 * (D / 4); idx += 32) {
    const int kk = idx / (D / 4), n4 = (idx % (D / 4)) * 4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (key0 + kk < Nk) v = *reinterpret_cast<const float4*>(Vh + size_t(key0 + kk) * D + n4);
    const float vals[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int n = n4 + e;
      const uint32_t byte = (kk & 31) * 4;
      const uint32_t o = (kk >> 5) * (D * 128) + n * 128 + ((((byte >> 4) ^ (n & 7)) << 4) | (byte & 15));
      *reinterpret_cast<float*>(dst + o) = round_tf32(vals[e]);
    }
  }
}

// GEN: some tensor map is 4-D (a layout whose heads and batches do not merge
// into one index); otherwise every map is the 3-D (d, N, B·H) form.
// DROP: dropout on P (16-bit types only), masks drawn in the softmax warps.
// BIAS: an additive bias on the scaled scores (16-bit types only).
template <typename T, int D, bool CAUSAL, bool GEN, bool DROP, bool BIAS, int NT>
__global__ void __launch_bounds__(FwdTraits<T, D, NT, BIAS>::THREADS, FwdTraits<T, D, NT, BIAS>::CTAS_PER_SM)
    fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
               const __grid_constant__ CUtensorMap tmBias, FwdParams p) {
  using Tr = FwdTraits<T, D, NT, BIAS && !ElemTraits<T>::tf32>;
  // staged bias tiles (16-bit types)
  constexpr bool SBIAS = BIAS && !ElemTraits<T>::tf32;
  constexpr bool TF32 = ElemTraits<T>::tf32;
  // the rounded-P row sums by the tensor core (with dropout the product sees
  // the dropped weights, so the sums stay in the softmax threads)
  constexpr bool RSUM = Tr::ONES && !DROP;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  FwdBarriers* bars = reinterpret_cast<FwdBarriers*>(
      Tr::TIGHT && smem - smem_raw >= 256 ? smem_raw : smem + Tr::SMEM_BAR);
  volatile int* abort_flag = &bars->abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int n_qb = p.n_qblocks;
  int bh, blk;
  grouped_order(blockIdx.x, p.B * p.H, n_qb, p.head_group, bh, blk);
  const int qb = CAUSAL ? n_qb - 1 - blk : blk;  // causal: the last query blocks see the most keys
  const int q_row0 = qb * 128 * Tr::TILES;
  const int off = p.Nk - p.Nq;  // bottom-right causal alignment (full Nk)
  const int nk = keys_of(p.kv_len, bh, p.H, p.Nk);  // keys this batch element sees

  int kv_end = nk;
  if (CAUSAL) {
    const int q_last = min(q_row0 + 128 * Tr::TILES - 1, p.Nq - 1);
    kv_end = min(nk, q_last + off + 1);
  }
  // at least one (then fully masked) tile, so that every role runs its loop
  // once and an empty row still ends with O = 0 and L = -inf
  const int n_kv = max(1, (kv_end + Tr::BN - 1) / Tr::BN);

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->q_full[i], 1);
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->p_full[i], 128);
      mbar_init(&bars->o_full[i], 1);
    }
    for (int i = 0; i < 8; ++i) {
      mbar_init(&bars->kv_full[i], 1);
      mbar_init(&bars->kv_empty[i], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars->bias_full[t], 1);
      mbar_init(&bars->bias_empty[t], 128);
    }
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == Tr::MMA_WARP) {
    tmem_alloc(&bars->tmem_base, Tr::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == Tr::PRODUCER_WARP && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    if constexpr (SBIAS) tma_prefetch_desc(&tmBias);
  }
  if constexpr (RSUM) {
    if (warp == Tr::PRODUCER_WARP) {
      const uint32_t one2 = ElemTraits<T>::pack2(1.f, 1.f);
      for (int i = lane; i < Tr::ONES_TILE / 16; i += 32)
        reinterpret_cast<uint4*>(smem + Tr::OFF_ONES)[i] = make_uint4(one2, one2, one2, one2);
      fence_async_smem();  // the tensor core reads it
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  uint8_t* sQ[2] = {smem, smem + Tr::TILE};  // (the second only with two tiles)
  uint8_t* sKV = smem + Tr::TILES * Tr::TILE;
  uint8_t* sBias = smem + Tr::OFF_BIAS;  // SBIAS: [TILES][BN / 64 blocks][rows][128 B], swizzled

  if (warp > Tr::PRODUCER_WARP) {
    // idle warps of the producer/MMA warpgroup
    regs_dec<Tr::REGS_OTHER>();
  } else if (warp == Tr::PRODUCER_WARP) {
    // ------------------------------------------------------------ producer
    regs_dec<Tr::REGS_OTHER>();
    // Lane 0 issues the TMA loads (16-bit types).  fp32 tiles are staged by
    // the whole warp instead (see stage_rows_tf32).
    auto load_tile = [&](int which, uint8_t* dst, uint64_t* bar, int row) {
      // which: 0 = Q, 1 = K, 2 = V
      if constexpr (TF32) {
        const float* src = reinterpret_cast<const float*>(which == 0 ? p.Q : which == 1 ? p.K : p.V);
        if (which == 2)
          stage_v_transposed_tf32<D>(src, bh, p.Nk, row, dst, lane);
        else
          stage_rows_tf32<D>(src, bh, which == 0 ? p.Nq : p.Nk, row, dst, lane);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(bar);
      } else if (lane == 0) {
        const CUtensorMap* map = which == 0 ? &tmQ : which == 1 ? &tmK : &tmV;
        // (a tile may start past the end only by the CTA's second Q tile:
        // TMA fills its rows with zeros)
        if (!FA_INBOUNDS(bh < p.B * p.H && row >= 0 && row < (which == 0 ? p.Nq + 128 : p.Nk))) return;
        const int bytes = which == 0 ? Tr::TILE : Tr::KV_TILE, chunk = which == 0 ? Tr::CHUNK : Tr::KV_CHUNK;
        mbar_arrive_expect_tx(bar, bytes);
#pragma unroll
        for (int c = 0; c < Tr::DC; ++c)
          tma_load_bh(dst + c * chunk, map, GEN && ((p.map4d >> which) & 1), bar, c * Tr::AW, row, bh, p.H);
      }
    };
    auto load_kv = [&](int i) {  // i-th K/V tile in consumption order: K0 V0 K1 V1 ...
      const int slot = i % Tr::NS;
      bool ok = true;
      if (i >= Tr::NS)
        ok = MBAR_WAIT(&bars->kv_empty[slot], ((i / Tr::NS) - 1) & 1, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) return false;
      load_tile((i & 1) ? 2 : 1, sKV + slot * Tr::KV_TILE, &bars->kv_full[slot], (i >> 1) * Tr::BN);
      return true;
    };
    // SBIAS: K/V tile j's bias tile of each Q tile (BN / 64 swizzled blocks
    // of 64 keys; one row each when the bias is shared by all query rows, the
    // blocks a swizzle atom apart), once that tile's softmax warps have
    // copied out tile j − 1's.  Zero past Nq and Nk.
    auto load_bias = [&](int j) {
      for (int t = 0; t < Tr::TILES; ++t) {
        bool ok = j == 0 || MBAR_WAIT(&bars->bias_empty[t], (j - 1) & 1, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) return false;
        if (lane == 0 && FA_INBOUNDS(bh < p.B * p.H && j * Tr::BN < p.Nk)) {
          const int rows = p.bias_rows, half = rows > 1 ? rows * 128 : 1024;
          mbar_arrive_expect_tx(&bars->bias_full[t], (Tr::BN / 64) * rows * 128);
#pragma unroll
          for (int h = 0; h < Tr::BN / 64; ++h)
            tma_load_4d(sBias + t * Tr::BIAS_TILE + h * half, &tmBias, &bars->bias_full[t], j * Tr::BN + 64 * h,
                        rows > 1 ? q_row0 + 128 * t : 0, (bh % p.H) % p.bias_H, (bh / p.H) % p.bias_B);
        }
      }
      return true;
    };
    load_tile(0, sQ[0], &bars->q_full[0], q_row0);
    if constexpr (SBIAS) load_bias(0);
    load_kv(0);
    if constexpr (Tr::TILES == 2) load_tile(0, sQ[1], &bars->q_full[1], q_row0 + 128);
    for (int i = 1; i < 2 * n_kv; ++i) {
      if constexpr (SBIAS)
        if ((i & 1) == 0 && !load_bias(i >> 1)) break;
      if (!load_kv(i)) break;
    }
    if (lane == 0) {
      // Drain: wait until every issued load has landed before the CTA may exit.
      for (int i = max(0, 2 * n_kv - Tr::NS); i < 2 * n_kv; ++i)
        MBAR_WAIT(&bars->kv_full[i % Tr::NS], (i / Tr::NS) & 1, abort_flag);
      MBAR_WAIT(&bars->q_full[0], 0, abort_flag);
      if constexpr (Tr::TILES == 2) MBAR_WAIT(&bars->q_full[1], 0, abort_flag);
      if constexpr (SBIAS)
        for (int t = 0; t < Tr::TILES; ++t) MBAR_WAIT(&bars->bias_full[t], (n_kv - 1) & 1, abort_flag);
    }
  } else if (warp == Tr::MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    regs_dec<Tr::REGS_OTHER>();
    // The whole warp runs the loop (warp-uniform waits and descriptor
    // arithmetic); the elected lane issues the MMAs and commits.
    {
      const bool leader = elect_one();
      // score buffers: tile t (two tiles), or buffer b of the one tile (NT = 3)
      const uint32_t tS[2] = {tmem, tmem + Tr::BN};
      const uint32_t tO[2] = {tmem + Tr::COL_O, tmem + Tr::COL_O + D};
      const uint32_t aQ[2] = {smem_u32(sQ[0]), smem_u32(sQ[1])};
      const uint32_t aKV = smem_u32(sKV);

      // Operand descriptors are built once per tile; inside the unrolled
      // loops each MMA only adds a compile-time offset (in 16-byte units), so
      // the issuing thread keeps ahead of the tensor core.
      const uint64_t descQ[2] = {sw128_desc(aQ[0], 16, 1024), sw128_desc(aQ[1], 16, 1024)};
      // S of Q tile t (or into score buffer b: sb) = Q_t · K(slot)ᵀ
      auto issue_qk = [&](int t, int slot, int sb) {
        const uint64_t da = descQ[t];
        const uint64_t db = sw128_desc(aKV + slot * Tr::KV_TILE, 16, 1024);
#pragma unroll
        for (int ks = 0; ks < D / Tr::KSTEP; ++ks) {
          const uint64_t oa = uint64_t((ks >> 2) * (Tr::CHUNK / 16) + (ks & 3) * 2);
          const uint64_t ob = uint64_t((ks >> 2) * (Tr::KV_CHUNK / 16) + (ks & 3) * 2);
          if (leader) mma_ss<TF32>(tS[sb], da + oa, db + ob, Tr::IDESC_QK, ks > 0);
        }
      };
      // O of Q tile t += P (score buffer sb) · V(slot)
      auto issue_pv = [&](int t, int slot, bool acc, int sb) {
        const uint32_t vb = aKV + slot * Tr::KV_TILE;
        // 16-bit: V tile [key][d] is an MN-major B operand; step = KSTEP key rows.
        // TF32: V tile was stored transposed ([d][key], K-major); step = 32 bytes.
        const uint64_t db = TF32 ? sw128_desc(vb, 16, 1024) : sw128_desc(vb, Tr::KV_CHUNK, 1024);
#pragma unroll
        for (int ks = 0; ks < Tr::BN / Tr::KSTEP; ++ks) {
          const uint64_t o = TF32 ? uint64_t((ks >> 2) * (D * 8) + (ks & 3) * 2)
                                  : uint64_t(ks * Tr::KSTEP * 8);
          if (leader) mma_ts<TF32>(tO[t], tS[sb] + ks * 8, db + o, Tr::IDESC_PV, (acc || ks > 0) ? 1u : 0u);
        }
      };
      // RSUM: the row sums of P (score buffer sb) += P · ones
      auto issue_rsum = [&](int sb, bool acc) {
        const uint64_t db = sw128_desc(smem_u32(smem + Tr::OFF_ONES), 16, 1024);
#pragma unroll
        for (int ks = 0; ks < Tr::BN / Tr::KSTEP; ++ks)
          if (leader)
            mma_ts<false>(tmem + Tr::COL_R, tS[sb] + ks * 8, db + uint64_t(ks * 2), Tr::IDESC_R,
                          (acc || ks > 0) ? 1u : 0u);
      };
      auto commit = [&](uint64_t* bar) {
        if (leader) tc_commit(bar);
      };
      auto kv_wait = [&](int i) {
        return MBAR_WAIT_WARP(&bars->kv_full[i % Tr::NS], (i / Tr::NS) & 1, abort_flag);
      };

      if constexpr (Tr::SBUF == 2) {
        // One tile, two score buffers: S(0) and S(1) first; then for each j,
        // once the softmax has written P(j) into buffer j % 2, P(j)·V(j) and
        // S(j+2) into the same buffer (in issue order after P·V read P).  The
        // softmax of tile j+1 runs while these products do.  K/V come in the
        // producer's order K0 V0 K1 V1 …: K(j+1) is taken before V(j).
        bool ok = MBAR_WAIT_WARP(&bars->q_full[0], 0, abort_flag) && kv_wait(0);
        tc_fence_after();
        if (ok) issue_qk(0, 0, 0);
        commit(&bars->s_full[0]);
        commit(&bars->kv_empty[0]);  // K_0's slot, once S(0) has read it
        if (ok && n_kv > 1) {
          ok = kv_wait(2);
          tc_fence_after();
          if (ok) issue_qk(0, 2 % Tr::NS, 1);
          commit(&bars->s_full[1]);
          commit(&bars->kv_empty[2 % Tr::NS]);
        }
        for (int j = 0; j < n_kv && ok; ++j) {
          const int b = j & 1, iv = 2 * j + 1, ik = 2 * j + 4;
          const int sv = iv % Tr::NS, sk = ik % Tr::NS;
          ok = kv_wait(iv) && MBAR_WAIT_WARP(&bars->p_full[b], (j >> 1) & 1, abort_flag);
          tc_fence_after();
          if (!ok) break;
          issue_pv(0, sv, j > 0, b);
          if constexpr (RSUM) issue_rsum(b, j > 0);
          commit(&bars->o_full[0]);
          if (j + 1 == n_kv) commit(&bars->o_full[1]);  // the tile's last product, for the epilogue
          commit(&bars->kv_empty[sv]);
          if (j + 2 < n_kv) {
            ok = kv_wait(ik);
            tc_fence_after();
            if (!ok) break;
            issue_qk(0, sk, b);
            commit(&bars->s_full[b]);
            commit(&bars->kv_empty[sk]);
          }
        }
      } else {
      bool ok = MBAR_WAIT_WARP(&bars->q_full[0], 0, abort_flag) && kv_wait(0);
      tc_fence_after();
      if (ok) issue_qk(0, 0, 0);
      commit(&bars->s_full[0]);
      ok = ok && MBAR_WAIT_WARP(&bars->q_full[1], 0, abort_flag);
      tc_fence_after();
      if (ok) issue_qk(1, 0, 1);
      commit(&bars->s_full[1]);
      commit(&bars->kv_empty[0]);
      for (int j = 0; j < n_kv && ok; ++j) {
        const int iv = 2 * j + 1, ik = 2 * j + 2;
        const int sv = iv % Tr::NS, sk = ik % Tr::NS;
        ok = kv_wait(iv);
        ok = ok && MBAR_WAIT_WARP(&bars->p_full[0], j & 1, abort_flag);
        tc_fence_after();
        if (!ok) break;
        issue_pv(0, sv, j > 0, 0);
        commit(&bars->o_full[0]);
        const bool more = j + 1 < n_kv;
        if (more) {
          ok = kv_wait(ik);
          tc_fence_after();
          if (!ok) break;
          issue_qk(0, sk, 0);
          commit(&bars->s_full[0]);
        }
        ok = MBAR_WAIT_WARP(&bars->p_full[1], j & 1, abort_flag);
        tc_fence_after();
        if (!ok) break;
        issue_pv(1, sv, j > 0, 1);
        commit(&bars->o_full[1]);
        commit(&bars->kv_empty[sv]);
        if (more) {
          issue_qk(1, sk, 1);
          commit(&bars->s_full[1]);
          commit(&bars->kv_empty[sk]);
        }
      }
      }
    }
  } else {
    // ------------------------------------------------------------ softmax
    regs_inc<Tr::REGS_SOFTMAX>();
    const int t = warp >> 2;         // which Q tile
    const int quad = warp & 3;       // TMEM lane quadrant of this warp
    const int r = quad * 32 + lane;  // row in the tile = TMEM lane
    const int qi = q_row0 + t * 128 + r;
    const uint32_t lane_off = uint32_t(quad * 32) << 16;
    const uint32_t tS0 = tmem + lane_off + t * 128;  // S of tile t (or score buffer 0)
    const uint32_t tO = tmem + lane_off + Tr::COL_O + t * D;
    const float sl2 = p.scale_log2;
    const int tile_first_row = q_row0 + t * 128;

    float m_ref = -INFINITY;  // reference maximum, scaled log2 units
    float row_sum = 0.f;    // Σ exp2 of the scores: gives the logsumexp L
    float row_sum_p = 0.f;  // Σ of P as rounded for the P·V product: normalises O
    bool ok = true;

    // staged bias tile of this Q tile: chunk c (8 keys) of row rr in the
    // 64-key block c / 8, position (c % 8) ^ (rr % 8) of the row's 128 bytes
    const uint8_t* btile = sBias + t * Tr::BIAS_TILE;
    for (int j = 0; j < n_kv; ++j) {
      // Bias: this row's BN values for the tile's columns, copied out of the
      // staged tile before S arrives (zero past Nk or past Nq), which is then
      // released for the next K/V tile's.
      uint4 bv[SBIAS ? Tr::BN / 8 : 1];
      if constexpr (SBIAS) {
        ok = __all_sync(0xffffffffu, MBAR_WAIT(&bars->bias_full[t], j & 1, abort_flag));
        if (!ok) break;
        if (p.bias_rows > 1) {
#pragma unroll
          for (int v = 0; v < Tr::BN / 8; ++v)
            bv[v] = *reinterpret_cast<const uint4*>(btile + (v >> 3) * (128 * 128) + r * 128 +
                                                   (((v & 7) ^ (r & 7)) << 4));
        } else {  // one row shared by all queries
#pragma unroll
          for (int v = 0; v < Tr::BN / 8; ++v)
            bv[v] = *reinterpret_cast<const uint4*>(btile + (v >> 3) * 1024 + ((v & 7) << 4));
        }
        // The values are still in flight when the tile is released, and the
        // next tile is written by TMA (the async proxy): without a proxy
        // fence that write overtook these reads now and then (seen as rows of
        // L and O that changed from run to run).
        fence_async_smem();
        mbar_arrive(&bars->bias_empty[t]);
      }
      // score buffer of K/V tile j: the tile's own, or j % 2 of two
      const int sb = Tr::SBUF == 2 ? (j & 1) : t;
      const uint32_t sph = Tr::SBUF == 2 ? ((j >> 1) & 1) : (j & 1);
      const uint32_t tS = tS0 + (Tr::SBUF == 2 ? (j & 1) * Tr::BN : 0);
      ok = __all_sync(0xffffffffu, MBAR_WAIT(&bars->s_full[sb], sph, abort_flag));
      tc_fence_after();
      if (!ok) break;
      uint32_t su[Tr::BN / 32][32];
      if constexpr (BIAS && !TF32) {
        // 32 columns at a time, each plus its bias / scale (so the bias
        // registers free up as the scores arrive)
#pragma unroll
        for (int q = 0; q < Tr::BN / 32; ++q) {
          tmem_ld32(tS + 32 * q, su[q]);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const int c = 32 * q + e;
            const uint32_t w = (c & 7) < 2 ? bv[c >> 3].x : (c & 7) < 4 ? bv[c >> 3].y
                             : (c & 7) < 6 ? bv[c >> 3].z : bv[c >> 3].w;
            const float2 b2 = ElemTraits<T>::unpack2(w);
            const float2 r2 = upk2(ffma2(pk2(b2.x, b2.y), pk2(p.bias_mul, p.bias_mul),
                                         pk2(__uint_as_float(su[q][e]), __uint_as_float(su[q][e + 1]))));
            su[q][e] = __float_as_uint(r2.x);
            su[q][e + 1] = __float_as_uint(r2.y);
          }
        }
      } else {
        // All 32-column loads in flight, one wait.
#pragma unroll
        for (int q = 0; q < Tr::BN / 32; ++q) tmem_ld32(tS + 32 * q, su[q]);
        tmem_ld_wait();
      }
      float* s = reinterpret_cast<float*>(&su[0][0]);
      const int k0 = j * Tr::BN;
      const bool tail = k0 + Tr::BN > nk;
      const bool diag = CAUSAL && (k0 + Tr::BN - 1 > tile_first_row + off);
      if (tail || diag) {
        int lim = nk - k0;
        if (CAUSAL) lim = min(lim, qi + off + 1 - k0);
#pragma unroll
        for (int c = 0; c < Tr::BN; ++c)
          if (c >= lim) s[c] = -INFINITY;
      }
      // Row maximum: independent chains of 3-input max, one per 32 columns.
      float mq[Tr::BN / 32];
#pragma unroll
      for (int q = 0; q < Tr::BN / 32; ++q) {
        const float* v = s + 32 * q;
        float a = fmax3(v[0], v[1], v[2]);
#pragma unroll
        for (int i = 3; i < 31; i += 2) a = fmax3(a, v[i], v[i + 1]);
        mq[q] = fmaxf(a, v[31]);
      }
      float mx = fmaxf(mq[0], mq[1]);
#pragma unroll
      for (int q = 2; q < Tr::BN / 32; q += 2) mx = fmax3(mx, mq[q], mq[q + 1]);
      const float m_tile = mx * sl2;
      const bool upd = m_tile > m_ref + kRescaleThreshold;
      float alpha = 1.f;
      if (upd) {
        alpha = ex2(m_ref - m_tile);  // 0 when m_ref is -inf
        row_sum *= alpha;
        row_sum_p *= alpha;
        m_ref = m_tile;
      }
      if (j > 0 && __any_sync(0xffffffffu, upd)) {
        // Correction: O (which holds tiles < j) moves onto the new maximum.
        ok = __all_sync(0xffffffffu, MBAR_WAIT(&bars->o_full[t], (j - 1) & 1, abort_flag));
        tc_fence_after();
        if (!ok) break;
#pragma unroll 1
        for (int c = 0; c < D + (RSUM ? 32 : 0); c += 32) {  // (RSUM: the row sums follow O)
          uint32_t u[32];
          tmem_ld32(tO + c, u);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(__uint_as_float(u[e]) * alpha);
          tmem_st32(tO + c, u);
        }
      }
      const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
      const uint64_t c2 = pk2(sl2, sl2), negm2 = pk2(-m_use, -m_use);
      // Four independent partial sums (one per 32-column quarter) of the
      // unrounded P (for L) and of P as rounded for the P·V product (to
      // normalise O, so that a row's weights add up to one exactly: with a
      // peaky softmax the rounding of the largest P would otherwise show in O).
      uint64_t sum2[4], sum2_p[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) sum2[q] = sum2_p[q] = pk2(0.f, 0.f);
      if constexpr (TF32) {
#pragma unroll
        for (int c = 0; c < Tr::BN; c += 32) {
          uint32_t u[32];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const uint64_t x = ffma2(pk2(s[c + e], s[c + e + 1]), c2, negm2);
            const float2 pe = exp2_pair<false>(x);
            const float r0 = round_tf32(pe.x), r1 = round_tf32(pe.y);
            sum2[c / 32] = fadd2(sum2[c / 32], pk2(pe.x, pe.y));
            sum2_p[c / 32] = fadd2(sum2_p[c / 32], pk2(r0, r1));
            u[e] = __float_as_uint(r0);
            u[e + 1] = __float_as_uint(r1);
          }
          tmem_st32(tS + c, u);
        }
      } else {
#pragma unroll
        for (int c = 0; c < Tr::BN; c += 64) {
          // Dropout: keep bytes of this row's columns k0 + c .. k0 + c + 63
          // (pair e of the half sits in keep[e / 2], bytes 2·(e % 2) and up).
          uint32_t keep[DROP ? 16 : 1];
          if constexpr (DROP) {
#pragma unroll
            for (int g = 0; g < 4; ++g) keep16_row(p.drop, bh, qi, k0 + c + 16 * g, keep + 4 * g);
          }
          uint32_t u[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int q = (c + 2 * e) / 32;
            const uint64_t x = ffma2(pk2(s[c + 2 * e], s[c + 2 * e + 1]), c2, negm2);
            // every emu_period-th pair of exponentials on the FMA pipe
            constexpr int EP = emu_period(Tr::TILES);
            const float2 pe = (EP > 0 && e % EP == EP - 1) ? exp2_pair<true>(x)
                                                                  : exp2_pair<false>(x);
            u[e] = ElemTraits<T>::pack2(pe.x, pe.y);
            sum2[q] = fadd2(sum2[q], pk2(pe.x, pe.y));
            if constexpr (!RSUM) {
              const float2 pr = ElemTraits<T>::unpack2(u[e]);
              sum2_p[q] = fadd2(sum2_p[q], pk2(pr.x, pr.y));
            }
            // the product sees the dropped weights; the sums above do not
            if constexpr (DROP) u[e] &= keep_pair_mask(keep[e / 2], (2 * e) & 3);
          }
          tmem_st32(tS + c / 2, u);
        }
      }
      {
        const float2 a = upk2(fadd2(fadd2(sum2[0], sum2[1]), fadd2(sum2[2], sum2[3])));
        const float2 b = upk2(fadd2(fadd2(sum2_p[0], sum2_p[1]), fadd2(sum2_p[2], sum2_p[3])));
        row_sum += a.x + a.y;
        row_sum_p += b.x + b.y;
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars->p_full[sb]);
    }

    // ------------------------------------------------------------ epilogue
    // the tile's last product (with two score buffers the per-product
    // barrier may be two phases behind here, so the last product has its own)
    if (ok)
      ok = __all_sync(0xffffffffu, Tr::SBUF == 2 ? MBAR_WAIT(&bars->o_full[1], 0, abort_flag)
                                                 : MBAR_WAIT(&bars->o_full[t], (n_kv - 1) & 1, abort_flag));
    tc_fence_after();
    if (ok) {
      if constexpr (RSUM) {  // the row sum of the rounded P, after O in TMEM
        uint32_t u[32];
        tmem_ld32(tO + D, u);
        tmem_ld_wait();
        row_sum_p = __uint_as_float(u[0]);
      }
      // A row whose every score was masked (m_ref still -inf) has O = 0: the
      // FMA-pipe exponentials leave it tiny but nonzero weights otherwise.
      float inv = (row_sum_p > 0.f && m_ref != -INFINITY) ? 1.f / row_sum_p : 0.f;
      if constexpr (DROP) inv *= p.drop.scale;  // kept weights scaled by 256 / T
      const bool live = qi < p.Nq;
      if constexpr (TF32) {
        float* orow = reinterpret_cast<float*>(p.O) + (size_t(bh) * p.Nq + (live ? qi : 0)) * D;
#pragma unroll 1
        for (int c = 0; c < D; c += 32) {
          uint32_t u[32];
          tmem_ld32(tO + c, u);
          tmem_ld_wait();
          if (live) {
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
              float4 v = make_float4(__uint_as_float(u[e]) * inv, __uint_as_float(u[e + 1]) * inv,
                                     __uint_as_float(u[e + 2]) * inv,
                                     __uint_as_float(u[e + 3]) * inv);
              *reinterpret_cast<float4*>(orow + c + e) = v;
            }
          }
        }
      } else {
        // O/ℓ to the tile's Q buffer (every MMA of the tile is complete), in
        // the 128-byte swizzled layout of the loads; TMA writes it below.
        uint8_t* stage = smem + t * Tr::TILE;  // = sQ[t], without indexing the array
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          uint32_t u[32];
          tmem_ld32(tO + c, u);
          tmem_ld_wait();
#pragma unroll
          for (int c8 = 0; c8 < 32; c8 += 8) {
            const int col = c + c8;  // first column of this 16-byte chunk
            const int blk = col / Tr::AW, ch = (col % Tr::AW) / 8;
            uint4 v;
            v.x = ElemTraits<T>::pack2(__uint_as_float(u[c8]) * inv, __uint_as_float(u[c8 + 1]) * inv);
            v.y = ElemTraits<T>::pack2(__uint_as_float(u[c8 + 2]) * inv, __uint_as_float(u[c8 + 3]) * inv);
            v.z = ElemTraits<T>::pack2(__uint_as_float(u[c8 + 4]) * inv, __uint_as_float(u[c8 + 5]) * inv);
            v.w = ElemTraits<T>::pack2(__uint_as_float(u[c8 + 6]) * inv, __uint_as_float(u[c8 + 7]) * inv);
            *reinterpret_cast<uint4*>(stage + blk * Tr::CHUNK + r * 128 + ((ch ^ (r & 7)) << 4)) = v;
          }
        }
        fence_async_smem();
      }
      if (live && FA_INBOUNDS(bh < p.B * p.H && qi < p.Nq))
        p.L[size_t(bh) * p.Nq + qi] =
            row_sum > 0.f ? (m_ref + lg2(row_sum)) * kLn2 : -INFINITY;
    }
    if constexpr (!TF32) {
      // The tile's 128 rows are staged: one thread stores its D/64 column
      // blocks (rows past Nq are clipped by the tensor map) and waits until
      // TMA has read them before the CTA may exit.
      if (named_bar_and(1 + t, 128, ok) && r == 0 &&
          FA_INBOUNDS(bh < p.B * p.H && tile_first_row < p.Nq + 128)) {
#pragma unroll
        for (int blk = 0; blk < Tr::DC; ++blk)
          tma_store_bh(&tmO, GEN && ((p.map4d >> 3) & 1), smem + t * Tr::TILE + blk * Tr::CHUNK, blk * Tr::AW,
                       tile_first_row, bh, p.H);
        bulk_commit();
        bulk_wait_read0();
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == Tr::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, Tr::TMEM_COLS);
  }
}

}  // namespace

template <typename T, int D, bool CAUSAL, bool GEN, bool DROP = false, bool BIAS = false,
          int NT = fwd_tiles(ElemTraits<T>::tf32, D)>
static cudaError_t launch_fwd_t(const FwdLaunch& a) {
  using Tr = FwdTraits<T, D, NT, BIAS && !ElemTraits<T>::tf32>;
  if (a.params.tiles != NT) return cudaErrorInvalidValue;  // the grid was sized for another count
  auto kern = fwd_kernel<T, D, CAUSAL, GEN, DROP, BIAS, NT>;
  cudaError_t e = set_smem_once(reinterpret_cast<const void*>(kern), Tr::SMEM_BYTES, Tr::TIGHT);
  if (e != cudaSuccess) return e;
  // setmaxnreg redistributes the registers the CTA was launched with; refuse
  // to launch if the compiled register count cannot cover the split.
  static int regs_ok = -1;
  if (regs_ok < 0) {
    cudaFuncAttributes attr;
    e = cudaFuncGetAttributes(&attr, reinterpret_cast<const void*>(kern));
    if (e != cudaSuccess) return e;
    regs_ok = attr.numRegs * Tr::THREADS >= 128 * Tr::TILES * Tr::REGS_SOFTMAX + 128 * Tr::REGS_OTHER;
  }
  if (!regs_ok) return cudaErrorInvalidConfiguration;
  dim3 grid(a.params.n_qblocks * a.params.H * a.params.B);
  kern<<<grid, Tr::THREADS, Tr::SMEM_BYTES, a.stream>>>(a.tmQ, a.tmK, a.tmV, a.tmO, a.tmBias, a.params);
  return cudaGetLastError();
}

int fwd_tiles_for(int dtype, int d, int Nq, int Nk, bool causal, bool drop, bool bias) {
  const int dflt = fwd_tiles(dtype == FA_FP32, d);
  if (dtype == FA_FP32) return dflt;
  // d = 64: one tile over 64-key K/V tiles at every length measured (µs,
  // interleaved A/B, both orders, against two tiles): B4 H16 N1024 41.3–42.2
  // vs 43.0–43.1, causal N = 1024 90.3 vs 108.6, N = 2048 142 vs 163,
  // N = 4096 244 vs 270, N = 8192 448–453 vs 485–489, B1 H32 N16384 1671 vs
  // 1813; non-causal N = 4096 450 vs 466, N = 8192 857 vs 888.
  // With a bias: one tile with 64-key bias tiles and four K/V slots, against
  // two tiles with 128-key bias tiles and two K/V slots (forward µs, d = 128
  // bf16, head-shared [1, H, N, N] bias unless noted, interleaved A/B, both
  // orders): non-causal N = 4096 406–432 vs 456–498, N = 8192 834–869 vs
  // 1004–1046, N = 3072 (full bias) 244–261 vs 280–305; causal N = 2048
  // 225–239 vs 259–274, N = 12288 1891–1948 vs 2100–2175, N = 16384
  // 1631–1735 vs 1847–1917.
  if (bias || d != 128 || drop) return 3;
  // 128-key K/V tiles a 128-row query tile sees, on average (bottom-right
  // causal: query tile i sees about i + 1 + (Nk − Nq) / 128 of them).  One Q
  // tile over 64-key K/V tiles with double-buffered scores, against two Q
  // tiles over one K/V stream (forward µs, d = 128 bf16, interleaved A/B,
  // both orders): causal N = 1024 104.6 vs 120.8, N = 2048 160.8 vs 177.6,
  // N = 4096 275–276 vs 281–282, N = 8192 506–510 vs 506–523, N = 16384 ×3
  // even; non-causal N = 2048 289 vs 296, N = 4096 508–509 vs 491–492,
  // N = 8192 972–1050 vs 937–1044.
  const double kv_tiles = (Nk + 127) / 128;
  const double q_tiles = (Nq + 127) / 128;
  const double avg = causal ? std::min(kv_tiles, (q_tiles + 1) / 2 + double(Nk - Nq) / 128) : kv_tiles;
  return avg >= (causal ? 48.0 : 24.0) ? 2 : 3;
}

cudaError_t launch_fwd(int dtype, int d, bool causal, const FwdLaunch& a) {
  const bool gen = a.params.map4d != 0;  // only 4-D tensor maps differ: every access is TMA
  const bool drop = a.params.drop.t4 != 0;
  const bool bias = a.params.bias != nullptr;
  // dropout and bias run in general-layout variants only
#define FA_FWD_CASE(TY, DD)                                                                      \
  {                                                                                              \
    if (bias)                                                                                    \
      return causal ? (drop ? launch_fwd_t<TY, DD, true, true, true, true, 3>(a)                \
                            : launch_fwd_t<TY, DD, true, true, false, true, 3>(a))              \
                    : (drop ? launch_fwd_t<TY, DD, false, true, true, true, 3>(a)               \
                            : launch_fwd_t<TY, DD, false, true, false, true, 3>(a));            \
    if (drop)                                                                                    \
      return causal ? launch_fwd_t<TY, DD, true, true, true>(a)                                  \
                    : launch_fwd_t<TY, DD, false, true, true>(a);                                \
    if (a.params.tiles == 2)                                                                     \
      return causal ? (gen ? launch_fwd_t<TY, DD, true, true, false, false, 2>(a)                \
                           : launch_fwd_t<TY, DD, true, false, false, false, 2>(a))              \
                    : (gen ? launch_fwd_t<TY, DD, false, true, false, false, 2>(a)               \
                           : launch_fwd_t<TY, DD, false, false, false, false, 2>(a));            \
    return causal ? (gen ? launch_fwd_t<TY, DD, true, true>(a) : launch_fwd_t<TY, DD, true, false>(a)) \
                  : (gen ? launch_fwd_t<TY, DD, false, true>(a) : launch_fwd_t<TY, DD, false, false>(a)); \
  }
  if (dtype == FA_BF16) {
    if (d == 64) FA_FWD_CASE(__nv_bfloat16, 64)
    if (d == 128) FA_FWD_CASE(__nv_bfloat16, 128)
  } else if (dtype == FA_FP16) {
    if (d == 64) FA_FWD_CASE(__half, 64)
    if (d == 128) FA_FWD_CASE(__half, 128)
  } else if (dtype == FA_FP32) {  // contiguous, no dropout (the host rejects the rest)
    if (d == 64) return causal ? launch_fwd_t<float, 64, true, false>(a) : launch_fwd_t<float, 64, false, false>(a);
  }
#undef FA_FWD_CASE
  return cudaErrorInvalidValue;
}

FA_ERROR_ACCESSOR(take_error_fwd)


}  // namespace fa
