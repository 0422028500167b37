// Backward attention kernels for sm_100a.
//
// FlashAttention V1/V2 study notes (51CTO):
//   section "算法的改进": the backward needs only the row logsumexp L from
//     the forward; P is rebuilt block by block as exp(scale·S − L) instead of
//     being stored.
//   section "Thread Block Level 并行": the backward is parallel along the K/V
//     sequence ("vertical slices"): one CTA per K/V block, looping over the
//     query blocks, so dK and dV stay on chip and are written once.
//   section "Warp Level 并行": dV = Pᵀ dO, dP = dO Vᵀ, dS = P ∘ (dP − D),
//     dQ = dS K, dK = dSᵀ Q (with the scale on dQ and dK and
//     D = rowsum(dO ∘ O), the exact softmax gradient).  Here dS is kept
//     unscaled in the products and the scale is applied once to the fp32
//     results (dK in its epilogue, dQ in the finalise kernel).
//   section "Sequence Parallel": dQ receives a contribution from every K/V
//     block, so it is reduced across CTAs, either by atomic adds into one
//     buffer or by one buffer per K/V block and a separate reduction kernel.
//     Both are implemented (dq_mode 1 and 2); mode 1 is the default.  The
//     section's compromise, partial buffers shared by groups of K/V blocks
//     with atomic adds inside a group, is mode 3: G fp32 accumulators, K/V
//     block kb reduce-adding into accumulator kb mod G (so K/V blocks of one
//     head that run at the same time add into different buffers).
//
// Kernels: bwd_preprocess (−D = −rowsum(dO ∘ O) and −L·log2e into padded
// buffers, dQ accumulator cleared), bwd_main (below), bwd_dq_finalise
// (sum / convert).
//
// bwd_main, B200 design.  Persistent: one CTA per SM takes work items (a K/V
// block of 128 keys of one head) from a global counter, heaviest first within
// groups of heads, each when its previous item is one step from the end; K is
// double buffered so the next item's K loads while the current item runs, V
// is reloaded once the current item's last dPᵀ has read it.  A step handles
// BM = 128 query rows of the item.
// The two score-like products are computed transposed (keys on TMEM lanes):
// Sᵀ = K Qᵀ and dPᵀ = V dOᵀ, so that the thread owning key row k holds
// Pᵀ[k, :] and dSᵀ[k, :].  Pᵀ goes back to TMEM as the A operand of
// dV += Pᵀ dO; dSᵀ goes to shared memory (one buffer, key rows, 128-byte
// swizzled), where it is the K-major A operand of dK += dSᵀ Q and the
// MN-major operand of the dQ product:
//   d = 128: dQᵀ = Kᵀ dSᵀ (M = d = 128), reduced from registers with one
//            coalesced red.global.add.f32 per warp and query row;
//   d = 64:  dQ = dS K (M = BM = 128), staged in shared memory as two
//            128-byte-swizzled [128 × 32] fp32 halves and reduced with two
//            TMA tensor reduce-adds (cp.reduce.async.bulk.tensor .add.f32).
// Roles (512 threads, setmaxnreg split 136 / 136 / 104 registers):
//   warpgroups 0 and 1: thread = key row; warpgroup c computes P and dS for
//                query columns [64c, 64c + 64) of each step;
//   warpgroup 2: moves dQ of the step from TMEM to the fp32 accumulator,
//                and writes each work item's dK and dV (so the compute
//                warpgroups go straight on to the next item);
//   warp 12: tcgen05.mma issuer, TMEM owner; warp 13: Q / dO producer;
//   warp 14: work-item scheduler and K / V loads.
// TMEM (512 columns): Sᵀ | dPᵀ | dV | dK (128, 128, d, d).  Per step the
// MMA order is dV, next Sᵀ, dQ, dK, next dPᵀ: dQ lands in the dPᵀ columns
// (read by then), warpgroup 2 drains it while dK runs, and the next dPᵀ
// waits until warpgroup 2 has the dQ values in registers.  Q (with −L·log2e
// and −D) has two stages at d = 128 and three at d = 64, dO one.
#define FA_SITE_BASE 20000
#include <algorithm>

#include "common.cuh"
#include "dropout.cuh"
#include "launch.h"

namespace fa {

namespace {

// ------------------------------------------------------------------ bulk copies
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void red_add_f32(float* dst, float v) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(dst), "f"(v) : "memory");
}
constexpr float kLog2e = 1.4426950408889634f;

template <typename T, int D, bool BIAS = false>
struct BwdTraits {
  static constexpr int ES = 2;
  static constexpr int BN = 128;                     // keys per CTA (TMEM lanes)
  static constexpr int BM = 128;                     // query rows per step
  // Compute warpgroups.  Four (32 query columns each, 768 threads, 72
  // registers per compute thread) measured 2 % slower at causal N = 2048
  // d = 128 and no faster at d = 64: the P phase is not shortened by more
  // warps per sub-partition.
  static constexpr int NCW = 2;
  // One pair of exponentials in EXP2_EMU of the P phase on the FMA pipe (0 =
  // none).  Measured (interleaved A/B, periods 2, 4, 8 and none): d = 64 is
  // fastest with 1 in 8 (B4 H16 N1024 backward 84.1 -> 79.2 us), d = 128
  // with none (causal N = 2048: 463.9 us, 466.1 with 1 in 8).
  static constexpr int EXP2_EMU = D == 64 ? 8 : 0;
  static constexpr int CWC = BM / NCW;               // query columns per compute warpgroup
  // d = 128: dQᵀ = Kᵀ dSᵀ with d on the TMEM lanes, so that a warp adds one
  // 128-byte line of the accumulator per query row.  (dQ = dS K with rows on
  // the lanes and four-wide reductions of each thread's row measured 30 %
  // slower: the L2 takes reductions per request, and 16-byte requests
  // scattered over 32 rows are 8 times as many as 128-byte lines.)
  static constexpr bool DQ_T = D == 128;
  static constexpr bool DQ_STAGED = D == 64;           // dQ staged in smem, TMA tensor reduce-add
  static constexpr int KV_TILE = BN * D * ES;        // bytes of the K (or V) tile
  static constexpr int KV_CHUNK = BN * 128;          // one 128-byte column block of it
  static constexpr int Q_TILE = BM * D * ES;         // bytes of a Q (or dO) tile
  static constexpr int Q_CHUNK = BM * 128;
  static constexpr int DS_TILE = BN * BM * ES;       // dSᵀ, rows = keys, q contiguous
  // dQ staging (d = 64 only): the whole [BM × 64] fp32 tile (32 KB) goes to
  // shared memory as two swizzled halves and out with two tensor reduce-adds;
  // d = 128 reduces dQᵀ from registers and needs no staging.
  static constexpr int DQ_STAGE = DQ_STAGED ? BM * D * 4 : 0;
  // shared-memory offsets (all 1024-aligned).  K is double buffered (the
  // next work item's K loads while this item runs); Q has QS stages (the
  // next step's Sᵀ needs one while this step's dK still reads the current
  // one); V and dO are single buffered.
  // The bias variants stage each step's [BM queries × BN keys] bias tile in
  // shared memory (one TMA load).  At d = 128 its 32 KB take the second K
  // buffer (K is then single buffered); at d = 64 there is room after the rest.
  static constexpr int BIAS_TILE = BIAS ? BM * BN * ES : 0;
  static constexpr bool K_SINGLE = BIAS && D == 128;
  static constexpr int KBUF = K_SINGLE ? 1 : 2;      // K buffers
  // Q stages: three at d = 64 (room to spare), so a stage is reloaded two
  // steps after its dK product released it; two at d = 128.
  static constexpr int QS = D == 64 ? 3 : 2;
  static constexpr int OFF_K = 0;                    // 2 buffers
  static constexpr int OFF_V = OFF_K + 2 * KV_TILE;
  static constexpr int OFF_Q = OFF_V + KV_TILE;      // QS stages
  static constexpr int OFF_DO = OFF_Q + QS * Q_TILE;
  static constexpr int OFF_DS = OFF_DO + Q_TILE;
  static constexpr int OFF_DQ = OFF_DS + DS_TILE;
  static constexpr int OFF_LD = OFF_DQ + DQ_STAGE;   // L·log2e and D per Q stage
  static constexpr int OFF_BAR = OFF_LD + QS * 2 * BM * 4;
  static constexpr int OFF_BIAS = K_SINGLE ? OFF_K + KV_TILE : (OFF_BAR + 512 + 1023) / 1024 * 1024;
  // the base is checked to be 1024-aligned
  static constexpr int SMEM_BYTES = (BIAS && !K_SINGLE) ? OFF_BIAS + BIAS_TILE : OFF_BAR + 512;
  // TMEM columns: Sᵀ | dPᵀ (dQ of the step lands here after dK read dSᵀ) | dV | dK
  static constexpr int COL_S = 0;
  static constexpr int COL_DP = BM;
  static constexpr int COL_DV = 2 * BM;
  static constexpr int COL_DK = COL_DV + D;
  static_assert(COL_DK + D <= 512, "TMEM budget");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared-memory budget");
  // Warps: the compute warpgroups, then the dQ warpgroup, then MMA issue,
  // Q / dO producer, scheduler + K / V loads and one idle warp.
  static constexpr int THREADS = 128 * (NCW + 2);
  static constexpr int WARP_DQ0 = 4 * NCW;
  static constexpr int WARP_MMA = WARP_DQ0 + 4;
  static constexpr int WARP_PROD = WARP_MMA + 1;
  static constexpr int WARP_SCHED = WARP_MMA + 2;
  // setmaxnreg split; 128·(NCW·REGS_COMPUTE + REGS_DQ + REGS_OTHER) must not
  // exceed the registers the CTA is launched with (THREADS × LAUNCH_REGS).
  static constexpr int LAUNCH_REGS = (65536 / THREADS) / 8 * 8;
  static constexpr int REGS_COMPUTE = 136;
  static constexpr int REGS_DQ = 136;
  static constexpr int REGS_OTHER = 104;
  static_assert(128 * (NCW * REGS_COMPUTE + REGS_DQ + REGS_OTHER) <= THREADS * LAUNCH_REGS,
                "register split");
  static constexpr uint32_t F = ElemTraits<T>::fmt;
  static constexpr uint32_t IDESC_ST = make_idesc(F, 128, BM, 0, 0);   // Sᵀ, dPᵀ
  static constexpr uint32_t IDESC_GRAD = make_idesc(F, 128, D, 0, 1);  // dV (A in TMEM), dK (A = dSᵀ K-major)
  static constexpr uint32_t IDESC_DQ = make_idesc(F, 128, DQ_T ? BM : D, 1, 1);
};


// The kernel is persistent: a CTA takes work items (K/V block, head) in turn
// and numbers its steps across items (g).  The per-step barriers complete
// once per step except q_full / q_empty (one per Q stage, every QS-th
// step); v_full, v_free, dkv_done and dkv_free complete once per work item,
// k_full[b] / k_free[b] once per item that uses K buffer b (every other
// item), item_full[s] once per item published in ring slot s.  A producer
// of any of them cannot run two phases ahead of its waiter (each signal
// needs the waiter's previous phase to have been seen), so parity waits are
// unambiguous.
struct BwdBarriers {
  uint64_t k_full[2];
  uint64_t k_free[2];
  uint64_t v_full;
  uint64_t v_free;
  uint64_t q_full[3];     // Q stage s (of QS) holds its step's Q, −L·log2e and −D
  uint64_t q_empty[3];
  uint64_t do_full;
  uint64_t do_empty;
  uint64_t s_full;
  uint64_t dp_full;
  uint64_t p_ready;
  uint64_t ds_ready;
  uint64_t dq_full;
  uint64_t dq_empty;
  uint64_t ds_free;
  uint64_t dkv_done;      // the item's last dK / dV products are complete
  uint64_t dkv_free;      // the epilogue has read the item's dK / dV from TMEM
  uint64_t bias_full;     // BIAS: the step's bias tile has landed (once per step)
  uint64_t bias_empty;    // BIAS: the compute warpgroups have copied it out
  uint64_t item_full[4];  // the scheduler published work item `it` in slot it % 4
  int item_idx[4];        // its index in the grouped order, or -1 after the last
  uint32_t tmem_base;
  int abort_flag;
};

// Query-tile range of K/V block `kb`: with bottom-right causal alignment the
// first query that sees key kb*BN is kb*BN - (Nk - Nq).
template <int BM, bool CAUSAL>
__device__ __forceinline__ void q_tile_range(int kb, int Nq, int Nk, int& i0, int& n) {
  int first = 0;
  if (CAUSAL) first = max(0, kb * 128 - (Nk - Nq));
  i0 = first / BM;
  const int nt = (Nq + BM - 1) / BM;
  n = max(0, nt - i0);
}

// The fp32 dQ buffer is S slabs of [B·H, Nq_pad, d]: one accumulator
// (mode 1), one partial per K/V block (mode 2), or dq_groups accumulators
// (mode 3).  K/V block kb writes slab dq_slab(p, kb).
[[maybe_unused]] __device__ __forceinline__ int dq_slabs(const BwdParams& p) {
  return p.dq_mode == 2 ? p.n_kblocks : p.dq_mode == 3 ? p.dq_groups : 1;
}
__device__ __forceinline__ int dq_slab(const BwdParams& p, int kb) {
  return p.dq_mode == 2 ? kb : p.dq_mode == 3 ? kb % p.dq_groups : 0;
}

// GEN: some tensor has a general layout (4-D tensor maps or plain strided
// accesses); otherwise every access uses the contiguous [B·H, N, d] form.
// DROP: the forward dropped weights; the compute warps redraw its keep mask.
// BIAS: the forward added a bias to the scaled scores; P is rebuilt with it.
template <typename T, int D, bool CAUSAL, bool GEN, bool DROP, bool BIAS>
__global__ void __launch_bounds__(BwdTraits<T, D, BIAS>::THREADS, 1)
    bwd_main_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                    const __grid_constant__ CUtensorMap tmdQ,
                    const __grid_constant__ CUtensorMap tmBias, BwdParams p) {
  using Tr = BwdTraits<T, D, BIAS>;
  constexpr int BM = Tr::BM;
  constexpr int CWC = Tr::CWC;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // The layout uses all but a few hundred bytes of shared memory, with no
  // slack to align the base: it must already start on a 1024-byte boundary
  // (the 128-byte swizzle atoms and the MMA descriptors assume it).
  if ((smem_u32(smem_raw) & 1023u) != 0) {
    if (threadIdx.x == 0) atomicOr(&g_fa_error, kErrLayout);
    return;
  }
  uint8_t* smem = smem_raw;
  BwdBarriers* bars = reinterpret_cast<BwdBarriers*>(smem + Tr::OFF_BAR);
  volatile int* abort_flag = &bars->abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int off = p.Nk - p.Nq;
  const int n_items = p.n_kblocks * p.B * p.H;

  // Work item j: (K/V block kb, head bh) in the grouped order (causal: the
  // first key blocks are seen by the most query tiles) and its query-tile
  // range [i0, i0 + n_q).  A block wholly past the batch element's key
  // padding length has no steps (its dK and dV rows are written as zeros).
  auto item = [&](int j, int& bh, int& kb, int& i0, int& n_q) {
    grouped_order(j, p.B * p.H, p.n_kblocks, p.head_group, bh, kb);
    q_tile_range<BM, CAUSAL>(kb, p.Nq, p.Nk, i0, n_q);
    if (p.kv_len && kb * Tr::BN >= keys_of(p.kv_len, bh, p.H, p.Nk)) n_q = 0;
  };
  // The it-th work item of this CTA, as the scheduler published it in the
  // item ring; false after the last one (or on abort).
  auto take_item = [&](int it, int& j) -> bool {
    if (!MBAR_WAIT(&bars->item_full[it & 3], (it >> 2) & 1, abort_flag)) return false;
    j = *reinterpret_cast<volatile int*>(&bars->item_idx[it & 3]);
    return j >= 0;
  };

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->k_full[b], 1);
      mbar_init(&bars->k_free[b], 1);
    }
    for (int b = 0; b < 3; ++b) {
      mbar_init(&bars->q_full[b], 1);
      mbar_init(&bars->q_empty[b], 1);
    }
    mbar_init(&bars->v_full, 1);
    mbar_init(&bars->v_free, 1);
    mbar_init(&bars->do_full, 1);
    mbar_init(&bars->do_empty, 1);
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->dp_full, 1);
    mbar_init(&bars->p_ready, 128 * Tr::NCW);
    mbar_init(&bars->ds_ready, 128 * Tr::NCW);
    mbar_init(&bars->dq_full, 1);
    mbar_init(&bars->dq_empty, 128);
    mbar_init(&bars->ds_free, 1);
    mbar_init(&bars->dkv_done, 1);
    mbar_init(&bars->dkv_free, 128);
    mbar_init(&bars->bias_full, 1);
    mbar_init(&bars->bias_empty, 128 * Tr::NCW);
    for (int k = 0; k < 4; ++k) mbar_init(&bars->item_full[k], 1);
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == Tr::WARP_MMA) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == Tr::WARP_PROD && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmdO);
    if constexpr (Tr::DQ_STAGED) tma_prefetch_desc(&tmdQ);
    if constexpr (BIAS) tma_prefetch_desc(&tmBias);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  uint8_t* sK0 = smem + Tr::OFF_K;  // two K buffers, KV_TILE apart
  uint8_t* sV = smem + Tr::OFF_V;
  uint8_t* sQ = smem + Tr::OFF_Q;
  uint8_t* sdO = smem + Tr::OFF_DO;
  uint8_t* sdS = smem + Tr::OFF_DS;
  uint8_t* sdQ = smem + Tr::OFF_DQ;  // d = 64: two [128 rows × 128 B] swizzled halves
  float* sLD = reinterpret_cast<float*>(smem + Tr::OFF_LD);  // [stage][2][BM]
  uint8_t* sBias = smem + Tr::OFF_BIAS;  // BIAS: [BM queries][BN keys] of the input type

  // Register split (the CTA launches with LAUNCH_REGS per thread): the
  // compute and dQ warpgroups hold a step's TMEM columns in registers, the
  // last warpgroup (MMA issue, loads, scheduling) needs few.  Each role sets
  // its own count.
  if (warp >= Tr::WARP_SCHED) {
    regs_set<Tr::REGS_OTHER, Tr::LAUNCH_REGS>();
    if (warp == Tr::WARP_SCHED && lane == 0) {
      // ---------------------------------------------------- scheduler + K/V loads
      // Work items are handed out dynamically in the grouped order: the first
      // wave by CTA index, the rest from a global counter, each taken when
      // the previous item has issued its last dPᵀ (about one step before it
      // ends), so no CTA holds a claim on work it cannot start soon.  The
      // item's K goes to buffer it % 2 (the previous item still reads the
      // other; the bias variants at d = 128 have one K buffer, which the
      // previous item's last dQ product released), its V to the one V buffer,
      // which that last dPᵀ released.
      bool ok = true;
      int it = 0;
      for (;; ++it) {
        int j = blockIdx.x;
        if (it >= 1) {
          ok = ok && MBAR_WAIT(&bars->v_free, (it - 1) & 1, abort_flag);
          j = int(gridDim.x) + atomicAdd(p.item_ctr, 1);
        }
        const bool last = !ok || j >= n_items;
        bars->item_idx[it & 3] = last ? -1 : j;
        mbar_arrive(&bars->item_full[it & 3]);  // release: the index is visible to the waiters
        if (last) break;
        int bh, kb, i0, n_q;
        item(j, bh, kb, i0, n_q);
        const int key0 = kb * Tr::BN, b = it % Tr::KBUF;
        if (it >= Tr::KBUF && !MBAR_WAIT(&bars->k_free[b], ((it / Tr::KBUF) - 1) & 1, abort_flag)) {
          ok = false;
          continue;
        }
        if (!FA_INBOUNDS(bh < p.B * p.H && kb < p.n_kblocks && key0 < p.Nk)) {
          ok = false;
          continue;
        }
        mbar_arrive_expect_tx(&bars->k_full[b], Tr::KV_TILE);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_bh(sK0 + b * Tr::KV_TILE + c * Tr::KV_CHUNK, &tmK, GEN && ((p.map4d >> 1) & 1),
                      &bars->k_full[b], c * 64, key0, bh, p.H);
        mbar_arrive_expect_tx(&bars->v_full, Tr::KV_TILE);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_bh(sV + c * Tr::KV_CHUNK, &tmV, GEN && ((p.map4d >> 2) & 1), &bars->v_full, c * 64, key0, bh,
                      p.H);
      }
      // Drain every issued load before the CTA may exit (it items loaded).
      for (int k = max(0, it - Tr::KBUF); k < it; ++k)
        MBAR_WAIT(&bars->k_full[k % Tr::KBUF], (k / Tr::KBUF) & 1, abort_flag);
      if (it > 0) MBAR_WAIT(&bars->v_full, (it - 1) & 1, abort_flag);
    }
  } else if (warp == Tr::WARP_PROD) {
    // ------------------------------------------------------------ Q / dO producer
    regs_set<Tr::REGS_OTHER, Tr::LAUNCH_REGS>();
    if (lane == 0) {
      bool ok = true;
      int g = 0, it = 0;
      for (int j; ok && take_item(it, j); ++it) {
        int bh, kb, i0, n_q;
        item(j, bh, kb, i0, n_q);
        for (int i = 0; i < n_q && ok; ++i) {
          const int gs = g + i, s = gs % Tr::QS;
          const int q0 = (i0 + i) * BM;
          if constexpr (BIAS) {
            // the step's [BM queries × BN keys] bias tile (zero past Nq and
            // Nk), once the compute warpgroups have copied out step gs-1's
            if (gs >= 1 && !MBAR_WAIT(&bars->bias_empty, (gs - 1) & 1, abort_flag)) {
              ok = false;
              break;
            }
            if (!FA_INBOUNDS(kb * Tr::BN < p.Nk && q0 < p.Nq && bh < p.B * p.H)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&bars->bias_full, p.bias_rows * Tr::BN * Tr::ES);
            tma_load_4d(sBias, &tmBias, &bars->bias_full, kb * Tr::BN, p.bias_rows > 1 ? q0 : 0,
                        (bh % p.H) % p.bias_H, (bh / p.H) % p.bias_B);
          }
          // Q (with −L·log2e and −D) into stage s, once step gs-2 has released it
          if (gs >= Tr::QS && !MBAR_WAIT(&bars->q_empty[s], ((gs / Tr::QS) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          uint64_t* bar = &bars->q_full[s];
          if (!FA_INBOUNDS(bh < p.B * p.H && q0 + BM <= p.Nq_pad && q0 < p.Nq)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar, Tr::Q_TILE + 2 * BM * 4);
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            tma_load_bh(sQ + s * Tr::Q_TILE + c * Tr::Q_CHUNK, &tmQ, GEN && (p.map4d & 1), bar, c * 64, q0, bh,
                        p.H);
          const size_t row = size_t(bh) * p.Nq_pad + q0;
          bulk_load(sLD + (s * 2 + 0) * BM, p.neg_Lsc + row, BM * 4, bar);
          bulk_load(sLD + (s * 2 + 1) * BM, p.neg_D + row, BM * 4, bar);
          // dO into its single buffer, once step gs-1's dV product has read it
          if (gs >= 1 && !MBAR_WAIT(&bars->do_empty, (gs - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bars->do_full, Tr::Q_TILE);
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            tma_load_bh(sdO + c * Tr::Q_CHUNK, &tmdO, GEN && ((p.map4d >> 4) & 1), &bars->do_full, c * 64, q0, bh,
                        p.H);
        }
        g += n_q;
      }
      // Drain every issued load before the CTA may exit.
      for (int gs = max(0, g - Tr::QS); gs < g; ++gs)
        MBAR_WAIT(&bars->q_full[gs % Tr::QS], (gs / Tr::QS) & 1, abort_flag);
      if (g > 0) MBAR_WAIT(&bars->do_full, (g - 1) & 1, abort_flag);
      if (BIAS && g > 0) MBAR_WAIT(&bars->bias_full, (g - 1) & 1, abort_flag);
    }
  } else if (warp == Tr::WARP_MMA) {
    // ------------------------------------------------------------ MMA issuer
    regs_set<Tr::REGS_OTHER, Tr::LAUNCH_REGS>();
    // The whole warp runs the loop (warp-uniform waits and descriptor
    // arithmetic); the elected lane issues the MMAs and commits.
    {
      const bool leader = elect_one();
      auto commit = [&](uint64_t* bar) {
        if (leader) tc_commit(bar);
      };
      const uint32_t aK0 = smem_u32(sK0), aV = smem_u32(sV), aQ = smem_u32(sQ), adO = smem_u32(sdO);
      const uint32_t adS = smem_u32(sdS);
      const uint32_t colS = tmem + Tr::COL_S, colDP = tmem + Tr::COL_DP;
      const uint32_t colDV = tmem + Tr::COL_DV, colDK = tmem + Tr::COL_DK;
      // Operand descriptors are built once; inside the unrolled loops each
      // MMA only adds a compile-time offset (16-byte units).
      const uint64_t dK_k0 = sw128_desc(aK0, 16, 1024), dV_k = sw128_desc(aV, 16, 1024);
      const uint64_t dK_mn0 = sw128_desc(aK0, Tr::KV_CHUNK, 1024);
      const uint64_t dQ_k0 = sw128_desc(aQ, 16, 1024), dO_k = sw128_desc(adO, 16, 1024);
      const uint64_t dQ_mn0 = sw128_desc(aQ, Tr::Q_CHUNK, 1024);
      const uint64_t dO_mn = sw128_desc(adO, Tr::Q_CHUNK, 1024);
      const uint64_t dS_mn = sw128_desc(adS, Tr::BN * 128, 1024);
      const uint64_t dS_k = sw128_desc(adS, 16, 1024);
      auto stg = [](uint64_t d0, int s) { return d0 + uint64_t(s) * uint64_t(Tr::Q_TILE >> 4); };
      auto kbuf = [](uint64_t d0, int b) { return d0 + uint64_t(b) * uint64_t(Tr::KV_TILE >> 4); };

      // Sᵀ (or dPᵀ) = X[128 keys × D] · Y[BM × D]ᵀ, both K-major.
      auto mma_st = [&](uint32_t dcol, uint64_t dx, uint64_t dy) {
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t oa = uint64_t((ks >> 2) * (Tr::KV_CHUNK / 16) + (ks & 3) * 2);
          const uint64_t ob = uint64_t((ks >> 2) * (Tr::Q_CHUNK / 16) + (ks & 3) * 2);
          if (leader) mma_ss<false>(dcol, dx + oa, dy + ob, Tr::IDESC_ST, ks > 0);
        }
      };
      // dV [128 × D] += Pᵀ[128 × BM] (TMEM) · dO[BM × D] (MN-major).  Pᵀ
      // (pairs of the input type) was written by the two compute warpgroups,
      // each into the first half of the columns it had read, so k-step ks
      // sits at column (ks / kPerWg)·CWC + (ks % kPerWg)·8.
      auto mma_dv = [&](bool acc) {
        constexpr int kPerWg = CWC / 16;
#pragma unroll
        for (int ks = 0; ks < BM / 16; ++ks)
          if (leader) mma_ts<false>(colDV, colS + (ks / kPerWg) * CWC + (ks % kPerWg) * 8,
                        dO_mn + uint64_t(ks * 128), Tr::IDESC_GRAD, (acc || ks > 0) ? 1u : 0u);
      };
      // dK [128 × D] += dSᵀ [128 keys × BM] (shared memory, K-major: key rows of
      // BM query values in 64-column blocks) · Q [BM × D] (MN-major).
      auto mma_dk = [&](uint64_t dy, bool acc) {
#pragma unroll
        for (int ks = 0; ks < BM / 16; ++ks) {
          const uint64_t oa = uint64_t((ks >> 2) * (Tr::BN * 128 / 16) + (ks & 3) * 2);
          if (leader) mma_ss<false>(colDK, dS_k + oa, dy + uint64_t(ks * 128), Tr::IDESC_GRAD,
                        (acc || ks > 0) ? 1u : 0u);
        }
      };
      // dQᵀ [D × BM] = Kᵀ · dSᵀ  (d = 128), or dQ [BM × D] = dS · K (d = 64);
      // both operands MN-major, K dimension = the 128 keys.
      auto mma_dq = [&](uint64_t dkmn) {
#pragma unroll
        for (int ks = 0; ks < Tr::BN / 16; ++ks) {
          const uint64_t o = uint64_t(ks * 128);
          if (leader) {
            if constexpr (Tr::DQ_T)
              mma_ss<false>(colDP, dkmn + o, dS_mn + o, Tr::IDESC_DQ, ks > 0);
            else
              mma_ss<false>(colDP, dS_mn + o, dkmn + o, Tr::IDESC_DQ, ks > 0);
          }
        }
      };

      bool ok = true;
      int g = 0, it = 0;
      for (int j; ok && __all_sync(0xffffffffu, take_item(it, j)); ++it) {
        int bh, kb, i0, n_q;
        item(j, bh, kb, i0, n_q);
        (void)bh;
        (void)i0;
        int b = it % Tr::KBUF;
        // With one K buffer the index is the constant 0, and the compiler then
        // keeps every product's descriptors live across items (spilling);
        // hidden from it, they are formed per item as with two buffers.
        if constexpr (Tr::KBUF == 1) asm volatile("" : "+r"(b));
        const uint64_t dK_k = kbuf(dK_k0, b), dK_mn = kbuf(dK_mn0, b);
        ok = MBAR_WAIT_WARP(&bars->k_full[b], (it / Tr::KBUF) & 1, abort_flag);
        if (ok && n_q > 0)
          ok = MBAR_WAIT_WARP(&bars->q_full[g % Tr::QS], (g / Tr::QS) & 1, abort_flag) &&
               MBAR_WAIT_WARP(&bars->do_full, g & 1, abort_flag);
        tc_fence_after();
        if (!ok) break;
        if (n_q > 0) {
          mma_st(colS, dK_k, stg(dQ_k0, g % Tr::QS));
          commit(&bars->s_full);
          // dPᵀ(0) needs V, and the previous item's last dQ out of the dPᵀ columns
          ok = MBAR_WAIT_WARP(&bars->v_full, it & 1, abort_flag);
          if (ok && g > 0) ok = MBAR_WAIT_WARP(&bars->dq_empty, (g - 1) & 1, abort_flag);
          tc_fence_after();
          if (!ok) break;
          mma_st(colDP, dV_k, dO_k);
          commit(&bars->dp_full);
          if (n_q == 1) commit(&bars->v_free);  // the item's last dPᵀ
        } else {
          ok = MBAR_WAIT_WARP(&bars->v_full, it & 1, abort_flag);
          tc_fence_after();
          if (!ok) break;
          commit(&bars->v_free);
        }
        // dV and dK restart from zero: the previous item's epilogue must
        // have read them.
        if (it > 0) {
          ok = MBAR_WAIT_WARP(&bars->dkv_free, (it - 1) & 1, abort_flag);
          tc_fence_after();
          if (!ok) break;
        }
        // Per step: dV (needs Pᵀ), the next Sᵀ into the same columns (in
        // issue order after dV read them), dQ into the dPᵀ columns (read by
        // the compute warpgroups by then), dK, and last the next dPᵀ, once
        // warpgroup 2 has drained dQ from those columns.
        for (int i = 0; i < n_q; ++i) {
          const int gs = g + i, s = gs % Tr::QS, sn = (gs + 1) % Tr::QS;
          const bool more = i + 1 < n_q;
          ok = MBAR_WAIT_WARP(&bars->p_ready, gs & 1, abort_flag);
          tc_fence_after();
          if (!ok) break;
          mma_dv(i > 0);
          commit(&bars->do_empty);
          if (more) {
            ok = MBAR_WAIT_WARP(&bars->q_full[sn], ((gs + 1) / Tr::QS) & 1, abort_flag);
            tc_fence_after();
            if (!ok) break;
            mma_st(colS, dK_k, stg(dQ_k0, sn));
            commit(&bars->s_full);
          }
          ok = MBAR_WAIT_WARP(&bars->ds_ready, gs & 1, abort_flag);
          tc_fence_after();
          if (!ok) break;
          // dQ first, so warpgroup 2 drains it while the tensor core runs dK.
          mma_dq(dK_mn);
          commit(&bars->dq_full);
          if (!more) commit(&bars->k_free[b]);  // the item's last product reading K
          mma_dk(stg(dQ_mn0, s), i > 0);
          commit(&bars->q_empty[s]);
          commit(&bars->ds_free);
          if (more) {
            ok = MBAR_WAIT_WARP(&bars->dq_empty, gs & 1, abort_flag) &&
                 MBAR_WAIT_WARP(&bars->do_full, (gs + 1) & 1, abort_flag);
            tc_fence_after();
            if (!ok) break;
            mma_st(colDP, dV_k, dO_k);
            commit(&bars->dp_full);
            if (i + 2 == n_q) commit(&bars->v_free);  // the item's last dPᵀ
          }
        }
        if (!ok) break;
        if (n_q == 0) commit(&bars->k_free[b]);
        commit(&bars->dkv_done);  // after the item's last dK (or at once if it has no steps)
        g += n_q;
      }
    }
  } else if (warp < Tr::WARP_DQ0) {
    // ------------------------------------------------------------ P / dS (thread = key)
    // NCW warpgroups; warpgroup cw handles query columns [cw·CWC, (cw+1)·CWC)
    // of each step for all 128 key rows.
    regs_set<Tr::REGS_COMPUTE, Tr::LAUNCH_REGS>();
    const int cw = warp >> 2;
    const int quad = warp & 3;
    const int kr = quad * 32 + lane;  // key row in the tile = TMEM lane
    const uint32_t lane_off = uint32_t(quad * 32) << 16;
    const float sl2 = p.scale_log2;
    const uint32_t tS = tmem + lane_off + Tr::COL_S;
    const uint32_t tDP = tmem + lane_off + Tr::COL_DP;
    bool ok = true;
    int g = 0, it = 0;
    for (int j; ok && __all_sync(0xffffffffu, take_item(it, j)); ++it) {
      int bh, kb, i0, n_q;
      item(j, bh, kb, i0, n_q);
      const int key0 = kb * Tr::BN;
      const int key = key0 + kr;
      const bool key_live = key < keys_of(p.kv_len, bh, p.H, p.Nk);
      const int qmin = key - off;  // first query row that sees this key
      for (int i = 0; i < n_q; ++i) {
        const int gs = g + i, s = gs % Tr::QS;
        const int q0 = (i0 + i) * BM + cw * CWC;  // first query column of this warpgroup
        // −L·log2e and −D of this warpgroup's query columns (16-byte aligned)
        const float4* sL4 = reinterpret_cast<const float4*>(sLD + (s * 2 + 0) * BM + cw * CWC);
        const float4* sD4 = reinterpret_cast<const float4*>(sLD + (s * 2 + 1) * BM + cw * CWC);
        // Dropout: keep bytes of this key for query columns q0 .. q0 + CWC − 1
        // (column pair q, q + 1 in keep[q / 4], bytes q % 4 and up), drawn
        // before S arrives.
        uint32_t keep[DROP ? CWC / 4 : 1];
        if constexpr (DROP) {
#pragma unroll
          for (int g16 = 0; g16 < CWC / 16; ++g16) keep16_col(p.drop, bh, key, q0 + 16 * g16, keep + 4 * g16);
        }
        // Bias: this key's values for the CWC query columns, as packed pairs
        // (zero past Nq or past Nk: the tile's load fills them with zeros).
        uint32_t bpk[BIAS ? CWC / 2 : 1];
        if constexpr (BIAS) {
          // out of the step's staged tile (row = query, BN keys contiguous;
          // a warp's lanes read 64 consecutive bytes of a row), then the tile
          // is released so the producer can load the next step's
          ok = __all_sync(0xffffffffu, MBAR_WAIT(&bars->bias_full, gs & 1, abort_flag));
          if (!ok) break;
          const uint16_t* bt = reinterpret_cast<const uint16_t*>(sBias) + kr;
          if (p.bias_rows > 1) {
            bt += cw * CWC * Tr::BN;
#pragma unroll
            for (int c = 0; c < CWC; c += 2)
              bpk[c >> 1] = uint32_t(bt[c * Tr::BN]) | (uint32_t(bt[(c + 1) * Tr::BN]) << 16);
          } else {  // one row shared by all queries
            const uint32_t v = bt[0];
#pragma unroll
            for (int c = 0; c < CWC; c += 2) bpk[c >> 1] = v | (v << 16);
          }
          // (the next tile is written by TMA, another proxy: a proxy fence
          // orders these reads before that write, as in the forward)
          fence_async_smem();
          mbar_arrive(&bars->bias_empty);
        }
        // ---- P = exp2(S·c − L·log2e), causal / ragged masking
        ok = __all_sync(0xffffffffu, MBAR_WAIT(&bars->s_full, gs & 1, abort_flag));
        tc_fence_after();
        if (!ok) break;
        const bool need_mask = !key_live || (CAUSAL && (key0 + Tr::BN - 1 > q0 + off));
        uint32_t Pk[CWC / 2];  // P as packed pairs of the input type
        const uint64_t c2 = pk2(sl2, sl2);
        // Load the warpgroup's CWC columns at once (one TMEM round trip), then
        // 32 at a time: exponentiate, pack to pairs of the input type, store Pᵀ
        // back to TMEM into the columns this warpgroup has read (the other
        // warpgroup may still be reading its own half).  The packed P stays in
        // registers for dS, so dS uses the same rounded P as the dV product.
        uint32_t u[CWC];
#pragma unroll
        for (int c = 0; c < CWC; c += 32)
          tmem_ld32(tS + cw * CWC + c, *reinterpret_cast<uint32_t(*)[32]>(u + c));
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < CWC; c += 32) {
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            const float4 nl = sL4[(c + e) >> 2];
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              const int q = c + e + 2 * h2;
              uint64_t nlq = h2 ? pk2(nl.z, nl.w) : pk2(nl.x, nl.y);
              if constexpr (BIAS) {  // − L·log2e + bias·log2e
                const float2 b2 = ElemTraits<T>::unpack2(bpk[q >> 1]);
                nlq = ffma2(pk2(b2.x, b2.y), pk2(p.bias_l2, p.bias_l2), nlq);
              }
              const float2 x = upk2(ffma2(pk2(__uint_as_float(u[q]), __uint_as_float(u[q + 1])), c2, nlq));
              float p0, p1;
              if (Tr::EXP2_EMU > 0 && (q >> 1) % (Tr::EXP2_EMU > 0 ? Tr::EXP2_EMU : 1) == Tr::EXP2_EMU - 1) {
                const float2 pe = exp2_pair_fma<true>(x);  // exactly 0 for masked entries
                p0 = pe.x;
                p1 = pe.y;
              } else {
                p0 = ex2(x.x);
                p1 = ex2(x.y);
              }
              if (need_mask) {
                if (!key_live || (CAUSAL && q0 + q < qmin)) p0 = 0.f;
                if (!key_live || (CAUSAL && q0 + q + 1 < qmin)) p1 = 0.f;
              }
              Pk[q >> 1] = ElemTraits<T>::pack2(p0, p1);
            }
          }
          if constexpr (DROP) {
            // the dV product sees the dropped weights (its 256/T factor is
            // applied in the epilogue); dS below needs the undropped P
            uint32_t pm[16];
#pragma unroll
            for (int w = 0; w < 16; ++w) {
              const int pi = (c >> 1) + w;  // pair index: columns 2·pi, 2·pi + 1
              pm[w] = Pk[pi] & keep_pair_mask(keep[pi >> 1], (2 * pi) & 3);
            }
            tmem_st16(tS + cw * CWC + c / 2, pm);
          } else {
            tmem_st16(tS + cw * CWC + c / 2, Pk + (c >> 1));
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bars->p_ready);

        // ---- dS = P ∘ (dP − D), to shared memory (row = key, BM query
        // values contiguous, 128-byte swizzled, 64 values per column block):
        // the A operand of dK += dSᵀ Q and an operand of dQ.  The softmax
        // scale is left out here (one multiply per element fewer on the
        // busiest warps) and applied to the fp32 dK and dQ sums.
        ok = __all_sync(0xffffffffu, MBAR_WAIT(&bars->dp_full, gs & 1, abort_flag));
        if (ok && gs >= 1)
          ok = __all_sync(0xffffffffu, MBAR_WAIT(&bars->ds_free, (gs - 1) & 1, abort_flag));
        tc_fence_after();
        if (!ok) break;
#pragma unroll
        for (int c = 0; c < CWC; c += 32) {
          // −D of the chunk's 32 query columns first, so that the
          // shared-memory loads run during the TMEM load (which, like every
          // tcgen05 wait, orders memory, so the compiler cannot hoist them);
          // then one 32-column TMEM load per chunk (measured faster here than
          // loading all CWC columns before the arithmetic)
          float4 ndc[8];
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) ndc[e4] = sD4[(c >> 2) + e4];
          tmem_ld32(tDP + cw * CWC + c, *reinterpret_cast<uint32_t(*)[32]>(u + c));
          tmem_ld_wait();
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            const float4 nd = ndc[e >> 2];
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              const int q = c + e + 2 * h2;
              uint64_t t;
              if constexpr (DROP) {
                // dP ∘ Z · 256/T − D
                const uint32_t sb = __float_as_uint(p.drop.scale);
                const uint64_t z = pk2(__uint_as_float(keep_word_mask(keep[q >> 2], q & 3) & sb),
                                       __uint_as_float(keep_word_mask(keep[q >> 2], (q & 3) + 1) & sb));
                t = ffma2(pk2(__uint_as_float(u[q]), __uint_as_float(u[q + 1])), z,
                          h2 ? pk2(nd.z, nd.w) : pk2(nd.x, nd.y));
              } else {
                t = fadd2(pk2(__uint_as_float(u[q]), __uint_as_float(u[q + 1])),
                          h2 ? pk2(nd.z, nd.w) : pk2(nd.x, nd.y));
              }
              const float2 pq = ElemTraits<T>::unpack2(Pk[q >> 1]);
              const float2 ds = upk2(fmul2(t, pk2(pq.x, pq.y)));
              w[(e >> 1) + h2] = ElemTraits<T>::pack2(ds.x, ds.y);
            }
          }
#pragma unroll
          for (int c16 = 0; c16 < 4; ++c16) {
            const int col = cw * CWC + c + c16 * 8;  // first query column of this 16-byte chunk
            const int blk = col >> 6, ch = (col >> 3) & 7;
            *reinterpret_cast<uint4*>(sdS + blk * (Tr::BN * 128) + kr * 128 + ((ch ^ (kr & 7)) << 4)) =
                make_uint4(w[c16 * 4], w[c16 * 4 + 1], w[c16 * 4 + 2], w[c16 * 4 + 3]);
          }
        }
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(&bars->ds_ready);
      }
      g += n_q;
    }
  } else {
    // ------------------------------------------------------------ dQ (the warpgroup after the compute ones)
    regs_set<Tr::REGS_DQ, Tr::LAUNCH_REGS>();
    const int quad = warp & 3;
    const int r = quad * 32 + lane;  // TMEM lane: d index (dQᵀ) or query row (dQ)
    const uint32_t lane_off = uint32_t(quad * 32) << 16;
    const uint32_t tQ = tmem + lane_off + Tr::COL_DP;  // dQ of the step sits in the dPᵀ columns
    const bool leader = (warp == Tr::WARP_DQ0 && lane == 0);
    bool ok = true;
    int g = 0, it = 0;
    for (int j; ok && named_bar_and(1, 128, take_item(it, j)); ++it) {
      int bh, kb, i0, n_q;
      item(j, bh, kb, i0, n_q);
      for (int i = 0; i < n_q; ++i) {
        const int gs = g + i;
        const int q0 = (i0 + i) * BM;
        ok = named_bar_and(1, 128, MBAR_WAIT(&bars->dq_full, gs & 1, abort_flag));
        tc_fence_after();
        if (!ok) break;
        if constexpr (Tr::DQ_T) {
          // thread = d index r, TMEM column q = query row q0 + q.  All BM
          // columns come to registers first, so the dPᵀ columns are released
          // after one TMEM round trip; then for each q a warp adds 32
          // consecutive floats (one 128-byte line) of the fp32 accumulator
          // (mode 1), or stores them into this K/V block's partial (mode 2).
          uint32_t v[BM];
#pragma unroll
          for (int c = 0; c < BM; c += 32) tmem_ld32(tQ + c, *reinterpret_cast<uint32_t(*)[32]>(v + c));
          tmem_ld_wait();
          tc_fence_before();
          mbar_arrive(&bars->dq_empty);  // the dPᵀ columns may take the next dPᵀ
          const int slab = dq_slab(p, kb);
          float* dst = p.dQacc + ((size_t(slab) * p.B * p.H + bh) * p.Nq_pad + q0) * D + r;
          if (!FA_INBOUNDS(bh < p.B * p.H && q0 + BM <= p.Nq_pad && slab < dq_slabs(p))) {
          } else if (p.dq_mode == 2) {
#pragma unroll
            for (int q = 0; q < BM; ++q) dst[q * D] = __uint_as_float(v[q]);
          } else {
#pragma unroll
            for (int q = 0; q < BM; ++q) {
              red_add_f32(dst + q * D, __uint_as_float(v[q]));
              // A short pause every 8 reductions spreads them over the
              // step: the L2 takes them at its own rate (~5 TB/s), and a
              // burst fills the SM's load/store queue, which the compute
              // warps' TMEM and shared-memory accesses wait behind.
              // Measured: backward 481 -> 466 us at causal B8 H16 N2048.
              if ((q & 7) == 7) __nanosleep(64);
            }
          }
        } else {
          uint32_t v[D];  // thread = query row r: its D values
#pragma unroll
          for (int c = 0; c < D; c += 32) tmem_ld32(tQ + c, *reinterpret_cast<uint32_t(*)[32]>(v + c));
          tmem_ld_wait();
          tc_fence_before();
          mbar_arrive(&bars->dq_empty);  // the dP columns may take the next dPᵀ
          // The previous bulk operation must have finished reading the staging buffer.
          if (leader) bulk_wait_read0();
          named_bar(1, 128);
          // The row's 64 values go to two 128-byte-swizzled halves (columns
          // 0-31, 32-63): 16-byte chunk j of row r at chunk position
          // j ^ (r % 8), the tensor map's 128-byte swizzle.  Static register
          // indices, and the 8 rows of a store phase hit 8 different chunks.
#pragma unroll
          for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int c = 32 * h + 4 * j;
              float4 x;
              x.x = __uint_as_float(v[c + 0]);
              x.y = __uint_as_float(v[c + 1]);
              x.z = __uint_as_float(v[c + 2]);
              x.w = __uint_as_float(v[c + 3]);
              *reinterpret_cast<float4*>(sdQ + h * (BM * 128) + r * 128 + ((j ^ (r & 7)) << 4)) = x;
            }
          }
          fence_async_smem();
          named_bar(1, 128);
          const int slab = dq_slab(p, kb);
          if (leader && FA_INBOUNDS(bh < p.B * p.H && q0 + BM <= p.Nq_pad && slab < dq_slabs(p))) {
            // rows of the buffer viewed as [rows, 64] fp32 (x = column, y = row)
            const int row = (slab * p.B * p.H + bh) * p.Nq_pad + q0;
            if (p.dq_mode == 2) {
              tma_store_2d(&tmdQ, sdQ, 0, row);
              tma_store_2d(&tmdQ, sdQ + BM * 128, 32, row);
            } else {
              tma_reduce_add_2d(&tmdQ, sdQ, 0, row);
              tma_reduce_add_2d(&tmdQ, sdQ + BM * 128, 32, row);
            }
            bulk_commit();
          }
        }
      }
      if (!ok) break;
      // ---- dK, dV of the item (thread = key row r): out of TMEM 32 columns
      // at a time, packed to the dtype, straight to global memory.  This
      // warpgroup is otherwise idle until the next item's first dQ, so the
      // compute warpgroups go on to the next item's P at once; the
      // accumulators are released after the last TMEM load.
      ok = named_bar_and(1, 128, MBAR_WAIT(&bars->dkv_done, it & 1, abort_flag));
      tc_fence_after();
      if (!ok) break;
      {
        const int key = kb * Tr::BN + r;
        const bool live = key < p.Nk;
        const int krow = live ? key : 0;
#pragma unroll
        for (int which = 0; which < 2; ++which) {
          const uint32_t tcol = tmem + lane_off + (which ? Tr::COL_DK : Tr::COL_DV);
          T* out = reinterpret_cast<T*>(which ? p.dK : p.dV) +
                   row_offset<GEN, D>(which ? p.s_dk : p.s_dv, bh, p.H, p.Nk, krow);
#pragma unroll
          for (int c = 0; c < D; c += 32) {
            uint32_t v[32];
            tmem_ld32(tcol + c, v);
            tmem_ld_wait();
            if (which == 1 && c + 32 == D) {
              tc_fence_before();
              mbar_arrive(&bars->dkv_free);
            }
            // dK: the softmax scale left out of dS; dV: the kept weights'
            // 256/T factor under dropout
            if (which == 1 || DROP) {
              const float mul = which == 1 ? p.scale : p.drop.scale;
#pragma unroll
              for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * mul);
            }
            if (live && FA_INBOUNDS(bh < p.B * p.H && krow < p.Nk)) {
#pragma unroll
              for (int e = 0; e < 32; e += 8) {
                uint4 x = make_uint4(0u, 0u, 0u, 0u);
                if (n_q > 0) {
                  x.x = ElemTraits<T>::pack2(__uint_as_float(v[e]), __uint_as_float(v[e + 1]));
                  x.y = ElemTraits<T>::pack2(__uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
                  x.z = ElemTraits<T>::pack2(__uint_as_float(v[e + 4]), __uint_as_float(v[e + 5]));
                  x.w = ElemTraits<T>::pack2(__uint_as_float(v[e + 6]), __uint_as_float(v[e + 7]));
                }
                *reinterpret_cast<uint4*>(out + c + e) = x;
              }
            }
          }
        }
      }
      g += n_q;
    }
    if (leader) bulk_wait0();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == Tr::WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// −D = −rowsum(dO ∘ O) and −L·log2e into padded buffers (−inf on padding
// rows, so their P is 0), stored negated so the main kernel adds them; in
// mode 1 the fp32 dQ accumulator is cleared.
// A group of D/8 lanes handles one row (8 elements per lane).  Heads go in
// the reverse of the main kernel's order (blocks run in index order, a
// head's row blocks consecutive), so the first heads the main kernel takes
// are the last ones written here, still in L2.
template <typename T, int D, bool GEN>
__global__ void __launch_bounds__(256) bwd_preprocess_kernel(BwdParams p) {
  constexpr int LPR = D / 8;
  constexpr int RPB = 256 / LPR;  // rows per block
  const int g = threadIdx.x / LPR, sl = threadIdx.x % LPR;
  const unsigned nrb = unsigned(p.Nq_pad + RPB - 1) / RPB;  // row blocks per head (1-D grid)
  const int bh = p.B * p.H - 1 - int(blockIdx.x / nrb);
  const int q = int(blockIdx.x % nrb) * RPB + g;
  if (blockIdx.x == 0 && threadIdx.x == 0) *p.item_ctr = 0;
  if (q >= p.Nq_pad || !FA_INBOUNDS(bh < p.B * p.H)) return;
  float dsum = 0.f;
  float lsc = INFINITY;
  if (q < p.Nq) {
    const T* orow = reinterpret_cast<const T*>(p.O) + row_offset<GEN, D>(p.s_o, bh, p.H, p.Nq, q);
    const T* dorow = reinterpret_cast<const T*>(p.dO) + row_offset<GEN, D>(p.s_do, bh, p.H, p.Nq, q);
    const uint4 a = *reinterpret_cast<const uint4*>(orow + sl * 8);
    const uint4 c = *reinterpret_cast<const uint4*>(dorow + sl * 8);
    const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, cw[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 x = ElemTraits<T>::unpack2(aw[k]), y = ElemTraits<T>::unpack2(cw[k]);
      dsum = fmaf(x.x, y.x, dsum);
      dsum = fmaf(x.y, y.y, dsum);
    }
    lsc = p.L[size_t(bh) * p.Nq + q] * kLog2e;
  }
#pragma unroll
  for (int o = LPR / 2; o > 0; o >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, o);
  const size_t row = size_t(bh) * p.Nq_pad + q;
  if (sl == 0) {
    p.neg_D[row] = q < p.Nq ? -dsum : 0.f;
    // a row that sees no key (L = -inf) keeps P = 0 whatever its scores and
    // bias are, as the padding rows do
    p.neg_Lsc[row] = lsc == -INFINITY ? -INFINITY : -lsc;
  }
  if (p.dq_mode != 2) {  // the accumulator(s) of modes 1 and 3 start from zero
    const int n = p.dq_mode == 3 ? p.dq_groups : 1;
    const size_t slab = size_t(p.B) * p.H * p.Nq_pad * D;
    for (int s = 0; s < n; ++s) {
      float4* z = reinterpret_cast<float4*>(p.dQacc + s * slab + row * D + sl * 8);
      z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
      z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
}

// dQ = scale · Σ (dQ accumulator or per-K/V-block partials), cast to the
// dtype (the main kernel's dS leaves the softmax scale out).
// Heads in the reverse of the main kernel's order too: its last heads'
// accumulators are the ones still in L2.
template <typename T, int D, bool CAUSAL, bool GEN>
__global__ void __launch_bounds__(256) bwd_dq_finalise_kernel(BwdParams p) {
  constexpr int LPR = D / 8;
  constexpr int RPB = 256 / LPR;
  const int g = threadIdx.x / LPR, sl = threadIdx.x % LPR;
  const unsigned nrb = unsigned(p.Nq + RPB - 1) / RPB;  // row blocks per head (1-D grid)
  const int bh = p.B * p.H - 1 - int(blockIdx.x / nrb);
  const int q = int(blockIdx.x % nrb) * RPB + g;
  if (q >= p.Nq || !FA_INBOUNDS(bh >= 0 && bh < p.B * p.H)) return;
  float acc[8];
  const size_t row = size_t(bh) * p.Nq_pad + q;
  if (p.dq_mode >= 2) {
    // the partials of K/V blocks 0 .. last (mode 2), or the accumulators
    // they added into (mode 3: block kb into kb mod G)
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] = 0.f;
    int last = p.n_kblocks - 1;
    if (CAUSAL) last = min(last, (q + p.Nk - p.Nq) / 128);
    if (p.dq_mode == 3) last = min(last, p.dq_groups - 1);
    const size_t stride = size_t(p.B) * p.H * p.Nq_pad * D;
    for (int j = 0; j <= last && FA_INBOUNDS(j < dq_slabs(p)); ++j) {
      const float4* src = reinterpret_cast<const float4*>(p.dQacc + j * stride + row * D + sl * 8);
      const float4 x = src[0], y = src[1];
      acc[0] += x.x; acc[1] += x.y; acc[2] += x.z; acc[3] += x.w;
      acc[4] += y.x; acc[5] += y.y; acc[6] += y.z; acc[7] += y.w;
    }
  } else {
    const float4* src = reinterpret_cast<const float4*>(p.dQacc + row * D + sl * 8);
    const float4 x = src[0], y = src[1];
    acc[0] = x.x; acc[1] = x.y; acc[2] = x.z; acc[3] = x.w;
    acc[4] = y.x; acc[5] = y.y; acc[6] = y.z; acc[7] = y.w;
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) acc[k] *= p.scale;
  uint4 o;
  o.x = ElemTraits<T>::pack2(acc[0], acc[1]);
  o.y = ElemTraits<T>::pack2(acc[2], acc[3]);
  o.z = ElemTraits<T>::pack2(acc[4], acc[5]);
  o.w = ElemTraits<T>::pack2(acc[6], acc[7]);
  T* dqrow = reinterpret_cast<T*>(p.dQ) + row_offset<GEN, D>(p.s_dq, bh, p.H, p.Nq, q);
  *reinterpret_cast<uint4*>(dqrow + sl * 8) = o;
}

// fp32 backward on the CUDA cores (fp32 inputs only; a parity path, not a
// fast one).  Same structure as the tensor-core kernel: one CTA per block of
// 64 keys, query rows visited one at a time, P rebuilt from L, D = dO·O per
// row, dK/dV accumulated in shared memory and written once, dQ added with
// fp32 atomics into the (zeroed) output.
template <int D, bool CAUSAL>
__global__ void __launch_bounds__(256) bwd_fp32_simt_kernel(BwdParams p) {
  constexpr int BK = 64;
  extern __shared__ float fsm[];
  float* sK = fsm;               // [BK][D]
  float* sV = sK + BK * D;       // [BK][D]
  float* sdK = sV + BK * D;      // [BK][D]
  float* sdV = sdK + BK * D;     // [BK][D]
  float* sq = sdV + BK * D;      // [D]
  float* sdo = sq + D;           // [D]
  float* sp = sdo + D;           // [BK]
  float* sds = sp + BK;          // [BK]
  __shared__ float sred[2];
  const int tid = threadIdx.x;
  const int kb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int bh = b * p.H + h;
  const int key0 = kb * BK;
  const int off = p.Nk - p.Nq;
  const float* Q = reinterpret_cast<const float*>(p.Q) + size_t(bh) * p.Nq * D;
  const float* K = reinterpret_cast<const float*>(p.K) + size_t(bh) * p.Nk * D;
  const float* V = reinterpret_cast<const float*>(p.V) + size_t(bh) * p.Nk * D;
  const float* O = reinterpret_cast<const float*>(p.O) + size_t(bh) * p.Nq * D;
  const float* dO = reinterpret_cast<const float*>(p.dO) + size_t(bh) * p.Nq * D;
  float* dQ = reinterpret_cast<float*>(p.dQ) + size_t(bh) * p.Nq * D;
  for (int i = tid; i < BK * D; i += 256) {
    const int k = i / D;
    const bool live = key0 + k < p.Nk;
    sK[i] = live ? K[size_t(key0) * D + i] : 0.f;
    sV[i] = live ? V[size_t(key0) * D + i] : 0.f;
    sdK[i] = 0.f;
    sdV[i] = 0.f;
  }
  __syncthreads();
  const int q_first = CAUSAL ? max(0, key0 - off) : 0;
  const int k_sub = tid >> 2, part = tid & 3;  // 4 threads per key
  for (int q = q_first; q < p.Nq; ++q) {
    for (int c = tid; c < D; c += 256) {
      sq[c] = Q[size_t(q) * D + c];
      sdo[c] = dO[size_t(q) * D + c];
    }
    if (tid < 32) {  // D_q = dO_q · O_q
      float acc = 0.f;
      for (int c = tid; c < D; c += 32) acc = fmaf(dO[size_t(q) * D + c], O[size_t(q) * D + c], acc);
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (tid == 0) sred[0] = acc;
    }
    __syncthreads();
    {
      const int key = key0 + k_sub;
      float s = 0.f, dp = 0.f;
      for (int c = part; c < D; c += 4) {
        s = fmaf(sq[c], sK[k_sub * D + c], s);
        dp = fmaf(sdo[c], sV[k_sub * D + c], dp);
      }
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      s += __shfl_xor_sync(0xffffffffu, s, 2);
      dp += __shfl_xor_sync(0xffffffffu, dp, 1);
      dp += __shfl_xor_sync(0xffffffffu, dp, 2);
      const bool vis = key < p.Nk && (!CAUSAL || key <= q + off);
      const float L = p.L[size_t(bh) * p.Nq + q];
      const float pr = vis ? expf(s * p.scale - L) : 0.f;
      if (part == 0) {
        sp[k_sub] = pr;
        sds[k_sub] = pr * (dp - sred[0]) * p.scale;
      }
    }
    __syncthreads();
    for (int i = tid; i < BK * D; i += 256) {
      const int k = i / D, c = i % D;
      sdV[i] = fmaf(sp[k], sdo[c], sdV[i]);
      sdK[i] = fmaf(sds[k], sq[c], sdK[i]);
    }
    for (int c = tid; c < D; c += 256) {
      float acc = 0.f;
      for (int k = 0; k < BK; ++k) acc = fmaf(sds[k], sK[k * D + c], acc);
      atomicAdd(&dQ[size_t(q) * D + c], acc);
    }
    __syncthreads();
  }
  float* dK = reinterpret_cast<float*>(p.dK) + size_t(bh) * p.Nk * D;
  float* dV = reinterpret_cast<float*>(p.dV) + size_t(bh) * p.Nk * D;
  for (int i = tid; i < BK * D; i += 256) {
    if (key0 + i / D < p.Nk) {
      dK[size_t(key0) * D + i] = sdK[i];
      dV[size_t(key0) * D + i] = sdV[i];
    }
  }
}

template <int D, bool CAUSAL>
static cudaError_t launch_bwd_fp32(const BwdLaunch& a) {
  const BwdParams& p = a.params;
  cudaError_t e = cudaMemsetAsync(p.dQ, 0, size_t(p.B) * p.H * p.Nq * D * sizeof(float), a.stream);
  if (e != cudaSuccess) return e;
  const int smem = (4 * 64 * D + 2 * D + 2 * 64) * sizeof(float);
  auto kern = bwd_fp32_simt_kernel<D, CAUSAL>;
  e = set_smem_once(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  kern<<<dim3((p.Nk + 63) / 64, p.H, p.B), 256, smem, a.stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

template <typename T, int D, bool CAUSAL, bool GEN, bool DROP = false, bool BIAS = false>
static cudaError_t launch_bwd_t(const BwdLaunch& a) {
  using Tr = BwdTraits<T, D, BIAS>;
  const BwdParams& p = a.params;
  constexpr int RPB = 256 / (D / 8);
  const int BH = p.B * p.H;
  // 1-D grids over (head, row block): B·H may exceed a grid's second dimension
  bwd_preprocess_kernel<T, D, GEN><<<unsigned((p.Nq_pad + RPB - 1) / RPB) * unsigned(BH), 256, 0, a.stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  auto kern = bwd_main_kernel<T, D, CAUSAL, GEN, DROP, BIAS>;
  e = set_smem_once(reinterpret_cast<const void*>(kern), Tr::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  // setmaxnreg.inc draws on the registers the CTA was launched with: refuse
  // to launch if the compiled count cannot cover the split.
  static int regs_ok = -1;
  if (regs_ok < 0) {
    cudaFuncAttributes attr;
    e = cudaFuncGetAttributes(&attr, reinterpret_cast<const void*>(kern));
    if (e != cudaSuccess) return e;
    regs_ok = attr.numRegs * Tr::THREADS >=
              128 * (Tr::NCW * Tr::REGS_COMPUTE + Tr::REGS_DQ + Tr::REGS_OTHER);
  }
  if (!regs_ok) return cudaErrorInvalidConfiguration;
  if (a.ev_start) {
    e = cudaEventRecord(a.ev_start, a.stream);
    if (e != cudaSuccess) return e;
  }
  // persistent: one CTA per SM (or per work item, if fewer)
  const int grid = std::min(p.n_kblocks * BH, sm_count());
  kern<<<grid, Tr::THREADS, Tr::SMEM_BYTES, a.stream>>>(a.tmQ, a.tmK, a.tmV, a.tmdO, a.tmdQ, a.tmBias, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (a.ev_stop) {
    e = cudaEventRecord(a.ev_stop, a.stream);
    if (e != cudaSuccess) return e;
  }
  bwd_dq_finalise_kernel<T, D, CAUSAL, GEN><<<unsigned((p.Nq + RPB - 1) / RPB) * unsigned(BH), 256, 0, a.stream>>>(p);
  return cudaGetLastError();
}

int bwd_block_rows(int d) { (void)d; return 128; }

cudaError_t launch_bwd(int dtype, int d, bool causal, const BwdLaunch& a) {
  const BwdParams& p = a.params;
  const bool gen = p.map4d != 0 || !contiguous_strides(p.s_o, p.H, p.Nq, d) ||
                   !contiguous_strides(p.s_do, p.H, p.Nq, d) ||
                   !contiguous_strides(p.s_dq, p.H, p.Nq, d) ||
                   !contiguous_strides(p.s_dk, p.H, p.Nk, d) ||
                   !contiguous_strides(p.s_dv, p.H, p.Nk, d);
  const bool drop = p.drop.t4 != 0;
  const bool bias = p.bias != nullptr;
  // dropout and bias run in general-layout variants only
#define FA_BWD_CASE(TY, DD)                                                        \
  {                                                                                \
    if (bias)                                                                      \
      return causal ? (drop ? launch_bwd_t<TY, DD, true, true, true, true>(a)     \
                            : launch_bwd_t<TY, DD, true, true, false, true>(a))   \
                    : (drop ? launch_bwd_t<TY, DD, false, true, true, true>(a)    \
                            : launch_bwd_t<TY, DD, false, true, false, true>(a)); \
    if (drop)                                                                      \
      return causal ? launch_bwd_t<TY, DD, true, true, true>(a)                    \
                    : launch_bwd_t<TY, DD, false, true, true>(a);                  \
    return causal ? (gen ? launch_bwd_t<TY, DD, true, true>(a)                     \
                         : launch_bwd_t<TY, DD, true, false>(a))                   \
                  : (gen ? launch_bwd_t<TY, DD, false, true>(a)                    \
                         : launch_bwd_t<TY, DD, false, false>(a));                 \
  }
  if (dtype == FA_BF16) {
    if (d == 64) FA_BWD_CASE(__nv_bfloat16, 64)
    if (d == 128) FA_BWD_CASE(__nv_bfloat16, 128)
  } else if (dtype == FA_FP16) {
    if (d == 64) FA_BWD_CASE(__half, 64)
    if (d == 128) FA_BWD_CASE(__half, 128)
  } else if (dtype == FA_FP32) {
    if (d == 64) return causal ? launch_bwd_fp32<64, true>(a) : launch_bwd_fp32<64, false>(a);
    if (d == 128) return causal ? launch_bwd_fp32<128, true>(a) : launch_bwd_fp32<128, false>(a);
  }
#undef FA_BWD_CASE
  return cudaErrorNotSupported;
}

FA_ERROR_ACCESSOR(take_error_bwd)


}  // namespace fa
