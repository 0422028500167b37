// Host-side launch interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cstddef>
#include <cuda.h>
#include <cuda_runtime.h>

namespace fa {

// Element strides of one [B, H, N, d] attention tensor (d contiguous).
struct Strides {
  long long b, h, n;
};

inline bool contiguous_strides(const Strides& s, int H, int N, int d) {
  return s.n == d && s.h == (long long)N * d && s.b == (long long)H * N * d;
}

// Element offset of row n of head bh = b·H + h: the general strided form, or
// the contiguous [B·H, N, D] one when GEN is false.
template <bool GEN, int D>
__host__ __device__ __forceinline__ long long row_offset(const Strides& s, int bh, int H, int N, int n) {
  if constexpr (GEN)
    return (bh / H) * s.b + (bh % H) * s.h + n * s.n;
  else
    return ((long long)bh * N + n) * D;
}

// Dropout of the attention weights (see dropout.cuh); t4 == 0 means none.
struct DropoutParams {
  uint32_t rk[10][2];  // Philox round keys: the seed's (low, high) words plus r·(Weyl constants)
  uint32_t offset;     // Philox counter word 3
  uint32_t t4;         // keep threshold T (1..255) in each of the four bytes
  float scale;         // 256 / T, applied to the kept weights
};

struct FwdParams {
  const void* Q;  // raw inputs (read directly only by the fp32 path)
  const void* K;
  const void* V;
  void* O;
  float* L;
  int B, H, Nq, Nk;
  float scale_log2;  // scale * log2(e)
  int tiles;         // kernel shape (fwd_tiles_for): 2 = two 128-row Q tiles per CTA, 3 = one over 64-key K/V tiles
  int n_qblocks;     // ceil(Nq / query rows per CTA): one CTA per block of query rows
  int head_group;    // heads per launch-order group (see head_group_for)
  int map4d;         // bit per tensor map (Q 0, K 1, V 2, O 3): 4-D (d, N, H, B), else 3-D (d, N, B·H)
  DropoutParams drop;
  const int* kv_len;  // key padding: keys of batch element b are [0, kv_len[b]); null = all Nk
  const void* bias;   // additive bias on the scaled scores, [B', H', Nq, Nk] input dtype; null = none
  Strides s_bias;     // its element strides (0 broadcasts a batch or head; columns contiguous)
  float bias_mul;     // 1 / scale: the bias in units of the unscaled scores
  int bias_H, bias_B; // the bias tensor map's head and batch extents (1 where it broadcasts)
  int bias_rows;      // rows of a staged bias tile: 128, or 1 for a bias shared by all query rows
};

struct FwdLaunch {
  CUtensorMap tmQ, tmK, tmV;
  CUtensorMap tmO;  // output, written by TMA stores (16-bit types)
  CUtensorMap tmBias;  // bias: (key, query, head, batch), 128-byte-swizzled boxes of 64 keys
  FwdParams params;
  cudaStream_t stream;
};

// Forward kernel for a call: 2 (two 128-row Q tiles per CTA over 128-key K/V
// tiles) or 3 (one Q tile over 64-key K/V tiles with double-buffered scores).
int fwd_tiles_for(int dtype, int d, int Nq, int Nk, bool causal, bool drop, bool bias);
cudaError_t launch_fwd(int dtype, int d, bool causal, const FwdLaunch& a);

struct BwdParams {
  const void* Q;
  const void* K;
  const void* V;
  const void* O;
  const void* dO;
  const float* L;
  void* dQ;
  void* dK;
  void* dV;
  float* neg_D;    // [B*H, Nq_pad] -rowsum(dO * O), padded rows zero
  float* neg_Lsc;  // [B*H, Nq_pad] -L * log2(e), padded rows -inf
  float* dQacc;   // fp32 [S, B*H, Nq_pad, d]: S = 1 (mode 1), nkv (mode 2), dq_groups (mode 3)
  int* item_ctr;  // work items handed out beyond the first wave (zeroed by the preprocess)
  int B, H, Nq, Nk, Nq_pad;
  float scale;        // softmax scale
  float scale_log2;   // scale * log2(e)
  int n_kblocks;      // ceil(Nk / 128)
  int dq_mode;        // 1 = reduce-add into one buffer, 2 = per-K/V-block partials,
                      // 3 = reduce-add into dq_groups buffers (K/V block kb into kb mod dq_groups)
  int dq_groups;      // buffers of mode 3 (1..16)
  int head_group;     // heads per launch-order group (see head_group_for)
  Strides s_o, s_do, s_dq, s_dk, s_dv;  // plain (non-TMA) accesses; Q, K, V, dO go through tensor maps
  int map4d;  // bit per tensor map (Q 0, K 1, V 2, dO 4): 4-D (d, N, H, B), else 3-D (d, N, B·H)
  DropoutParams drop;
  const int* kv_len;  // key padding, as in FwdParams
  const void* bias;   // additive bias, as in FwdParams
  Strides s_bias;
  float bias_l2;      // log2(e): the bias in the backward's log2 units
  int bias_H, bias_B; // the bias tensor map's head and batch extents (1 where it broadcasts)
  int bias_rows;      // query rows of the staged bias tile: 128, or 1 for a bias shared by all rows
};

struct BwdLaunch {
  CUtensorMap tmQ, tmK, tmV, tmdO;
  CUtensorMap tmdQ;  // d = 64: the fp32 dQ accumulator as a [rows, 64] tensor (tensor reduce-add)
  CUtensorMap tmBias;  // bias: (key, query, head, batch), boxes of 128 keys × 128 queries
  BwdParams params;
  cudaStream_t stream;
  cudaEvent_t ev_start, ev_stop;  // optional timing events around the main kernel
};

cudaError_t launch_bwd(int dtype, int d, bool causal, const BwdLaunch& a);

// Streaming multiprocessors of the current device (cached per device).
int sm_count();

// Heads per launch-order group: as many as keep the bytes one head's CTAs
// share (K and V in the forward; Q, dO, the fp32 dQ accumulator, L and D in
// the backward) within a slice of L2, at least 1 and at most B·H.
#ifndef FA_L2_GROUP_BYTES
#define FA_L2_GROUP_BYTES (48ull << 20)
#endif
inline int head_group_for(size_t bytes_per_head, int BH) {
  size_t g = bytes_per_head ? FA_L2_GROUP_BYTES / bytes_per_head : size_t(BH);
  if (g < 1) g = 1;
  if (g > size_t(BH)) g = size_t(BH);
  return int(g);
}
// Query rows per backward step (the TMA box height of Q and dO).
int bwd_block_rows(int d);

struct DecodeParams {
  const void* Q;
  const void* K;
  const void* V;
  void* O;
  float* L;
  float* Opart;  // [B*H, S, d] normalised partial outputs
  float* Lpart;  // [B*H, S] natural-log logsumexp of each part (-inf if empty)
  int BH, Nk, splits, keys_per_split;
  float scale_log2;
  int H;
  const int* kv_len;  // key padding (keys [0, kv_len[b]) of batch element b); null = all Nk
};

cudaError_t launch_decode(int dtype, int d, const DecodeParams& p, cudaStream_t s);
// Library-owned scratch of fa_decode_noalloc (decode.cu): its size, and its
// device address on the current device.
size_t decode_scratch_bytes();
cudaError_t decode_scratch_ptr(void** out);

// Read-and-clear accessors of each kernel file's device error word.
cudaError_t take_error_fwd(int* word, int* site);
cudaError_t take_error_bwd(int* word, int* site);
cudaError_t take_error_decode(int* word, int* site);
cudaError_t launch_selftest_wait(unsigned long long limit_ns, cudaStream_t stream);

// Sets the dynamic shared-memory limit of `kernel` on the current device once.
// Sets a kernel's dynamic shared-memory size once per device (and, with
// max_carveout, asks for the largest shared-memory carveout of the SM).
cudaError_t set_smem_once(const void* kernel, int bytes, bool max_carveout = false);

}  // namespace fa
