// C ABI of the attention library: argument checks, TMA descriptor set-up,
// workspace layout and kernel launches.  No device memory is allocated here
// and nothing synchronises except fa_status.
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "fa.h"
#include "launch.h"

namespace fa {

namespace {

constexpr int kMaxDevices = 64;

std::atomic<int> g_dq_mode{0};    // 0 auto, 1 reduce-add, 2 partial buffers, 3 grouped
std::atomic<int> g_dq_groups{4};  // accumulators of mode 3
cudaEvent_t g_ev_start = nullptr, g_ev_stop = nullptr;  // fa_bwd_set_timing_events
std::atomic<int> g_last_site{0};  // fa_last_timeout_site
std::atomic<int> g_last_cuda{0};  // fa_last_cuda_error

// FA_ERR_CUDA, remembering the code behind it (a cudaError_t, or 100000 +
// the CUresult of a failed tensor-map encoding) for fa_last_cuda_error.
int cuda_fail(int code) {
  g_last_cuda = code;
  return FA_ERR_CUDA;
}
int from_cuda(cudaError_t e) { return e == cudaSuccess ? FA_OK : cuda_fail(int(e)); }

// A named NVTX range around each computing entry point, so that profiler
// timelines show the library's calls (a no-op unless a tool is attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// Tensor-map encoding is a driver call, which needs a current context on the
// calling thread; a thread that has made no runtime call yet (an autograd
// worker, a fresh host thread) has none.  cudaSetDevice makes the current
// device's primary context current on this thread.
cudaError_t ensure_context() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  return e != cudaSuccess ? e : cudaSetDevice(dev);
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

int elem_size(int dtype) { return dtype == FA_FP32 ? 4 : 2; }

CUtensorMapDataType tma_type(int dtype) {
  switch (dtype) {
    case FA_BF16: return CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    case FA_FP16: return CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    default: return CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  }
}

// Tensor map over a [B, H, N, d] tensor with element strides l (d
// contiguous).  When batches are exactly H heads apart (l.b == H·l.h, as in a
// contiguous tensor) heads and batches merge into one index: a 3-D map
// (x = d, y = row, z = b·H + h); otherwise a 4-D map (x, y, z = h, w = b),
// and *is4d says which.  The box is one 128-byte swizzled column block of
// `box_rows` rows; rows past N read as zero (and stores there are dropped).
bool make_map(CUtensorMap* m, const void* ptr, int dtype, int d, int N, int H, int B,
              const fa_layout& l, int box_rows, bool* is4d) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) {
    g_last_cuda = int(cudaErrorSymbolNotFound);
    return false;
  }
  const int es = elem_size(dtype);
  const bool merge = l.b == (long long)H * l.h;
  *is4d = !merge;
  cuuint64_t dims[4] = {cuuint64_t(d), cuuint64_t(N), cuuint64_t(merge ? B * H : H), cuuint64_t(B)};
  cuuint64_t strides[3] = {cuuint64_t(l.n) * es, cuuint64_t(l.h) * es, cuuint64_t(l.b) * es};
  cuuint32_t box[4] = {cuuint32_t(128 / es), cuuint32_t(box_rows), 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(m, tma_type(dtype), merge ? 3 : 4, const_cast<void*>(ptr), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) g_last_cuda = 100000 + int(r);
  return r == CUDA_SUCCESS;
}

// Tensor map of an additive bias for staging [rows × keys] tiles: 4-D (key,
// query, head, batch), whose query, head or batch extent is 1 where the bias
// broadcasts (stride 0, which a tensor map cannot hold; the stride given for
// such a dimension is never stepped over).  A bias shared by all query rows
// gives 1-row boxes.  Reads past Nq and Nk are zero-filled.  Sets the
// extents the kernels index with.
CUresult encode_bias_map(CUtensorMap* m, const void* bias, const fa_layout& lb, int dtype, int B,
                         int H, int Nq, int Nk, int box_keys, bool swizzle128, int* bias_H,
                         int* bias_B, int* bias_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return CUDA_ERROR_NOT_FOUND;
  *bias_H = lb.h ? H : 1;
  *bias_B = lb.b ? B : 1;
  *bias_rows = lb.n ? 128 : 1;
  const cuuint64_t es = cuuint64_t(elem_size(dtype));
  const cuuint64_t unit = (cuuint64_t(Nk) * es + 15) / 16 * 16;
  cuuint64_t dims[4] = {cuuint64_t(Nk), lb.n ? cuuint64_t(Nq) : 1, cuuint64_t(*bias_H),
                        cuuint64_t(*bias_B)};
  cuuint64_t strides[3] = {lb.n ? cuuint64_t(lb.n) * es : unit, lb.h ? cuuint64_t(lb.h) * es : unit,
                           lb.b ? cuuint64_t(lb.b) * es : unit};
  cuuint32_t box[4] = {cuuint32_t(box_keys), cuuint32_t(*bias_rows), 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(m, tma_type(dtype), 4, const_cast<void*>(bias), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE,
             swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

fa_layout contiguous_layout(int H, int N, int d) {
  return fa_layout{(long long)H * N * d, (long long)N * d, (long long)d};
}

bool is_contiguous(const fa_layout& l, int H, int N, int d) {
  const fa_layout c = contiguous_layout(H, N, d);
  return l.b == c.b && l.h == c.h && l.n == c.n;
}

// Strides the kernels accept: non-negative, each a multiple of 16 bytes (the
// tensor-map rule; it also keeps every row 16-byte aligned).
bool valid_layout(const fa_layout* l, int dtype) {
  if (!l) return false;
  const long long es = elem_size(dtype);
  const long long v[3] = {l->b, l->h, l->n};
  for (long long x : v)
    if (x < 0 || (x * es) % 16 != 0 || x * es >= (1ll << 40)) return false;
  return true;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_common(int B, int H, int Nq, int Nk, int d, float scale, int dtype) {
  if (B <= 0 || H <= 0 || Nq <= 0 || Nk <= 0 || d <= 0) return FA_ERR_INVALID;
  if (!std::isfinite(scale) || scale <= 0.f) return FA_ERR_INVALID;
  if (dtype != FA_FP32 && dtype != FA_BF16 && dtype != FA_FP16) return FA_ERR_INVALID;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (B > 65535 || H > 65535) return FA_ERR_UNSUPPORTED;
  if (int64_t(B) * H > (int64_t(1) << 31) - 1) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int bwd_pad_rows(int Nq) { return int(round_up(size_t(Nq), 128)); }

int effective_dq_mode(int B, int H, int Nq, int Nk, int d) {
  const int forced = g_dq_mode.load();
  if (forced != 0) return forced;
  (void)B; (void)H; (void)Nq; (void)Nk; (void)d;
  return 1;  // reduce-add: measured faster (partials cost nkv× the dQ traffic)
}

struct BwdWorkspace {
  size_t d_off, l_off, dq_off, ctr_off, total;
};

BwdWorkspace bwd_layout(int B, int H, int Nq, int Nk, int d, int mode, int groups) {
  const size_t BH = size_t(B) * H;
  const size_t rows = size_t(bwd_pad_rows(Nq));
  const size_t nkv = (size_t(Nk) + 127) / 128;
  BwdWorkspace w;
  w.d_off = 0;
  w.l_off = round_up(BH * rows * sizeof(float), 256);
  w.dq_off = w.l_off + round_up(BH * rows * sizeof(float), 256);
  const size_t slabs = mode == 2 ? nkv : mode == 3 ? size_t(groups) : 1;
  const size_t dq = BH * rows * size_t(d) * sizeof(float) * slabs;
  w.ctr_off = w.dq_off + round_up(dq, 256);  // work-item counter of the main kernel
  w.total = w.ctr_off + 256;
  return w;
}

int decode_auto_splits(int BH, int Nk) {
  // Enough CTAs for many waves over 148 SMs (so the ragged last wave costs
  // little), but parts of at least 256 keys.
  const int target = 148 * 8 * 16;
  int s = (target + BH - 1) / BH;
  s = std::max(1, std::min(s, 128));
  const int max_by_len = std::max(1, Nk / 256);
  return std::min(s, max_by_len);
}

int decode_keys_per_split(int Nk, int splits) {
  int kps = (Nk + splits - 1) / splits;
  return int(round_up(size_t(kps), 64));
}

}  // namespace

cudaError_t set_smem_once(const void* kernel, int bytes, bool max_carveout) {
  static std::mutex mu;
  static int done_n[kMaxDevices] = {0};
  constexpr int kTracked = 128;  // more than the kernel variants of the library
  static const void* done_k[kMaxDevices][kTracked];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(mu);
  const bool track = dev >= 0 && dev < kMaxDevices;
  if (track)
    for (int i = 0; i < done_n[dev]; ++i)
      if (done_k[dev][i] == kernel) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && max_carveout)
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess && track && done_n[dev] < kTracked) done_k[dev][done_n[dev]++] = kernel;
  return e;
}

int sm_count() {
  static std::mutex mu;
  static int n_sm[kMaxDevices] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  std::lock_guard<std::mutex> lk(mu);
  if (n_sm[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    n_sm[dev] = n;
  }
  return n_sm[dev];
}

// Dropout parameters from the C struct: FA_OK with *out filled (t4 = 0 when
// there is no dropout), or FA_ERR_INVALID for a probability outside [0, 1)
// or one that keeps nothing after rounding.  The keep threshold is
// T = round((1 − p)·256), computed in double from the float p.
int dropout_params(const fa_dropout* dr, DropoutParams* out) {
  std::memset(out, 0, sizeof(*out));
  if (!dr || dr->p == 0.0f) return FA_OK;
  const double pd = dr->p;
  if (!(pd >= 0.0 && pd < 1.0)) return FA_ERR_INVALID;  // also rejects NaN
  const long t = std::lrint((1.0 - pd) * 256.0);
  if (t < 1) return FA_ERR_INVALID;
  if (t >= 256) return FA_OK;  // rounds to keeping everything: no dropout
  // Philox4x32-10 key schedule: round r uses the seed's words plus r times
  // the Weyl constants (mod 2^32); computed once here, read by every draw.
  uint32_t k0 = uint32_t(dr->seed & 0xFFFFFFFFull), k1 = uint32_t(dr->seed >> 32);
  for (int r = 0; r < 10; ++r) {
    out->rk[r][0] = k0;
    out->rk[r][1] = k1;
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  out->offset = dr->offset;
  out->t4 = uint32_t(t) * 0x01010101u;
  out->scale = float(256.0 / double(t));
  return FA_OK;
}

}  // namespace fa

using namespace fa;

extern "C" {

int fa_fwd_ex(const void* Q, const void* K, const void* V, void* O, float* L, const fa_layout* lq,
              const fa_layout* lk, const fa_layout* lv, const fa_layout* lo, int B, int H, int Nq,
              int Nk, int d, int causal, float scale, int dtype, const fa_dropout* dropout,
              const int* kv_len, const void* bias, const fa_layout* lbias, void* stream) {
  NvtxRange nvtx_range("fa_fwd_ex");
  int st = check_common(B, H, Nq, Nk, d, scale, dtype);
  if (st != FA_OK) return st;
  if (!Q || !K || !V || !O || !L) return FA_ERR_INVALID;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(L))
    return FA_ERR_INVALID;
  if (!valid_layout(lq, dtype) || !valid_layout(lk, dtype) || !valid_layout(lv, dtype) ||
      !valid_layout(lo, dtype))
    return FA_ERR_INVALID;
  if (dtype == FA_FP32 && d != 64) return FA_ERR_UNSUPPORTED;
  // the fp32 path stages its tiles with plain loads of contiguous tensors
  if (dtype == FA_FP32 && !(is_contiguous(*lq, H, Nq, d) && is_contiguous(*lk, H, Nk, d) &&
                            is_contiguous(*lv, H, Nk, d) && is_contiguous(*lo, H, Nq, d)))
    return FA_ERR_UNSUPPORTED;
  if (causal && Nq > Nk) return FA_ERR_UNSUPPORTED;
  if (int64_t((Nq + 127) / 128) * B * H > INT32_MAX) return FA_ERR_UNSUPPORTED;  // 1-D grid
  DropoutParams drop;
  st = dropout_params(dropout, &drop);
  if (st != FA_OK) return st;
  if (drop.t4 && dtype == FA_FP32) return FA_ERR_UNSUPPORTED;
  if (kv_len && (reinterpret_cast<uintptr_t>(kv_len) & 3u)) return FA_ERR_INVALID;
  if (kv_len && dtype == FA_FP32) return FA_ERR_UNSUPPORTED;
  if (bias && (!aligned16(bias) || !valid_layout(lbias, dtype))) return FA_ERR_INVALID;
  if (bias && dtype == FA_FP32) return FA_ERR_UNSUPPORTED;
  const int BH = B * H;
  FwdLaunch a;
  std::memset(&a, 0, sizeof(a));
  a.params.drop = drop;
  a.params.kv_len = kv_len;
  st = from_cuda(ensure_context());
  if (st != FA_OK) return st;
  if (bias) {
    a.params.bias = bias;
    a.params.s_bias = Strides{lbias->b, lbias->h, lbias->n};
    a.params.bias_mul = 1.0f / scale;
    // the forward stages [128 rows × 128 keys] tiles as two 128-byte-swizzled
    // halves of 64 keys
    const CUresult r = encode_bias_map(&a.tmBias, bias, *lbias, dtype, B, H, Nq, Nk, 64, true,
                                       &a.params.bias_H, &a.params.bias_B, &a.params.bias_rows);
    if (r != CUDA_SUCCESS) return cuda_fail(100000 + int(r));
  }
  // Q tiles per CTA and K/V tile rows (3: one Q tile over 64-key K/V tiles)
  a.params.tiles = fwd_tiles_for(dtype, d, Nq, Nk, causal != 0, drop.t4 != 0, bias != nullptr);
  const int kv_rows = a.params.tiles == 3 ? 64 : 128;
  bool m4[4];
  if (!make_map(&a.tmQ, Q, dtype, d, Nq, H, B, *lq, 128, &m4[0]) ||
      !make_map(&a.tmK, K, dtype, d, Nk, H, B, *lk, kv_rows, &m4[1]) ||
      !make_map(&a.tmV, V, dtype, d, Nk, H, B, *lv, kv_rows, &m4[2]) ||
      !make_map(&a.tmO, O, dtype, d, Nq, H, B, *lo, 128, &m4[3]))
    return FA_ERR_CUDA;
  for (int i = 0; i < 4; ++i) a.params.map4d |= int(m4[i]) << i;
  a.params.Q = Q;
  a.params.K = K;
  a.params.V = V;
  a.params.O = O;
  a.params.L = L;
  a.params.B = B;
  a.params.H = H;
  a.params.Nq = Nq;
  a.params.Nk = Nk;
  a.params.scale_log2 = scale * 1.4426950408889634f;
  const int rows = a.params.tiles == 2 ? 256 : 128;  // query rows per CTA
  a.params.n_qblocks = (Nq + rows - 1) / rows;
  a.params.head_group = head_group_for(size_t(Nk) * d * 2 * elem_size(dtype), BH);
  a.stream = static_cast<cudaStream_t>(stream);
  return from_cuda(launch_fwd(dtype, d, causal != 0, a));
}

int fa_fwd(const void* Q, const void* K, const void* V, void* O, float* L, int B, int H, int Nq,
           int Nk, int d, int causal, float scale, int dtype, void* stream) {
  const fa_layout lq = contiguous_layout(H, Nq, d), lk = contiguous_layout(H, Nk, d);
  return fa_fwd_ex(Q, K, V, O, L, &lq, &lk, &lk, &lq, B, H, Nq, Nk, d, causal, scale, dtype, nullptr,
                   nullptr, nullptr, nullptr, stream);
}

size_t fa_bwd_workspace_bytes(int B, int H, int Nq, int Nk, int d, int dtype) {
  if (check_common(B, H, Nq, Nk, d, 1.0f, dtype) != FA_OK) return 0;
  return bwd_layout(B, H, Nq, Nk, d, effective_dq_mode(B, H, Nq, Nk, d), g_dq_groups.load()).total;
}

int fa_set_bwd_dq_mode(int mode) {
  if (mode < 0 || mode > 3) return FA_ERR_INVALID;
  const int prev = g_dq_mode.exchange(mode);
  return prev;
}

int fa_set_bwd_dq_groups(int groups) {
  if (groups < 1 || groups > 16) return FA_ERR_INVALID;
  return g_dq_groups.exchange(groups);
}

int fa_bwd_ex(const void* Q, const void* K, const void* V, const void* O, const void* dO,
              const float* L, void* dQ, void* dK, void* dV, const fa_layout* lq,
              const fa_layout* lk, const fa_layout* lv, const fa_layout* lo, const fa_layout* ldo,
              const fa_layout* ldq, const fa_layout* ldk, const fa_layout* ldv, int B, int H,
              int Nq, int Nk, int d, int causal, float scale, int dtype, const fa_dropout* dropout,
              const int* kv_len, const void* bias, const fa_layout* lbias, void* workspace,
              size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("fa_bwd_ex");
  int st = check_common(B, H, Nq, Nk, d, scale, dtype);
  if (st != FA_OK) return st;
  const void* ptrs[] = {Q, K, V, O, dO, L, dQ, dK, dV};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return FA_ERR_INVALID;
  const fa_layout* lays[] = {lq, lk, lv, lo, ldo, ldq, ldk, ldv};
  for (const fa_layout* l : lays)
    if (!valid_layout(l, dtype)) return FA_ERR_INVALID;
  if (dtype == FA_FP32 && d != 64) return FA_ERR_UNSUPPORTED;
  if (dtype == FA_FP32) {  // the CUDA-core fp32 path reads and writes contiguous tensors
    const int rows[] = {Nq, Nk, Nk, Nq, Nq, Nq, Nk, Nk};
    for (int i = 0; i < 8; ++i)
      if (!is_contiguous(*lays[i], H, rows[i], d)) return FA_ERR_UNSUPPORTED;
  }
  if (causal && Nq > Nk) return FA_ERR_UNSUPPORTED;
  // 1-D grids: (head, row block) for the per-row kernels, work items per (K/V block, head)
  if (int64_t((bwd_pad_rows(Nq) + 15) / 16) * B * H > INT32_MAX ||
      int64_t((Nk + 127) / 128) * B * H > INT32_MAX)
    return FA_ERR_UNSUPPORTED;
  DropoutParams drop;
  st = dropout_params(dropout, &drop);
  if (st != FA_OK) return st;
  if (drop.t4 && dtype == FA_FP32) return FA_ERR_UNSUPPORTED;
  if (kv_len && (reinterpret_cast<uintptr_t>(kv_len) & 3u)) return FA_ERR_INVALID;
  if (kv_len && dtype == FA_FP32) return FA_ERR_UNSUPPORTED;
  if (bias && (!aligned16(bias) || !valid_layout(lbias, dtype))) return FA_ERR_INVALID;
  if (bias && dtype == FA_FP32) return FA_ERR_UNSUPPORTED;
  const int mode = effective_dq_mode(B, H, Nq, Nk, d);
  const int groups = g_dq_groups.load();
  const BwdWorkspace w = bwd_layout(B, H, Nq, Nk, d, mode, groups);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || ws_bytes < w.total)
    return FA_ERR_WORKSPACE;
  const int BH = B * H;
  BwdLaunch a;
  std::memset(&a, 0, sizeof(a));
  const int bm = bwd_block_rows(d);
  // (the fp32 path stages its operands without TMA)
  // (dK and dV are written with plain stores: their strides go to the kernel)
  st = from_cuda(ensure_context());
  if (st != FA_OK) return st;
  bool m4[5] = {false, false, false, false, false};
  if (dtype != FA_FP32 &&
      (!make_map(&a.tmQ, Q, dtype, d, Nq, H, B, *lq, bm, &m4[0]) ||
       !make_map(&a.tmK, K, dtype, d, Nk, H, B, *lk, 128, &m4[1]) ||
       !make_map(&a.tmV, V, dtype, d, Nk, H, B, *lv, 128, &m4[2]) ||
       !make_map(&a.tmdO, dO, dtype, d, Nq, H, B, *ldo, bm, &m4[4])))
    return FA_ERR_CUDA;
  BwdParams& p = a.params;
  p.Q = Q; p.K = K; p.V = V; p.O = O; p.dO = dO; p.L = L;
  p.dQ = dQ; p.dK = dK; p.dV = dV;
  p.neg_D = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + w.d_off);
  p.neg_Lsc = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + w.l_off);
  p.dQacc = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + w.dq_off);
  p.item_ctr = reinterpret_cast<int*>(static_cast<uint8_t*>(workspace) + w.ctr_off);
  p.B = B; p.H = H; p.Nq = Nq; p.Nk = Nk;
  p.Nq_pad = bwd_pad_rows(Nq);
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.n_kblocks = (Nk + 127) / 128;
  p.dq_mode = mode;
  p.dq_groups = groups;
  p.head_group = head_group_for(size_t(p.Nq_pad) * (size_t(d) * (2 * elem_size(dtype) + 4) + 8), BH);
  auto to_strides = [](const fa_layout* l) { return Strides{l->b, l->h, l->n}; };
  p.s_o = to_strides(lo);
  p.s_do = to_strides(ldo);
  p.s_dq = to_strides(ldq);
  p.s_dk = to_strides(ldk);
  p.s_dv = to_strides(ldv);
  for (int i = 0; i < 5; ++i) p.map4d |= int(m4[i]) << i;  // Q 0, K 1, V 2, dO 4
  if (dtype != FA_FP32 && d == 64) {
    // The d = 64 kernel reduces each step's dQ tile into the fp32 accumulator
    // (or stores it into its K/V block's partial) through a 2-D map over the
    // whole buffer: [rows, 64] fp32, boxes of 32 columns (128 bytes,
    // 128-byte swizzle) by 128 rows.
    const uint64_t slabs = mode == 2 ? uint64_t(p.n_kblocks) : mode == 3 ? uint64_t(groups) : 1u;
    const uint64_t rows = uint64_t(BH) * p.Nq_pad * slabs;
    if (rows > uint64_t(INT32_MAX)) return FA_ERR_UNSUPPORTED;  // TMA row coordinates are int32
    EncodeTiledFn enc = encode_fn();
    cuuint64_t dims[2] = {cuuint64_t(d), cuuint64_t(rows)};
    cuuint64_t strides[1] = {cuuint64_t(d) * sizeof(float)};
    cuuint32_t box[2] = {32, 128};
    cuuint32_t estr[2] = {1, 1};
    if (!enc) return cuda_fail(int(cudaErrorSymbolNotFound));
    const CUresult r = enc(&a.tmdQ, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, p.dQacc, dims, strides, box,
                           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cuda_fail(100000 + int(r));
  }
  p.drop = drop;
  p.kv_len = kv_len;
  if (bias) {
    p.bias = bias;
    p.s_bias = Strides{lbias->b, lbias->h, lbias->n};
    p.bias_l2 = 1.4426950408889634f;
    // The backward stages each step's [128 queries × 128 keys] bias tile with
    // one TMA load (no swizzle: a warp reads 64 consecutive bytes of a row).
    const CUresult r = encode_bias_map(&a.tmBias, bias, *lbias, dtype, B, H, Nq, Nk, 128, false,
                                       &p.bias_H, &p.bias_B, &p.bias_rows);
    if (r != CUDA_SUCCESS) return cuda_fail(100000 + int(r));
  }
  a.stream = static_cast<cudaStream_t>(stream);
  a.ev_start = g_ev_start;
  a.ev_stop = g_ev_stop;
  return from_cuda(launch_bwd(dtype, d, causal != 0, a));
}

int fa_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO,
           const float* L, void* dQ, void* dK, void* dV, int B, int H, int Nq, int Nk, int d,
           int causal, float scale, int dtype, void* workspace, size_t ws_bytes, void* stream) {
  const fa_layout lq = contiguous_layout(H, Nq, d), lk = contiguous_layout(H, Nk, d);
  return fa_bwd_ex(Q, K, V, O, dO, L, dQ, dK, dV, &lq, &lk, &lk, &lq, &lq, &lq, &lk, &lk, B, H, Nq,
                   Nk, d, causal, scale, dtype, nullptr, nullptr, nullptr, nullptr, workspace,
                   ws_bytes, stream);
}

size_t fa_decode_workspace_bytes(int B, int H, int Nk, int d, int num_splits) {
  if (B <= 0 || H <= 0 || Nk <= 0 || (d != 64 && d != 128) || num_splits < 0) return 0;
  const int BH = B * H;
  int s = num_splits > 0 ? num_splits : decode_auto_splits(BH, Nk);
  s = std::min(s, Nk);
  const int kps = decode_keys_per_split(Nk, s);
  s = (Nk + kps - 1) / kps;
  return round_up(size_t(BH) * s * d * sizeof(float), 256) + round_up(size_t(BH) * s * 4, 256);
}

int fa_decode_ex(const void* Q, const void* K, const void* V, void* O, float* L, int B, int H,
                 int Nk, int d, float scale, int dtype, int num_splits, const int* kv_len,
                 void* workspace, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("fa_decode_ex");
  int st = check_common(B, H, 1, Nk, d, scale, dtype);
  if (st != FA_OK) return st;
  if (dtype == FA_FP32) return FA_ERR_UNSUPPORTED;
  if (num_splits < 0) return FA_ERR_INVALID;
  if (kv_len && (reinterpret_cast<uintptr_t>(kv_len) & 3u)) return FA_ERR_INVALID;
  const void* ptrs[] = {Q, K, V, O, L};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return FA_ERR_INVALID;
  const int BH = B * H;
  int s = num_splits > 0 ? num_splits : decode_auto_splits(BH, Nk);
  s = std::min(s, Nk);
  if (s > 65535 || int64_t(s) * BH > INT32_MAX) return FA_ERR_UNSUPPORTED;  // 1-D grid of (head, part)
  const int kps = decode_keys_per_split(Nk, s);
  s = (Nk + kps - 1) / kps;
  const size_t need = fa_decode_workspace_bytes(B, H, Nk, d, num_splits);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || ws_bytes < need)
    return FA_ERR_WORKSPACE;
  DecodeParams p;
  p.Q = Q; p.K = K; p.V = V; p.O = O; p.L = L;
  p.Opart = static_cast<float*>(workspace);
  p.Lpart = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                     round_up(size_t(BH) * s * d * sizeof(float), 256));
  p.BH = BH;
  p.Nk = Nk;
  p.splits = s;
  p.keys_per_split = kps;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.H = H;
  p.kv_len = kv_len;
  return from_cuda(launch_decode(dtype, d, p, static_cast<cudaStream_t>(stream)));
}

int fa_decode(const void* Q, const void* K, const void* V, void* O, float* L, int B, int H, int Nk,
              int d, float scale, int dtype, int num_splits, void* workspace, size_t ws_bytes,
              void* stream) {
  return fa_decode_ex(Q, K, V, O, L, B, H, Nk, d, scale, dtype, num_splits, nullptr, workspace,
                      ws_bytes, stream);
}

int fa_decode_noalloc(const void* Q, const void* K, const void* V, void* O, float* L, int B, int H,
                      int Nk, int d, float scale, int dtype, int num_splits, void* stream) {
  NvtxRange nvtx_range("fa_decode_noalloc");
  int st = check_common(B, H, 1, Nk, d, scale, dtype);
  if (st != FA_OK) return st;
  if (dtype == FA_FP32) return FA_ERR_UNSUPPORTED;
  if (num_splits < 0) return FA_ERR_INVALID;
  const void* ptrs[] = {Q, K, V, O, L};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return FA_ERR_INVALID;
  const int BH = B * H;
  // Scratch bytes for s parts: partial outputs [BH, s, d] then logsumexps [BH, s].
  auto need_for = [&](int s) {
    return round_up(size_t(BH) * s * d * sizeof(float), 256) + round_up(size_t(BH) * s * 4, 256);
  };
  const size_t cap = decode_scratch_bytes();
  int s = num_splits > 0 ? num_splits : decode_auto_splits(BH, Nk);
  s = std::min(s, Nk);
  if (num_splits == 0)
    while (s > 1 && need_for(s) > cap) --s;  // automatic: fewer parts until they fit
  if (s > 65535 || int64_t(s) * BH > INT32_MAX) return FA_ERR_UNSUPPORTED;  // 1-D grid of (head, part)
  const int kps = decode_keys_per_split(Nk, s);
  s = (Nk + kps - 1) / kps;
  if (need_for(s) > cap) return FA_ERR_WORKSPACE;  // beyond the built-in scratch
  void* scratch = nullptr;
  st = from_cuda(decode_scratch_ptr(&scratch));
  if (st != FA_OK) return st;
  DecodeParams p;
  p.Q = Q; p.K = K; p.V = V; p.O = O; p.L = L;
  p.Opart = static_cast<float*>(scratch);
  p.Lpart = reinterpret_cast<float*>(static_cast<uint8_t*>(scratch) +
                                     round_up(size_t(BH) * s * d * sizeof(float), 256));
  p.BH = BH;
  p.Nk = Nk;
  p.splits = s;
  p.keys_per_split = kps;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.H = H;
  p.kv_len = nullptr;
  return from_cuda(launch_decode(dtype, d, p, static_cast<cudaStream_t>(stream)));
}

int fa_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(int(e));
  int word = 0, site = 0;
  if ((e = take_error_fwd(&word, &site)) != cudaSuccess) return cuda_fail(int(e));
  if ((e = take_error_bwd(&word, &site)) != cudaSuccess) return cuda_fail(int(e));
  if ((e = take_error_decode(&word, &site)) != cudaSuccess) return cuda_fail(int(e));
  if (site != 0) g_last_site = site;
  if (word & 2) return FA_ERR_CUDA;  // a kernel found its shared memory misaligned (kErrLayout)
  if (word & 4) return FA_ERR_BOUNDS;  // a debug build's index check failed (kErrBounds)
  if (word != 0) return FA_ERR_TIMEOUT;
  return FA_OK;
}

int fa_bwd_set_timing_events(void* start, void* stop) {
  if (start && stop) {
    g_ev_start = static_cast<cudaEvent_t>(start);
    g_ev_stop = static_cast<cudaEvent_t>(stop);
  } else {
    g_ev_start = g_ev_stop = nullptr;
  }
  return FA_OK;
}

int fa_last_timeout_site(void) { return g_last_site.load(); }

int fa_last_cuda_error(void) { return g_last_cuda.load(); }

int fa_selftest_wait_timeout(unsigned int limit_us, void* stream) {
  if (limit_us < 1 || limit_us > 1000000) return FA_ERR_INVALID;
  return from_cuda(launch_selftest_wait(1000ull * limit_us, static_cast<cudaStream_t>(stream)));
}

#ifdef FA_DEBUG
const char* fa_version(void) { return "fa-b200 0.1 (sm_100a, debug index checks)"; }
#else
const char* fa_version(void) { return "fa-b200 0.1 (sm_100a)"; }
#endif

}  // extern "C"
