// Split-KV decode (one query row per batch·head) and its logsumexp combine.
//
// FlashAttention V1/V2 study notes (51CTO), section "Sequence Parallel",
// Flash-Decoding paragraph: with a single query row there is no parallelism
// along Q, so the K/V sequence is cut into parts processed by different
// CTAs, each running the forward online softmax over its part; a reduction
// kernel then rescales the parts and adds them.  Each part here stores its
// output already normalised (O_s) together with its natural-log logsumexp
// L_s; the combine computes L = log Σ_s exp(L_s) and O = Σ_s exp(L_s − L) O_s.
//
// Nq = 1 makes this a matrix-vector product per head (about 1 flop per byte
// of K/V), so it runs on the CUDA cores and is bound by HBM bandwidth: every
// K/V byte is read exactly once with 16-byte non-allocating loads, several
// rows in flight per warp.
#define FA_SITE_BASE 30000
#include "common.cuh"
#include "launch.h"

#include <mutex>

namespace fa {

namespace {

constexpr int kDecodeThreads = 256;
constexpr int kUnroll = 4;

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

template <typename T>
__device__ __forceinline__ void to_f8(const uint4& u, float (&f)[8]);
template <>
__device__ __forceinline__ void to_f8<__nv_bfloat16>(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t = ElemTraits<__nv_bfloat16>::unpack2(w[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}
template <>
__device__ __forceinline__ void to_f8<__half>(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t = ElemTraits<__half>::unpack2(w[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

// One CTA per (part, batch·head).  A group of LPK = D/8 lanes owns one key
// row at a time (8 elements per lane); a warp covers 32/LPK keys per load.
template <typename T, int D>
__global__ void __launch_bounds__(kDecodeThreads)
    decode_split_kernel(DecodeParams p) {
  constexpr int LPK = D / 8;                // lanes per key row
  constexpr int KPW = 32 / LPK;             // key rows per warp per load
  constexpr int NW = kDecodeThreads / 32;   // warps
  constexpr int GROUPS = NW * KPW;          // independent softmax states per CTA
  // one CTA per (head, part), parts of a head consecutive (a 1-D grid: B·H
  // may exceed the 65535 of a grid's second dimension)
  const int part = int(blockIdx.x % unsigned(p.splits)), bh = int(blockIdx.x / unsigned(p.splits));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane / LPK, sl = lane % LPK;  // key slot in the warp, lane in the group

  // this part's keys, cut at the batch element's key-padding length (a part
  // past it is empty: L_part = -inf, weight 0 in the combine)
  const int k_begin = part * p.keys_per_split;
  int k_end = min(keys_of(p.kv_len, bh, p.H, p.Nk), k_begin + p.keys_per_split);
  if (!FA_INBOUNDS(part < p.splits && bh < p.BH && (k_end <= k_begin || k_begin < p.Nk))) k_end = k_begin;

  // q slice, pre-multiplied by scale·log2(e) so scores come out in log2 units.
  float q[8];
  {
    const T* qp = reinterpret_cast<const T*>(p.Q) + size_t(bh) * D + sl * 8;
    uint4 u = *reinterpret_cast<const uint4*>(qp);
    to_f8<T>(u, q);
#pragma unroll
    for (int i = 0; i < 8; ++i) q[i] *= p.scale_log2;
  }
  const T* Kh = reinterpret_cast<const T*>(p.K) + size_t(bh) * p.Nk * D + sl * 8;
  const T* Vh = reinterpret_cast<const T*>(p.V) + size_t(bh) * p.Nk * D + sl * 8;

  float m = -INFINITY, l = 0.f, acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;

  // Each iteration the CTA covers NW*KPW*kUnroll consecutive keys.
  const int step = GROUPS * kUnroll;
  for (int base = k_begin; base < k_end; base += step) {
    uint4 ku[kUnroll], vu[kUnroll];
    int key[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      key[u] = base + (u * NW + warp) * KPW + sub;
      const int kk = key[u] < k_end ? key[u] : k_begin;  // clamp: valid address, masked below
      ku[u] = ld_stream(Kh + size_t(kk) * D);
      vu[u] = ld_stream(Vh + size_t(kk) * D);
    }
    float s[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      float kf[8];
      to_f8<T>(ku[u], kf);
      float acc_s = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) acc_s = fmaf(q[i], kf[i], acc_s);
#pragma unroll
      for (int o = LPK / 2; o > 0; o >>= 1) acc_s += __shfl_xor_sync(0xffffffffu, acc_s, o);
      s[u] = key[u] < k_end ? acc_s : -INFINITY;
    }
    float mx = s[0];
#pragma unroll
    for (int u = 1; u < kUnroll; ++u) mx = fmaxf(mx, s[u]);
    const float m_new = fmaxf(m, mx);
    // While a group has seen no key yet (m_new = -inf) it keeps l = 0 and
    // acc = 0: use 0 as the reference so no inf - inf appears.
    const float m_use = m_new == -INFINITY ? 0.f : m_new;
    const float alpha = ex2(m - m_use);
    l *= alpha;
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] *= alpha;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const float pu = ex2(s[u] - m_use);
      l += pu;
      float vf[8];
      to_f8<T>(vu[u], vf);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = fmaf(pu, vf[i], acc[i]);
    }
    m = m_new;
  }

  // Combine the CTA's GROUPS states through shared memory.
  __shared__ float sm_m[GROUPS], sm_l[GROUPS];
  __shared__ float sm_acc[GROUPS][D];
  const int g = warp * KPW + sub;
  if (sl == 0) {
    sm_m[g] = m;
    sm_l[g] = l;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) sm_acc[g][sl * 8 + i] = acc[i];
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += kDecodeThreads) {
    float M = -INFINITY;
    for (int gg = 0; gg < GROUPS; ++gg) M = fmaxf(M, sm_m[gg]);
    float lt = 0.f, o = 0.f;
    if (M != -INFINITY) {
      for (int gg = 0; gg < GROUPS; ++gg) {
        const float w = ex2(sm_m[gg] - M);  // 0 for an empty group
        lt = fmaf(sm_l[gg], w, lt);
        o = fmaf(sm_acc[gg][c], w, o);
      }
    }
    const size_t idx = size_t(bh) * p.splits + part;
    if (!FA_INBOUNDS(part < p.splits && bh < p.BH)) continue;
    p.Opart[idx * D + c] = lt > 0.f ? o / lt : 0.f;
    if (c == 0) p.Lpart[idx] = lt > 0.f ? (M + lg2(lt)) * kLn2 : -INFINITY;
  }
}

// One CTA per batch·head, one thread per output element.
template <typename T, int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(DecodeParams p) {
  const int bh = blockIdx.x, c = threadIdx.x;
  if (!FA_INBOUNDS(bh < p.BH && c < D)) return;
  const float* Lp = p.Lpart + size_t(bh) * p.splits;
  const float* Op = p.Opart + size_t(bh) * p.splits * D;
  float M = -INFINITY;
  for (int s = 0; s < p.splits; ++s) M = fmaxf(M, Lp[s]);
  float out = 0.f, Lrow = -INFINITY;
  if (M != -INFINITY) {
    float sum = 0.f;
    for (int s = 0; s < p.splits; ++s) sum += __expf(Lp[s] - M);
    Lrow = M + __logf(sum);
    for (int s = 0; s < p.splits; ++s) out = fmaf(__expf(Lp[s] - Lrow), Op[size_t(s) * D + c], out);
  }
  T* O = reinterpret_cast<T*>(p.O) + size_t(bh) * D;
  O[c] = ElemTraits<T>::from_float(out);
  if (c == 0) p.L[bh] = Lrow;
}

}  // namespace

template <typename T, int D>
static cudaError_t launch_decode_t(const DecodeParams& p, cudaStream_t s) {
  decode_split_kernel<T, D><<<unsigned(p.splits) * unsigned(p.BH), kDecodeThreads, 0, s>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_combine_kernel<T, D><<<p.BH, D, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_decode(int dtype, int d, const DecodeParams& p, cudaStream_t s) {
  if (dtype == FA_BF16) {
    if (d == 64) return launch_decode_t<__nv_bfloat16, 64>(p, s);
    if (d == 128) return launch_decode_t<__nv_bfloat16, 128>(p, s);
  } else if (dtype == FA_FP16) {
    if (d == 64) return launch_decode_t<__half, 64>(p, s);
    if (d == 128) return launch_decode_t<__half, 128>(p, s);
  }
  return cudaErrorInvalidValue;
}

// ------------------------------------------------------------------
// Scratch of fa_decode_noalloc: the partial outputs and logsumexps of the
// split-KV decode, kept in a device array that belongs to this library
// instead of a workspace the caller allocates.  Every GPU that loads the
// library holds these 8 MiB until the process exits.  All calls on a device
// share the array and it keeps whatever the last call left there; nothing
// in it has to start at zero, because a call writes every partial result
// its combine step reads.  Two calls whose kernels overlap on the GPU (on
// different streams or from different host threads) race on it.
constexpr size_t kDecodeScratchBytes = FA_DECODE_NOALLOC_SCRATCH_BYTES;  // 8 MiB
static __device__ __align__(256) unsigned char g_decode_scratch[kDecodeScratchBytes];

size_t decode_scratch_bytes() { return kDecodeScratchBytes; }

// In host code g_decode_scratch names a host-side stand-in, not device
// memory, so its device address on the current device is looked up with
// cudaGetSymbolAddress, once per device (by the first no-alloc call made
// with that device current), and cached.  The cache is keyed by the unique
// ID of the device's context as well: a cudaDeviceReset (or any other
// teardown of the primary context) reloads the module, possibly at another
// address, and the next call then looks the address up again instead of
// handing the kernels a stale one.
namespace {
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Unique ID of the current context (0 if it cannot be read).
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}
}  // namespace

cudaError_t decode_scratch_ptr(void** out) {
  static std::mutex mu;
  static void* cached[64] = {};
  static unsigned long long cached_ctx[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  // make the device's primary context current (a no-op when it already is),
  // so that its ID can be read
  e = cudaSetDevice(dev);
  if (e != cudaSuccess) return e;
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lk(mu);
  if (cached[dev] == nullptr || ctx == 0 || cached_ctx[dev] != ctx) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_decode_scratch);
    if (e != cudaSuccess) return e;
    cached[dev] = ptr;
    cached_ctx[dev] = ctx;
  }
  *out = cached[dev];
  return cudaSuccess;
}

// Failure-detection self-test: one thread waits, through the same bounded
// wait the kernels use, on an mbarrier that nothing ever arrives at; after
// limit_ns it records a timeout (error word + site) and returns.
__global__ void selftest_wait_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, FA_SITE_BASE + __LINE__, limit_ns);
}

cudaError_t launch_selftest_wait(unsigned long long limit_ns, cudaStream_t stream) {
  selftest_wait_kernel<<<1, 32, 0, stream>>>(limit_ns);
  return cudaGetLastError();
}

FA_ERROR_ACCESSOR(take_error_decode)

}  // namespace fa
