/*
 * fa.h — C ABI of the B200 (sm_100a) fused exact-attention library.
 *
 * The library computes exact scaled-dot-product attention
 *     O = softmax(scale · Q Kᵀ [+ causal mask]) V
 * fused into tiled kernels with an online softmax, and its gradient.
 *
 *   FlashAttention1 post (CSDN), section "具体算法": S = Q Kᵀ, P = softmax(S),
 *     O = P V, computed block by block with a running row maximum and a
 *     running denominator so that S and P never reach device memory.
 *   FlashAttention V1/V2 study notes (51CTO), section "算法的改进": the
 *     forward writes the row logsumexp L once; the backward rebuilds P from
 *     L instead of storing it.  Causal: blocks wholly above the diagonal are
 *     skipped, only the diagonal block is masked.
 *   Same notes, section "Sequence Parallel": the backward runs one K/V block
 *     per CTA and reduces dQ across CTAs; Flash-Decoding splits K/V of a
 *     single query across CTAs and combines the parts by their logsumexp.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor arguments are DEVICE pointers to contiguous row-major arrays
 *    allocated and owned by the caller.  The library never allocates device
 *    memory on these paths and never synchronises (except fa_status).
 *  - Q, O, dO, dQ: [B, H, Nq, d];  K, V, dK, dV: [B, H, Nk, d];  L, D: [B, H, Nq]
 *    (d fastest).  Element type of Q/K/V/O/dO/dQ/dK/dV is `dtype`; L is
 *    always float32 and holds the NATURAL-log logsumexp of the scaled,
 *    masked scores of each query row.
 *  - Every pointer must be 16-byte aligned.
 *  - causal != 0 uses bottom-right alignment: key j is visible to query i iff
 *    j <= i + (Nk - Nq).  Causal requires Nq <= Nk, so no row is empty.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Work is
 *    enqueued on it and the call returns without waiting.
 *  - Supported: d in {64, 128}; dtype FA_BF16 or FA_FP16 for every d, FA_FP32
 *    (computed with TF32 tensor-core products and fp32 softmax) for d = 64.
 *  - Return value: FA_OK, or a negative fa_status_t detected synchronously
 *    before anything is enqueued (invalid arguments, unsupported shape,
 *    workspace too small) or at launch (FA_ERR_CUDA).  Faults and bounded-
 *    wait timeouts inside kernels are reported later by fa_status().
 */
#ifndef FA_B200_H_
#define FA_B200_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { FA_FP32 = 0, FA_BF16 = 1, FA_FP16 = 2 } fa_dtype;

/* Size of the device scratch array that fa_decode_noalloc uses (below). */
#define FA_DECODE_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID = -1,     /* null pointer, size <= 0, non-finite scale, misaligned pointer */
  FA_ERR_UNSUPPORTED = -2, /* d not in {64,128}, fp32 with d=128, causal with Nq > Nk,
                              B or H > 65535, a grid of more than 2^31 - 1 blocks */
  FA_ERR_WORKSPACE = -3,   /* workspace pointer null or smaller than the query says */
  FA_ERR_CUDA = -4,        /* a CUDA runtime error at launch or in fa_status */
  FA_ERR_TIMEOUT = -5,     /* a kernel's bounded wait expired (reported by fa_status) */
  FA_ERR_BOUNDS = -6       /* debug builds only: a kernel index check failed (reported by
                              fa_status; the access was skipped) */
} fa_status_t;

/* Forward.  Writes O [B,H,Nq,d] (dtype) and L [B,H,Nq] (float32, natural
 * log).  FlashAttention V1/V2 study notes (51CTO), sections "算法的改进" and
 * "Thread Block Level 并行": one CTA per block of query rows, the K/V
 * sequence streamed through shared memory, O and L written once. */
int fa_fwd(const void* Q, const void* K, const void* V, void* O, float* L, int B, int H, int Nq,
           int Nk, int d, int causal, float scale, int dtype, void* stream);

/* Element strides of one attention tensor viewed as [B, H, N, d], the d
 * elements of a row contiguous: b between batches, h between heads, n between
 * rows.  A contiguous [B, H, N, d] tensor has {H·N·d, N·d, d}; a [B, N, H, d]
 * tensor (sequence before head) has {N·H·d, d, H·d}.  Each stride times the
 * element size must be a non-negative multiple of 16 bytes.  The 51CTO notes,
 * section "Sequence Parallel": the backward kernel shown there takes a batch,
 * head, row and column stride for every tensor it touches. */
typedef struct {
  long long b, h, n;
} fa_layout;

/* Dropout of the attention weights.  The study notes on FlashAttention V1/V2
 * (51CTO), section "算法的改进", mention the dropout steps of the V1
 * algorithm; the library applies them to the normalised weights:
 * O = (P ∘ Z · 256/T) V with Z a 0/1 keep mask, while L stays the logsumexp
 * of the undropped scores.  The keep threshold is T = round((1 − p)·256)
 * (computed in double from the float p), so a weight survives with
 * probability T/256.  Z is drawn inside the kernels by the counter-based
 * generator Philox4x32-10 (Salmon et al., "Parallel Random Numbers: As Easy
 * as 1, 2, 3", SC'11): 4×4 blocks of the [Nq, Nk] weights of head index
 * bh = b·H + h, block (query rows 4r.., keys 4c..) from counter
 * (c, r, bh, offset) and key (seed low word, seed high word); word i of the
 * output belongs to query row 4r + i and byte j of that word (least
 * significant first) to key 4c + j; a weight is kept iff its byte is below T.
 * The backward redraws the same Z from the same seed and offset, so the two
 * calls must get the same fa_dropout. */
typedef struct {
  float p;                 /* probability of dropping a weight, in [0, 1); 0 = none */
  unsigned long long seed; /* generator key */
  unsigned int offset;     /* counter word 3: a separate stream per call */
} fa_dropout;

/* Additive bias (`bias`, `lbias`, for fa_fwd_ex and fa_bwd_ex): NULL, or a
 * device tensor of the input dtype viewed as [B, H, Nq, Nk] through the
 * element strides in `lbias` {b, h, n} (row = query; key columns contiguous;
 * a stride of 0 broadcasts over batches or heads).  It is added to the
 * scaled scores before the masks and the softmax, S' = scale·Q Kᵀ + bias,
 * in natural-log units (-inf hides a key), and L is the logsumexp of S'.
 * The 51CTO notes' background list names adding a bias as the first change
 * one writes one's own kernel for.  The bias is an input constant: the
 * backward rebuilds P with it and returns no gradient for it.  The pointer
 * must be 16-byte aligned and each stride a non-negative multiple of 16
 * bytes (rows padded to a multiple of 8 keys), else FA_ERR_INVALID; fp32 has
 * no bias (FA_ERR_UNSUPPORTED).
 *
 * Key padding (`kv_len`, for fa_fwd_ex and fa_bwd_ex): NULL, or a DEVICE
 * array of B int32 lengths; batch element b then sees only keys
 * j < kv_len[b] (values are clamped to [0, Nk] on the device).  It is the
 * additive 0 / -inf mask of batched sequences padded to Nk, ANDed with the
 * causal mask, whose bottom-right alignment still uses the full Nq and Nk.
 * The FlashAttention1 post (CSDN), section "引言/动机", lists the fused chain
 * as matmul, scale, mask, softmax: the mask acts on the scaled scores before
 * the softmax.  A row that sees no key gets O = 0 and L = -inf; keys past
 * the length get dK = dV = 0.  The pointer must be 4-byte aligned
 * (FA_ERR_INVALID); fp32 has no key padding (FA_ERR_UNSUPPORTED).
 *
 * fa_fwd for tensors with arbitrary strides (one fa_layout each for Q, K, V
 * and O; L stays contiguous [B, H, Nq]), optional dropout (NULL or p = 0:
 * none), optional key padding and an optional additive bias (both above).
 * fa_fwd is this call with contiguous layouts, no dropout, no padding and
 * no bias.
 * Layout errors and a dropout probability outside [0, 1) (or one that keeps
 * nothing after rounding): FA_ERR_INVALID; a non-contiguous fp32 tensor or
 * fp32 with dropout: FA_ERR_UNSUPPORTED (the fp32 path reads contiguous
 * tensors and has no dropout). */
int fa_fwd_ex(const void* Q, const void* K, const void* V, void* O, float* L, const fa_layout* lq,
              const fa_layout* lk, const fa_layout* lv, const fa_layout* lo, int B, int H, int Nq,
              int Nk, int d, int causal, float scale, int dtype, const fa_dropout* dropout,
              const int* kv_len, const void* bias, const fa_layout* lbias, void* stream);

/* Bytes of device workspace fa_bwd needs for this problem (0 on invalid
 * arguments).  The workspace holds D = rowsum(dO ∘ O) [B,H,Nq] and the fp32
 * dQ accumulator; its contents on entry do not matter. */
size_t fa_bwd_workspace_bytes(int B, int H, int Nq, int Nk, int d, int dtype);

/* Backward.  Given the forward's inputs, its O and L, and dO, writes dQ, dK,
 * dV (dtype, shapes of Q, K, V).  Recomputes P = exp(scale·S − L) block by
 * block (the N×N matrix is never stored), D = rowsum(dO ∘ O) first.  The
 * 51CTO notes, sections "算法的改进" and "Sequence Parallel".  `workspace`
 * must hold fa_bwd_workspace_bytes(...) bytes, 256-byte aligned. */
int fa_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO,
           const float* L, void* dQ, void* dK, void* dV, int B, int H, int Nq, int Nk, int d,
           int causal, float scale, int dtype, void* workspace, size_t ws_bytes, void* stream);

/* fa_bwd for tensors with arbitrary strides (layouts of Q, K, V, O, dO, dQ,
 * dK, dV in that order; L stays contiguous), the forward's dropout (the
 * same fa_dropout as the forward call, or NULL), its key padding and its
 * bias (P is rebuilt with the bias; no bias gradient is returned).  With dropout the gradient
 * is the exact one for the drawn Z: dV = (P ∘ Z · s)ᵀ dO,
 * dP = (dO Vᵀ) ∘ Z · s, dS = P ∘ (dP − D), s = 256/T.  fa_bwd is this call
 * with contiguous layouts, no dropout, no padding and no bias.  Errors as
 * for fa_fwd_ex and fa_bwd. */
int fa_bwd_ex(const void* Q, const void* K, const void* V, const void* O, const void* dO,
              const float* L, void* dQ, void* dK, void* dV, const fa_layout* lq,
              const fa_layout* lk, const fa_layout* lv, const fa_layout* lo, const fa_layout* ldo,
              const fa_layout* ldq, const fa_layout* ldk, const fa_layout* ldv, int B, int H,
              int Nq, int Nk, int d, int causal, float scale, int dtype, const fa_dropout* dropout,
              const int* kv_len, const void* bias, const fa_layout* lbias, void* workspace,
              size_t ws_bytes, void* stream);

/* How fa_bwd reduces the dQ contributions of the different K/V blocks:
 *   0 = automatic (the measured faster strategy for the shape),
 *   1 = fp32 reductions (red.add) into one accumulator,
 *   2 = one fp32 partial buffer per K/V block, then a reduction kernel,
 *   3 = fp32 reductions into G accumulators, K/V block kb adding into
 *       accumulator kb mod G (G from fa_set_bwd_dq_groups), then the same
 *       reduction kernel over the G buffers.
 * The 51CTO notes, section "Sequence Parallel", describe 1 and 2, and mode 3
 * is their compromise (partial buffers shared by groups of K/V blocks, with
 * atomic adds inside a group).  The workspace grows with the buffers: ×1, ×
 * the K/V block count, ×G.  Returns the previous mode, or FA_ERR_INVALID for
 * an unknown mode.  Process-wide; fa_bwd_workspace_bytes follows it. */
int fa_set_bwd_dq_mode(int mode);

/* G, the accumulator count of dQ mode 3 (1 to 16; 4 initially).  Returns
 * the previous G, or FA_ERR_INVALID outside 1..16.  Process-wide. */
int fa_set_bwd_dq_groups(int groups);

/* Bytes of workspace fa_decode needs for `num_splits` parts (0 = the count
 * fa_decode would choose itself). */
size_t fa_decode_workspace_bytes(int B, int H, int Nk, int d, int num_splits);

/* Split-KV decode forward for one query row per (batch, head):
 * Q [B,H,1,d], K,V [B,H,Nk,d] -> O [B,H,1,d] (dtype), L [B,H,1] (float32).
 * No mask.  Each of `num_splits` parts (0 = automatic) runs the online
 * softmax over its slice of K/V and writes a normalised partial output and
 * its logsumexp; a combine kernel then rescales and adds them
 * (the 51CTO notes, Flash-Decoding paragraph of "Sequence Parallel"). */
int fa_decode(const void* Q, const void* K, const void* V, void* O, float* L, int B, int H, int Nk,
              int d, float scale, int dtype, int num_splits, void* workspace, size_t ws_bytes,
              void* stream);

/* fa_decode with key padding: `kv_len` is NULL or a DEVICE array of B int32
 * lengths (4-byte aligned), and the query of batch element b attends to keys
 * j < kv_len[b] only (clamped to [0, Nk]): a KV cache whose sequences are
 * padded to Nk.  Parts past a length are empty and get weight 0 in the
 * combine; a length of 0 gives O = 0 and L = -inf.  The mask acts on the
 * scaled scores before the softmax (the FlashAttention1 post (CSDN),
 * section "引言/动机": matmul, scale, mask, softmax).  The workspace is
 * fa_decode's. */
int fa_decode_ex(const void* Q, const void* K, const void* V, void* O, float* L, int B, int H,
                 int Nk, int d, float scale, int dtype, int num_splits, const int* kv_len,
                 void* workspace, size_t ws_bytes, void* stream);

/* fa_decode_noalloc: the split-KV decode of fa_decode for callers that
 * cannot allocate device memory.  The pages have no counterpart for it.
 *
 * Some callers own every byte of device memory themselves and hand a
 * library only its input and output buffers: a plugin or runtime whose
 * interface has no way to pass a workspace, or a service whose device
 * memory is fixed once it has started.  They cannot provide fa_decode's
 * workspace and must not call cudaMalloc.  This entry point needs no
 * workspace: the per-part partial outputs and logsumexps go to a scratch
 * array that the library itself holds in device memory (a file-scope
 * __device__ array of FA_DECODE_NOALLOC_SCRATCH_BYTES = 8 MiB, present on
 * every GPU that loads the library until the process exits).  It calls no
 * cudaMalloc, cudaFree or allocating library routine.
 *
 * Arguments and results are those of fa_decode without the workspace.  The
 * scratch needed is about B*H*num_splits*(d+1)*4 bytes: with num_splits = 0
 * the number of parts is reduced until it fits; FA_ERR_WORKSPACE is returned,
 * before anything is enqueued, when an explicit num_splits does not fit or
 * when even one part per (batch, head) does not (B*H*(d+1)*4 bytes above the
 * 8 MiB, i.e. B*H above about 16000 at d = 128).
 *
 * The first call on each device looks up the array's device address (with
 * that device current) and caches it; make that first call before any
 * stream capture.  The cache remembers the device's context too: after a
 * cudaDeviceReset the next call looks the address up again (in the new
 * context) rather than reusing the old one.  All calls share the one array and it keeps the last
 * call's contents (nothing in it needs to start at zero); calls whose
 * kernels overlap on the GPU, on different streams or host threads, race on
 * it and must be serialised by the caller. */
int fa_decode_noalloc(const void* Q, const void* K, const void* V, void* O, float* L, int B, int H,
                      int Nk, int d, float scale, int dtype, int num_splits, void* stream);

/* Synchronises `stream`, then returns and clears the device error word:
 * FA_OK, FA_ERR_TIMEOUT if a kernel's bounded wait expired, FA_ERR_CUDA if
 * the stream reports a CUDA error or a kernel found its shared memory
 * misaligned (it then did nothing), and, in a library built with FA_DEBUG,
 * FA_ERR_BOUNDS if a kernel found an index outside its buffer (the access
 * was skipped; fa_last_timeout_site names the check).  The debug build
 * (libfa_b200_debug.so, same ABI) checks every plain global access and TMA
 * coordinate of the kernels against the buffer it addresses, in place of a
 * memory checker. */
int fa_status(void* stream);

/* Diagnostic: identifies the first kernel wait that timed out (or, in a
 * debug build, the first failed index check) among those fa_status has
 * reported (10000 + line in the forward kernel file, 20000 + line in the
 * backward file, 30000 + line in the decode file); 0 if none has.  No
 * counterpart on the pages. */
int fa_last_timeout_site(void);

/* Diagnostic: the CUDA error behind the most recent FA_ERR_CUDA of any call
 * (a cudaError_t value, or 100000 + the CUresult of a failed tensor-map
 * encoding); 0 if no call has returned FA_ERR_CUDA.  Process-wide. */
int fa_last_cuda_error(void);

/* Measurement hook (no counterpart on the pages, which only say to profile
 * kernels with Nsight Compute, 51CTO notes, section "FlashAttention V2相比V1有
 * 哪些改进").  When both are non-NULL, every later fa_bwd call records the
 * cudaEvent_t `start` on its stream just before the main backward kernel and
 * `stop` just after it, so callers can time that kernel alone with
 * cudaEventElapsedTime.  The events are created and owned by the caller.
 * Pass NULLs to switch it off.  Process-wide; returns FA_OK. */
int fa_bwd_set_timing_events(void* start, void* stop);

/* Failure-detection self-test (no counterpart on the pages).  Enqueues on
 * `stream` one thread that waits, through the kernels' own bounded wait, on
 * a barrier nothing arrives at, for `limit_us` microseconds (1..1000000),
 * then records a timeout as any kernel wait would: the next fa_status
 * returns FA_ERR_TIMEOUT and fa_last_timeout_site names that wait (30000 +
 * line).  Nothing faults or traps; the context stays usable.  Returns
 * FA_ERR_INVALID for a limit out of range, else FA_OK (FA_ERR_CUDA if the
 * launch fails). */
int fa_selftest_wait_timeout(unsigned int limit_us, void* stream);

/* Library version string (static storage). */
const char* fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_H_ */
