/*
 * fa_b200.h -- C ABI of the exact-attention library for NVIDIA B200 (sm_100a).
 *
 * The operation (every page cites it; the definitions used here):
 *   Standard attention, "YOLO11 ... FlashAttention-2" page, section 1.2, with
 *   the 1/sqrt(d) score factor of that page's section 3.2 and of the LLM
 *   explainer page (aitangshan.cn), section 1:
 *       S = scale * Q K^T,  P = softmax_rows(S),  O = P V,
 *       LSE_i = log(sum_j exp(S_ij))            (natural log, per query row)
 *   computed FlashAttention-2 style (LLM explainer page, sections 4.1-4.3
 *   and 5.2): outer loop over Q tiles, inner loop over K/V tiles, online
 *   softmax with a running max and running sum; S and P never reach global
 *   memory.  The backward pass (same page, section 6.2, recompute strategy)
 *   rebuilds P from Q, K and the saved LSE and returns the textbook gradients
 *   dV = P^T dO, dS = P o (dO V^T - rowsum(dO o O)), dQ = scale dS K,
 *   dK = scale dS^T Q.  Non-causal, no dropout, no bias.
 *
 * Layout and types
 *   q, k, v, o, dout, dq, dk, dv: contiguous [B, N, H, d] device arrays of
 *   16-bit floats (bf16 for the unsuffixed entry points, fp16 for *_f16);
 *   token stride H*d elements, head stride d.  lse: contiguous [B, H, N]
 *   fp32 device array (natural log).  Every pointer must be 16-byte aligned.
 *   d is 64, 96, 128 or 256; B, H, N >= 1; each tensor
 *   holds fewer than 2^31 elements.  scale is any finite float (normally
 *   1/sqrt(d)).  Arithmetic: 16-bit inputs, fp32 accumulation and softmax,
 *   outputs rounded to nearest even.
 *
 * Ownership
 *   The caller allocates and owns every buffer.  Inputs are read only.
 *   fa_fwd writes o and lse; fa_bwd overwrites dq, dk, dv (it does not
 *   accumulate into them).  Scratch memory (split-K/V partial results, the
 *   fp32 dQ accumulator, the rowsum term) is allocated and released by the
 *   library, stream-ordered on `stream`, from a memory pool the library
 *   creates per device (cudaMemPoolCreate, cudaMallocFromPoolAsync,
 *   cudaFreeAsync).  The pool keeps up to 1 GiB of freed scratch mapped
 *   between calls, so that a call after a synchronisation does not map new
 *   device memory; the caller's default memory pool is not touched.
 *
 * Errors and execution
 *   Every call validates its arguments before any launch and returns FA_OK
 *   or a negative FA_ERR_* code; on error no output is touched.  Work is
 *   enqueued on `stream` and runs asynchronously: launch failures are
 *   reported by the return value, faults inside a kernel surface at the
 *   caller's next synchronisation.  Device-side waits are bounded: a wait
 *   that gives up records a code readable with fa_get_device_status() and
 *   the kernel returns instead of hanging.
 */
#ifndef FA_B200_H
#define FA_B200_H

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *cudaStream_t;
typedef struct CUevent_st *cudaEvent_t;

enum fa_status {
    FA_OK = 0,
    FA_ERR_NULL = -1,        /* a required pointer is NULL                      */
    FA_ERR_SHAPE = -2,       /* B, H or N < 1, or a tensor of 2^31+ elements    */
    FA_ERR_HEADDIM = -3,     /* d not supported by this entry point             */
    FA_ERR_ALIGN = -4,       /* a pointer is not 16-byte aligned                */
    FA_ERR_LAUNCH = -5,      /* the CUDA runtime rejected a launch or a call    */
    FA_ERR_NOMEM = -6,       /* scratch allocation failed                       */
    FA_ERR_DEVICE = -7,      /* current device is not compute capability 10.0   */
    FA_ERR_SCALE = -8,       /* scale is NaN or infinite                        */
    FA_ERR_SCRATCH = -9,     /* fa_bwd_noalloc: the problem needs more scratch than
                                its fixed buffer holds                           */
    FA_ERR_FLAGS = -10,      /* *_ex: unknown flag bits                          */
    FA_ERR_DTYPE = -11       /* *_ex: unknown element type                       */
};

/* Element types of the *_ex entry points. */
enum fa_dtype { FA_BF16 = 0, FA_FP16 = 1 };

/*
 * Flags of the *_ex entry points.
 * FA_FLAG_CAUSAL: the causal mask of autoregressive models (LLM explainer
 *   page, section 7.1): query row i attends to key rows j <= i only (the
 *   same position index in Q and K/V), i.e. S_ij = -inf for j > i before the
 *   softmax; the LSE and the gradients are those of the masked problem.
 */
enum fa_flag { FA_FLAG_CAUSAL = 1u };

/*
 * Forward pass, bf16.  Writes o [B,N,H,d] and lse [B,H,N].
 * The LLM explainer page, sections 4.1-4.3 and 5.2.
 */
int fa_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
           int B, int H, int N, int d, float scale, cudaStream_t stream);

/* Forward pass, fp16; otherwise identical to fa_fwd. */
int fa_fwd_f16(const void *q, const void *k, const void *v, void *o, float *lse,
               int B, int H, int N, int d, float scale, cudaStream_t stream);

/*
 * Forward pass with an element type (FA_BF16 / FA_FP16) and flags
 * (FA_FLAG_*; 0 gives exactly fa_fwd / fa_fwd_f16).  Arguments, layout and
 * errors as fa_fwd, plus FA_ERR_DTYPE and FA_ERR_FLAGS.  With FA_FLAG_CAUSAL
 * the K/V tiles wholly above a Q tile's diagonal are skipped.
 */
int fa_fwd_ex(const void *q, const void *k, const void *v, void *o, float *lse,
              int B, int H, int N, int d, float scale, int dtype, unsigned flags,
              cudaStream_t stream);

/*
 * Forward pass on 8-bit inputs.  The pages point this way through the
 * multiplied gains of reduced-precision inputs with FlashAttention-2 (YOLO11
 * page, section 5.3) and 8-bit deployment (YOLO integration page, deployment
 * paragraph).  q, k, v: contiguous [B, N, H, d] device arrays of
 * OCP FP8 E4M3 bytes (1 sign, 4 exponent, 3 mantissa bits, bias 7, no
 * infinities; torch.float8_e4m3fn), each with a per-tensor descale factor:
 * the attention computed is the one of (descale_q q, descale_k k, descale_v v)
 * with `scale`, i.e. S = scale descale_q descale_k q k^T, O = descale_v
 * softmax(S) v.  o: [B, N, H, d] bf16; lse: [B, H, N] fp32, natural log of
 * that S.  d must be 128 (FA_ERR_HEADDIM otherwise); flags as fa_fwd_ex
 * (FA_FLAG_CAUSAL).  Arithmetic: Q K^T and P V on the 8-bit tensor-core path
 * with fp32 accumulation; the softmax in fp32; P is rounded to E4M3 (round
 * to nearest even) before P V, while the row sums use the unrounded values.
 * A non-finite descale, or scale * descale_q * descale_k not finite, gives
 * FA_ERR_SCALE.  Pointers 16-byte aligned; ownership and errors as fa_fwd.
 */
int fa_fwd_fp8(const void *q, const void *k, const void *v, void *o, float *lse,
               int B, int H, int N, int d, float scale, float descale_q,
               float descale_k, float descale_v, unsigned flags, cudaStream_t stream);

/*
 * Backward pass, bf16, by recompute (LLM explainer page, section 6.2).
 * Inputs q, k, v, o (the forward output), dout (upstream gradient of o) and
 * lse (the forward's).  Overwrites dq, dk, dv [B,N,H,d].  d is 64, 96, 128
 * or 256 (d = 64: 128-query inner tiles; d = 96, 128, 256: 64-query inner
 * tiles with dQ produced transposed, since five 128-column accumulators
 * exceed tensor memory; at d = 256 two blocks per key tile each produce one
 * 128-wide half of dQ, dK, dV); other d return FA_ERR_HEADDIM.
 */
int fa_bwd(const void *q, const void *k, const void *v, const void *o,
           const void *dout, const float *lse, void *dq, void *dk, void *dv,
           int B, int H, int N, int d, float scale, cudaStream_t stream);

/* Backward pass, fp16; otherwise identical to fa_bwd. */
int fa_bwd_f16(const void *q, const void *k, const void *v, const void *o,
               const void *dout, const float *lse, void *dq, void *dk, void *dv,
               int B, int H, int N, int d, float scale, cudaStream_t stream);

/*
 * Backward pass with an element type and flags, as fa_fwd_ex.  With
 * FA_FLAG_CAUSAL, o and lse must come from the causal forward (fa_fwd_ex
 * with the same flag); query tiles wholly before a key tile are skipped.
 */
int fa_bwd_ex(const void *q, const void *k, const void *v, const void *o,
              const void *dout, const float *lse, void *dq, void *dk, void *dv,
              int B, int H, int N, int d, float scale, int dtype, unsigned flags,
              cudaStream_t stream);

/*
 * Packed Q, K, V (the YOLOv12 image page's flash_attn_qkvpacked_func input):
 * qkv is one contiguous [B, N, 3, H, d] device array of the element type
 * `dtype` whose slices 0, 1, 2 along the third axis are Q, K, V (token stride
 * 3*H*d).  fa_fwd_qkvpacked writes o [B,N,H,d] and lse [B,H,N] exactly as
 * fa_fwd_ex on the three slices would; fa_bwd_qkvpacked takes o, dout
 * [B,N,H,d] and lse and overwrites dqkv, a [B, N, 3, H, d] array holding dQ,
 * dK, dV in the same slices.  Flags, errors and d as fa_fwd_ex / fa_bwd_ex;
 * each of qkv and dqkv must hold fewer than 2^31 elements.
 */
int fa_fwd_qkvpacked(const void *qkv, void *o, float *lse, int B, int H, int N, int d,
                     float scale, int dtype, unsigned flags, cudaStream_t stream);
int fa_bwd_qkvpacked(const void *qkv, const void *o, const void *dout, const float *lse,
                     void *dqkv, int B, int H, int N, int d, float scale, int dtype,
                     unsigned flags, cudaStream_t stream);

/*
 * Variable-length batches (the YOLOv12 image page's
 * flash_attn_varlen_qkvpacked_func form, unpacked): B sequences of different
 * lengths packed along one token axis of `total` tokens.  q, k, v, o, dout,
 * dq, dk, dv are contiguous [total, H, d] device arrays; lse is [H, total]
 * fp32.  cu_seqlens is a device array of B + 1 int32 with cu_seqlens[0] = 0,
 * non-decreasing, cu_seqlens[B] = total: sequence b is tokens
 * [cu_seqlens[b], cu_seqlens[b+1]), and attention (with FA_FLAG_CAUSAL, the
 * causal mask by position within the sequence) stays inside each sequence.
 * max_seqlen must be at least the longest sequence.  The library does not
 * read cu_seqlens on the host: the kernels clamp each sequence into
 * [0, total) and to max_seqlen tokens, so malformed contents cannot cause an
 * out-of-bounds access (the results are then meaningless).  Rows of tokens
 * that no sequence covers are not written.  Errors as fa_fwd_ex /
 * fa_bwd_ex; FA_ERR_ALIGN if cu_seqlens is not 4-byte aligned.
 */
int fa_fwd_varlen(const void *q, const void *k, const void *v, void *o, float *lse,
                  const int *cu_seqlens, int B, int total, int max_seqlen, int H, int d,
                  float scale, int dtype, unsigned flags, cudaStream_t stream);
int fa_bwd_varlen(const void *q, const void *k, const void *v, const void *o,
                  const void *dout, const float *lse, void *dq, void *dk, void *dv,
                  const int *cu_seqlens, int B, int total, int max_seqlen, int H, int d,
                  float scale, int dtype, unsigned flags, cudaStream_t stream);

/*
 * Host copy of the rule the varlen kernels apply to sequence b: its first
 * token and length after clamping cu_seqlens[b], cu_seqlens[b+1] into
 * [0, total] and to at most max_seqlen tokens.  cu_seqlens_host is host
 * memory here.  Returns FA_OK, FA_ERR_NULL or FA_ERR_SHAPE.
 */
int fa_varlen_bounds(const int *cu_seqlens_host, int b, int max_seqlen, int total, int *tok0,
                     int *len);

/*
 * Backward pass, bf16, for callers that cannot allocate device memory.
 * The pages have no counterpart to this entry point; it exists for hosts
 * such as plugin runtimes with their own static memory plan, code that runs
 * where allocation is forbidden or unsafe, and callers that must not touch
 * the device allocator at all.  fa_bwd needs scratch memory (an fp32 dQ
 * accumulator plus two fp32 vectors per query row) and takes it from a
 * stream-ordered memory pool; this variant computes the same result with the same
 * kernels but takes the scratch from one fixed buffer compiled into the
 * library, so it calls no cudaMalloc, cudaFree or other allocating routine.
 *
 * Arguments, layout, ownership and results are those of fa_bwd, for d = 64
 * only (other d return FA_ERR_HEADDIM).
 * Limit: the scratch needed is B * H * ceil(N/128) * 128 * (4*d + 8) bytes
 * and must not exceed 64 MiB (67,108,864 bytes); larger problems are
 * rejected with FA_ERR_SCRATCH before any launch.  Every GPU that loads the
 * library holds the 64 MiB buffer until the process exits.
 *
 * The first call in a CUDA context looks up the buffer's device address
 * (cudaGetSymbolAddress, with the device current) and keeps it for that
 * context only: the cache is keyed by the context's unique ID (cuCtxGetId),
 * so after cudaDeviceReset, or with another context current, the next call
 * looks the address up again.  Make the first call in a context before any
 * stream capture.  All calls share the one buffer and it keeps the previous call's
 * contents (the part that must start at zero is cleared by every call):
 * calls whose work overlaps on the GPU -- on different streams, or from
 * different host threads without ordering -- race on it and give wrong
 * results.  Order such calls, for example on a single stream.
 */
int fa_bwd_noalloc(const void *q, const void *k, const void *v, const void *o,
                   const void *dout, const float *lse, void *dq, void *dk, void *dv,
                   int B, int H, int N, int d, float scale, cudaStream_t stream);

/*
 * Forward work decomposition (host logic only: no GPU, no CUDA call).
 * Describes how fa_fwd / fa_fwd_f16 split a [B,N,H,d] problem over a device
 * with sm_count SMs, for tests and tuning.  A unit is unit_rows query rows of
 * one (batch, head); with n_split > 1 each unit covers one share of the K/V
 * tiles and a second kernel merges the shares' partial results (exactly, by
 * their log-sum-exps); with balanced = 1 every block takes an equal,
 * contiguous range of (unit, K/V tile) steps, so units are cut into pieces
 * whose partial results the block holding K/V tile 0 merges.
 */
typedef struct fa_fwd_plan {
    int kernel;          /* 1: two 128-row Q tiles a unit, 0: one tile a unit   */
    int unit_rows;       /* query rows per unit (256 or 128)                    */
    int kv_tile_rows;    /* rows per K/V tile (128)                              */
    int n_units;         /* B * H * ceil(N / unit_rows) * n_split               */
    int n_kv_tiles;      /* ceil(N / kv_tile_rows)                              */
    int n_split;         /* K/V shares per unit                                 */
    int grid;            /* blocks launched (at most sm_count)                  */
    int balanced;        /* 1: balanced step ranges (cooperative launch)        */
    long long scratch_bytes; /* device scratch the call allocates               */
} fa_fwd_plan_t;

/*
 * Fills *plan.  Returns FA_OK, FA_ERR_NULL, FA_ERR_SHAPE (B, H, N or
 * sm_count below 1) or FA_ERR_HEADDIM.
 */
int fa_fwd_plan(int B, int H, int N, int d, int sm_count, fa_fwd_plan_t *plan);

/* fa_fwd_plan for fa_fwd_ex with the given flags (FA_ERR_FLAGS on unknown bits).
 * Causal units cover only the K/V tiles up to their diagonal, are never cut
 * or split, and are walked longest first. */
int fa_fwd_plan_ex(int B, int H, int N, int d, unsigned flags, int sm_count,
                   fa_fwd_plan_t *plan);

/*
 * Host-only description of the backward's decomposition for a fixed-length
 * batch on a device with sm_count SMs: *n_split blocks per 128-key tile
 * (each takes an equal share of the tile's query tiles, and an extra kernel
 * sums their fp32 dK, dV partials) and *grid_blocks blocks in all.  The split
 * is used only without FA_FLAG_CAUSAL, when it fills the waves of
 * one-block-per-SM launches clearly better (at least 8 query tiles a block).
 * At d = 256 the grid has two blocks per key tile (one per half of d) and no
 * split.  Returns FA_OK, FA_ERR_NULL, FA_ERR_FLAGS, FA_ERR_SHAPE or
 * FA_ERR_HEADDIM (d other than 64, 96, 128, 256).
 */
int fa_bwd_plan(int B, int H, int N, int d, unsigned flags, int sm_count, int *n_split,
                int *grid_blocks);

/*
 * The pieces block `block` (0 <= block < plan.grid) processes, in order,
 * 6 ints each: unit index, first K/V tile, end K/V tile, store kind
 * (0: whole result, 1: partial rows to the block's slot, 2: merge with the
 * partial rows of blocks first_peer .. first_peer + n_peers - 1), first_peer,
 * n_peers.  Writes at most max_pieces pieces and returns the number the block
 * has (>= 0), or a negative FA_ERR_* code.  The same code decides the pieces
 * inside the kernel.
 */
int fa_fwd_plan_pieces(int B, int H, int N, int d, int sm_count, int block, int *pieces,
                       int max_pieces);

/* fa_fwd_plan_pieces for fa_fwd_ex with the given flags. */
int fa_fwd_plan_pieces_ex(int B, int H, int N, int d, unsigned flags, int sm_count, int block,
                          int *pieces, int max_pieces);

/* Static description of a status code.  Never NULL. */
const char *fa_status_string(int status);

/*
 * Reads the device-side status word of the current device (0 = no kernel
 * of this library gave up a bounded wait since the last clear).  Synchronises
 * the device.  If clear is non-zero the word is reset to 0.  Returns FA_OK or
 * FA_ERR_LAUNCH.
 */
int fa_get_device_status(unsigned long long *status_out, int clear);

/*
 * Self-test of the bounded-wait path: launches one block that waits on a
 * barrier nothing will complete, with the given limit in microseconds
 * (1..10,000,000).  The kernel gives up, records a status and returns; the
 * call synchronises and writes the recorded status to *status_out (non-zero
 * when the wait gave up as designed).  Leaves the device usable.
 */
int fa_selftest_bounded_wait(unsigned int limit_us, unsigned long long *status_out);

/*
 * Diagnostic: y[i] = 2^x[i] for n device floats (n >= 1), computed by the
 * FMA-pipe exponential that the forward softmax uses for part of each row's
 * columns instead of the hardware ex2 (range reduction x = n + f, |f| <= 1/2,
 * and a degree-3 polynomial for 2^f; relative error below 1e-4 for
 * -125 <= x <= 127; inputs below -125 give about 2^-125).  Enqueued on
 * `stream`; returns FA_OK, FA_ERR_NULL, FA_ERR_SHAPE or a launch error.
 */
int fa_selftest_exp2(const float *x, float *y, int n, cudaStream_t stream);

/*
 * Instrumentation for benchmarks.  Arms CUDA events that the library records
 * on the launching stream immediately before and immediately after the main
 * kernel (fa_fwd_kernel / fa_bwd_kernel) of the next forward / backward call.
 * Each armed pair is used once and then disarmed; pass NULL to leave a pair
 * unarmed.  The events stay owned by the caller.  Process-wide, not tied to a
 * thread.  Always returns FA_OK.
 */
int fa_set_kernel_events(cudaEvent_t fwd_start, cudaEvent_t fwd_stop,
                         cudaEvent_t bwd_start, cudaEvent_t bwd_stop);

/* Number of kernel launches this library has issued since it was loaded. */
unsigned long long fa_kernel_launches(void);

/*
 * Number of scratch allocations this library has requested from its memory
 * pool since it was loaded (one per forward call that needs split-K/V or
 * balanced-schedule partials, one per backward call; fa_bwd_noalloc makes
 * none).  Diagnostic only.
 */
unsigned long long fa_scratch_allocs(void);

/*
 * The cudaError_t value behind the most recent FA_ERR_LAUNCH returned by any
 * call of this library in the process (0 if none).  Diagnostic only.
 */
int fa_last_cuda_error(void);

/* Library version, major*10000 + minor*100 + patch. */
int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_H */
