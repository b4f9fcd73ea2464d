/*
 * flce.h -- C ABI of a fused linear cross-entropy (FLCE) for NVIDIA B200
 * (sm_100a): the LM-head projection, an optional logit softcap, log-softmax
 * cross-entropy against integer labels with ignore_index, 'sum' / 'mean'
 * reduction with the num_tokens contract, forward and backward, without ever
 * writing the [tokens, vocab] logits to device memory.
 *
 * What is computed (one row i per token, N rows, vocabulary V, hidden H):
 *   Z    = hidden . weight^T                       (LM-head projection; weight is
 *                                                   [vocab, hidden]: NeMo AutoModel
 *                                                   linear_ce API, forward(lm_weight))
 *   L    = softcap * tanh(Z / softcap), or L = Z when softcap == 0
 *                                                  (modelscope/twinkle PR #335,
 *                                                   "PR information" item 3; NeMo
 *                                                   logit_softcapping=0 means off)
 *   lse_i = log sum_v exp(L_iv)
 *   loss_i = lse_i - L_i,y_i for rows with y_i != ignore_index, else 0
 *                                                  (F.cross_entropy semantics:
 *                                                   modelscope/twinkle PR #335,
 *                                                   "Experiment results")
 *   n     = #rows with y_i != ignore_index (a label outside [0, V) is an error,
 *           reported asynchronously; its row is treated as ignored)
 *   'sum'  -> loss = sum_i loss_i,             num_tokens = n
 *   'mean' -> loss = sum_i loss_i / max(n, 1), num_tokens = 0
 *                                                  (modelscope/twinkle PR #335,
 *                                                   item 1; the max(n, 1) clamp that
 *                                                   makes an all-ignored batch give 0,
 *                                                   never NaN: inclusionAI/
 *                                                   Ling-3.1-flash discussion #7)
 * The loss, lse and every stored intermediate are float32 (Modalities PR #464,
 * "The problem": the stored tensors and the returned scalar must not be bf16);
 * the loss sum is accumulated in float64.
 *
 * Backward (textbook derivative of the above):
 *   g     = grad_output * grad_scale * ('mean' ? 1 / max(n, 1) : 1)
 *   dZ_iv = g * (exp(L_iv - lse_i) - [v == y_i]) * (softcap > 0 ? 1 - (L_iv/softcap)^2 : 1),
 *           0 on ignored rows
 *   d_hidden = dZ . weight        [N, H] float32 or bf16, overwritten or accumulated
 *   d_weight = dZ^T . hidden      [V, H] float32 or bf16, overwritten or accumulated
 * grad_scale is the caller's micro-batch / token-count weighting
 * (modelscope/twinkle PR #335, item 2: 1.0 for 'sum' per micro-batch; the
 * trainer divides a 'sum' loss's gradient by the global non-padding token
 * count, NeMo AutoModel forward(num_label_tokens)).
 *
 * Conventions shared by every call:
 *  - All tensor arguments are DEVICE pointers on the current CUDA device,
 *    row-major and densely packed, 16-byte aligned (torch allocations are).
 *    hidden is [N, H], weight is [V, H], labels is int64 [N].
 *  - dtype FLCE_BF16: hidden/weight hold bfloat16; the tensor-core path runs.
 *    H must be a multiple of 8 (16-byte rows for the TMA engine).
 *    dtype FLCE_FP32: hidden/weight hold float32; a CUDA-core path runs
 *    (a correctness path for small problems, not tuned).
 *  - stream is a cudaStream_t (NULL = legacy default stream).  Every call is
 *    asynchronous on that stream and returns after enqueueing its kernels,
 *    without synchronising, so flce_forward and flce_backward may be captured
 *    into a CUDA graph (after one uncaptured call with the same shapes, which
 *    sets the kernels' shared-memory attributes) and replayed with the inputs
 *    updated in place; flce_get_status synchronises and must stay outside.
 *  - The caller owns every buffer, including the workspace (at least
 *    flce_workspace_bytes(...) bytes, 256-byte aligned).  The library does not
 *    allocate device memory and keeps no per-call state.  Calls that share a
 *    workspace must be ordered on one stream.
 *  - Return value: argument and launch errors are reported synchronously.
 *    Errors found by the kernels (a label outside [0, V) that is not
 *    ignore_index, a pipeline wait that ran out of time) are recorded in a
 *    status word inside the workspace.  flce_forward and flce_backward clear
 *    it first, so flce_get_status() (which synchronises the stream) returns
 *    the errors of the latest call on that workspace.  Nothing aborts or traps.
 */
#ifndef FLCE_H
#define FLCE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum flce_status {
  FLCE_OK = 0,
  FLCE_ERR_ARG = 1,          /* null pointer, bad enum, negative softcap, misaligned pointer */
  FLCE_ERR_SHAPE = 2,        /* N < 0, V < 1, H < 8, H % 8 != 0 (bf16), sizes too large */
  FLCE_ERR_LABEL_RANGE = 3,  /* (async) a label outside [0, V) that is not ignore_index */
  FLCE_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed */
  FLCE_ERR_UNSUPPORTED = 5,  /* device is not sm_100 */
  FLCE_ERR_TIMEOUT = 6,      /* (async) a bounded pipeline wait inside a kernel ran out */
  FLCE_ERR_WORKSPACE = 7     /* workspace smaller than flce_workspace_bytes() */
} flce_status;

typedef enum flce_reduction { FLCE_SUM = 0, FLCE_MEAN = 1 } flce_reduction;

typedef enum flce_dtype { FLCE_BF16 = 0, FLCE_FP32 = 1 } flce_dtype;

/* Library options (flce_set_option).  They are process-wide, apply to every
 * device, and keep their value until set again; every call reads them once,
 * when it starts.  None changes the result beyond fp32 summation order: they
 * select between equivalent schedules (for measurements and tests) and set
 * limits.  Nothing else (no environment variable) changes what the library
 * runs.  Defaults in brackets. */
typedef enum flce_option {
  FLCE_OPT_CTA_GROUP = 0,       /* [2] tensor-core tiles of CTA pairs (256 rows); 1: single CTAs (128 rows) */
  FLCE_OPT_BWD_COMPACT = 1,     /* [1] the backward leaves ignored rows out of its GEMMs; 0: keeps every row
                                   (and then also skips the exact fp32 label-term correction) */
  FLCE_OPT_BWD_FUSE = 2,        /* [1] dHidden and dWeight GEMMs of a backward chunk share one launch; 0: two */
  FLCE_OPT_MN3D = 3,            /* [1] MN-major operands load through 3-D chunk views; 0: 2-D views */
  FLCE_OPT_CHUNK_TOKENS = 4,    /* [16384] token rows of a backward chunk (256 .. 2^20, rounded up to 256) */
  FLCE_OPT_CHUNK_VOCAB = 5,     /* [16384] vocab columns of a backward chunk (256 .. 2^20, rounded up to 256);
                                   the dZ block of the workspace is chunk_tokens x chunk_vocab bf16 and,
                                   with FLCE_OPT_BWD_COMPACT, a compact-order dHidden block chunk_tokens x H
                                   fp32 follows it, so flce_workspace_bytes must be called with the same
                                   chunk and compaction options as the calls that use the workspace */
  FLCE_OPT_WAIT_TIMEOUT_MS = 6, /* [1000] limit of every bounded wait inside a kernel (10 .. 60000) */
  FLCE_OPT_GRAD_TILE_N = 7,     /* [512] columns of a dHidden / dWeight tile: 512 or 256 (512 needs CTA pairs;
                                   with FLCE_OPT_CTA_GROUP = 1 tiles are 256 wide) */
  FLCE_OPT_DZ_TILE_N = 8,       /* [0] columns of a backward dZ tile: 256 or 512 (as above); 0: 512
                                   without softcap, 256 with softcap */
  FLCE_OPT_FWD_TILE_N = 9,      /* [512] columns of a forward tile: 512 or 256 (as above) */
  FLCE_OPT_FWD_GROUP_M = 10,    /* [16] row tiles per raster group of the forward GEMM (1 .. 64): the
                                   group's hidden rows stay in L2 while the weight streams past */
  FLCE_OPT_DZ_GROUP_M = 11,     /* [16] the same for the backward dZ GEMM */
  FLCE_OPT_GRAD_GROUP_M = 12,   /* [8] the same for the dHidden / dWeight GEMMs */
  FLCE_OPT_FWD_DYNAMIC = 13,    /* [1] forward tiles are handed out by an atomic counter; 0: round-robin */
  FLCE_OPT_DZ_BUFFERS = 14,     /* [1] backward dZ blocks in the workspace: 1, or 2 (each chunk's dZ GEMM
                                   then runs beside the previous chunk's gradient GEMMs) */
  FLCE_OPT_FWD_COMPACT = 15,    /* [1] the bf16 forward compacts the rows that take part in the loss and
                                   runs its GEMM on those alone; 0: on every row (same results) */
  FLCE_OPT_COUNT_ = 16          /* number of options (not an option) */
} flce_option;

/* Set option `option` to `value`.  FLCE_ERR_ARG for an unknown option or a
 * value outside its range; the option is then unchanged. */
flce_status flce_set_option(int32_t option, int64_t value);

/* Current value of `option` into *value.  FLCE_ERR_ARG for an unknown option
 * or a NULL value. */
flce_status flce_get_option(int32_t option, int64_t* value);

/* Bytes of workspace that flce_forward / flce_backward need for this shape.
 * Returns 0 for invalid sizes.  Pure host computation. */
size_t flce_workspace_bytes(int64_t N, int64_t H, int64_t V, int32_t dtype);

/* The same for a flce_backward call with these flags: FLCE_DHIDDEN_BF16 and
 * FLCE_DWEIGHT_BF16 add fp32 scratch for the gradient before its single
 * rounding (4*N*H and 4*V*H bytes).  Returns 0 for invalid sizes or flags. */
size_t flce_workspace_bytes_ex(int64_t N, int64_t H, int64_t V, int32_t dtype, int32_t flags);

/* Forward.
 *   loss        device float[1]   'sum' or 'mean' loss (float32)
 *   num_tokens  device int64[1]   n for 'sum', 0 for 'mean'
 *   lse         device float[N]   log-sum-exp of every row that takes part in the loss;
 *                                 0 for a row whose label is ignore_index (or outside
 *                                 [0, V)): neither the loss nor its gradient depends on
 *                                 those rows, so their logits are not computed.
 *                                 flce_backward reads it.
 * ignore_index may be any int64; a row is ignored iff labels[i] == ignore_index.
 * softcap must be >= 0 (0 = off).  The async status word is cleared first. */
flce_status flce_forward(const void* hidden, const void* weight, const int64_t* labels,
                         int64_t N, int64_t H, int64_t V, int64_t ignore_index, float softcap,
                         int32_t reduction, int32_t dtype, float* loss, int64_t* num_tokens,
                         float* lse, void* workspace, size_t workspace_bytes, void* stream);

/* flce_forward with the returned loss multiplied by loss_scale (applied in
 * float64 before the single rounding to float32; num_tokens and lse are
 * unchanged).  loss_scale = 1 / n_global normalises a 'sum' loss by a global
 * non-padding token count (NeMo AutoModel linear_ce API, forward(
 * num_label_tokens)); the matching backward takes grad_scale = loss_scale.
 * A NaN or infinite loss_scale is FLCE_ERR_ARG. */
flce_status flce_forward_ex(const void* hidden, const void* weight, const int64_t* labels,
                            int64_t N, int64_t H, int64_t V, int64_t ignore_index, float softcap,
                            int32_t reduction, int32_t dtype, float loss_scale, float* loss,
                            int64_t* num_tokens, float* lse, void* workspace,
                            size_t workspace_bytes, void* stream);

/* flce_forward_ex with, in addition, the global number of label tokens that
 * normalises a 'sum' loss (NeMo AutoModel linear_ce API, forward(
 * num_label_tokens): the count of non-padding target tokens across the
 * micro-batches and ranks that share one optimizer step).
 *   num_label_tokens >= 0, 'sum': loss = loss_scale * (sum_i loss_i) /
 *       max(num_label_tokens, 1), evaluated in float64 before the single
 *       rounding to float32 (the max(., 1) clamp keeps a batch without target
 *       tokens at 0, never NaN: inclusionAI/Ling-3.1-flash discussion #7, "Why
 *       use num_items_in_batch for MTP?");
 *   num_label_tokens < 0 (none given), or 'mean' (which divides by its own
 *       count): as flce_forward_ex.
 * num_tokens and lse are unchanged by either scale.  The matching backward is
 * flce_backward_ex with the same num_label_tokens and grad_scale = loss_scale. */
flce_status flce_forward_ex2(const void* hidden, const void* weight, const int64_t* labels,
                             int64_t N, int64_t H, int64_t V, int64_t ignore_index, float softcap,
                             int32_t reduction, int32_t dtype, float loss_scale,
                             int64_t num_label_tokens, float* loss, int64_t* num_tokens,
                             float* lse, void* workspace, size_t workspace_bytes, void* stream);

/* flce_backward flags. */
#define FLCE_ACCUMULATE_DHIDDEN 1 /* d_hidden += gradient (else overwritten) */
#define FLCE_ACCUMULATE_DWEIGHT 2 /* d_weight += gradient (else overwritten) */
#define FLCE_DHIDDEN_BF16 4       /* d_hidden is bf16 [N*H] (else float) */
#define FLCE_DWEIGHT_BF16 8       /* d_weight is bf16 [V*H] (else float) */

/* Backward of the loss returned by flce_forward with the same arguments.
 *   lse          device float[N]  from flce_forward
 *   grad_output  device float[1]  upstream gradient of the loss; NULL means 1.0
 *   grad_scale   host float       extra factor (micro-batch / token weighting)
 *   num_valid    device int64[1]  n (the true count, also for 'mean');
 *                                 NULL: the library counts it on the device
 *   d_hidden     device float[N*H]  overwritten, or accumulated into
 *                (bf16[N*H] with FLCE_DHIDDEN_BF16)
 *   d_weight     device float[V*H]  overwritten, or accumulated into
 *                (bf16[V*H] with FLCE_DWEIGHT_BF16)
 *                Either may be NULL: that gradient is then not computed (a
 *                frozen LM head needs no dWeight GEMM: a third of the work);
 *                at least one must be given.
 *   flags        any OR of FLCE_ACCUMULATE_DHIDDEN, FLCE_ACCUMULATE_DWEIGHT,
 *                FLCE_DHIDDEN_BF16, FLCE_DWEIGHT_BF16, or 0.
 * A bf16 output is computed in fp32 scratch inside the workspace (size it with
 * flce_workspace_bytes_ex) and rounded once, to nearest even: overwrite gives
 * bf16(g), accumulate gives bf16(float(old) + g).  Ignored rows of a
 * non-accumulated d_hidden are exact zeros either way.
 * Accumulating into d_weight across the micro-batches of one optimizer step
 * (each with grad_scale = 1 / the step's total non-ignored count) gives the
 * token-weighted gradient of the whole batch (modelscope/twinkle PR #335,
 * item 2).  The call clears the workspace status word and records in it a
 * label outside [0, V) that is not ignore_index (FLCE_ERR_LABEL_RANGE); such a
 * row is treated as ignored (zero gradient, not counted), as in the forward. */
flce_status flce_backward(const void* hidden, const void* weight, const int64_t* labels,
                          const float* lse, int64_t N, int64_t H, int64_t V,
                          int64_t ignore_index, float softcap, int32_t reduction, int32_t dtype,
                          const float* grad_output, float grad_scale, const int64_t* num_valid,
                          float* d_hidden, float* d_weight, int32_t flags, void* workspace,
                          size_t workspace_bytes, void* stream);

/* flce_backward for the loss of flce_forward_ex2: with num_label_tokens >= 0
 * and 'sum', the gradient factor g is divided by max(num_label_tokens, 1)
 * (computed in float64 with grad_scale, then rounded once to float32);
 * num_label_tokens < 0 or 'mean': exactly flce_backward.  Every other argument
 * as flce_backward. */
flce_status flce_backward_ex(const void* hidden, const void* weight, const int64_t* labels,
                             const float* lse, int64_t N, int64_t H, int64_t V,
                             int64_t ignore_index, float softcap, int32_t reduction,
                             int32_t dtype, const float* grad_output, float grad_scale,
                             int64_t num_label_tokens, const int64_t* num_valid,
                             float* d_hidden, float* d_weight, int32_t flags, void* workspace,
                             size_t workspace_bytes, void* stream);

/* Size of the library-owned device buffer behind flce_forward_noalloc. */
#define FLCE_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)

/* Forward that allocates nothing and takes no workspace.  The pages have no
 * counterpart to this entry point; it exists for callers that cannot allocate
 * device memory at all: op/plugin interfaces that hand a kernel only its input
 * and output buffers with no allocator, and programs that reserve the whole
 * device memory in their own pool at start-up, where an extra cudaMalloc
 * either fails or synchronises the device.
 *
 * Same arguments and results as flce_forward, minus the workspace.  Its
 * scratch (per-vocab-tile softmax partials, label logits, loss partials) lives
 * in one static __device__ buffer of FLCE_NOALLOC_SCRATCH_BYTES that every
 * device which loads this library keeps until the process exits.
 *  - Sizes whose forward scratch exceeds that buffer (about
 *    8 * N * ceil(V / 256) bytes for bf16) return FLCE_ERR_SHAPE and launch
 *    nothing; flce_forward with a caller workspace has no such limit.
 *  - The first call on each device looks the buffer's device address up
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture.
 *  - Every call on a device shares the one buffer, and the buffer keeps the
 *    last call's contents (the call clears the part that must start at zero).
 *    Calls whose kernels overlap on the GPU (different streams, or several
 *    host threads) race on it: order them on one stream.
 *  - status: optional device uint32[1]; receives the asynchronous error bits of
 *    this call (1 = label outside [0, V) and not ignore_index, 2 = a bounded
 *    pipeline wait ran out), 0 if none.  NULL skips it.
 * It never calls cudaMalloc, cudaFree or any allocating library routine. */
flce_status flce_forward_noalloc(const void* hidden, const void* weight, const int64_t* labels,
                                 int64_t N, int64_t H, int64_t V, int64_t ignore_index,
                                 float softcap, int32_t reduction, int32_t dtype, float* loss,
                                 int64_t* num_tokens, float* lse, uint32_t* status, void* stream);

/* Synchronise `stream`, then return the asynchronous error recorded in the
 * workspace by the latest flce_forward or flce_backward on it (FLCE_OK if
 * none; a label-range error is reported before a timeout). */
flce_status flce_get_status(const void* workspace, void* stream);

/* Self-test of failure reporting: launches one tiny kernel whose thread waits
 * on an mbarrier that nothing arrives on, through the same bounded wait the
 * GEMM pipelines use, with a limit of timeout_ms (1..10000).  The wait runs
 * out, the kernel records the timeout bit in the workspace status word and
 * returns, so the following flce_get_status() reports FLCE_ERR_TIMEOUT and the
 * CUDA context stays usable.  No fault, trap or hang is involved; the next
 * flce_forward clears the status.  (Test hook; no counterpart on the pages.) */
flce_status flce_selftest_wait_timeout(void* workspace, int32_t timeout_ms, void* stream);

/* Human-readable name of a status code (static storage). */
const char* flce_status_string(int32_t status);

/* ABI version of this library (major * 10000 + minor * 100 + patch). */
int32_t flce_version(void);

/* Number of kernels this library has launched in this process. */
uint64_t flce_launch_count(void);

/* Launch-time accounting, for benchmarks.  When enabled, the library records
 * a CUDA event pair around every kernel it launches (on the call's stream).
 * flce_profile_read synchronises those events and returns, for one kernel
 * kind, the summed device time in milliseconds and the number of launches
 * since the last read of that kind, then forgets them.
 * Kinds: 0 forward GEMM+softmax stats, 1 forward merge/loss, 2 backward dZ
 * GEMM, 3 backward dHidden+dWeight GEMMs (one launch per chunk), 4 unused,
 * 5 small helper kernels, 6 fp32 CUDA-core path. */
flce_status flce_profile_enable(int32_t enable);
flce_status flce_profile_read(int32_t kind, double* total_ms, int64_t* launches);

#ifdef __cplusplus
}
#endif

#endif /* FLCE_H */
