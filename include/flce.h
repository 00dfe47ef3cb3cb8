/*
 * flce.h - C ABI of the B200 (sm_100a) fused LM-head projection + cross-entropy.
 *
 * The operation (NeMo-AutoModel pages "nemo_automodel.components.loss.linear_ce",
 * FusedLinearCrossEntropy, and "nemo_automodel.components.models.inkling2.loss",
 * Inkling2FusedLinearCrossEntropy, class docstring):
 *
 *   z[n, v]  = sum_h hidden[n, h] * Wb[v, h]            BF16 x BF16, FP32 accumulate
 *   zc[n, v] = c * tanh(z[n, v] / c)  (c > 0), else z   FP32 logit softcap
 *   lse[n]   = log sum_{v < V} exp(zc[n, v])            rows >= V never enter the softmax
 *   l[n]     = lse[n] - zc[n, y_n]  if y_n != ignore_index, else 0
 *   loss     = sum_n l[n]  (/ num_label_tokens if > 0),  or mean, or per token
 *
 * with Wb = the first V = unpadded_vocab rows of the head, rounded to BF16 (RNE)
 * when the head is FP32 (inkling2 page: "An FP32 head is rounded to BF16").
 * The backward recomputes the logits and returns dhidden (BF16) and dweight
 * (the head's dtype, rows >= V exactly 0); no [N, V] tensor is ever written.
 *
 * Conventions for every entry point
 *  - All tensor pointers are DEVICE pointers on the current CUDA device,
 *    row-major and contiguous; the caller allocates and owns every buffer and
 *    the library allocates no device memory.  Work is enqueued on `stream`
 *    (a cudaStream_t; NULL = the legacy default stream) and runs
 *    asynchronously; outputs are valid once the stream has reached that point.
 *  - hidden:  BF16 [N, H];  weight: [Vp, H], BF16 or FP32 (w_dtype);
 *    labels: int64 [N], not shifted (labels[n] is the target of hidden[n]).
 *  - H must be a multiple of 8 (16-byte rows for the tensor-memory-access
 *    engine); hidden, weight, dhidden, dweight and workspace must be 16-byte
 *    aligned; labels, loss and lse 8- resp. 4-byte aligned.
 *  - Arguments are checked on the host before anything is enqueued; a bad
 *    argument returns an error status and enqueues nothing.  Nothing throws or
 *    aborts across this boundary.  FLCE_ERR_CUDA from a launch means kernels
 *    the call enqueued before it may still run; the call's outputs are then
 *    undefined.
 *  - After one call of an entry point per device and dtype (which queries the
 *    device, resolves the tensor-map encoder and caches launch shapes),
 *    flce_forward / flce_backward / flce_ce_* only enqueue work on `stream`
 *    (kernels, and in flce_forward one 4-byte memset that zeroes a tile
 *    counter in the workspace), so a sequence of them can be captured into a
 *    CUDA graph and replayed with the same buffers.
 *  - Labels outside [0, V) that are not ignore_index cannot be checked on the
 *    host without a device read; the kernels treat them as ignored (zero loss,
 *    zero gradient) and raise FLCE_ERR_BAD_LABEL in a per-device error word
 *    that flce_get_error() reports and clears.
 */
#ifndef FLCE_H_
#define FLCE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef void* flce_stream_t; /* a cudaStream_t */

typedef enum {
  FLCE_OK = 0,
  FLCE_ERR_INVALID_ARG = 1, /* bad size, pointer, alignment or option        */
  FLCE_ERR_WORKSPACE = 2,   /* workspace NULL or smaller than required       */
  FLCE_ERR_UNSUPPORTED = 3, /* no sm_100a device, or more tiles than supported */
  FLCE_ERR_CUDA = 4,        /* a CUDA runtime call or kernel launch failed   */
  FLCE_ERR_BAD_LABEL = 5,   /* (flce_get_error) a label outside [0,V) seen   */
  FLCE_ERR_TIMEOUT = 6      /* (flce_get_error) a pipeline wait ran out      */
} flce_status;

typedef enum { FLCE_SUM = 0, FLCE_MEAN = 1, FLCE_NONE = 2 } flce_reduction;
typedef enum { FLCE_BF16 = 0, FLCE_F32 = 1 } flce_dtype;

/*
 * Bytes of workspace that flce_forward and flce_backward want for this shape
 * (one buffer serves both).  Pure host arithmetic.  Returns 0 for invalid
 * sizes.  unpadded_vocab <= 0 means padded_vocab.  The backward also accepts a
 * smaller workspace (down to flce_workspace_min_size) and then streams the
 * vocabulary in narrower chunks.
 */
size_t flce_workspace_size(int64_t n_tokens, int64_t hidden, int64_t padded_vocab,
                           int64_t unpadded_vocab, int w_dtype);
size_t flce_workspace_min_size(int64_t n_tokens, int64_t hidden, int64_t padded_vocab,
                               int64_t unpadded_vocab, int w_dtype);

/*
 * FP32 head without a BF16 copy (inkling2 page, Inkling2FusedLinearCrossEntropy
 * class docstring: an FP32 head is rounded to BF16, "the cast FSDP applies").
 * With this flag, flce_forward_ex and flce_backward_ex do not write the
 * head's BF16 copy (V*H*2 bytes) into the workspace: the GEMMs that read the
 * head load its FP32 rows and round them to BF16 (nearest even, the same
 * rounding as the copy) in shared memory, inside the kernel.  Results are
 * bit-identical to the copy's; the workspace shrinks by the copy, and the
 * GEMMs move twice the head bytes and convert every head tile once per tile
 * row, so they run slower than the copy path: on one B200, 8192 tokens with
 * H = 5376 and V = 256000 take about twice as long per forward + backward
 * (0.51x the tokens/s) in a workspace of 1.85 GB instead of 4.61 GB.
 * The flag has no effect with a BF16 head.
 * The _ex sizes take the same flags (0 or FLCE_FUSED_HEAD_CAST; any other
 * bit gives 0).
 */
#define FLCE_FUSED_HEAD_CAST 2u
size_t flce_workspace_size_ex(int64_t n_tokens, int64_t hidden, int64_t padded_vocab,
                              int64_t unpadded_vocab, int w_dtype, unsigned int flags);
size_t flce_workspace_min_size_ex(int64_t n_tokens, int64_t hidden, int64_t padded_vocab,
                                  int64_t unpadded_vocab, int w_dtype, unsigned int flags);

/*
 * Forward: the loss and the per-token logsumexp.
 *   Defines: linear_ce page, FusedLinearCrossEntropy(ignore_index=-100,
 *   logit_softcapping=0, reduction='sum') and forward(hidden_states, labels,
 *   lm_weight, num_label_tokens); inkling2 page for unpadded_vocab and the
 *   BF16/FP32 contract.
 *   unpadded_vocab   V: rows of the head that enter the softmax; <= 0 means Vp.
 *   ignore_index     label value that contributes neither loss nor gradient.
 *   softcap          c >= 0; 0 disables the softcap.
 *   reduction        FLCE_SUM (default of the pages), FLCE_MEAN or FLCE_NONE.
 *   num_label_tokens > 0: divide the summed loss by it (FLCE_SUM only);
 *                    <= 0: no normalisation.
 *   loss   out, FP32: [1] for SUM/MEAN (MEAN with no valid label gives NaN),
 *          [N] per-token losses for NONE.
 *   lse    out, FP32 [N]: per-token logsumexp of the capped logits (all
 *          tokens, ignored ones included); flce_backward consumes it.
 *   workspace, ws_bytes: device scratch of at least
 *          flce_workspace_size(...) bytes; contents are overwritten.
 * Returns FLCE_OK or an error status.  N == 0 is valid (loss 0, NaN for MEAN).
 */
int flce_forward(const void* hidden, const void* weight, int w_dtype, const int64_t* labels,
                 int64_t n_tokens, int64_t hidden_size, int64_t padded_vocab,
                 int64_t unpadded_vocab, int64_t ignore_index, float softcap,
                 int reduction, int64_t num_label_tokens, float* loss, float* lse,
                 void* workspace, size_t ws_bytes, flce_stream_t stream);

/*
 * flce_forward with option flags: 0 or FLCE_FUSED_HEAD_CAST (see above; the
 * workspace then needs flce_workspace_size_ex(..., FLCE_FUSED_HEAD_CAST)
 * bytes).  Any other bit set: FLCE_ERR_INVALID_ARG.
 * flce_forward(...) is flce_forward_ex(..., 0, stream).
 */
int flce_forward_ex(const void* hidden, const void* weight, int w_dtype,
                    const int64_t* labels, int64_t n_tokens, int64_t hidden_size,
                    int64_t padded_vocab, int64_t unpadded_vocab, int64_t ignore_index,
                    float softcap, int reduction, int64_t num_label_tokens, float* loss,
                    float* lse, void* workspace, size_t ws_bytes, unsigned int flags,
                    flce_stream_t stream);

/*
 * Backward: gradients of the loss above, recomputing the logits.
 *   Defines: chunked_ce page, _ChunkedCrossEntropySum.backward (recompute the
 *   FP32 softmax instead of storing it); inkling2 page ("Gradients reach the"
 *   padded head through the slice and cast: rows >= V get exactly 0).
 *   Same shape/option arguments as flce_forward.
 *   grad_loss  in, FP32 device: [1] for SUM/MEAN, [N] for NONE.
 *   lse        in, FP32 [N]: the lse written by flce_forward on the same inputs.
 *   dhidden    out, BF16 [N, H] (overwritten).
 *   dweight    out, [Vp, H] in w_dtype (overwritten; rows [V, Vp) set to 0).
 *   workspace  >= flce_workspace_min_size(...) bytes; with less than
 *              flce_workspace_size(...) the vocabulary is processed in
 *              narrower chunks (same result, more passes over dhidden).
 * Ignored tokens get exactly-zero dhidden rows and add nothing to dweight.
 */
int flce_backward(const void* hidden, const void* weight, int w_dtype, const int64_t* labels,
                  int64_t n_tokens, int64_t hidden_size, int64_t padded_vocab,
                  int64_t unpadded_vocab, int64_t ignore_index, float softcap,
                  int reduction, int64_t num_label_tokens, const float* grad_loss,
                  const float* lse, void* dhidden, void* dweight,
                  void* workspace, size_t ws_bytes, flce_stream_t stream);

/*
 * flce_backward with option flags.  The pages compute the head's BF16 copy
 * once per step (inkling2 page, Inkling2FusedLinearCrossEntropy class
 * docstring: an FP32 head is rounded to BF16, "the cast FSDP applies", and the
 * gradient flows back through that cast); this lets the backward reuse the
 * copy the forward made instead of casting again.
 *   flags  0, or FLCE_BWD_HEAD_COPY_VALID: the caller promises that the first
 *          V*H*2 bytes of `workspace` (rounded up to 1 KiB) still hold the BF16
 *          copy of weight[:V] that flce_forward wrote there -- the forward ran
 *          on this workspace with this weight pointer, shape and w_dtype, and
 *          neither the head nor those workspace bytes changed since.  The
 *          backward then skips its own FP32 -> BF16 cast of the head (one read
 *          of V*H*4 bytes and one write of V*H*2).  The flag is ignored for a
 *          BF16 head, which is used in place.  The library cannot check the
 *          promise: a stale copy gives wrong gradients without an error.
 *          Or FLCE_FUSED_HEAD_CAST: no copy is used or written; the recompute
 *          and dhidden GEMMs round the FP32 head in the kernel (the workspace
 *          then needs flce_workspace_min_size_ex(..., FLCE_FUSED_HEAD_CAST)
 *          bytes at least).  Both flags at once, or any other bit set:
 *          FLCE_ERR_INVALID_ARG.
 * flce_backward(...) is flce_backward_ex(..., 0, stream).
 */
#define FLCE_BWD_HEAD_COPY_VALID 1u
int flce_backward_ex(const void* hidden, const void* weight, int w_dtype,
                     const int64_t* labels, int64_t n_tokens, int64_t hidden_size,
                     int64_t padded_vocab, int64_t unpadded_vocab, int64_t ignore_index,
                     float softcap, int reduction, int64_t num_label_tokens,
                     const float* grad_loss, const float* lse, void* dhidden, void* dweight,
                     void* workspace, size_t ws_bytes, unsigned int flags,
                     flce_stream_t stream);

/*
 * Synchronises `stream`, then reads and clears the calling device's error word:
 * FLCE_ERR_BAD_LABEL if a kernel saw a label outside [0, V) that was not
 * ignore_index, FLCE_ERR_TIMEOUT if a pipeline wait gave up (the affected
 * output is then incomplete), FLCE_ERR_CUDA if the synchronisation failed,
 * else FLCE_OK.  The word is shared by every call on the device since the
 * last read.
 */
int flce_get_error(flce_stream_t stream);

/* Static description of a status code. */
const char* flce_status_string(int status);

/* Algorithmic FLOPs of one forward + backward for a shape, for reports:
 * 8*N*V*H (forward GEMM, recompute GEMM, dW GEMM, dh GEMM; V unpadded). */
double flce_flops_fwd_bwd(int64_t n_tokens, int64_t hidden_size, int64_t unpadded_vocab);

/*
 * Self-test of the tensor-core GEMM the path is built on (no counterpart on
 * the pages; for tests):  D[M, N] (FP32, row-major) = A . B^T over K, with
 *   A: a_mn == 0 -> BF16 [M, K] (K contiguous); a_mn == 1 -> BF16 [K, M];
 *   B: b_mn == 0 -> BF16 [N, K];                b_mn == 1 -> BF16 [K, N].
 * Sizes must be positive, N, K (K-contiguous operands) and M/N (MN-contiguous
 * operands) multiples of 8.  Device pointers, asynchronous on `stream`.
 */
int flce_selftest_gemm(const void* a, const void* b, float* d, int64_t m, int64_t n,
                       int64_t k, int a_mn, int b_mn, flce_stream_t stream);

/*
 * Self-test of the bounded pipeline waits (no counterpart on the pages):
 * launches one block that waits on a barrier nothing ever arrives on, with a
 * limit of `timeout_us` microseconds (1..2000000).  The kernel gives up, sets
 * the timeout bit of the error word and returns; the context stays usable.
 * flce_get_error() then reports FLCE_ERR_TIMEOUT.
 */
int flce_selftest_wait_timeout(unsigned int timeout_us, flce_stream_t stream);

/*
 * Cross entropy on given logits: the pages' ChunkedCrossEntropy
 * ("nemo_automodel.components.loss.chunked_ce": ChunkedCrossEntropy.forward(
 * logits, labels, mask, num_label_tokens), _ChunkedCrossEntropySum.forward /
 * backward, compute_cross_entropy).
 *   logits     [N, V] rows ld elements apart (ld >= V), BF16 (dtype 0) or FP32
 *              (dtype 1), 16-byte aligned base; read, never written.
 *   labels     int64 [N]; mask: optional uint8 [N] (NULL = none) -- a zero
 *              entry makes that position ignored, as the page's `mask` does.
 *   ignore_index, reduction, num_label_tokens, loss, lse: as flce_forward.
 *   dlogits    (backward) [N, V], rows ld apart, the logits' dtype, 16-byte
 *              aligned base: s_n * (softmax(logits)[n] - onehot(y_n)), zero
 *              rows for ignored / masked positions.
 *   workspace  >= flce_ce_workspace_size(N) bytes.
 * No FP32 copy of the logits is made: one pass over them in the forward, one
 * read + one write in the backward.  Same error conventions as flce_forward.
 */
size_t flce_ce_workspace_size(int64_t n_tokens);
int flce_ce_forward(const void* logits, int dtype, const int64_t* labels, const uint8_t* mask,
                    int64_t n_tokens, int64_t vocab, int64_t ld, int64_t ignore_index,
                    int reduction, int64_t num_label_tokens, float* loss, float* lse,
                    void* workspace, size_t ws_bytes, flce_stream_t stream);
int flce_ce_backward(const void* logits, int dtype, const int64_t* labels, const uint8_t* mask,
                     int64_t n_tokens, int64_t vocab, int64_t ld, int64_t ignore_index,
                     int reduction, int64_t num_label_tokens, const float* grad_loss,
                     const float* lse, void* dlogits, void* workspace, size_t ws_bytes,
                     flce_stream_t stream);

/*
 * Forward that allocates nothing and takes no workspace (the pages have no
 * counterpart; it exists for callers that cannot supply scratch memory, such
 * as a plugin inside a framework whose allocator owns the whole device, or a
 * service that allows no device allocation once running).
 *   Arguments and results are those of flce_forward without workspace /
 *   ws_bytes; the caller still passes every input and output.
 *   Scratch: a 32 MiB array in this library's device memory, present on every
 *   GPU that loads the library until the process exits.  A problem whose
 *   forward scratch (8 B x ceil(V/256) x N for the logsumexp partials, plus
 *   4 B x N) exceeds 32 MiB is refused with FLCE_ERR_WORKSPACE and nothing is
 *   enqueued; e.g. N = 4096 tokens with V = 128256 needs 15.7 MiB (16.4 MB)
 *   and fits.  An FP32 head takes the FLCE_FUSED_HEAD_CAST path (rounded to
 *   BF16 inside the GEMM), so it needs no room for a BF16 copy.
 *   The array is shared by every call on a device and keeps whatever the last
 *   call left in it; the forward writes every scratch byte before reading it,
 *   so nothing has to be cleared between calls.  Calls that overlap on the GPU
 *   (different streams, or different host threads) race on the array: order
 *   them on one stream or synchronise between them.
 *   The first call on each device looks up the array's device address with
 *   cudaGetSymbolAddress (with that device current); make that first call
 *   before any stream capture.  The address is looked up again whenever the
 *   device's CUDA context has changed (after cudaDeviceReset, for instance),
 *   so that call too belongs outside a capture.
 */
int flce_forward_noalloc(const void* hidden, const void* weight, int w_dtype,
                         const int64_t* labels, int64_t n_tokens, int64_t hidden_size,
                         int64_t padded_vocab, int64_t unpadded_vocab, int64_t ignore_index,
                         float softcap, int reduction, int64_t num_label_tokens, float* loss,
                         float* lse, flce_stream_t stream);

/*
 * Launch accounting for benchmarks (no counterpart on the pages).
 *
 * flce_launch_count: kernels this library has launched in this process.
 * flce_profile_start: from now on, bracket every kernel launch of this library
 *   with CUDA events on its stream (process-wide, any stream).  Returns
 *   FLCE_ERR_INVALID_ARG if profiling is already on.
 * flce_profile_stop: synchronise those events, stop recording and report one
 *   flce_kernel_stat per kernel family that launched: launches, summed device
 *   time between its events, and the algorithmic work the launches did
 *   (FLOPs of the contraction; HBM bytes a single-pass kernel must move).
 *   Writes at most `capacity` entries to `stats` and the family count to
 *   *count.
 */
typedef struct {
  char name[32];
  int64_t launches;
  double total_ms;
  double flops;
  double bytes;
} flce_kernel_stat;

unsigned long long flce_launch_count(void);
int flce_profile_start(void);
int flce_profile_stop(flce_kernel_stat* stats, int capacity, int* count);

#ifdef __cplusplus
}
#endif
#endif /* FLCE_H_ */
