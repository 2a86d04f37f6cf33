/*
 * sfn.h -- C ABI of libsfn: the predictor-gated bank-wise top-k sparse
 * SwiGLU FFN on NVIDIA B200 (sm_100a) -- its forward pass (whole layer or one
 * bank shard), its backward with the surrogate top-k gradient, and the
 * pages' Dense-4x comparison.
 *
 * The method: "Continual LLM Upcycling: A Predictor-Gated Bank-Wise Sparsity
 * Training Recipe for Dense-to-Sparse LLMs" (arXiv 2606.10722).  Passages are
 * cited by page and section:
 *   [arch]  gist.science summary, "Methodologie / 1. Architectuur:
 *           Predictor-Gated Sparse SwiGLU" -- a low-rank predictor
 *           R^d -> R^448 -> R^{d_i} acts on the token hidden state before the
 *           FFN; its logits replace the dense SwiGLU gate; d_i = 14336 is cut
 *           into fixed banks of 64 with a hard top-16 per bank (d_s = 3584);
 *           in the forward pass inactive channels are exactly zero.
 *   [hw]    same page, "3. Hardware Implicaties" -- with dedicated kernels
 *           the gate, up and down projections all skip inactive channels.
 *   [abs]   the paper's abstract (catalyzex.com / searcharxiv.com author
 *           pages) -- per token and layer a low-rank predictor gives
 *           FFN-channel routing logits; a bank-wise top-k keeps 16 channels
 *           in every 64-channel bank, 4x sparsity.
 *
 * Readings of what the pages leave open (fixed here, identical in the CPU
 * oracle):
 *   - the predictor is p = B (A x): no bias, no inner activation;
 *   - each kept channel j computes a_j = sigma(p_j) * (Wg[j].x) * (Wu[j].x)
 *     (sigma(p) takes the place of the gate's sigma in silu);
 *     y = sum_{kept j} a_j * W_down[:, j];
 *   - banks are contiguous channel ranges [b*bank, (b+1)*bank);
 *   - a bank keeps the k largest logits; equal logits go to the lower
 *     channel index; +0 equals -0; NaN ranks below every number.
 *
 * Layouts (all row-major and contiguous; every pointer is a DEVICE pointer):
 *   x      [T][d]        hidden states (bf16 or f32)
 *   A      [r][d]        first predictor factor
 *   B      [d_i][r]      second predictor factor
 *   Wg, Wu [d_i][d]      gate / up projection rows
 *   Wd     [d_i][d]      DOWN PROJECTION STORED CHANNEL-MAJOR: row j of Wd
 *                        is column j of W_down ([d][d_i]), i.e. Wd = W_down^T,
 *                        so the 16 kept channels of a bank are 16 contiguous
 *                        rows of d elements.
 *   y      [T][d]        output (same element type as x)
 *   logits [T][d_i]      float32
 *   mask   [T][d_i/bank] uint64; bit i of word b is channel b*bank + i;
 *                        bits at and above `bank` are zero.
 *
 * Ownership and execution: the caller owns every buffer; the library keeps
 * no pointer after a call returns.  Every call only enqueues work on
 * `stream` (cudaStream_t; NULL is the legacy default stream) and returns
 * without synchronising; results are ready when the stream is.  No call
 * copies between host and device.  The only allocations are the
 * stream-ordered scratch of sfn_sparse_ffn_forward and sfn_predict
 * (cudaMallocAsync / cudaFreeAsync on `stream`); the other entry points
 * take caller scratch.  Calls on different streams may run concurrently if
 * their outputs and scratch do not overlap.  Results are deterministic: a
 * fixed reduction order and no floating-point atomics, so a rerun is
 * bit-identical.
 *
 * Errors: every argument is checked on the host before anything is
 * enqueued; on any error status nothing is written.  T == 0 returns SFN_OK
 * without enqueueing work (pointers are then not inspected).  A launch
 * failure is reported as SFN_ERR_CUDA; faults during execution surface at
 * the caller's next synchronisation, as for any CUDA work.  There is no CPU
 * fallback: without a usable sm_100 device every compute call returns
 * SFN_ERR_CUDA.
 */
#ifndef SFN_H_
#define SFN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; declared here so this header needs no CUDA
 * include. */
typedef struct CUstream_st *sfn_stream_t;

typedef enum sfn_status {
  SFN_OK = 0,
  SFN_ERR_INVALID_VALUE = 1, /* T < 0; d, d_i or r <= 0; d_i % bank != 0;
                                not 1 <= k <= bank <= 64; required pointer
                                NULL; unknown dtype */
  SFN_ERR_MISALIGNED = 2,    /* a pointer not 16-byte aligned, or d or r not
                                a multiple of 16 bytes of its element type */
  SFN_ERR_UNSUPPORTED = 3,   /* a valid shape outside the built kernels'
                                limits: d > 8192, r > 2048, d_i > 2^24;
                                on the CUDA-core path also d not a
                                multiple of 64 (bf16) / 32 (f32), or
                                d > 4096 for f32 */
  SFN_ERR_WORKSPACE = 4,     /* *_ws scratch NULL, misaligned or smaller than
                                sfn_workspace_bytes() */
  SFN_ERR_CUDA = 5           /* a CUDA runtime call or launch failed */
} sfn_status;

typedef enum sfn_dtype {
  SFN_DTYPE_BF16 = 0, /* x, A, B, Wg, Wu, Wd, y in bf16; fp32 accumulation */
  SFN_DTYPE_F32 = 1   /* everything in float32 */
} sfn_dtype;

/* Static, NUL-terminated description of a status code. */
const char *sfn_status_string(sfn_status s);

/* ABI version of this header (incremented on any signature change). */
int sfn_abi_version(void);

/* The message behind the last SFN_ERR_CUDA (the CUDA runtime's) returned on
 * this host thread (static string; "no error" if none). */
const char *sfn_last_error_string(void);

/* Number of kernels this library has launched in this process (all
 * devices, all threads).  Diagnostic counter; never reset. */
uint64_t sfn_kernel_launch_count(void);

/*
 * Predictor logits [arch]: for every token t, h = A x_t (R^d -> R^r), then
 * logits[t] = B h (R^r -> R^{d_i}).  Accumulation is float32; h is kept in
 * float32 between the two factors.
 * sfn_predict: x, A, B are bf16 (uint16 bit patterns); sfn_predict_f32:
 * float32.  logits is float32 [T][d_i].
 */
sfn_status sfn_predict(const void *x, const void *A, const void *B, float *logits,
                       int64_t T, int d, int d_i, int r, sfn_stream_t stream);
sfn_status sfn_predict_f32(const float *x, const float *A, const float *B, float *logits,
                           int64_t T, int d, int d_i, int r, sfn_stream_t stream);

/*
 * Bank-wise hard top-k [arch], [abs]: in every bank of `bank` consecutive
 * channels of logits[t], set the bits of the k largest logits (ties to the
 * lower index, NaN lowest).  Exactly k bits are set in every word.
 * logits float32 [T][d_i] -> mask uint64 [T][d_i/bank].
 */
sfn_status sfn_bank_topk(const float *logits, uint64_t *mask, int64_t T, int d_i,
                         int bank, int k, sfn_stream_t stream);

/*
 * Bytes of scratch the *_ws forward variants need for this shape and
 * element type (0 when T == 0).  Returns 0 for invalid arguments.
 */
size_t sfn_workspace_bytes(int64_t T, int d, int d_i, int r, int bank, int k,
                           sfn_dtype dtype);

/*
 * The whole sparse FFN forward [arch], [hw]: predictor logits, bank-wise
 * top-k mask, then for the kept channels only a_j = sigma(p_j) * (Wg[j].x) *
 * (Wu[j].x) and y = sum_j a_j Wd[j, :].  Unkept channels are never read.
 * x, A, B, Wg, Wu, Wd, y are bf16 (uint16 bit patterns); mask, if not NULL,
 * receives the mask used.  Scratch is taken stream-ordered from the
 * device's default memory pool and returned before the call's work ends.
 */
sfn_status sfn_sparse_ffn_forward(const void *x, const void *A, const void *B,
                                  const void *Wg, const void *Wu, const void *Wd, void *y,
                                  uint64_t *mask, int64_t T, int d, int d_i, int r,
                                  int bank, int k, sfn_stream_t stream);

/* As sfn_sparse_ffn_forward, with caller scratch `workspace` (device, 256-byte
 * aligned, at least sfn_workspace_bytes(..., SFN_DTYPE_BF16) bytes).  The
 * scratch must not be used by other work until this call's work is done. */
sfn_status sfn_sparse_ffn_forward_ws(const void *x, const void *A, const void *B,
                                     const void *Wg, const void *Wu, const void *Wd,
                                     void *y, uint64_t *mask, int64_t T, int d, int d_i,
                                     int r, int bank, int k, void *workspace,
                                     size_t workspace_bytes, sfn_stream_t stream);

/*
 * The bf16 forward without any allocation.  The paper has no counterpart:
 * this entry point exists for callers that cannot allocate device memory
 * when they run the layer -- a plugin interface that hands the layer only
 * its input and output pointers, a serving process whose allocator already
 * owns the GPU's memory, or a latency-critical loop that must not risk
 * cudaMalloc's implicit synchronisation.
 *
 * Arguments, layouts, results and checks are those of sfn_sparse_ffn_forward.
 * The scratch is one fixed device array of SFN_STATIC_SCRATCH_BYTES inside
 * the library, which the CUDA runtime keeps in the memory of every GPU that
 * loads this library's code until the process exits.  The call allocates
 * and frees nothing.
 *   - A shape whose scratch need (sfn_workspace_bytes(..., SFN_DTYPE_BF16))
 *     exceeds SFN_STATIC_SCRATCH_BYTES is rejected with SFN_ERR_WORKSPACE
 *     before anything is enqueued.  For the 4096 x 14336 layer (r 448,
 *     bank 64, k 16) every T up to 81 fits, and T = 129 to 132 (the
 *     many-token kernels' split sums need more scratch at 82 to 128 tokens
 *     and from 133); sfn_workspace_bytes() tells for any shape.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current) and caches it; make
 *     that first call before any stream capture.  cudaDeviceReset unloads
 *     the library's module from that device and invalidates the cached
 *     address (as it does the device error word's, see sfn_device_errors):
 *     do not call the library on a device after resetting it in the same
 *     process.
 *   - Every call shares the one array per device.  Calls whose work overlaps
 *     on the GPU (other streams, other host threads) race on it and produce
 *     wrong results: serialise them.  The array keeps the previous call's
 *     contents; each call writes every scratch byte before reading it, so
 *     nothing needs clearing.
 */
#define SFN_STATIC_SCRATCH_BYTES (16u << 20)
sfn_status sfn_sparse_ffn_forward_static(const void *x, const void *A, const void *B,
                                         const void *Wg, const void *Wu, const void *Wd,
                                         void *y, uint64_t *mask, int64_t T, int d, int d_i,
                                         int r, int bank, int k, sfn_stream_t stream);

/*
 * Which kernels compute the forward.  The result is the same either way
 * (within rounding; the mask may differ only at exact-threshold ties of the
 * differently rounded logits).
 *   SFN_PATH_CUDA_CORE  gather kernels that read only the kept rows (few
 *                       tokens: every T, any bank <= 64, bf16 or f32);
 *   SFN_PATH_TENSOR     tcgen05 tensor-core GEMMs over 128-token tiles with
 *                       the top-k and the sigma(p) g u mask fused into their
 *                       epilogues (bf16, bank 64, d and d_i multiples of
 *                       256, r a multiple of 64 up to 512); when all tokens
 *                       fit one tile (T <= 128) the logits GEMM, the top-k
 *                       and the masked gate/up are one kernel;
 *   SFN_PATH_AUTO       the tensor path from T >= 6 when the shape allows
 *                       it, the CUDA-core path otherwise.
 */
typedef enum sfn_path {
  SFN_PATH_AUTO = 0,
  SFN_PATH_CUDA_CORE = 1,
  SFN_PATH_TENSOR = 2
} sfn_path;

/* sfn_sparse_ffn_forward_ws with an explicit path.  SFN_PATH_TENSOR on a
 * shape the tensor path does not cover returns SFN_ERR_UNSUPPORTED.
 * sfn_workspace_bytes() covers both paths. */
sfn_status sfn_sparse_ffn_forward_path(const void *x, const void *A, const void *B,
                                       const void *Wg, const void *Wu, const void *Wd,
                                       void *y, uint64_t *mask, int64_t T, int d, int d_i,
                                       int r, int bank, int k, sfn_path path, void *workspace,
                                       size_t workspace_bytes, sfn_stream_t stream);

/*
 * One bank shard of the layer, for splitting a layer's banks over devices
 * (banks are independent through the top-k and the three projections, so a
 * device that holds banks [b0, b1) computes their contribution to y and the
 * devices sum their partial outputs, e.g. with an all-reduce).
 *
 * B, Wg, Wu and Wd point at the shard's first row (channel b0 * bank) and
 * d_i is the shard's channel count (a multiple of bank); A and x are the
 * whole predictor factor and input.  y_partial [T][d] receives, in float32
 * and without rounding, sum over the shard's kept channels of a_j Wd[j];
 * mask (may be NULL) the shard's mask words.  The sum of y_partial over a
 * partition of the banks, rounded to bf16, is the layer's y.  bf16 inputs;
 * scratch sfn_workspace_bytes(T, d, d_i (the shard's), r, bank, k,
 * SFN_DTYPE_BF16); path and errors as sfn_sparse_ffn_forward_path.
 */
sfn_status sfn_sparse_ffn_forward_partial(const void *x, const void *A, const void *B,
                                          const void *Wg, const void *Wu, const void *Wd,
                                          float *y_partial, uint64_t *mask, int64_t T, int d,
                                          int d_i, int r, int bank, int k, sfn_path path,
                                          void *workspace, size_t workspace_bytes,
                                          sfn_stream_t stream);

/*
 * The pages' "Dense-4x" comparison (gist.science summary, "Resultaten": a
 * dense model made 4x sparse post hoc from the activation amplitude).
 * Reading: the standard SwiGLU FFN without a predictor -- act_j =
 * silu(Wg[j].x) * (Wu[j].x) with silu(z) = z sigma(z); in every bank keep the
 * k channels of largest |act_j| (ties to the lower index), zero the rest;
 * y = sum_j act_j Wd[j, :].  bf16 in and out (x, Wg, Wu, Wd, y); mask, if not
 * NULL, receives the kept channels.  Runs on the tensor cores: bank must be
 * 64 and d, d_i multiples of 256 (else SFN_ERR_UNSUPPORTED).  Scratch: at
 * least sfn_dense4x_workspace_bytes() bytes, 256-byte aligned.
 */
size_t sfn_dense4x_workspace_bytes(int64_t T, int d, int d_i, int bank, int k);
sfn_status sfn_dense4x_forward(const void *x, const void *Wg, const void *Wu, const void *Wd,
                               void *y, uint64_t *mask, int64_t T, int d, int d_i, int bank,
                               int k, void *workspace, size_t workspace_bytes,
                               sfn_stream_t stream);

/*
 * Backward of the layer, for training the predictor ("1. Architectuur",
 * Executie / Backward Pass: the non-differentiable top-k gets a soft,
 * sigmoid-like surrogate gradient around the selection threshold).
 *
 * Given dy = dL/dy [T][d] for the forward above on the same inputs, writes
 * the gradients of L with respect to every input:
 *   dx [T][d], dA [r][d], dB [d_i][r], dWg, dWu, dWd [d_i][d]  (float32)
 * Any of them may be NULL (not computed).  They are overwritten, not
 * accumulated.  mask (may be NULL) receives the forward's mask [T][d_i/bank].
 *
 * Surrogate (a reading; the pages give no formula): bank b's threshold
 * tau_b = (p_(k) + p_(k+1)) / 2, the midpoint of its k-th and (k+1)-th
 * logits, held constant; the forward mask m stays hard; in the backward
 * dm_j/dp_j := sigma'((p_j - tau_b) / temperature) / temperature.  With
 * k = bank there is no threshold and no surrogate term.  The surrogate term
 * needs g_j u_j of every channel, so the backward is dense in gate and up.
 *
 * bf16 inputs (x, A, B, Wg, Wu, Wd, dy); logits are recomputed with the
 * forward's own kernels (the same mask as the forward for the same T), the
 * elementwise chain rule runs in this library's kernels, and the dense
 * contractions run on its tcgen05 tensor-core GEMM (bf16 operands, float32
 * accumulation and output).  temperature must be finite and > 0 (else
 * SFN_ERR_INVALID_VALUE); d, d_i and r must be multiples of 64 (else
 * SFN_ERR_UNSUPPORTED).  Scratch: at least sfn_backward_workspace_bytes()
 * bytes, 256-byte aligned (1.4 GB for 4096 tokens of the 4096 x 14336
 * layer).  Other errors as sfn_sparse_ffn_forward_ws.
 */
size_t sfn_backward_workspace_bytes(int64_t T, int d, int d_i, int r, int bank, int k);
sfn_status sfn_sparse_ffn_backward(const void *x, const void *A, const void *B, const void *Wg,
                                   const void *Wu, const void *Wd, const void *dy,
                                   float temperature, float *dx, float *dA, float *dB,
                                   float *dWg, float *dWu, float *dWd, uint64_t *mask,
                                   int64_t T, int d, int d_i, int r, int bank, int k,
                                   void *workspace, size_t workspace_bytes,
                                   sfn_stream_t stream);

/* float32 twins of the two forward entry points. */
sfn_status sfn_sparse_ffn_forward_f32(const float *x, const float *A, const float *B,
                                      const float *Wg, const float *Wu, const float *Wd,
                                      float *y, uint64_t *mask, int64_t T, int d, int d_i,
                                      int r, int bank, int k, sfn_stream_t stream);
sfn_status sfn_sparse_ffn_forward_f32_ws(const float *x, const float *A, const float *B,
                                         const float *Wg, const float *Wu, const float *Wd,
                                         float *y, uint64_t *mask, int64_t T, int d,
                                         int d_i, int r, int bank, int k, void *workspace,
                                         size_t workspace_bytes, sfn_stream_t stream);

/*
 * Per-stage timing (diagnostics; no counterpart in the paper).  Between
 * sfn_timing_begin() and sfn_timing_end(), every kernel the library launches
 * is bracketed by two CUDA events recorded on its stream.  sfn_timing_end()
 * waits for those events, then writes for each stage s < n the summed
 * kernel time in milliseconds (ms[s]) and the number of launches
 * (launches[s]); either array may be NULL.  Not for use during stream
 * capture.  Process-wide; not meant for concurrent use from several threads.
 * Stage ids are the SFN_STAGE_* values; sfn_stage_name() names them.
 */
enum {
  SFN_STAGE_PRED_H = 0,       /* h = A x                                */
  SFN_STAGE_LOGITS_TOPK = 1,  /* p = B h, bank top-k, sigma(p) of kept  */
  SFN_STAGE_FFN = 2,          /* kept gate/up/down rows -> partial y    */
  SFN_STAGE_REDUCE = 3,       /* partial rows -> y (few tokens)         */
  SFN_STAGE_BANK_TOPK = 4,    /* standalone top-k on given logits       */
  SFN_STAGE_TC_H = 5,         /* tensor cores: h = A x, split hi/lo     */
  SFN_STAGE_TC_LOGITS_TOPK = 6, /* tensor cores: logits + fused top-k   */
  SFN_STAGE_TC_GATEUP = 7,    /* tensor cores: masked sigma(p) g u      */
  SFN_STAGE_TC_DOWN = 8,      /* tensor cores: y = act W_down           */
  SFN_STAGE_DENSE4X_GATEUP = 10, /* Dense-4x: silu(g) u + amplitude top-k */
  SFN_STAGE_BWD_TAU = 11,     /* backward: mask and thresholds          */
  SFN_STAGE_BWD_ELEM = 12,    /* backward: surrogate chain rule         */
  SFN_STAGE_BWD_GEMM = 13,    /* backward: tensor-core contractions     */
  SFN_STAGE_COUNT = 16        /* room for the stage ids of this library */
};
sfn_status sfn_timing_begin(void);

/*
 * Device error word of the current device (diagnostics; no counterpart in
 * the paper).  Kernels never trap: a pipeline wait that gives up after about
 * two seconds, or a failed index check, sets a bit here and the kernel
 * returns early (its outputs are then invalid).  Bits: 1 = a bounded wait
 * timed out, 2 = an index check failed.  This call synchronises the device,
 * writes the word to *bits and, if `clear`, resets it to 0.  The word's
 * address is looked up once per device and cached; cudaDeviceReset
 * invalidates it (and every other per-device cache of the library).
 */
sfn_status sfn_device_errors(unsigned *bits, int clear);

/*
 * Self-test of the bounded waits above (diagnostics; no counterpart in the
 * paper).  Launches one warp on `stream` that waits, through the same
 * bounded-wait code as every pipeline of this library, on a shared-memory
 * barrier that nothing ever completes, giving up after `limit_cycles` SM
 * clock cycles (1 .. 10^9, about half a second at most; else
 * SFN_ERR_INVALID_VALUE).  The wait then sets bit 1 of the device error word
 * and the kernel returns; *gave_up (device int, may be NULL) receives 1 if
 * every lane gave up.  No copy or MMA is in flight, so nothing is left
 * behind: the device stays usable for later calls.
 */
sfn_status sfn_debug_wait_timeout(long long limit_cycles, int *gave_up, sfn_stream_t stream);
sfn_status sfn_timing_end(double *ms, uint64_t *launches, int n);
const char *sfn_stage_name(int stage);

#ifdef __cplusplus
}
#endif

#endif /* SFN_H_ */
