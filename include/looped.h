/* looped.h - C ABI of the B200 (sm_100a) looped weight-shared decoder.
 *
 * The method: a decoder of 32 stored layers whose block of layers 4-27 runs
 * twice with shared weights, B(B(h)), between a prelude (layers 0-3) and a
 * coda (layers 28-31, then the output head): 4 + 24 + 24 + 4 = 56 layer
 * executions per forward pass ("How Does SenseNova-Loop Get More Depth Without
 * More Parameters?", section "What is the looped decoder in SenseNova-Loop?").
 * Inside the block two residual streams are joined by manifold-constrained
 * hyper-connections whose read, mix and write maps are learned, the mix being
 * projected by 20 Sinkhorn row/column normalisations (same page, section
 * "What does two-stream mHC do?").  Each 4-layer group is 3 linear-attention
 * layers then 1 full-attention layer (same page, section "How does the hybrid
 * attention pattern work?").  Shapes: hidden 4096, FFN 12288, vocabulary
 * 248,320, contexts to 262,144 ("SenseTime's SenseNova-Loop-9B Runs Its Own
 * Layers Twice, and It's Open Source", key-specs table).
 *
 * Conventions for every call:
 *   - Status: 0 (LOOP_OK) or a negative LOOP_E* code; nothing is launched
 *     when a call fails its argument checks.  loop_last_error() gives a text.
 *   - Pointers named d_* are device pointers owned by the caller; they must
 *     stay valid until the work queued on `stream` has finished.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Every call is asynchronous on that stream; one model must not
 *     be used from two streams at once.
 *   - The model owns its weights, its KV cache / linear-attention state arena
 *     and its workspaces (device memory allocated by loop_model_create and
 *     released by loop_model_destroy).
 */
#ifndef LOOPED_H
#define LOOPED_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LOOP_API __attribute__((visibility("default")))
#else
#define LOOP_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

enum {
  LOOP_OK = 0,
  LOOP_EINVAL = -1,       /* bad argument or configuration                    */
  LOOP_ENOMEM = -2,       /* device allocation failed (nothing is leaked)      */
  LOOP_ECUDA = -3,        /* a CUDA call failed                                */
  LOOP_ERANGE = -4,       /* batch > max_batch or context > max_ctx            */
  LOOP_EUNSUPPORTED = -5, /* valid configuration this library does not run     */
  LOOP_ETIMEOUT = -6      /* a device-side wait gave up (see loop_device_status) */
};

enum { LOOP_F32 = 0, LOOP_BF16 = 1 };
enum { LOOP_TOKENS_TO_LOGITS = 0, LOOP_HIDDEN_TO_HIDDEN = 1 };
enum { LOOP_ALL_POSITIONS = 1u }; /* flag of loop_prefill, loop_extend, loop_prefill_ragged: logits for every position */
enum { LOOP_KIND_LINEAR = 0, LOOP_KIND_FULL = 1 };
enum { LOOP_REGION_PRELUDE = 0, LOOP_REGION_BLOCK = 1, LOOP_REGION_CODA = 2 };

/* The checkpoint's execution configuration: loop range, pass count and mHC
 * settings travel with the weights, because a plain layer-by-layer runner
 * would execute the wrong order ("How Does SenseNova-Loop Get More Depth
 * Without More Parameters?", section "How do you run SenseNova-Loop-9B-Preview?").
 * The loop-9B values are given in brackets. */
typedef struct {
  int32_t n_prelude, n_block, n_loops, n_coda; /* [4, 24, 2, 4]; n_prelude, n_block multiples of group */
  int32_t group, full_slot;                    /* [4, 3]: layer p is full attention iff p % group == full_slot */
  int32_t hidden, ffn, vocab;                  /* [4096, 12288, 248320]; vocab unused for HIDDEN_TO_HIDDEN */
  int32_t n_q, n_kv, head_dim;                 /* full attention, GQA [32, 8, 128] */
  int32_t n_lin, lin_dim, lin_chunk;           /* gated linear attention [32, 128, 64] */
  int32_t n_streams, sinkhorn_iters;           /* mHC [2, 20]; this library runs n_streams == 2 */
  float rope_base, norm_eps;                   /* [1e4, 1e-6] */
  int32_t dtype;                               /* LOOP_F32 or LOOP_BF16 (mHC parameters are always fp32) */
  int32_t io_mode;                             /* LOOP_TOKENS_TO_LOGITS or LOOP_HIDDEN_TO_HIDDEN */
  int32_t max_batch, max_ctx;                  /* sequences and positions per sequence the caches hold */
  int32_t kv_pages;                            /* KV pages of 64 positions in each full-attention execution's
                                                  pool; 0 = max_batch * ceil(max_ctx / 64), enough for every
                                                  sequence at max_ctx (see "KV cache" below) */
} loop_config;

/* KV cache.  Each full-attention execution keeps its keys and values in a
 * pool of pages of 64 positions; one page table per sequence, shared by all
 * executions (every execution of a sequence holds the same positions), maps
 * each block of 64 positions to a page.  A prefill (or ragged prefill) of a
 * sequence returns its pages to the pool and takes what its new length needs;
 * decode and extend take a page when a sequence crosses a block boundary.  With
 * kv_pages below max_batch * ceil(max_ctx / 64) the sequences share a smaller
 * pool (continuous batching of sequences of different lengths); a call whose
 * sequences would need more pages than are free returns LOOP_ERANGE and
 * changes nothing. */

typedef struct loop_model loop_model;

/* Number of layer executions n_prelude + n_block * n_loops + n_coda, or a
 * negative status for an invalid configuration. */
LOOP_API int32_t loop_num_exec(const loop_config* cfg);

/* Execution table (host memory, 5 int32 per execution): physical layer,
 * pass, kind (LOOP_KIND_*), cache slot, region (LOOP_REGION_*).  Prelude
 * execution e runs layer e; block execution n_prelude + p * n_block + j runs
 * layer n_prelude + j in pass p (B(B(h))); the coda runs the remaining layers.
 * The k-th full-attention execution owns KV slot k and the k-th linear one
 * owns state slot k, so each pass keeps its own caches.  Returns the number of
 * executions or a negative status. */
LOOP_API int32_t loop_schedule(const loop_config* cfg, int32_t* table);

/* Number of weight tensors in the canonical order used by loop_model_create:
 * [0] embedding [vocab][hidden] (empty for HIDDEN_TO_HIDDEN), [1] final norm
 * gain [hidden]; then per physical layer 10 tensors: attention-norm gain, W_q,
 * W_k, W_v, W_g (linear layers only; empty for full attention), W_o, FFN-norm
 * gain, W_gate, W_up, W_down (matrices stored [out][in]); then per block layer
 * and sublayer (attention, FFN) the mHC gain gamma [n*hidden] and projection
 * Phi [2n + n*n][n*hidden].  Negative status for an invalid configuration. */
LOOP_API int32_t loop_num_weights(const loop_config* cfg);

/* Create a model of the execution configuration *cfg: the loop range
 * (n_prelude, n_block, n_coda), the pass count n_loops and the mHC settings
 * that a checkpoint carries and an engine must honour ("How Does
 * SenseNova-Loop Get More Depth Without More Parameters?", section "How do you
 * run SenseNova-Loop-9B-Preview?"); the 32-layer, 56-execution shape of the
 * 9B model is the same page's section "What is the looped decoder in
 * SenseNova-Loop?".  Invalid configurations give LOOP_EINVAL, valid ones this
 * library does not run LOOP_EUNSUPPORTED.  host_weights == NULL draws every matrix from the seeded
 * SplitMix64 generator on the device (0.02 * N(0,1), rounded to the model
 * dtype; norm gains 1); otherwise host_weights[i] points to host fp32 values of
 * tensor i in the canonical order above (copied and converted; the caller
 * keeps ownership).  Allocates the weights, the per-execution KV cache and
 * linear-attention state for max_batch x max_ctx, and the workspaces.  Blocks
 * until the model is ready.  On failure *out is NULL and nothing is leaked. */
LOOP_API int32_t loop_model_create(const loop_config* cfg, const float* const* host_weights, uint64_t seed,
                          loop_model** out);

/* The looped forward pass over a prompt: embedding, prelude layers once, the
 * shared block n_loops times on its own output with the two mHC streams, the
 * coda and the tied output head ("How Does SenseNova-Loop Get More Depth
 * Without More Parameters?", section "What is the looped decoder in
 * SenseNova-Loop?"; the hybrid 3:1 linear/full attention pattern and its
 * caches from the section "How does the hybrid attention pattern work?").
 * Prefill B sequences of S tokens from position 0 (resets their caches).
 * TOKENS_TO_LOGITS: d_tokens int32 [B][S] (each in [0, vocab)); d_out fp32
 *   [B][vocab] with the logits of each sequence's last position, or
 *   [B][S][vocab] when flags has LOOP_ALL_POSITIONS.
 * HIDDEN_TO_HIDDEN: d_hidden fp32 [B][S][hidden] in, d_out fp32 [B][S][hidden]
 *   out (the collapsed streams; no embedding, final norm or head).
 * Writes each execution's KV (positions 0..S-1) and final linear-attention
 * state into its own slot; afterwards the sequences have length S.
 * LOOP_ERANGE if B > max_batch, S > max_ctx or the KV page pool cannot hold
 * the B sequences. */
LOOP_API int32_t loop_prefill(loop_model* m, const int32_t* d_tokens, const float* d_hidden, int32_t B, int32_t S,
                     float* d_out, uint32_t flags, void* stream);

/* The same looped forward pass for one new token per sequence, reading and
 * extending each execution's own KV cache and fixed-size linear-attention state
 * ("How Does SenseNova-Loop Get More Depth Without More Parameters?", sections
 * "What is the looped decoder in SenseNova-Loop?" and "How does the hybrid
 * attention pattern work?": the full-attention cache grows with the context,
 * the linear-attention state does not; both passes keep their own).
 * One decode step for sequences 0..B-1: d_tokens int32 [B] is the next token
 * of each sequence, processed at its current length; d_logits fp32 [B][vocab].
 * Appends one KV position per full-attention execution, advances every
 * linear-attention state, then adds 1 to each sequence length.
 * LOOP_ERANGE if a sequence would pass max_ctx or no KV page is free.
 * After the first step, a step's kernels are replayed from a CUDA graph
 * captured on a private stream (one per batch size and 1,024-position context
 * range; not while per-launch timing or a capture is on): the tokens are copied
 * into a model buffer first and the logits out of one afterwards, all on
 * `stream`. */
LOOP_API int32_t loop_decode_step(loop_model* m, const int32_t* d_tokens, int32_t B, float* d_logits, void* stream);

/* Append k tokens to each of sequences 0..B-1 in one pass: d_tokens int32
 * [B][k] continues each sequence at its current length, exactly as k calls of
 * loop_decode_step would, but with all k positions of a sequence in the same
 * projections (the step a multi-token-prediction or speculative-verification
 * loop runs; the pages list MTP as available for faster inference: "SenseTime's
 * SenseNova-Loop-9B Runs Its Own Layers Twice, and It's Open Source", section
 * "Running it", and "How Does SenseNova-Loop Get More Depth Without More
 * Parameters?", section "How do you run SenseNova-Loop-9B-Preview?").
 * d_out fp32 [B][vocab] (last appended position) or [B][k][vocab] with
 * LOOP_ALL_POSITIONS.  Appends k KV positions per full-attention execution,
 * advances every linear-attention state by k tokens, then adds k to each
 * sequence length.  TOKENS_TO_LOGITS models only (LOOP_EINVAL otherwise);
 * LOOP_ERANGE if a sequence would pass max_ctx, B > max_batch, the KV pages
 * would run out, or B * k
 * exceeds the model's per-call token budget (max(max_ctx, min(max_batch *
 * max_ctx, 65536)) tokens). */
LOOP_API int32_t loop_extend(loop_model* m, const int32_t* d_tokens, int32_t B, int32_t k, float* d_out,
                             uint32_t flags, void* stream);

/* Prefill sequences b0 .. b0+B-1 from position 0, each with its own length
 * h_lens[i] (host int32 [B], each in [1, max_ctx]), leaving every other
 * sequence's caches and length untouched: new requests enter free slots while
 * the others keep decoding (loop_decode_step handles sequences of different
 * lengths).  d_tokens int32, the B sequences packed one after another
 * (sum of h_lens tokens).  d_out fp32 [B][vocab] (each sequence's last
 * position) or, with LOOP_ALL_POSITIONS, the packed [sum h_lens][vocab].
 * Each sequence runs as its own pass through the same kernels as
 * loop_prefill, so its results equal a loop_prefill of that sequence alone.
 * TOKENS_TO_LOGITS models only; LOOP_ERANGE if the KV pages would run out,
 * b0 + B > max_batch or a length
 * is outside [1, max_ctx]. */
LOOP_API int32_t loop_prefill_ragged(loop_model* m, const int32_t* d_tokens, const int32_t* h_lens, int32_t b0,
                                     int32_t B, float* d_out, uint32_t flags, void* stream);

/* Sinkhorn projection of `count` n x n matrices (fp32, row-major, device):
 * P = exp(L - max L) with the library's fixed exponential (Cody-Waite
 * reduction and a degree-7 Taylor polynomial, fused multiply-adds), then
 * `iters` times: divide each row by its sum, then each column by its sum
 * (sums left to right, IEEE division).  The result is bit-identical across
 * runs and to any implementation of that same definition.  The mixing map of
 * the mHC streams ("How Does SenseNova-Loop Get More Depth Without More
 * Parameters?", section "What does two-stream mHC do?").  n in [1, 8]. */
LOOP_API int32_t mhc_sinkhorn(const float* d_logits, float* d_out, int32_t count, int32_t n, int32_t iters, void* stream);

/* One mHC read site for T tokens with n = 2 streams ("How Does SenseNova-Loop
 * Get More Depth Without More Parameters?", section "What does two-stream mHC
 * do?": how a layer reads from the streams and how they are mixed):
 *   r = sqrt(mean over both streams of s^2 + eps),  l = ((s / r) * gamma) . Phi,
 *   H_pre = sigmoid(l[0:2]), H_post = 2 sigmoid(l[2:4]),
 *   H_res = Sinkhorn_iters(exp(l[4:8] as 2 x 2)),
 *   x = H_pre[0] s_0 + H_pre[1] s_1,  x_hat = x / sqrt(mean(x^2) + eps) * gain.
 * d_streams fp32 [2][T][H] (stream 0 rows, then stream 1 rows); d_gamma fp32
 * [2H]; d_phi fp32 [8][2H] (rows pre0, pre1, post0, post1, res00, res01, res10,
 * res11); d_gain fp32 [H]; outputs d_coef fp32 [T][8] in that row order and
 * d_xhat [T][H] (xhat_dtype LOOP_F32 or LOOP_BF16).  d_scratch: device buffer
 * of at least 18 * T floats owned by the caller (partial projections; its
 * contents on entry do not matter).  H a multiple of 4, at most 6144. */
LOOP_API int32_t mhc_prologue(const float* d_streams, int64_t T, int32_t H, const float* d_gamma,
                              const float* d_phi, const float* d_gain, int32_t iters, float eps, float* d_coef,
                              void* d_xhat, int32_t xhat_dtype, float* d_scratch, void* stream);

/* mhc_prologue for callers that cannot allocate device memory: code running
 * under a framework or serving runtime whose memory pool owns every device
 * allocation, or a latency-critical path that cannot afford the implicit
 * synchronisation of cudaMalloc / cudaFree.  The pages have no counterpart;
 * this is a calling convention of the library, not part of the method.
 * Same arguments and results as mhc_prologue, without d_scratch: the scratch
 * is a fixed array of 18 x 65,536 floats (4.7 MB) compiled into the library,
 * which every GPU that loads the library holds until the process exits.
 * Allocates nothing.  T > 65,536 returns LOOP_ERANGE.  The first call on a
 * device looks up the array's device address (cudaGetSymbolAddress) with that
 * device current and keeps it until the process exits; make that first call
 * before any stream capture, and make no call on a device after a
 * cudaDeviceReset of it (the kept address is then no longer valid).  All calls
 * on a device share the array and leave their values in it; calls that
 * overlap on the GPU (for instance on two streams) race and must not be
 * issued.  No part of the array needs to start at zero. */
LOOP_API int32_t mhc_prologue_noalloc(const float* d_streams, int64_t T, int32_t H, const float* d_gamma,
                                      const float* d_phi, const float* d_gain, int32_t iters, float eps,
                                      float* d_coef, void* d_xhat, int32_t xhat_dtype, void* stream);

/* Release everything loop_model_create allocated for the execution
 * configuration (weights, the per-execution caches of both passes, workspaces;
 * "How Does SenseNova-Loop Get More Depth Without More Parameters?", section
 * "How do you run SenseNova-Loop-9B-Preview?").  Waits for the model's queued
 * work.  NULL is ignored. */
LOOP_API void loop_model_destroy(loop_model* m);

/* ---- inspection (tests and tools) ---- */

/* Current length of sequence b (host value kept in step with the device). */
LOOP_API int32_t loop_seq_len(const loop_model* m, int32_t b);

/* Copy a cache slot to d_out (device, fp32): kind LOOP_KIND_FULL gives K then
 * V, each [B][n_kv][len][head_dim]; LOOP_KIND_LINEAR gives the state
 * [B][n_lin][lin_dim][lin_dim] (S[k][v]). */
LOOP_API int32_t loop_cache_read(loop_model* m, int32_t kind, int32_t slot, int32_t B, int32_t len, float* d_out,
                        void* stream);

/* Copy weight tensor `index` (canonical order, see loop_num_weights) to d_out
 * (device, fp32) in its canonical row-major [out][in] layout. */
LOOP_API int32_t loop_weight_read(loop_model* m, int32_t index, float* d_out, void* stream);

/* Capture (tests and inspection): while armed, every forward of this model
 * (prefill, extend, decode) copies, for sequence 0 of the call and heads
 * [head0, head0 + nheads) of execution `exec`, the inputs and output of its
 * attention step into caller device buffers (model dtype; NULL skips one):
 *   linear attention: d_q, d_k, d_v [nheads][S][lin_dim] (q, k L2-normalised),
 *     d_gate fp32 [nheads][S] (log g), d_o [S][nheads * lin_dim];
 *   full attention: d_q [nheads][S][head_dim] (after RoPE), d_o as above, and
 *     d_k, d_v [nk][len][head_dim] for the nk kv heads those query heads read
 *     (len = the sequence's length after the call), copied from the cache.
 * S is the number of new tokens of the call.  Up to 8 captures can be armed;
 * exec < 0 disarms all.  The buffers must stay valid while armed. */
LOOP_API int32_t loop_capture(loop_model* m, int32_t exec, int32_t head0, int32_t nheads, void* d_q, void* d_k,
                              void* d_v, float* d_gate, void* d_o);

/* The projection primitive on its own: C[M][N] (row stride ldc, fp32) =
 * A[M][K] W[N][K]^T with A, W bf16 row-major device arrays.  use_tensor_cores
 * selects the tcgen05 kernel (K a multiple of 64; LOOP_EUNSUPPORTED otherwise)
 * or the CUDA-core kernel. */
LOOP_API int32_t loop_gemm_bf16(const void* d_A, const void* d_W, int64_t M, int64_t N, int64_t K, float* d_C,
                                int64_t ldc, int32_t use_tensor_cores, void* stream);

/* Kernel classes for loop_timing_read. */
enum {
  LOOP_K_GEMM = 0,             /* projection GEMMs and the output head */
  LOOP_K_ATTENTION = 1,        /* causal GQA attention (prefill and decode) */
  LOOP_K_LINEAR_ATTENTION = 2, /* gated linear attention */
  LOOP_K_MHC = 3,              /* mHC prologue */
  LOOP_K_NORM = 4,             /* RMSNorm, embedding, stream expand/collapse */
  LOOP_K_OTHER = 5,
  LOOP_K_CLASSES = 6
};

/* Enable (1) or disable (0) per-launch timing: while enabled every kernel
 * the model launches is bracketed by CUDA events on its stream. */
LOOP_API int32_t loop_set_timing(loop_model* m, int32_t enable);

/* Totals for kernel class `cls` since the last reset: device time in ms,
 * launches, and algorithmic work (FLOPs for LOOP_K_GEMM, LOOP_K_ATTENTION and
 * LOOP_K_LINEAR_ATTENTION; bytes that must move for the others).  Waits for
 * the recorded events.  reset != 0 clears the totals afterwards. */
LOOP_API int32_t loop_timing_read(loop_model* m, int32_t cls, double* total_ms, int64_t* launches, double* work,
                                  int32_t reset);

/* Number of kernels this model has launched since it was created. */
LOOP_API int64_t loop_launch_count(const loop_model* m);

/* Sticky device status word: 0, or bits for what went wrong in a kernel: 1
 * TMA producer wait, 2 MMA-issuer wait, 4 epilogue / consumer wait, 8 other
 * wait timed out (the kernel then returned early); 16 a token id outside
 * [0, vocab) was embedded as zeros; 32 the self-test timeout fired.  Reading it synchronises the
 * device.  loop_clear_device_status() resets it. */
LOOP_API int32_t loop_device_status(void);
LOOP_API void loop_clear_device_status(void);

/* Failure-detection self-test: one kernel waits on an mbarrier phase that
 * never completes, with a limit of timeout_ms; the wait gives up, records bit
 * 32 (self-test) in the status word and the kernel returns normally, so the
 * context stays usable.  Synchronises; returns the status word (the caller
 * clears it with loop_clear_device_status) or a negative LOOP_E* code. */
LOOP_API int32_t loop_selftest_timeout(int32_t timeout_ms);

/* Text of the last failed call on this thread ("" if none). */
LOOP_API const char* loop_last_error(void);

#ifdef __cplusplus
}
#endif
#endif
