/* Oracle for the looped weight-shared decoder: TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow CPU forward pass (fp64 arithmetic, fp32 storage) of the
 * SenseNova-Loop-style looped decoder, written from the method's description:
 *   - looped execution B(B(h)): layers 0-3 once, the shared block 4-27 twice,
 *     layers 28-31 and the output head once, 56 executions from 32 stored
 *     layers ("SenseTime's Loop-9B runs its own layers twice", section "The
 *     trick: run the middle of the network twice"; "How Does SenseNova-Loop
 *     Get More Depth Without More Parameters?", section "What is the looped
 *     decoder in SenseNova-Loop?");
 *   - two-stream mHC with read / mix / write maps, the mix projected by 20
 *     Sinkhorn normalisations (same explainer, section "What does two-stream
 *     mHC do?");
 *   - 3 linear-attention layers then 1 full-attention layer per 4-layer group
 *     (same explainer, section "How does the hybrid attention pattern work?").
 * Everything the pages leave open (the linear-attention variant, head
 * counts, norms, the mHC parameterisation) follows the workload definitions
 * the library is built for; each choice is listed in the design notes.
 *
 * Only tests/, the smoke entry and the bench's CPU-baseline leg may load this
 * library.  It shares no code with the CUDA library.
 */
#ifndef LOOP_ORACLE_H
#define LOOP_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Field-for-field the same layout as the CUDA library's loop_config: both
 * describe the checkpoint's execution configuration (loop range, pass count,
 * mHC settings), so the two must agree on it. */
typedef struct {
  int32_t n_prelude, n_block, n_loops, n_coda;
  int32_t group, full_slot;
  int32_t hidden, ffn, vocab;
  int32_t n_q, n_kv, head_dim;
  int32_t n_lin, lin_dim, lin_chunk;
  int32_t n_streams, sinkhorn_iters;
  float rope_base, norm_eps;
  int32_t dtype;   /* 0 = fp32 everywhere, 1 = bf16 weights and GEMM operands */
  int32_t io_mode; /* 0 = tokens -> logits, 1 = hidden -> hidden             */
  int32_t max_batch, max_ctx;
  int32_t kv_pages; /* the library's KV page-pool size; the oracle keeps a dense cache and ignores it */
} oracle_config;

enum { ORACLE_FULL = 1, ORACLE_LINEAR = 0 };
enum { ORACLE_PRELUDE = 0, ORACLE_BLOCK = 1, ORACLE_CODA = 2 };
enum { ORACLE_ALL_POSITIONS = 1 };

/* generator (SplitMix64, counter based) */
uint64_t oracle_rng_u64(uint64_t seed, uint64_t stream, uint64_t j);
double oracle_rng_normal(uint64_t seed, uint64_t stream, uint64_t i);

/* spec-defined exponential and Sinkhorn */
float oracle_exp_spec(float x);
void oracle_sinkhorn_f32(const float* logits, float* out, int64_t count, int32_t n, int32_t iters);
void oracle_sinkhorn_f64(const double* logits, double* out, int64_t count, int32_t n, int32_t iters);

/* execution table: per execution 5 ints (phys, pass, kind, slot, region) */
int32_t oracle_num_exec(const oracle_config* c);
int32_t oracle_schedule(const oracle_config* c, int32_t* table);

/* unit operations (fp64), exposed for the pins */
void oracle_rmsnorm(const double* x, const double* gain, double* y, int64_t rows, int32_t dim, double eps);
void oracle_gla_recurrent(const double* q, const double* k, const double* v, const double* g,
                          double* o, double* state, int32_t T, int32_t dk, int32_t dv);
void oracle_attention_naive(const double* q, const double* k, const double* v, double* o,
                            int32_t Tq, int32_t Tk, int32_t q0, int32_t d);
void oracle_rope(double* x, int32_t T, int32_t n_heads, int32_t d, const int32_t* pos, double base);
void oracle_mhc_site(const double* s, const double* gamma_m, const double* phi, const double* gain,
                     int32_t n, int32_t H, int32_t iters, double eps, double* coef, double* xhat);
void oracle_mhc_write(double* s, const double* coef, const double* y, int32_t n, int32_t H);

/* the model's three sublayers on caller arrays (the model runs the same
 * functions): full attention (K/V cache slot [B][n_kv][max_ctx][head_dim],
 * appended at start[b] ..), gated linear attention (state [B][n_lin][d][d],
 * updated in place) and the SwiGLU FFN; xh and y are [B*S][hidden] fp64 */
int32_t oracle_attention_sublayer(const oracle_config* c, const float* wq, const float* wk, const float* wv,
                                  const float* wo, float* kcache, float* vcache, const double* xh, int32_t B,
                                  int32_t S, const int32_t* start, double* y);
int32_t oracle_gla_sublayer(const oracle_config* c, const float* wq, const float* wk, const float* wv,
                            const float* wg, const float* wo, double* state, const double* xh, int32_t B, int32_t S,
                            double* y);
int32_t oracle_ffn_sublayer(const oracle_config* c, const float* w_gate, const float* w_up, const float* w_down,
                            const double* xh, int64_t T, double* y);

/* whole model */
void* oracle_model_create(const oracle_config* c, uint64_t seed, const float* const* weights);
int32_t oracle_num_weights(const oracle_config* c);
int64_t oracle_weight_numel(void* m, int32_t index);
int32_t oracle_get_weight(void* m, int32_t index, float* out);
int32_t oracle_prefill(void* m, const int32_t* tokens, const float* hidden, int32_t B, int32_t S,
                       float* out, uint32_t flags);
int32_t oracle_decode_step(void* m, const int32_t* tokens, int32_t B, float* logits);
int32_t oracle_seq_len(void* m, int32_t b);
/* copies slot `slot` of the KV cache (kind FULL: K then V, [B][n_kv][len][d]) or
 * the GLA state (kind LINEAR: [B][n_lin][dk][dv]) for sequences 0..B-1 */
int32_t oracle_cache_read(void* m, int32_t kind, int32_t slot, int32_t B, int32_t len, float* out);
/* test-only: load a cache slot (the layout of oracle_cache_read), set a
 * sequence's length, replace a weight tensor */
int32_t oracle_cache_write(void* m, int32_t kind, int32_t slot, int32_t B, int32_t len, const float* in);
int32_t oracle_set_seq_len(void* m, int32_t b, int32_t len);
int32_t oracle_set_weight(void* m, int32_t index, const float* in);
void oracle_model_destroy(void* m);

#ifdef __cplusplus
}
#endif
#endif
