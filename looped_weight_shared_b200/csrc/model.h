// Internal declarations of the looped-decoder library: the model object, its
// workspace, and the launchers each kernel file provides.
#pragma once

#include <cuda_runtime.h>

#include <atomic>
#include <string>
#include <vector>

#include "../../include/looped.h"
#include "common.cuh"

namespace loopk {

// Raise a kernel's dynamic shared-memory limit on the current device, once per
// device (the setting belongs to that device's context); `done` is the
// caller's per-kernel bitmask of devices already set.
template <typename F>
cudaError_t set_smem_limit(F* kernel, int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

// Output modes of a projection (a GEMM C = A W^T plus what follows it).
enum class Epi {
  F32,         // C fp32 [M][N] (row stride ldc) - logits
  RESID,       // h[M][H] += C                     (prelude / coda residual)
  MHC_WRITE,   // s_i = sum_j res[i][j] s_j + post[i] C   (two streams)
  SWIGLU,      // a[M][F] = silu(C gate) * C up; weight rows interleaved per 128
  QKV_LINEAR,  // q, k (L2-normalised), v -> [B][n_lin][S][d]; log sigmoid(gate) -> [B][n_lin][S]
  QKV_FULL,    // RoPE(q) -> [B][n_q][S][hd]; RoPE(k), v -> cache [B][n_kv][max_ctx][hd]
};

struct EpiArgs {
  Epi mode = Epi::F32;
  float* c = nullptr;  // F32: output; RESID: h
  int64_t ldc = 0;
  float* s = nullptr;  // MHC_WRITE: streams [2][M][H]
  const float* coef = nullptr;  // MHC_WRITE: [M][8]
  void* a = nullptr;            // SWIGLU output [M][F]
  void* q = nullptr;            // QKV: q [B][heads][S][d]
  void* k = nullptr;            // QKV_LINEAR: k; QKV_FULL: this execution's K page pool
  void* v = nullptr;            // QKV_LINEAR: v; QKV_FULL: V page pool
  float* gl = nullptr;          // QKV_LINEAR: log-gates [B][n_lin][S]
  const float2* rope = nullptr; // QKV_FULL: (cos, sin) [max_ctx][hd/2]
  const int32_t* start = nullptr;  // QKV_FULL: start position of each sequence
  int S = 1;                    // tokens per sequence in this call
  int heads_q = 0, heads_kv = 0, hd = 0;
  const int32_t* table = nullptr;  // QKV_FULL: KV page table of the call's first sequence
  int pps = 0;                     // QKV_FULL: pages per sequence (table row stride)
  int n_lin = 0;
  float eps = 1e-6f;
  // MHC_WRITE on the tensor-core path: also the next mHC site's partial
  // projections of the new streams (next_phig = that site's Phi * gamma,
  // [8][2H]), written to part [M][2 N / 256][9]; NULL: none
  const float* next_phig = nullptr;
  float* part = nullptr;
};

struct LayerW {
  bool full = false;
  void* w_in = nullptr;   // linear: [3 n_lin d + n_lin][H] (q | k | v | gate); full: [(n_q + 2 n_kv) hd][H]
  void* w_o = nullptr;    // [H][n d]
  void* w_gu = nullptr;   // [2F][H]: block j of 256 rows = gate rows 128j.. then up rows 128j..
  void* w_down = nullptr; // [H][F]
  float* attn_gain = nullptr;
  float* ffn_gain = nullptr;
  int64_t n_in = 0, n_o_in = 0;
};

struct SiteW {
  float* gamma = nullptr;  // [2H]
  float* phi = nullptr;    // [8][2H]
  float* phig = nullptr;   // [8][2H] Phi * gamma entry by entry (for projections formed in a GEMM epilogue)
};

struct Work {
  int64_t t_max = 0;
  float* h = nullptr;       // [T][H]
  float* s = nullptr;       // [2][T][H]
  void* xh = nullptr;       // [T][H]
  float* coef = nullptr;    // [T][8]
  void* q = nullptr;        // [T][max(n_q hd, n_lin d)]
  void* k = nullptr;        // [T][n_lin d]
  void* v = nullptr;        // [T][n_lin d]
  float* gl = nullptr;      // [T][n_lin]
  void* o = nullptr;        // [T][max(n_q hd, n_lin d)]
  void* a = nullptr;        // [T][F]
  float* cbuf = nullptr;    // [T][max N] projection scratch of the unfused path
  void* xf = nullptr;       // [rows][H] final-norm output
  int32_t* zeros = nullptr; // start positions of a prefill (all 0)
  float* mhc_part = nullptr;  // [T][parts][9] partial projections of the mHC prologue
  int64_t mhc_part_floats = 0;
  bool part_formed = false;   // the last projection also wrote the next site's partials into mhc_part
  float* cpart = nullptr;     // split-K partial sums of the decode GEMM [32][64][max N]
  int64_t cpart_floats = 0;
  float* dec_attn = nullptr;  // decode attention chunk partials [B][n_q][ctx / 128][130]
  float* gla_seg = nullptr;   // segment states of a segmented linear-attention prefill
  int64_t gla_seg_floats = 0;
};

// One armed capture of an execution's attention inputs and outputs (test and
// inspection hook, see loop_capture).
struct Capture {
  int exec = -1, head0 = 0, nheads = 0;
  void* q = nullptr;
  void* k = nullptr;
  void* v = nullptr;
  float* g = nullptr;
  void* o = nullptr;
};

struct TimedLaunch {
  int cls;
  double work;
  cudaEvent_t a, b;
};

struct Model {
  loop_config c{};
  // launch accounting
  int64_t launches = 0;
  bool timing = false;
  std::vector<TimedLaunch> pending;
  std::vector<cudaEvent_t> event_pool;
  double t_ms[LOOP_K_CLASSES] = {};
  double t_work[LOOP_K_CLASSES] = {};
  int64_t t_count[LOOP_K_CLASSES] = {};
  int n_phys = 0, n_exec = 0, n_full = 0, n_lin = 0;
  std::vector<int32_t> table;
  size_t esize = 4;
  void* embed = nullptr;
  float* final_gain = nullptr;
  std::vector<LayerW> L;
  std::vector<SiteW> sites;
  std::vector<void*> kc, vc;    // per full-attention slot: page pool [n_pages][n_kv][KV_PAGE][hd]
  int pps = 0;                  // KV pages per sequence: ceil(max_ctx / KV_PAGE)
  int n_pages = 0;              // pages in each execution's pool
  int32_t* d_table = nullptr;   // [max_batch][pps] page of each block of KV_PAGE positions (all slots)
  std::vector<int32_t> h_table; // host copy
  std::vector<int32_t> n_held;  // pages each sequence holds
  std::vector<int32_t> free_pages;
  std::vector<float*> st;       // per linear slot [max_batch][n_lin][d][d] fp32
  int32_t* d_seq_len = nullptr;
  std::vector<int32_t> seq_len;
  float2* rope = nullptr;       // [max_ctx][hd/2]
  Work w;
  std::vector<void*> allocs;
  bool use_tc = false;          // tcgen05 path for bf16 projections
  bool decoding = false;        // inside loop_decode_step: projections use the decode GEMM
  bool extending = false;       // inside loop_extend: sequences start past 0 (attention starts at seq_len)
  std::vector<Capture> captures;
  // decode steps replayed from CUDA graphs: one graph per (batch, decode-
  // attention chunk count), captured on a private stream after one eager step
  struct DecodeGraph {
    int B = 0, nch = 0;
    int64_t kernels = 0;
    cudaGraphExec_t exec = nullptr;
  };
  std::vector<DecodeGraph> graphs;
  cudaStream_t cap_stream = nullptr;
  bool decoded_eagerly = false;
  int32_t* dec_tok = nullptr;   // [max_batch] the step's tokens (graph input)
  float* dec_logits = nullptr;  // [max_batch][vocab] the step's logits (graph output)
};

bool bf16_model(const Model& m);

// Record the text loop_last_error() returns on this thread.
void set_last_error(const std::string& msg);

// Device address of the library's status word (this device), or NULL.
int* status_ptr();
int status_read();
void status_clear();

// ---- launchers (each returns cudaGetLastError()) ----
cudaError_t launch_fill_normal(void* dst, bool bf16, int64_t rows, int64_t cols, int64_t dst_row0,
                               uint64_t seed, uint64_t stream, int64_t src_row0, double scale, cudaStream_t st);
cudaError_t launch_fill_const(float* dst, int64_t n, float v, cudaStream_t st);
cudaError_t launch_embed(const int32_t* tok, const void* E, bool bf16, int64_t T, int H, int V, float* h,
                         cudaStream_t st);
cudaError_t launch_rmsnorm(const float* x, int64_t rows, int H, int64_t row_step, int64_t row_off,
                           const float* gain, float eps, void* y, bool bf16, cudaStream_t st);
// two or three kernels; `part` is scratch of 9 x parts floats per token
// (parts even, dividing the stream width into equal float4 runs; 2 by
// default).  fused_read selects the reader that forms the coefficients
// itself (fewer launches for a few tokens) at every width; otherwise hidden
// 4096 uses a coefficient kernel and a one-pass reader.
cudaError_t launch_mhc_prologue(const float* s, int64_t T, int H, const float* gamma, const float* phi,
                                const float* gain, int iters, float eps, float* coef, void* xh, bool bf16,
                                float* part, cudaStream_t st, int parts = 2, bool fused_read = false);
size_t mhc_partial_smem(int H);
// out[c][i] = phi[c][i] * gamma[i], c < 8, i < D
cudaError_t launch_mhc_phig(const float* gamma, const float* phi, int64_t D, float* out, cudaStream_t st);
// hidden 4096, the partial projections already formed ([T][parts][9], summed
// in part order, e.g. by the mHC-write epilogue of the projection before):
// the coefficient kernel and the one-pass reader
cudaError_t launch_mhc_coef_read(const float* part, int parts, const float* s, int64_t T, int H, const float* gain,
                                 int iters, float eps, float* coef, void* xh, bool bf16, cudaStream_t st);
// one launch per site for a few tokens (decode), hidden 4096
bool mhc_token_supported(int H);
cudaError_t launch_mhc_token(const float* s, int64_t T, int H, const float* gamma, const float* phi,
                             const float* gain, int iters, float eps, float* coef, void* xh, bool bf16, cudaStream_t st);
cudaError_t launch_expand(const float* h, float* s, int64_t n, cudaStream_t st);
cudaError_t launch_collapse(const float* s, float* h, int64_t n, cudaStream_t st);
cudaError_t launch_sinkhorn(const float* l, float* out, int64_t count, int n, int iters, cudaStream_t st);

cudaError_t launch_gemm_simt(const void* A, const void* W, bool bf16, int64_t M, int64_t N, int64_t K,
                             float* C, int64_t ldc, cudaStream_t st);
// C holds `splits` slices of M x ldc (split-K partial sums, added in order).
cudaError_t launch_epilogue_unfused(const float* C, int64_t ldc, int64_t M, int64_t N, const EpiArgs& e, bool bf16,
                                    cudaStream_t st, int splits = 1);
cudaError_t launch_attention_simple(const void* q, const void* K, const void* V, void* o, bool bf16, int B, int S,
                                    int nq, int nkv, int hd, const int32_t* table, int pps, const int32_t* start,
                                    cudaStream_t st);
cudaError_t launch_gla_recurrent(const void* q, const void* k, const void* v, const float* gl, float* state, void* o,
                                 bool bf16, int B, int S, int nh, int d, cudaStream_t st);
cudaError_t launch_rope_table(float2* tab, int64_t ctx, int hd, double base, cudaStream_t st);
// K or V of sequences 0..B-1, positions 0..len-1 -> dst fp32 [B][nkv][len][hd]
cudaError_t launch_cache_to_f32(const void* src, bool bf16, const int32_t* table, int pps, int B, int nkv, int len,
                                int hd, float* dst, cudaStream_t st);
// K or V rows 0..len-1 of sequence b, kv head h -> dst [len][hd] in the model dtype
cudaError_t launch_cache_rows(const void* src, size_t esize, const int32_t* table, int pps, int nkv, int b, int h,
                              int len, int hd, void* dst, cudaStream_t st);
// set table[idx[i]] = page[i] for n entries (passed by value)
cudaError_t launch_table_set(int32_t* table, const int32_t* idx, const int32_t* page, int n, cudaStream_t st);
cudaError_t launch_advance(int32_t* seq_len, int B, cudaStream_t st, int by = 1);
cudaError_t launch_selftest_timeout(uint64_t limit_ns, int* result, cudaStream_t st);
cudaError_t launch_set_len(int32_t* seq_len, int B, int S, cudaStream_t st);
cudaError_t launch_weight_to_f32(const void* src, bool bf16, int64_t rows, int64_t cols, int64_t src_row0,
                                 float* dst, cudaStream_t st);

// flash attention on tcgen05 (bf16, head_dim 128) for S queries per sequence
// at positions start[b] .. (start NULL: from 0)
bool flash_tc_supported(int hd, int nq, int nkv);
cudaError_t launch_flash_tc(const void* q, const void* K, const void* V, void* o, int B, int S, int nq, int nkv,
                            const int32_t* table, int pps, int64_t pool_rows, const int32_t* start, cudaStream_t st);

// decode attention (flash-decoding over 1024-key chunks; bf16, head_dim 128, group 4)
bool decode_attention_supported(int hd, int nq, int nkv);
int decode_attention_chunks(int max_len);  // grid width for the longest sequence
int64_t decode_attention_scratch_floats(int B, int nq, int64_t ctx);
cudaError_t launch_attention_decode(const void* q, const void* K, const void* V, void* o, int B, int nq, int nkv,
                                    const int32_t* table, int pps, int64_t pool_rows, int max_len,
                                    const int32_t* start, float* scratch, cudaStream_t st);

// chunked gated linear attention for prefill (bf16, d = 128)
bool gla_chunk_supported(int d);
// seg_scratch (may be NULL, scratch_floats floats) lets a small batch run as
// parallel segments of each sequence
cudaError_t launch_gla_chunked(const void* q, const void* k, const void* v, const float* gl, float* state, void* o,
                               int B, int S, int nh, float* seg_scratch, int64_t scratch_floats, cudaStream_t st);

// one decode step of gated linear attention (bf16, d = 128)
cudaError_t launch_gla_decode(const void* q, const void* k, const void* v, const float* gl, float* state, void* o,
                              int B, int nh, cudaStream_t st);

// tcgen05 GEMM (bf16): C = A[M][K] W[N][K]^T with a fused epilogue.  Returns
// cudaErrorNotSupported when the shapes are outside what it handles.
cudaError_t launch_gemm_tc(const void* A, const void* W, int64_t M, int64_t N, int64_t K, const EpiArgs& e,
                           cudaStream_t st);
bool gemm_tc_supported(int64_t M, int64_t N, int64_t K, const EpiArgs& e);

// decode GEMM (M <= 64 tokens): swap-AB, split-K; P[split][M][ldp] fp32 partials
bool gemm_skinny_supported(int64_t M, int64_t N, int64_t K);
int gemm_skinny_splits(int64_t N, int64_t K);
cudaError_t launch_gemm_skinny(const void* X, const void* W, int64_t M, int64_t N, int64_t K, int splits, float* P,
                               int64_t ldp, cudaStream_t st);

}  // namespace loopk
