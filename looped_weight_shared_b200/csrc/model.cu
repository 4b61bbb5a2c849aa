// C ABI of the looped decoder: configuration checks, the execution table,
// weight storage and generation, the cache arena, and the scheduler that runs
// the 56 layer executions of a forward pass.
//
// Looped execution follows "How Does SenseNova-Loop Get More Depth Without
// More Parameters?", section "What is the looped decoder in SenseNova-Loop?":
// prelude layers once, the shared block n_loops times on its own output,
// then the coda and the output head.  Inside the block the residual is two
// mHC streams (section "What does two-stream mHC do?"); the streams start as
// copies of h at the block entry and are summed back into h at its exit.

#include <cuda.h>

#include <algorithm>
#include <cstring>
#include <memory>
#include <string>
#include <vector>

#include "model.h"

namespace loopk {

namespace {

thread_local std::string g_last_error;

int32_t fail(int32_t code, const std::string& msg) {
  g_last_error = msg;
  return code;
}

#define LOOP_CU(call)                                                                       \
  do {                                                                                      \
    cudaError_t e_ = (call);                                                                \
    if (e_ != cudaSuccess) return fail(LOOP_ECUDA, std::string(#call) + ": " + cudaGetErrorString(e_)); \
  } while (0)

enum Slot { W_ATTN_GAIN, W_Q, W_K, W_V, W_G, W_O, W_FFN_GAIN, W_GATE, W_UP, W_DOWN, W_PER_LAYER };

constexpr uint64_t kStreamEmbed = 1;
uint64_t layer_stream(int layer, int kind) { return 1000 + 100 * (uint64_t)layer + kind; }
uint64_t site_stream(int site) { return 100000 + 10 * (uint64_t)site + 1; }

bool valid(const loop_config* c) {
  if (!c) return false;
  if (c->n_prelude < 0 || c->n_block <= 0 || c->n_loops <= 0 || c->n_coda < 0) return false;
  if (c->group <= 0 || c->full_slot < 0 || c->full_slot >= c->group) return false;
  if (c->n_prelude % c->group != 0 || c->n_block % c->group != 0) return false;
  if (c->hidden <= 0 || c->ffn <= 0 || c->n_streams <= 0 || c->sinkhorn_iters < 0) return false;
  if (c->n_q <= 0 || c->n_kv <= 0 || c->n_q % c->n_kv != 0 || c->head_dim <= 0 || c->head_dim % 2 != 0) return false;
  if (c->n_lin <= 0 || c->lin_dim <= 0 || c->lin_chunk <= 0) return false;
  if (c->dtype != LOOP_F32 && c->dtype != LOOP_BF16) return false;
  if (c->io_mode != LOOP_TOKENS_TO_LOGITS && c->io_mode != LOOP_HIDDEN_TO_HIDDEN) return false;
  if (c->io_mode == LOOP_TOKENS_TO_LOGITS && c->vocab <= 0) return false;
  if (c->max_batch <= 0 || c->max_ctx <= 0 || c->kv_pages < 0) return false;
  if (!(c->norm_eps >= 0.f) || !(c->rope_base > 0.f)) return false;
  return true;
}

// What this library runs (valid configurations outside it are LOOP_EUNSUPPORTED).
const char* unsupported(const loop_config* c) {
  if (c->n_streams != 2) return "this library runs n_streams == 2";
  if (c->hidden % 4 != 0) return "hidden must be a multiple of 4";
  if (c->hidden > 6144) return "hidden must be <= 6144 (mHC prologue keeps Phi in shared memory)";
  if (c->ffn % 128 != 0) return "ffn must be a multiple of 128";
  if (c->head_dim != 32 && c->head_dim != 64 && c->head_dim != 128) return "head_dim must be 32, 64 or 128";
  if ((size_t)c->lin_dim * c->lin_dim * 4 + 8 * (size_t)c->lin_dim > 232448)
    return "lin_dim must be <= 240 (the recurrent kernel keeps the state in shared memory)";
  return nullptr;
}

int64_t weight_rows(const loop_config& c, int index, int64_t* cols) {
  const int n_phys = c.n_prelude + c.n_block + c.n_coda;
  const int64_t H = c.hidden, F = c.ffn;
  *cols = H;
  if (index == 0) return c.io_mode == LOOP_TOKENS_TO_LOGITS ? c.vocab : 0;
  if (index == 1) { *cols = 1; return H; }
  int i = index - 2;
  if (i < W_PER_LAYER * n_phys) {
    const int phys = i / W_PER_LAYER, slot = i % W_PER_LAYER;
    const bool full = phys % c.group == c.full_slot;
    const int64_t nq = full ? (int64_t)c.n_q * c.head_dim : (int64_t)c.n_lin * c.lin_dim;
    const int64_t nkv = full ? (int64_t)c.n_kv * c.head_dim : (int64_t)c.n_lin * c.lin_dim;
    switch (slot) {
      case W_ATTN_GAIN: case W_FFN_GAIN: *cols = 1; return H;
      case W_Q: return nq;
      case W_K: case W_V: return nkv;
      case W_G: return full ? 0 : c.n_lin;
      case W_O: *cols = nq; return H;
      case W_GATE: case W_UP: return F;
      case W_DOWN: *cols = F; return H;
    }
  }
  i -= W_PER_LAYER * n_phys;
  const int64_t n = c.n_streams;
  if (i < 4 * c.n_block) {
    if (i % 2 == 0) { *cols = 1; return n * H; }
    *cols = n * H;
    return 2 * n + n * n;
  }
  return -1;
}

uint16_t bf16_bits_rne(float x) {
  uint32_t b;
  std::memcpy(&b, &x, 4);
  if ((b & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((b >> 16) | 0x40);  // NaN stays NaN
  b += 0x7FFFu + ((b >> 16) & 1u);
  return (uint16_t)(b >> 16);
}

}  // namespace

bool bf16_model(const Model& m) { return m.c.dtype == LOOP_BF16; }

void set_last_error(const std::string& msg) { g_last_error = msg; }

}  // namespace loopk

using namespace loopk;

struct loop_model {
  Model m;
};

namespace {

int32_t build_table(const loop_config* c, int32_t* table) {
  const int n_exec = c->n_prelude + c->n_block * c->n_loops + c->n_coda;
  int nf = 0, nl = 0;
  for (int e = 0; e < n_exec; ++e) {
    int phys, pass, region;
    if (e < c->n_prelude) {
      phys = e; pass = 0; region = LOOP_REGION_PRELUDE;
    } else if (e < c->n_prelude + c->n_block * c->n_loops) {
      const int j = e - c->n_prelude;
      pass = j / c->n_block;
      phys = c->n_prelude + j % c->n_block;
      region = LOOP_REGION_BLOCK;
    } else {
      phys = c->n_prelude + c->n_block + (e - c->n_prelude - c->n_block * c->n_loops);
      pass = 0;
      region = LOOP_REGION_CODA;
    }
    const int kind = (phys % c->group == c->full_slot) ? LOOP_KIND_FULL : LOOP_KIND_LINEAR;
    int32_t* row = table + 5 * e;
    row[0] = phys;
    row[1] = pass;
    row[2] = kind;
    row[3] = kind == LOOP_KIND_FULL ? nf++ : nl++;
    row[4] = region;
  }
  return n_exec;
}

void release(Model& m) {
  if (!m.allocs.empty()) cudaDeviceSynchronize();
  for (auto& g : m.graphs)
    if (g.exec) cudaGraphExecDestroy(g.exec);
  m.graphs.clear();
  if (m.cap_stream) cudaStreamDestroy(m.cap_stream);
  m.cap_stream = nullptr;
  for (void* p : m.allocs) cudaFree(p);
  m.allocs.clear();
  for (auto& t : m.pending) {
    cudaEventDestroy(t.a);
    cudaEventDestroy(t.b);
  }
  m.pending.clear();
  for (auto e : m.event_pool) cudaEventDestroy(e);
  m.event_pool.clear();
}

void* dev_alloc(Model& m, size_t bytes) {
  if (bytes == 0) bytes = 16;
  void* p = nullptr;
  if (cudaMalloc(&p, bytes) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  m.allocs.push_back(p);
  return p;
}

// Copy rows [src_row0, +rows) of a host fp32 matrix into rows [dst_row0, ...)
// of a device matrix of the model dtype.
int32_t put_rows(Model& m, void* dst, int64_t dst_row0, int64_t cols, const float* src, int64_t src_row0,
                 int64_t rows, bool keep_f32) {
  const int64_t n = rows * cols;
  if (n == 0) return LOOP_OK;
  if (bf16_model(m) && !keep_f32) {
    std::vector<uint16_t> tmp(n);
    for (int64_t i = 0; i < n; ++i) tmp[i] = bf16_bits_rne(src[src_row0 * cols + i]);
    LOOP_CU(cudaMemcpy((uint16_t*)dst + dst_row0 * cols, tmp.data(), n * 2, cudaMemcpyHostToDevice));
  } else {
    LOOP_CU(cudaMemcpy((float*)dst + dst_row0 * cols, src + src_row0 * cols, n * 4, cudaMemcpyHostToDevice));
  }
  return LOOP_OK;
}

// Fill the rows of one canonical tensor either from the caller's host values
// or from its seeded stream.
int32_t fill_rows(Model& m, const float* const* hw, uint64_t seed, int index, uint64_t stream, void* dst,
                  int64_t dst_row0, int64_t src_row0, int64_t rows, int64_t cols) {
  if (rows == 0) return LOOP_OK;
  if (hw) {
    if (!hw[index]) return fail(LOOP_EINVAL, "weights[" + std::to_string(index) + "] is NULL");
    return put_rows(m, dst, dst_row0, cols, hw[index], src_row0, rows, false);
  }
  LOOP_CU(launch_fill_normal(dst, bf16_model(m), rows, cols, dst_row0, seed, stream, src_row0, 0.02, 0));
  return LOOP_OK;
}

int32_t fill_f32(Model& m, const float* const* hw, uint64_t seed, int index, uint64_t stream, float* dst, int64_t n,
                 bool ones) {
  if (hw) {
    if (!hw[index]) return fail(LOOP_EINVAL, "weights[" + std::to_string(index) + "] is NULL");
    return put_rows(m, dst, 0, n, hw[index], 0, 1, true);
  }
  if (ones) LOOP_CU(launch_fill_const(dst, n, 1.0f, 0));
  else LOOP_CU(launch_fill_normal(dst, false, 1, n, 0, seed, stream, 0, 0.02, 0));
  return LOOP_OK;
}

int32_t create_impl(const loop_config* cfg, const float* const* hw, uint64_t seed, Model& m) {
  const loop_config& c = *cfg;
  m.c = c;
  m.n_phys = c.n_prelude + c.n_block + c.n_coda;
  m.n_exec = c.n_prelude + c.n_block * c.n_loops + c.n_coda;
  m.table.resize(5 * m.n_exec);
  build_table(cfg, m.table.data());
  for (int e = 0; e < m.n_exec; ++e) (m.table[5 * e + 2] == LOOP_KIND_FULL ? m.n_full : m.n_lin)++;
  const bool bf = c.dtype == LOOP_BF16;
  m.esize = bf ? 2 : 4;
  const int64_t H = c.hidden, F = c.ffn, es = m.esize;
  const int64_t nl = c.n_lin, ld = c.lin_dim, nq = c.n_q, nkv = c.n_kv, hd = c.head_dim;
  m.use_tc = bf;
  int32_t rc;
#define LOOP_ALLOC(ptr, type, bytes)                                              \
  do {                                                                            \
    ptr = (type)dev_alloc(m, (size_t)(bytes));                                    \
    if (!ptr) return fail(LOOP_ENOMEM, std::string("cudaMalloc failed: ") + #ptr); \
  } while (0)
#define LOOP_RC(x) \
  do {             \
    rc = (x);      \
    if (rc != LOOP_OK) return rc; \
  } while (0)

  // embedding / final norm
  if (c.io_mode == LOOP_TOKENS_TO_LOGITS) {
    LOOP_ALLOC(m.embed, void*, (int64_t)c.vocab * H * es);
    LOOP_RC(fill_rows(m, hw, seed, 0, kStreamEmbed, m.embed, 0, 0, c.vocab, H));
  }
  LOOP_ALLOC(m.final_gain, float*, H * 4);
  LOOP_RC(fill_f32(m, hw, seed, 1, 0, m.final_gain, H, true));
  // layers
  m.L.resize(m.n_phys);
  for (int p = 0; p < m.n_phys; ++p) {
    LayerW& L = m.L[p];
    const int wi = 2 + W_PER_LAYER * p;
    L.full = p % c.group == c.full_slot;
    const int64_t nqr = L.full ? nq * hd : nl * ld, nkr = L.full ? nkv * hd : nl * ld;
    L.n_in = nqr + 2 * nkr + (L.full ? 0 : nl);
    L.n_o_in = nqr;
    LOOP_ALLOC(L.attn_gain, float*, H * 4);
    LOOP_ALLOC(L.ffn_gain, float*, H * 4);
    LOOP_ALLOC(L.w_in, void*, L.n_in * H * es);
    LOOP_ALLOC(L.w_o, void*, H * nqr * es);
    LOOP_ALLOC(L.w_gu, void*, 2 * F * H * es);
    LOOP_ALLOC(L.w_down, void*, H * F * es);
    LOOP_RC(fill_f32(m, hw, seed, wi + W_ATTN_GAIN, 0, L.attn_gain, H, true));
    LOOP_RC(fill_f32(m, hw, seed, wi + W_FFN_GAIN, 0, L.ffn_gain, H, true));
    LOOP_RC(fill_rows(m, hw, seed, wi + W_Q, layer_stream(p, W_Q), L.w_in, 0, 0, nqr, H));
    LOOP_RC(fill_rows(m, hw, seed, wi + W_K, layer_stream(p, W_K), L.w_in, nqr, 0, nkr, H));
    LOOP_RC(fill_rows(m, hw, seed, wi + W_V, layer_stream(p, W_V), L.w_in, nqr + nkr, 0, nkr, H));
    if (!L.full) LOOP_RC(fill_rows(m, hw, seed, wi + W_G, layer_stream(p, W_G), L.w_in, nqr + 2 * nkr, 0, nl, H));
    LOOP_RC(fill_rows(m, hw, seed, wi + W_O, layer_stream(p, W_O), L.w_o, 0, 0, H, nqr));
    for (int64_t j = 0; j < F / 128; ++j) {  // interleave gate / up in blocks of 128 rows
      LOOP_RC(fill_rows(m, hw, seed, wi + W_GATE, layer_stream(p, W_GATE), L.w_gu, 256 * j, 128 * j, 128, H));
      LOOP_RC(fill_rows(m, hw, seed, wi + W_UP, layer_stream(p, W_UP), L.w_gu, 256 * j + 128, 128 * j, 128, H));
    }
    LOOP_RC(fill_rows(m, hw, seed, wi + W_DOWN, layer_stream(p, W_DOWN), L.w_down, 0, 0, H, F));
  }
  // mHC sites (fp32)
  m.sites.resize(2 * c.n_block);
  for (int s = 0; s < 2 * c.n_block; ++s) {
    const int wi = 2 + W_PER_LAYER * m.n_phys + 2 * s;
    LOOP_ALLOC(m.sites[s].gamma, float*, 2 * H * 4);
    LOOP_ALLOC(m.sites[s].phi, float*, 8 * 2 * H * 4);
    LOOP_RC(fill_f32(m, hw, seed, wi, 0, m.sites[s].gamma, 2 * H, true));
    LOOP_RC(fill_f32(m, hw, seed, wi + 1, site_stream(s), m.sites[s].phi, 16 * H, false));
    if (bf && m.use_tc && H == 4096) {  // the prefill forms this site's projections in a GEMM epilogue
      LOOP_ALLOC(m.sites[s].phig, float*, 8 * 2 * H * 4);
      LOOP_CU(launch_mhc_phig(m.sites[s].gamma, m.sites[s].phi, 2 * H, m.sites[s].phig, 0));
    }
  }
  // KV cache: one page pool per full-attention execution and one page table
  // per sequence shared by all of them (every execution of a sequence holds
  // the same positions)
  const int64_t Bm = c.max_batch, ctx = c.max_ctx;
  m.pps = (int)((ctx + KV_PAGE - 1) / KV_PAGE);
  m.n_pages = c.kv_pages > 0 ? c.kv_pages : (int)(Bm * m.pps);
  const int64_t pool = (int64_t)m.n_pages * nkv * KV_PAGE * hd * es;
  m.kc.assign(m.n_full, nullptr);
  m.vc.assign(m.n_full, nullptr);
  for (int i = 0; i < m.n_full; ++i) {  // zeroed: positions never written hold finite values
    LOOP_ALLOC(m.kc[i], void*, pool);
    LOOP_ALLOC(m.vc[i], void*, pool);
    LOOP_CU(cudaMemset(m.kc[i], 0, pool));
    LOOP_CU(cudaMemset(m.vc[i], 0, pool));
  }
  LOOP_ALLOC(m.d_table, int32_t*, Bm * m.pps * 4);
  LOOP_CU(cudaMemset(m.d_table, 0, Bm * m.pps * 4));  // unheld blocks point at page 0 (in bounds)
  m.h_table.assign(Bm * m.pps, 0);
  m.n_held.assign(Bm, 0);
  m.free_pages.clear();
  for (int p = m.n_pages - 1; p >= 0; --p) m.free_pages.push_back(p);
  m.st.assign(m.n_lin, nullptr);
  for (int i = 0; i < m.n_lin; ++i) {
    LOOP_ALLOC(m.st[i], float*, Bm * nl * ld * ld * 4);
    LOOP_CU(cudaMemset(m.st[i], 0, Bm * nl * ld * ld * 4));
  }
  LOOP_ALLOC(m.d_seq_len, int32_t*, Bm * 4);
  LOOP_CU(cudaMemset(m.d_seq_len, 0, Bm * 4));
  m.seq_len.assign(Bm, 0);
  LOOP_ALLOC(m.rope, float2*, ctx * (hd / 2) * sizeof(float2));
  LOOP_CU(launch_rope_table(m.rope, ctx, (int)hd, (double)c.rope_base, 0));
  // workspace for up to t_max tokens per forward
  Work& w = m.w;
  w.t_max = std::max<int64_t>(std::max<int64_t>(ctx, std::min<int64_t>(Bm * ctx, 65536)), Bm);
  const int64_t T = w.t_max;
  const int64_t qw = std::max(nq * hd, nl * ld);
  LOOP_ALLOC(w.h, float*, T * H * 4);
  LOOP_ALLOC(w.s, float*, 2 * T * H * 4);
  LOOP_ALLOC(w.xh, void*, T * H * es);
  LOOP_ALLOC(w.coef, float*, T * 8 * 4);
  w.mhc_part_floats = std::max<int64_t>(T * 18, 512 * 16 * 9);
  if (H % 256 == 0) w.mhc_part_floats = std::max<int64_t>(w.mhc_part_floats, T * (2 * H / 256) * 9);
  LOOP_ALLOC(w.mhc_part, float*, w.mhc_part_floats * 4);
  if (m.use_tc && H % 64 == 0) {  // decode GEMM partials: up to 32 splits x 64 tokens x the widest projection
    int64_t maxn = std::max<int64_t>(2 * F, H);
    for (auto& L : m.L) maxn = std::max(maxn, L.n_in);
    w.cpart_floats = 32 * 64 * maxn;
    LOOP_ALLOC(w.cpart, float*, w.cpart_floats * 4);
  }
  if (bf && c.io_mode == LOOP_TOKENS_TO_LOGITS) {  // decode graph input / output
    LOOP_ALLOC(m.dec_tok, int32_t*, Bm * 4);
    LOOP_ALLOC(m.dec_logits, float*, Bm * c.vocab * 4);
    LOOP_CU(cudaStreamCreateWithFlags(&m.cap_stream, cudaStreamNonBlocking));
  }
  if (bf && gla_chunk_supported((int)ld)) {  // one state per SM: the most a segmented prefill uses
    w.gla_seg_floats = 160 * ld * ld;
    LOOP_ALLOC(w.gla_seg, float*, w.gla_seg_floats * 4);
  }
  if (bf && decode_attention_supported((int)hd, (int)nq, (int)nkv))
    LOOP_ALLOC(w.dec_attn, float*, decode_attention_scratch_floats((int)Bm, (int)nq, ctx) * 4);
  LOOP_ALLOC(w.q, void*, T * qw * es);
  LOOP_ALLOC(w.k, void*, T * nl * ld * es);
  LOOP_ALLOC(w.v, void*, T * nl * ld * es);
  LOOP_ALLOC(w.gl, float*, T * nl * 4);
  LOOP_ALLOC(w.o, void*, T * qw * es);
  LOOP_ALLOC(w.a, void*, T * F * es);
  LOOP_ALLOC(w.zeros, int32_t*, Bm * 4);
  LOOP_CU(cudaMemset(w.zeros, 0, Bm * 4));
  // the fp32 scratch of the unfused path, only when some projection needs it
  bool unfused = !m.use_tc || H % 64 != 0 || F % 128 != 0;
  if (m.use_tc) {
    EpiArgs ql;
    ql.mode = Epi::QKV_LINEAR; ql.hd = (int)ld; ql.n_lin = (int)nl;
    EpiArgs qf;
    qf.mode = Epi::QKV_FULL; qf.hd = (int)hd; qf.heads_q = (int)nq; qf.heads_kv = (int)nkv;
    EpiArgs oe;
    oe.mode = Epi::RESID;
    unfused = unfused || !gemm_tc_supported(1, 3 * nl * ld + nl, H, ql) ||
              !gemm_tc_supported(1, (nq + 2 * nkv) * hd, H, qf) || !gemm_tc_supported(1, H, nq * hd, oe) ||
              !gemm_tc_supported(1, H, nl * ld, oe);
  }
  if (unfused) {
    int64_t maxn = 2 * F;
    for (auto& L : m.L) maxn = std::max(maxn, L.n_in);
    maxn = std::max(maxn, H);
    LOOP_ALLOC(w.cbuf, float*, T * maxn * 4);
  }
  LOOP_CU(cudaDeviceSynchronize());
  return LOOP_OK;
#undef LOOP_ALLOC
#undef LOOP_RC
}

cudaEvent_t take_event(Model& m) {
  if (!m.event_pool.empty()) {
    cudaEvent_t e = m.event_pool.back();
    m.event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return e;
}

// Run `launch` (which enqueues `kernels` kernels on st) and account for it.
template <typename F>
cudaError_t timed(Model& m, int cls, double work, int kernels, cudaStream_t st, F&& launch) {
  cudaEvent_t a = nullptr, b = nullptr;
  if (m.timing) {
    a = take_event(m);
    b = take_event(m);
    if (a) cudaEventRecord(a, st);
  }
  cudaError_t err = launch();
  m.launches += kernels;
  if (m.timing && a && b) {
    cudaEventRecord(b, st);
    m.pending.push_back({cls, work, a, b});
  }
  return err;
}

void drain_timing(Model& m) {
  for (auto& t : m.pending) {
    float ms = 0.f;
    if (cudaEventSynchronize(t.b) == cudaSuccess && cudaEventElapsedTime(&ms, t.a, t.b) == cudaSuccess) {
      m.t_ms[t.cls] += ms;
      m.t_work[t.cls] += t.work;
      m.t_count[t.cls] += 1;
    } else {
      cudaGetLastError();
    }
    m.event_pool.push_back(t.a);
    m.event_pool.push_back(t.b);
  }
  m.pending.clear();
}

// ---- KV pages: a free list on the host; a call's table changes go to the
// device as kernel arguments, in stream order ----
int64_t pages_for(int64_t len) { return (len + KV_PAGE - 1) / KV_PAGE; }

// Give sequence b pages for positions [0, len), appending to what it holds
// (the caller has checked that enough pages are free).
void pages_grow(Model& m, int b, int64_t len, std::vector<int32_t>& idx, std::vector<int32_t>& pg) {
  while (m.n_held[b] < pages_for(len)) {
    const int32_t p = m.free_pages.back();
    m.free_pages.pop_back();
    const int32_t i = b * m.pps + m.n_held[b]++;
    m.h_table[i] = p;
    idx.push_back(i);
    pg.push_back(p);
  }
}

void pages_release(Model& m, int b) {
  for (int j = m.n_held[b] - 1; j >= 0; --j) m.free_pages.push_back(m.h_table[b * m.pps + j]);
  m.n_held[b] = 0;
}

int32_t pages_upload(Model& m, const std::vector<int32_t>& idx, const std::vector<int32_t>& pg, cudaStream_t st) {
  if (idx.empty()) return LOOP_OK;
  LOOP_CU(timed(m, LOOP_K_OTHER, 0.0, (int)((idx.size() + 239) / 240), st,
                [&] { return launch_table_set(m.d_table, idx.data(), pg.data(), (int)idx.size(), st); }));
  return LOOP_OK;
}

// Restart sequences b0 .. b0 + n - 1 at lengths len(i) (their old pages go
// back first).  LOOP_ERANGE, with nothing changed, if the pool is too small.
template <typename Len>
int32_t pages_reset(Model& m, int b0, int n, Len len, cudaStream_t st) {
  int64_t avail = (int64_t)m.free_pages.size(), need = 0;
  for (int i = 0; i < n; ++i) {
    avail += m.n_held[b0 + i];
    need += pages_for(len(i));
  }
  if (need > avail) return fail(LOOP_ERANGE, "KV page pool exhausted");
  std::vector<int32_t> idx, pg;
  for (int i = 0; i < n; ++i) pages_release(m, b0 + i);
  for (int i = 0; i < n; ++i) pages_grow(m, b0 + i, len(i), idx, pg);
  return pages_upload(m, idx, pg, st);
}

// Let sequences 0 .. B - 1 grow by k positions.
int32_t pages_extend(Model& m, int B, int k, cudaStream_t st) {
  int64_t need = 0;
  for (int b = 0; b < B; ++b) need += std::max<int64_t>(0, pages_for((int64_t)m.seq_len[b] + k) - m.n_held[b]);
  if (need > (int64_t)m.free_pages.size()) return fail(LOOP_ERANGE, "KV page pool exhausted");
  std::vector<int32_t> idx, pg;
  for (int b = 0; b < B; ++b) pages_grow(m, b, (int64_t)m.seq_len[b] + k, idx, pg);
  return pages_upload(m, idx, pg, st);
}

// A projection: C = A W^T followed by its epilogue.
cudaError_t project(Model& m, const void* A, const void* W, int64_t M, int64_t N, int64_t K, const EpiArgs& e,
                    cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  const double flops = 2.0 * (double)M * (double)N * (double)K;
  m.w.part_formed = false;
  if (m.decoding && m.use_tc && m.w.cpart && gemm_skinny_supported(M, N, K)) {
    // decode: weight-streaming split-K GEMM, then the epilogue over the partials
    // (prefills never take it, so a prefill row is computed the same way
    // whatever the batch and length)
    const int splits = gemm_skinny_splits(N, K);
    const bool direct = e.mode == Epi::F32 && splits == 1;
    float* P = direct ? e.c : m.w.cpart;
    const int64_t ldp = direct ? e.ldc : N;
    if (!direct && (int64_t)splits * M * N > m.w.cpart_floats) return cudaErrorInvalidValue;
    cudaError_t err = timed(m, LOOP_K_GEMM, flops, 1, st,
                            [&] { return launch_gemm_skinny(A, W, M, N, K, splits, P, ldp, st); });
    if (err != cudaSuccess || direct) return err;
    return timed(m, LOOP_K_OTHER, 0.0, 1, st,
                 [&] { return launch_epilogue_unfused(P, N, M, N, e, bf16_model(m), st, splits); });
  }
  if (m.use_tc && gemm_tc_supported(M, N, K, e)) {
    const cudaError_t err = timed(m, LOOP_K_GEMM, flops, 1, st, [&] { return launch_gemm_tc(A, W, M, N, K, e, st); });
    m.w.part_formed = err == cudaSuccess && e.mode == Epi::MHC_WRITE && e.part != nullptr;
    return err;
  }
  float* C = e.mode == Epi::F32 ? e.c : m.w.cbuf;
  const int64_t ldc = e.mode == Epi::F32 ? e.ldc : N;
  cudaError_t err = timed(m, LOOP_K_GEMM, flops, 1, st,
                          [&] { return launch_gemm_simt(A, W, bf16_model(m), M, N, K, C, ldc, st); });
  if (err != cudaSuccess) return err;
  if (e.mode == Epi::F32) return cudaSuccess;
  return timed(m, LOOP_K_OTHER, 0.0, 1, st,
               [&] { return launch_epilogue_unfused(C, ldc, M, N, e, bf16_model(m), st); });
}

// Causal GQA attention of the current q against this execution's KV page
// pools; `table` is the page table of the call's first sequence.
cudaError_t attention(Model& m, const void* Kc, const void* Vc, const int32_t* table, int B, int S,
                      const int32_t* d_start, cudaStream_t st) {
  const loop_config& c = m.c;
  const bool bf = bf16_model(m);
  const int64_t pool_rows = (int64_t)m.n_pages * c.n_kv * KV_PAGE;
  // algorithmic FLOPs: QK^T and PV over the causal keys of every query
  double pairs = (double)B * S * (S + 1) / 2.0;
  if (m.extending)
    for (int b = 0; b < B; ++b) pairs += (double)S * m.seq_len[b];
  const double flops = 4.0 * pairs * c.head_dim * c.n_q;
  if (bf && S == 1 && m.w.dec_attn && decode_attention_supported(c.head_dim, c.n_q, c.n_kv)) {
    // one new token per sequence: its key position is seq_len[b]; the keys
    // read are the contexts (+1) of the B sequences
    int max_len = 0;
    double keys = 0;
    for (int b = 0; b < B; ++b) {
      max_len = std::max(max_len, m.seq_len[b] + 1);
      keys += m.seq_len[b] + 1;
    }
    const double dflops = 4.0 * keys * c.head_dim * c.n_q;
    return timed(m, LOOP_K_ATTENTION, dflops, 2, st, [&] {
      return launch_attention_decode(m.w.q, Kc, Vc, m.w.o, B, c.n_q, c.n_kv, table, m.pps, pool_rows, max_len,
                                     d_start, m.w.dec_attn, st);
    });
  }
  if (bf && S > 1 && flash_tc_supported(c.head_dim, c.n_q, c.n_kv))  // prefill from 0, or extend from seq_len
    return timed(m, LOOP_K_ATTENTION, flops, 1, st, [&] {
      return launch_flash_tc(m.w.q, Kc, Vc, m.w.o, B, S, c.n_q, c.n_kv, table, m.pps, pool_rows,
                             m.extending ? d_start : nullptr, st);
    });
  return timed(m, LOOP_K_ATTENTION, flops, 1, st, [&] {
    return launch_attention_simple(m.w.q, Kc, Vc, m.w.o, bf, B, S, c.n_q, c.n_kv, c.head_dim, table, m.pps, d_start,
                                   st);
  });
}

// Gated linear attention of the current q, k, v against this execution's state slot.
cudaError_t linear_attention(Model& m, float* state, int B, int S, cudaStream_t st) {
  const loop_config& c = m.c;
  const bool bf = bf16_model(m);
  const double d = c.lin_dim;
  if (bf && S > 1 && gla_chunk_supported(c.lin_dim)) {
    // chunked form: Q K^T, (.)V, Q S and K^T V per chunk of 64 tokens
    const double flops = 4.0 * (double)B * S * c.n_lin * d * (64.0 + d);
    return timed(m, LOOP_K_LINEAR_ATTENTION, flops, 1, st, [&] {
      return launch_gla_chunked(m.w.q, m.w.k, m.w.v, m.w.gl, state, m.w.o, B, S, c.n_lin, m.w.gla_seg,
                                m.w.gla_seg_floats, st);
    });
  }
  const double flops = 4.0 * (double)B * S * c.n_lin * d * d;
  if (bf && S == 1 && gla_chunk_supported(c.lin_dim))
    return timed(m, LOOP_K_LINEAR_ATTENTION, flops, 1, st, [&] {
      return launch_gla_decode(m.w.q, m.w.k, m.w.v, m.w.gl, state, m.w.o, B, c.n_lin, st);
    });
  return timed(m, LOOP_K_LINEAR_ATTENTION, flops, 1, st, [&] {
    return launch_gla_recurrent(m.w.q, m.w.k, m.w.v, m.w.gl, state, m.w.o, bf, B, S, c.n_lin, c.lin_dim, st);
  });
}

// Copy what an armed capture asks for, for sequence 0 of this call (b0 == 0):
// the attention inputs q (k, v and the log-gates for linear attention; K, V
// from the cache slot for full attention) and the output o of heads
// [head0, head0 + nheads), all S positions of this call.
cudaError_t capture(Model& m, const Capture& cp, bool full, const void* Kc, const void* Vc, int S, cudaStream_t st) {
  const loop_config& c = m.c;
  const int64_t es = m.esize;
  const int64_t nh = full ? c.n_q : c.n_lin, d = full ? c.head_dim : c.lin_dim;
  const int64_t h0 = cp.head0, n = cp.nheads;
  // q (and k, v, gates of linear attention): [B][heads][S][d], heads contiguous per sequence
  if (cp.q)
    if (cudaError_t e = cudaMemcpyAsync(cp.q, (const char*)m.w.q + h0 * S * d * es, n * S * d * es,
                                        cudaMemcpyDeviceToDevice, st); e != cudaSuccess) return e;
  if (full) {
    // K, V of the kv heads of those query heads, positions 0 .. start + S - 1 of the call
    const int64_t grp = c.n_q / c.n_kv, kh0 = h0 / grp, nk = (h0 + n - 1) / grp - kh0 + 1;
    const int64_t len = (m.extending || m.decoding) ? (int64_t)m.seq_len[0] + S : S;
    for (int64_t j = 0; j < nk; ++j) {  // gathered from sequence 0's pages
      if (cp.k)
        if (cudaError_t e = launch_cache_rows(Kc, es, m.d_table, m.pps, c.n_kv, 0, (int)(kh0 + j), (int)len, (int)d,
                                              (char*)cp.k + j * len * d * es, st); e != cudaSuccess) return e;
      if (cp.v)
        if (cudaError_t e = launch_cache_rows(Vc, es, m.d_table, m.pps, c.n_kv, 0, (int)(kh0 + j), (int)len, (int)d,
                                              (char*)cp.v + j * len * d * es, st); e != cudaSuccess) return e;
    }
  } else {
    if (cp.k)
      if (cudaError_t e = cudaMemcpyAsync(cp.k, (const char*)m.w.k + h0 * S * d * es, n * S * d * es,
                                          cudaMemcpyDeviceToDevice, st); e != cudaSuccess) return e;
    if (cp.v)
      if (cudaError_t e = cudaMemcpyAsync(cp.v, (const char*)m.w.v + h0 * S * d * es, n * S * d * es,
                                          cudaMemcpyDeviceToDevice, st); e != cudaSuccess) return e;
    if (cp.g)
      if (cudaError_t e = cudaMemcpyAsync(cp.g, m.w.gl + h0 * S, n * S * 4, cudaMemcpyDeviceToDevice, st);
          e != cudaSuccess) return e;
  }
  // o: [T][heads * d]; rows 0 .. S - 1, the columns of the captured heads
  if (cp.o)
    return cudaMemcpy2DAsync(cp.o, n * d * es, (const char*)m.w.o + h0 * d * es, nh * d * es, n * d * es, S,
                             cudaMemcpyDeviceToDevice, st);
  return cudaSuccess;
}

// One forward pass over sequences [b0, b0 + B) with S new tokens each,
// starting at positions d_start[0..B).  `out` is this group's output.
int32_t forward(Model& m, const int32_t* tokens, const float* hidden, int b0, int B, int S, const int32_t* d_start,
                float* out, uint32_t flags, bool last_only, cudaStream_t st) {
  const loop_config& c = m.c;
  const bool bf = bf16_model(m);
  const int64_t T = (int64_t)B * S, H = c.hidden, F = c.ffn;
  const int64_t nl = c.n_lin, ld = c.lin_dim, nq = c.n_q, nkv = c.n_kv, hd = c.head_dim;
  const int64_t es = m.esize;
  Work& w = m.w;
  if (c.io_mode == LOOP_TOKENS_TO_LOGITS)
    LOOP_CU(timed(m, LOOP_K_NORM, (double)T * H * (es + 4), 1, st,
                  [&] { return launch_embed(tokens, m.embed, bf, T, (int)H, c.vocab, w.h, st); }));
  else LOOP_CU(cudaMemcpyAsync(w.h, hidden, T * H * 4, cudaMemcpyDeviceToDevice, st));
  const int first_block = c.n_prelude, last_block = c.n_prelude + c.n_block * c.n_loops - 1;
  float* s_buf = w.s;  // streams [2][T][H]
  // A prefill's mHC-write projections also form the next site's partial
  // projections (hidden 4096, tensor-core path), so that site reads its
  // streams once instead of twice.
  const bool fuse_sites = !m.decoding && bf && m.use_tc && H == 4096;
  bool part_ready = false;  // w.mhc_part holds the current streams' partials for this site
  for (int e = 0; e < m.n_exec; ++e) {
    const int32_t* row = &m.table[5 * e];
    const int phys = row[0], kind = row[2], slot = row[3], region = row[4];
    const LayerW& L = m.L[phys];
    const bool in_block = region == LOOP_REGION_BLOCK;
    if (e == first_block)
      LOOP_CU(timed(m, LOOP_K_NORM, 12.0 * T * H, 1, st, [&] { return launch_expand(w.h, s_buf, T * H, st); }));
    for (int sub = 0; sub < 2; ++sub) {
      const float* gain = sub == 0 ? L.attn_gain : L.ffn_gain;
      if (in_block) {
        const SiteW& site = m.sites[2 * (phys - c.n_prelude) + sub];
        if (m.decoding && mhc_token_supported((int)H)) {  // decode: one CTA per token, one launch
          LOOP_CU(timed(m, LOOP_K_MHC, (double)T * (8.0 * H + es * H + 32.0), 1, st, [&] {
            return launch_mhc_token(s_buf, T, (int)H, site.gamma, site.phi, gain, c.sinkhorn_iters, c.norm_eps,
                                    w.coef, w.xh, bf, st);
          }));
        } else if (part_ready) {  // partials formed by the projection that wrote the streams
          LOOP_CU(timed(m, LOOP_K_MHC, (double)T * (8.0 * H + es * H + 32.0), 2, st, [&] {
            return launch_mhc_coef_read(w.mhc_part, (int)(2 * H / 256), s_buf, T, (int)H, gain, c.sinkhorn_iters,
                                        c.norm_eps, w.coef, w.xh, bf, st);
          }));
        } else {
          // decode at other widths: cut Phi into 16 parts so the partial kernel spreads over the
          // SMs and use the reader that forms the coefficients itself; a prefill always uses 2
          // parts and (at hidden 4096) the coefficient kernel, so each row's arithmetic is the
          // same at any length
          const int parts = (m.decoding && H % 32 == 0 && T * 16 * 9 <= w.mhc_part_floats) ? 16 : 2;
          LOOP_CU(timed(m, LOOP_K_MHC, (double)T * (8.0 * H + es * H + 32.0), (H == 4096 && !m.decoding) ? 3 : 2,
                        st, [&] {
                          return launch_mhc_prologue(s_buf, T, (int)H, site.gamma, site.phi, gain, c.sinkhorn_iters,
                                                     c.norm_eps, w.coef, w.xh, bf, w.mhc_part, st, parts, m.decoding);
                        }));
        }
      } else {
        LOOP_CU(timed(m, LOOP_K_NORM, (double)T * H * (4 + es), 1, st,
                      [&] { return launch_rmsnorm(w.h, T, (int)H, 1, 0, gain, c.norm_eps, w.xh, bf, st); }));
      }
      part_ready = false;
      EpiArgs out_epi;
      if (in_block) {
        out_epi.mode = Epi::MHC_WRITE;
        out_epi.s = s_buf;
        out_epi.coef = w.coef;
        // the loop region's next site (none after its last write)
        const SiteW* next = nullptr;
        if (sub == 0) next = &m.sites[2 * (phys - c.n_prelude) + 1];
        else if (e < last_block) next = &m.sites[2 * (m.table[5 * (e + 1)] - c.n_prelude)];
        if (fuse_sites && next && next->phig) {
          out_epi.next_phig = next->phig;
          out_epi.part = w.mhc_part;
        }
      } else {
        out_epi.mode = Epi::RESID;
        out_epi.c = w.h;
      }
      if (sub == 0) {
        if (kind == LOOP_KIND_FULL) {
          void* Kc = m.kc[slot];
          void* Vc = m.vc[slot];
          const int32_t* table = m.d_table + (int64_t)b0 * m.pps;
          EpiArgs qe;
          qe.mode = Epi::QKV_FULL;
          qe.q = w.q; qe.k = Kc; qe.v = Vc;
          qe.rope = m.rope; qe.start = d_start; qe.S = S;
          qe.heads_q = (int)nq; qe.heads_kv = (int)nkv; qe.hd = (int)hd; qe.table = table; qe.pps = m.pps;
          LOOP_CU(project(m, w.xh, L.w_in, T, L.n_in, H, qe, st));
          LOOP_CU(attention(m, Kc, Vc, table, B, S, d_start, st));
          for (const Capture& cp : m.captures)
            if (cp.exec == e && b0 == 0) LOOP_CU(capture(m, cp, true, Kc, Vc, S, st));
        } else {
          float* state = m.st[slot] + (int64_t)b0 * nl * ld * ld;
          EpiArgs qe;
          qe.mode = Epi::QKV_LINEAR;
          qe.q = w.q; qe.k = w.k; qe.v = w.v; qe.gl = w.gl;
          qe.S = S; qe.n_lin = (int)nl; qe.hd = (int)ld; qe.eps = c.norm_eps;
          LOOP_CU(project(m, w.xh, L.w_in, T, L.n_in, H, qe, st));
          LOOP_CU(linear_attention(m, state, B, S, st));
          for (const Capture& cp : m.captures)
            if (cp.exec == e && b0 == 0) LOOP_CU(capture(m, cp, false, nullptr, nullptr, S, st));
        }
        LOOP_CU(project(m, w.o, L.w_o, T, H, L.n_o_in, out_epi, st));
        part_ready = out_epi.part != nullptr && w.part_formed;
      } else {
        EpiArgs ge;
        ge.mode = Epi::SWIGLU;
        ge.a = w.a;
        LOOP_CU(project(m, w.xh, L.w_gu, T, 2 * F, H, ge, st));
        LOOP_CU(project(m, w.a, L.w_down, T, H, F, out_epi, st));
        part_ready = out_epi.part != nullptr && w.part_formed;
      }
    }
    if (e == last_block)
      LOOP_CU(timed(m, LOOP_K_NORM, 12.0 * T * H, 1, st, [&] { return launch_collapse(s_buf, w.h, T * H, st); }));
  }
  if (c.io_mode == LOOP_HIDDEN_TO_HIDDEN) {
    LOOP_CU(cudaMemcpyAsync(out, w.h, T * H * 4, cudaMemcpyDeviceToDevice, st));
    return LOOP_OK;
  }
  const bool all = (flags & LOOP_ALL_POSITIONS) && !last_only;
  const int64_t rows = all ? T : B;
  LOOP_CU(timed(m, LOOP_K_NORM, (double)rows * H * (4 + es), 1, st, [&] {
    return launch_rmsnorm(w.h, rows, (int)H, all ? 1 : S, all ? 0 : S - 1, m.final_gain, c.norm_eps, w.xh, bf, st);
  }));
  EpiArgs le;
  le.mode = Epi::F32;
  le.c = out;
  le.ldc = c.vocab;
  LOOP_CU(project(m, w.xh, m.embed, rows, c.vocab, H, le, st));
  return LOOP_OK;
}

// A decode step from a CUDA graph: the step's launches, captured once per
// (batch, decode-attention chunk count) on a private stream, replayed on the
// caller's stream between a copy of the tokens in and of the logits out.
// Returns false (nothing launched) when the step must run eagerly: per-launch
// timing is on, a loop_capture is armed, no eager step has set up the kernels
// yet, or capture failed.
bool decode_graph(Model& m, const int32_t* d_tokens, int B, float* d_logits, cudaStream_t st, int32_t* rc) {
  if (m.timing || !m.decoded_eagerly || !m.cap_stream || !m.dec_tok || !m.dec_logits || !m.captures.empty())
    return false;
  int max_len = 0;
  for (int b = 0; b < B; ++b) max_len = std::max(max_len, m.seq_len[b] + 1);
  const int nch = decode_attention_chunks(max_len);
  Model::DecodeGraph* g = nullptr;
  for (auto& x : m.graphs)
    if (x.B == B && x.nch == nch) g = &x;
  if (!g) {
    Model::DecodeGraph ng;
    ng.B = B;
    ng.nch = nch;
    const int64_t l0 = m.launches;
    cudaGraph_t graph = nullptr;
    if (cudaStreamBeginCapture(m.cap_stream, cudaStreamCaptureModeRelaxed) != cudaSuccess) {
      cudaGetLastError();
      return false;
    }
    m.decoding = true;
    const int32_t frc = forward(m, m.dec_tok, nullptr, 0, B, 1, m.d_seq_len, m.dec_logits, 0, true, m.cap_stream);
    m.decoding = false;
    const cudaError_t ec = cudaStreamEndCapture(m.cap_stream, &graph);
    ng.kernels = m.launches - l0;  // what the graph launches; capturing launched nothing
    m.launches = l0;
    bool ok = frc == LOOP_OK && ec == cudaSuccess && graph;
    if (ok) ok = cudaGraphInstantiate(&ng.exec, graph, 0) == cudaSuccess;
    if (graph) cudaGraphDestroy(graph);
    if (!ok) {
      cudaGetLastError();
      if (ng.exec) cudaGraphExecDestroy(ng.exec);
      return false;
    }
    m.graphs.push_back(ng);
    g = &m.graphs.back();
  }
  cudaError_t e = cudaMemcpyAsync(m.dec_tok, d_tokens, (size_t)B * 4, cudaMemcpyDeviceToDevice, st);
  if (e == cudaSuccess) e = cudaGraphLaunch(g->exec, st);
  m.launches += g->kernels;
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(d_logits, m.dec_logits, (size_t)B * m.c.vocab * 4, cudaMemcpyDeviceToDevice, st);
  *rc = e == cudaSuccess ? LOOP_OK : fail(LOOP_ECUDA, std::string("decode graph: ") + cudaGetErrorString(e));
  return true;
}

}  // namespace

extern "C" {

int32_t loop_num_exec(const loop_config* cfg) {
  if (!valid(cfg)) return fail(LOOP_EINVAL, "invalid loop_config");
  return cfg->n_prelude + cfg->n_block * cfg->n_loops + cfg->n_coda;
}

int32_t loop_schedule(const loop_config* cfg, int32_t* table) {
  if (!valid(cfg)) return fail(LOOP_EINVAL, "invalid loop_config");
  if (!table) return fail(LOOP_EINVAL, "table is NULL");
  return build_table(cfg, table);
}

int32_t loop_num_weights(const loop_config* cfg) {
  if (!valid(cfg)) return fail(LOOP_EINVAL, "invalid loop_config");
  return 2 + W_PER_LAYER * (cfg->n_prelude + cfg->n_block + cfg->n_coda) + 4 * cfg->n_block;
}

int32_t loop_model_create(const loop_config* cfg, const float* const* host_weights, uint64_t seed, loop_model** out) {
  if (!out) return fail(LOOP_EINVAL, "out is NULL");
  *out = nullptr;
  if (!valid(cfg)) return fail(LOOP_EINVAL, "invalid loop_config");
  if (const char* why = unsupported(cfg)) return fail(LOOP_EUNSUPPORTED, why);
  auto mp = std::make_unique<loop_model>();
  const int32_t rc = create_impl(cfg, host_weights, seed, mp->m);
  if (rc != LOOP_OK) {
    const std::string msg = g_last_error;
    release(mp->m);
    g_last_error = msg;
    return rc;
  }
  *out = mp.release();
  return LOOP_OK;
}

int32_t loop_prefill(loop_model* mp, const int32_t* d_tokens, const float* d_hidden, int32_t B, int32_t S,
                     float* d_out, uint32_t flags, void* stream) {
  if (!mp || !d_out) return fail(LOOP_EINVAL, "model or output is NULL");
  Model& m = mp->m;
  const loop_config& c = m.c;
  if (B <= 0 || S <= 0) return fail(LOOP_EINVAL, "B and S must be positive");
  if (B > c.max_batch || S > c.max_ctx) return fail(LOOP_ERANGE, "B > max_batch or S > max_ctx");
  if (c.io_mode == LOOP_TOKENS_TO_LOGITS && !d_tokens) return fail(LOOP_EINVAL, "d_tokens is NULL");
  if (c.io_mode == LOOP_HIDDEN_TO_HIDDEN && !d_hidden) return fail(LOOP_EINVAL, "d_hidden is NULL");
  cudaStream_t st = (cudaStream_t)stream;
  if (int32_t rc = pages_reset(m, 0, B, [&](int) { return (int64_t)S; }, st); rc != LOOP_OK) return rc;
  const int64_t nl = c.n_lin, ld = c.lin_dim, H = c.hidden;
  const int group = (int)std::max<int64_t>(1, std::min<int64_t>(B, m.w.t_max / S));
  const bool all = flags & LOOP_ALL_POSITIONS;
  for (int b0 = 0; b0 < B; b0 += group) {
    const int nb = std::min(group, B - b0);
    for (int i = 0; i < m.n_lin; ++i)
      LOOP_CU(cudaMemsetAsync(m.st[i] + (int64_t)b0 * nl * ld * ld, 0, (size_t)nb * nl * ld * ld * 4, st));
    float* out;
    if (c.io_mode == LOOP_HIDDEN_TO_HIDDEN) out = d_out + (int64_t)b0 * S * H;
    else out = d_out + (int64_t)b0 * (all ? S : 1) * c.vocab;
    const int32_t rc = forward(m, d_tokens ? d_tokens + (int64_t)b0 * S : nullptr,
                               d_hidden ? d_hidden + (int64_t)b0 * S * H : nullptr, b0, nb, S, m.w.zeros, out, flags,
                               false, st);
    if (rc != LOOP_OK) return rc;
  }
  LOOP_CU(timed(m, LOOP_K_OTHER, 0.0, 1, st, [&] { return launch_set_len(m.d_seq_len, B, S, st); }));
  for (int b = 0; b < B; ++b) m.seq_len[b] = S;
  return LOOP_OK;
}

int32_t loop_decode_step(loop_model* mp, const int32_t* d_tokens, int32_t B, float* d_logits, void* stream) {
  if (!mp || !d_tokens || !d_logits) return fail(LOOP_EINVAL, "NULL argument");
  Model& m = mp->m;
  if (m.c.io_mode != LOOP_TOKENS_TO_LOGITS) return fail(LOOP_EINVAL, "decode needs TOKENS_TO_LOGITS");
  if (B <= 0) return fail(LOOP_EINVAL, "B must be positive");
  if (B > m.c.max_batch) return fail(LOOP_ERANGE, "B > max_batch");
  for (int b = 0; b < B; ++b)
    if (m.seq_len[b] + 1 > m.c.max_ctx) return fail(LOOP_ERANGE, "sequence would pass max_ctx");
  cudaStream_t st = (cudaStream_t)stream;
  if (int32_t rc = pages_extend(m, B, 1, st); rc != LOOP_OK) return rc;
  int32_t rc = LOOP_EINVAL;
  if (!decode_graph(m, d_tokens, B, d_logits, st, &rc)) {  // eager: per-launch timing, first step, no graph
    m.decoding = true;
    rc = forward(m, d_tokens, nullptr, 0, B, 1, m.d_seq_len, d_logits, 0, true, st);
    m.decoding = false;
    if (rc == LOOP_OK) m.decoded_eagerly = true;
  }
  if (rc != LOOP_OK) return rc;
  LOOP_CU(timed(m, LOOP_K_OTHER, 0.0, 1, st, [&] { return launch_advance(m.d_seq_len, B, st); }));
  for (int b = 0; b < B; ++b) m.seq_len[b] += 1;
  return LOOP_OK;
}

int32_t loop_extend(loop_model* mp, const int32_t* d_tokens, int32_t B, int32_t k, float* d_out, uint32_t flags,
                    void* stream) {
  if (!mp || !d_tokens || !d_out) return fail(LOOP_EINVAL, "NULL argument");
  Model& m = mp->m;
  if (m.c.io_mode != LOOP_TOKENS_TO_LOGITS) return fail(LOOP_EINVAL, "extend needs TOKENS_TO_LOGITS");
  if (B <= 0 || k <= 0) return fail(LOOP_EINVAL, "B and k must be positive");
  if (B > m.c.max_batch) return fail(LOOP_ERANGE, "B > max_batch");
  if ((int64_t)B * k > m.w.t_max) return fail(LOOP_ERANGE, "B * k exceeds the per-call token budget");
  for (int b = 0; b < B; ++b)
    if ((int64_t)m.seq_len[b] + k > m.c.max_ctx) return fail(LOOP_ERANGE, "sequence would pass max_ctx");
  cudaStream_t st = (cudaStream_t)stream;
  if (int32_t rc = pages_extend(m, B, k, st); rc != LOOP_OK) return rc;
  // the positions of sequence b are seq_len[b] .. seq_len[b] + k - 1: every kernel takes
  // its start from d_seq_len, and attention uses the kernel that honours per-sequence starts
  m.extending = true;
  const int32_t rc = forward(m, d_tokens, nullptr, 0, B, k, m.d_seq_len, d_out, flags, false, st);
  m.extending = false;
  if (rc != LOOP_OK) return rc;
  LOOP_CU(timed(m, LOOP_K_OTHER, 0.0, 1, st, [&] { return launch_advance(m.d_seq_len, B, st, k); }));
  for (int b = 0; b < B; ++b) m.seq_len[b] += k;
  return LOOP_OK;
}

int32_t loop_prefill_ragged(loop_model* mp, const int32_t* d_tokens, const int32_t* h_lens, int32_t b0, int32_t B,
                            float* d_out, uint32_t flags, void* stream) {
  if (!mp || !d_tokens || !h_lens || !d_out) return fail(LOOP_EINVAL, "NULL argument");
  Model& m = mp->m;
  const loop_config& c = m.c;
  if (c.io_mode != LOOP_TOKENS_TO_LOGITS) return fail(LOOP_EINVAL, "ragged prefill needs TOKENS_TO_LOGITS");
  if (B <= 0 || b0 < 0) return fail(LOOP_EINVAL, "B must be positive and b0 >= 0");
  if ((int64_t)b0 + B > c.max_batch) return fail(LOOP_ERANGE, "b0 + B > max_batch");
  for (int i = 0; i < B; ++i)
    if (h_lens[i] < 1 || h_lens[i] > c.max_ctx) return fail(LOOP_ERANGE, "a length is outside [1, max_ctx]");
  cudaStream_t st = (cudaStream_t)stream;
  if (int32_t rc = pages_reset(m, b0, B, [&](int i) { return (int64_t)h_lens[i]; }, st); rc != LOOP_OK) return rc;
  const int64_t nl = c.n_lin, ld = c.lin_dim;
  const bool all = flags & LOOP_ALL_POSITIONS;
  int64_t off = 0;
  for (int i = 0; i < B; ++i) {
    const int b = b0 + i, S = h_lens[i];
    for (int j = 0; j < m.n_lin; ++j)
      LOOP_CU(cudaMemsetAsync(m.st[j] + (int64_t)b * nl * ld * ld, 0, (size_t)nl * ld * ld * 4, st));
    float* out = d_out + (all ? off : i) * c.vocab;
    const int32_t rc = forward(m, d_tokens + off, nullptr, b, 1, S, m.w.zeros, out, flags, false, st);
    if (rc != LOOP_OK) return rc;
    LOOP_CU(timed(m, LOOP_K_OTHER, 0.0, 1, st, [&] { return launch_set_len(m.d_seq_len + b, 1, S, st); }));
    m.seq_len[b] = S;
    off += S;
  }
  return LOOP_OK;
}

int32_t mhc_sinkhorn(const float* d_logits, float* d_out, int32_t count, int32_t n, int32_t iters, void* stream) {
  if (!d_logits || !d_out) return fail(LOOP_EINVAL, "NULL argument");
  if (count < 0 || n < 1 || n > 8 || iters < 0) return fail(LOOP_EINVAL, "count >= 0, 1 <= n <= 8, iters >= 0");
  LOOP_CU(launch_sinkhorn(d_logits, d_out, count, n, iters, (cudaStream_t)stream));
  return LOOP_OK;
}

int32_t mhc_prologue(const float* d_streams, int64_t T, int32_t H, const float* d_gamma, const float* d_phi,
                     const float* d_gain, int32_t iters, float eps, float* d_coef, void* d_xhat, int32_t xhat_dtype,
                     float* d_scratch, void* stream) {
  if (!d_streams || !d_gamma || !d_phi || !d_gain || !d_coef || !d_xhat || !d_scratch)
    return fail(LOOP_EINVAL, "NULL argument");
  if (T < 0 || H <= 0 || H % 4 != 0 || H > 6144 || iters < 0 || !(eps >= 0.f))
    return fail(LOOP_EINVAL, "T >= 0, H a multiple of 4 and <= 6144, iters >= 0, eps >= 0");
  if (xhat_dtype != LOOP_F32 && xhat_dtype != LOOP_BF16) return fail(LOOP_EINVAL, "bad xhat_dtype");
  LOOP_CU(launch_mhc_prologue(d_streams, T, H, d_gamma, d_phi, d_gain, iters, eps, d_coef, d_xhat,
                              xhat_dtype == LOOP_BF16, d_scratch, (cudaStream_t)stream));
  return LOOP_OK;
}

void loop_model_destroy(loop_model* mp) {
  if (!mp) return;
  release(mp->m);
  delete mp;
}

int32_t loop_seq_len(const loop_model* mp, int32_t b) {
  if (!mp || b < 0 || b >= mp->m.c.max_batch) return fail(LOOP_EINVAL, "bad model or sequence index");
  return mp->m.seq_len[b];
}

int32_t loop_cache_read(loop_model* mp, int32_t kind, int32_t slot, int32_t B, int32_t len, float* d_out,
                        void* stream) {
  if (!mp || !d_out) return fail(LOOP_EINVAL, "NULL argument");
  Model& m = mp->m;
  const loop_config& c = m.c;
  if (B <= 0 || B > c.max_batch) return fail(LOOP_ERANGE, "bad B");
  cudaStream_t st = (cudaStream_t)stream;
  if (kind == LOOP_KIND_FULL) {
    if (slot < 0 || slot >= m.n_full || len < 0 || len > c.max_ctx) return fail(LOOP_EINVAL, "bad slot or len");
    const int64_t n = (int64_t)B * c.n_kv * len * c.head_dim;
    LOOP_CU(launch_cache_to_f32(m.kc[slot], bf16_model(m), m.d_table, m.pps, B, c.n_kv, len, c.head_dim, d_out, st));
    LOOP_CU(launch_cache_to_f32(m.vc[slot], bf16_model(m), m.d_table, m.pps, B, c.n_kv, len, c.head_dim, d_out + n,
                                st));
    return LOOP_OK;
  }
  if (kind != LOOP_KIND_LINEAR || slot < 0 || slot >= m.n_lin) return fail(LOOP_EINVAL, "bad kind or slot");
  const int64_t n = (int64_t)B * c.n_lin * c.lin_dim * c.lin_dim;
  LOOP_CU(cudaMemcpyAsync(d_out, m.st[slot], n * 4, cudaMemcpyDeviceToDevice, st));
  return LOOP_OK;
}

int32_t loop_weight_read(loop_model* mp, int32_t index, float* d_out, void* stream) {
  if (!mp || !d_out) return fail(LOOP_EINVAL, "NULL argument");
  Model& m = mp->m;
  const loop_config& c = m.c;
  int64_t cols = 0;
  const int64_t rows = weight_rows(c, index, &cols);
  if (rows < 0) return fail(LOOP_EINVAL, "bad weight index");
  cudaStream_t st = (cudaStream_t)stream;
  const bool bf = bf16_model(m);
  if (index == 0) {
    LOOP_CU(launch_weight_to_f32(m.embed, bf, rows, cols, 0, d_out, st));
    return LOOP_OK;
  }
  if (index == 1) {
    LOOP_CU(cudaMemcpyAsync(d_out, m.final_gain, rows * 4, cudaMemcpyDeviceToDevice, st));
    return LOOP_OK;
  }
  int i = index - 2;
  if (i < W_PER_LAYER * m.n_phys) {
    const LayerW& L = m.L[i / W_PER_LAYER];
    const int slot = i % W_PER_LAYER;
    const int64_t H = c.hidden;
    const int64_t nqr = L.n_o_in, nkr = L.full ? (int64_t)c.n_kv * c.head_dim : (int64_t)c.n_lin * c.lin_dim;
    switch (slot) {
      case W_ATTN_GAIN: LOOP_CU(cudaMemcpyAsync(d_out, L.attn_gain, H * 4, cudaMemcpyDeviceToDevice, st)); break;
      case W_FFN_GAIN: LOOP_CU(cudaMemcpyAsync(d_out, L.ffn_gain, H * 4, cudaMemcpyDeviceToDevice, st)); break;
      case W_Q: LOOP_CU(launch_weight_to_f32(L.w_in, bf, rows, cols, 0, d_out, st)); break;
      case W_K: LOOP_CU(launch_weight_to_f32(L.w_in, bf, rows, cols, nqr, d_out, st)); break;
      case W_V: LOOP_CU(launch_weight_to_f32(L.w_in, bf, rows, cols, nqr + nkr, d_out, st)); break;
      case W_G: LOOP_CU(launch_weight_to_f32(L.w_in, bf, rows, cols, nqr + 2 * nkr, d_out, st)); break;
      case W_O: LOOP_CU(launch_weight_to_f32(L.w_o, bf, rows, cols, 0, d_out, st)); break;
      case W_GATE:
      case W_UP:
        for (int64_t j = 0; j < c.ffn / 128; ++j)
          LOOP_CU(launch_weight_to_f32(L.w_gu, bf, 128, cols, 256 * j + (slot == W_UP ? 128 : 0),
                                       d_out + 128 * j * cols, st));
        break;
      case W_DOWN: LOOP_CU(launch_weight_to_f32(L.w_down, bf, rows, cols, 0, d_out, st)); break;
    }
    return LOOP_OK;
  }
  i -= W_PER_LAYER * m.n_phys;
  const SiteW& s = m.sites[i / 2];
  LOOP_CU(cudaMemcpyAsync(d_out, i % 2 == 0 ? s.gamma : s.phi, rows * cols * 4, cudaMemcpyDeviceToDevice, st));
  return LOOP_OK;
}

int32_t loop_capture(loop_model* mp, int32_t exec, int32_t head0, int32_t nheads, void* d_q, void* d_k, void* d_v,
                     float* d_gate, void* d_o) {
  if (!mp) return fail(LOOP_EINVAL, "model is NULL");
  Model& m = mp->m;
  if (exec < 0) {
    m.captures.clear();
    return LOOP_OK;
  }
  if (exec >= m.n_exec) return fail(LOOP_EINVAL, "exec out of range");
  const bool full = m.table[5 * exec + 2] == LOOP_KIND_FULL;
  const int nh = full ? m.c.n_q : m.c.n_lin;
  if (head0 < 0 || nheads <= 0 || head0 + nheads > nh) return fail(LOOP_EINVAL, "bad head range");
  if (m.captures.size() >= 8) return fail(LOOP_ERANGE, "at most 8 captures");
  Capture cp;
  cp.exec = exec;
  cp.head0 = head0;
  cp.nheads = nheads;
  cp.q = d_q;
  cp.k = d_k;
  cp.v = d_v;
  cp.g = d_gate;
  cp.o = d_o;
  m.captures.push_back(cp);
  return LOOP_OK;
}

int32_t loop_set_timing(loop_model* mp, int32_t enable) {
  if (!mp) return fail(LOOP_EINVAL, "model is NULL");
  mp->m.timing = enable != 0;
  return LOOP_OK;
}

int32_t loop_timing_read(loop_model* mp, int32_t cls, double* total_ms, int64_t* launches, double* work,
                         int32_t reset) {
  if (!mp || cls < 0 || cls >= LOOP_K_CLASSES) return fail(LOOP_EINVAL, "bad model or class");
  Model& m = mp->m;
  drain_timing(m);
  if (total_ms) *total_ms = m.t_ms[cls];
  if (launches) *launches = m.t_count[cls];
  if (work) *work = m.t_work[cls];
  if (reset) {
    for (int i = 0; i < LOOP_K_CLASSES; ++i) m.t_ms[i] = m.t_work[i] = 0, m.t_count[i] = 0;
  }
  return LOOP_OK;
}

int64_t loop_launch_count(const loop_model* mp) { return mp ? mp->m.launches : -1; }

int32_t loop_device_status(void) {
  if (cudaDeviceSynchronize() != cudaSuccess) return fail(LOOP_ECUDA, "device error");
  const int v = status_read();
  if (v < 0) return fail(LOOP_ECUDA, "status read failed");
  return v;
}

void loop_clear_device_status(void) { status_clear(); }

int32_t loop_selftest_timeout(int32_t timeout_ms) {
  if (timeout_ms < 1 || timeout_ms > 10000) return fail(LOOP_EINVAL, "timeout_ms in [1, 10000]");
  int* d = nullptr;
  if (cudaMalloc(&d, sizeof(int)) != cudaSuccess) {
    cudaGetLastError();
    return fail(LOOP_ENOMEM, "cudaMalloc failed");
  }
  int r = -1;
  cudaError_t e = launch_selftest_timeout((uint64_t)timeout_ms * 1000000ull, d, 0);
  if (e == cudaSuccess) e = cudaMemcpy(&r, d, sizeof(int), cudaMemcpyDeviceToHost);
  cudaFree(d);
  if (e != cudaSuccess) return fail(LOOP_ECUDA, cudaGetErrorString(e));
  if (r != 0) return fail(LOOP_ECUDA, "the self-test wait completed, which nothing should cause");
  return loop_device_status();
}

const char* loop_last_error(void) { return g_last_error.c_str(); }

int32_t loop_gemm_bf16(const void* d_A, const void* d_W, int64_t M, int64_t N, int64_t K, float* d_C, int64_t ldc,
                       int32_t use_tensor_cores, void* stream) {
  if (!d_A || !d_W || !d_C) return fail(LOOP_EINVAL, "NULL argument");
  if (M < 0 || N <= 0 || K <= 0 || ldc < N) return fail(LOOP_EINVAL, "bad shape");
  EpiArgs e;
  e.mode = Epi::F32;
  e.c = d_C;
  e.ldc = ldc;
  cudaStream_t st = (cudaStream_t)stream;
  if (use_tensor_cores) {
    if (!gemm_tc_supported(M, N, K, e)) return fail(LOOP_EUNSUPPORTED, "K must be a multiple of 64");
    LOOP_CU(launch_gemm_tc(d_A, d_W, M, N, K, e, st));
  } else {
    LOOP_CU(launch_gemm_simt(d_A, d_W, true, M, N, K, d_C, ldc, st));
  }
  return LOOP_OK;
}

}  // extern "C"
