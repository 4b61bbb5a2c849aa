// The unfused path: a CUDA-core GEMM into an fp32 scratch buffer followed by
// one kernel per epilogue, a warp-per-query causal GQA attention with online
// softmax, and the token-by-token gated-linear-attention recurrence.  This
// path runs the fp32 model (tensor cores cannot multiply fp32 exactly) and
// every shape the tensor-core kernels do not take.

#include <algorithm>

#include "model.h"

namespace loopk {

// ---------------------------------------------------------------------------
// C[M][N] (row stride ldc) = A[M][K] * W[N][K]^T, fp32 accumulation
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) gemm_simt_kernel(const T* __restrict__ A, const T* __restrict__ W, int64_t M,
                                                        int64_t N, int64_t K, float* __restrict__ C, int64_t ldc) {
  __shared__ float As[16][64 + 4];
  __shared__ float Ws[16][64 + 4];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const int64_t m0 = (int64_t)blockIdx.y * 64, n0 = (int64_t)blockIdx.x * 64;
  float acc[4][4] = {};
  for (int64_t k0 = 0; k0 < K; k0 += 16) {
#pragma unroll
    for (int l = 0; l < 4; ++l) {
      const int idx = threadIdx.x + l * 256;
      const int r = idx / 16, kk = idx % 16;
      const bool kin = k0 + kk < K;
      As[kk][r] = (m0 + r < M && kin) ? to_f(A[(m0 + r) * K + k0 + kk]) : 0.f;
      Ws[kk][r] = (n0 + r < N && kin) ? to_f(W[(n0 + r) * K + k0 + kk]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Ws[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] += a[i] * b[j];
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t m = m0 + ty * 4 + i, n = n0 + tx * 4 + j;
      if (m < M && n < N) C[m * ldc + n] = acc[i][j];
    }
}

cudaError_t launch_gemm_simt(const void* A, const void* W, bool bf, int64_t M, int64_t N, int64_t K, float* C,
                             int64_t ldc, cudaStream_t st) {
  if (M == 0 || N == 0) return cudaSuccess;
  dim3 grid((unsigned)((N + 63) / 64), (unsigned)((M + 63) / 64));
  if (bf) gemm_simt_kernel<bf16><<<grid, 256, 0, st>>>((const bf16*)A, (const bf16*)W, M, N, K, C, ldc);
  else gemm_simt_kernel<float><<<grid, 256, 0, st>>>((const float*)A, (const float*)W, M, N, K, C, ldc);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// epilogues over the scratch C (optionally `splits` split-K slices of M x ldc
// each, summed in slice order)
// ---------------------------------------------------------------------------
struct CView {
  const float* c;
  int64_t ldc, slice;
  int splits;
  LOOP_DEV float operator()(int64_t r, int64_t col) const {
    float v = c[r * ldc + col];
    for (int k = 1; k < splits; ++k) v += c[k * slice + r * ldc + col];
    return v;
  }
};
__global__ void epi_resid_kernel(CView C, int64_t M, int64_t N, float* h) {
  const int64_t n = M * N;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / N, c = i % N;
    h[i] += C(r, c);
  }
}

__global__ void epi_f32_kernel(CView C, int64_t M, int64_t N, float* out, int64_t ldo) {
  const int64_t n = M * N;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / N, c = i % N;
    out[r * ldo + c] = C(r, c);
  }
}

__global__ void epi_mhc_kernel(CView C, int64_t M, int64_t N, float* s, const float* coef) {
  const int64_t n = M * N;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / N, c = i % N;
    const float* cf = coef + r * 8;
    const float y = C(r, c);
    const float s0 = s[i], s1 = s[n + i];
    s[i] = cf[4] * s0 + cf[5] * s1 + cf[2] * y;
    s[n + i] = cf[6] * s0 + cf[7] * s1 + cf[3] * y;
  }
}

template <typename T>
__global__ void epi_swiglu_kernel(CView C, int64_t M, int64_t F, T* a) {
  griddep_launch_dependents();  // the down projection after this may start streaming its weights
  const int64_t n = M * F;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / F, f = i % F;
    const int64_t blk = f / 128, j = f % 128;
    const float g = C(r, blk * 256 + j), u = C(r, blk * 256 + 128 + j);
    a[i] = from_f<T>(g * sigmoidf_(g) * u);
  }
}

// one warp per (token, head); d <= 128
template <typename T>
__global__ void epi_qkv_linear_kernel(CView C, int64_t M, int S, int nh, int d, float eps, T* q, T* k, T* v,
                                      float* gl) {
  const int64_t w = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= M * nh) return;
  const int64_t r = w / nh;
  const int h = (int)(w % nh);
  const int64_t b = r / S, t = r % S;
  float sq = 0.f, sk = 0.f;
  for (int i = lane; i < d; i += 32) {
    const float a = C(r, (int64_t)h * d + i), c = C(r, (int64_t)(nh + h) * d + i);
    sq += a * a;
    sk += c * c;
  }
  sq = warp_sum(sq);
  sk = warp_sum(sk);
  const float iq = rsqrtf(sq + eps), ik = rsqrtf(sk + eps);
  const int64_t o = ((b * nh + h) * S + t) * d;
  for (int i = lane; i < d; i += 32) {
    q[o + i] = from_f<T>(C(r, (int64_t)h * d + i) * iq);
    k[o + i] = from_f<T>(C(r, (int64_t)(nh + h) * d + i) * ik);
    v[o + i] = from_f<T>(C(r, (int64_t)(2 * nh + h) * d + i));
  }
  if (lane == 0) gl[(b * nh + h) * S + t] = log_sigmoidf_(C(r, (int64_t)3 * nh * d + h));
}

// one warp per (token, head) over q heads, then k heads, then v heads
template <typename T>
__global__ void epi_qkv_full_kernel(CView C, int64_t M, int S, int nq, int nkv, int hd, const float2* rope,
                                    const int32_t* start, const int32_t* table, int pps, T* q, T* K, T* V) {
  const int64_t w = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int nheads = nq + 2 * nkv;
  if (w >= M * nheads) return;
  const int64_t r = w / nheads;
  const int h = (int)(w % nheads);
  const int64_t b = r / S, t = r % S;
  const int64_t pos = start[b] + t;
  const int64_t c0 = (int64_t)h * hd;
  const int half = hd / 2;
  T* dst;
  bool rot = true;
  if (h < nq) {
    dst = q + ((b * nq + h) * S + t) * hd;
  } else if (h < nq + nkv) {
    dst = K + kv_row(table, pps, nkv, b, h - nq, pos) * hd;
  } else {
    dst = V + kv_row(table, pps, nkv, b, h - nq - nkv, pos) * hd;
    rot = false;
  }
  for (int i = lane; i < half; i += 32) {
    const float a = C(r, c0 + i), c = C(r, c0 + i + half);
    if (rot) {
      const float2 cs = rope[pos * half + i];
      dst[i] = from_f<T>(a * cs.x - c * cs.y);
      dst[i + half] = from_f<T>(c * cs.x + a * cs.y);
    } else {
      dst[i] = from_f<T>(a);
      dst[i + half] = from_f<T>(c);
    }
  }
}

cudaError_t launch_epilogue_unfused(const float* C, int64_t ldc, int64_t M, int64_t N, const EpiArgs& e, bool bf,
                                    cudaStream_t st, int splits) {
  if (M == 0) return cudaSuccess;
  auto grid_for = [](int64_t n) { return (unsigned)std::min<int64_t>((n + 255) / 256, 148 * 32); };
  const CView cv{C, ldc, M * ldc, splits};
  switch (e.mode) {
    case Epi::F32:
      if (splits > 1 || C != e.c) epi_f32_kernel<<<grid_for(M * N), 256, 0, st>>>(cv, M, N, e.c, e.ldc);
      break;
    case Epi::RESID:
      epi_resid_kernel<<<grid_for(M * N), 256, 0, st>>>(cv, M, N, e.c);
      break;
    case Epi::MHC_WRITE:
      epi_mhc_kernel<<<grid_for(M * N), 256, 0, st>>>(cv, M, N, e.s, e.coef);
      break;
    case Epi::SWIGLU:
      if (bf) epi_swiglu_kernel<bf16><<<grid_for(M * N / 2), 256, 0, st>>>(cv, M, N / 2, (bf16*)e.a);
      else epi_swiglu_kernel<float><<<grid_for(M * N / 2), 256, 0, st>>>(cv, M, N / 2, (float*)e.a);
      break;
    case Epi::QKV_LINEAR: {
      const int64_t warps = M * e.n_lin;
      const unsigned g = (unsigned)((warps * 32 + 255) / 256);
      if (bf)
        epi_qkv_linear_kernel<bf16><<<g, 256, 0, st>>>(cv, M, e.S, e.n_lin, e.hd, e.eps, (bf16*)e.q, (bf16*)e.k,
                                                       (bf16*)e.v, e.gl);
      else
        epi_qkv_linear_kernel<float><<<g, 256, 0, st>>>(cv, M, e.S, e.n_lin, e.hd, e.eps, (float*)e.q, (float*)e.k,
                                                        (float*)e.v, e.gl);
      break;
    }
    case Epi::QKV_FULL: {
      const int64_t warps = M * (e.heads_q + 2 * e.heads_kv);
      const unsigned g = (unsigned)((warps * 32 + 255) / 256);
      if (bf)
        epi_qkv_full_kernel<bf16><<<g, 256, 0, st>>>(cv, M, e.S, e.heads_q, e.heads_kv, e.hd, e.rope, e.start,
                                                     e.table, e.pps, (bf16*)e.q, (bf16*)e.k, (bf16*)e.v);
      else
        epi_qkv_full_kernel<float><<<g, 256, 0, st>>>(cv, M, e.S, e.heads_q, e.heads_kv, e.hd, e.rope, e.start,
                                                      e.table, e.pps, (float*)e.q, (float*)e.k, (float*)e.v);
      break;
    }
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// causal GQA attention, one warp per (sequence, q head, query); online softmax
// q [B][nq][S][hd]; K, V paged caches (see kv_row); o [B*S][nq*hd]
// ---------------------------------------------------------------------------
template <typename T, int EPL>
__global__ void attention_simple_kernel(const T* q, const T* K, const T* V, T* o, int B, int S, int nq, int nkv,
                                        const int32_t* table, int pps, const int32_t* start) {
  const int64_t w = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int hd = EPL * 32;
  if (w >= (int64_t)B * nq * S) return;
  const int t = (int)(w % S);
  const int h = (int)((w / S) % nq);
  const int b = (int)(w / ((int64_t)S * nq));
  const int kh = h / (nq / nkv);
  const int64_t pos = start[b] + t;
  const float scale = rsqrtf((float)hd);
  float qv[EPL], acc[EPL];
  const T* qr = q + (((int64_t)b * nq + h) * S + t) * hd;
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    qv[i] = to_f(qr[lane + 32 * i]) * scale;
    acc[i] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  for (int64_t j = 0; j <= pos; ++j) {
    const int64_t kr = kv_row(table, pps, nkv, b, kh, j) * hd;
    float sc = 0.f;
#pragma unroll
    for (int i = 0; i < EPL; ++i) sc += qv[i] * to_f(K[kr + lane + 32 * i]);
    sc = warp_sum(sc);
    const float mn = fmaxf(m, sc);
    const float corr = __expf(m - mn), p = __expf(sc - mn);
    l = l * corr + p;
#pragma unroll
    for (int i = 0; i < EPL; ++i) acc[i] = acc[i] * corr + p * to_f(V[kr + lane + 32 * i]);
    m = mn;
  }
  T* orow = o + ((int64_t)b * S + t) * nq * hd + (int64_t)h * hd;
#pragma unroll
  for (int i = 0; i < EPL; ++i) orow[lane + 32 * i] = from_f<T>(acc[i] / l);
}

cudaError_t launch_attention_simple(const void* q, const void* K, const void* V, void* o, bool bf, int B, int S,
                                    int nq, int nkv, int hd, const int32_t* table, int pps, const int32_t* start,
                                    cudaStream_t st) {
  const int64_t warps = (int64_t)B * nq * S;
  if (warps == 0) return cudaSuccess;
  const unsigned g = (unsigned)((warps * 32 + 255) / 256);
#define LOOP_ATT(EPL)                                                                                            \
  if (bf)                                                                                                        \
    attention_simple_kernel<bf16, EPL><<<g, 256, 0, st>>>((const bf16*)q, (const bf16*)K, (const bf16*)V,       \
                                                          (bf16*)o, B, S, nq, nkv, table, pps, start);           \
  else                                                                                                           \
    attention_simple_kernel<float, EPL><<<g, 256, 0, st>>>((const float*)q, (const float*)K, (const float*)V,    \
                                                           (float*)o, B, S, nq, nkv, table, pps, start);
  switch (hd) {
    case 32: LOOP_ATT(1); break;
    case 64: LOOP_ATT(2); break;
    case 128: LOOP_ATT(4); break;
    default: return cudaErrorInvalidValue;
  }
#undef LOOP_ATT
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// gated linear attention, token by token:  S_t = g_t S_{t-1} + k_t v_t^T,
// o_t = q_t S_t.  One CTA per (sequence, head), thread e owns column e of the
// state (kept in shared memory), gl holds log g.
// q, k, v [B][nh][S][d]; gl [B][nh][S]; state [B][nh][d][d]; o [B*S][nh*d]
// ---------------------------------------------------------------------------
template <typename T>
__global__ void gla_recurrent_kernel(const T* q, const T* k, const T* v, const float* gl, float* state, T* o, int S,
                                     int nh, int d) {
  extern __shared__ float sm[];
  float* Sm = sm;            // [d][d]
  float* qs = sm + d * d;    // [d]
  float* ks = qs + d;        // [d]
  const int bh = blockIdx.x;
  const int b = bh / nh, h = bh % nh;
  const int e = threadIdx.x;
  float* st = state + (int64_t)bh * d * d;
  for (int a = 0; a < d; ++a) Sm[a * d + e] = st[a * d + e];
  const int64_t base = (int64_t)bh * S;
  for (int t = 0; t < S; ++t) {
    __syncthreads();
    qs[e] = to_f(q[(base + t) * d + e]);
    ks[e] = to_f(k[(base + t) * d + e]);
    __syncthreads();
    const float g = __expf(gl[base + t]);
    const float ve = to_f(v[(base + t) * d + e]);
    float acc = 0.f;
    for (int a = 0; a < d; ++a) {
      const float sv = g * Sm[a * d + e] + ks[a] * ve;
      Sm[a * d + e] = sv;
      acc += qs[a] * sv;
    }
    o[((int64_t)b * S + t) * nh * d + (int64_t)h * d + e] = from_f<T>(acc);
  }
  for (int a = 0; a < d; ++a) st[a * d + e] = Sm[a * d + e];
}

cudaError_t launch_gla_recurrent(const void* q, const void* k, const void* v, const float* gl, float* state, void* o,
                                 bool bf, int B, int S, int nh, int d, cudaStream_t st) {
  if (B == 0 || S == 0) return cudaSuccess;
  const size_t smem = sizeof(float) * ((size_t)d * d + 2 * d);
  if (smem > 232448) return cudaErrorInvalidValue;
  static std::atomic<uint64_t> set_bf{0}, set_f{0};  // raised to the per-block maximum once per device
  if (bf) {
    if (cudaError_t e = set_smem_limit(gla_recurrent_kernel<bf16>, 232448, set_bf); e != cudaSuccess) return e;
    gla_recurrent_kernel<bf16><<<B * nh, d, smem, st>>>((const bf16*)q, (const bf16*)k, (const bf16*)v, gl, state,
                                                        (bf16*)o, S, nh, d);
  } else {
    if (cudaError_t e = set_smem_limit(gla_recurrent_kernel<float>, 232448, set_f); e != cudaSuccess) return e;
    gla_recurrent_kernel<float><<<B * nh, d, smem, st>>>((const float*)q, (const float*)k, (const float*)v, gl,
                                                         state, (float*)o, S, nh, d);
  }
  return cudaGetLastError();
}

}  // namespace loopk
