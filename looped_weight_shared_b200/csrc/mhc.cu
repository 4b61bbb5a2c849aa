// Row-wise kernels of the looped decoder: the seeded weight generator, the
// embedding gather, RMSNorm, the fused mHC prologue (coefficients, Sinkhorn,
// stream read, RMSNorm), stream expand/collapse and the standalone Sinkhorn.
//
// mHC follows "How Does SenseNova-Loop Get More Depth Without More
// Parameters?", section "What does two-stream mHC do?": per site and token,
//   r = RMS of the flattened streams (s_0, s_1),   l = ((s / r) * gamma) . Phi,
//   H_pre = sigmoid(l[0:2]), H_post = 2 sigmoid(l[2:4]),
//   H_res = Sinkhorn_20(exp(l[4:8] as 2x2)),   x = sum_i H_pre[i] s_i,
//   x_hat = RMSNorm(x) * gain.

#include <math.h>

#include <algorithm>

#include "model.h"

namespace loopk {

__device__ int g_status = 0;

int* status_ptr() {
  int* p = nullptr;
  if (cudaGetSymbolAddress((void**)&p, g_status) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return p;
}

// ---------------------------------------------------------------------------
// SplitMix64 counter stream (Steele, Lea, Flood 2014) and Box-Muller normals.
// ---------------------------------------------------------------------------
LOOP_DEV uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}
__host__ __device__ inline uint64_t mix64_h(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}
LOOP_DEV double box_muller(uint64_t key, uint64_t i) {
  const uint64_t p = i >> 1;
  const uint64_t g = 0x9E3779B97F4A7C15ull;
  const double u1 = (double)((mix64(key + (2 * p + 1) * g) >> 11) + 1) * 0x1.0p-53;
  const double u2 = (double)(mix64(key + (2 * p + 2) * g) >> 11) * 0x1.0p-53;
  const double r = sqrt(-2.0 * log(u1));
  const double t = 2.0 * 3.141592653589793238462643383279502884 * u2;
  return (i & 1) ? r * sin(t) : r * cos(t);
}

// dst rows [dst_row0, dst_row0 + rows) of a [*][cols] matrix get stream rows
// [src_row0, src_row0 + rows): element (r, c) is counter index r * cols + c.
__global__ void fill_normal_kernel(void* dst, int bf, int64_t rows, int64_t cols, int64_t dst_row0, uint64_t key,
                                   int64_t src_row0, double scale) {
  const int64_t n = rows * cols;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / cols, c = i % cols;
    const float x = (float)(scale * box_muller(key, (uint64_t)((src_row0 + r) * cols + c)));
    const int64_t o = (dst_row0 + r) * cols + c;
    if (bf) ((bf16*)dst)[o] = __float2bfloat16_rn(x);
    else ((float*)dst)[o] = x;
  }
}

cudaError_t launch_fill_normal(void* dst, bool bf, int64_t rows, int64_t cols, int64_t dst_row0, uint64_t seed,
                               uint64_t stream, int64_t src_row0, double scale, cudaStream_t st) {
  const uint64_t key = mix64_h(mix64_h(seed) + stream);
  const int64_t n = rows * cols;
  const int blocks = (int)std::min<int64_t>((n + 255) / 256, 148 * 32);
  fill_normal_kernel<<<blocks, 256, 0, st>>>(dst, bf, rows, cols, dst_row0, key, src_row0, scale);
  return cudaGetLastError();
}

__global__ void fill_const_kernel(float* d, int64_t n, float v) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    d[i] = v;
}
cudaError_t launch_fill_const(float* d, int64_t n, float v, cudaStream_t st) {
  fill_const_kernel<<<(int)std::min<int64_t>((n + 255) / 256, 4096), 256, 0, st>>>(d, n, v);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// embedding gather: h[t] = E[tok[t]] (fp32 residual); out-of-range ids flag
// the status word and give zeros
// ---------------------------------------------------------------------------
template <typename T>
__global__ void embed_kernel(const int32_t* tok, const T* E, int H, int V, float* h) {
  const int64_t t = blockIdx.x;
  const int32_t id = tok[t];
  const bool ok = id >= 0 && id < V;
  if (!ok && threadIdx.x == 0) atomicOr(&g_status, STATUS_BAD_TOKEN);
  const T* src = E + (int64_t)(ok ? id : 0) * H;
  for (int i = threadIdx.x; i < H; i += blockDim.x) h[t * H + i] = ok ? to_f(src[i]) : 0.f;
}
cudaError_t launch_embed(const int32_t* tok, const void* E, bool bf, int64_t T, int H, int V, float* h,
                         cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  if (bf) embed_kernel<bf16><<<(unsigned)T, 256, 0, st>>>(tok, (const bf16*)E, H, V, h);
  else embed_kernel<float><<<(unsigned)T, 256, 0, st>>>(tok, (const float*)E, H, V, h);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// RMSNorm: y[r] = x[src] / sqrt(mean(x[src]^2) + eps) * gain, src = r*step+off
// ---------------------------------------------------------------------------
template <typename T>
__global__ void rmsnorm_kernel(const float* x, int H, int64_t step, int64_t off, const float* gain, float eps, T* y) {
  __shared__ float red[32];
  griddep_launch_dependents();  // a decode GEMM after this may start streaming its weights
  const int64_t r = blockIdx.x;
  const float* xr = x + (r * step + off) * H;
  float ss = 0.f;
  for (int i = threadIdx.x; i < H; i += blockDim.x) ss += xr[i] * xr[i];
  ss = block_sum(ss, red);
  const float inv = rsqrtf(ss / H + eps);
  for (int i = threadIdx.x; i < H; i += blockDim.x) y[r * H + i] = from_f<T>(xr[i] * inv * gain[i]);
}
// The same for H = 512 NPL: 128 threads keep the row's NPL float4 each in
// registers (one pass over the row), one block reduction, vector stores.
template <typename T, int NPL>
__global__ void __launch_bounds__(128)
    rmsnorm_vec_kernel(const float* __restrict__ x, int64_t step, int64_t off, const float* __restrict__ gain,
                       float eps, T* __restrict__ y) {
  constexpr int H = 512 * NPL;
  __shared__ float red[4];
  griddep_launch_dependents();  // a decode GEMM after this may start streaming its weights
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t r = blockIdx.x;
  const float4* xr = reinterpret_cast<const float4*>(x + (r * step + off) * H);
  float4 a[NPL];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    a[i] = xr[tid + 128 * i];
    ss += a[i].x * a[i].x + a[i].y * a[i].y + a[i].z * a[i].z + a[i].w * a[i].w;
  }
  ss = warp_sum(ss);
  if (lane == 0) red[warp] = ss;
  __syncthreads();
  const float inv = rsqrtf((red[0] + red[1] + red[2] + red[3]) / H + eps);
  const float4* g4 = reinterpret_cast<const float4*>(gain);
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const float4 g = g4[tid + 128 * i];
    const float x0 = a[i].x * inv * g.x, x1 = a[i].y * inv * g.y, x2 = a[i].z * inv * g.z, x3 = a[i].w * inv * g.w;
    if constexpr (sizeof(T) == 2) {
      uint2 u;
      u.x = pack_bf16x2(x0, x1);
      u.y = pack_bf16x2(x2, x3);
      reinterpret_cast<uint2*>(y + r * H)[tid + 128 * i] = u;
    } else {
      reinterpret_cast<float4*>(y + r * H)[tid + 128 * i] = make_float4(x0, x1, x2, x3);
    }
  }
}

cudaError_t launch_rmsnorm(const float* x, int64_t rows, int H, int64_t step, int64_t off, const float* gain,
                           float eps, void* y, bool bf, cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  if (H % 512 == 0) {
#define LOOP_RMS(NPL)                                                                                          \
  case NPL:                                                                                                    \
    if (bf) rmsnorm_vec_kernel<bf16, NPL><<<(unsigned)rows, 128, 0, st>>>(x, step, off, gain, eps, (bf16*)y);   \
    else rmsnorm_vec_kernel<float, NPL><<<(unsigned)rows, 128, 0, st>>>(x, step, off, gain, eps, (float*)y);    \
    return cudaGetLastError();
    switch (H / 512) {
      LOOP_RMS(1)
      LOOP_RMS(2)
      LOOP_RMS(4)
      LOOP_RMS(8)
      LOOP_RMS(12)
      default: break;
    }
#undef LOOP_RMS
  }
  if (bf) rmsnorm_kernel<bf16><<<(unsigned)rows, 256, 0, st>>>(x, H, step, off, gain, eps, (bf16*)y);
  else rmsnorm_kernel<float><<<(unsigned)rows, 256, 0, st>>>(x, H, step, off, gain, eps, (float*)y);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// The library's fixed exponential and Sinkhorn (bit-exact contract).  Every
// operation is an explicitly rounded IEEE operation so the compiler cannot
// contract or reorder it: Cody-Waite x = k ln2 + r with ln2 split into the
// 15-bit head 22713/32768 and its remainder, degree-7 Taylor polynomial by
// Horner with fused multiply-adds, then an exact scaling by 2^k.
// ---------------------------------------------------------------------------
LOOP_DEV float scale_pow2(float p, int k) {
  // one rounding at most: the first factor is exact, the second rounds once
  if (k > 127) return __fmul_rn(__fmul_rn(p, __int_as_float(254 << 23)), __int_as_float((k - 127 + 127) << 23));
  if (k >= -125) return __fmul_rn(p, __int_as_float((k + 127) << 23));
  return __fmul_rn(__fmul_rn(p, __int_as_float((k + 64 + 127) << 23)), __int_as_float((-64 + 127) << 23));
}
LOOP_DEV float exp_fixed(float x) {
  if (isnan(x)) return x;
  if (x < -104.0f) return 0.0f;
  if (x > 88.72f) return __int_as_float(0x7f800000);
  const float log2e = 1.44269504088896340736f;
  const float ln2_hi = 0.693145751953125f;
  const float ln2_lo = 1.42860682030941723212e-6f;
  const float k = rintf(__fmul_rn(x, log2e));
  float r = __fmaf_rn(-k, ln2_hi, x);
  r = __fmaf_rn(-k, ln2_lo, r);
  float p = 1.0f / 5040.0f;
  p = __fmaf_rn(p, r, 1.0f / 720.0f);
  p = __fmaf_rn(p, r, 1.0f / 120.0f);
  p = __fmaf_rn(p, r, 1.0f / 24.0f);
  p = __fmaf_rn(p, r, 1.0f / 6.0f);
  p = __fmaf_rn(p, r, 0.5f);
  p = __fmaf_rn(p, r, 1.0f);
  p = __fmaf_rn(p, r, 1.0f);
  return scale_pow2(p, (int)k);
}

template <int N>
LOOP_DEV void sinkhorn_fixed(const float* l, float* P, int iters) {
  float mx = l[0];
#pragma unroll
  for (int i = 1; i < N * N; ++i) mx = l[i] > mx ? l[i] : mx;
#pragma unroll
  for (int i = 0; i < N * N; ++i) P[i] = exp_fixed(__fsub_rn(l[i], mx));
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int r = 0; r < N; ++r) {
      float s = 0.f;
#pragma unroll
      for (int c = 0; c < N; ++c) s = __fadd_rn(s, P[r * N + c]);
#pragma unroll
      for (int c = 0; c < N; ++c) P[r * N + c] = __fdiv_rn(P[r * N + c], s);
    }
#pragma unroll
    for (int c = 0; c < N; ++c) {
      float s = 0.f;
#pragma unroll
      for (int r = 0; r < N; ++r) s = __fadd_rn(s, P[r * N + c]);
#pragma unroll
      for (int r = 0; r < N; ++r) P[r * N + c] = __fdiv_rn(P[r * N + c], s);
    }
  }
}

template <int N>
__global__ void sinkhorn_kernel(const float* l, float* out, int64_t count, int iters) {
  const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i >= count) return;
  float a[N * N], P[N * N];
#pragma unroll
  for (int j = 0; j < N * N; ++j) a[j] = l[i * N * N + j];
  sinkhorn_fixed<N>(a, P, iters);
#pragma unroll
  for (int j = 0; j < N * N; ++j) out[i * N * N + j] = P[j];
}

cudaError_t launch_sinkhorn(const float* l, float* out, int64_t count, int n, int iters, cudaStream_t st) {
  if (count == 0) return cudaSuccess;
  const unsigned g = (unsigned)((count + 127) / 128);
  switch (n) {
    case 1: sinkhorn_kernel<1><<<g, 128, 0, st>>>(l, out, count, iters); break;
    case 2: sinkhorn_kernel<2><<<g, 128, 0, st>>>(l, out, count, iters); break;
    case 3: sinkhorn_kernel<3><<<g, 128, 0, st>>>(l, out, count, iters); break;
    case 4: sinkhorn_kernel<4><<<g, 128, 0, st>>>(l, out, count, iters); break;
    case 5: sinkhorn_kernel<5><<<g, 128, 0, st>>>(l, out, count, iters); break;
    case 6: sinkhorn_kernel<6><<<g, 128, 0, st>>>(l, out, count, iters); break;
    case 7: sinkhorn_kernel<7><<<g, 128, 0, st>>>(l, out, count, iters); break;
    case 8: sinkhorn_kernel<8><<<g, 128, 0, st>>>(l, out, count, iters); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// mHC prologue for n = 2 streams, in two HBM-streaming kernels.
//
// (A) mhc_partial: the flattened stream vector u = (s_0, s_1) of a token has
//     2H entries, cut into `parts` equal parts (2 for long inputs; more when
//     few tokens must still spread over many SMs); CTA (blk, part) forms
//     Phi * gamma over its part once in shared memory and every warp streams
//     4 tokens of that part with float4 loads, so each value read is used 4
//     times; the sums run as packed fp32x2 FMAs over column pairs.  It writes,
//     per token and part, the 8 partial projections sum_i s_i gamma_i Phi_ci
//     and the partial sum of squares.
// (B) mhc_read: one warp per token folds the two halves into
//     l = (sum / r), r = sqrt(sum of squares / 2H + eps), forms H_pre, H_post
//     and H_res = Sinkhorn(exp(l[4:8])), then reads x = H_pre0 s_0 + H_pre1 s_1
//     and writes RMSNorm(x) * gain.  The stream rows are read twice (sum of
//     squares, then the write), the second time from L1/L2.
// ---------------------------------------------------------------------------
constexpr int MHCA_WARPS = 12, MHCA_TOK = 4;  // tokens per warp
constexpr int MHCA_THREADS = MHCA_WARPS * 32;
constexpr int MHCB_WARPS = 8;

__global__ void __launch_bounds__(MHCA_THREADS, 1)
    mhc_partial_kernel(const float* __restrict__ s, int64_t T, int H, const float* __restrict__ gamma,
                       const float* __restrict__ phi, int parts, float* __restrict__ part) {
  extern __shared__ float4 sm4[];
  const int p = blockIdx.y;
  const int D = 2 * H, PL = D / parts, PL4 = PL / 4;
  const int i0 = p * PL;                  // this part's first entry of the flattened streams
  const int stream = i0 / H, col0 = i0 % H;  // a part lies inside one stream
  float4* sw = sm4;  // [8][PL4]: Phi * gamma over this part, formed once per CTA
  for (int i = threadIdx.x; i < PL4; i += MHCA_THREADS) {
    const float4 g = reinterpret_cast<const float4*>(gamma + i0)[i];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const float4 ph = reinterpret_cast<const float4*>(phi + (int64_t)c * D + i0)[i];
      sw[c * PL4 + i] = make_float4(ph.x * g.x, ph.y * g.y, ph.z * g.z, ph.w * g.w);
    }
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t0 = ((int64_t)blockIdx.x * MHCA_WARPS + warp) * MHCA_TOK;
  if (t0 >= T) return;
  const int ntok = (int)(T - t0 < MHCA_TOK ? T - t0 : MHCA_TOK);
  const int H4 = H / 4;
  const float4* base = reinterpret_cast<const float4*>(s + ((int64_t)stream * T + t0) * H + col0);
  // per token: 8 projections and the sum of squares, each as a pair of
  // partial sums (even and odd columns) so the products run as packed fp32x2 FMAs
  float2 acc[MHCA_TOK][9];
#pragma unroll
  for (int j = 0; j < MHCA_TOK; ++j)
#pragma unroll
    for (int c = 0; c < 9; ++c) acc[j][c] = make_float2(0.f, 0.f);
#pragma unroll 2
  for (int f = lane; f < PL4; f += 32) {
    float4 v[MHCA_TOK];
#pragma unroll
    for (int j = 0; j < MHCA_TOK; ++j) v[j] = j < ntok ? __ldcs(base + (int64_t)j * H4 + f) : make_float4(0, 0, 0, 0);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const float4 w = sw[c * PL4 + f];
#pragma unroll
      for (int j = 0; j < MHCA_TOK; ++j) {
        acc[j][c] = ffma2(make_float2(v[j].x, v[j].y), make_float2(w.x, w.y), acc[j][c]);
        acc[j][c] = ffma2(make_float2(v[j].z, v[j].w), make_float2(w.z, w.w), acc[j][c]);
      }
    }
#pragma unroll
    for (int j = 0; j < MHCA_TOK; ++j) {
      acc[j][8] = ffma2(make_float2(v[j].x, v[j].y), make_float2(v[j].x, v[j].y), acc[j][8]);
      acc[j][8] = ffma2(make_float2(v[j].z, v[j].w), make_float2(v[j].z, v[j].w), acc[j][8]);
    }
  }
#pragma unroll
  for (int j = 0; j < MHCA_TOK; ++j)
#pragma unroll
    for (int c = 0; c < 9; ++c) {
      const float r = warp_sum(acc[j][c].x + acc[j][c].y);
      if (lane == c && j < ntok) part[((t0 + j) * parts + p) * 9 + c] = r;
    }
}

template <typename T>
__global__ void __launch_bounds__(MHCB_WARPS * 32)
    mhc_read_kernel(const float* __restrict__ s, int64_t Ttot, int H, const float* __restrict__ part, int parts,
                    const float* __restrict__ gain, int iters, float eps, float* __restrict__ coef, T* __restrict__ xh) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * MHCB_WARPS + warp;
  if (t >= Ttot) return;
  const float* pp = part + t * parts * 9;
  float tot[9];
#pragma unroll
  for (int c = 0; c < 9; ++c) tot[c] = pp[c];
  for (int q = 1; q < parts; ++q)
#pragma unroll
    for (int c = 0; c < 9; ++c) tot[c] += pp[q * 9 + c];
  const float rinv = rsqrtf(tot[8] / (2 * H) + eps);
  float l[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) l[c] = tot[c] * rinv;
  float P[4];
  sinkhorn_fixed<2>(l + 4, P, iters);  // every lane computes the same coefficients
  const float pre0 = sigmoidf_(l[0]), pre1 = sigmoidf_(l[1]);
  if (lane < 8) {
    const float v = lane == 0 ? pre0 : lane == 1 ? pre1 : lane == 2 ? 2.f * sigmoidf_(l[2])
                  : lane == 3 ? 2.f * sigmoidf_(l[3]) : P[lane - 4];
    coef[t * 8 + lane] = v;
  }
  const int H4 = H / 4;
  const float4* s0 = reinterpret_cast<const float4*>(s + t * H);
  const float4* s1 = reinterpret_cast<const float4*>(s + (Ttot + t) * H);
  float ss = 0.f;
#pragma unroll 4
  for (int f = lane; f < H4; f += 32) {
    const float4 a = s0[f], b = s1[f];
    const float x0 = pre0 * a.x + pre1 * b.x, x1 = pre0 * a.y + pre1 * b.y;
    const float x2 = pre0 * a.z + pre1 * b.z, x3 = pre0 * a.w + pre1 * b.w;
    ss += x0 * x0 + x1 * x1 + x2 * x2 + x3 * x3;
  }
  ss = warp_sum(ss);
  const float nrm = rsqrtf(ss / H + eps);
  const float4* g4 = reinterpret_cast<const float4*>(gain);
#pragma unroll 4
  for (int f = lane; f < H4; f += 32) {
    const float4 a = s0[f], b = s1[f], g = g4[f];
    const float x0 = (pre0 * a.x + pre1 * b.x) * nrm * g.x, x1 = (pre0 * a.y + pre1 * b.y) * nrm * g.y;
    const float x2 = (pre0 * a.z + pre1 * b.z) * nrm * g.z, x3 = (pre0 * a.w + pre1 * b.w) * nrm * g.w;
    if constexpr (sizeof(T) == 2) {
      uint2 u;
      u.x = pack_bf16x2(x0, x1);
      u.y = pack_bf16x2(x2, x3);
      reinterpret_cast<uint2*>(xh + t * H)[f] = u;
    } else {
      reinterpret_cast<float4*>(xh + t * H)[f] = make_float4(x0, x1, x2, x3);
    }
  }
}

// Coefficients of every token from its partial sums, one thread per token:
// r, l = sum / r, H_pre, H_post and H_res = Sinkhorn(exp(l[4:8])).
__global__ void __launch_bounds__(128)
    mhc_coef_kernel(const float* __restrict__ part, int parts, int64_t T, int D, int iters, float eps,
                    float* __restrict__ coef) {
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  const float* pp = part + t * parts * 9;
  float tot[9];
#pragma unroll
  for (int c = 0; c < 9; ++c) tot[c] = pp[c];
  for (int q = 1; q < parts; ++q)
#pragma unroll
    for (int c = 0; c < 9; ++c) tot[c] += pp[q * 9 + c];
  const float rinv = rsqrtf(tot[8] / D + eps);
  float l[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) l[c] = tot[c] * rinv;
  float P[4];
  sinkhorn_fixed<2>(l + 4, P, iters);
  float4* co = reinterpret_cast<float4*>(coef + t * 8);
  co[0] = make_float4(sigmoidf_(l[0]), sigmoidf_(l[1]), 2.f * sigmoidf_(l[2]), 2.f * sigmoidf_(l[3]));
  co[1] = make_float4(P[0], P[1], P[2], P[3]);
}

// One-pass reader for H = 512 * NPL (coefficients already formed): one
// 128-thread CTA per token keeps its NPL float4 of both streams in registers,
// so the stream rows are read once.
template <typename T, int NPL>
__global__ void __launch_bounds__(128)
    mhc_read1_kernel(const float* __restrict__ s, int64_t Ttot, const float* __restrict__ coef,
                     const float* __restrict__ gain, float eps, T* __restrict__ xh) {
  constexpr int H = 512 * NPL;
  __shared__ float red[4];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t t = blockIdx.x;
  const float4* s0 = reinterpret_cast<const float4*>(s + t * H);
  const float4* s1 = reinterpret_cast<const float4*>(s + (Ttot + t) * H);
  float4 a[NPL], b[NPL];
#pragma unroll
  for (int i = 0; i < NPL; ++i) a[i] = __ldcs(s0 + tid + 128 * i);
#pragma unroll
  for (int i = 0; i < NPL; ++i) b[i] = __ldcs(s1 + tid + 128 * i);
  const float pre0 = coef[t * 8], pre1 = coef[t * 8 + 1];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    a[i] = make_float4(pre0 * a[i].x + pre1 * b[i].x, pre0 * a[i].y + pre1 * b[i].y, pre0 * a[i].z + pre1 * b[i].z,
                       pre0 * a[i].w + pre1 * b[i].w);
    ss += a[i].x * a[i].x + a[i].y * a[i].y + a[i].z * a[i].z + a[i].w * a[i].w;
  }
  ss = warp_sum(ss);
  if (lane == 0) red[warp] = ss;
  __syncthreads();
  const float nrm = rsqrtf((red[0] + red[1] + red[2] + red[3]) / H + eps);
  const float4* g4 = reinterpret_cast<const float4*>(gain);
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const float4 g = g4[tid + 128 * i];
    const float x0 = a[i].x * nrm * g.x, x1 = a[i].y * nrm * g.y, x2 = a[i].z * nrm * g.z, x3 = a[i].w * nrm * g.w;
    if constexpr (sizeof(T) == 2) {
      uint2 u;
      u.x = pack_bf16x2(x0, x1);
      u.y = pack_bf16x2(x2, x3);
      reinterpret_cast<uint2*>(xh + t * H)[tid + 128 * i] = u;
    } else {
      reinterpret_cast<float4*>(xh + t * H)[tid + 128 * i] = make_float4(x0, x1, x2, x3);
    }
  }
}

// Whole mHC read site for a few tokens (decode): one 256-thread CTA per token
// streams the token's two stream rows once (each thread keeps NK float4 of
// both streams), dots them with gamma * Phi read from L2, reduces the 9 sums
// over the CTA, forms the coefficients in one thread (Sinkhorn included), and
// normalises x = H_pre s from registers.  One launch, no scratch.
template <typename T, int NK>
__global__ void __launch_bounds__(256)
    mhc_token_kernel(const float* __restrict__ s, int64_t Ttot, const float* __restrict__ gamma,
                     const float* __restrict__ phi, const float* __restrict__ gain, int iters, float eps,
                     float* __restrict__ coef, T* __restrict__ xh) {
  constexpr int H = 1024 * NK, H4 = H / 4, D = 2 * H;
  __shared__ float red[8][9];
  griddep_launch_dependents();  // the decode GEMM after this may start streaming its weights
  __shared__ float cf[2];
  __shared__ float red2[8];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t t = blockIdx.x;
  const float4* s0 = reinterpret_cast<const float4*>(s + t * H);
  const float4* s1 = reinterpret_cast<const float4*>(s + (Ttot + t) * H);
  float4 a[NK], b[NK];
#pragma unroll
  for (int k = 0; k < NK; ++k) a[k] = s0[tid + 256 * k];
#pragma unroll
  for (int k = 0; k < NK; ++k) b[k] = s1[tid + 256 * k];
  float acc[9];
#pragma unroll
  for (int c = 0; c < 9; ++c) acc[c] = 0.f;
  const float4* g4 = reinterpret_cast<const float4*>(gamma);
#pragma unroll
  for (int k = 0; k < 2 * NK; ++k) {
    const float4 v = k < NK ? a[k] : b[k - NK];
    const int f = (k < NK ? 0 : H4) + tid + 256 * (k % NK);
    const float4 g = g4[f];
    const float4 w = make_float4(v.x * g.x, v.y * g.y, v.z * g.z, v.w * g.w);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const float4 p = reinterpret_cast<const float4*>(phi + (int64_t)c * D)[f];
      acc[c] += w.x * p.x + w.y * p.y + w.z * p.z + w.w * p.w;
    }
    acc[8] += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
  }
#pragma unroll
  for (int c = 0; c < 9; ++c) {
    const float r = warp_sum(acc[c]);
    if (lane == 0) red[warp][c] = r;
  }
  __syncthreads();
  if (tid == 0) {
    float tot[9];
    for (int c = 0; c < 9; ++c) {
      float x = 0.f;
      for (int w = 0; w < 8; ++w) x += red[w][c];
      tot[c] = x;
    }
    const float rinv = rsqrtf(tot[8] / D + eps);
    float l[8];
    for (int c = 0; c < 8; ++c) l[c] = tot[c] * rinv;
    float P[4];
    sinkhorn_fixed<2>(l + 4, P, iters);
    const float pre0 = sigmoidf_(l[0]), pre1 = sigmoidf_(l[1]);
    cf[0] = pre0;
    cf[1] = pre1;
    float4* co = reinterpret_cast<float4*>(coef + t * 8);
    co[0] = make_float4(pre0, pre1, 2.f * sigmoidf_(l[2]), 2.f * sigmoidf_(l[3]));
    co[1] = make_float4(P[0], P[1], P[2], P[3]);
  }
  __syncthreads();
  const float pre0 = cf[0], pre1 = cf[1];
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < NK; ++k) {
    a[k] = make_float4(pre0 * a[k].x + pre1 * b[k].x, pre0 * a[k].y + pre1 * b[k].y, pre0 * a[k].z + pre1 * b[k].z,
                       pre0 * a[k].w + pre1 * b[k].w);
    ss += a[k].x * a[k].x + a[k].y * a[k].y + a[k].z * a[k].z + a[k].w * a[k].w;
  }
  ss = warp_sum(ss);
  if (lane == 0) red2[warp] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w) tot += red2[w];
  const float nrm = rsqrtf(tot / H + eps);
  const float4* gn = reinterpret_cast<const float4*>(gain);
#pragma unroll
  for (int k = 0; k < NK; ++k) {
    const int f = tid + 256 * k;
    const float4 g = gn[f];
    const float x0 = a[k].x * nrm * g.x, x1 = a[k].y * nrm * g.y, x2 = a[k].z * nrm * g.z, x3 = a[k].w * nrm * g.w;
    if constexpr (sizeof(T) == 2) {
      uint2 u;
      u.x = pack_bf16x2(x0, x1);
      u.y = pack_bf16x2(x2, x3);
      reinterpret_cast<uint2*>(xh + t * H)[f] = u;
    } else {
      reinterpret_cast<float4*>(xh + t * H)[f] = make_float4(x0, x1, x2, x3);
    }
  }
}

bool mhc_token_supported(int H) { return H == 4096; }

cudaError_t launch_mhc_token(const float* s, int64_t T, int H, const float* gamma, const float* phi,
                             const float* gain, int iters, float eps, float* coef, void* xh, bool bf, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  if (H != 4096) return cudaErrorInvalidValue;
  if (bf) mhc_token_kernel<bf16, 4><<<(unsigned)T, 256, 0, st>>>(s, T, gamma, phi, gain, iters, eps, coef, (bf16*)xh);
  else mhc_token_kernel<float, 4><<<(unsigned)T, 256, 0, st>>>(s, T, gamma, phi, gain, iters, eps, coef, (float*)xh);
  return cudaGetLastError();
}

size_t mhc_partial_smem(int H) { return (size_t)8 * H * sizeof(float); }  // Phi * gamma of half the streams

__global__ void mhc_phig_kernel(const float* __restrict__ gamma, const float* __restrict__ phi, int64_t D,
                                float* __restrict__ out) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < 8 * D; i += (int64_t)gridDim.x * blockDim.x)
    out[i] = phi[i] * gamma[i % D];
}
cudaError_t launch_mhc_phig(const float* gamma, const float* phi, int64_t D, float* out, cudaStream_t st) {
  mhc_phig_kernel<<<(unsigned)std::min<int64_t>((8 * D + 255) / 256, 1024), 256, 0, st>>>(gamma, phi, D, out);
  return cudaGetLastError();
}

cudaError_t launch_mhc_coef_read(const float* part, int parts, const float* s, int64_t T, int H, const float* gain,
                                 int iters, float eps, float* coef, void* xh, bool bf, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  if (H != 4096 || parts < 1) return cudaErrorInvalidValue;
  mhc_coef_kernel<<<(unsigned)((T + 127) / 128), 128, 0, st>>>(part, parts, T, 2 * H, iters, eps, coef);
  if (bf) mhc_read1_kernel<bf16, 8><<<(unsigned)T, 128, 0, st>>>(s, T, coef, gain, eps, (bf16*)xh);
  else mhc_read1_kernel<float, 8><<<(unsigned)T, 128, 0, st>>>(s, T, coef, gain, eps, (float*)xh);
  return cudaGetLastError();
}

cudaError_t launch_mhc_prologue(const float* s, int64_t T, int H, const float* gamma, const float* phi,
                                const float* gain, int iters, float eps, float* coef, void* xh, bool bf,
                                float* part, cudaStream_t st, int parts, bool fused_read) {
  if (T == 0) return cudaSuccess;
  if (H % 4 != 0 || H > 6144) return cudaErrorInvalidValue;
  if (parts < 2 || parts % 2 != 0 || (2 * H) % (4 * parts) != 0 || H % (2 * H / parts) != 0)
    return cudaErrorInvalidValue;
  const int smem = (int)(mhc_partial_smem(H) * 2 / parts);
  static std::atomic<uint64_t> smem_set{0};  // the limit for the widest H, raised once per device
  if (cudaError_t e = set_smem_limit(mhc_partial_kernel, (int)mhc_partial_smem(6144), smem_set); e != cudaSuccess)
    return e;
  const int64_t per_cta = (int64_t)MHCA_WARPS * MHCA_TOK;
  dim3 ga((unsigned)((T + per_cta - 1) / per_cta), (unsigned)parts);
  mhc_partial_kernel<<<ga, MHCA_THREADS, smem, st>>>(s, T, H, gamma, phi, parts, part);
  if (H == 4096 && !fused_read) {  // the 9B width: coefficients, then one pass over the streams
    mhc_coef_kernel<<<(unsigned)((T + 127) / 128), 128, 0, st>>>(part, parts, T, 2 * H, iters, eps, coef);
    if (bf) mhc_read1_kernel<bf16, 8><<<(unsigned)T, 128, 0, st>>>(s, T, coef, gain, eps, (bf16*)xh);
    else mhc_read1_kernel<float, 8><<<(unsigned)T, 128, 0, st>>>(s, T, coef, gain, eps, (float*)xh);
    return cudaGetLastError();
  }
  const unsigned gb = (unsigned)((T + MHCB_WARPS - 1) / MHCB_WARPS);
  if (bf)
    mhc_read_kernel<bf16><<<gb, MHCB_WARPS * 32, 0, st>>>(s, T, H, part, parts, gain, iters, eps, coef, (bf16*)xh);
  else
    mhc_read_kernel<float><<<gb, MHCB_WARPS * 32, 0, st>>>(s, T, H, part, parts, gain, iters, eps, coef,
                                                           (float*)xh);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// streams: expand s_0 = s_1 = h at loop entry, collapse h = s_0 + s_1 at exit
// ---------------------------------------------------------------------------
__global__ void expand_kernel(const float4* h, float4* s, int64_t n4) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x) {
    const float4 v = h[i];
    s[i] = v;
    s[i + n4] = v;
  }
}
__global__ void collapse_kernel(const float4* s, float4* h, int64_t n4) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x) {
    const float4 a = s[i], b = s[i + n4];
    h[i] = make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
  }
}
cudaError_t launch_expand(const float* h, float* s, int64_t n, cudaStream_t st) {
  const int64_t n4 = n / 4;
  expand_kernel<<<(unsigned)std::min<int64_t>((n4 + 255) / 256, 148 * 16), 256, 0, st>>>((const float4*)h,
                                                                                         (float4*)s, n4);
  return cudaGetLastError();
}
cudaError_t launch_collapse(const float* s, float* h, int64_t n, cudaStream_t st) {
  const int64_t n4 = n / 4;
  collapse_kernel<<<(unsigned)std::min<int64_t>((n4 + 255) / 256, 148 * 16), 256, 0, st>>>((const float4*)s,
                                                                                           (float4*)h, n4);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// RoPE table: (cos, sin) of pos * base^(-2i/hd), angle in fp64
// ---------------------------------------------------------------------------
__global__ void rope_table_kernel(float2* tab, int64_t ctx, int half, double base, int hd) {
  const int64_t n = ctx * half;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t p = i / half;
    const int j = (int)(i % half);
    const double ang = (double)p * pow(base, -2.0 * j / hd);
    double sn, cs;
    sincos(ang, &sn, &cs);
    tab[i] = make_float2((float)cs, (float)sn);
  }
}
cudaError_t launch_rope_table(float2* tab, int64_t ctx, int hd, double base, cudaStream_t st) {
  const int64_t n = ctx * (hd / 2);
  rope_table_kernel<<<(unsigned)std::min<int64_t>((n + 255) / 256, 148 * 16), 256, 0, st>>>(tab, ctx, hd / 2, base,
                                                                                           hd);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// inspection helpers
// ---------------------------------------------------------------------------
template <typename T>
__global__ void cache_to_f32_kernel(const T* src, const int32_t* table, int pps, int B, int nkv, int len, int hd,
                                    float* dst) {
  const int64_t n = (int64_t)B * nkv * len * hd;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t e = i % hd, p = (i / hd) % len, bh = i / ((int64_t)hd * len);
    dst[i] = to_f(src[kv_row(table, pps, nkv, bh / nkv, (int)(bh % nkv), p) * hd + e]);
  }
}
cudaError_t launch_cache_to_f32(const void* src, bool bf, const int32_t* table, int pps, int B, int nkv, int len,
                                int hd, float* dst, cudaStream_t st) {
  const int64_t n = (int64_t)B * nkv * len * hd;
  if (n == 0) return cudaSuccess;
  const unsigned g = (unsigned)std::min<int64_t>((n + 255) / 256, 148 * 16);
  if (bf) cache_to_f32_kernel<bf16><<<g, 256, 0, st>>>((const bf16*)src, table, pps, B, nkv, len, hd, dst);
  else cache_to_f32_kernel<float><<<g, 256, 0, st>>>((const float*)src, table, pps, B, nkv, len, hd, dst);
  return cudaGetLastError();
}

// rows 0..len-1 of (sequence b, kv head h), 16 bytes per thread
__global__ void cache_rows_kernel(const uint4* src, const int32_t* table, int pps, int nkv, int b, int h, int len,
                                  int row16, uint4* dst) {
  const int64_t n = (int64_t)len * row16;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t p = i / row16, e = i % row16;
    dst[i] = src[kv_row(table, pps, nkv, b, h, p) * row16 + e];
  }
}
cudaError_t launch_cache_rows(const void* src, size_t esize, const int32_t* table, int pps, int nkv, int b, int h,
                              int len, int hd, void* dst, cudaStream_t st) {
  if (len == 0) return cudaSuccess;
  const int row16 = (int)(hd * esize / 16);
  const unsigned g = (unsigned)std::min<int64_t>(((int64_t)len * row16 + 255) / 256, 148 * 16);
  cache_rows_kernel<<<g, 256, 0, st>>>((const uint4*)src, table, pps, nkv, b, h, len, row16, (uint4*)dst);
  return cudaGetLastError();
}

// table[idx[i]] = page[i]: the page-table entries a call changes, passed by
// value so the update is ordered on the stream without a host copy
constexpr int kTableBatch = 240;
struct TableSet {
  int32_t idx[kTableBatch], page[kTableBatch];
};
__global__ void table_set_kernel(int32_t* table, TableSet u, int n) {
  const int i = threadIdx.x;
  if (i < n) table[u.idx[i]] = u.page[i];
}
cudaError_t launch_table_set(int32_t* table, const int32_t* idx, const int32_t* page, int n, cudaStream_t st) {
  for (int o = 0; o < n; o += kTableBatch) {
    TableSet u;
    const int k = std::min(kTableBatch, n - o);
    for (int i = 0; i < k; ++i) {
      u.idx[i] = idx[o + i];
      u.page[i] = page[o + i];
    }
    table_set_kernel<<<1, 256, 0, st>>>(table, u, k);
    if (cudaError_t e = cudaGetLastError(); e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

template <typename T>
__global__ void weight_to_f32_kernel(const T* src, int64_t n, float* dst) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    dst[i] = to_f(src[i]);
}
cudaError_t launch_weight_to_f32(const void* src, bool bf, int64_t rows, int64_t cols, int64_t src_row0, float* dst,
                                 cudaStream_t st) {
  const int64_t n = rows * cols;
  if (n == 0) return cudaSuccess;
  const unsigned g = (unsigned)std::min<int64_t>((n + 255) / 256, 148 * 16);
  if (bf) weight_to_f32_kernel<bf16><<<g, 256, 0, st>>>((const bf16*)src + src_row0 * cols, n, dst);
  else weight_to_f32_kernel<float><<<g, 256, 0, st>>>((const float*)src + src_row0 * cols, n, dst);
  return cudaGetLastError();
}

__global__ void advance_kernel(int32_t* len, int B, int by) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) len[b] += by;
}
__global__ void set_len_kernel(int32_t* len, int B, int S) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) len[b] = S;
}
cudaError_t launch_set_len(int32_t* len, int B, int S, cudaStream_t st) {
  set_len_kernel<<<(B + 127) / 128, 128, 0, st>>>(len, B, S);
  return cudaGetLastError();
}
cudaError_t launch_advance(int32_t* len, int B, cudaStream_t st, int by) {
  advance_kernel<<<(B + 127) / 128, 128, 0, st>>>(len, B, by);
  return cudaGetLastError();
}

}  // namespace loopk

namespace loopk {
int status_read() {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return -1;
  return v;
}
void status_clear() {
  const int z = 0;
  cudaMemcpyToSymbol(g_status, &z, sizeof(int));
}
}  // namespace loopk

namespace loopk {
// A wait that nothing will end: one thread waits on a fresh mbarrier whose
// phase never completes, with a short limit, so the timeout path runs.
__global__ void selftest_timeout_kernel(uint64_t limit_ns, int* status, int* result) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) *result = mbar_wait(&bar, 0, status, STATUS_SELFTEST, limit_ns) ? 1 : 0;
}
cudaError_t launch_selftest_timeout(uint64_t limit_ns, int* result, cudaStream_t st) {
  selftest_timeout_kernel<<<1, 32, 0, st>>>(limit_ns, status_ptr(), result);
  return cudaGetLastError();
}
}  // namespace loopk
