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
  const int64_t r = blockIdx.x;
  const float* xr = x + (r * step + off) * H;
  float ss = 0.f;
  for (int i = threadIdx.x; i < H; i += blockDim.x) ss += xr[i] * xr[i];
  ss = block_sum(ss, red);
  const float inv = rsqrtf(ss / H + eps);
  for (int i = threadIdx.x; i < H; i += blockDim.x) y[r * H + i] = from_f<T>(xr[i] * inv * gain[i]);
}
cudaError_t launch_rmsnorm(const float* x, int64_t rows, int H, int64_t step, int64_t off, const float* gain,
                           float eps, void* y, bool bf, cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
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
// Fused mHC prologue for n = 2 streams.  One CTA handles TOK tokens so the
// projection Phi [8][2H] is read once per TOK tokens.  Pass 1 accumulates the
// squared norm and the 8 projections of (s * gamma); one thread per token
// then forms the coefficients (Sinkhorn included); pass 2 reads
// x = H_pre[0] s_0 + H_pre[1] s_1 and writes RMSNorm(x) * gain.
// ---------------------------------------------------------------------------
constexpr int MHC_TOK = 8;
constexpr int MHC_THREADS = 256;

template <typename T>
__global__ void __launch_bounds__(MHC_THREADS) mhc_prologue_kernel(const float* __restrict__ s, int64_t Ttot, int H,
                                                                   const float* __restrict__ gamma,
                                                                   const float* __restrict__ phi,
                                                                   const float* __restrict__ gain, int iters,
                                                                   float eps, float* __restrict__ coef,
                                                                   T* __restrict__ xh) {
  __shared__ float red[MHC_THREADS / 32][MHC_TOK][9];
  __shared__ float cf[MHC_TOK][8];
  __shared__ float nrm[MHC_TOK];
  const int64_t t0 = (int64_t)blockIdx.x * MHC_TOK;
  const int ntok = (int)(Ttot - t0 < MHC_TOK ? Ttot - t0 : MHC_TOK);
  const int D = 2 * H;
  float acc[MHC_TOK][9];
#pragma unroll
  for (int j = 0; j < MHC_TOK; ++j)
#pragma unroll
    for (int c = 0; c < 9; ++c) acc[j][c] = 0.f;

  for (int i = threadIdx.x; i < D; i += MHC_THREADS) {
    const int stream = i >= H ? 1 : 0;
    const int col = i - stream * H;
    float ph[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) ph[c] = phi[(int64_t)c * D + i];
    const float g = gamma[i];
#pragma unroll
    for (int j = 0; j < MHC_TOK; ++j) {
      if (j < ntok) {
        const float v = s[((int64_t)stream * Ttot + t0 + j) * H + col];
        acc[j][8] += v * v;
        const float w = v * g;
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[j][c] += w * ph[c];
      }
    }
  }
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
  for (int j = 0; j < MHC_TOK; ++j)
#pragma unroll
    for (int c = 0; c < 9; ++c) {
      const float r = warp_sum(acc[j][c]);
      if (lane == 0) red[wid][j][c] = r;
    }
  __syncthreads();
  if (threadIdx.x < ntok) {
    const int j = threadIdx.x;
    float tot[9];
    for (int c = 0; c < 9; ++c) {
      float a = 0.f;
      for (int w = 0; w < MHC_THREADS / 32; ++w) a += red[w][j][c];
      tot[c] = a;
    }
    const float rinv = rsqrtf(tot[8] / D + eps);
    float l[8];
    for (int c = 0; c < 8; ++c) l[c] = tot[c] * rinv;
    float P[4];
    sinkhorn_fixed<2>(l + 4, P, iters);
    cf[j][0] = sigmoidf_(l[0]);
    cf[j][1] = sigmoidf_(l[1]);
    cf[j][2] = 2.f * sigmoidf_(l[2]);
    cf[j][3] = 2.f * sigmoidf_(l[3]);
    for (int c = 0; c < 4; ++c) cf[j][4 + c] = P[c];
    for (int c = 0; c < 8; ++c) coef[(t0 + j) * 8 + c] = cf[j][c];
  }
  __syncthreads();
  // pass 2: x = pre0 s0 + pre1 s1, then RMSNorm(x) * gain
  float ss[MHC_TOK];
#pragma unroll
  for (int j = 0; j < MHC_TOK; ++j) ss[j] = 0.f;
  for (int i = threadIdx.x; i < H; i += MHC_THREADS) {
#pragma unroll
    for (int j = 0; j < MHC_TOK; ++j) {
      if (j < ntok) {
        const float x = cf[j][0] * s[(t0 + j) * H + i] + cf[j][1] * s[(Ttot + t0 + j) * H + i];
        ss[j] += x * x;
      }
    }
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < MHC_TOK; ++j) {
    const float r = warp_sum(ss[j]);
    if (lane == 0) red[wid][j][0] = r;
  }
  __syncthreads();
  if (threadIdx.x < ntok) {
    float a = 0.f;
    for (int w = 0; w < MHC_THREADS / 32; ++w) a += red[w][threadIdx.x][0];
    nrm[threadIdx.x] = rsqrtf(a / H + eps);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < H; i += MHC_THREADS) {
    const float gi = gain[i];
#pragma unroll
    for (int j = 0; j < MHC_TOK; ++j) {
      if (j < ntok) {
        const float x = cf[j][0] * s[(t0 + j) * H + i] + cf[j][1] * s[(Ttot + t0 + j) * H + i];
        xh[(t0 + j) * H + i] = from_f<T>(x * nrm[j] * gi);
      }
    }
  }
}

cudaError_t launch_mhc_prologue(const float* s, int64_t T, int H, const float* gamma, const float* phi,
                                const float* gain, int iters, float eps, float* coef, void* xh, bool bf,
                                cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  const unsigned g = (unsigned)((T + MHC_TOK - 1) / MHC_TOK);
  if (bf)
    mhc_prologue_kernel<bf16><<<g, MHC_THREADS, 0, st>>>(s, T, H, gamma, phi, gain, iters, eps, coef, (bf16*)xh);
  else
    mhc_prologue_kernel<float><<<g, MHC_THREADS, 0, st>>>(s, T, H, gamma, phi, gain, iters, eps, coef, (float*)xh);
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
__global__ void cache_to_f32_kernel(const T* src, int B, int nkv, int64_t ctx, int len, int hd, float* dst) {
  const int64_t n = (int64_t)B * nkv * len * hd;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t e = i % hd, p = (i / hd) % len, bh = i / ((int64_t)hd * len);
    dst[i] = to_f(src[(bh * ctx + p) * hd + e]);
  }
}
cudaError_t launch_cache_to_f32(const void* src, bool bf, int B, int nkv, int64_t ctx, int len, int hd, float* dst,
                                cudaStream_t st) {
  const int64_t n = (int64_t)B * nkv * len * hd;
  if (n == 0) return cudaSuccess;
  const unsigned g = (unsigned)std::min<int64_t>((n + 255) / 256, 148 * 16);
  if (bf) cache_to_f32_kernel<bf16><<<g, 256, 0, st>>>((const bf16*)src, B, nkv, ctx, len, hd, dst);
  else cache_to_f32_kernel<float><<<g, 256, 0, st>>>((const float*)src, B, nkv, ctx, len, hd, dst);
  return cudaGetLastError();
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

__global__ void advance_kernel(int32_t* len, int B) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) len[b] += 1;
}
__global__ void set_len_kernel(int32_t* len, int B, int S) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) len[b] = S;
}
cudaError_t launch_set_len(int32_t* len, int B, int S, cudaStream_t st) {
  set_len_kernel<<<(B + 127) / 128, 128, 0, st>>>(len, B, S);
  return cudaGetLastError();
}
cudaError_t launch_advance(int32_t* len, int B, cudaStream_t st) {
  advance_kernel<<<(B + 127) / 128, 128, 0, st>>>(len, B);
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
