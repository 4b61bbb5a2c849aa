// Chunked gated linear attention (prefill) on the tensor cores.
//
// The layer (one of the 3 linear-attention layers of every 4-layer group,
// "How Does SenseNova-Loop Get More Depth Without More Parameters?", section
// "How does the hybrid attention pattern work?") keeps a fixed-size state per
// head: S_t = g_t S_{t-1} + k_t v_t^T, o_t = q_t S_t.  Over a chunk of C = 64
// tokens with b_t the running sum of log g inside the chunk this is exactly
//   O   = ((Q K^T) * D) V + diag(exp b) Q S_prev,   D_ts = exp(b_t - b_s) [s <= t]
//   S'  = exp(b_last) S_prev + K^T (diag(exp(b_last - b)) V).
//
// One CTA (8 warps) owns (sequence, head, 64-column slice of the value
// dimension) and walks the chunks in order; its 128 x 64 fp32 state slice
// stays in MMA accumulator registers for the whole sequence (16 rows per
// warp).  Outputs: warp w computes rows 16 (w % 4) .. + 15 and value columns
// 32 (w / 4) .. + 31 of the chunk.  Q, K and the V slice of each
// chunk are staged by TMA (128-byte swizzle, double-buffered).  Products run
// on bf16 mma.sync m16n8k16 with fp32 accumulation.  The three operands that
// are not model activations - the state, the decayed scores (Q K^T) * D and
// the decayed values - enter their products as bf16 hi + lo pairs (~16
// significant bits), so the chunked form loses no accuracy against the
// token-by-token recurrence.

#include <cuda.h>

#include "model.h"

namespace loopk {

namespace {

constexpr int C = 64, DK = 128, DV = 64, WARPS = 8, THREADS = WARPS * 32;
constexpr int QK_BYTES = C * DK * 2;            // Q or K tile: two boxes [64][64]
constexpr int V_BYTES = C * DV * 2;             // V slice: one box [64][64]
constexpr int STAGE_BYTES = 2 * QK_BYTES + V_BYTES;
constexpr int SS_BYTES = DK * DV * 2;           // bf16 copy of the state slice
constexpr int SMEM = 2 * STAGE_BYTES + 2 * SS_BYTES + 2 * V_BYTES + 2 * C * 4 + 64 + 1024;

__global__ void __launch_bounds__(THREADS, 1)
    gla_chunk_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                     const __grid_constant__ CUtensorMap tv, const float* __restrict__ gl, float* __restrict__ state,
                     bf16* __restrict__ out, int S, int nh, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage0 = smem;
  uint8_t* shi = smem + 2 * STAGE_BYTES;
  uint8_t* slo = shi + SS_BYTES;
  uint8_t* vhat = slo + SS_BYTES;      // hi part of diag(exp(b_last - b)) V
  uint8_t* vhat_lo = vhat + V_BYTES;    // and its remainder
  float* lg = reinterpret_cast<float*>(vhat_lo + V_BYTES);
  float* bv = lg + C;
  uint64_t* full = reinterpret_cast<uint64_t*>(bv + C);

  const int slice = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3, mi = lane >> 3, ri = lane & 7;
  const int nch = (S + C - 1) / C;
  const int row0 = (b * nh + h) * S;  // first row of this head in the [B nh S][128] views
  const float* glh = gl + (int64_t)(b * nh + h) * S;
  float* st = state + (int64_t)(b * nh + h) * DK * 128 + slice * DV;

  if (tid == 0) {
    mbar_init(&full[0], 1);
    mbar_init(&full[1], 1);
    fence_mbar_init();
  }
  __syncthreads();
  auto issue = [&](int c) {
    uint8_t* sg = stage0 + (c & 1) * STAGE_BYTES;
    uint64_t* bar = &full[c & 1];
    const int row = row0 + c * C;
    mbar_expect_tx(bar, STAGE_BYTES);
    tma_load_2d(sg, &tq, bar, 0, row);
    tma_load_2d(sg + QK_BYTES / 2, &tq, bar, 64, row);
    tma_load_2d(sg + QK_BYTES, &tk, bar, 0, row);
    tma_load_2d(sg + QK_BYTES + QK_BYTES / 2, &tk, bar, 64, row);
    tma_load_2d(sg + 2 * QK_BYTES, &tv, bar, slice * DV, row);
  };
  if (tid == 0) {
    prefetch_tmap(&tq);
    prefetch_tmap(&tk);
    prefetch_tmap(&tv);
    issue(0);
    if (nch > 1) issue(1);
  }

  // state slice: warp w owns rows 16w .. 16w + 15 (one m16 tile) x 64 columns
  float acc[8][4];
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
    const int r = warp * 16 + g, c = nt * 8 + 2 * t;
    acc[nt][0] = st[(int64_t)r * 128 + c];
    acc[nt][1] = st[(int64_t)r * 128 + c + 1];
    acc[nt][2] = st[(int64_t)(r + 8) * 128 + c];
    acc[nt][3] = st[(int64_t)(r + 8) * 128 + c + 1];
  }

  const uint32_t shi_u = smem_u32(shi), slo_u = smem_u32(slo), vhat_u = smem_u32(vhat),
                 vlo_u = smem_u32(vhat_lo);
  const int rg = warp & 3, ch = warp >> 2;  // output phase: rows 16 rg .., value columns 32 ch ..
  for (int c = 0; c < nch; ++c) {
    const int c0 = c * C;
    const int valid = min(C, S - c0);
    // gates of this chunk (0 past the end) and their running sums b
    if (tid < C) lg[tid] = tid < valid ? glh[c0 + tid] : 0.f;
    const bool ok = mbar_wait(&full[c & 1], (c >> 1) & 1, status, STATUS_WAIT_OTHER);
    if (__syncthreads_or(!ok)) break;
    if (warp == 0) {
      const float x0 = lg[2 * lane], x1 = lg[2 * lane + 1];
      const float pair = x0 + x1;
      float inc = pair;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
      }
      const float ex = inc - pair;
      bv[2 * lane] = ex + x0;
      bv[2 * lane + 1] = inc;
    }
    // current state as bf16 hi + lo, row-major [dk][64] with the 128-byte swizzle
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int r = warp * 16 + g + 8 * hf;
        const float x0 = acc[nt][2 * hf], x1 = acc[nt][2 * hf + 1];
        const __nv_bfloat162 hi = __floats2bfloat162_rn(x0, x1);
        const float2 hf2 = __bfloat1622float2(hi);
        const __nv_bfloat162 lo = __floats2bfloat162_rn(x0 - hf2.x, x1 - hf2.y);
        const uint32_t off = (uint32_t)(r * 128 + ((nt ^ (r & 7)) << 4) + 4 * t);
        *reinterpret_cast<__nv_bfloat162*>(shi + off) = hi;
        *reinterpret_cast<__nv_bfloat162*>(slo + off) = lo;
      }
    __syncthreads();
    const float b_last = bv[C - 1];
    uint8_t* sg = stage0 + (c & 1) * STAGE_BYTES;
    const uint32_t q_u = smem_u32(sg), k_u = q_u + QK_BYTES, v_u = q_u + 2 * QK_BYTES;
    // V-hat = diag(exp(b_last - b)) V as hi + lo, zero past the end of the sequence
    for (int ci = tid; ci < C * 8; ci += THREADS) {
      const int r = ci >> 3, chk = ci & 7;
      const uint32_t off = (uint32_t)(r * 128 + ((chk ^ (r & 7)) << 4));
      const float f = r < valid ? __expf(b_last - bv[r]) : 0.f;
      uint4 u = *reinterpret_cast<const uint4*>(sg + 2 * QK_BYTES + off);
      uint4 w;
      __nv_bfloat162* p = reinterpret_cast<__nv_bfloat162*>(&u);
      __nv_bfloat162* pl = reinterpret_cast<__nv_bfloat162*>(&w);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 x = __bfloat1622float2(p[e]);
        const float y0 = x.x * f, y1 = x.y * f;
        p[e] = __floats2bfloat162_rn(y0, y1);
        const float2 hi = __bfloat1622float2(p[e]);
        pl[e] = __floats2bfloat162_rn(y0 - hi.x, y1 - hi.y);
      }
      *reinterpret_cast<uint4*>(vhat + off) = u;
      *reinterpret_cast<uint4*>(vhat_lo + off) = w;
    }
    __syncthreads();

    // ---- outputs: rows 16 rg .. 16 rg + 15, value columns 32 ch .. 32 ch + 31 ----
    {
      uint32_t qf[8][4];
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        ldsm_x4(q_u + sw(rg * 16 + (mi & 1) * 8 + ri, kk * 2 + (mi >> 1), C), qf[kk][0], qf[kk][1], qf[kk][2],
                qf[kk][3]);
      float a[8][4];
#pragma unroll
      for (int i = 0; i < 8; ++i) a[i][0] = a[i][1] = a[i][2] = a[i][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
#pragma unroll
        for (int nt = 0; nt < 8; nt += 2) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(k_u + sw(nt * 8 + (mi >> 1) * 8 + ri, kk * 2 + (mi & 1), C), b0, b1, b2, b3);
          mma_bf16(a[nt], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b0, b1);
          mma_bf16(a[nt + 1], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b2, b3);
        }
      const int tq0 = rg * 16 + g, tq1 = tq0 + 8;
      const float bt0 = bv[tq0], bt1 = bv[tq1];
      uint32_t pa[8][2], pl[8][2];  // (Q K^T) * D as bf16 hi + lo
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        float d[4];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int sk = nt * 8 + 2 * t + e;
          const float bs = bv[sk];
          d[e] = (sk <= tq0 && sk < valid) ? __expf(bt0 - bs) : 0.f;
          d[2 + e] = (sk <= tq1 && sk < valid) ? __expf(bt1 - bs) : 0.f;
        }
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const float x0 = a[nt][2 * hf] * d[2 * hf], x1 = a[nt][2 * hf + 1] * d[2 * hf + 1];
          const __nv_bfloat162 hi = __floats2bfloat162_rn(x0, x1);
          const float2 h2 = __bfloat1622float2(hi);
          pa[nt][hf] = *reinterpret_cast<const uint32_t*>(&hi);
          pl[nt][hf] = pack_bf16x2(x0 - h2.x, x1 - h2.y);
        }
      }
      // inter-chunk first: o = exp(b_t) Q S_prev (S as hi + lo), then the
      // intra-chunk (A * D) V accumulates onto it
      float o[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
#pragma unroll
        for (int nt = 0; nt < 4; nt += 2) {
          uint32_t b0, b1, b2, b3;
          const uint32_t off = sw(kk * 16 + (mi & 1) * 8 + ri, ch * 4 + nt + (mi >> 1), DK);
          ldsm_x4_t(shi_u + off, b0, b1, b2, b3);
          mma_bf16(o[nt], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b0, b1);
          mma_bf16(o[nt + 1], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b2, b3);
          ldsm_x4_t(slo_u + off, b0, b1, b2, b3);
          mma_bf16(o[nt], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b0, b1);
          mma_bf16(o[nt + 1], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b2, b3);
        }
      const float e0 = __expf(bt0), e1 = __expf(bt1);
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        o[nt][0] *= e0;
        o[nt][1] *= e0;
        o[nt][2] *= e1;
        o[nt][3] *= e1;
      }
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
#pragma unroll
        for (int nt = 0; nt < 4; nt += 2) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(v_u + sw(kk * 16 + (mi & 1) * 8 + ri, ch * 4 + nt + (mi >> 1), C), b0, b1, b2, b3);
          mma_bf16(o[nt], pa[2 * kk][0], pa[2 * kk][1], pa[2 * kk + 1][0], pa[2 * kk + 1][1], b0, b1);
          mma_bf16(o[nt + 1], pa[2 * kk][0], pa[2 * kk][1], pa[2 * kk + 1][0], pa[2 * kk + 1][1], b2, b3);
          mma_bf16(o[nt], pl[2 * kk][0], pl[2 * kk][1], pl[2 * kk + 1][0], pl[2 * kk + 1][1], b0, b1);
          mma_bf16(o[nt + 1], pl[2 * kk][0], pl[2 * kk][1], pl[2 * kk + 1][0], pl[2 * kk + 1][1], b2, b3);
        }
      const int64_t ld = (int64_t)nh * 128;
      bf16* r0p = out + ((int64_t)b * S + c0 + tq0) * ld + h * 128 + slice * DV + ch * 32;
      bf16* r1p = out + ((int64_t)b * S + c0 + tq1) * ld + h * 128 + slice * DV + ch * 32;
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        const int col = nt * 8 + 2 * t;
        if (tq0 < valid) *reinterpret_cast<uint32_t*>(r0p + col) = pack_bf16x2(o[nt][0], o[nt][1]);
        if (tq1 < valid) *reinterpret_cast<uint32_t*>(r1p + col) = pack_bf16x2(o[nt][2], o[nt][3]);
      }
    }
    // ---- state update: S = exp(b_last) S + K^T V-hat (rows 16 warp ..) ----
    {
      const float dl = __expf(b_last);
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[nt][e] *= dl;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        uint32_t af[4];
        ldsm_x4_t(k_u + sw(kk * 16 + (mi >> 1) * 8 + ri, 2 * warp + (mi & 1), C), af[0], af[1], af[2], af[3]);
#pragma unroll
        for (int nt = 0; nt < 8; nt += 2) {
          uint32_t b0, b1, b2, b3;
          const uint32_t off = sw(kk * 16 + (mi & 1) * 8 + ri, nt + (mi >> 1), C);
          ldsm_x4_t(vhat_u + off, b0, b1, b2, b3);
          mma_bf16(acc[nt], af[0], af[1], af[2], af[3], b0, b1);
          mma_bf16(acc[nt + 1], af[0], af[1], af[2], af[3], b2, b3);
          ldsm_x4_t(vlo_u + off, b0, b1, b2, b3);
          mma_bf16(acc[nt], af[0], af[1], af[2], af[3], b0, b1);
          mma_bf16(acc[nt + 1], af[0], af[1], af[2], af[3], b2, b3);
        }
      }
    }
    __syncthreads();  // every read of this stage, the state copy and V-hat is done
    if (tid == 0 && c + 2 < nch) issue(c + 2);
  }
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
    const int r = warp * 16 + g, c = nt * 8 + 2 * t;
    st[(int64_t)r * 128 + c] = acc[nt][0];
    st[(int64_t)r * 128 + c + 1] = acc[nt][1];
    st[(int64_t)(r + 8) * 128 + c] = acc[nt][2];
    st[(int64_t)(r + 8) * 128 + c + 1] = acc[nt][3];
  }
}

// ---------------------------------------------------------------------------
// One decode step of gated linear attention (d = 128): S = g S + k v^T,
// o = q S.  CTA (32-column slice of S, head, sequence), 256 threads: thread
// (row group rg = tid / 32, column c = tid % 32) updates rows 16 rg .. 16 rg + 15
// of its column with 16 independent loads, and the 8 row groups' parts of
// q S are summed in shared memory.  The state is read and written once.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
    gla_decode_kernel(const bf16* __restrict__ q, const bf16* __restrict__ k, const bf16* __restrict__ v,
                      const float* __restrict__ gl, float* __restrict__ state, bf16* __restrict__ out, int nh) {
  __shared__ float qs[DK], ks[DK], red[8][32];
  const int slice = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, rg = tid >> 5, c = tid & 31;
  const int64_t bh = (int64_t)b * nh + h;
  if (tid < DK) {
    qs[tid] = __bfloat162float(q[bh * DK + tid]);
    ks[tid] = __bfloat162float(k[bh * DK + tid]);
  }
  __syncthreads();
  const int col = slice * 32 + c;
  const float g = __expf(gl[bh]);
  const float vc = __bfloat162float(v[bh * DK + col]);
  float* st = state + bh * DK * 128 + col;
  float sv[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) sv[i] = st[(int64_t)(rg * 16 + i) * 128];
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int r = rg * 16 + i;
    sv[i] = g * sv[i] + ks[r] * vc;
    acc += qs[r] * sv[i];
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) st[(int64_t)(rg * 16 + i) * 128] = sv[i];
  red[rg][c] = acc;
  __syncthreads();
  if (rg == 0) {
    float o = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) o += red[j][c];
    out[(int64_t)b * nh * 128 + h * 128 + col] = __float2bfloat16_rn(o);
  }
}

}  // namespace

bool gla_chunk_supported(int d) { return d == DK; }

// q, k, v [B][nh][1][128] bf16; gl [B][nh]; state [B][nh][128][128] fp32
// (updated in place); o [B][nh * 128] bf16.
cudaError_t launch_gla_decode(const void* q, const void* k, const void* v, const float* gl, float* state, void* o,
                              int B, int nh, cudaStream_t st) {
  if (B == 0) return cudaSuccess;
  dim3 grid(128 / 32, (unsigned)nh, (unsigned)B);
  gla_decode_kernel<<<grid, 256, 0, st>>>((const bf16*)q, (const bf16*)k, (const bf16*)v, gl, state, (bf16*)o, nh);
  return cudaGetLastError();
}

// q, k, v [B][nh][S][128] bf16; gl [B][nh][S] log-gates; state [B][nh][128][128]
// fp32 (read, then replaced by the final state); o [B*S][nh*128] bf16.
cudaError_t launch_gla_chunked(const void* q, const void* k, const void* v, const float* gl, float* state, void* o,
                               int B, int S, int nh, cudaStream_t st) {
  if (B == 0 || S == 0) return cudaSuccess;
  CUtensorMap mq, mk, mv;
  const int64_t rows = (int64_t)B * nh * S;
  if (!map_rows128(&mq, q, rows, C) || !map_rows128(&mk, k, rows, C) || !map_rows128(&mv, v, rows, C))
    return cudaErrorInvalidValue;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(gla_chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  dim3 grid(128 / DV, (unsigned)nh, (unsigned)B);
  gla_chunk_kernel<<<grid, THREADS, SMEM, st>>>(mq, mk, mv, gl, state, (bf16*)o, S, nh, status_ptr());
  return cudaGetLastError();
}

}  // namespace loopk
