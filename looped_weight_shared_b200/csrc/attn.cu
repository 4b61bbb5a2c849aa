// Causal GQA flash attention for the prefill of the full-attention layers:
// O = softmax(Q K^T / sqrt(128) + causal mask) V with kv head = q head / 4
// ("How Does SenseNova-Loop Get More Depth Without More Parameters?", section
// "How does the hybrid attention pattern work?": periodic full-attention layers
// with grouped KV heads).
//
// One CTA computes 128 queries of one head.  A producer warp stages Q once and
// K/V tiles of 64 keys through a 3-deep ring with TMA (128-byte swizzle); 8
// compute warps (16 query rows each) run S = Q K^T and O += P V on the tensor
// cores (bf16 mma.sync m16n8k16, fp32 accumulation) with the online softmax in
// registers.  Key tiles past the causal frontier are never loaded.

#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "model.h"

namespace loopk {

namespace {

constexpr int BQ = 128, BKV = 64, D = 128, NS = 3;
constexpr int WARPS = 8;
constexpr int THREADS = (WARPS + 1) * 32;
constexpr int Q_BYTES = BQ * D * 2;
constexpr int KV_BYTES = BKV * D * 2;  // one K or V tile
constexpr int SMEM = Q_BYTES + NS * 2 * KV_BYTES + 1024 + 128;

__global__ void __launch_bounds__(THREADS, 1)
    flash_fwd_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                     const __grid_constant__ CUtensorMap tv, bf16* __restrict__ out, int S, int nq, int nkv,
                     int64_t ctx, float scale_log2, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sq = smem;
  uint8_t* skv = smem + Q_BYTES;  // stage s: K at skv + 2 s KV_BYTES, V after it
  uint64_t* qfull = reinterpret_cast<uint64_t*>(smem + Q_BYTES + NS * 2 * KV_BYTES);
  uint64_t* kvfull = qfull + 1;
  uint64_t* kvempty = kvfull + NS;

  const int nqb = (S + BQ - 1) / BQ;
  const int qb = nqb - 1 - (int)blockIdx.x;  // longest rows first
  const int h = blockIdx.y, b = blockIdx.z;
  const int kvh = h / (nq / nkv);
  const int q0 = qb * BQ;
  const int last_key = min(q0 + BQ, S) - 1;
  const int ntiles = last_key / BKV + 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(qfull, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&kvfull[s], 1);
      mbar_init(&kvempty[s], WARPS);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == WARPS) {
    if (lane == 0) {
      prefetch_tmap(&tq);
      prefetch_tmap(&tk);
      prefetch_tmap(&tv);
      const int qrow = (b * nq + h) * S + q0;
      mbar_expect_tx(qfull, Q_BYTES);
      tma_load_2d(sq, &tq, qfull, 0, qrow);
      tma_load_2d(sq + Q_BYTES / 2, &tq, qfull, 64, qrow);
      const int64_t krow0 = ((int64_t)b * nkv + kvh) * ctx;
      for (int j = 0; j < ntiles; ++j) {
        const int s = j % NS;
        const uint32_t ph = (j / NS) & 1;
        if (!mbar_wait(&kvempty[s], ph ^ 1, status, STATUS_WAIT_PRODUCER)) break;
        uint8_t* kt = skv + 2 * s * KV_BYTES;
        uint8_t* vt = kt + KV_BYTES;
        const int row = (int)(krow0 + (int64_t)j * BKV);
        mbar_expect_tx(&kvfull[s], 2 * KV_BYTES);
        tma_load_2d(kt, &tk, &kvfull[s], 0, row);
        tma_load_2d(kt + KV_BYTES / 2, &tk, &kvfull[s], 64, row);
        tma_load_2d(vt, &tv, &kvfull[s], 0, row);
        tma_load_2d(vt + KV_BYTES / 2, &tv, &kvfull[s], 64, row);
      }
    }
    return;
  }

  // ---- compute warps ----
  const int g = lane >> 2, t = lane & 3;
  const int mi = lane >> 3, ri = lane & 7;
  const uint32_t sq_u = smem_u32(sq);
  const uint32_t skv_u = smem_u32(skv);
  bool ok = __all_sync(0xffffffffu, mbar_wait(qfull, 0, status, STATUS_WAIT_EPILOGUE));
  uint32_t qf[8][4];
  if (ok) {
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const int row = warp * 16 + (mi & 1) * 8 + ri;
      ldsm_x4(sq_u + sw(row, kk * 2 + (mi >> 1), BQ), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
    }
  }
  float o[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  const int qp0 = q0 + warp * 16 + g, qp1 = qp0 + 8;

  for (int j = 0; j < ntiles && ok; ++j) {
    const int s = j % NS;
    const uint32_t ph = (j / NS) & 1;
    ok = __all_sync(0xffffffffu, mbar_wait(&kvfull[s], ph, status, STATUS_WAIT_EPILOGUE));
    if (!ok) break;
    const uint32_t kt = skv_u + 2 * s * KV_BYTES;
    const uint32_t vt = kt + KV_BYTES;
    // S = Q K^T for 16 rows x 64 keys
    float sc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) sc[i][0] = sc[i][1] = sc[i][2] = sc[i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
      for (int nt = 0; nt < 8; nt += 2) {
        uint32_t b0, b1, b2, b3;
        const int key = nt * 8 + (mi >> 1) * 8 + ri;
        ldsm_x4(kt + sw(key, kk * 2 + (mi & 1), BKV), b0, b1, b2, b3);
        mma_bf16(sc[nt], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b0, b1);
        mma_bf16(sc[nt + 1], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b2, b3);
      }
    }
    // scale, causal mask, online softmax (rows g and g + 8 of this warp)
    const int kbase = j * BKV;
    const bool need_mask = kbase + BKV - 1 > q0 + warp * 16;
    float mx0 = m0, mx1 = m1;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int kp = kbase + nt * 8 + 2 * t + e;
        float v0 = sc[nt][e] * scale_log2, v1 = sc[nt][2 + e] * scale_log2;
        if (need_mask) {
          if (kp > qp0) v0 = -INFINITY;
          if (kp > qp1) v1 = -INFINITY;
        }
        sc[nt][e] = v0;
        sc[nt][2 + e] = v1;
        mx0 = fmaxf(mx0, v0);
        mx1 = fmaxf(mx1, v1);
      }
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float c0 = ex2(m0 - mx0), c1 = ex2(m1 - mx1);
    m0 = mx0;
    m1 = mx1;
    float rs0 = 0.f, rs1 = 0.f;
    uint32_t pa[8][2];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const float p0 = ex2(sc[nt][0] - mx0), p1 = ex2(sc[nt][1] - mx0);
      const float p2 = ex2(sc[nt][2] - mx1), p3 = ex2(sc[nt][3] - mx1);
      rs0 += p0 + p1;
      rs1 += p2 + p3;
      pa[nt][0] = pack_bf16x2(p0, p1);
      pa[nt][1] = pack_bf16x2(p2, p3);
    }
    l0 = l0 * c0 + rs0;
    l1 = l1 * c1 + rs1;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      o[i][0] *= c0;
      o[i][1] *= c0;
      o[i][2] *= c1;
      o[i][3] *= c1;
    }
    // O += P V  (P as the A operand straight from the S registers)
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const uint32_t a0 = pa[2 * kk][0], a1 = pa[2 * kk][1], a2 = pa[2 * kk + 1][0], a3 = pa[2 * kk + 1][1];
#pragma unroll
      for (int nt = 0; nt < 16; nt += 2) {
        uint32_t b0, b1, b2, b3;
        const int key = kk * 16 + (mi & 1) * 8 + ri;
        ldsm_x4_t(vt + sw(key, nt + (mi >> 1), BKV), b0, b1, b2, b3);
        mma_bf16(o[nt], a0, a1, a2, a3, b0, b1);
        mma_bf16(o[nt + 1], a0, a1, a2, a3, b2, b3);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&kvempty[s]);
  }
  // normalise and store O as [token][head * 128 + dim]
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const float i0 = l0 > 0.f ? 1.f / l0 : 0.f, i1 = l1 > 0.f ? 1.f / l1 : 0.f;
  const int64_t ld = (int64_t)nq * D;
  bf16* r0 = out + ((int64_t)b * S + qp0) * ld + (int64_t)h * D;
  bf16* r1 = out + ((int64_t)b * S + qp1) * ld + (int64_t)h * D;
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) {
    const int col = nt * 8 + 2 * t;
    if (qp0 < S) *reinterpret_cast<uint32_t*>(r0 + col) = pack_bf16x2(o[nt][0] * i0, o[nt][1] * i0);
    if (qp1 < S) *reinterpret_cast<uint32_t*>(r1 + col) = pack_bf16x2(o[nt][2] * i1, o[nt][3] * i1);
  }
}


// ---------------------------------------------------------------------------
// Decode attention (one new query per sequence): split the context into
// chunks of 128 keys.  CTA (chunk, kv head, sequence) bulk-copies the chunk's
// K and V rows (contiguous in the cache) into shared memory and scores the 4
// query heads of the group: each warp takes 32 keys, lanes split the 128
// dims so every K row is read once and coalesced.  It writes the chunk's
// unnormalised o, its max m (log2 domain) and sum l; a combine kernel merges
// the chunks.  K/V are read from HBM exactly once per step.
// ---------------------------------------------------------------------------
constexpr int DEC_KEYS = 128, DEC_G = 4, DEC_THREADS = 128;
constexpr int DEC_SMEM = 2 * DEC_KEYS * D * 2 + DEC_G * D * 4 + DEC_G * DEC_KEYS * 4 + 64 + 128;

__global__ void __launch_bounds__(DEC_THREADS)
    attn_decode_partial_kernel(const bf16* __restrict__ q, const bf16* __restrict__ K, const bf16* __restrict__ V,
                               const int32_t* __restrict__ start, int nq, int nkv, int64_t ctx, int nchunks,
                               float scale_log2, float* __restrict__ po, float* __restrict__ pml, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  bf16* ks = reinterpret_cast<bf16*>(smem);
  bf16* vs = ks + DEC_KEYS * D;
  float* qs = reinterpret_cast<float*>(vs + DEC_KEYS * D);  // [G][128]
  float* ps = qs + DEC_G * D;                                // [G][keys]
  uint64_t* bar = reinterpret_cast<uint64_t*>(ps + DEC_G * DEC_KEYS);
  const int chunk = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = nq / nkv;
  const int L = start[b] + 1;  // keys 0 .. start[b] (the new token's K/V are already in the cache)
  const int k0 = chunk * DEC_KEYS;
  const int64_t out_base = ((int64_t)b * nq + kvh * G) * nchunks + chunk;
  if (k0 >= L) {  // past this sequence's end: an empty partial
    if (tid < G) {
      pml[(out_base + (int64_t)tid * nchunks) * 2] = -INFINITY;
      pml[(out_base + (int64_t)tid * nchunks) * 2 + 1] = 0.f;
    }
    return;
  }
  const int nk = min(DEC_KEYS, L - k0);
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (tid == 0) {
    const int64_t row = ((int64_t)b * nkv + kvh) * ctx + k0;
    mbar_expect_tx(bar, 2u * nk * D * 2);
    bulk_load(ks, K + row * D, nk * D * 2, bar);
    bulk_load(vs, V + row * D, nk * D * 2, bar);
  }
  for (int i = tid; i < G * D; i += DEC_THREADS)
    qs[i] = __bfloat162float(q[((int64_t)b * nq + kvh * G + i / D) * D + i % D]) * scale_log2;
  const bool ok = mbar_wait(bar, 0, status, STATUS_WAIT_OTHER);
  if (__syncthreads_or(!ok)) return;
  // scores: warp w handles keys w, w + 4, ...; lane owns dims 4 lane .. 4 lane + 3
  float qv[DEC_G][4];
#pragma unroll
  for (int h = 0; h < DEC_G; ++h)
#pragma unroll
    for (int e = 0; e < 4; ++e) qv[h][e] = qs[h * D + 4 * lane + e];
  for (int j = warp; j < nk; j += DEC_THREADS / 32) {
    const uint2 kr = *reinterpret_cast<const uint2*>(ks + j * D + 4 * lane);
    const float2 k01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kr.x));
    const float2 k23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kr.y));
#pragma unroll
    for (int h = 0; h < DEC_G; ++h) {
      float d = qv[h][0] * k01.x + qv[h][1] * k01.y + qv[h][2] * k23.x + qv[h][3] * k23.y;
      d = warp_sum(d);
      if (lane == 0) ps[h * DEC_KEYS + j] = d;
    }
  }
  __syncthreads();
  // per head: max and exp2 over the chunk (warp h handles head h)
  if (warp < DEC_G) {
    const int h = warp;
    float m = -INFINITY;
    for (int j = lane; j < nk; j += 32) m = fmaxf(m, ps[h * DEC_KEYS + j]);
    m = warp_max(m);
    float l = 0.f;
    for (int j = lane; j < nk; j += 32) {
      const float p = ex2(ps[h * DEC_KEYS + j] - m);
      ps[h * DEC_KEYS + j] = p;
      l += p;
    }
    l = warp_sum(l);
    if (lane == 0) {
      pml[(out_base + (int64_t)h * nchunks) * 2] = m;
      pml[(out_base + (int64_t)h * nchunks) * 2 + 1] = l;
    }
  }
  __syncthreads();
  // o[h][d] = sum_j p[h][j] V[j][d]: thread t owns dim t
  float acc[DEC_G] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
  for (int j = 0; j < nk; ++j) {
    const float v = __bfloat162float(vs[j * D + tid]);
#pragma unroll
    for (int h = 0; h < DEC_G; ++h) acc[h] += ps[h * DEC_KEYS + j] * v;
  }
#pragma unroll
  for (int h = 0; h < DEC_G; ++h) po[(out_base + (int64_t)h * nchunks) * D + tid] = acc[h];
}

__global__ void __launch_bounds__(D)
    attn_decode_combine_kernel(const float* __restrict__ po, const float* __restrict__ pml, int nq, int nchunks,
                               bf16* __restrict__ out) {
  const int h = blockIdx.x, b = blockIdx.y, t = threadIdx.x;
  const int64_t base = ((int64_t)b * nq + h) * nchunks;
  float M = -INFINITY;
  for (int c = 0; c < nchunks; ++c) M = fmaxf(M, pml[(base + c) * 2]);
  float l = 0.f, o = 0.f;
  for (int c = 0; c < nchunks; ++c) {
    const float m = pml[(base + c) * 2];
    if (m == -INFINITY) continue;
    const float w = ex2(m - M);
    l += w * pml[(base + c) * 2 + 1];
    o += w * po[(base + c) * D + t];
  }
  out[((int64_t)b * nq + h) * D + t] = __float2bfloat16_rn(l > 0.f ? o / l : 0.f);
}

}  // namespace

static PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    else
      cudaGetLastError();
  }
  return fn;
}

bool map_rows128(CUtensorMap* m, const void* ptr, int64_t rows, int box_rows) {
  auto enc = encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {128, (cuuint64_t)rows};
  cuuint64_t strides[1] = {256};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool flash_supported(int hd, int nq, int nkv) { return hd == D && nq % nkv == 0; }

// q [B][nq][S][128], K/V cache [B][nkv][ctx][128] (positions 0..S-1 valid),
// o [B*S][nq*128].  All sequences start at position 0.
cudaError_t launch_flash_prefill(const void* q, const void* K, const void* V, void* o, int B, int S, int nq, int nkv,
                                 int64_t ctx, cudaStream_t st) {
  if (B == 0 || S == 0) return cudaSuccess;
  CUtensorMap mq, mk, mv;
  if (!map_rows128(&mq, q, (int64_t)B * nq * S, BQ) || !map_rows128(&mk, K, (int64_t)B * nkv * ctx, BKV) ||
      !map_rows128(&mv, V, (int64_t)B * nkv * ctx, BKV))
    return cudaErrorInvalidValue;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(flash_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)D);
  dim3 grid((unsigned)((S + BQ - 1) / BQ), (unsigned)nq, (unsigned)B);
  flash_fwd_kernel<<<grid, THREADS, SMEM, st>>>(mq, mk, mv, (bf16*)o, S, nq, nkv, ctx, scale_log2, status_ptr());
  return cudaGetLastError();
}

bool decode_attention_supported(int hd, int nq, int nkv) { return hd == D && nq == DEC_G * nkv; }

int64_t decode_attention_scratch_floats(int B, int nq, int64_t ctx) {
  const int64_t nch = (ctx + DEC_KEYS - 1) / DEC_KEYS;
  return (int64_t)B * nq * nch * (D + 2);
}

// q [B][nq][1][128]; K/V cache [B][nkv][ctx][128] with the new position
// already written; start[b] = position of the new token; o [B][nq*128].
// scratch: decode_attention_scratch_floats(B, nq, ctx) floats.
cudaError_t launch_attention_decode(const void* q, const void* K, const void* V, void* o, int B, int nq, int nkv,
                                    int64_t ctx, int max_len, const int32_t* start, float* scratch, cudaStream_t st) {
  if (B == 0) return cudaSuccess;
  static bool attr = false;
  if (!attr) {
    cudaError_t e =
        cudaFuncSetAttribute(attn_decode_partial_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, DEC_SMEM);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  const int nch = (max_len + DEC_KEYS - 1) / DEC_KEYS;
  float* po = scratch;
  float* pml = scratch + (int64_t)B * nq * nch * D;
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)D);
  dim3 g1((unsigned)nch, (unsigned)nkv, (unsigned)B);
  attn_decode_partial_kernel<<<g1, DEC_THREADS, DEC_SMEM, st>>>((const bf16*)q, (const bf16*)K, (const bf16*)V, start,
                                                                nq, nkv, ctx, nch, scale_log2, po, pml, status_ptr());
  dim3 g2((unsigned)nq, (unsigned)B);
  attn_decode_combine_kernel<<<g2, D, 0, st>>>(po, pml, nq, nch, (bf16*)o);
  return cudaGetLastError();
}

}  // namespace loopk
