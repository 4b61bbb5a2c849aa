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

}  // namespace loopk
