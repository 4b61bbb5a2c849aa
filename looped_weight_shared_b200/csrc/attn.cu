// Causal GQA attention for one new token per sequence (decode), over the KV
// cache of a full-attention execution: o = softmax(q K^T / sqrt(128)) V with
// kv head = q head / 4 ("How Does SenseNova-Loop Get More Depth Without More
// Parameters?", section "How does the hybrid attention pattern work?").  The
// prefill kernel is in attn_tc.cu.  Also the TMA map helper shared by the
// attention and linear-attention kernels.

#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "model.h"

namespace loopk {

namespace {

constexpr int D = 128;

// ---------------------------------------------------------------------------
// Decode attention (one new query per sequence, GQA group of 4).  CTA
// (chunk of 1024 keys, kv head, sequence): a producer warp streams 64-key K/V
// tiles by TMA (128-byte swizzle) into a 4-slot ring, one slot per compute
// warp; each compute warp runs S = Q K^T and O += P V on the tensor cores with
// the 4 query heads of the group as rows 0-3 of a 16-row tile, keeping its own
// online softmax.  The 4 warps merge in shared memory and the CTA writes the
// chunk's unnormalised o with its max m (log2 domain) and sum l; a combine
// kernel merges the chunks.  K/V are read from HBM once per step.
// ---------------------------------------------------------------------------
constexpr int DEC_CHUNK = 1024, DEC_TILE = 64, DEC_G = 4, DEC_WARPS = 4;
constexpr int DEC_THREADS = (DEC_WARPS + 1) * 32;
constexpr int DEC_Q_BYTES = 16 * D * 2;            // 16 rows x 128, two swizzled boxes of [16][64]
constexpr int DEC_KV_BYTES = 2 * DEC_TILE * D * 2;  // K and V tiles of one ring slot
constexpr int DEC_SMEM = DEC_Q_BYTES + DEC_WARPS * DEC_KV_BYTES + DEC_WARPS * DEC_G * (D + 2) * 4 + 128 + 1024;

__global__ void __launch_bounds__(DEC_THREADS, 1)
    attn_decode_partial_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                               const bf16* __restrict__ q, const int32_t* __restrict__ start, int nq, int nkv,
                               const int32_t* __restrict__ table, int pps, int nchunks, float scale_log2,
                               float* __restrict__ po,
                               float* __restrict__ pml, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sq = smem;
  uint8_t* ring = smem + DEC_Q_BYTES;  // slot w: K at ring + w * DEC_KV_BYTES, V after it
  float* co = reinterpret_cast<float*>(ring + DEC_WARPS * DEC_KV_BYTES);  // [warp][head][128]
  float* cm = co + DEC_WARPS * DEC_G * D;                                 // [warp][head] max
  float* cl = cm + DEC_WARPS * DEC_G;                                     // [warp][head] sum
  uint64_t* full = reinterpret_cast<uint64_t*>(cl + DEC_WARPS * DEC_G);
  uint64_t* empty = full + DEC_WARPS;

  const int chunk = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int k0 = chunk * DEC_CHUNK;
  // The producer looks up the chunk's page rows first, so the loads' latency
  // passes under the Q staging below (entries past the sequence are read, in
  // bounds, and not used).
  int rows[DEC_CHUNK / DEC_TILE];
  if (warp == DEC_WARPS && lane == 0) {
#pragma unroll
    for (int j = 0; j < DEC_CHUNK / DEC_TILE; ++j)
      rows[j] = (int)kv_row(table, pps, nkv, b, kvh, (int64_t)min(k0 / DEC_TILE + j, pps - 1) * DEC_TILE);
  }
  const int L = start[b] + 1;  // keys 0 .. start[b]; the new token's K/V are already in the cache
  const int64_t obase = ((int64_t)b * nq + kvh * DEC_G) * nchunks + chunk;
  if (k0 >= L) {  // past this sequence's end: an empty partial
    if (tid < DEC_G) {
      pml[(obase + (int64_t)tid * nchunks) * 2] = -INFINITY;
      pml[(obase + (int64_t)tid * nchunks) * 2 + 1] = 0.f;
    }
    return;
  }
  const int nk = min(DEC_CHUNK, L - k0);
  const int ntiles = (nk + DEC_TILE - 1) / DEC_TILE;
  if (tid == 0) {
    for (int w = 0; w < DEC_WARPS; ++w) {
      mbar_init(&full[w], 1);
      mbar_init(&empty[w], 1);
    }
    fence_mbar_init();
  }
  // Q rows 0-3 = the group's query heads, rows 4-15 zero (bf16, swizzled)
  for (int i = tid; i < 16 * D; i += DEC_THREADS) {
    const int r = i / D, d = i % D;
    const bf16 v = r < DEC_G ? q[((int64_t)b * nq + kvh * DEC_G + r) * D + d] : __float2bfloat16_rn(0.f);
    *reinterpret_cast<bf16*>(sq + sw(r, d >> 3, 16) + (d & 7) * 2) = v;
  }
  __syncthreads();

  if (warp == DEC_WARPS) {  // producer
    if (lane == 0) {
      prefetch_tmap(&tk);
      prefetch_tmap(&tv);
#pragma unroll  // unrolled so rows[] stays in registers
      for (int j = 0; j < DEC_CHUNK / DEC_TILE; ++j) {
        if (j >= ntiles) break;
        const int s = j % DEC_WARPS;
        const uint32_t ph = (j / DEC_WARPS) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, status, STATUS_WAIT_PRODUCER)) break;
        uint8_t* kt = ring + s * DEC_KV_BYTES;
        uint8_t* vt = kt + DEC_KV_BYTES / 2;
        const int row = rows[j];  // a whole page
        mbar_expect_tx(&full[s], DEC_KV_BYTES);
        tma_load_2d(kt, &tk, &full[s], 0, row);
        tma_load_2d(kt + DEC_KV_BYTES / 4, &tk, &full[s], 64, row);
        tma_load_2d(vt, &tv, &full[s], 0, row);
        tma_load_2d(vt + DEC_KV_BYTES / 4, &tv, &full[s], 64, row);
      }
    }
    return;
  }

  const int g = lane >> 2, t = lane & 3, mi = lane >> 3, ri = lane & 7;
  const uint32_t sq_u = smem_u32(sq), ring_u = smem_u32(ring);
  uint32_t qf[8][4];
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
    ldsm_x4(sq_u + sw((mi & 1) * 8 + ri, kk * 2 + (mi >> 1), 16), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
  float o[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m = -INFINITY, l = 0.f;  // row g (valid for g < 4)
  bool ok = true;
  for (int j = warp; j < ntiles && ok; j += DEC_WARPS) {
    const int s = j % DEC_WARPS;
    const uint32_t ph = (j / DEC_WARPS) & 1;
    ok = __all_sync(0xffffffffu, mbar_wait(&full[s], ph, status, STATUS_WAIT_EPILOGUE));
    if (!ok) break;
    const uint32_t kt = ring_u + s * DEC_KV_BYTES, vt = kt + DEC_KV_BYTES / 2;
    float sc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) sc[i][0] = sc[i][1] = sc[i][2] = sc[i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
#pragma unroll
      for (int nt = 0; nt < 8; nt += 2) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kt + sw(nt * 8 + (mi >> 1) * 8 + ri, kk * 2 + (mi & 1), DEC_TILE), b0, b1, b2, b3);
        mma_bf16(sc[nt], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b0, b1);
        mma_bf16(sc[nt + 1], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b2, b3);
      }
    const int kvalid = nk - j * DEC_TILE;  // keys of this tile inside the sequence
    float mx = m;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int kc = nt * 8 + 2 * t + e;
        const float v = kc < kvalid ? sc[nt][e] * scale_log2 : -INFINITY;
        sc[nt][e] = v;
        mx = fmaxf(mx, v);
      }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float corr = ex2(m - mx);
    m = mx;
    float rs = 0.f;
    uint32_t pa[8][2];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const float p0 = ex2(sc[nt][0] - mx), p1 = ex2(sc[nt][1] - mx);
      rs += p0 + p1;
      pa[nt][0] = pack_bf16x2(p0, p1);
      pa[nt][1] = 0u;  // rows 8-15 carry no query
    }
    l = l * corr + rs;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      o[i][0] *= corr;
      o[i][1] *= corr;
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
#pragma unroll
      for (int nt = 0; nt < 16; nt += 2) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(vt + sw(kk * 16 + (mi & 1) * 8 + ri, nt + (mi >> 1), DEC_TILE), b0, b1, b2, b3);
        mma_bf16(o[nt], pa[2 * kk][0], pa[2 * kk][1], pa[2 * kk + 1][0], pa[2 * kk + 1][1], b0, b1);
        mma_bf16(o[nt + 1], pa[2 * kk][0], pa[2 * kk][1], pa[2 * kk + 1][0], pa[2 * kk + 1][1], b2, b3);
      }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
  l += __shfl_xor_sync(0xffffffffu, l, 1);
  l += __shfl_xor_sync(0xffffffffu, l, 2);
  if (g < DEC_G) {
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      co[(warp * DEC_G + g) * D + nt * 8 + 2 * t] = o[nt][0];
      co[(warp * DEC_G + g) * D + nt * 8 + 2 * t + 1] = o[nt][1];
    }
    if (t == 0) {
      cm[warp * DEC_G + g] = m;
      cl[warp * DEC_G + g] = l;
    }
  }
  asm volatile("bar.sync 1, %0;" ::"n"(DEC_WARPS * 32));  // the compute warps only
  // merge the 4 warps: thread t < 128 owns dim t of every head
  for (int h = 0; h < DEC_G; ++h) {
    float M = -INFINITY;
    for (int w = 0; w < DEC_WARPS; ++w) M = fmaxf(M, cm[w * DEC_G + h]);
    float acc = 0.f, ls = 0.f;
    for (int w = 0; w < DEC_WARPS; ++w) {
      const float mw = cm[w * DEC_G + h];
      if (mw == -INFINITY) continue;
      const float f = ex2(mw - M);
      acc += f * co[(w * DEC_G + h) * D + tid];
      ls += f * cl[w * DEC_G + h];
    }
    po[(obase + (int64_t)h * nchunks) * D + tid] = acc;
    if (tid == 0) {
      pml[(obase + (int64_t)h * nchunks) * 2] = M;
      pml[(obase + (int64_t)h * nchunks) * 2 + 1] = ls;
    }
  }
}

__global__ void __launch_bounds__(D)
    attn_decode_combine_kernel(const float* __restrict__ po, const float* __restrict__ pml, int nq, int nchunks,
                               bf16* __restrict__ out) {
  const int h = blockIdx.x, b = blockIdx.y, t = threadIdx.x;
  griddep_launch_dependents();  // the output projection after this may start streaming its weights
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

bool decode_attention_supported(int hd, int nq, int nkv) { return hd == D && nq == DEC_G * nkv; }

int decode_attention_chunks(int max_len) { return (max_len + DEC_CHUNK - 1) / DEC_CHUNK; }

int64_t decode_attention_scratch_floats(int B, int nq, int64_t ctx) {
  const int64_t nch = (ctx + DEC_CHUNK - 1) / DEC_CHUNK;
  return (int64_t)B * nq * nch * (D + 2);
}

// q [B][nq][1][128]; K/V paged pools of pool_rows rows (see kv_row) with the
// new position already written; start[b] = position of the new token;
// o [B][nq*128].  scratch: decode_attention_scratch_floats(B, nq, max_ctx) floats.
cudaError_t launch_attention_decode(const void* q, const void* K, const void* V, void* o, int B, int nq, int nkv,
                                    const int32_t* table, int pps, int64_t pool_rows, int max_len,
                                    const int32_t* start, float* scratch, cudaStream_t st) {
  if (B == 0) return cudaSuccess;
  static_assert(DEC_TILE == KV_PAGE, "a decode tile is one KV page");
  CUtensorMap mk, mv;
  if (!map_rows128(&mk, K, pool_rows, DEC_TILE) || !map_rows128(&mv, V, pool_rows, DEC_TILE))
    return cudaErrorInvalidValue;
  static std::atomic<uint64_t> smem_set{0};
  if (cudaError_t e = set_smem_limit(attn_decode_partial_kernel, DEC_SMEM, smem_set); e != cudaSuccess) return e;
  const int nch = decode_attention_chunks(max_len);
  float* po = scratch;
  float* pml = scratch + (int64_t)B * nq * nch * D;
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)D);
  dim3 g1((unsigned)nch, (unsigned)nkv, (unsigned)B);
  attn_decode_partial_kernel<<<g1, DEC_THREADS, DEC_SMEM, st>>>(mk, mv, (const bf16*)q, start, nq, nkv, table, pps,
                                                                nch, scale_log2, po, pml, status_ptr());
  dim3 g2((unsigned)nq, (unsigned)B);
  attn_decode_combine_kernel<<<g2, D, 0, st>>>(po, pml, nq, nch, (bf16*)o);
  return cudaGetLastError();
}

}  // namespace loopk
