// Causal GQA flash attention for prefill on the 5th-generation tensor cores
// (tcgen05): O = softmax(Q K^T / sqrt(128) + causal mask) V, kv head = q head / 4 ("How Does SenseNova-Loop Get More
// Depth Without More Parameters?", section "How does the hybrid attention
// pattern work?").
//
// One CTA computes 128 queries of one head over key tiles of 128:
//   warp 0      TMA producer: Q once, then K and V tiles into a 2-slot ring
//               (128-byte swizzle);
//   warp 1      one thread issues tcgen05.mma: S_j = Q K_j^T into one of two
//               128-column TMEM buffers, then O += P_{j-1} V_{j-1} into a
//               third (P from shared memory as the K-major A operand, V read
//               in place as an MN-major B operand);
//   warp 2      allocates / frees TMEM;
//   warps 4-7   softmax: thread r owns query row r, loads its S row from TMEM,
//               keeps the running max and sum, writes P (bf16) to shared
//               memory, and rescales its O row in TMEM only when the max grew
//               by more than 2^8 since the last rescale (the stale max then
//               bounds P by 256); at the end O / l is stored.
// Every mbarrier wait is bounded; the whole warp leaves together before any
// warp-collective TMEM access.

#include <cuda.h>

#include "model.h"

namespace loopk {

namespace {

constexpr int BQ = 128, BKV = 128, D = 128, NS = 2;
constexpr int THREADS = 256;
constexpr int Q_BYTES = BQ * D * 2;      // 32 KB: two boxes [128][64]
constexpr int KV_TILE = BKV * D * 2;     // 32 KB: two boxes [128][64]
constexpr int P_BYTES = BQ * BKV * 2;    // 32 KB
constexpr int SMEM = Q_BYTES + NS * 2 * KV_TILE + P_BYTES + 1024 + 256;
constexpr int TMEM_COLS = 512;           // S buffers at 0 and 128, O at 256
constexpr uint32_t IDESC_S = idesc_bf16_f32(BQ, BKV);
constexpr uint32_t IDESC_PV = idesc_bf16_f32(BQ, D, true);
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units

// K-major SW128 descriptor of a [rows][128] bf16 tile stored as two boxes of
// [rows][64]: k-step kk covers columns 16 kk .. 16 kk + 15.
LOOP_DEV uint64_t kmajor_desc(uint32_t base, int rows, int kk) {
  return smem_desc_sw128(base + (uint32_t)((kk >> 2) * rows * 128 + (kk & 3) * 32), 1024);
}

__global__ void __launch_bounds__(THREADS, 1)
    flash_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                    const __grid_constant__ CUtensorMap tv, bf16* __restrict__ out, int S, int nq, int nkv,
                    int64_t ctx, float scale_log2, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sq = smem;
  uint8_t* skv = smem + Q_BYTES;  // slot s: K at skv + 2 s KV_TILE, V after it
  uint8_t* sp = skv + NS * 2 * KV_TILE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sp + P_BYTES);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + NS;
  uint64_t* s_full = kv_empty + NS;
  uint64_t* s_free = s_full + 2;
  uint64_t* p_full = s_free + 2;
  uint64_t* o_done = p_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_done + 1);

  const int nqb = (S + BQ - 1) / BQ;
  const int qb = nqb - 1 - (int)blockIdx.x;  // longest rows first
  const int h = blockIdx.y, b = blockIdx.z;
  const int kvh = h / (nq / nkv);
  const int q0 = qb * BQ;
  const int ntiles = (min(q0 + BQ, S) - 1) / BKV + 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 4);
    }
    mbar_init(p_full, 4);
    mbar_init(o_done, 1);
    fence_mbar_init();
  }
  if (warp == 2) tmem_alloc(tmem_slot, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_s[2] = {tmem, tmem + 128};
  const uint32_t t_o = tmem + 256;

  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tq);
    prefetch_tmap(&tk);
    prefetch_tmap(&tv);
    const int qrow = (b * nq + h) * S + q0;
    mbar_expect_tx(q_full, Q_BYTES);
    tma_load_2d(sq, &tq, q_full, 0, qrow);
    tma_load_2d(sq + Q_BYTES / 2, &tq, q_full, 64, qrow);
    const int64_t krow0 = ((int64_t)b * nkv + kvh) * ctx;
    for (int j = 0; j < ntiles; ++j) {
      const int s = j % NS;
      if (!mbar_wait(&kv_empty[s], ((j / NS) & 1) ^ 1, status, STATUS_WAIT_PRODUCER)) break;
      uint8_t* kt = skv + 2 * s * KV_TILE;
      uint8_t* vt = kt + KV_TILE;
      const int row = (int)(krow0 + (int64_t)j * BKV);
      mbar_expect_tx(&kv_full[s], 2 * KV_TILE);
      tma_load_2d(kt, &tk, &kv_full[s], 0, row);
      tma_load_2d(kt + KV_TILE / 2, &tk, &kv_full[s], 64, row);
      tma_load_2d(vt, &tv, &kv_full[s], 0, row);
      tma_load_2d(vt + KV_TILE / 2, &tv, &kv_full[s], 64, row);
    }
  } else if (warp == 1 && lane == 0) {
    const uint32_t q_u = smem_u32(sq), p_u = smem_u32(sp), kv_u = smem_u32(skv);
    bool ok = mbar_wait(q_full, 0, status, STATUS_WAIT_MMA);
    auto issue_pv = [&](int jj) -> bool {  // O += P_jj V_jj
      if (!mbar_wait(p_full, jj & 1, status, STATUS_WAIT_MMA)) return false;
      tc_fence_after();
      const uint32_t vt = kv_u + (2 * (jj % NS) + 1) * KV_TILE;
#pragma unroll
      for (int kk = 0; kk < BKV / 16; ++kk)
        tc_mma_f16(t_o, kmajor_desc(p_u, BQ, kk), smem_desc_sw128_lbo(vt + kk * 2048, KV_TILE / 2, 1024), IDESC_PV,
                   (jj > 0 || kk > 0) ? 1u : 0u);
      tc_commit(&kv_empty[jj % NS]);
      tc_commit(o_done);
      return true;
    };
    for (int j = 0; j < ntiles && ok; ++j) {
      const int sb = j & 1;
      if (!mbar_wait(&kv_full[j % NS], (j / NS) & 1, status, STATUS_WAIT_MMA)) { ok = false; break; }
      if (j >= 2 && !mbar_wait(&s_free[sb], ((j - 2) >> 1) & 1, status, STATUS_WAIT_MMA)) { ok = false; break; }
      tc_fence_after();
      const uint32_t kt = kv_u + 2 * (j % NS) * KV_TILE;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        tc_mma_f16(t_s[sb], kmajor_desc(q_u, BQ, kk), kmajor_desc(kt, BKV, kk), IDESC_S, kk > 0 ? 1u : 0u);
      tc_commit(&s_full[sb]);
      if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
    }
    if (ok) issue_pv(ntiles - 1);
  } else if (warp >= 4) {
    const int quarter = warp & 3;
    const int r = 32 * quarter + lane;  // query row in the block
    const int qpos = q0 + r;
    const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;
    uint8_t* prow = sp;
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < ntiles && ok; ++j) {
      const int sb = j & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&s_full[sb], (j >> 1) & 1, status, STATUS_WAIT_EPILOGUE));
      if (!ok) break;
      tc_fence_after();
      float sv[BKV];
#pragma unroll
      for (int c = 0; c < BKV / 32; ++c) {
        float v[32];
        tmem_ld32(t_s[sb] + lane_off + 32 * c, v);
        tc_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) sv[32 * c + i] = v[i];
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[sb]);
      const int kbase = j * BKV;
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < BKV; ++i) {
        const float x = (kbase + i <= qpos) ? sv[i] * scale_log2 : -INFINITY;
        sv[i] = x;
        mx = fmaxf(mx, x);
      }
      float corr = 1.f;
      if (mx > m_ref + RESCALE_THRESHOLD) {
        corr = ex2(m_ref - mx);  // 0 on the first tile
        m_ref = mx;
      }
      float rs = 0.f;
      uint32_t pk[BKV / 2];
#pragma unroll
      for (int i = 0; i < BKV / 2; ++i) {
        const float p0 = ex2(sv[2 * i] - m_ref), p1 = ex2(sv[2 * i + 1] - m_ref);
        rs += p0 + p1;
        pk[i] = pack_bf16x2(p0, p1);
      }
      l = l * corr + rs;
      // P_{j-1} V_{j-1} must be done before O is rescaled and P is overwritten
      if (j >= 1) {
        ok = __all_sync(0xffffffffu, mbar_wait(o_done, (j - 1) & 1, status, STATUS_WAIT_EPILOGUE));
        if (!ok) break;
        tc_fence_after();
        if (__any_sync(0xffffffffu, corr != 1.f)) {
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            float v[32];
            tmem_ld32(t_o + lane_off + 32 * c, v);
            tc_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] *= corr;
            tmem_st32(t_o + lane_off + 32 * c, v);
          }
          tc_wait_st();
        }
      }
      // P row r: 16 chunks of 8 keys, 128-byte swizzle, two boxes of 64 keys
#pragma unroll
      for (int c = 0; c < BKV / 8; ++c) {
        const uint32_t off = (uint32_t)((c >> 3) * BQ * 128 + r * 128 + (((c & 7) ^ (r & 7)) << 4));
        *reinterpret_cast<uint4*>(prow + off) = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(o_done, (ntiles - 1) & 1, status, STATUS_WAIT_EPILOGUE));
    if (ok) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      bf16* orow = out + ((int64_t)b * S + qpos) * ((int64_t)nq * D) + (int64_t)h * D;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        float v[32];
        tmem_ld32(t_o + lane_off + 32 * c, v);
        tc_wait_ld();
        if (qpos < S) {
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[i] = make_uint4(pack_bf16x2(v[8 * i] * inv, v[8 * i + 1] * inv),
                                pack_bf16x2(v[8 * i + 2] * inv, v[8 * i + 3] * inv),
                                pack_bf16x2(v[8 * i + 4] * inv, v[8 * i + 5] * inv),
                                pack_bf16x2(v[8 * i + 6] * inv, v[8 * i + 7] * inv));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace

bool flash_tc_supported(int hd, int nq, int nkv) { return hd == D && nq % nkv == 0; }

// q [B][nq][S][128], K/V cache [B][nkv][ctx][128] (positions 0..S-1 valid),
// o [B*S][nq*128].  All sequences start at position 0.
cudaError_t launch_flash_tc(const void* q, const void* K, const void* V, void* o, int B, int S, int nq, int nkv,
                            int64_t ctx, cudaStream_t st) {
  if (B == 0 || S == 0) return cudaSuccess;
  CUtensorMap mq, mk, mv;
  if (!map_rows128(&mq, q, (int64_t)B * nq * S, BQ) || !map_rows128(&mk, K, (int64_t)B * nkv * ctx, BKV) ||
      !map_rows128(&mv, V, (int64_t)B * nkv * ctx, BKV))
    return cudaErrorInvalidValue;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(flash_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)D);
  dim3 grid((unsigned)((S + BQ - 1) / BQ), (unsigned)nq, (unsigned)B);
  flash_tc_kernel<<<grid, THREADS, SMEM, st>>>(mq, mk, mv, (bf16*)o, S, nq, nkv, ctx, scale_log2, status_ptr());
  return cudaGetLastError();
}

}  // namespace loopk
