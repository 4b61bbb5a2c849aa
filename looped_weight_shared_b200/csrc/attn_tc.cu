// Causal GQA flash attention for prefill on the 5th-generation tensor cores
// (tcgen05): O = softmax(Q K^T / sqrt(128) + causal mask) V, kv head = q head / 4 ("How Does SenseNova-Loop Get More
// Depth Without More Parameters?", section "How does the hybrid attention
// pattern work?").
//
// One CTA computes two 128-query tiles (X = 0, 1: queries q0 .. q0 + 255 of
// the call, which may continue a sequence: query i at position start + i) of
// one head against the 64-key tiles both need, sharing each K/V tile:
//   warp 0      TMA producer: Q of both tiles once, then K and V tiles into a
//               4-slot ring (128-byte swizzle);
//   warps 1, 10 one lane each issues the tcgen05.mma of one query tile (warp 1
//               for tile 0, warp 10 for tile 1, so neither tile's issue order
//               waits on the other's softmax; warp 1 also allocates TMEM).
//               Each query tile has two score buffers in TMEM, so the scores
//               of key tile j + 1 are computed while the softmax of tile j
//               runs:  S_X(j+1) = Q_X K_{j+1}^T into buffer (j + 1) % 2, then
//               O_X += P_X(j) V_j with P_X(j) read from TMEM (written over
//               S_X(j)) and V read in place as an MN-major B operand;
//   warps 2-5   softmax of tile 0, warps 6-9 softmax of tile 1: thread r owns
//               query row r of its tile (TMEM lane r), loads its 64 scores,
//               keeps the running max and sum, writes P (bf16 pairs) back over
//               S, and rescales its O row in TMEM only when the max grew by
//               more than 2^8 since the last rescale (the stale max then
//               bounds P by 256), after the previous P V product is done; at
//               the end O / l is stored.
// TMEM: S/P buffers of 64 columns at 64 (2 X + b), O_0 at 256, O_1 at 384.
// Every mbarrier wait is bounded; the whole warp leaves together before any
// warp-collective TMEM access.

#include <cuda.h>

#include "model.h"

namespace loopk {

namespace {

constexpr int BQ = 128, BKV = 64, D = 128, NS = 4;
constexpr int THREADS = 352;             // producer, MMA tile 0, 2 softmax warpgroups, MMA tile 1
constexpr int Q_BYTES = BQ * D * 2;      // 32 KB: two boxes [128][64]
constexpr int KV_TILE = BKV * D * 2;     // 16 KB: two boxes [64][64]
constexpr int SMEM = 2 * Q_BYTES + NS * 2 * KV_TILE + 1024 + 256;
static_assert(SMEM <= 232448, "shared memory per block");
constexpr int TMEM_COLS = 512;
constexpr uint32_t T_O = 256;            // O_X at T_O + 128 X
constexpr uint32_t IDESC_S = idesc_bf16_f32(BQ, BKV);
constexpr uint32_t IDESC_PV = idesc_bf16_f32(BQ, D, true);
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units

LOOP_DEV float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// P for the 64 keys of one row: p = 2^(s scale - m_ref) as bf16 pairs into
// pk, their sum added to rs2.  The exponent argument is one packed fp32x2
// FMA, the power of two ex2.approx on the MUFU unit (evaluating part of them
// as a polynomial on the FMA pipe measured slower here: with one MMA issuer
// per query tile the softmax is not MUFU-bound).
LOOP_DEV void softmax_row(const float (&sv)[BKV], float2 sc, float2 nm, float (&pk)[32], float2& rs2) {
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const float2 xx = ffma2(make_float2(sv[2 * i], sv[2 * i + 1]), sc, nm);
    const float2 pp = make_float2(ex2(xx.x), ex2(xx.y));
    rs2 = fadd2(rs2, pp);
    pk[i] = __uint_as_float(pack_bf16x2(pp.x, pp.y));
  }
}

// K-major SW128 descriptor of a [rows][128] bf16 tile stored as two boxes of
// [rows][64]: k-step kk covers columns 16 kk .. 16 kk + 15.
LOOP_DEV uint64_t kmajor_desc(uint32_t base, int rows, int kk) {
  return smem_desc_sw128(base + (uint32_t)((kk >> 2) * rows * 128 + (kk & 3) * 32), 1024);
}

__global__ void __launch_bounds__(THREADS, 1)
    flash_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                    const __grid_constant__ CUtensorMap tv, bf16* __restrict__ out, int S, int nq, int nkv,
                    const int32_t* __restrict__ table, int pps, const int32_t* __restrict__ start, int packed,
                    float scale_log2, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sq = smem;                 // tile X at sq + X Q_BYTES
  uint8_t* skv = smem + 2 * Q_BYTES;  // slot s: K at skv + 2 s KV_TILE, V after it
  uint64_t* bars = reinterpret_cast<uint64_t*>(skv + NS * 2 * KV_TILE);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + NS;
  uint64_t* s_full = kv_empty + NS;  // [X][buffer]
  uint64_t* p_full = s_full + 4;     // [X][buffer]
  uint64_t* pv_done = p_full + 4;    // [X]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(pv_done + 2);

  // Unpacked: CTA (query-tile pair, query head, sequence).  Packed (a few new
  // tokens per sequence, grp * S <= 128): CTA (kv head, sequence) whose one
  // tile holds the S queries of each of the grp query heads sharing that kv
  // head, row r = (head kvh * grp + r / S, query r % S): the heads' q rows are
  // adjacent in q, so one box loads them, and K/V are read once per kv head.
  const int grp = nq / nkv;
  const int npair = (S + 2 * BQ - 1) / (2 * BQ);
  const int q0 = packed ? 0 : 2 * BQ * (npair - 1 - (int)blockIdx.x);  // a head's longest pairs first
  const int b = blockIdx.z;
  const int kvh = packed ? (int)blockIdx.y : (int)blockIdx.y / grp;
  const int h = packed ? kvh * grp : (int)blockIdx.y;  // the (first) query head
  // query i of the call sits at position p0 + i and sees keys 0 .. p0 + i
  const int p0 = start ? start[b] : 0;
  // key tiles each query tile needs (0: the second tile is past the end)
  const int nt[2] = {(p0 + min(q0 + BQ, S) - 1) / BKV + 1,
                     !packed && q0 + BQ < S ? (p0 + min(q0 + 2 * BQ, S) - 1) / BKV + 1 : 0};
  const int ntiles = max(nt[0], nt[1]);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 2);  // one commit per query tile (the longer tile commits for a missing one)
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 4);
    }
    mbar_init(&pv_done[0], 1);
    mbar_init(&pv_done[1], 1);
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tq);
    prefetch_tmap(&tk);
    prefetch_tmap(&tv);
    const int qrow = (b * nq + h) * S + q0;
    const int ntq = nt[1] > 0 ? 2 : 1;
    mbar_expect_tx(q_full, ntq * Q_BYTES);
    for (int x = 0; x < ntq; ++x) {
      tma_load_2d(sq + x * Q_BYTES, &tq, q_full, 0, qrow + x * BQ);
      tma_load_2d(sq + x * Q_BYTES + Q_BYTES / 2, &tq, q_full, 64, qrow + x * BQ);
    }
    // key tile j is page j; its row is looked up one tile ahead, under the wait
    int next_row = ntiles > 0 ? (int)kv_row(table, pps, nkv, b, kvh, 0) : 0;
    for (int j = 0; j < ntiles; ++j) {
      const int s = j % NS;
      const int row = next_row;
      if (j + 1 < ntiles) next_row = (int)kv_row(table, pps, nkv, b, kvh, (int64_t)(j + 1) * BKV);
      if (!mbar_wait(&kv_empty[s], ((j / NS) & 1) ^ 1, status, STATUS_WAIT_PRODUCER)) break;
      uint8_t* kt = skv + 2 * s * KV_TILE;
      uint8_t* vt = kt + KV_TILE;
      mbar_expect_tx(&kv_full[s], 2 * KV_TILE);
      tma_load_2d(kt, &tk, &kv_full[s], 0, row);
      tma_load_2d(kt + KV_TILE / 2, &tk, &kv_full[s], 64, row);
      tma_load_2d(vt, &tv, &kv_full[s], 0, row);
      tma_load_2d(vt + KV_TILE / 2, &tv, &kv_full[s], 64, row);
    }
  } else if ((warp == 1 || warp == 10) && lane == 0) {
    const int x = warp == 1 ? 0 : 1;  // the query tile this thread issues for
    const int y = 1 - x;
    const uint32_t q_u = smem_u32(sq), kv_u = smem_u32(skv);
    auto slot = [&](int j) { return kv_u + 2 * (j % NS) * KV_TILE; };
    auto sbuf = [&](int j) { return tmem + (uint32_t)(64 * (2 * x + (j & 1))); };
    // S_X(j) = Q_X K_j^T into buffer j % 2
    auto issue_s = [&](int j) {
      tc_fence_after();
      const uint32_t kt = slot(j);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        tc_mma_f16(sbuf(j), kmajor_desc(q_u + x * Q_BYTES, BQ, kk), kmajor_desc(kt, BKV, kk), IDESC_S,
                   kk > 0 ? 1u : 0u);
      tc_commit(&s_full[2 * x + (j & 1)]);
    };
    // O_X += P_X(j) V_j, P_X(j) read from TMEM (the first 32 columns of its buffer)
    auto issue_pv = [&](int j) {
      tc_fence_after();
      const uint32_t vt = slot(j) + KV_TILE;
#pragma unroll
      for (int kk = 0; kk < BKV / 16; ++kk)
        tc_mma_f16_ts(tmem + T_O + 128 * x, sbuf(j) + 8 * kk, smem_desc_sw128_lbo(vt + kk * 2048, KV_TILE / 2, 1024),
                      IDESC_PV, (j > 0 || kk > 0) ? 1u : 0u);
      tc_commit(&pv_done[x]);
    };
    auto kv_ready = [&](int j) { return mbar_wait(&kv_full[j % NS], (j / NS) & 1, status, STATUS_WAIT_MMA); };
    bool ok = nt[x] > 0 && mbar_wait(q_full, 0, status, STATUS_WAIT_MMA) && kv_ready(0);
    if (ok) issue_s(0);
    for (int j = 0; j < nt[x] && ok; ++j) {
      if (j + 1 < nt[x]) {
        // buffer (j + 1) % 2 held P_X(j - 1): its product must be done
        ok = kv_ready(j + 1) && (j == 0 || mbar_wait(&pv_done[x], (j - 1) & 1, status, STATUS_WAIT_MMA));
        if (!ok) break;
        issue_s(j + 1);
      }
      ok = mbar_wait(&p_full[2 * x + (j & 1)], (j >> 1) & 1, status, STATUS_WAIT_MMA);
      if (!ok) break;
      issue_pv(j);
      // K_j, V_j are free once both tiles' products of key tile j are done;
      // the longer tile also commits for key tiles the other does not use
      tc_commit(&kv_empty[j % NS]);
      if (j >= nt[y]) tc_commit(&kv_empty[j % NS]);
    }
  } else if (warp >= 2 && warp < 10) {
    const int x = (warp - 2) >> 2;    // query tile of this warpgroup
    const int quarter = warp & 3;     // TMEM lanes 32 quarter .. (fixed by the warp's rank)
    const int r = 32 * quarter + lane;
    const int qx0 = q0 + BQ * x;  // the tile's first query (its smallest position is p0 + qx0)
    // this row's query (within the call) and head; rows past the queries are computed but not stored
    const bool rvalid = packed ? r < grp * S : qx0 + r < S;
    const int qpos = packed ? (rvalid ? r % S : 0) : qx0 + r;
    const int hrow = packed ? h + (rvalid ? r / S : 0) : h;
    const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;
    const uint32_t t_o = tmem + T_O + 128 * x + lane_off;
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nt[x] && ok; ++j) {
      const int bi = 2 * x + (j & 1);
      const uint32_t t_s = tmem + (uint32_t)(64 * bi) + lane_off;
      ok = __all_sync(0xffffffffu, mbar_wait(&s_full[bi], (j >> 1) & 1, status, STATUS_WAIT_EPILOGUE));
      if (!ok) break;
      tc_fence_after();
      float sv[BKV];
      tmem_ld32(t_s, *reinterpret_cast<float(*)[32]>(sv));
      tmem_ld32(t_s + 32, *reinterpret_cast<float(*)[32]>(sv + 32));
      tc_wait_ld();
      const int kbase = j * BKV;
      const bool masked = kbase + BKV - 1 > p0 + qx0;  // some key of the tile lies past some row's position
      if (masked) {
#pragma unroll
        for (int i = 0; i < BKV; ++i)
          if (kbase + i > p0 + qpos) sv[i] = -INFINITY;
      }
      float mraw = sv[0];
#pragma unroll
      for (int i = 1; i + 1 < BKV; i += 2) mraw = max3f(mraw, sv[i], sv[i + 1]);
      mraw = fmaxf(mraw, sv[BKV - 1]);
      const float mx = mraw * scale_log2;
      float corr = 1.f;
      if (mx > m_ref + RESCALE_THRESHOLD) {
        corr = ex2(m_ref - mx);  // 0 on the first tile
        m_ref = mx;
      }
      // p = 2^(s scale - m_ref), two lanes per packed FMA and add
      const float2 sc = make_float2(scale_log2, scale_log2), nm = make_float2(-m_ref, -m_ref);
      float2 rs2 = make_float2(0.f, 0.f);
      {
        float pk[32];
        softmax_row(sv, sc, nm, pk, rs2);
        tmem_st32(t_s, pk);
      }
      l = l * corr + (rs2.x + rs2.y);
      // pv_done is waited by parity, which is exact only while at most one
      // product is pending.  At step j that holds: the issuer saw PV(j - 2)
      // done before it issued S(j), and PV(j) needs this step's P.  So the
      // product of the previous key tile is awaited here before O is
      // rescaled, and always at the last key tile, so that the final wait
      // below also has at most one pending (without it, PV(nt - 2) and
      // PV(nt - 1) could both be pending there, a parity that matches a
      // completed phase, and O would be read early).
      const bool rescale = __any_sync(0xffffffffu, corr != 1.f);
      if (j >= 1 && (rescale || j == nt[x] - 1)) {
        ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[x], (j - 1) & 1, status, STATUS_WAIT_EPILOGUE));
        if (!ok) break;
      }
      if (j >= 1 && rescale) {
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          float v[32];
          tmem_ld32(t_o + 32 * c, v);
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] *= corr;
          tmem_st32(t_o + 32 * c, v);
        }
      }
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[bi]);
    }
    if (ok && nt[x] > 0) ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[x], (nt[x] - 1) & 1, status, STATUS_WAIT_EPILOGUE));
    if (ok && nt[x] > 0) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      bf16* orow = out + ((int64_t)b * S + qpos) * ((int64_t)nq * D) + (int64_t)hrow * D;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        float v[32];
        tmem_ld32(t_o + 32 * c, v);
        tc_wait_ld();
        if (rvalid) {
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
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace

bool flash_tc_supported(int hd, int nq, int nkv) { return hd == D && nq % nkv == 0; }

// q [B][nq][S][128], K/V paged pools of pool_rows rows (see kv_row), o
// [B*S][nq*128].  The S queries of sequence b sit at positions start[b] ..
// start[b] + S - 1 (start NULL: from 0) and their keys, positions 0 ..
// start[b] + S - 1, are in the cache.
cudaError_t launch_flash_tc(const void* q, const void* K, const void* V, void* o, int B, int S, int nq, int nkv,
                            const int32_t* table, int pps, int64_t pool_rows, const int32_t* start, cudaStream_t st) {
  if (B == 0 || S == 0) return cudaSuccess;
  static_assert(BKV == KV_PAGE, "a key tile is one KV page");
  CUtensorMap mq, mk, mv;
  if (!map_rows128(&mq, q, (int64_t)B * nq * S, BQ) || !map_rows128(&mk, K, pool_rows, BKV) ||
      !map_rows128(&mv, V, pool_rows, BKV))
    return cudaErrorInvalidValue;
  static std::atomic<uint64_t> smem_set{0};
  if (cudaError_t e = set_smem_limit(flash_tc_kernel, SMEM, smem_set); e != cudaSuccess) return e;
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)D);
  const int packed = start && (int64_t)S * (nq / nkv) <= BQ;  // a few new tokens: heads of a group share a tile
  dim3 grid(packed ? 1u : (unsigned)((S + 2 * BQ - 1) / (2 * BQ)), packed ? (unsigned)nkv : (unsigned)nq, (unsigned)B);
  flash_tc_kernel<<<grid, THREADS, SMEM, st>>>(mq, mk, mv, (bf16*)o, S, nq, nkv, table, pps, start, packed,
                                               scale_log2, status_ptr());
  return cudaGetLastError();
}

}  // namespace loopk
