// Tensor-core projection GEMM for sm_100a: C = A[M][K] W[N][K]^T in bf16 with
// fp32 accumulation in tensor memory, followed by the projection's epilogue
// (residual add, mHC stream write, SwiGLU, q/k/v split with L2 norm or RoPE
// and KV-cache write, or plain fp32 logits).
//
// Persistent kernel, one CTA per SM, warp-specialised:
//   warp 0      TMA producer: A tile 128 x 64 and W tile 256 x 64 per stage,
//               128-byte swizzle, 4 stages in shared memory;
//   warp 1      one thread issues tcgen05.mma (M = 128, N = 256, K = 16) into
//               one of two 256-column TMEM accumulators;
//   warp 2      allocates / frees the 512 TMEM columns;
//   warps 4-11  epilogue, two warpgroups splitting the tile's columns:
//               tcgen05.ld of the accumulator rows (warp w reads TMEM lanes
//               32 (w % 4) ..), fused output, then release the accumulator
//               so the next tile's MMAs overlap this epilogue.
// Every wait on an mbarrier gives up after ~2 s and flags the status word.

#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "model.h"

namespace loopk {

namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int EPI_OFF = STAGES * STAGE_BYTES + 256;  // after the barriers: 8 epilogue warps x 4 KB
constexpr int SMEM_BYTES = EPI_OFF + 8 * 4096 + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory per block");
constexpr int THREADS = 256;       // skinny kernel: 4 role warps + 4 epilogue warps
constexpr int GEMM_THREADS = 384;  // main kernel: 4 role warps + 8 epilogue warps (two column halves)
constexpr int TMEM_COLS = 512;
// tile raster: group_m row blocks sweep the N blocks together (the host picks
// group_m per launch: more row blocks when a row block's A is small, so each
// W tile is read fewer times while the group's A stays in L2)
constexpr int GROUP_M_SMALL_K = 32, GROUP_M_LARGE_K = 16;
constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN);

struct EpiP {
  int M, N;
  int group_m;  // raster group (row blocks)
  float* c;
  int64_t ldc;
  float* s;
  const float* coef;
  bf16* a;
  bf16* q;
  bf16* k;
  bf16* v;
  float* gl;
  const float2* rope;
  const int32_t* start;
  int S, hq, hkv, n_lin;
  const int32_t* table;  // QKV_FULL: KV page table (the call's first sequence) and its row stride
  int pps;
  float eps;
  // MHC_WRITE: the next mHC site's Phi * gamma [8][2N], and where the
  // partial projections of the new streams go, [M][2 N / BN][9] (NULL: none)
  const float* pphig;
  float* ppart;
};

LOOP_DEV void ld_chunk(uint32_t taddr, float (&v)[32]) {
  tmem_ld32(taddr, v);
  tc_wait_ld();
}

LOOP_DEV void store_bf16x32(bf16* dst, const float (&v)[32], float scale) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 u;
    u.x = pack_bf16x2(v[8 * i + 0] * scale, v[8 * i + 1] * scale);
    u.y = pack_bf16x2(v[8 * i + 2] * scale, v[8 * i + 3] * scale);
    u.z = pack_bf16x2(v[8 * i + 4] * scale, v[8 * i + 5] * scale);
    u.w = pack_bf16x2(v[8 * i + 6] * scale, v[8 * i + 7] * scale);
    d[i] = u;
  }
}

// L2-normalise (optional) one 128-column head held in TMEM and store it bf16.
// Every lane runs the TMEM loads (warp-collective); only rows < M store.
LOOP_DEV void head_store(uint32_t t0, bf16* dst, bool l2, float eps, bool valid) {
  float scale = 1.f;
  float v[32];
  if (l2) {
    float ss = 0.f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      ld_chunk(t0 + 32 * c, v);
#pragma unroll
      for (int j = 0; j < 32; ++j) ss += v[j] * v[j];
    }
    scale = rsqrtf(ss + eps);
  }
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    ld_chunk(t0 + 32 * c, v);
    if (valid) store_bf16x32(dst + 32 * c, v, scale);
  }
}

// Rotate-half RoPE on one 128-column head held in TMEM, then store bf16.
LOOP_DEV void head_store_rope(uint32_t t0, bf16* dst, const float2* cs_row, bool valid) {
#pragma unroll 1
  for (int c = 0; c < 2; ++c) {
    float a[32], b[32];
    ld_chunk(t0 + 32 * c, a);
    ld_chunk(t0 + 64 + 32 * c, b);
    if (!valid) continue;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const float2 cs = cs_row[32 * c + j];
      const float x = a[j], y = b[j];
      a[j] = x * cs.x - y * cs.y;
      b[j] = y * cs.x + x * cs.y;
    }
    store_bf16x32(dst + 32 * c, a, 1.f);
    store_bf16x32(dst + 64 + 32 * c, b, 1.f);
  }
}

// r[k] holds this lane's part of a sum for row group k (k = 0..7); the 8 lanes
// whose low 3 bits are 0..7 and whose other bits agree hold the other parts.
// Returns the total for row group (lane & 7), reduced in a fixed tree.
LOOP_DEV float reduce_scatter8(const float (&r)[8], int lane) {
  const bool b2 = lane & 4, b1 = lane & 2, b0 = lane & 1;
  float t[4], u[2];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float keep = b2 ? r[k + 4] : r[k], give = b2 ? r[k] : r[k + 4];
    t[k] = keep + __shfl_xor_sync(0xffffffffu, give, 4);
  }
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const float keep = b1 ? t[k + 2] : t[k], give = b1 ? t[k] : t[k + 2];
    u[k] = keep + __shfl_xor_sync(0xffffffffu, give, 2);
  }
  const float keep = b0 ? u[1] : u[0], give = b0 ? u[0] : u[1];
  return keep + __shfl_xor_sync(0xffffffffu, give, 1);
}

// a . w0 + b . w1 over the 8 entries, as packed fp32x2 FMAs
LOOP_DEV float dot8(float4 a, float4 b, float4 w0, float4 w1) {
  float2 s = ffma2(make_float2(a.x, a.y), make_float2(w0.x, w0.y), make_float2(0.f, 0.f));
  s = ffma2(make_float2(a.z, a.w), make_float2(w0.z, w0.w), s);
  s = ffma2(make_float2(b.x, b.y), make_float2(w1.x, w1.y), s);
  s = ffma2(make_float2(b.z, b.w), make_float2(w1.z, w1.w), s);
  return s.x + s.y;
}

// tcgen05.ld / wait::ld are warp-collective: every lane of the warp executes
// them in lockstep, and only the memory accesses of rows >= M are skipped.
// Two epilogue warpgroups share a tile: `half` 0 takes the first 128
// columns (or the first head, or gate/up chunks 0-1), `half` 1 the rest.
// xs: this warp's 4 KB shared-memory tile (used by the residual and mHC-write modes).
template <Epi MODE>
LOOP_DEV void epilogue_tile(uint32_t tacc, int row, int n0, int half, const EpiP& p, float* xs) {
  const bool valid = row < p.M;
  if constexpr (MODE == Epi::F32) {
#pragma unroll 1
    for (int c = 4 * half; c < 4 * half + 4; ++c) {
      const int n = n0 + 32 * c;
      if (n >= p.N) break;
      float v[32];
      ld_chunk(tacc + 32 * c, v);
      if (!valid) continue;
      float* dst = p.c + (int64_t)row * p.ldc + n;
      if (n + 32 <= p.N && (p.ldc % 4) == 0) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
          reinterpret_cast<float4*>(dst)[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
      } else {
        for (int j = 0; j < 32 && n + j < p.N; ++j) dst[j] = v[j];
      }
    }
  } else if constexpr (MODE == Epi::RESID || MODE == Epi::MHC_WRITE) {
    // Read-modify-write of fp32 rows (the residual, or both mHC streams).  A
    // thread holds one accumulator row, so the warp first passes each 32 x 32
    // chunk through its shared-memory tile (16-byte slots XOR-swizzled by row,
    // conflict-free both ways); then 8 lanes cover one row's 128 contiguous
    // bytes and every load or store instruction touches 4 rows, not 32.
    const int lane = threadIdx.x & 31;
    const int row0 = row - lane;  // the warp's first row
    float4* xs4 = reinterpret_cast<float4*>(xs);
    const int64_t plane = (int64_t)p.M * p.N;
    // next-site projections: this lane ends with the 9 sums of row 4 (lane & 7)
    // + (lane >> 3) over the warp's 128 columns of both streams
    const bool proj = MODE == Epi::MHC_WRITE && p.pphig != nullptr;
    float pacc[9];
#pragma unroll
    for (int j = 0; j < 9; ++j) pacc[j] = 0.f;
#pragma unroll 1
    for (int c = 4 * half; c < 4 * half + 4; ++c) {
      const int n = n0 + 32 * c;
      float v[32];
      ld_chunk(tacc + 32 * c, v);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        xs4[lane * 8 + (j ^ (lane & 7))] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
      __syncwarp();
      const int col4 = lane & 7;
      float4 y[8], a[8], b[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int rr = 4 * k + (lane >> 3);
        y[k] = xs4[rr * 8 + (col4 ^ (rr & 7))];
        if (row0 + rr < p.M) {
          const int64_t off = (int64_t)(row0 + rr) * p.N + n + 4 * col4;
          if constexpr (MODE == Epi::RESID) {
            a[k] = *reinterpret_cast<const float4*>(p.c + off);
          } else {
            a[k] = __ldcs(reinterpret_cast<const float4*>(p.s + off));
            b[k] = __ldcs(reinterpret_cast<const float4*>(p.s + plane + off));
          }
        } else {
          a[k] = b[k] = make_float4(0.f, 0.f, 0.f, 0.f);  // rows past M add nothing to the projections
        }
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int rr = 4 * k + (lane >> 3);
        if (row0 + rr >= p.M) continue;
        const int64_t off = (int64_t)(row0 + rr) * p.N + n + 4 * col4;
        if constexpr (MODE == Epi::RESID) {
          *reinterpret_cast<float4*>(p.c + off) =
              make_float4(a[k].x + y[k].x, a[k].y + y[k].y, a[k].z + y[k].z, a[k].w + y[k].w);
        } else {
          // (pre0, pre1, post0, post1) and (res00, res01, res10, res11) of the row
          const float4 c0 = __ldg(reinterpret_cast<const float4*>(p.coef + (int64_t)(row0 + rr) * 8));
          const float4 c1 = __ldg(reinterpret_cast<const float4*>(p.coef + (int64_t)(row0 + rr) * 8) + 1);
          float4 x, z;
          x.x = c1.x * a[k].x + c1.y * b[k].x + c0.z * y[k].x;
          x.y = c1.x * a[k].y + c1.y * b[k].y + c0.z * y[k].y;
          x.z = c1.x * a[k].z + c1.y * b[k].z + c0.z * y[k].z;
          x.w = c1.x * a[k].w + c1.y * b[k].w + c0.z * y[k].w;
          z.x = c1.z * a[k].x + c1.w * b[k].x + c0.w * y[k].x;
          z.y = c1.z * a[k].y + c1.w * b[k].y + c0.w * y[k].y;
          z.z = c1.z * a[k].z + c1.w * b[k].z + c0.w * y[k].z;
          z.w = c1.z * a[k].w + c1.w * b[k].w + c0.w * y[k].w;
          *reinterpret_cast<float4*>(p.s + off) = x;
          *reinterpret_cast<float4*>(p.s + plane + off) = z;
          a[k] = x;  // kept for the next site's projections
          b[k] = z;
        }
      }
      if (proj) {
        // sum_i u_i gamma_i Phi_ci over this chunk's 32 columns of both
        // streams (c < 8), and sum_i u_i^2 (c = 8), for each of the lane's 8 rows
        const int col = n + 4 * col4;
#pragma unroll
        for (int j = 0; j < 9; ++j) {
          float r[8];
          const float4 w0 = j < 8 ? __ldg(reinterpret_cast<const float4*>(p.pphig + (int64_t)j * 2 * p.N + col))
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
          const float4 w1 = j < 8 ? __ldg(reinterpret_cast<const float4*>(p.pphig + (int64_t)j * 2 * p.N + p.N + col))
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int k = 0; k < 8; ++k) r[k] = j < 8 ? dot8(a[k], b[k], w0, w1) : dot8(a[k], b[k], a[k], b[k]);
          pacc[j] += reduce_scatter8(r, lane);
        }
      }
      __syncwarp();  // the tile is rewritten by the next chunk
    }
    if (proj) {
      const int prow = row0 + 4 * (lane & 7) + (lane >> 3);
      if (prow < p.M) {
        float* dst = p.ppart + ((int64_t)prow * (2 * p.N / BN) + 2 * (n0 / BN) + half) * 9;
#pragma unroll
        for (int j = 0; j < 9; ++j) dst[j] = pacc[j];
      }
    }
  } else if constexpr (MODE == Epi::SWIGLU) {
    const int F = p.N / 2;
    bf16* dst = p.a + (int64_t)row * F + n0 / 2;
#pragma unroll 1
    for (int c = 2 * half; c < 2 * half + 2; ++c) {
      float g[32], u[32];
      ld_chunk(tacc + 32 * c, g);
      ld_chunk(tacc + 128 + 32 * c, u);
      if (!valid) continue;
#pragma unroll
      for (int j = 0; j < 32; ++j) g[j] = g[j] / (1.f + __expf(-g[j])) * u[j];
      store_bf16x32(dst + 32 * c, g, 1.f);
    }
  } else if constexpr (MODE == Epi::QKV_LINEAR) {
    const int d = 128, nl = p.n_lin;
    const int b = row / p.S, t = row % p.S;
    const int region = n0 / (nl * d);  // 0 q, 1 k, 2 v, 3 gate
    if (region < 3) {
      bf16* base = region == 0 ? p.q : (region == 1 ? p.k : p.v);
      const int head = (n0 - region * nl * d) / d + half;
      bf16* dst = base + (((int64_t)b * nl + head) * p.S + t) * d;
      head_store(tacc + 128 * half, dst, region < 2, p.eps, valid);
    } else if (half == 0) {
      float v[32];
#pragma unroll 1
      for (int c = 0; c * 32 < nl; ++c) {
        ld_chunk(tacc + 32 * c, v);
        if (!valid) continue;
        for (int j = 0; j < 32 && 32 * c + j < nl; ++j) {
          const int head = 32 * c + j;
          const float z = v[j];
          p.gl[((int64_t)b * nl + head) * p.S + t] = z >= 0.f ? -log1pf(__expf(-z)) : z - log1pf(__expf(z));
        }
      }
    }
  } else if constexpr (MODE == Epi::QKV_FULL) {
    const int d = 128;
    const int b = row / p.S, t = row % p.S;
    const int64_t pos = valid ? p.start[b] + t : 0;
    const float2* cs = p.rope + pos * (d / 2);
    {
      const int head = n0 / d + half;
      const uint32_t t0 = tacc + 128 * half;
      if (head < p.hq) {
        head_store_rope(t0, p.q + (((int64_t)b * p.hq + head) * p.S + t) * d, cs, valid);
      } else if (head < p.hq + p.hkv) {
        const int64_t kr = valid ? kv_row(p.table, p.pps, p.hkv, b, head - p.hq, pos) : 0;
        head_store_rope(t0, p.k + kr * d, cs, valid);
      } else {
        const int64_t vr = valid ? kv_row(p.table, p.pps, p.hkv, b, head - p.hq - p.hkv, pos) : 0;
        head_store(t0, p.v + vr * d, false, 0.f, valid);
      }
    }
  }
}

LOOP_DEV void tile_coords(int tile, int num_m, int num_n, int group_m, int& mb, int& nb) {
  const int per_group = group_m * num_n;
  const int g = tile / per_group;
  const int first = g * group_m;
  const int gsz = min(num_m - first, group_m);
  const int r = tile % per_group;
  mb = first + r % gsz;
  nb = r / gsz;
}

template <Epi MODE>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tma, const __grid_constant__ CUtensorMap tmb, int M, int N,
                   int K, EpiP p, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sa = smem;
  uint8_t* sb = smem + STAGES * A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 8);  // one arrival per epilogue warp
    }
    fence_mbar_init();
  }
  if (warp == 2) tmem_alloc(tmem_slot, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int num_m = (M + BM - 1) / BM, num_n = (N + BN - 1) / BN, tiles = num_m * num_n;
  const int kbs = K / BK;

  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tma);
    prefetch_tmap(&tmb);
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
      int mb, nb;
      tile_coords(tile, num_m, num_n, p.group_m, mb, nb);
      for (int kb = 0; kb < kbs; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1, status, STATUS_WAIT_PRODUCER)) { ok = false; break; }
        mbar_expect_tx(&full[stage], STAGE_BYTES);
        tma_load_2d(sa + stage * A_BYTES, &tma, &full[stage], kb * BK, mb * BM);
        tma_load_2d(sb + stage * B_BYTES, &tmb, &full[stage], kb * BK, nb * BN);
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
      }
    }
  } else if (warp == 1 && lane == 0) {
    int stage = 0;
    uint32_t phase = 0;
    int local = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x, ++local) {
      const int acc = local & 1;
      const uint32_t aphase = (local >> 1) & 1;
      if (!mbar_wait(&tempty[acc], aphase ^ 1, status, STATUS_WAIT_MMA)) break;
      tc_fence_after();
      const uint32_t d = tmem + acc * BN;
      for (int kb = 0; kb < kbs; ++kb) {
        if (!mbar_wait(&full[stage], phase, status, STATUS_WAIT_MMA)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a0 = smem_u32(sa + stage * A_BYTES), b0 = smem_u32(sb + stage * B_BYTES);
#pragma unroll
        for (int k = 0; k < BK / 16; ++k) {
          const uint64_t ad = smem_desc_sw128(a0 + 32 * k, 1024);
          const uint64_t bd = smem_desc_sw128(b0 + 32 * k, 1024);
          tc_mma_f16(d, ad, bd, IDESC, (kb | k) != 0);
        }
        tc_commit(&empty[stage]);
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
      }
      if (ok) tc_commit(&tfull[acc]);
    }
  } else if (warp >= 4) {
    const int q = warp & 3;
    int local = 0;
    for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++local) {
      const int acc = local & 1;
      const uint32_t aphase = (local >> 1) & 1;
      int mb, nb;
      tile_coords(tile, num_m, num_n, p.group_m, mb, nb);
      const bool got = mbar_wait(&tfull[acc], aphase, status, STATUS_WAIT_EPILOGUE);
      if (!__all_sync(0xffffffffu, got)) break;  // the whole warp leaves together
      tc_fence_after();
      const uint32_t tacc = tmem + acc * BN + ((uint32_t)(32 * q) << 16);
      epilogue_tile<MODE>(tacc, mb * BM + 32 * q + lane, nb * BN, (warp - 4) >> 2, p,
                          reinterpret_cast<float*>(smem + EPI_OFF) + (warp - 4) * 1024);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Skinny GEMM for decode (M <= 64 tokens): the weight is the streamed operand.
// Swap-AB so the weight rows fill the M = 128 side of tcgen05.mma and the
// tokens are N = 64.  Work items are (128-row weight tile, slice of K)
// (split-K, so even N = 4096 keeps every SM streaming weights); a persistent
// CTA per SM walks its items with the TMA ring and two TMEM accumulators
// carried across items, so the epilogue of one item overlaps the next.
// Output: fp32 partial sums P[split][token][n] (row stride ldp), reduced by
// the epilogue kernels.
// ---------------------------------------------------------------------------
constexpr int SK_BN = 64, SK_BK = 128, SK_STAGES = 4;
constexpr int SK_A_BYTES = BM * SK_BK * 2;     // weight tile 128 x 128: two 64-column boxes
constexpr int SK_B_BYTES = SK_BN * SK_BK * 2;  // token tile 64 x 128: two 64-column boxes
constexpr int SK_STAGE = SK_A_BYTES + SK_B_BYTES;
constexpr int SK_SMEM = SK_STAGES * SK_STAGE + 1024 + 256;
static_assert(SK_SMEM <= 232448, "shared memory per block");
constexpr uint32_t SK_IDESC = idesc_bf16_f32(BM, SK_BN);

__global__ void __launch_bounds__(THREADS, 1)
    gemm_skinny_kernel(const __grid_constant__ CUtensorMap tmw, const __grid_constant__ CUtensorMap tmx, int M, int N,
                       int K, int splits, float* __restrict__ P, int64_t ldp, int* status) {
  // persistent: CTA b takes items b, b + grid, ...; item = (split, weight tile)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sw_ = smem;
  uint8_t* sx = smem + SK_STAGES * SK_A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + SK_STAGES * SK_STAGE);
  uint64_t* empty = full + SK_STAGES;
  uint64_t* tfull = empty + SK_STAGES;  // 2 accumulators
  uint64_t* tempty = tfull + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles = (N + BM - 1) / BM, items = tiles * splits;
  const int kbs = K / SK_BK;
  if (threadIdx.x == 0) {
    for (int s = 0; s < SK_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);
    }
    fence_mbar_init();
  }
  if (warp == 2) tmem_alloc(tmem_slot, 2 * SK_BN);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmw);
    prefetch_tmap(&tmx);
    auto load_w = [&](int stage, int kb, int tile) {
      tma_load_2d(sw_ + stage * SK_A_BYTES, &tmw, &full[stage], kb * SK_BK, tile * BM);
      tma_load_2d(sw_ + stage * SK_A_BYTES + SK_A_BYTES / 2, &tmw, &full[stage], kb * SK_BK + 64, tile * BM);
    };
    auto load_x = [&](int stage, int kb) {
      tma_load_2d(sx + stage * SK_B_BYTES, &tmx, &full[stage], kb * SK_BK, 0);
      tma_load_2d(sx + stage * SK_B_BYTES + SK_B_BYTES / 2, &tmx, &full[stage], kb * SK_BK + 64, 0);
    };
    // The weights do not depend on the kernels before this one: the first
    // ring's worth of weight tiles is requested before waiting for them, the
    // token tiles of those stages after.
    int npre = 0, pre_kb[SK_STAGES];
    for (int it = blockIdx.x; it < items && npre < SK_STAGES; it += gridDim.x) {
      const int split = it / tiles, tile = it % tiles;
      const int kb0 = (int)((int64_t)kbs * split / splits), kb1 = (int)((int64_t)kbs * (split + 1) / splits);
      for (int kb = kb0; kb < kb1 && npre < SK_STAGES; ++kb) {
        mbar_expect_tx(&full[npre], SK_STAGE);
        load_w(npre, kb, tile);
        pre_kb[npre++] = kb;
      }
    }
    griddep_wait();
    for (int i = 0; i < npre; ++i) load_x(i, pre_kb[i]);
    int stage = npre % SK_STAGES;
    uint32_t phase = npre == SK_STAGES ? 1u : 0u;
    bool ok = true;
    int idx = 0;
    for (int it = blockIdx.x; it < items && ok; it += gridDim.x) {
      const int split = it / tiles, tile = it % tiles;
      const int kb0 = (int)((int64_t)kbs * split / splits), kb1 = (int)((int64_t)kbs * (split + 1) / splits);
      for (int kb = kb0; kb < kb1; ++kb, ++idx) {
        if (idx < npre) continue;  // requested above
        if (!mbar_wait(&empty[stage], phase ^ 1, status, STATUS_WAIT_PRODUCER)) { ok = false; break; }
        mbar_expect_tx(&full[stage], SK_STAGE);
        load_w(stage, kb, tile);
        load_x(stage, kb);
        if (++stage == SK_STAGES) { stage = 0; phase ^= 1; }
      }
    }
  } else if (warp == 1 && lane == 0) {
    int stage = 0;
    uint32_t phase = 0;
    int local = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < items && ok; it += gridDim.x, ++local) {
      const int split = it / tiles;
      const int kb0 = (int)((int64_t)kbs * split / splits), kb1 = (int)((int64_t)kbs * (split + 1) / splits);
      const int acc = local & 1;
      if (!mbar_wait(&tempty[acc], ((local >> 1) & 1) ^ 1, status, STATUS_WAIT_MMA)) break;
      tc_fence_after();
      const uint32_t d = tmem + acc * SK_BN;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(&full[stage], phase, status, STATUS_WAIT_MMA)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a0 = smem_u32(sw_ + stage * SK_A_BYTES), b0 = smem_u32(sx + stage * SK_B_BYTES);
#pragma unroll
        for (int k = 0; k < SK_BK / 16; ++k) {
          const uint32_t ka = (uint32_t)((k >> 2) * (SK_A_BYTES / 2) + (k & 3) * 32);
          const uint32_t kx = (uint32_t)((k >> 2) * (SK_B_BYTES / 2) + (k & 3) * 32);
          tc_mma_f16(d, smem_desc_sw128(a0 + ka, 1024), smem_desc_sw128(b0 + kx, 1024), SK_IDESC,
                     (kb > kb0 || k > 0) ? 1u : 0u);
        }
        tc_commit(&empty[stage]);
        if (++stage == SK_STAGES) { stage = 0; phase ^= 1; }
      }
      if (ok) tc_commit(&tfull[acc]);
    }
  } else if (warp >= 4) {
    const int q = warp & 3;
    int local = 0;
    griddep_wait();  // the partials may still be read by the kernel before this one
    for (int it = blockIdx.x; it < items; it += gridDim.x, ++local) {
      const int split = it / tiles, tile = it % tiles;
      const int acc = local & 1;
      const bool got = mbar_wait(&tfull[acc], (local >> 1) & 1, status, STATUS_WAIT_EPILOGUE);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const int n = tile * BM + 32 * q + lane;
      float* dst = P + (int64_t)split * M * ldp + n;
#pragma unroll 1
      for (int c = 0; c < SK_BN / 32; ++c) {
        float v[32];
        ld_chunk(tmem + acc * SK_BN + ((uint32_t)(32 * q) << 16) + 32 * c, v);
        if (n < N) {
          for (int j = 0; j < 32 && 32 * c + j < M; ++j) dst[(int64_t)(32 * c + j) * ldp] = v[j];
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * SK_BN);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

// 2-D bf16 tensor map over a row-major [rows][K] matrix, box 64 x box_rows,
// 128-byte swizzle; rows past the end read as zeros.
bool make_map(CUtensorMap* map, const void* ptr, int64_t rows, int64_t K, int box_rows) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int num_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

template <Epi MODE>
cudaError_t launch_mode(const CUtensorMap& ma, const CUtensorMap& mb, int M, int N, int K, const EpiP& p,
                        cudaStream_t st) {
  static std::atomic<uint64_t> smem_set{0};
  if (cudaError_t e = set_smem_limit(gemm_tc_kernel<MODE>, SMEM_BYTES, smem_set); e != cudaSuccess) return e;
  const int tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
  const int grid = std::min(tiles, num_sms());
  gemm_tc_kernel<MODE><<<grid, GEMM_THREADS, SMEM_BYTES, st>>>(ma, mb, M, N, K, p, status_ptr());
  return cudaGetLastError();
}

}  // namespace

bool gemm_skinny_supported(int64_t M, int64_t N, int64_t K) { return M >= 1 && M <= SK_BN && K % SK_BK == 0 && N > 0; }

int gemm_skinny_splits(int64_t N, int64_t K) {
  // split-K count minimising the busiest CTA's work: items per CTA times
  // (weight k-blocks per item + ~4 k-block equivalents of fp32 partials
  // written and read back per item)
  const int64_t tiles = (N + BM - 1) / BM, kbs = K / SK_BK, sms = num_sms();
  int best = 1;
  double best_cost = (double)((tiles + sms - 1) / sms) * (double)kbs;  // one split writes no partials
  for (int s = 2; s <= 16 && s <= kbs; ++s) {
    const double cost = (double)((tiles * s + sms - 1) / sms) * ((double)kbs / s + 2.0);
    if (cost < best_cost * 0.97) {
      best_cost = cost;
      best = s;
    }
  }
  return best;
}

cudaError_t launch_gemm_skinny(const void* X, const void* W, int64_t M, int64_t N, int64_t K, int splits, float* P,
                               int64_t ldp, cudaStream_t st) {
  if (!gemm_skinny_supported(M, N, K) || splits < 1) return cudaErrorNotSupported;
  CUtensorMap mw, mx;
  if (!make_map(&mw, W, N, K, BM) || !make_map(&mx, X, M, K, SK_BN)) return cudaErrorInvalidValue;
  static std::atomic<uint64_t> smem_set{0};
  if (cudaError_t e = set_smem_limit(gemm_skinny_kernel, SK_SMEM, smem_set); e != cudaSuccess) return e;
  const int items = (int)((N + BM - 1) / BM) * splits;
  // programmatic dependent launch: the CTAs start (barriers, TMEM, the first
  // weight tiles) while the kernel before them finishes
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)std::min(items, num_sms()));
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = SK_SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemm_skinny_kernel, mw, mx, (int)M, (int)N, (int)K, splits, P, ldp, status_ptr());
}

bool gemm_tc_supported(int64_t M, int64_t N, int64_t K, const EpiArgs& e) {
  if (M <= 0 || K % BK != 0 || M > (int64_t)1 << 30 || N > (int64_t)1 << 30) return false;
  switch (e.mode) {
    case Epi::F32: return true;
    case Epi::RESID:
    case Epi::MHC_WRITE: return N % BN == 0;
    case Epi::SWIGLU: return N % BN == 0;
    case Epi::QKV_LINEAR: return e.hd == 128 && ((int64_t)e.n_lin * 128) % BN == 0 && e.n_lin <= BN;
    case Epi::QKV_FULL: return e.hd == 128 && N % BN == 0 && ((int64_t)e.heads_q * 128) % BN == 0 &&
                               ((int64_t)e.heads_kv * 128) % BN == 0;
  }
  return false;
}

cudaError_t launch_gemm_tc(const void* A, const void* W, int64_t M, int64_t N, int64_t K, const EpiArgs& e,
                           cudaStream_t st) {
  if (!gemm_tc_supported(M, N, K, e)) return cudaErrorNotSupported;
  CUtensorMap ma, mb;
  if (!make_map(&ma, A, M, K, BM) || !make_map(&mb, W, N, K, BN)) return cudaErrorInvalidValue;
  EpiP p{};
  p.M = (int)M;
  p.N = (int)N;
  p.group_m = K <= 4096 ? GROUP_M_SMALL_K : GROUP_M_LARGE_K;
  p.c = e.c;
  p.ldc = e.ldc;
  p.s = e.s;
  p.coef = e.coef;
  p.a = (bf16*)e.a;
  p.q = (bf16*)e.q;
  p.k = (bf16*)e.k;
  p.v = (bf16*)e.v;
  p.gl = e.gl;
  p.rope = e.rope;
  p.start = e.start;
  p.S = e.S;
  p.hq = e.heads_q;
  p.hkv = e.heads_kv;
  p.n_lin = e.n_lin;
  p.table = e.table;
  p.pps = e.pps;
  p.eps = e.eps;
  p.pphig = e.next_phig;
  p.ppart = e.part;
  switch (e.mode) {
    case Epi::F32: return launch_mode<Epi::F32>(ma, mb, (int)M, (int)N, (int)K, p, st);
    case Epi::RESID: return launch_mode<Epi::RESID>(ma, mb, (int)M, (int)N, (int)K, p, st);
    case Epi::MHC_WRITE: return launch_mode<Epi::MHC_WRITE>(ma, mb, (int)M, (int)N, (int)K, p, st);
    case Epi::SWIGLU: return launch_mode<Epi::SWIGLU>(ma, mb, (int)M, (int)N, (int)K, p, st);
    case Epi::QKV_LINEAR: return launch_mode<Epi::QKV_LINEAR>(ma, mb, (int)M, (int)N, (int)K, p, st);
    case Epi::QKV_FULL: return launch_mode<Epi::QKV_FULL>(ma, mb, (int)M, (int)N, (int)K, p, st);
  }
  return cudaErrorNotSupported;
}

}  // namespace loopk
