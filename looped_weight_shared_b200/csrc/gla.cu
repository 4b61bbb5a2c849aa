// Gated linear attention: the chunked prefill on the 5th-generation tensor
// cores (tcgen05) and the one-token decode step.
//
// The layer (one of the 3 linear-attention layers of every 4-layer group,
// "How Does SenseNova-Loop Get More Depth Without More Parameters?", section
// "How does the hybrid attention pattern work?") keeps a fixed-size state per
// head: S_t = g_t S_{t-1} + k_t v_t^T, o_t = q_t S_t.  Over a tile of T
// tokens with b_t the running sum of log g inside the tile this is exactly
//   O  = diag(exp b) Q S_prev + ((Q K^T) * D) V,   D_ts = exp(b_t - b_s) [s <= t]
//   S' = exp(b_last) S_prev + K^T (diag(exp(b_last - b)) V).
// The prefill kernel takes T = 128: two of the pages' 64-token chunks, whose
// joint intra-tile block is the same sum computed in one product (the
// chunked form is exact for any chunk length), so every product is a full
// M = 128 tensor-core tile.
//
// One CTA per (sequence, head) walks the tiles in order (18 warps):
//   warp 0      TMA producer: Q, K and V of the tile ([128][128] bf16 each,
//               two 64-column boxes, 128-byte swizzle), each refilled as soon
//               as the products that read it are done;
//   warp 1      allocates / frees the 512 TMEM columns; one thread issues
//               the tcgen05.mma products:
//                 P   = Q K^T                       (TMEM, fp32)
//                 O_x = Q S_prev                    (S as bf16 hi + lo, MN-major)
//                 R  += K^T V^                      (K read MN-major as A)
//                 O_a = A V                         (A from TMEM, hi + lo)
//               where R is the fp32 state, resident in TMEM for the whole
//               sequence;
//   warps 2-17  each owns one TMEM lane quarter (warp % 4) and a quarter
//               of the 128 columns (so each step of the per-tile chain below
//               is split 16 ways): the decayed scores A = P * D written back
//               over P as bf16 hi + lo (the A operand of O_a), V^ = diag(exp(
//               b_last - b)) V as hi + lo in shared memory, the state step
//               (R -> S_prev hi + lo in shared memory, R *= exp(b_last)), and
//               the output exp(b_t) O_x + O_a.
// The three operands that are not model activations (the state, the decayed
// scores and the decayed values) enter their products as bf16 hi + lo pairs
// (~16 significant bits), so the chunked form keeps the accuracy of the
// token-by-token recurrence.  Every mbarrier wait gives up after ~2 s and
// flags the status word.

#include <cuda.h>

#include <algorithm>

#include "model.h"

namespace loopk {

namespace {

constexpr int DK = 128;
constexpr int CT = 128;                       // tokens per tile
constexpr int TILE = CT * 128 * 2;            // one [128][128] bf16 operand: two boxes [128][64]
constexpr int THREADS = 576;  // producer, MMA issuer + TMEM allocator, 16 epilogue warps
constexpr int OFF_Q = 0, OFF_K = TILE, OFF_V = 2 * TILE, OFF_SHI = 3 * TILE, OFF_SLO = 4 * TILE,
              OFF_VHI = 5 * TILE, OFF_VLO = 6 * TILE, OFF_B2 = 7 * TILE;
constexpr int NB2 = 3;                        // gate buffers (tiles t, t + 1 and one in flight)
enum { B_QF, B_KF, B_VF, B_QE, B_KE, B_VE, B_PF, B_DS, B_OF, B_GR, B_SR, B_VR, B_AR, B_OE, NBARS };
constexpr int OFF_BAR = OFF_B2 + NB2 * CT * 4;
constexpr int SMEM = OFF_BAR + NBARS * 8 + 16 + 1024;
static_assert(SMEM <= 232448, "shared memory per block");
// TMEM columns: state R, scores P (then A), inter-tile O_x, intra-tile O_a
constexpr uint32_t T_R = 0, T_P = 128, T_OX = 256, T_OA = 384;
constexpr uint32_t ID_KK = idesc_bf16_f32(128, 128);               // A, B K-major
constexpr uint32_t ID_KM = idesc_bf16_f32(128, 128, true);         // B MN-major
constexpr uint32_t ID_MM = idesc_bf16_f32(128, 128, true, true);   // A, B MN-major
constexpr float LOG2E = 1.4426950408889634f;

// K-major descriptor of a [128][128] operand, k-step kk (16 columns)
LOOP_DEV uint64_t kdesc(uint32_t base, int kk) {
  return smem_desc_sw128(base + (uint32_t)((kk >> 2) * CT * 128 + (kk & 3) * 32), 1024);
}
// MN-major descriptor of a [128 k][128 mn] operand, k-step kk (16 rows)
LOOP_DEV uint64_t mdesc(uint32_t base, int kk) { return smem_desc_sw128_lbo(base + (uint32_t)kk * 2048, TILE / 2, 1024); }
// TMEM column of the A hi part for k-step kk: each 32-column group of P holds
// the hi pairs of its 32 keys in its first 16 columns and the lo pairs after
LOOP_DEV uint32_t a_col(int kk) { return (uint32_t)(32 * (kk >> 1) + 8 * (kk & 1)); }

LOOP_DEV void split_pack(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  const float2 hf = __bfloat1622float2(h);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = pack_bf16x2(x0 - hf.x, x1 - hf.y);
}

__global__ void __launch_bounds__(THREADS, 1)
    gla_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                  const __grid_constant__ CUtensorMap tv, const float* __restrict__ gl,
                  const float* __restrict__ init_state, float* __restrict__ seg_states,
                  float* __restrict__ final_state, bf16* __restrict__ out, int S, int nh, int nseg, int seg_tiles,
                  int pass, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* b2s = reinterpret_cast<float*>(smem + OFF_B2);  // [NB2][CT] running log2 gates
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + NBARS);

  const int h = blockIdx.x, b = blockIdx.y, seg = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // this CTA's segment: tokens t0 .. t0 + Sl - 1 of the sequence, walked as a
  // sequence of its own from the segment's start state
  const int t0 = seg * seg_tiles * CT;
  const int Sl = min(S - t0, seg_tiles * CT);
  const int nch = (Sl + CT - 1) / CT;
  const int row0 = (b * nh + h) * S + t0;  // first row of this segment in the [B nh S][128] views
  const int64_t bh = (int64_t)b * nh + h;
  // start state (NULL: zero) and where the end state goes (NULL: nowhere).
  // One segment: init_state to final_state.  Several (seg_states holds nseg
  // states per head): pass 1 runs segments 0 .. nseg - 2 from zero and leaves
  // segment p's local end state in slot p + 1; gla_scan_kernel turns slot p
  // into the true start state of segment p; pass 2 runs every segment from its
  // slot and the last one writes final_state.
  const float* s_in = nullptr;
  float* s_out = nullptr;
  if (nseg == 1) {
    s_in = init_state + bh * DK * 128;
    s_out = final_state + bh * DK * 128;
  } else if (pass == 1) {
    s_out = seg_states + (bh * nseg + seg + 1) * (int64_t)DK * 128;
  } else {
    s_in = seg_states + (bh * nseg + seg) * (int64_t)DK * 128;
    if (seg == nseg - 1) s_out = final_state + bh * DK * 128;
  }

  if (threadIdx.x == 0) {
    for (int i = 0; i < NBARS; ++i) mbar_init(&bar[i], i >= B_SR ? 16u : 1u);
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t su = smem_u32(smem);

  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tq);
    prefetch_tmap(&tk);
    prefetch_tmap(&tv);
    const CUtensorMap* maps[3] = {&tq, &tk, &tv};
    for (int c = 0; c < nch; ++c) {
      const int row = row0 + c * CT;
      bool ok = true;
      for (int o = 0; o < 3 && ok; ++o) {  // Q, K, V in the order the products release them
        if (c > 0 && !mbar_wait(&bar[B_QE + o], (c - 1) & 1, status, STATUS_WAIT_PRODUCER)) { ok = false; break; }
        uint8_t* dst = smem + o * TILE;
        mbar_expect_tx(&bar[B_QF + o], TILE);
        tma_load_2d(dst, maps[o], &bar[B_QF + o], 0, row);
        tma_load_2d(dst + TILE / 2, maps[o], &bar[B_QF + o], 64, row);
      }
      if (!ok) break;
    }
  } else if (warp == 1 && lane == 0) {
    auto scores = [&]() {
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) tc_mma_f16(tmem + T_P, kdesc(su + OFF_Q, kk), kdesc(su + OFF_K, kk), ID_KK, kk > 0);
      tc_commit(&bar[B_PF]);
    };
    bool ok = mbar_wait(&bar[B_QF], 0, status, STATUS_WAIT_MMA) && mbar_wait(&bar[B_KF], 0, status, STATUS_WAIT_MMA);
    if (ok) {
      tc_fence_after();
      scores();
    }
    for (int c = 0; c < nch && ok; ++c) {
      const uint32_t par = c & 1;
      // O_x = Q S_prev once the state step has written S_prev and the last
      // tile's outputs have been read
      ok = mbar_wait(&bar[B_SR], par, status, STATUS_WAIT_MMA) &&
           (c == 0 || mbar_wait(&bar[B_OE], (c - 1) & 1, status, STATUS_WAIT_MMA));
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) tc_mma_f16(tmem + T_OX, kdesc(su + OFF_Q, kk), mdesc(su + OFF_SHI, kk), ID_KM, kk > 0);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) tc_mma_f16(tmem + T_OX, kdesc(su + OFF_Q, kk), mdesc(su + OFF_SLO, kk), ID_KM, 1u);
      tc_commit(&bar[B_QE]);
      // R += K^T V^
      if (!mbar_wait(&bar[B_VR], par, status, STATUS_WAIT_MMA)) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) tc_mma_f16(tmem + T_R, mdesc(su + OFF_K, kk), mdesc(su + OFF_VHI, kk), ID_MM, 1u);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) tc_mma_f16(tmem + T_R, mdesc(su + OFF_K, kk), mdesc(su + OFF_VLO, kk), ID_MM, 1u);
      tc_commit(&bar[B_DS]);
      tc_commit(&bar[B_KE]);
      // O_a = A V, A from TMEM
      ok = mbar_wait(&bar[B_AR], par, status, STATUS_WAIT_MMA) && mbar_wait(&bar[B_VF], par, status, STATUS_WAIT_MMA);
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) tc_mma_f16_ts(tmem + T_OA, tmem + T_P + a_col(kk), mdesc(su + OFF_V, kk), ID_KM, kk > 0);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) tc_mma_f16_ts(tmem + T_OA, tmem + T_P + a_col(kk) + 16, mdesc(su + OFF_V, kk), ID_KM, 1u);
      tc_commit(&bar[B_OF]);
      tc_commit(&bar[B_VE]);
      if (c + 1 < nch) {
        // the next scores overwrite A: wait for this tile's products first
        ok = mbar_wait(&bar[B_OF], par, status, STATUS_WAIT_MMA) &&
             mbar_wait(&bar[B_QF], (c + 1) & 1, status, STATUS_WAIT_MMA) &&
             mbar_wait(&bar[B_KF], (c + 1) & 1, status, STATUS_WAIT_MMA);
        if (!ok) break;
        tc_fence_after();
        scores();
      }
    }
  } else if (warp >= 2) {
    const int ew = warp - 2;
    const int quarter = warp & 3;     // TMEM lanes 32 quarter .. (fixed by the warp's rank)
    const int cb = 32 * (ew >> 2);    // this warp's 32 columns
    const int r = 32 * quarter + lane;  // the row this thread owns: token t, key s or state row
    const uint32_t lo_lane = (uint32_t)(32 * quarter) << 16;
    const float* glh = gl + bh * S + t0;
    bool ok = true;

    // running sums of the log gates of tile j, in log2 units (0 past the end)
    auto gates = [&](int j) -> bool {
      if (ew != 0) return true;
      if (j >= 1 && !__all_sync(0xffffffffu, mbar_wait(&bar[B_SR], (j - 1) & 1, status, STATUS_WAIT_EPILOGUE)))
        return false;  // every warp has read the gate buffer this one reuses
      const int c0 = j * CT, valid = min(CT, Sl - c0);
      float x[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) x[i] = 4 * lane + i < valid ? glh[c0 + 4 * lane + i] : 0.f;
      x[1] += x[0];
      x[2] += x[1];
      x[3] += x[2];
      float inc = x[3];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
      }
      const float ex = inc - x[3];
      float* dst = b2s + (j % NB2) * CT + 4 * lane;
#pragma unroll
      for (int i = 0; i < 4; ++i) dst[i] = (ex + x[i]) * LOG2E;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[B_GR]);
      return true;
    };
    // state step for tile j: S_prev = R (the initial state for j = 0) into
    // shared memory as hi + lo, then R = exp(b_last) S_prev
    auto state_step = [&](int j) -> bool {
      if (!__all_sync(0xffffffffu, mbar_wait(&bar[B_GR], j & 1, status, STATUS_WAIT_EPILOGUE))) return false;
      if (j >= 1) {
        if (!__all_sync(0xffffffffu, mbar_wait(&bar[B_DS], (j - 1) & 1, status, STATUS_WAIT_EPILOGUE))) return false;
        tc_fence_after();
      }
      const float dl = ex2(b2s[(j % NB2) * CT + CT - 1]);
      const float* src = s_in ? s_in + r * 128 : nullptr;
      {  // this thread's 32 columns
        const int col = cb;
        float s[32];
        if (j == 0) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 v = src ? reinterpret_cast<const float4*>(src + col)[i] : make_float4(0.f, 0.f, 0.f, 0.f);
            s[4 * i] = v.x;
            s[4 * i + 1] = v.y;
            s[4 * i + 2] = v.z;
            s[4 * i + 3] = v.w;
          }
        } else {
          tmem_ld32(tmem + T_R + lo_lane + col, s);
          tc_wait_ld();
        }
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint4 hi, lo;
          split_pack(s[8 * ch], s[8 * ch + 1], hi.x, lo.x);
          split_pack(s[8 * ch + 2], s[8 * ch + 3], hi.y, lo.y);
          split_pack(s[8 * ch + 4], s[8 * ch + 5], hi.z, lo.z);
          split_pack(s[8 * ch + 6], s[8 * ch + 7], hi.w, lo.w);
          const uint32_t off = sw(r, col / 8 + ch, CT);
          *reinterpret_cast<uint4*>(smem + OFF_SHI + off) = hi;
          *reinterpret_cast<uint4*>(smem + OFF_SLO + off) = lo;
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) s[i] *= dl;
        tmem_st32(tmem + T_R + lo_lane + col, s);
      }
      tc_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[B_SR]);
      return true;
    };
    // the final state of the sequence back to global memory
    auto state_out = [&](int last) -> bool {
      if (!s_out) return true;
      if (!__all_sync(0xffffffffu, mbar_wait(&bar[B_DS], last & 1, status, STATUS_WAIT_EPILOGUE))) return false;
      tc_fence_after();
      float* dst = s_out + r * 128;
      {  // this thread's 32 columns
        const int col = cb;
        float s[32];
        tmem_ld32(tmem + T_R + lo_lane + col, s);
        tc_wait_ld();
#pragma unroll
        for (int i = 0; i < 8; ++i)
          reinterpret_cast<float4*>(dst + col)[i] = make_float4(s[4 * i], s[4 * i + 1], s[4 * i + 2], s[4 * i + 3]);
      }
      return true;
    };
    // V^ = diag(exp(b_last - b)) V as hi + lo, zero past the end of the sequence
    auto vhat = [&](int j) -> bool {
      if (!__all_sync(0xffffffffu, mbar_wait(&bar[B_VF], j & 1, status, STATUS_WAIT_EPILOGUE))) return false;
      const float* bb = b2s + (j % NB2) * CT;
      const int valid = min(CT, Sl - j * CT);
      const float w = r < valid ? ex2(bb[CT - 1] - bb[r]) : 0.f;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        const uint32_t off = sw(r, cb / 8 + ch, CT);
        const uint4 u = *reinterpret_cast<const uint4*>(smem + OFF_V + off);
        const uint32_t in[4] = {u.x, u.y, u.z, u.w};
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&in[e]));
          split_pack(x.x * w, x.y * w, hi[e], lo[e]);
        }
        *reinterpret_cast<uint4*>(smem + OFF_VHI + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(smem + OFF_VLO + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[B_VR]);
      return true;
    };
    // A = (Q K^T) * D over P, as bf16 hi + lo pairs (row t = r, keys cb ..)
    auto decayed_scores = [&](int j) -> bool {
      if (!__all_sync(0xffffffffu, mbar_wait(&bar[B_PF], j & 1, status, STATUS_WAIT_EPILOGUE))) return false;
      tc_fence_after();
      const float* bb = b2s + (j % NB2) * CT;
      const int valid = min(CT, Sl - j * CT);
      const float bt = bb[r];
      const bool row_ok = r < valid;
      {  // this thread's 32 keys
        const int col = cb;
        float p[32];
        tmem_ld32(tmem + T_P + lo_lane + col, p);
        tc_wait_ld();
        uint32_t hi[16], lo[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int s0 = col + 2 * i;
          const float x0 = (row_ok && s0 <= r) ? p[2 * i] * ex2(bt - bb[s0]) : 0.f;
          const float x1 = (row_ok && s0 + 1 <= r) ? p[2 * i + 1] * ex2(bt - bb[s0 + 1]) : 0.f;
          split_pack(x0, x1, hi[i], lo[i]);
        }
        tmem_st16(tmem + T_P + lo_lane + col, hi);
        tmem_st16(tmem + T_P + lo_lane + col + 16, lo);
      }
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[B_AR]);
      return true;
    };
    // o_t = exp(b_t) O_x + O_a for the valid rows of tile c
    auto output = [&](int c) -> bool {
      if (!__all_sync(0xffffffffu, mbar_wait(&bar[B_OF], c & 1, status, STATUS_WAIT_EPILOGUE))) return false;
      tc_fence_after();
      const int c0 = c * CT, valid = min(CT, Sl - c0);
      const float et = ex2(b2s[(c % NB2) * CT + r]);
      bf16* dst = out + ((int64_t)b * S + t0 + c0 + r) * ((int64_t)nh * 128) + h * 128;
      {  // this thread's 32 columns
        const int col = cb;
        float x[32], a[32];
        tmem_ld32(tmem + T_OX + lo_lane + col, x);
        tmem_ld32(tmem + T_OA + lo_lane + col, a);
        tc_wait_ld();
        if (r < valid) {
#pragma unroll
          for (int i = 0; i < 32; ++i) x[i] = fmaf(et, x[i], a[i]);
          uint4* d4 = reinterpret_cast<uint4*>(dst + col);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            d4[i] = make_uint4(pack_bf16x2(x[8 * i], x[8 * i + 1]), pack_bf16x2(x[8 * i + 2], x[8 * i + 3]),
                               pack_bf16x2(x[8 * i + 4], x[8 * i + 5]), pack_bf16x2(x[8 * i + 6], x[8 * i + 7]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[B_OE]);
      return true;
    };

    ok = gates(0) && state_step(0) && vhat(0) && decayed_scores(0);
    for (int c = 0; c < nch && ok; ++c) {
      if (c + 1 < nch)
        ok = gates(c + 1) && state_step(c + 1);
      else
        ok = state_out(c);
      ok = ok && output(c);
      if (ok && c + 1 < nch) ok = vhat(c + 1) && decayed_scores(c + 1);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// The chaining step between the two passes of a segmented prefill, one CTA
// per (sequence, head): slot 0 = the initial state, then for p = 1 .. nseg - 1
//   slot p = G_{p-1} slot (p - 1) + slot p,  G_{p-1} = exp(sum of log g over
// segment p - 1), where slot p held segment p - 1's local end state (its
// state from zero).  This is the recurrence S_t = g_t S_{t-1} + k_t v_t^T
// taken a segment at a time.  The gate sums are accumulated in fp64.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
    gla_scan_kernel(const float* __restrict__ gl, const float* __restrict__ init_state,
                    float* __restrict__ seg_states, int S, int nseg, int seg_tokens) {
  __shared__ double red[8];
  const int64_t bh = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  float* base = seg_states + bh * nseg * (int64_t)DK * 128;
  const float* init = init_state ? init_state + bh * DK * 128 : nullptr;
  float cur[64];  // this thread's 64 state entries of the current slot
#pragma unroll
  for (int i = 0; i < 64; ++i) {
    const int e = i * 256 + tid;
    cur[i] = init ? init[e] : 0.f;
    base[e] = cur[i];
  }
  for (int p = 1; p < nseg; ++p) {
    const float* g = gl + bh * S + (int64_t)(p - 1) * seg_tokens;
    double acc = 0.0;
    for (int t = tid; t < seg_tokens; t += 256) acc += (double)g[t];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) red[wid] = acc;
    __syncthreads();
    double tot = 0.0;
#pragma unroll
    for (int w = 0; w < 8; ++w) tot += red[w];
    __syncthreads();
    const float decay = (float)exp(tot);
    float* slot = base + (int64_t)p * DK * 128;
#pragma unroll
    for (int i = 0; i < 64; ++i) {
      const int e = i * 256 + tid;
      cur[i] = fmaf(decay, cur[i], slot[e]);
      slot[e] = cur[i];
    }
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
  griddep_launch_dependents();  // the output projection after this may start streaming its weights
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
// seg_scratch (may be NULL) holds scratch_floats floats; with room, a batch
// with fewer (sequence, head) pairs than SMs is cut into segments of whole
// tiles so the segments run in parallel (two passes and a scan).
cudaError_t launch_gla_chunked(const void* q, const void* k, const void* v, const float* gl, float* state, void* o,
                               int B, int S, int nh, float* seg_scratch, int64_t scratch_floats, cudaStream_t st) {
  if (B == 0 || S == 0) return cudaSuccess;
  CUtensorMap mq, mk, mv;
  const int64_t rows = (int64_t)B * nh * S;
  if (!map_rows128(&mq, q, rows, CT) || !map_rows128(&mk, k, rows, CT) || !map_rows128(&mv, v, rows, CT))
    return cudaErrorInvalidValue;
  static std::atomic<uint64_t> smem_set{0};
  if (cudaError_t e = set_smem_limit(gla_tc_kernel, SMEM, smem_set); e != cudaSuccess) return e;
  const int nch = (S + CT - 1) / CT;
  int nseg = 1;
  if (seg_scratch) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int pairs = B * nh;
    nseg = std::max(1, std::min(sms / std::max(pairs, 1), nch / 8));  // at least 8 tiles a segment
    while (nseg > 1 && (int64_t)pairs * nseg * DK * 128 > scratch_floats) --nseg;
  }
  const int seg_tiles = (nch + nseg - 1) / nseg;
  nseg = (nch + seg_tiles - 1) / seg_tiles;  // no empty segment
  int* status = status_ptr();
  if (nseg == 1) {
    gla_tc_kernel<<<dim3((unsigned)nh, (unsigned)B, 1), THREADS, SMEM, st>>>(
        mq, mk, mv, gl, state, nullptr, state, (bf16*)o, S, nh, 1, seg_tiles, 2, status);
    return cudaGetLastError();
  }
  gla_tc_kernel<<<dim3((unsigned)nh, (unsigned)B, (unsigned)(nseg - 1)), THREADS, SMEM, st>>>(
      mq, mk, mv, gl, nullptr, seg_scratch, nullptr, (bf16*)o, S, nh, nseg, seg_tiles, 1, status);
  gla_scan_kernel<<<(unsigned)(B * nh), 256, 0, st>>>(gl, state, seg_scratch, S, nseg, seg_tiles * CT);
  gla_tc_kernel<<<dim3((unsigned)nh, (unsigned)B, (unsigned)nseg), THREADS, SMEM, st>>>(
      mq, mk, mv, gl, nullptr, seg_scratch, state, (bf16*)o, S, nh, nseg, seg_tiles, 2, status);
  return cudaGetLastError();
}

}  // namespace loopk
