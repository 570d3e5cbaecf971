// tc_linear.cuh - tensor-core (tcgen05) kernel of TTT-Linear and TTT-Linear +
// LN + residual for bf16 Q, K, V, d = 64, b = 16.
//
// Method: the dual form of the TTT write-up (§03.7) over mini-batches of b = 16
// tokens (§03.6), f(x) = x W or x + LN(x W) (§03.9), loss ||f(k; W) - v||^2
// (§03.5).
//
// Work decomposition.  One CTA of 4 warps owns one (batch, head) sequence for
// its whole length and keeps the fp32 state W in registers.  Tokens are taken
// in chunks of 64 (four mini-batches), so that every tensor-core product has
// M = 128 rows: the 64 K rows of the chunk stacked over its 64 Q rows.  With
// W_c the state at the start of the chunk and G_m (m = 0..3) the gradients of
// the loss w.r.t. the pre-activation of mini-batch m (taken at that mini-batch's
// own base state), the state at the start of mini-batch m is
//   W_m = W_c - sum_{j<m} K_j^T diag(eta_j) G_j,
// so that, exactly,
//   K_m W_m = (K W_c)_m - sum_{j<m} (K_m K_j^T) diag(eta_j) G_j
//   Q_t W_t = (Q W_c)_t - sum_{s<=t} (q_t . k_s) eta_s G_s    (the dual-form output)
//   W_next  = W_c - K^T diag(eta) G.
// Per chunk:
//   1. TMA: K, Q (64 x 64 bf16 each, 128-byte swizzle) and V, eta.
//   2. tcgen05: P = [K; Q] W_c (TMEM cols 0..63) and S = [K; Q] K^T (cols 64..127).
//   3. Every thread masks its own row of S in TMEM into the A operand of step 4:
//      K rows keep the columns of earlier mini-batches, Q rows keep s <= t (the
//      causal mask of the dual form, diagonal included), stored as bf16 hi + lo.
//   4. For m = 0..3: the warp owning mini-batch m reads its 16 rows of P (already
//      corrected for mini-batches < m), computes G_m (LN backward fused in
//      registers), writes eta*G_m as bf16 hi + lo, and issues
//      P -= A[:, m] (eta G_m) on the tensor core, which applies mini-batch m's
//      update to every later K row and to every Q row at once.
//   5. After the last mini-batch the Q rows of P hold Q W - tril(Q K^T) diag(eta) G:
//      warps 2-3 apply LN + residual and store Z while the tensor core computes
//      dW = K^T (eta G); every thread then updates its 32 fp32 state elements and
//      rewrites the bf16 hi + lo operand copy of W for the next chunk.
// Precision: every fp32 operand (W, eta*G, the masked Q K^T) enters the tensor
// core as a bf16 pair hi + lo (error ~2^-16 relative); K and Q are exact bf16;
// accumulation is fp32.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "device_status.cuh"
#include "sm100.cuh"

namespace ttt {
namespace tc {

using namespace ::ttt::sm100;

constexpr int D = 64;
constexpr int CHUNK = 64;  // tokens per chunk (4 mini-batches of 16)
constexpr int MB = 16;     // mini-batch size of this kernel
constexpr int THREADS = 128;
constexpr uint32_t TMEM_COLS = 128;

// Shared-memory map (bytes from a 1024-byte aligned base).
constexpr uint32_t OFF_K = 0;         // K tile [64][64] bf16, 128B swizzle
constexpr uint32_t OFF_Q = 8192;      // Q tile, directly after K: [K; Q] is one 128-row operand
constexpr uint32_t OFF_WHI = 16384;   // W hi [d_in][d_out] bf16
constexpr uint32_t OFF_WLO = 24576;   // W lo
constexpr uint32_t OFF_GHI = 32768;   // eta*G hi [token][d_out] bf16
constexpr uint32_t OFF_GLO = 40960;   // V tile on arrival; eta*G lo once mini-batch m is done
constexpr uint32_t OFF_ETA = 49152;   // eta of the chunk, 64 floats
constexpr uint32_t OFF_GAMMA = 49408; // LN gamma, 64 floats
constexpr uint32_t OFF_BETA = 49664;  // LN beta, 64 floats
constexpr uint32_t OFF_BAR = 49920;   // mbarriers
constexpr uint32_t OFF_TSLOT = 49984; // TMEM base address
constexpr uint32_t OFF_ABORT = 49988; // set when a bounded wait expired
constexpr uint32_t SMEM_USED = 50000;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // + alignment slack

// mbarriers: K/V/eta loads; Q load; MMA P,S; mini-batch 0,1,2 updates; last update; dW.
enum { BAR_LOAD = 0, BAR_PS = 1, BAR_C0 = 2, BAR_LAST = 5, BAR_DW = 6, BAR_LOADQ = 7, NUM_BARS = 8 };

struct Params {
  const __nv_bfloat16 *Q;  // for the residual of the output (read back from L2)
  const float *eta;
  const float *W0;
  const float *gamma, *beta;
  float eps;
  int H, T;
  float *Z;
  float *W_out;
};

__device__ __forceinline__ float quad_sum(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  x += __shfl_xor_sync(0xffffffffu, x, 2);
  return x;
}

// Waits, or flags the CTA as aborted and records the timeout if the wait expires.
__device__ __forceinline__ void wait_or_abort(uint64_t *bar, uint32_t parity, volatile int *abort) {
  if (*abort) return;
  if (!mbar_wait(bar, parity)) {
    *abort = 1;
    record_device_error(-5 /* TTT_ERR_TIMEOUT */);
  }
}

template <bool LN>
__global__ void __launch_bounds__(THREADS, 4)
    linear_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int unit = blockIdx.x;
  const int head = unit % p.H;
  const int T = p.T;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
  uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + OFF_TSLOT);
  volatile int *abort = reinterpret_cast<volatile int *>(sm + OFF_ABORT);
  float *eta_s = reinterpret_cast<float *>(sm + OFF_ETA);
  float *gam_s = reinterpret_cast<float *>(sm + OFF_GAMMA);
  float *bet_s = reinterpret_cast<float *>(sm + OFF_BETA);
  const uint32_t aK = smem_u32(sm + OFF_K);
  const uint32_t aWhi = smem_u32(sm + OFF_WHI), aWlo = smem_u32(sm + OFF_WLO);
  const uint32_t aGhi = smem_u32(sm + OFF_GHI), aGlo = smem_u32(sm + OFF_GLO);

  if (tid == 0) {
    for (int i = 0; i < NUM_BARS; ++i) mbar_init(&bars[i], 1);
    *abort = 0;
    fence_mbarrier_init();
    prefetch_tensormap(&tmQ);
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
  }
  if (warp == 0) {
    tmem_alloc(tslot, TMEM_COLS);
    tmem_relinquish();
  }
  if (LN && tid < D) {
    gam_s[tid] = p.gamma[head * D + tid];
    bet_s[tid] = p.beta[head * D + tid];
  }

  // Each thread owns 32 elements of the fp32 state: row wi, columns wc0..wc0+31.
  const int wi = 32 * (warp & 1) + lane;
  const int wc0 = 32 * (warp >> 1);
  float wm[32];
  {
    const float4 *src = reinterpret_cast<const float4 *>(p.W0 + (size_t)head * D * D + wi * D + wc0);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float4 v = src[q];
      wm[4 * q + 0] = v.x;
      wm[4 * q + 1] = v.y;
      wm[4 * q + 2] = v.z;
      wm[4 * q + 3] = v.w;
    }
  }
  // bf16 hi + lo copy of this thread's part of W (operand of P = [K;Q] W).
  auto write_w_operand = [&]() {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t hi[4], lo[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) split_bf16x2(wm[8 * q + 2 * e], wm[8 * q + 2 * e + 1], hi[e], lo[e]);
      const uint32_t off = sw128_offset(wi, wc0 + 8 * q);
      *reinterpret_cast<uint4 *>(sm + OFF_WHI + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<uint4 *>(sm + OFF_WLO + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
  };
  write_w_operand();

  const int nchunks = (T + CHUNK - 1) / CHUNK;
  const size_t tok_base = (size_t)unit * T;

  // Loads are split so that each tile is fetched as soon as its buffer is free:
  // Q once P and S are computed, K / V / eta once dW is computed.
  auto issue_loads_kv = [&](int c) {
    const int ntok = min(CHUNK, T - c * CHUNK);
    mbar_arrive_expect_tx(&bars[BAR_LOAD], 2u * 8192u + (uint32_t)ntok * 4u);
    tma_load_3d(sm + OFF_K, &tmK, 0, c * CHUNK, unit, &bars[BAR_LOAD]);
    tma_load_3d(sm + OFF_GLO, &tmV, 0, c * CHUNK, unit, &bars[BAR_LOAD]);
    bulk_load(eta_s, p.eta + tok_base + (size_t)c * CHUNK, (uint32_t)ntok * 4u, &bars[BAR_LOAD]);
  };
  auto issue_load_q = [&](int c) {
    mbar_arrive_expect_tx(&bars[BAR_LOADQ], 8192u);
    tma_load_3d(sm + OFF_Q, &tmQ, 0, c * CHUNK, unit, &bars[BAR_LOADQ]);
  };

  fence_proxy_async_smem();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tb = *tslot;
  const uint32_t tP = tb, tS = tb + 64;  // column bases of P and S (lane 0)
  if (tid == 0 && nchunks > 0) {
    issue_loads_kv(0);
    issue_load_q(0);
  }

  constexpr uint32_t ID_PW = idesc_bf16_f32(128, 64, false, true, false);   // [K;Q] x W
  constexpr uint32_t ID_S = idesc_bf16_f32(128, 64, false, false, false);   // [K;Q] x K^T
  constexpr uint32_t ID_UPD = idesc_bf16_f32(128, 64, false, true, true);   // P -= A x (eta G)
  constexpr uint32_t ID_DW = idesc_bf16_f32(128, 64, true, true, false);    // [K^T;K^T] x (eta G)

  for (int c = 0; c < nchunks; ++c) {
    const int ntok = min(CHUNK, T - c * CHUNK);
    const int nmb = ntok / MB;
    const uint32_t par = (uint32_t)c & 1u;

    // ---- 1-2: tiles in, P = [K;Q] W and S = [K;Q] K^T ----------------------------
    wait_or_abort(&bars[BAR_LOAD], par, abort);
    wait_or_abort(&bars[BAR_LOADQ], par, abort);
    if (tid == 0 && !*abort) {
      tc_fence_after_sync();
#pragma unroll
      for (int k = 0; k < 4; ++k)
        umma_ss(tP, smem_desc_sw128(aK + 32 * k, 16, 1024), smem_desc_sw128(aWhi + 2048 * k, 8192, 1024),
                ID_PW, k > 0);
#pragma unroll
      for (int k = 0; k < 4; ++k)
        umma_ss(tP, smem_desc_sw128(aK + 32 * k, 16, 1024), smem_desc_sw128(aWlo + 2048 * k, 8192, 1024),
                ID_PW, true);
#pragma unroll
      for (int k = 0; k < 4; ++k)
        umma_ss(tS, smem_desc_sw128(aK + 32 * k, 16, 1024), smem_desc_sw128(aK + 32 * k, 16, 1024),
                ID_S, k > 0);
      umma_commit(&bars[BAR_PS]);
    }
    if (ntok < CHUNK) {  // ragged last chunk: absent tokens contribute nothing to dW
      for (int x = tid; x < (CHUNK - ntok) * 32; x += THREADS) {
        const int row = ntok + x / 32, col = 2 * (x % 32);
        *reinterpret_cast<uint32_t *>(sm + OFF_GHI + sw128_offset(row, col)) = 0u;
        *reinterpret_cast<uint32_t *>(sm + OFF_GLO + sw128_offset(row, col)) = 0u;
      }
    }
    wait_or_abort(&bars[BAR_PS], par, abort);
    tc_fence_after_sync();

    // ---- 3: mask this thread's row of S into the A operand (in place, per block) ----
    {
      const int r = 32 * warp + lane;  // TMEM lane = row: K rows 0..63, Q rows 64..127
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t v[16];
        tmem_ld_32x32b_x16(tmem_addr(tS, 32 * warp, 16 * j), v);
        tmem_wait_ld();
        uint32_t hi[8], lo[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int s0 = 16 * j + 2 * e;
          bool keep0, keep1;
          if (r < CHUNK) {
            keep0 = keep1 = j < (r >> 4);  // earlier mini-batches only
          } else {
            keep0 = s0 <= r - CHUNK;  // causal, diagonal included
            keep1 = s0 + 1 <= r - CHUNK;
          }
          const float a = keep0 ? __uint_as_float(v[2 * e]) : 0.f;
          const float b = keep1 ? __uint_as_float(v[2 * e + 1]) : 0.f;
          split_bf16x2(a, b, hi[e], lo[e]);
        }
        tmem_st_32x32b_x8(tmem_addr(tS, 32 * warp, 16 * j), hi);
        tmem_st_32x32b_x8(tmem_addr(tS, 32 * warp, 16 * j + 8), lo);
      }
      tmem_wait_st();
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    // The Q buffer is free (P and S are done).  Issued only after this barrier:
    // every thread has then passed its wait on this chunk's Q phase, so the Q
    // barrier cannot complete twice while a thread still waits on it.
    if (tid == 0 && c + 1 < nchunks && !*abort) issue_load_q(c + 1);

    // ---- 4: the mini-batch chain (warp 0: mini-batches 0-1, warp 1: 2-3) ---------
    if (warp < 2) {
      const int q4 = lane & 3;
#pragma unroll 1
      for (int m = 2 * warp; m < 2 * warp + 2 && m < nmb; ++m) {
        if (m > 0) wait_or_abort(&bars[BAR_C0 + m - 1], par, abort);
        tc_fence_after_sync();
        uint32_t yr[32];
        tmem_ld_16x256b_x8(tmem_addr(tP, 32 * warp + 16 * (m & 1), 0), yr);
        tmem_wait_ld();
        const int r0 = 16 * m + (lane >> 2), r1 = r0 + 8;
        float g0[16], g1[16];  // y = the P rows, then the gradient w.r.t. y
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          g0[2 * j] = __uint_as_float(yr[4 * j + 0]);
          g0[2 * j + 1] = __uint_as_float(yr[4 * j + 1]);
          g1[2 * j] = __uint_as_float(yr[4 * j + 2]);
          g1[2 * j + 1] = __uint_as_float(yr[4 * j + 3]);
        }
        const uint32_t sbase = smem_u32(sm);
        auto ld2 = [&](uint32_t off, int row, int col) {
          return unpack_bf16x2(lds_u32(sbase + off + sw128_offset(row, col)));
        };
        const float e0 = eta_s[r0], e1 = eta_s[r1];
        // Stores eta * (dl/dy) of one column pair of both rows as bf16 hi + lo; the
        // lo half overwrites V, which this thread has read for exactly these cells.
        auto store_grad = [&](int col, float ga0, float ga1, float gb0, float gb1) {
          uint32_t h0, l0, h1, l1;
          split_bf16x2(e0 * ga0, e0 * ga1, h0, l0);
          split_bf16x2(e1 * gb0, e1 * gb1, h1, l1);
          *reinterpret_cast<uint32_t *>(sm + OFF_GHI + sw128_offset(r0, col)) = h0;
          *reinterpret_cast<uint32_t *>(sm + OFF_GLO + sw128_offset(r0, col)) = l0;
          *reinterpret_cast<uint32_t *>(sm + OFF_GHI + sw128_offset(r1, col)) = h1;
          *reinterpret_cast<uint32_t *>(sm + OFF_GLO + sw128_offset(r1, col)) = l1;
        };
        if (!LN) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int col = 8 * j + 2 * q4;
            const float2 va = ld2(OFF_GLO, r0, col), vb = ld2(OFF_GLO, r1, col);
            store_grad(col, 2.f * (g0[2 * j] - va.x), 2.f * (g0[2 * j + 1] - va.y),
                       2.f * (g1[2 * j] - vb.x), 2.f * (g1[2 * j + 1] - vb.y));
          }
        } else {
          // LN backward of ||k + gamma*xhat + beta - v||^2 w.r.t. y: with
          // dx = dl/dxhat = 2 (k + gamma xhat + beta - v) gamma,
          // dl/dy = rstd (dx - mean(dx) - xhat mean(dx xhat)).
          float s0 = 0.f, s1 = 0.f;
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            s0 += g0[e];
            s1 += g1[e];
          }
          const float mean0 = quad_sum(s0) * (1.f / D), mean1 = quad_sum(s1) * (1.f / D);
          float q0 = 0.f, q1 = 0.f;
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            g0[e] -= mean0;
            g1[e] -= mean1;
            q0 += g0[e] * g0[e];
            q1 += g1[e] * g1[e];
          }
          const float rstd0 = rsqrtf(quad_sum(q0) * (1.f / D) + p.eps);
          const float rstd1 = rsqrtf(quad_sum(q1) * (1.f / D) + p.eps);
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            g0[e] *= rstd0;  // xhat
            g1[e] *= rstd1;
          }
          auto dxhat = [&](int col, float xa0, float xa1, float xb0, float xb1, float &d00,
                           float &d01, float &d10, float &d11) {
            const float2 ka = ld2(OFF_K, r0, col), kb = ld2(OFF_K, r1, col);
            const float2 va = ld2(OFF_GLO, r0, col), vb = ld2(OFF_GLO, r1, col);
            const float2 gm = lds_f2(sbase + OFF_GAMMA + 4 * col);
            const float2 bt = lds_f2(sbase + OFF_BETA + 4 * col);
            d00 = 2.f * (ka.x + gm.x * xa0 + bt.x - va.x) * gm.x;
            d01 = 2.f * (ka.y + gm.y * xa1 + bt.y - va.y) * gm.y;
            d10 = 2.f * (kb.x + gm.x * xb0 + bt.x - vb.x) * gm.x;
            d11 = 2.f * (kb.y + gm.y * xb1 + bt.y - vb.y) * gm.y;
          };
          float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            float d00, d01, d10, d11;
            dxhat(8 * j + 2 * q4, g0[2 * j], g0[2 * j + 1], g1[2 * j], g1[2 * j + 1], d00, d01, d10, d11);
            a0 += d00 + d01;
            a1 += d10 + d11;
            b0 += d00 * g0[2 * j] + d01 * g0[2 * j + 1];
            b1 += d10 * g1[2 * j] + d11 * g1[2 * j + 1];
          }
          const float mg0 = quad_sum(a0) * (1.f / D), mg1 = quad_sum(a1) * (1.f / D);
          const float mx0 = quad_sum(b0) * (1.f / D), mx1 = quad_sum(b1) * (1.f / D);
#pragma unroll
          for (int j = 0; j < 8; ++j) {  // second pass: recompute dx, finish and store
            const int col = 8 * j + 2 * q4;
            float d00, d01, d10, d11;
            dxhat(col, g0[2 * j], g0[2 * j + 1], g1[2 * j], g1[2 * j + 1], d00, d01, d10, d11);
            store_grad(col, rstd0 * (d00 - mg0 - g0[2 * j] * mx0),
                       rstd0 * (d01 - mg0 - g0[2 * j + 1] * mx0),
                       rstd1 * (d10 - mg1 - g1[2 * j] * mx1),
                       rstd1 * (d11 - mg1 - g1[2 * j + 1] * mx1));
          }
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0 && !*abort) {
          tc_fence_after_sync();
          const uint64_t bhi = smem_desc_sw128(aGhi + 2048 * m, 8192, 1024);
          const uint64_t blo = smem_desc_sw128(aGlo + 2048 * m, 8192, 1024);
          umma_ts(tP, tS + 16 * m, bhi, ID_UPD, true);
          umma_ts(tP, tS + 16 * m, blo, ID_UPD, true);
          umma_ts(tP, tS + 16 * m + 8, bhi, ID_UPD, true);
          umma_commit(&bars[m == nmb - 1 ? BAR_LAST : BAR_C0 + m]);
        }
        __syncwarp();
      }
    }

    // ---- 5: the last update done -> dW on the tensor core, output on CUDA cores ----
    wait_or_abort(&bars[BAR_LAST], par, abort);
    tc_fence_after_sync();
    if (tid == 0 && !*abort) {
#pragma unroll
      for (int k = 0; k < 4; ++k)
        umma_ss(tS, smem_desc_sw128(aK + 2048 * k, 0, 1024), smem_desc_sw128(aGhi + 2048 * k, 8192, 1024),
                ID_DW, k > 0);
#pragma unroll
      for (int k = 0; k < 4; ++k)
        umma_ss(tS, smem_desc_sw128(aK + 2048 * k, 0, 1024), smem_desc_sw128(aGlo + 2048 * k, 8192, 1024),
                ID_DW, true);
      umma_commit(&bars[BAR_DW]);
    }
    if (warp >= 2) {
      const int q4 = lane & 3;
      float *Zc = p.Z + (tok_base + (size_t)c * CHUNK) * D;
      const __nv_bfloat16 *Qc = p.Q + (tok_base + (size_t)c * CHUNK) * D;
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        uint32_t zr[32];
        tmem_ld_16x256b_x8(tmem_addr(tP, 32 * warp + 16 * h, 0), zr);
        tmem_wait_ld();
        const int t0 = 32 * (warp - 2) + 16 * h + (lane >> 2), t1 = t0 + 8;
        float z0[16], z1[16];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          z0[2 * j] = __uint_as_float(zr[4 * j + 0]);
          z0[2 * j + 1] = __uint_as_float(zr[4 * j + 1]);
          z1[2 * j] = __uint_as_float(zr[4 * j + 2]);
          z1[2 * j + 1] = __uint_as_float(zr[4 * j + 3]);
        }
        if (LN) {
          float s0 = 0.f, s1 = 0.f;
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            s0 += z0[e];
            s1 += z1[e];
          }
          const float mean0 = quad_sum(s0) * (1.f / D), mean1 = quad_sum(s1) * (1.f / D);
          float q0 = 0.f, q1 = 0.f;
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            z0[e] -= mean0;
            z1[e] -= mean1;
            q0 += z0[e] * z0[e];
            q1 += z1[e] * z1[e];
          }
          const float rstd0 = rsqrtf(quad_sum(q0) * (1.f / D) + p.eps);
          const float rstd1 = rsqrtf(quad_sum(q1) * (1.f / D) + p.eps);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int col = 8 * j + 2 * q4;
            const float2 qa = t0 < ntok ? __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(Qc + t0 * D + col))
                                        : make_float2(0.f, 0.f);
            const float2 qb = t1 < ntok ? __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(Qc + t1 * D + col))
                                        : make_float2(0.f, 0.f);
            const float2 gm = lds_f2(smem_u32(sm) + OFF_GAMMA + 4 * col);
            const float2 bt = lds_f2(smem_u32(sm) + OFF_BETA + 4 * col);
            if (t0 < ntok)
              *reinterpret_cast<float2 *>(Zc + t0 * D + col) =
                  make_float2(qa.x + gm.x * (z0[2 * j] * rstd0) + bt.x,
                              qa.y + gm.y * (z0[2 * j + 1] * rstd0) + bt.y);
            if (t1 < ntok)
              *reinterpret_cast<float2 *>(Zc + t1 * D + col) =
                  make_float2(qb.x + gm.x * (z1[2 * j] * rstd1) + bt.x,
                              qb.y + gm.y * (z1[2 * j + 1] * rstd1) + bt.y);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int col = 8 * j + 2 * q4;
            if (t0 < ntok) *reinterpret_cast<float2 *>(Zc + t0 * D + col) = make_float2(z0[2 * j], z0[2 * j + 1]);
            if (t1 < ntok) *reinterpret_cast<float2 *>(Zc + t1 * D + col) = make_float2(z1[2 * j], z1[2 * j + 1]);
          }
        }
      }
    }

    // ---- 6: state update W -= dW and the next chunk's operand copy --------------
    wait_or_abort(&bars[BAR_DW], par, abort);
    tc_fence_after_sync();
    // K, V (lo half of eta*G) and eta are free once dW is done; every thread passed
    // this chunk's wait on their barrier before the A-operand barrier above.
    if (tid == 0 && c + 1 < nchunks && !*abort) issue_loads_kv(c + 1);
    {
      uint32_t dw[32];
      tmem_ld_32x32b_x32(tmem_addr(tS, 32 * warp, wc0), dw);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; ++e) wm[e] -= __uint_as_float(dw[e]);
      write_w_operand();
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (*abort) break;
  }

  // Final state.
  {
    float4 *dst = reinterpret_cast<float4 *>(p.W_out + (size_t)unit * D * D + wi * D + wc0);
#pragma unroll
    for (int q = 0; q < 8; ++q)
      dst[q] = make_float4(wm[4 * q], wm[4 * q + 1], wm[4 * q + 2], wm[4 * q + 3]);
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tb, TMEM_COLS);
  }
}

}  // namespace tc
}  // namespace ttt
