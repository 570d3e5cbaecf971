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
// M = 128 rows: the 64 K rows and the 64 Q rows of the chunk, interleaved by
// mini-batch as [K0; Q0; K1; Q1; K2; Q2; K3; Q3] (16 rows each).  TMEM lane =
// operand row, so warp m (which can read TMEM lanes 32m..32m+31) holds exactly
// the K and Q rows of mini-batch m.  With W_c the state at the start of the
// chunk and G_m the gradient of the loss w.r.t. the pre-activation of
// mini-batch m (taken at that mini-batch's own base state), the state at the
// start of mini-batch m is W_m = W_c - sum_{j<m} K_j^T diag(eta_j) G_j, so that
//   K_m W_m = (K W_c)_m - sum_{j<m} (K_m K_j^T) diag(eta_j) G_j
//   q_t W_t = (Q W_c)_t - sum_{s<=t} (q_t . k_s) eta_s G_s    (dual-form output)
//   W_next  = W_c - K^T diag(eta) G.
// Per chunk:
//   1. TMA: K and Q (16-row boxes into the interleaved operand, 128-byte
//      swizzle), V, eta.
//   2. tcgen05: P = [K;Q] W_c (TMEM cols 0..63), S = [K;Q] K^T (cols 64..127).
//   3. Every thread masks its own row of S in TMEM into the A operand of step 4:
//      K rows keep the columns of earlier mini-batches, Q rows keep s <= t (the
//      causal mask of the dual form, diagonal included), as bf16 hi + lo.
//   4. For m = 0..3, warp m: reads its 16 K rows of P (already corrected for
//      mini-batches < m), computes G_m (LN backward in registers), writes
//      eta*G_m as bf16 hi + lo, and issues P -= A[:, m] (eta G_m), which applies
//      mini-batch m's update to every later K row and every Q row at once.
//   5. Then the Q rows of P hold Q W - tril(Q K^T) diag(eta) G: each warp applies
//      LN + residual to its 16 Q rows and stores Z while the tensor core computes
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
constexpr uint32_t OFF_A = 0;          // [K0;Q0;K1;Q1;K2;Q2;K3;Q3], 16 rows x 128 B each
constexpr uint32_t OFF_WHI = 16384;    // W hi [d_in][d_out] bf16
constexpr uint32_t OFF_WLO = 24576;    // W lo
constexpr uint32_t OFF_GHI = 32768;    // eta*G hi [token][d_out] bf16
constexpr uint32_t OFF_GLO = 40960;    // V tile on arrival; eta*G lo once a mini-batch is done
constexpr uint32_t OFF_ETA = 49152;    // eta of the chunk, 64 floats
constexpr uint32_t OFF_GAMMA = 49408;  // LN gamma, 64 floats
constexpr uint32_t OFF_BETA = 49664;   // LN beta, 64 floats
constexpr uint32_t OFF_W2 = 49920;     // 2 gamma^2, 64 floats
constexpr uint32_t OFF_BAR = 50176;    // mbarriers (9 x 8 bytes)
constexpr uint32_t OFF_TSLOT = 50248;  // TMEM base address
constexpr uint32_t OFF_ABORT = 50252;  // set when a bounded wait expired
constexpr uint32_t SMEM_USED = 50256;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // + alignment slack

__host__ __device__ constexpr uint32_t k_block(int m) { return OFF_A + 4096u * m; }
__host__ __device__ constexpr uint32_t q_block(int m) { return OFF_A + 4096u * m + 2048u; }

// mbarriers: K/V/eta loads; MMA S; updates of mini-batches 0,1,2; last update;
// dW; Q loads (four arrivals: one per warp and Q block); MMA P.
enum { BAR_LOAD = 0, BAR_S = 1, BAR_C0 = 2, BAR_LAST = 5, BAR_DW = 6, BAR_LOADQ = 7, BAR_P = 8, NUM_BARS = 9 };

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

__device__ __forceinline__ float sum8(const float2 (&x)[8]) {
  const float2 a = __fadd2_rn(__fadd2_rn(x[0], x[1]), __fadd2_rn(x[2], x[3]));
  const float2 b = __fadd2_rn(__fadd2_rn(x[4], x[5]), __fadd2_rn(x[6], x[7]));
  const float2 c = __fadd2_rn(a, b);
  return c.x + c.y;
}

__device__ __forceinline__ float2 __fsub2(float2 a, float2 b) {
  return __fadd2_rn(a, make_float2(-b.x, -b.y));
}

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
  const uint32_t sbase = smem_u32(sm);
  const uint32_t aA = sbase + OFF_A;
  const uint32_t aWhi = sbase + OFF_WHI, aWlo = sbase + OFF_WLO;
  const uint32_t aGhi = sbase + OFF_GHI, aGlo = sbase + OFF_GLO;

  if (tid == 0) {
    for (int i = 0; i < NUM_BARS; ++i) mbar_init(&bars[i], i == BAR_LOADQ ? 4 : 1);
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
    const float g = p.gamma[head * D + tid];
    reinterpret_cast<float *>(sm + OFF_GAMMA)[tid] = g;
    reinterpret_cast<float *>(sm + OFF_BETA)[tid] = p.beta[head * D + tid];
    reinterpret_cast<float *>(sm + OFF_W2)[tid] = 2.f * g * g;
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
  const int q4 = lane & 3;
  const int fr = lane >> 2;  // row within a 16-row group (and +8) in the 16x256b layout

  // Loads are split so that each tile is fetched as soon as its buffer is free:
  // each warp refills its own Q block once it has written its output, thread 0
  // refills K / V / eta once dW is computed.
  auto issue_loads_kv = [&](int c) {
    const int ntok = min(CHUNK, T - c * CHUNK);
    mbar_arrive_expect_tx(&bars[BAR_LOAD], 4u * 2048u + 8192u + (uint32_t)ntok * 4u);
#pragma unroll
    for (int m = 0; m < 4; ++m) tma_load_3d(sm + k_block(m), &tmK, 0, c * CHUNK + MB * m, unit, &bars[BAR_LOAD]);
    tma_load_3d(sm + OFF_GLO, &tmV, 0, c * CHUNK, unit, &bars[BAR_LOAD]);
    bulk_load(eta_s, p.eta + tok_base + (size_t)c * CHUNK, (uint32_t)ntok * 4u, &bars[BAR_LOAD]);
  };
  // One of the four arrivals of the Q barrier: Q block m of chunk c.
  auto issue_load_q_block = [&](int c, int m) {
    mbar_arrive_expect_tx(&bars[BAR_LOADQ], 2048u);
    tma_load_3d(sm + q_block(m), &tmQ, 0, c * CHUNK + MB * m, unit, &bars[BAR_LOADQ]);
  };

  fence_proxy_async_smem();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tb = *tslot;
  const uint32_t tP = tb, tS = tb + 64;  // column bases of P and S (lane 0)
  if (tid == 0 && nchunks > 0) issue_loads_kv(0);
  if (lane == 0 && nchunks > 0) issue_load_q_block(0, warp);

  constexpr uint32_t ID_PW = idesc_bf16_f32(128, 64, false, true, false);  // [K;Q] x W
  constexpr uint32_t ID_S = idesc_bf16_f32(128, 16, false, false, false);  // [K;Q] x K_m^T
  constexpr uint32_t ID_UPD = idesc_bf16_f32(128, 64, false, true, true);  // P -= A x (eta G)
  constexpr uint32_t ID_DW = idesc_bf16_f32(128, 64, true, true, false);   // [K^T;K^T] x (eta G)

  for (int c = 0; c < nchunks; ++c) {
    const int ntok = min(CHUNK, T - c * CHUNK);
    const int nmb = ntok / MB;
    const uint32_t par = (uint32_t)c & 1u;

    // ---- 1-2: tiles in; S = [K;Q] K^T first (the masking needs it), then P = [K;Q] W
    wait_or_abort(&bars[BAR_LOAD], par, abort);
    wait_or_abort(&bars[BAR_LOADQ], par, abort);
    if (tid == 0 && !*abort) {
      tc_fence_after_sync();
#pragma unroll
      for (int n = 0; n < 4; ++n)
#pragma unroll
        for (int k = 0; k < 4; ++k)
          umma_ss(tS + 16 * n, smem_desc_sw128(aA + 32 * k, 16, 1024),
                  smem_desc_sw128(sbase + k_block(n) + 32 * k, 16, 1024), ID_S, k > 0);
      umma_commit(&bars[BAR_S]);
#pragma unroll
      for (int k = 0; k < 4; ++k)
        umma_ss(tP, smem_desc_sw128(aA + 32 * k, 16, 1024), smem_desc_sw128(aWhi + 2048 * k, 8192, 1024),
                ID_PW, k > 0);
#pragma unroll
      for (int k = 0; k < 4; ++k)
        umma_ss(tP, smem_desc_sw128(aA + 32 * k, 16, 1024), smem_desc_sw128(aWlo + 2048 * k, 8192, 1024),
                ID_PW, true);
      umma_commit(&bars[BAR_P]);
    }
    if (ntok < CHUNK) {  // ragged last chunk: absent tokens contribute nothing to dW
      for (int x = tid; x < (CHUNK - ntok) * 32; x += THREADS) {
        const int row = ntok + x / 32, col = 2 * (x % 32);
        *reinterpret_cast<uint32_t *>(sm + OFF_GHI + sw128_offset(row, col)) = 0u;
        *reinterpret_cast<uint32_t *>(sm + OFF_GLO + sw128_offset(row, col)) = 0u;
      }
    }

    // Everything of mini-batch `warp`'s LN backward that does not depend on P,
    // computed while the tensor core works: u = 2 gamma (k + beta - v) (or v for
    // the plain linear model) for this thread's two rows, and mean(u).
    const int m = warp;
    const int r0 = MB * m + fr, r1 = r0 + 8;  // tokens of this thread's two rows
    float2 u0[8], u1[8];
    float um0 = 0.f, um1 = 0.f;
    if (m < nmb) {
      const uint32_t kb = sbase + k_block(m);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int col = 8 * j + 2 * q4;
        const float2 va = unpack_bf16x2(lds_u32(aGlo + sw128_offset(r0, col)));
        const float2 vc = unpack_bf16x2(lds_u32(aGlo + sw128_offset(r1, col)));
        if (LN) {
          const float2 ka = unpack_bf16x2(lds_u32(kb + sw128_offset(fr, col)));
          const float2 kc = unpack_bf16x2(lds_u32(kb + sw128_offset(fr + 8, col)));
          const float2 gm = *reinterpret_cast<const float2 *>(sm + OFF_GAMMA + 4 * col);
          const float2 bt = *reinterpret_cast<const float2 *>(sm + OFF_BETA + 4 * col);
          const float2 g2 = __fadd2_rn(gm, gm);
          u0[j] = __fmul2_rn(g2, __fadd2_rn(ka, __fsub2(bt, va)));
          u1[j] = __fmul2_rn(g2, __fadd2_rn(kc, __fsub2(bt, vc)));
          um0 += u0[j].x + u0[j].y;
          um1 += u1[j].x + u1[j].y;
        } else {
          u0[j] = va;
          u1[j] = vc;
        }
      }
      if (LN) {
        um0 = quad_sum(um0) * (1.f / D);
        um1 = quad_sum(um1) * (1.f / D);
      }
    }
    const float e0 = eta_s[r0], e1 = eta_s[r1];

    wait_or_abort(&bars[BAR_S], par, abort);
    tc_fence_after_sync();
    __syncwarp();  // lanes leave the wait loop independently; TMEM access is warp-collective

    // ---- 3: mask this thread's row of S into the A operand (in place, per block) ------
    {
      const bool qrow = lane >= 16;
      const int t = MB * warp + (lane & 15);  // token of this row within the chunk
      // Column blocks j > warp are zero for every row of this warp (K rows keep
      // blocks < warp, Q rows blocks <= warp); TMEM loads and stores are
      // warp-collective, so the skip is decided per warp.
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t v[16], hi[8], lo[8];
        if (j <= warp) {
          tmem_ld_32x32b_x16(tmem_addr(tS, 32 * warp, 16 * j), v);
          tmem_wait_ld();
        }
        const bool all_zero = qrow ? (j > warp) : (j >= warp);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int s0 = MB * j + 2 * e;
          const float a = (!all_zero && (!qrow || s0 <= t)) ? __uint_as_float(v[2 * e]) : 0.f;
          const float b = (!all_zero && (!qrow || s0 + 1 <= t)) ? __uint_as_float(v[2 * e + 1]) : 0.f;
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

    // ---- 4: the mini-batch chain: warp m handles mini-batch m ------------------------
    if (m < nmb) {
      wait_or_abort(&bars[m == 0 ? BAR_P : BAR_C0 + m - 1], par, abort);
      tc_fence_after_sync();
      __syncwarp();
      uint32_t yr[32];
      tmem_ld_16x256b_x8(tmem_addr(tP, 32 * m, 0), yr);
      tmem_wait_ld();
      float2 y0[8], y1[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        y0[j] = make_float2(__uint_as_float(yr[4 * j + 0]), __uint_as_float(yr[4 * j + 1]));
        y1[j] = make_float2(__uint_as_float(yr[4 * j + 2]), __uint_as_float(yr[4 * j + 3]));
      }
      // Stores eta * (dl/dy) of one column pair of both rows as bf16 hi + lo; the
      // lo half overwrites V, which this thread has read for exactly these cells.
      auto store_grad = [&](int col, float2 g0, float2 g1) {
        uint32_t h0, l0, h1, l1;
        split_bf16x2(g0.x, g0.y, h0, l0);
        split_bf16x2(g1.x, g1.y, h1, l1);
        *reinterpret_cast<uint32_t *>(sm + OFF_GHI + sw128_offset(r0, col)) = h0;
        *reinterpret_cast<uint32_t *>(sm + OFF_GLO + sw128_offset(r0, col)) = l0;
        *reinterpret_cast<uint32_t *>(sm + OFF_GHI + sw128_offset(r1, col)) = h1;
        *reinterpret_cast<uint32_t *>(sm + OFF_GLO + sw128_offset(r1, col)) = l1;
      };
      if (!LN) {
        // dl/dy = 2 (y - v)
        const float2 f0 = make_float2(2.f * e0, 2.f * e0), f1 = make_float2(2.f * e1, 2.f * e1);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          store_grad(8 * j + 2 * q4, __fmul2_rn(f0, __fsub2(y0[j], u0[j])),
                     __fmul2_rn(f1, __fsub2(y1[j], u1[j])));
      } else {
        // LN backward of ||k + gamma xhat + beta - v||^2 w.r.t. y.  With
        // dx = dl/dxhat = u + w xhat (w = 2 gamma^2), A = mean(dx), B = mean(dx xhat):
        // dl/dy = rstd (dx - A - xhat B) = rstd (u + xhat (w - B) - A).
        const float mean0 = quad_sum(sum8(y0)) * (1.f / D);
        const float mean1 = quad_sum(sum8(y1)) * (1.f / D);
        const float2 nm0 = make_float2(-mean0, -mean0), nm1 = make_float2(-mean1, -mean1);
        float2 q0a = make_float2(0.f, 0.f), q0b = q0a, q1a = q0a, q1b = q0a;
#pragma unroll
        for (int j = 0; j < 8; j += 2) {
          y0[j] = __fadd2_rn(y0[j], nm0);
          y0[j + 1] = __fadd2_rn(y0[j + 1], nm0);
          y1[j] = __fadd2_rn(y1[j], nm1);
          y1[j + 1] = __fadd2_rn(y1[j + 1], nm1);
          q0a = __ffma2_rn(y0[j], y0[j], q0a);
          q0b = __ffma2_rn(y0[j + 1], y0[j + 1], q0b);
          q1a = __ffma2_rn(y1[j], y1[j], q1a);
          q1b = __ffma2_rn(y1[j + 1], y1[j + 1], q1b);
        }
        const float rstd0 = rsqrtf(quad_sum((q0a.x + q0b.x) + (q0a.y + q0b.y)) * (1.f / D) + p.eps);
        const float rstd1 = rsqrtf(quad_sum((q1a.x + q1b.x) + (q1a.y + q1b.y)) * (1.f / D) + p.eps);
        const float2 rs0 = make_float2(rstd0, rstd0), rs1 = make_float2(rstd1, rstd1);
        float2 wx0 = make_float2(0.f, 0.f), wx1 = wx0, ux0 = wx0, ux1 = wx0, wxx0 = wx0, wxx1 = wx0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float2 w2 = *reinterpret_cast<const float2 *>(sm + OFF_W2 + 4 * (8 * j + 2 * q4));
          y0[j] = __fmul2_rn(y0[j], rs0);  // xhat
          y1[j] = __fmul2_rn(y1[j], rs1);
          const float2 wa = __fmul2_rn(w2, y0[j]), wb = __fmul2_rn(w2, y1[j]);
          wx0 = __fadd2_rn(wx0, wa);
          wx1 = __fadd2_rn(wx1, wb);
          wxx0 = __ffma2_rn(wa, y0[j], wxx0);
          wxx1 = __ffma2_rn(wb, y1[j], wxx1);
          ux0 = __ffma2_rn(u0[j], y0[j], ux0);
          ux1 = __ffma2_rn(u1[j], y1[j], ux1);
        }
        const float A0 = um0 + quad_sum(wx0.x + wx0.y) * (1.f / D);
        const float A1 = um1 + quad_sum(wx1.x + wx1.y) * (1.f / D);
        const float B0 = quad_sum((ux0.x + ux0.y) + (wxx0.x + wxx0.y)) * (1.f / D);
        const float B1 = quad_sum((ux1.x + ux1.y) + (wxx1.x + wxx1.y)) * (1.f / D);
        const float2 f0 = make_float2(e0 * rstd0, e0 * rstd0), f1 = make_float2(e1 * rstd1, e1 * rstd1);
        const float2 nA0 = make_float2(-A0, -A0), nA1 = make_float2(-A1, -A1);
        const float2 nB0 = make_float2(-B0, -B0), nB1 = make_float2(-B1, -B1);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float2 w2 = *reinterpret_cast<const float2 *>(sm + OFF_W2 + 4 * (8 * j + 2 * q4));
          const float2 ga = __fmul2_rn(f0, __fadd2_rn(__ffma2_rn(y0[j], __fadd2_rn(w2, nB0), u0[j]), nA0));
          const float2 gb = __fmul2_rn(f1, __fadd2_rn(__ffma2_rn(y1[j], __fadd2_rn(w2, nB1), u1[j]), nA1));
          store_grad(8 * j + 2 * q4, ga, gb);
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

      // ---- 5: output of this mini-batch's Q rows.  After update m their value is
      // final: later updates add exactly zero to them (A is zero there).
      wait_or_abort(&bars[m == nmb - 1 ? BAR_LAST : BAR_C0 + m], par, abort);
      tc_fence_after_sync();
      __syncwarp();
      uint32_t zr[32];
      tmem_ld_16x256b_x8(tmem_addr(tP, 32 * m + 16, 0), zr);
      tmem_wait_ld();
      float2 z0[8], z1[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        z0[j] = make_float2(__uint_as_float(zr[4 * j + 0]), __uint_as_float(zr[4 * j + 1]));
        z1[j] = make_float2(__uint_as_float(zr[4 * j + 2]), __uint_as_float(zr[4 * j + 3]));
      }
      float *Zc = p.Z + (tok_base + (size_t)c * CHUNK) * D;
      const bool ok0 = r0 < ntok, ok1 = r1 < ntok;
      const uint32_t qb = sbase + q_block(m);
      if (LN) {
        const float mean0 = quad_sum(sum8(z0)) * (1.f / D);
        const float mean1 = quad_sum(sum8(z1)) * (1.f / D);
        const float2 nm0 = make_float2(-mean0, -mean0), nm1 = make_float2(-mean1, -mean1);
        float2 q0a = make_float2(0.f, 0.f), q0b = q0a, q1a = q0a, q1b = q0a;
#pragma unroll
        for (int j = 0; j < 8; j += 2) {
          z0[j] = __fadd2_rn(z0[j], nm0);
          z0[j + 1] = __fadd2_rn(z0[j + 1], nm0);
          z1[j] = __fadd2_rn(z1[j], nm1);
          z1[j + 1] = __fadd2_rn(z1[j + 1], nm1);
          q0a = __ffma2_rn(z0[j], z0[j], q0a);
          q0b = __ffma2_rn(z0[j + 1], z0[j + 1], q0b);
          q1a = __ffma2_rn(z1[j], z1[j], q1a);
          q1b = __ffma2_rn(z1[j + 1], z1[j + 1], q1b);
        }
        const float rstd0 = rsqrtf(quad_sum((q0a.x + q0b.x) + (q0a.y + q0b.y)) * (1.f / D) + p.eps);
        const float rstd1 = rsqrtf(quad_sum((q1a.x + q1b.x) + (q1a.y + q1b.y)) * (1.f / D) + p.eps);
        const float2 rs0 = make_float2(rstd0, rstd0), rs1 = make_float2(rstd1, rstd1);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int col = 8 * j + 2 * q4;
          const float2 gm = *reinterpret_cast<const float2 *>(sm + OFF_GAMMA + 4 * col);
          const float2 bt = *reinterpret_cast<const float2 *>(sm + OFF_BETA + 4 * col);
          const float2 qa = unpack_bf16x2(lds_u32(qb + sw128_offset(fr, col)));
          const float2 qc = unpack_bf16x2(lds_u32(qb + sw128_offset(fr + 8, col)));
          if (ok0)
            *reinterpret_cast<float2 *>(Zc + r0 * D + col) =
                __fadd2_rn(qa, __ffma2_rn(gm, __fmul2_rn(z0[j], rs0), bt));
          if (ok1)
            *reinterpret_cast<float2 *>(Zc + r1 * D + col) =
                __fadd2_rn(qc, __ffma2_rn(gm, __fmul2_rn(z1[j], rs1), bt));
        }
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int col = 8 * j + 2 * q4;
          if (ok0) *reinterpret_cast<float2 *>(Zc + r0 * D + col) = z0[j];
          if (ok1) *reinterpret_cast<float2 *>(Zc + r1 * D + col) = z1[j];
        }
      }
      // This warp's Q block is no longer needed: refill it with the next chunk.
      // The Q barrier completes only when all four warps have arrived, i.e. after
      // every thread has passed its wait on this chunk's Q phase.
      __syncwarp();
      if (lane == 0 && c + 1 < nchunks && !*abort) issue_load_q_block(c + 1, m);
    }

    // ---- 6: dW on the tensor core after the last update; state update -------------
    wait_or_abort(&bars[BAR_LAST], par, abort);
    tc_fence_after_sync();
    if (tid == 0 && !*abort) {
#pragma unroll
      for (int k = 0; k < 4; ++k)
        umma_ss(tS, smem_desc_sw128(sbase + k_block(k), 0, 1024), smem_desc_sw128(aGhi + 2048 * k, 8192, 1024),
                ID_DW, k > 0);
#pragma unroll
      for (int k = 0; k < 4; ++k)
        umma_ss(tS, smem_desc_sw128(sbase + k_block(k), 0, 1024), smem_desc_sw128(aGlo + 2048 * k, 8192, 1024),
                ID_DW, true);
      umma_commit(&bars[BAR_DW]);
    }
    wait_or_abort(&bars[BAR_DW], par, abort);
    tc_fence_after_sync();
    __syncwarp();
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
