// tc_mlp.cuh - tensor-core (tcgen05) kernel of TTT-MLP,
// f(x) = x + LN(GELU(x W1) W2), d = 64, hidden h = 256, bf16 Q, K, V, b = 16.
//
// Method: the dual form of the TTT write-up (§03.7) over mini-batches of b = 16
// tokens (§03.6) for the MLP variant (§03.9), loss ||f(k; W) - v||^2 (§03.5).
// Per mini-batch, with W1, W2 the state at its start (every gradient of the
// mini-batch is taken there), X1 = K W1, X2 = GELU(X1), X3 = X2 W2,
// G3 = dl/dX3 (through LN and the residual), G2 = (G3 W2^T) * GELU'(X1),
// E2 = diag(eta) G2, E3 = diag(eta) G3:
//   Zq1 = Q W1 - tril(Q K^T) E2,   Zq2 = GELU(Zq1)
//   Zq3 = Zq2 W2 - tril(Zq2 X2^T) E3,   Z = Q + LN(Zq3)
//   W1 <- W1 - K^T E2,   W2 <- W2 - X2^T E3.
// Every product is exact in the dual form: each layer is linear in its weight
// and all the mini-batch's gradients are taken at its base state.
//
// Work decomposition.  One CTA of 16 warps owns one (batch, head) sequence for
// its whole length; thread (i, j) owns hidden unit i (TMEM lane i % 128 of
// column half i / 128) and tokens 8 j .. 8 j + 7 of each mini-batch (or d
// columns 32 j .. 32 j + 31 of the state).  The fp32 state lives in tensor
// memory for the whole sequence: W1^T and W2 as [hidden][d] (lanes = hidden
// unit), and the two state updates are tensor-core products that accumulate
// into it in place.  Products whose output has a hidden dimension are computed
// hidden-major (M = 256 as two M = 128 halves), the two whose output is
// [d x tokens] with M = 64.  Per mini-batch:
//   P1   = W1^T [K;Q]^T                 (hidden x 32 tokens; A from TMEM)
//   X3^T = W2^T X2^T                    (d x 16, M = 64)
//   GW^T = W2 G3^T                      (hidden x 16; A from TMEM)
//   W2 -= X2^T E3,  W1^T -= E2^T K      (A from TMEM, accumulated into the state)
//   P1_q -= E2^T tril(Q K^T)^T          (Zq1: the Q columns of P1)
//   S2   = Zq2 X2^T                     (the 16 x 16 Gram over the hidden width:
//                                       4 blocks of 64 hidden units as one
//                                       M = 64 product whose diagonal 16 x 16
//                                       blocks are summed)
//   Zq3^T = W2'^T Zq2^T + E3^T striu(S2)^T   (W2' = W2 after this mini-batch's
//                                       update, hence the strictly upper mask:
//                                       Zq2 W2 = Zq2 W2' + S2 E3)
// and once per chunk of 64 tokens S1 = [K;Q] K^T for the masked Q K^T blocks.
// GELU, GELU', the LN forward and backward and the output LN run on the CUDA
// cores between the products.
//
// Operand precision.  The products that contract over the hidden width (X3,
// Zq3, the Gram) take fp16 operands (kind::f16, 10-bit mantissa, 16 elements
// of K per instruction): a copy of W2 refreshed after each update, X2 and Zq2.
// Every other product is kind::tf32 (10-bit mantissa, fp32 range) with the
// fp32 state read from tensor memory (truncated to tf32 by the tensor core) and
// the activations, gradients and masked Grams rounded to tf32 where they are
// written.  Accumulation is fp32; K and Q (bf16) are exact in tf32.  fp16
// overflows above 65504: the W2 copy and the activations X2, Zq2 stay far below
// that unless the inner model diverges.
//
// Product issue.  A tcgen05.mma instruction costs ~45 SM cycles to issue
// whatever its size, so the products are shaped for few instructions, and every
// product is issued by warp 0 converged (one lane elected inside the asm).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "device_status.cuh"
#include "sm100.cuh"

namespace ttt {
namespace tcmlp {

using namespace ::ttt::sm100;

constexpr int D = 64;
constexpr int HID = 256;
constexpr int MB = 16;      // mini-batch size of this kernel
constexpr int CHUNK = 64;   // tokens per TMA chunk (4 mini-batches)
constexpr int THREADS = 512;
constexpr uint32_t TMEM_COLS = 512;

// TMEM columns (lane = hidden unit within a half unless noted).
constexpr uint32_t C_W1 = 0;     // W1^T state, half h at 64 h (64 columns = d)
constexpr uint32_t C_W2 = 128;   // W2 state, half h at 128 + 64 h
constexpr uint32_t C_P1 = 256;   // P1 = W1^T [K;Q]^T, half h at 256 + 32 h; its K columns
                                 // (0-7, 16-23) then hold X2^T
constexpr uint32_t C_GW = 320;   // GW^T, half h at 320 + 16 h; then E2^T
constexpr uint32_t C_X3 = 352;   // X3^T (M = 64, lane offset 0) and Zq3^T (lane offset 16)
constexpr uint32_t C_S1 = 368;   // S1 = [K;Q] K^T of the chunk (M = 128, 64 columns)
constexpr uint32_t C_S2 = 432;   // the Gram blocks (M = 64, 64 columns)

// Shared-memory map (bytes from a 1024-byte aligned base).  "[a][r][128B]" means
// 128 bytes of row r of column block a.  K-major tiles and fp16 tiles use the
// 128-byte swizzle (16-byte granules), MN-major fp32 tiles the 128-byte swizzle
// on a 32-byte base (the only MN-major layout of kind::tf32).
constexpr uint32_t OFF_W2 = 0;          // W2 copy [hidden 256][64 d fp16], MN-major for W2^T
constexpr uint32_t OFF_KQ = 32768;      // [K;Q] of the chunk [d-block 2][row 128][128B] fp32, K-major
constexpr uint32_t OFF_X2 = 65536;      // X2  [hidden-block 4][token 16][64 fp16], K-major
constexpr uint32_t OFF_Z2 = 73728;      // Zq2 same layout
constexpr uint32_t OFF_KM = 81920;      // K of the mini-batch [d-block 2][token 16][128B] fp32, MN-major
constexpr uint32_t OFF_G3 = 86016;      // G3  [token 16][64 d fp16], K-major
constexpr uint32_t OFF_E3 = 90112;      // E3  same shape, MN-major
constexpr uint32_t OFF_S1 = 94208;      // masked Q K^T in P1's column order [row 32][128B]
constexpr uint32_t OFF_S2U = 98304;     // striu(S2) [query token 16][128B]
constexpr uint32_t OFF_STG = 100352;    // 2 stages x {K, Q, V} bf16 [64][128B] (TMA)
constexpr uint32_t STG_BYTES = 24576;
constexpr uint32_t OFF_ETA = 149504;    // 2 stages x 64 eta
constexpr uint32_t OFF_RED = 150016;    // [16][RS] fp32 rows (X3, Zq3) / Gram partials [4][16][17]
constexpr uint32_t OFF_GB = 154368;     // gamma [64], beta [64]
constexpr uint32_t OFF_BAR = 154880;    // mbarriers
constexpr uint32_t OFF_TSLOT = 154976;  // TMEM base address
constexpr uint32_t OFF_ABORT = 154980;  // set when a bounded wait expired
constexpr uint32_t SMEM_USED = 154984;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // + alignment slack
constexpr int RS = 68;                  // row stride (floats) of the [token][d] staging rows

enum {
  BAR_LOAD0 = 0, BAR_LOAD1 = 1, BAR_S1C = 2, BAR_P1 = 3, BAR_X3 = 4, BAR_GW = 5, BAR_UPD = 6,
  BAR_S2 = 7, BAR_ZQ3 = 8, BAR_DRAIN = 9, BAR_NEVER = 10, NUM_BARS = 11
};
// The warp that issues Zq3 and its correction (and, with the next warp, P1).
constexpr int ZQ3_WARP = 4;
constexpr long long WAIT_LIMIT = 1ll << 32;
constexpr long long INJECTED_WAIT_LIMIT = 1ll << 20;

struct Params {
  const float *eta;
  const float *W1_0, *W2_0;  // [H][d][hidden], [H][hidden][d]
  const float *gamma, *beta;
  float eps;
  int H, T;
  float *Z;
  float *W1_out, *W2_out;    // [units][d][hidden], [units][hidden][d]
  int inject_timeout;
};

// Byte offset of 4-byte element (row, col) in a [rows][128B] block of 32
// columns with the 128-byte swizzle (col < 32).
__device__ __forceinline__ uint32_t swz32(uint32_t row, uint32_t col) {
  return row * 128u + ((((col >> 2) ^ row) & 7u) << 4) + ((col & 3u) << 2);
}
// The same for 2-byte elements, 64 columns per row (col < 64).
__device__ __forceinline__ uint32_t swz16(uint32_t row, uint32_t col) {
  return row * 128u + ((((col >> 3) ^ row) & 7u) << 4) + ((col & 7u) << 1);
}
// 4-byte element (row, col) with the 32-byte-base swizzle (col < 32).
__device__ __forceinline__ uint32_t swzb32(uint32_t row, uint32_t col) {
  return row * 128u + ((((col >> 3) ^ row) & 3u) << 5) + ((col & 7u) << 2);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Phi(x) and phi(x) of the standard normal, for GELU(x) = x Phi(x) (the exact
// erf form) and GELU'(x) = Phi(x) + x phi(x).  erfc(z), z = |x| / sqrt(2), by
// the rational approximation of Abramowitz and Stegun, Handbook of Mathematical
// Functions, formula 7.1.26 (absolute error at most 1.5e-7):
//   erfc(z) = (a1 t + a2 t^2 + a3 t^3 + a4 t^4 + a5 t^5) exp(-z^2),
//   t = 1 / (1 + p z),
// so that Phi(x) = 1 - erfc(z) / 2 for x >= 0 and erfc(z) / 2 otherwise, with no
// cancellation on either side; exp(-z^2) = exp(-x^2 / 2) also gives phi.
__device__ __forceinline__ void normal_cdf_pdf(float x, float &cdf, float &pdf) {
  constexpr float P = 0.3275911f;
  constexpr float A1 = 0.254829592f, A2 = -0.284496736f, A3 = 1.421413741f;
  constexpr float A4 = -1.453152027f, A5 = 1.061405429f;
  constexpr float RSQRT2 = 0.70710678118654752f, RSQRT2PI = 0.39894228040143268f;
  const float z = fabsf(x) * RSQRT2;
  const float t = __fdividef(1.f, fmaf(P, z, 1.f));
  const float poly = t * fmaf(t, fmaf(t, fmaf(t, fmaf(t, A5, A4), A3), A2), A1);
  const float e = __expf(-0.5f * x * x);
  const float half_erfc = 0.5f * poly * e;
  cdf = x >= 0.f ? 1.f - half_erfc : half_erfc;
  pdf = RSQRT2PI * e;
}

__device__ __forceinline__ void mma_wait(uint64_t *bar, uint32_t parity, volatile int *abort,
                                         long long limit = WAIT_LIMIT) {
  if (mbar_try_wait(bar, parity)) return;
  if (*abort) return;
  if (!mbar_wait(bar, parity, limit)) {
    *abort = 1;
    record_device_error(-5 /* TTT_ERR_TIMEOUT */);
  }
}

__global__ void __launch_bounds__(THREADS, 1)
    mlp_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, as an offset into the shared array so that every
  // access through it stays a shared-memory access.
  uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qd = warp & 3;           // TMEM lane quarter of this warp
  const int half = (warp >> 2) & 1;  // hidden half of this thread
  const int th = warp >> 3;          // token half (tokens 8 th .. 8 th + 7) / d block
  const int hid = 128 * half + 32 * qd + lane;
  const int unit = blockIdx.x;
  const int head = unit % p.H;
  const int T = p.T;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
  uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + OFF_TSLOT);
  volatile int *abort = reinterpret_cast<volatile int *>(sm + OFF_ABORT);
  float *red = reinterpret_cast<float *>(sm + OFF_RED);
  const float *gam = reinterpret_cast<const float *>(sm + OFF_GB);
  const float *bet = gam + D;
  const uint32_t sbase = smem_u32(sm);

  if (tid == 0) {
    // P1, X3 and GW arrive once per half (two issuing warps); the drain once per
    // issuing warp.
    for (int i = 0; i < NUM_BARS; ++i)
      mbar_init(&bars[i], (i == BAR_P1 || i == BAR_X3 || i == BAR_GW) ? 2 : i == BAR_DRAIN ? 3 : 1);
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
  if (tid < D) {
    reinterpret_cast<float *>(sm + OFF_GB)[tid] = p.gamma[head * D + tid];
    reinterpret_cast<float *>(sm + OFF_GB)[D + tid] = p.beta[head * D + tid];
  }
  // The masked Q K^T tile keeps its K rows (0-7, 16-23) zero for good.
  for (int x = tid; x < 1024; x += THREADS) reinterpret_cast<float *>(sm + OFF_S1)[x] = 0.f;
  fence_proxy_async_smem();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tb = *tslot;
  const uint32_t tq = tmem_addr(tb, 32 * qd, 0);  // this warp's lane quarter

  // Writes 32 consecutive d of this thread's W2 row as fp16 into the W2 copy
  // (MN-major for W2^T: row = hidden unit, 64 d per 128-byte row).
  auto store_w2_row = [&](const uint32_t (&r)[32]) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      uint32_t h2[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        __half2 v = __floats2half2_rn(__uint_as_float(r[8 * u + 2 * e]), __uint_as_float(r[8 * u + 2 * e + 1]));
        h2[e] = *reinterpret_cast<uint32_t *>(&v);
      }
      *reinterpret_cast<uint4 *>(sm + OFF_W2 + swz16(hid, 32 * th + 8 * u)) = make_uint4(h2[0], h2[1], h2[2], h2[3]);
    }
  };

  // Initial state: this thread's 32 d of W1^T row `hid` and of W2 row `hid` into
  // TMEM; the W2 row also into the fp16 copy.
  {
    const float *w1 = p.W1_0 + (size_t)head * D * HID;
    const float *w2 = p.W2_0 + ((size_t)head * HID + hid) * D + 32 * th;
    uint32_t r[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(w1[(32 * th + e) * HID + hid]);
    tmem_st_32x32b_x16(tq + C_W1 + 64 * half + 32 * th, *reinterpret_cast<const uint32_t(*)[16]>(&r[0]));
    tmem_st_32x32b_x16(tq + C_W1 + 64 * half + 32 * th + 16, *reinterpret_cast<const uint32_t(*)[16]>(&r[16]));
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float4 v = reinterpret_cast<const float4 *>(w2)[e];
      r[4 * e] = __float_as_uint(v.x);
      r[4 * e + 1] = __float_as_uint(v.y);
      r[4 * e + 2] = __float_as_uint(v.z);
      r[4 * e + 3] = __float_as_uint(v.w);
    }
    tmem_st_32x32b_x16(tq + C_W2 + 64 * half + 32 * th, *reinterpret_cast<const uint32_t(*)[16]>(&r[0]));
    tmem_st_32x32b_x16(tq + C_W2 + 64 * half + 32 * th + 16, *reinterpret_cast<const uint32_t(*)[16]>(&r[16]));
    store_w2_row(r);
    tmem_wait_st();
  }

  const int nchunks = (T + CHUNK - 1) / CHUNK;
  const size_t tok_base = (size_t)unit * T;
  auto chunk_tokens = [&](int c) { return min(CHUNK, T - c * CHUNK); };
  int loads_issued = 0;
  auto issue_load = [&](int c) {
    const int s = c & 1;
    const int ntok = chunk_tokens(c);
    uint8_t *stg = sm + OFF_STG + s * STG_BYTES;
    mbar_arrive_expect_tx(&bars[BAR_LOAD0 + s], 3u * 8192u + (uint32_t)ntok * 4u);
    tma_load_3d(stg, &tmK, 0, c * CHUNK, unit, &bars[BAR_LOAD0 + s]);
    tma_load_3d(stg + 8192, &tmQ, 0, c * CHUNK, unit, &bars[BAR_LOAD0 + s]);
    tma_load_3d(stg + 16384, &tmV, 0, c * CHUNK, unit, &bars[BAR_LOAD0 + s]);
    bulk_load(sm + OFF_ETA + 256 * s, p.eta + tok_base + (size_t)c * CHUNK, (uint32_t)ntok * 4u,
              &bars[BAR_LOAD0 + s]);
    loads_issued = c + 1;
  };
  if (tid == 0) {
    if (nchunks > 0) issue_load(0);
    if (nchunks > 1) issue_load(1);
  }

  // Instruction descriptors.
  constexpr uint32_t ID_P1 = idesc_tf32_f32(128, 32, false, false, false);   // W1^T(TMEM) x [K;Q]
  constexpr uint32_t ID_X3 = idesc_f16_f32(64, 16, true, false, false);      // W2^T x X2 (and Zq2)
  constexpr uint32_t ID_GW = idesc_f16_f32(128, 16, false, false, false);    // W2 copy x G3, fp16
  constexpr uint32_t ID_UPD = idesc_tf32_f32(128, 64, false, true, true);    // state -= A(TMEM) B
  constexpr uint32_t ID_ZQ1 = idesc_tf32_f32(128, 32, false, false, true);   // P1 -= E2^T(TMEM) S1^T
  constexpr uint32_t ID_S1 = idesc_tf32_f32(128, 64, false, false, false);   // [K;Q] x K
  constexpr uint32_t ID_G2 = idesc_f16_f32(64, 64, false, false, false);     // Gram blocks
  constexpr uint32_t ID_ZC = idesc_tf32_f32(64, 16, true, false, false);     // Zq3 += E3^T S2u^T

  const uint32_t aW2 = sbase + OFF_W2, aKQ = sbase + OFF_KQ, aX2 = sbase + OFF_X2;
  const uint32_t aKM = sbase + OFF_KM, aZ2 = sbase + OFF_Z2, aG3 = sbase + OFF_G3;
  const uint32_t aE3 = sbase + OFF_E3, aS1 = sbase + OFF_S1, aS2U = sbase + OFF_S2U;

  // Phase counters of the MMA barriers (every thread waits on each in order).
  uint32_t n_s1c = 0, n_p1 = 0, n_x3 = 0, n_gw = 0, n_upd = 0, n_s2 = 0, n_zq3 = 0;

  // Products are issued by whole converged warps (one lane elected inside each
  // instruction's asm block) after a CTA barrier: warp 0 the chain's products and
  // the Gram, warp ZQ3_WARP Zq3 and its correction, then, with warp ZQ3_WARP + 1,
  // one half each of the next mini-batch's P1, so that P1 runs under the output LN.
  // Half h of P1 = W1^T [K;Q]^T for mini-batch m, committed on BAR_P1.
  auto issue_p1_half = [&](int m, int h) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint64_t b = smem_desc_sw128(aKQ + m * 4096 + (i >> 2) * 16384 + (i & 3) * 32, 16, 1024);
      umma_ts_tf32_w(tb + C_P1 + 32 * h, tb + C_W1 + 64 * h + 8 * i, b, ID_P1, i > 0);
    }
    umma_commit_w(&bars[BAR_P1]);
  };
  // W2^T (M = d, fp16) against a [16 token][hidden] fp16 operand (X2 or Zq2), hidden
  // steps i0 .. i1 - 1 of 16.
  auto issue_w2t = [&](uint32_t d_tmem, uint32_t aB, int i0 = 0, int i1 = 16) {
#pragma unroll
    for (int i = i0; i < i1; ++i) {
      const uint64_t a = smem_desc_sw128(aW2 + i * 2048, 8192, 1024);
      const uint64_t b = smem_desc_sw128(aB + (i >> 2) * 2048 + (i & 3) * 32, 16, 1024);
      umma_ss_w(d_tmem, a, b, ID_X3, i > i0);
    }
  };

  if (p.inject_timeout) mma_wait(&bars[BAR_NEVER], 0, abort, INJECTED_WAIT_LIMIT);

  for (int c = 0; c < nchunks && !*abort; ++c) {
    const int s = c & 1;
    const int ntok = chunk_tokens(c);
    const int nmb = ntok / MB;
    const uint8_t *stg = sm + OFF_STG + s * STG_BYTES;
    const float *eta_s = reinterpret_cast<const float *>(sm + OFF_ETA + 256 * s);
    mma_wait(&bars[BAR_LOAD0 + s], (uint32_t)(c >> 1) & 1u, abort);

    // ---- chunk head: K, Q (bf16, TMA) -> [K;Q] fp32 in the interleaved row order
    // (per mini-batch m: K 0-7, Q 0-7, K 8-15, Q 8-15 as 8-row groups 4m..4m+3).
    for (int x = tid; x < 2 * CHUNK * 16; x += THREADS) {
      const int isq = x >> 10, tc = (x >> 4) & 63, u = x & 15;
      const uint2 raw = *reinterpret_cast<const uint2 *>(
          stg + 8192 * isq + tc * 128 + ((((u >> 1) ^ tc) & 7) << 4) + (u & 1) * 8);
      const float2 lo = unpack_bf16x2(raw.x), hi = unpack_bf16x2(raw.y);
      const int m = tc >> 4, t = tc & 15;
      const int row = 8 * (4 * m + 2 * (t >> 3) + isq) + (t & 7);
      *reinterpret_cast<float4 *>(sm + OFF_KQ + (u >> 3) * 16384 + swz32(row, 4 * (u & 7))) =
          make_float4(lo.x, lo.y, hi.x, hi.y);
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == ZQ3_WARP || warp == ZQ3_WARP + 1) {
      __syncwarp();
      tc_fence_after_sync();
      issue_p1_half(0, warp - ZQ3_WARP);
      __syncwarp();
    }
    if (warp == 0) {
      __syncwarp();
      tc_fence_after_sync();
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t off = (i >> 2) * 16384 + (i & 3) * 32;
        umma_ss_tf32_w(tb + C_S1, smem_desc_sw128(aKQ + off, 16, 1024),
                       smem_desc_sw128(aKQ + off, 16, 2048), ID_S1, i > 0);
      }
      umma_commit_w(&bars[BAR_S1C]);
      __syncwarp();
    }

    for (int m = 0; m < nmb; ++m) {
      const int t0 = MB * m;  // first token of the mini-batch within the chunk
      // ---- X1 -> X2 = GELU(X1), GELU'(X1) (thread: hidden unit, 8 tokens) ----------
      mma_wait(&bars[BAR_P1], n_p1++ & 1u, abort);
      tc_fence_after_sync();
      __syncwarp();
      float d2[8];
      {
        uint32_t r[8];
        tmem_ld_32x32b_x8(tq + C_P1 + 32 * half + 16 * th, r);  // K tokens 8 th .. 8 th + 7
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float x1 = __uint_as_float(r[j]);
          float cdf, pdf;
          normal_cdf_pdf(x1, cdf, pdf);
          const float g = x1 * cdf;
          d2[j] = fmaf(x1, pdf, cdf);
          const int t = 8 * th + j;
          *reinterpret_cast<__half *>(sm + OFF_X2 + (hid >> 6) * 2048u + swz16(t, hid & 63)) = __float2half_rn(g);
          r[j] = __float_as_uint(round_tf32(g));
        }
        // X2^T over the consumed X1 columns: the A operand of the W2 update.
        tmem_st_32x32b_x8(tq + C_P1 + 32 * half + 16 * th, r);
        tmem_wait_st();
      }
      fence_proxy_async_smem();
      tc_fence_before_sync();
      __syncthreads();
      tc_fence_after_sync();
      // ---- X3^T = W2^T X2^T: hidden units 0-127 by warp 0 into lanes 0-15, 128-255
      // by warp ZQ3_WARP into lanes 16-31 of the same columns (summed when read) ----
      if (warp == 0 || warp == ZQ3_WARP) {
        __syncwarp();
        tc_fence_after_sync();
        if (warp == 0) issue_w2t(tb + C_X3, aX2, 0, 8);
        else issue_w2t(tmem_addr(tb, 16, C_X3), aX2, 8, 16);
        umma_commit_w(&bars[BAR_X3]);
        __syncwarp();
      }
      // K of the mini-batch, MN-major, for the W1 update (one float4 per thread).
      if (tid < 256) {
        const int t = tid >> 4, u = tid & 15, tc = t0 + t;
        const uint2 raw = *reinterpret_cast<const uint2 *>(
            stg + tc * 128 + ((((u >> 1) ^ tc) & 7) << 4) + (u & 1) * 8);
        const float2 lo = unpack_bf16x2(raw.x), hi = unpack_bf16x2(raw.y);
        *reinterpret_cast<float4 *>(sm + OFF_KM + (u >> 3) * 2048u + swzb32(t, 4 * (u & 7))) =
            make_float4(lo.x, lo.y, hi.x, hi.y);
      }
      mma_wait(&bars[BAR_X3], n_x3++ & 1u, abort);
      tc_fence_after_sync();
      __syncwarp();
      if (warp < 4) {
        uint32_t r[16];
        tmem_ld_32x32b_x16(tq + C_X3, r);  // lanes 0-15 / 16-31: the two hidden halves, d = 16 qd + lane % 16
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float v = __uint_as_float(r[j]) + __shfl_xor_sync(0xffffffffu, __uint_as_float(r[j]), 16);
          if (lane < 16) red[j * RS + 16 * qd + lane] = v;
        }
      }
      tc_fence_before_sync();
      __syncthreads();
      // ---- LN forward and backward of X3 (one warp per token, 2 d per lane) ------
      {
        const int t = warp, tc = t0 + t, dc = 2 * lane;
        const float2 x = *reinterpret_cast<const float2 *>(red + t * RS + dc);
        const float2 gm = *reinterpret_cast<const float2 *>(gam + dc);
        const float2 bt = *reinterpret_cast<const float2 *>(bet + dc);
        const uint32_t kvo = tc * 128 + ((((dc >> 3) ^ tc) & 7) << 4) + (dc & 7) * 2;
        const float2 kk = unpack_bf16x2(*reinterpret_cast<const uint32_t *>(stg + kvo));
        const float2 vv = unpack_bf16x2(*reinterpret_cast<const uint32_t *>(stg + 16384 + kvo));
        const float mean = warp_sum(x.x + x.y) * (1.f / D);
        const float d0 = x.x - mean, d1 = x.y - mean;
        const float r = rsqrtf(warp_sum(d0 * d0 + d1 * d1) * (1.f / D) + p.eps);
        const float h0 = d0 * r, h1 = d1 * r;
        // g = 2 (k + gamma xhat + beta - v); dl/dxhat = g gamma.
        const float a0 = 2.f * (kk.x + fmaf(gm.x, h0, bt.x) - vv.x) * gm.x;
        const float a1 = 2.f * (kk.y + fmaf(gm.y, h1, bt.y) - vv.y) * gm.y;
        const float ma = warp_sum(a0 + a1) * (1.f / D);
        const float mb = warp_sum(a0 * h0 + a1 * h1) * (1.f / D);
        const float g0 = r * (a0 - ma - h0 * mb), g1 = r * (a1 - ma - h1 * mb);
        const float e = eta_s[tc];
        const uint32_t blk = (dc >> 5) * 2048u;
        *reinterpret_cast<__half2 *>(sm + OFF_G3 + swz16(t, dc)) = __floats2half2_rn(g0, g1);
        *reinterpret_cast<float2 *>(sm + OFF_E3 + blk + swzb32(t, dc & 31)) =
            make_float2(round_tf32(e * g0), round_tf32(e * g1));
      }
      fence_proxy_async_smem();
      tc_fence_before_sync();
      __syncthreads();
      tc_fence_after_sync();
      // ---- GW^T = W2 G3^T: fp16, A = the W2 copy ([hidden][d], K-major), hidden
      // half h by warp 0 (h = 0) and warp ZQ3_WARP (h = 1) ---------------------------
      if (warp == 0 || warp == ZQ3_WARP) {
        __syncwarp();
        tc_fence_after_sync();
        const int h = warp == 0 ? 0 : 1;
#pragma unroll
        for (int k = 0; k < 4; ++k)
          umma_ss_w(tb + C_GW + 16 * h, smem_desc_sw128(aW2 + h * 16384 + 32 * k, 16, 1024),
                    smem_desc_sw128(aG3 + 32 * k, 16, 1024), ID_GW, k > 0);
        umma_commit_w(&bars[BAR_GW]);
        __syncwarp();
      }
      // ---- the masked Q K^T block of this mini-batch (warp m: its Q lanes) ---------
      if (m == 0) mma_wait(&bars[BAR_S1C], n_s1c++ & 1u, abort);
      tc_fence_after_sync();
      __syncwarp();
      if (warp == m) {
        uint32_t r[16];
        tmem_ld_32x32b_x16(tq + C_S1 + 16 * m, r);  // row = lane of quarter m, K tokens 0-15
        tmem_wait_ld();
        if (lane & 8) {  // Q rows: lanes 8-15 (tokens 0-7) and 24-31 (tokens 8-15)
          const int jq = (lane & 7) + 8 * (lane >> 4);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            float4 v;
            v.x = 4 * u + 0 <= jq ? round_tf32(__uint_as_float(r[4 * u + 0])) : 0.f;
            v.y = 4 * u + 1 <= jq ? round_tf32(__uint_as_float(r[4 * u + 1])) : 0.f;
            v.z = 4 * u + 2 <= jq ? round_tf32(__uint_as_float(r[4 * u + 2])) : 0.f;
            v.w = 4 * u + 3 <= jq ? round_tf32(__uint_as_float(r[4 * u + 3])) : 0.f;
            *reinterpret_cast<float4 *>(sm + OFF_S1 + swz32(lane, 4 * u)) = v;
          }
        }
      }
      // ---- G2 = GW * GELU'(X1), E2 = eta G2 (into TMEM over GW) ----------------------
      mma_wait(&bars[BAR_GW], n_gw++ & 1u, abort);
      tc_fence_after_sync();
      __syncwarp();
      {
        uint32_t r[8];
        tmem_ld_32x32b_x8(tq + C_GW + 16 * half + 8 * th, r);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 8; ++j)
          r[j] = __float_as_uint(round_tf32(eta_s[t0 + 8 * th + j] * (__uint_as_float(r[j]) * d2[j])));
        tmem_st_32x32b_x8(tq + C_GW + 16 * half + 8 * th, r);
        tmem_wait_st();
      }
      fence_proxy_async_smem();
      tc_fence_before_sync();
      __syncthreads();
      tc_fence_after_sync();
      // ---- W1^T -= E2^T K; W2 -= X2^T E3; Zq1 = P1_q - E2^T S1^T ----------------------
      if (warp == 0) {
        __syncwarp();
        tc_fence_after_sync();
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const uint64_t bk = smem_desc_sw128_b32(aKM + j * 1024, 2048, 512);
            const uint64_t be = smem_desc_sw128_b32(aE3 + j * 1024, 2048, 512);
            const uint64_t bs = smem_desc_sw128(aS1 + j * 32, 16, 1024);
            const uint32_t e2 = tb + C_GW + 16 * h + 8 * j;   // E2^T, tokens 8j..8j+7
            const uint32_t x2 = tb + C_P1 + 32 * h + 16 * j;  // X2^T, tokens 8j..8j+7
            umma_ts_tf32_w(tb + C_W1 + 64 * h, e2, bk, ID_UPD, true);
            umma_ts_tf32_w(tb + C_W2 + 64 * h, x2, be, ID_UPD, true);
            umma_ts_tf32_w(tb + C_P1 + 32 * h, e2, bs, ID_ZQ1, true);
          }
        umma_commit_w(&bars[BAR_UPD]);
        __syncwarp();
      }
      // ---- refresh the W2 copy from the updated state; Zq2 = GELU(Zq1) -------------
      mma_wait(&bars[BAR_UPD], n_upd++ & 1u, abort);
      tc_fence_after_sync();
      __syncwarp();
      {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tq + C_W2 + 64 * half + 32 * th, r);
        tmem_wait_ld();
        store_w2_row(r);
      }
      {
        uint32_t r[8];
        tmem_ld_32x32b_x8(tq + C_P1 + 32 * half + 8 + 16 * th, r);  // Q tokens 8 th .. 8 th + 7
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float z1 = __uint_as_float(r[j]);
          float cdf, pdf;
          normal_cdf_pdf(z1, cdf, pdf);
          *reinterpret_cast<__half *>(sm + OFF_Z2 + (hid >> 6) * 2048u + swz16(8 * th + j, hid & 63)) =
              __float2half_rn(z1 * cdf);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before_sync();
      __syncthreads();
      tc_fence_after_sync();
      // ---- the Gram of Zq2 X2^T (warp 0) and Zq3^T = W2'^T Zq2^T (warp ZQ3_WARP) ------
      if (warp == 0) {
        __syncwarp();
        tc_fence_after_sync();
#pragma unroll
        for (int i = 0; i < 4; ++i)
          umma_ss_w(tb + C_S2, smem_desc_sw128(aZ2 + i * 32, 16, 1024),
                    smem_desc_sw128(aX2 + i * 32, 16, 1024), ID_G2, i > 0);
        umma_commit_w(&bars[BAR_S2]);
        __syncwarp();
      }
      if (warp == ZQ3_WARP) {
        __syncwarp();
        tc_fence_after_sync();
        issue_w2t(tmem_addr(tb, 16, C_X3), aZ2);
        __syncwarp();
      }
      mma_wait(&bars[BAR_S2], n_s2++ & 1u, abort);
      tc_fence_after_sync();
      __syncwarp();
      if (warp < 4) {
        uint32_t r[16];
        tmem_ld_32x32b_x16(tq + C_S2 + 16 * qd, r);  // lanes 0-15: block qd, token lane
        tmem_wait_ld();
        if (lane < 16) {
#pragma unroll
          for (int j = 0; j < 16; ++j) red[(qd * 16 + lane) * 17 + j] = __uint_as_float(r[j]);
        }
      }
      tc_fence_before_sync();
      __syncthreads();
      if (tid < 256) {
        const int t = tid >> 4, sj = tid & 15;
        float v = 0.f;
#pragma unroll
        for (int g = 0; g < 4; ++g) v += red[(g * 16 + t) * 17 + sj];
        *reinterpret_cast<float *>(sm + OFF_S2U + swz32(t, sj)) = sj > t ? round_tf32(v) : 0.f;
      }
      fence_proxy_async_smem();
      tc_fence_before_sync();
      __syncthreads();
      tc_fence_after_sync();
      // ---- Zq3^T += E3^T striu(S2)^T (after Zq3, by the same warp); then the next
      // mini-batch's P1, which runs under the output LN ------------------------------
      if (warp == ZQ3_WARP) {
        __syncwarp();
        tc_fence_after_sync();
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const uint64_t a = smem_desc_sw128_b32(aE3 + j * 1024, 2048, 512);
          const uint64_t b = smem_desc_sw128(aS2U + j * 32, 16, 1024);
          umma_ss_tf32_w(tmem_addr(tb, 16, C_X3), a, b, ID_ZC, true);
        }
        umma_commit_w(&bars[BAR_ZQ3]);
        __syncwarp();
      }
      if ((warp == ZQ3_WARP || warp == ZQ3_WARP + 1) && m + 1 < nmb) {
        __syncwarp();
        tc_fence_after_sync();
        issue_p1_half(m + 1, warp - ZQ3_WARP);
        __syncwarp();
      }
      mma_wait(&bars[BAR_ZQ3], n_zq3++ & 1u, abort);
      tc_fence_after_sync();
      __syncwarp();
      if (warp < 4) {
        uint32_t r[16];
        tmem_ld_32x32b_x16(tq + C_X3, r);  // lanes 16-31: Zq3^T rows d = 16 qd + lane - 16
        tmem_wait_ld();
        if (lane >= 16) {
#pragma unroll
          for (int j = 0; j < 16; ++j) red[j * RS + 16 * qd + lane - 16] = __uint_as_float(r[j]);
        }
      }
      tc_fence_before_sync();
      __syncthreads();
      // ---- Z = Q + LN(Zq3) (one warp per token) --------------------------------------
      {
        const int t = warp, tc = t0 + t, dc = 2 * lane;
        const float2 x = *reinterpret_cast<const float2 *>(red + t * RS + dc);
        const float2 gm = *reinterpret_cast<const float2 *>(gam + dc);
        const float2 bt = *reinterpret_cast<const float2 *>(bet + dc);
        const float2 qq = unpack_bf16x2(*reinterpret_cast<const uint32_t *>(
            stg + 8192 + tc * 128 + ((((dc >> 3) ^ tc) & 7) << 4) + (dc & 7) * 2));
        const float mean = warp_sum(x.x + x.y) * (1.f / D);
        const float d0 = x.x - mean, d1 = x.y - mean;
        const float r = rsqrtf(warp_sum(d0 * d0 + d1 * d1) * (1.f / D) + p.eps);
        *reinterpret_cast<float2 *>(p.Z + (tok_base + (size_t)c * CHUNK + tc) * D + dc) =
            make_float2(qq.x + fmaf(gm.x, d0 * r, bt.x), qq.y + fmaf(gm.y, d1 * r, bt.y));
      }
      __syncthreads();  // the staging rows are rewritten by the next mini-batch
    }
    // The stage of chunk c is free: fetch chunk c + 2 into it.
    if (tid == 0 && c + 2 < nchunks && !*abort) issue_load(c + 2);
  }

  // An aborted CTA waits, with a bound, for its own loads and products in flight.
  __syncthreads();
  if (*abort) {
    if (tid == 0) {
      for (int k = 0; k < loads_issued; ++k)
        mbar_wait(&bars[BAR_LOAD0 + (k & 1)], (uint32_t)(k >> 1) & 1u, WAIT_LIMIT);
    }
    // Every warp that issues products commits once (a commit with nothing in flight
    // arrives at once), and those warps wait for all of them.
    const bool issuer = warp == 0 || warp == ZQ3_WARP || warp == ZQ3_WARP + 1;
    if (issuer) {
      __syncwarp();
      umma_commit_w(&bars[BAR_DRAIN]);
      __syncwarp();
      mbar_wait(&bars[BAR_DRAIN], 0, WAIT_LIMIT);
    }
    tc_fence_after_sync();
  }
  __syncthreads();
  tc_fence_after_sync();

  // Final state (every update has completed: each was waited on above).
  {
    float *w1 = p.W1_out + (size_t)unit * D * HID;
    float *w2 = p.W2_out + ((size_t)unit * HID + hid) * D + 32 * th;
    uint32_t r[32];
    tmem_ld_32x32b_x32(tq + C_W1 + 64 * half + 32 * th, r);
    tmem_wait_ld();
#pragma unroll
    for (int e = 0; e < 32; ++e) w1[(32 * th + e) * HID + hid] = __uint_as_float(r[e]);
    tmem_ld_32x32b_x32(tq + C_W2 + 64 * half + 32 * th, r);
    tmem_wait_ld();
#pragma unroll
    for (int e = 0; e < 8; ++e)
      reinterpret_cast<float4 *>(w2)[e] =
          make_float4(__uint_as_float(r[4 * e]), __uint_as_float(r[4 * e + 1]),
                      __uint_as_float(r[4 * e + 2]), __uint_as_float(r[4 * e + 3]));
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tb, TMEM_COLS);
  }
}

}  // namespace tcmlp
}  // namespace ttt
