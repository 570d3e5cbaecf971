// tc_linear.cuh - tensor-core (tcgen05) kernel of TTT-Linear and TTT-Linear +
// LN + residual for bf16 Q, K, V, d = 64, b = 16.
//
// Method: the dual form of the TTT write-up (§03.7) over mini-batches of b = 16
// tokens (§03.6), f(x) = x W or x + LN(x W) (§03.9), loss ||f(k; W) - v||^2
// (§03.5).
//
// Work decomposition.  One CTA of 4 warps owns one (batch, head) sequence for
// its whole length and keeps the fp32 state W in registers (in TMEM while the
// chain of a chunk runs, step 3 to 5).  Tokens are taken
// in chunks of 64 (four mini-batches), so that every tensor-core product has
// M = 128 rows: the 64 K rows and the 64 Q rows of the chunk.  With W_c the
// state at the start of the chunk and G_m the gradient of the loss w.r.t. the
// pre-activation of mini-batch m (taken at that mini-batch's own base state),
// W_m = W_c - sum_{j<m} K_j^T diag(eta_j) G_j, so that, exactly,
//   K_m W_m = (K W_c)_m - sum_{j<m} (K_m K_j^T) diag(eta_j) G_j
//   q_t W_t = (Q W_c)_t - sum_{s<=t} (q_t . k_s) eta_s G_s    (dual-form output)
//   W_next  = W_c - K^T diag(eta) G.
//
// Row layout of [K;Q] (= TMEM lanes of the products).  8-row group
// g = 8h + 2m + q holds tokens 16m + 8h + (0..7) of K (q = 0) or Q (q = 1): h
// is the half of mini-batch m.  So TMEM lane quarter w (warp w) holds half
// h = w / 2 of mini-batches 2(w % 2) and 2(w % 2) + 1, each as 8 K rows followed
// by the 8 Q rows of the same tokens (one 16-lane access returns both), every
// mini-batch is shared by two warps (m / 2 and 2 + m / 2), and the K rows alone
// sit in every other group (a uniform-stride operand: column n = 8i + r of
// S = [K;Q] K^T is token 16 (i % 4) + 8 (i / 4) + r).
//
// Per chunk:
//   1. TMA: K and Q (8-row boxes into that layout, 128-byte swizzle), V
//      (64 x 64), eta.
//   2. tcgen05: S = [K;Q] K^T (TMEM cols 64..127) and P = [K;Q] W_c (cols 0..63).
//   3. Every thread masks its own row of S in TMEM, in place, into the fp16 A
//      operand of step 4: K rows keep the columns of earlier mini-batches, Q
//      rows keep s <= t (the causal mask of the dual form, diagonal included);
//      it then parks its 32 state elements in its lane's S columns 96..127,
//      free until dW, and takes them back after its chain steps.
//   4. For m = 0..3, the two warps that hold mini-batch m read its K rows of P
//      (already corrected for mini-batches < m), compute G_m (LN backward in
//      registers, 16 elements per thread), write eta*G_m as fp16, turn their K
//      rows into fp16 in place, meet at a named barrier, and one of them issues
//      P -= A[:, m] (eta G_m) (A read from TMEM), which applies mini-batch m's
//      update to every later K row and every Q row at once.  Once their chain
//      steps are issued, the warps write the outputs of their Q rows, which are
//      final after their mini-batch's update (later updates add exactly zero to
//      them).
//   5. dW = K^T (eta G) on the tensor core (fp16) into the S columns (free
//      again); every thread updates its 32 fp32 state elements and rewrites the
//      bf16 hi + lo operand copy of W; then steps 1-3 of the next chunk follow
//      directly (the next K, V are fetched as soon as dW is done, each warp's Q
//      rows as soon as it has written its outputs).
// Precision: W enters P = [K;Q] W as a bf16 pair hi + lo (~2^-16 relative) against
// the exact bf16 K and Q; the masked Q K^T, eta*G and K enter the chain's
// corrections and dW as fp16 (2^-11 relative); accumulation is fp32 and the
// state stays fp32.
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
// Hardware named barriers (0 is __syncthreads): 1 and 2 pair the two warps of a
// chain step; NB_STATE_BACK gathers every warp's state back from TMEM before dW.
constexpr uint32_t NB_STATE_BACK = 3;
constexpr uint32_t TMEM_COLS = 128;

// Shared-memory map (bytes from a 1024-byte aligned base).
constexpr uint32_t OFF_A = 0;          // [K;Q] rows of the chunk in 8-row groups (see kq_group)
constexpr uint32_t OFF_WHI = 16384;    // W hi [d_in][d_out] bf16
constexpr uint32_t OFF_WLO = 24576;    // W lo
constexpr uint32_t OFF_GHI = 32768;    // eta*G [token][d_out] fp16
constexpr uint32_t OFF_GLO = 40960;    // V tile
constexpr uint32_t OFF_ETA = 49152;    // eta of the chunk, 64 floats
constexpr uint32_t OFF_GB = 49408;     // per column pair {gamma x2, beta x2}, 32 x 16 bytes
constexpr uint32_t OFF_UC = 49920;     // per column pair {2 gamma x2, 2 gamma beta x2}
constexpr uint32_t OFF_W2 = 50432;     // 2 gamma^2, 64 floats
constexpr uint32_t OFF_BAR = 50688;    // mbarriers (14 x 8 bytes)
constexpr uint32_t OFF_TSLOT = 50800;  // TMEM base address
constexpr uint32_t OFF_ABORT = 50804;  // set when a bounded wait expired
constexpr uint32_t SMEM_USED = 50808;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // + alignment slack

// 8-row group of token `row` of the chunk in the [K;Q] operand: K (q = 0) or Q
// (q = 1) of half (row / 8) % 2 of mini-batch row / 16.
__host__ __device__ __forceinline__ uint32_t kq_group(int row, int q) {
  return 8u * ((row >> 3) & 1) + 2u * (row >> 4) + (uint32_t)q;
}
__device__ __forceinline__ uint32_t kq_offset(int row, int q, int col) {
  return OFF_A + 1024u * kq_group(row, q) + sw128_offset(row & 7, col);
}

// One of the two lanes that a 16x256b load gives each thread (which = 0: lane
// base + i/4, which = 1: lane base + 8 + i/4), all 64 columns, as column pairs
// 8j + 2(i%4) + {0,1}; two 32-column loads keep the live registers low.
__device__ __forceinline__ void tmem_rows_16x256b(uint32_t taddr, int which, float2 (&y)[8]) {
  uint32_t r0[16], r1[16];
  tmem_ld_16x256b_x4(taddr, r0);
  tmem_ld_16x256b_x4(taddr + 32, r1);
  tmem_wait_ld();
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    y[j] = make_float2(__uint_as_float(r0[4 * j + 2 * which]), __uint_as_float(r0[4 * j + 2 * which + 1]));
    y[4 + j] = make_float2(__uint_as_float(r1[4 * j + 2 * which]), __uint_as_float(r1[4 * j + 2 * which + 1]));
  }
}

// mbarriers: K/V/eta loads; MMA S; updates of mini-batches 0,1,2; last update;
// dW; Q loads of warps 0..3; MMA P; the drain of an aborted CTA's products; one
// that nothing arrives at (the injected-timeout test).
enum {
  BAR_LOAD = 0, BAR_S = 1, BAR_C0 = 2, BAR_LAST = 5, BAR_DW = 6, BAR_LOADQ = 7, BAR_P = 11,
  BAR_DRAIN = 12, BAR_NEVER = 13, NUM_BARS = 14
};
// Bound of every wait (SM cycles, ~2 s) and of the injected one.
constexpr long long WAIT_LIMIT = 1ll << 32;
constexpr long long INJECTED_WAIT_LIMIT = 1ll << 20;

struct Params {
  const float *eta;
  const float *W0;
  const float *gamma, *beta;
  float eps;
  int H, T;
  float *Z;
  float *W_out;
  int inject_timeout;  // test hook: start with a wait that nothing completes
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
__device__ __forceinline__ void wait_or_abort(uint64_t *bar, uint32_t parity, volatile int *abort,
                                              long long limit = WAIT_LIMIT) {
  if (mbar_try_wait(bar, parity)) return;  // the common case: no shared-flag read
  if (*abort) return;
  if (!mbar_wait(bar, parity, limit)) {
    *abort = 1;
    record_device_error(-5 /* TTT_ERR_TIMEOUT */);
  }
}

// MINB = 4: <= 128 registers, so that 4 CTAs share an SM (a grid of up to 592
// units in one wave); MINB = 2: the register budget of 2 CTAs per SM, for grids
// that leave SMs to spare (the launch picks by wave count).
template <bool LN, int MINB = 4>
__global__ void __launch_bounds__(THREADS, MINB)
    linear_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, as an offset into the shared array so that every
  // access through it stays a shared-memory access.
  uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
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
  const int q4 = lane & 3;
  const int fr = lane >> 2;        // row within an 8-row group in the 16x256b layout
  const int mb0 = 2 * (warp & 1);  // this warp holds mini-batches mb0 and mb0 + 1 ...
  const int hh = warp >> 1;        // ... half hh of each

  if (tid == 0) {
    for (int i = 0; i < NUM_BARS; ++i) mbar_init(&bars[i], i == BAR_DRAIN ? 64 : 1);
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
    const float b = p.beta[head * D + tid];
    float *gb = reinterpret_cast<float *>(sm + OFF_GB + 16 * (tid >> 1)) + (tid & 1);
    float *uc = reinterpret_cast<float *>(sm + OFF_UC + 16 * (tid >> 1)) + (tid & 1);
    gb[0] = g;
    gb[2] = b;
    uc[0] = 2.f * g;
    uc[2] = 2.f * g * b;
    reinterpret_cast<float *>(sm + OFF_W2)[tid] = 2.f * g * g;
  }

  // Each thread owns 32 elements of the fp32 state: row wi, columns wc0..wc0+31
  // (the layout in which dW comes back from TMEM).
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
  auto chunk_tokens = [&](int c) { return min(CHUNK, T - c * CHUNK); };

  // Loads are split so that each tile is fetched as soon as its buffer is free:
  // each warp refills its own Q rows once it has written its outputs, thread 0
  // refills K / V / eta once dW is computed.
  // The last chunk whose loads this thread issued (thread 0: K, V, eta; lane 0
  // of each warp: its Q rows), for the drain of an aborted CTA.
  int kv_last = -1, q_last = -1;
  auto issue_loads_kv = [&](int c) {
    kv_last = c;
    const int ntok = chunk_tokens(c);
    mbar_arrive_expect_tx(&bars[BAR_LOAD], 8u * 1024u + 8192u + (uint32_t)ntok * 4u);
#pragma unroll
    for (int g = 0; g < 8; ++g)
      tma_load_3d(sm + OFF_A + 1024u * kq_group(8 * g, 0), &tmK, 0, c * CHUNK + 8 * g, unit, &bars[BAR_LOAD]);
    tma_load_3d(sm + OFF_GLO, &tmV, 0, c * CHUNK, unit, &bars[BAR_LOAD]);
    bulk_load(eta_s, p.eta + tok_base + (size_t)c * CHUNK, (uint32_t)ntok * 4u, &bars[BAR_LOAD]);
  };
  // This warp's 16 Q rows of chunk c, on the warp's own Q barrier.
  auto issue_load_q = [&](int c) {
    q_last = c;
    mbar_arrive_expect_tx(&bars[BAR_LOADQ + warp], 2048u);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int t0 = MB * (mb0 + i) + 8 * hh;
      tma_load_3d(sm + OFF_A + 1024u * kq_group(t0, 1), &tmQ, 0, c * CHUNK + t0, unit,
                  &bars[BAR_LOADQ + warp]);
    }
  };

  fence_proxy_async_smem();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tb = *tslot;
  const uint32_t tP = tb, tS = tb + 64;  // column bases of P and S (lane 0)
  if (tid == 0 && nchunks > 0) issue_loads_kv(0);
  if (lane == 0 && nchunks > 0) issue_load_q(0);

  constexpr uint32_t ID_P = idesc_bf16_f32(128, 64, false, true, false);   // [K;Q] x W
  constexpr uint32_t ID_S = idesc_bf16_f32(128, 64, false, false, false);  // [K;Q] x K^T
  constexpr uint32_t ID_UPD = idesc_f16_f32(128, 64, false, true, true);   // P -= A x (eta G), fp16
  constexpr uint32_t ID_DW = idesc_f16_f32(128, 64, true, true, false);    // [K^T;K^T] x (eta G), fp16

  // The P-independent part of the LN backward of this thread's K row of token
  // tk: u = 2 gamma (k + beta - v) = g2 (k - v) + g2b (or v for the plain linear
  // model) and mean(u), from k and v (kr, vr: bf16 pairs).
  uint32_t kr[8], vr[8];
  float2 u[8];
  float um = 0.f;
  auto load_kv = [&](int tk) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int col = 8 * j + 2 * q4;
      vr[j] = lds_u32(aGlo + sw128_offset(tk, col));
      kr[j] = lds_u32(sbase + kq_offset(tk, 0, col));
    }
  };
  auto make_u = [&]() {
    um = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float2 v = unpack_bf16x2(vr[j]);
      if (LN) {
        const float4 c = *reinterpret_cast<const float4 *>(sm + OFF_UC + 16 * (4 * j + q4));
        u[j] = __ffma2_rn(make_float2(c.x, c.y), __fsub2(unpack_bf16x2(kr[j]), v), make_float2(c.z, c.w));
        um += u[j].x + u[j].y;
      } else {
        u[j] = v;
      }
    }
    if (LN) um = quad_sum(um) * (1.f / D);
  };

  // Steps 1-3 of chunk c: wait for its tiles, issue S then P, mask S into the A
  // operand.  This thread's K and Q rows: token MB (mb0 + i) + 8 hh + fr, i = 0, 1.
  auto chunk_head = [&](int c) {
    const int ntok = chunk_tokens(c);
    const uint32_t par = (uint32_t)c & 1u;
    wait_or_abort(&bars[BAR_LOAD], par, abort);
#pragma unroll
    for (int w = 0; w < 4; ++w) wait_or_abort(&bars[BAR_LOADQ + w], par, abort);
    // Products are issued by one elected lane of a converged warp (the whole warp
    // computes the operand descriptors).  No product waits on the abort flag:
    // products issued after an expired wait are harmless (they complete, and the
    // drain at the end waits for them).
    if (warp == 0) {
      __syncwarp();
      tc_fence_after_sync();
      // S = [K;Q] K^T: B = the K rows alone (every other 8-row group, 2 KB apart).
#pragma unroll
      for (int k = 0; k < 4; ++k)
        umma_ss_w(tS, smem_desc_sw128(aA + 32 * k, 16, 1024), smem_desc_sw128(aA + 32 * k, 16, 2048), ID_S,
                  k > 0);
      umma_commit_w(&bars[BAR_S]);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint64_t ak = smem_desc_sw128(aA + 32 * k, 16, 1024);
        umma_ss_w(tP, ak, smem_desc_sw128(aWhi + 2048 * k, 8192, 1024), ID_P, k > 0);
        umma_ss_w(tP, ak, smem_desc_sw128(aWlo + 2048 * k, 8192, 1024), ID_P, true);
      }
      umma_commit_w(&bars[BAR_P]);
      __syncwarp();
    }
    if (ntok < CHUNK) {  // ragged last chunk: absent tokens contribute nothing to dW
      for (int x = tid; x < (CHUNK - ntok) * 32; x += THREADS) {
        const int row = ntok + x / 32, col = 2 * (x % 32);
        *reinterpret_cast<uint32_t *>(sm + OFF_GHI + sw128_offset(row, col)) = 0u;
      }
    }
    wait_or_abort(&bars[BAR_S], par, abort);
    tc_fence_after_sync();
    __syncwarp();  // lanes leave the wait loop independently; TMEM access is warp-collective
    {
      // This thread's row of [K;Q]: group 4 warp + lane / 8.
      const bool qrow = (lane >> 3) & 1;
      const int mrow = mb0 + (lane >> 4);             // its mini-batch
      const int t = MB * mrow + 8 * hh + (lane & 7);  // its token
      // A block j (tokens 16j..16j+15, natural order) is read from S columns
      // 8j..8j+7 (first half) and 32+8j..32+8j+7 (second half) and written back
      // as fp16 pairs over the first.  Blocks j > mb0 + 1 are zero for every row
      // of this warp (the choice is per warp: TMEM access is warp-collective).
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t pk[8];
        if (j <= mb0 + 1) {
          uint32_t v0[8], v1[8];
          tmem_ld_32x32b_x8(tmem_addr(tS, 32 * warp, 8 * j), v0);
          tmem_ld_32x32b_x8(tmem_addr(tS, 32 * warp, 32 + 8 * j), v1);
          tmem_wait_ld();
          const bool full = j < mrow;           // an earlier mini-batch: every column
          const bool diag = qrow && j == mrow;  // own mini-batch of a Q row: s <= t
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int s0 = MB * j + 2 * e;
            const uint32_t b0 = e < 4 ? v0[2 * e] : v1[2 * e - 8];
            const uint32_t b1 = e < 4 ? v0[2 * e + 1] : v1[2 * e - 7];
            const float a0 = (full || (diag && s0 <= t)) ? __uint_as_float(b0) : 0.f;
            const float a1 = (full || (diag && s0 + 1 <= t)) ? __uint_as_float(b1) : 0.f;
            pk[e] = pack_f16x2(a0, a1);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) pk[e] = 0u;
        }
        tmem_st_32x32b_x8(tmem_addr(tS, 32 * warp, 8 * j), pk);
      }
      // The fp32 state waits out the chain in this thread's TMEM lane, S columns
      // 32-63 (free from here until dW), so that its 32 registers serve the chain.
      {
        uint32_t w0r[16], w1r[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          w0r[e] = __float_as_uint(wm[e]);
          w1r[e] = __float_as_uint(wm[16 + e]);
        }
        tmem_st_32x32b_x16(tmem_addr(tS, 32 * warp, 32), w0r);
        tmem_st_32x32b_x16(tmem_addr(tS, 32 * warp, 48), w1r);
      }
      tmem_wait_st();
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
  };

  if (p.inject_timeout) wait_or_abort(&bars[BAR_NEVER], 0, abort, INJECTED_WAIT_LIMIT);
  if (nchunks > 0) chunk_head(0);

  for (int c = 0; c < nchunks; ++c) {
    const int ntok = chunk_tokens(c);
    const int nmb = ntok / MB;
    const uint32_t par = (uint32_t)c & 1u;

    // ---- 4: the mini-batch chain: mini-batch m on warps m/2 and 2 + m/2 ---------------
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int m = mb0 + i;
      if (m >= nmb) break;
      const int tk = MB * m + 8 * hh + fr;  // token of this thread's K row
      const float e0 = eta_s[tk];
      // The P-independent part of the LN backward, while the previous update is
      // in flight.
      load_kv(tk);
      make_u();
      // This thread's K row elements become fp16 in place (the dW operand); P and
      // S, the bf16 readers, are complete.  Under the 4-CTA register cap this is
      // done before the wait, so that the K elements are not held through the LN
      // backward.
      auto k_to_f16 = [&]() {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float2 k2 = unpack_bf16x2(kr[j]);
          *reinterpret_cast<uint32_t *>(sm + kq_offset(tk, 0, 8 * j + 2 * q4)) = pack_f16x2(k2.x, k2.y);
        }
      };
      if (MINB == 4) k_to_f16();
      wait_or_abort(&bars[m == 0 ? BAR_P : BAR_C0 + m - 1], par, abort);
      tc_fence_after_sync();
      __syncwarp();
      float2 y[8];
      tmem_rows_16x256b(tmem_addr(tP, 32 * warp + 16 * i, 0), 0, y);
      // Stores eta * (dl/dy) of one column pair as fp16.
      auto store_grad = [&](int col, float2 g) {
        *reinterpret_cast<uint32_t *>(sm + OFF_GHI + sw128_offset(tk, col)) = pack_f16x2(g.x, g.y);
      };
      if (!LN) {
        // dl/dy = 2 (y - v)
        const float2 f = make_float2(2.f * e0, 2.f * e0);
#pragma unroll
        for (int j = 0; j < 8; ++j) store_grad(8 * j + 2 * q4, __fmul2_rn(f, __fsub2(y[j], u[j])));
      } else {
        // LN backward of ||k + gamma xhat + beta - v||^2 w.r.t. y.  With
        // dx = dl/dxhat = u + w xhat (w = 2 gamma^2), A = mean(dx), B = mean(dx xhat):
        // dl/dy = r (dx - A - xhat B) = r (u + xhat (w - B) - A), r = 1/std(y).
        // With d = y - mean(y) and xhat = r d, every sum needed is a sum over d:
        // A = mean(u) + r sum(w d) / D, B = r sum(u d) / D + r^2 sum(w d^2) / D,
        // so one reduction round follows the one for the mean.
        const float mean = quad_sum(sum8(y)) * (1.f / D);
        const float2 nm = make_float2(-mean, -mean);
        float2 w2[8];
        float2 sdd = make_float2(0.f, 0.f), swd = sdd, swdd = sdd, sud = sdd;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          w2[j] = *reinterpret_cast<const float2 *>(sm + OFF_W2 + 4 * (8 * j + 2 * q4));
          y[j] = __fadd2_rn(y[j], nm);  // d
          const float2 t = __fmul2_rn(w2[j], y[j]);
          swd = __fadd2_rn(swd, t);
          swdd = __ffma2_rn(t, y[j], swdd);
          sdd = __ffma2_rn(y[j], y[j], sdd);
          sud = __ffma2_rn(u[j], y[j], sud);
        }
        const float vdd = quad_sum(sdd.x + sdd.y), vwd = quad_sum(swd.x + swd.y);
        const float vwdd = quad_sum(swdd.x + swdd.y), vud = quad_sum(sud.x + sud.y);
        const float r = rsqrtf(vdd * (1.f / D) + p.eps);
        const float A = um + r * vwd * (1.f / D);
        const float B = (r * vud + r * r * vwdd) * (1.f / D);
        const float2 f = make_float2(e0 * r, e0 * r), rr = make_float2(r, r);
        const float2 nA = make_float2(-A, -A), nB = make_float2(-B, -B);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float2 xh = __fmul2_rn(y[j], rr);
          store_grad(8 * j + 2 * q4, __fmul2_rn(f, __fadd2_rn(__ffma2_rn(xh, __fadd2_rn(w2[j], nB), u[j]), nA)));
        }
      }
      if (MINB != 4) k_to_f16();
      // Both halves of eta*G_m written: the pair's first warp issues the update.
      fence_proxy_async_smem();
      tc_fence_before_sync();
      named_barrier_sync(1 + (warp & 1), 64);
      if (hh == 0) {
        __syncwarp();
        tc_fence_after_sync();
        umma_ts_w(tP, tS + 8 * m, smem_desc_sw128(aGhi + 2048 * m, 8192, 1024), ID_UPD, true);
        umma_commit_w(&bars[m == nmb - 1 ? BAR_LAST : BAR_C0 + m]);
        __syncwarp();
      }
    }

    // The state back from TMEM; warps 1-3 count themselves toward the named
    // barrier NB_STATE_BACK, which warp 0 waits on before dW overwrites those columns.
    {
      uint32_t r0[16], r1[16];
      tmem_ld_32x32b_x16(tmem_addr(tS, 32 * warp, 32), r0);
      tmem_ld_32x32b_x16(tmem_addr(tS, 32 * warp, 48), r1);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        wm[e] = __uint_as_float(r0[e]);
        wm[16 + e] = __uint_as_float(r1[e]);
      }
      tc_fence_before_sync();
      if (warp != 0) named_barrier_arrive(NB_STATE_BACK, THREADS);
    }
    // Outputs of this warp's Q rows: after their mini-batch's update they are
    // final (later updates add exactly zero to them, A being zero there).
    float *Zc = p.Z + (tok_base + (size_t)c * CHUNK) * D;
    // Q residuals of both rows first, so that the Q rows can be refilled with the
    // next chunk before the outputs are computed.
    uint32_t qres[2][8];
    if (LN) {
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j)
          qres[i][j] = lds_u32(sbase + kq_offset(MB * (mb0 + i) + 8 * hh + fr, 1, 8 * j + 2 * q4));
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0 && c + 1 < nchunks && !*abort) issue_load_q(c + 1);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int m = mb0 + i;
      if (m >= nmb) break;
      const int tq = MB * m + 8 * hh + fr;  // token of this thread's Q row
      wait_or_abort(&bars[m == nmb - 1 ? BAR_LAST : BAR_C0 + m], par, abort);
      tc_fence_after_sync();
      __syncwarp();
      float2 z[8];
      tmem_rows_16x256b(tmem_addr(tP, 32 * warp + 16 * i, 0), 1, z);
      float *zrow = Zc + tq * D;
      if (LN) {
        const float mean = quad_sum(sum8(z)) * (1.f / D);
        const float2 nm = make_float2(-mean, -mean);
        float2 qa = make_float2(0.f, 0.f), qb = qa;
#pragma unroll
        for (int j = 0; j < 8; j += 2) {
          z[j] = __fadd2_rn(z[j], nm);
          z[j + 1] = __fadd2_rn(z[j + 1], nm);
          qa = __ffma2_rn(z[j], z[j], qa);
          qb = __ffma2_rn(z[j + 1], z[j + 1], qb);
        }
        const float rstd = rsqrtf(quad_sum((qa.x + qb.x) + (qa.y + qb.y)) * (1.f / D) + p.eps);
        const float2 rs = make_float2(rstd, rstd);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int col = 8 * j + 2 * q4;
          const float4 gb = *reinterpret_cast<const float4 *>(sm + OFF_GB + 16 * (4 * j + q4));
          const float2 gm = make_float2(gb.x, gb.y), bt = make_float2(gb.z, gb.w);
          const float2 q = unpack_bf16x2(qres[i][j]);
          *reinterpret_cast<float2 *>(zrow + col) = __fadd2_rn(q, __ffma2_rn(gm, __fmul2_rn(z[j], rs), bt));
        }
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) *reinterpret_cast<float2 *>(zrow + 8 * j + 2 * q4) = z[j];
      }
    }

    // ---- 5: dW on the tensor core after the last update; state update -------------
    wait_or_abort(&bars[BAR_LAST], par, abort);
    tc_fence_after_sync();
    if (warp == 0) {
      named_barrier_sync(NB_STATE_BACK, THREADS);  // every warp has its state back
      tc_fence_after_sync();
      __syncwarp();
      // dW = K^T (eta G) into the S columns (their operand is consumed).  Step k
      // takes the K rows of groups 4k and 4k + 2 (tokens of mini-batches
      // 2(k % 2), 2(k % 2) + 1, half k / 2), read twice (lbo 0) so that rows
      // 64..127 repeat rows 0..63 for warps 2-3, against the eta*G rows of the
      // same tokens (two 8-row groups 2 KB apart).
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint64_t ak = smem_desc_sw128(aA + 4096 * k, 0, 2048);
        const uint32_t gk = 4096u * (k & 1) + 1024u * (k >> 1);
        umma_ss_w(tS, ak, smem_desc_sw128(aGhi + gk, 8192, 2048), ID_DW, k > 0);
      }
      umma_commit_w(&bars[BAR_DW]);
      __syncwarp();
    }
    wait_or_abort(&bars[BAR_DW], par, abort);
    tc_fence_after_sync();
    __syncwarp();
    // K, V and eta are free once dW is done; every thread passed
    // this chunk's wait on their barrier in the chunk head.
    if (tid == 0 && c + 1 < nchunks && !*abort) issue_loads_kv(c + 1);
    {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t dw[16];
        tmem_ld_32x32b_x16(tmem_addr(tS, 32 * warp, wc0 + 16 * h), dw);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) wm[16 * h + e] -= __uint_as_float(dw[e]);
      }
      write_w_operand();
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();  // P and S of this chunk fully consumed; W operand written
    tc_fence_after_sync();
    if (*abort) break;
    if (c + 1 < nchunks) chunk_head(c + 1);
  }

  // An aborted CTA (a wait ran past its bound) waits, again with a bound, for
  // its own loads and products still in flight before it frees TMEM and exits.
  __syncthreads();
  if (*abort) {
    if (tid == 0 && kv_last >= 0) mbar_wait(&bars[BAR_LOAD], (uint32_t)kv_last & 1u, WAIT_LIMIT);
    if (lane == 0 && q_last >= 0) mbar_wait(&bars[BAR_LOADQ + warp], (uint32_t)q_last & 1u, WAIT_LIMIT);
    if (warp < 2) umma_commit(&bars[BAR_DRAIN]);  // every thread that may have issued products
    mbar_wait(&bars[BAR_DRAIN], 0, WAIT_LIMIT);
    tc_fence_after_sync();
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
