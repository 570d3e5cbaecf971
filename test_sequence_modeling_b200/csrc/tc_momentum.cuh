// tc_momentum.cuh - tensor-core (tcgen05) forward of TTT-Linear and TTT-Linear +
// LN with the momentum and decay update of the Titans article (§二.1(2): momentum
// on past surprise, a forget gate that decays the memory), kept to the TTT
// mini-batch rule (§03.6: every gradient of a mini-batch taken at its base
// state), for bf16 Q, K, V, d = 64, b = 16.
//
// Per token t, with g_t = k_t^T G_t the loss gradient at the base of t's
// mini-batch:  S_t = alpha_t S_{t-1} - eta_t g_t,  W_t = (1 - lambda_t) W_{t-1} + S_t.
//
// Dual form over a 64-token chunk with initial state (W_c, S_c), tokens
// tau, sigma = 0..63 of the chunk: the recursion is linear in W_c, S_c and the
// gradients, so
//   W_tau = Lam_tau W_c + C_tau S_c - sum_{sigma <= tau} c_{tau,sigma} eta_sigma g_sigma
//   S_tau = A_tau S_c            - sum_{sigma <= tau} a_{tau,sigma} eta_sigma g_sigma
// with Lam_tau = prod_{r <= tau} (1 - lambda_r), A_tau = prod_{r <= tau} alpha_r,
// C_tau = (1 - lambda_tau) C_{tau-1} + A_tau, a_{tau,sigma} = prod_{sigma < r <= tau}
// alpha_r and c_{tau,sigma} = (1 - lambda_tau) c_{tau-1,sigma} + a_{tau,sigma}
// (c_{s,s} = a_{s,s} = 1).  Walking sigma down from tau, with
// D_{tau,sigma} = prod_{sigma < v <= tau} (1 - lambda_v), the same coefficients
// follow without a division: c_{tau,sigma} = D_{tau,sigma} + alpha_{sigma+1}
// c_{tau,sigma+1}.  Hence, with X = [K;Q] W_c and Y = [K;Q] S_c,
//   K rows of mini-batch m (base = the state after token 16 m - 1):
//     k W_base = Lam_{16m-1} X + C_{16m-1} Y - sum_{sigma < 16m} c_{16m-1,sigma} eta (k . k_sigma) G_sigma
//   Q row of token tau:
//     q W_tau  = Lam_tau X + C_tau Y - sum_{sigma <= tau} c_{tau,sigma} eta (q . k_sigma) G_sigma
// (Lam_{-1} = 1, C_{-1} = 0).  The corrections are the linear kernel's chain with
// the causal 0/1 mask replaced by the coefficients, accumulated in a third
// accumulator; the next chunk's state is
//   W = Lam_L W_c + C_L S_c - (diag(c_{L,.}) K)^T (eta G),
//   S = A_L S_c - (diag(a_{L,.}) K)^T (eta G)      (L = the chunk's last token).
// alpha = lambda = 0 gives Lam = 1, C = 0, c = a = the causal mask: the TTT
// forward.
//
// Layout: the linear kernel's (one CTA of 4 warps per unit, [K;Q] rows in 8-row
// groups, each mini-batch's chain step shared by two warps), W and S in registers
// (fp32) and as bf16 hi + lo operands.  The chunk head computes X, Y and the
// Gram S = [K;Q] K^T on the tensor cores while one warp builds the coefficient
// table c_{tau,sigma} (a walk down each column sigma, tau ascending:
// c_{tau,sigma} = (1 - lambda_tau) c_{tau-1,sigma} + a_{tau,sigma}) and another
// the prefix scans; every thread then scales its row of S by its coefficient row
// (fp16, packed in place) and folds its rows of X and Y into one accumulator
// P = rho X + kappa Y, which the chain's corrections decrement.  The state update
// MMAs follow the last chain step directly, overlapping the last outputs.  TMEM:
// P, Y (then dS), dW, S: 256 columns, 2 CTAs per SM.  Precision: X, Y exact bf16
// K, Q against hi + lo pairs; the coefficient-weighted Gram, eta G and the
// weighted K of the state update as fp16; fp32 accumulation.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "device_status.cuh"
#include "sm100.cuh"
#include "tc_linear.cuh"

namespace ttt {
namespace tcmom {

using namespace ::ttt::sm100;
using ::ttt::tc::CHUNK;
using ::ttt::tc::D;
using ::ttt::tc::kq_group;
using ::ttt::tc::kq_offset;
using ::ttt::tc::MB;
using ::ttt::tc::quad_sum;
using ::ttt::tc::sum8;
using ::ttt::tc::THREADS;
using ::ttt::tc::tmem_rows_16x256b;
using ::ttt::tc::wait_or_abort;
using ::ttt::tc::WAIT_LIMIT;
using ::ttt::tc::INJECTED_WAIT_LIMIT;

constexpr uint32_t TMEM_COLS = 256;

// Shared-memory map (bytes from a 1024-byte aligned base).
constexpr uint32_t OFF_A = 0;          // [K;Q] rows in 8-row groups (tc::kq_group); K rows later c-weighted fp16
constexpr uint32_t OFF_WHI = 16384;    // W hi [d_in][d_out] bf16
constexpr uint32_t OFF_WLO = 24576;    // W lo
constexpr uint32_t OFF_SHI = 32768;    // S hi (W hi + 16 KB: the second atom of one B operand)
constexpr uint32_t OFF_SLO = 40960;    // S lo
constexpr uint32_t OFF_G = 49152;      // eta*G [token][d_out] fp16
constexpr uint32_t OFF_V = 57344;      // V tile; then a-weighted K [token][d_in] fp16 (natural order)
constexpr uint32_t OFF_ETA = 65536;    // eta, alpha, lambda of the chunk: 64 floats each
constexpr uint32_t OFF_ALPHA = 65792;
constexpr uint32_t OFF_LAM = 66048;
constexpr uint32_t OFF_PL = 66304;     // Lam_tau
constexpr uint32_t OFF_CC = 66560;     // C_tau
constexpr uint32_t OFF_CW = 66816;     // c_{L,sigma}
constexpr uint32_t OFF_AW = 67072;     // a_{L,sigma}
constexpr uint32_t OFF_FIN = 67328;    // Lam_L, C_L, A_L
constexpr uint32_t OFF_GB = 67344;     // per column pair {gamma x2, beta x2}
constexpr uint32_t OFF_UC = 67856;     // per column pair {2 gamma x2, 2 gamma beta x2}
constexpr uint32_t OFF_W2 = 68368;     // 2 gamma^2, 64 floats
constexpr uint32_t OFF_BAR = 68624;    // mbarriers (14 x 8 bytes)
constexpr uint32_t OFF_TSLOT = 68736;
constexpr uint32_t OFF_ABORT = 68740;
constexpr uint32_t OFF_COEF = 68752;   // c_{tau,sigma} [tau][sigma], fp32, row stride COEF_LD
constexpr int COEF_LD = 68;            // 17 x 16 bytes: 8 consecutive rows hit 8 distinct bank groups
constexpr uint32_t SMEM_USED = OFF_COEF + CHUNK * COEF_LD * 4;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;

enum {
  BAR_LOAD = 0, BAR_S = 1, BAR_C0 = 2, BAR_LAST = 5, BAR_DW = 6, BAR_LOADQ = 7, BAR_P = 11,
  BAR_DRAIN = 12, BAR_NEVER = 13, NUM_BARS = 14
};

struct Params {
  const float *eta, *alpha, *lambda;  // [units][T]
  const float *W0;                    // [H][D][D]
  const float *gamma, *beta;          // [H][D] (with LN only)
  float eps;
  int H, T;
  float *Z;                           // [units][T][D]
  float *W_out, *S_out;               // [units][D][D]
  int inject_timeout;
};

__device__ __forceinline__ float2 fsub2(float2 a, float2 b) { return __fadd2_rn(a, make_float2(-b.x, -b.y)); }

// Inclusive scan over the 64 tokens of the chunk (2 per lane: tokens lane and
// lane + 32) of x_t = d_t x_{t-1} + e_t, x_{-1} = 0: the composition of affine
// maps (d, e).  Returns x for both tokens of this lane.
__device__ __forceinline__ void affine_scan64(float (&d)[2], float (&e)[2], int lane) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const float pd = __shfl_up_sync(0xffffffffu, d[h], off);
      const float pe = __shfl_up_sync(0xffffffffu, e[h], off);
      if (lane >= off) {
        e[h] = fmaf(d[h], pe, e[h]);
        d[h] = pd * d[h];
      }
    }
  }
  // The second half continues from the first half's total (lane 31).
  const float td = __shfl_sync(0xffffffffu, d[0], 31), te = __shfl_sync(0xffffffffu, e[0], 31);
  e[1] = fmaf(d[1], te, e[1]);
  d[1] = td * d[1];
}

template <bool LN>
__global__ void __launch_bounds__(THREADS, 2)
    momentum_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int unit = blockIdx.x;
  const int head = unit % p.H;
  const int T = p.T;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
  uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + OFF_TSLOT);
  volatile int *abort = reinterpret_cast<volatile int *>(sm + OFF_ABORT);
  float *eta_s = reinterpret_cast<float *>(sm + OFF_ETA);
  float *alpha_s = reinterpret_cast<float *>(sm + OFF_ALPHA);
  float *lam_s = reinterpret_cast<float *>(sm + OFF_LAM);
  float *PL = reinterpret_cast<float *>(sm + OFF_PL);
  float *CC = reinterpret_cast<float *>(sm + OFF_CC);
  float *CW = reinterpret_cast<float *>(sm + OFF_CW);
  float *AW = reinterpret_cast<float *>(sm + OFF_AW);
  float *FIN = reinterpret_cast<float *>(sm + OFF_FIN);
  float *COEF = reinterpret_cast<float *>(sm + OFF_COEF);
  const uint32_t sbase = smem_u32(sm);
  const uint32_t aA = sbase + OFF_A;
  const uint32_t aWhi = sbase + OFF_WHI, aWlo = sbase + OFF_WLO;  // S hi, lo: 16 KB further
  const uint32_t aG = sbase + OFF_G, aV = sbase + OFF_V;
  const int q4 = lane & 3;
  const int fr = lane >> 2;
  const int mb0 = 2 * (warp & 1);
  const int hh = warp >> 1;

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
  if (tid < D) {
    const float g = LN ? p.gamma[head * D + tid] : 1.f;
    const float b = LN ? p.beta[head * D + tid] : 0.f;
    float *gb = reinterpret_cast<float *>(sm + OFF_GB + 16 * (tid >> 1)) + (tid & 1);
    float *uc = reinterpret_cast<float *>(sm + OFF_UC + 16 * (tid >> 1)) + (tid & 1);
    gb[0] = g;
    gb[2] = b;
    uc[0] = 2.f * g;
    uc[2] = 2.f * g * b;
    reinterpret_cast<float *>(sm + OFF_W2)[tid] = 2.f * g * g;
  }

  // This thread's 32 elements of W and S: row wi, columns wc0 .. wc0 + 31.
  const int wi = 32 * (warp & 1) + lane;
  const int wc0 = 32 * (warp >> 1);
  float wm[32], sv[32];
  {
    const float4 *src = reinterpret_cast<const float4 *>(p.W0 + (size_t)head * D * D + wi * D + wc0);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float4 v = src[q];
      wm[4 * q] = v.x;
      wm[4 * q + 1] = v.y;
      wm[4 * q + 2] = v.z;
      wm[4 * q + 3] = v.w;
    }
#pragma unroll
    for (int e = 0; e < 32; ++e) sv[e] = 0.f;
  }
  // bf16 hi + lo copies of this thread's part of W and S (the B operands of X, Y).
  auto write_operands = [&]() {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t hi[4], lo[4], shi[4], slo[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        split_bf16x2(wm[8 * q + 2 * e], wm[8 * q + 2 * e + 1], hi[e], lo[e]);
        split_bf16x2(sv[8 * q + 2 * e], sv[8 * q + 2 * e + 1], shi[e], slo[e]);
      }
      const uint32_t off = sw128_offset(wi, wc0 + 8 * q);
      *reinterpret_cast<uint4 *>(sm + OFF_WHI + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<uint4 *>(sm + OFF_WLO + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      *reinterpret_cast<uint4 *>(sm + OFF_SHI + off) = make_uint4(shi[0], shi[1], shi[2], shi[3]);
      *reinterpret_cast<uint4 *>(sm + OFF_SLO + off) = make_uint4(slo[0], slo[1], slo[2], slo[3]);
    }
  };
  write_operands();

  const int nchunks = (T + CHUNK - 1) / CHUNK;
  const size_t tok_base = (size_t)unit * T;
  auto chunk_tokens = [&](int c) { return min(CHUNK, T - c * CHUNK); };

  int kv_last = -1, q_last = -1;
  auto issue_loads_kv = [&](int c) {
    kv_last = c;
    const int ntok = chunk_tokens(c);
    mbar_arrive_expect_tx(&bars[BAR_LOAD], 8u * 1024u + 8192u + 3u * (uint32_t)ntok * 4u);
#pragma unroll
    for (int g = 0; g < 8; ++g)
      tma_load_3d(sm + OFF_A + 1024u * kq_group(8 * g, 0), &tmK, 0, c * CHUNK + 8 * g, unit, &bars[BAR_LOAD]);
    tma_load_3d(sm + OFF_V, &tmV, 0, c * CHUNK, unit, &bars[BAR_LOAD]);
    const size_t t0 = tok_base + (size_t)c * CHUNK;
    bulk_load(eta_s, p.eta + t0, (uint32_t)ntok * 4u, &bars[BAR_LOAD]);
    bulk_load(alpha_s, p.alpha + t0, (uint32_t)ntok * 4u, &bars[BAR_LOAD]);
    bulk_load(lam_s, p.lambda + t0, (uint32_t)ntok * 4u, &bars[BAR_LOAD]);
  };
  auto issue_load_q = [&](int c) {
    q_last = c;
    mbar_arrive_expect_tx(&bars[BAR_LOADQ + warp], 2048u);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int t0 = MB * (mb0 + i) + 8 * hh;
      tma_load_3d(sm + OFF_A + 1024u * kq_group(t0, 1), &tmQ, 0, c * CHUNK + t0, unit, &bars[BAR_LOADQ + warp]);
    }
  };

  fence_proxy_async_smem();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tb = *tslot;
  // P (first X), Y (then dS), dW, S.
  const uint32_t tX = tb, tY = tb + 64, tC = tb + 128, tS = tb + 192;
  if (tid == 0 && nchunks > 0) issue_loads_kv(0);
  if (lane == 0 && nchunks > 0) issue_load_q(0);

  constexpr uint32_t ID_S = idesc_bf16_f32(128, 64, false, false, false);   // [K;Q] x K^T
  constexpr uint32_t ID_P2 = idesc_bf16_f32(128, 128, false, true, false);  // [K;Q] x [W | S]
  constexpr uint32_t ID_CORR = idesc_f16_f32(128, 64, false, true, true);   // P -= A' x (eta G)
  constexpr uint32_t ID_DW = idesc_f16_f32(128, 64, true, true, false);     // [K'^T;K'^T] x (eta G)

  uint32_t kr[8], vr[8];
  float2 u[8];
  float um = 0.f;
  auto load_kv = [&](int tk) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int col = 8 * j + 2 * q4;
      vr[j] = lds_u32(aV + sw128_offset(tk, col));
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
        u[j] = __ffma2_rn(make_float2(c.x, c.y), fsub2(unpack_bf16x2(kr[j]), v), make_float2(c.z, c.w));
        um += u[j].x + u[j].y;
      } else {
        u[j] = v;  // the plain model's target
      }
    }
    if (LN) um = quad_sum(um) * (1.f / D);
  };
  // P = rho X + kappa Y - corrections of this thread's K (which = 0) or Q (which = 1)
  // row of the 16-lane block i.
  auto read_p = [&](int i, int which, float2 (&y)[8]) {
    tmem_rows_16x256b(tmem_addr(tX, 32 * warp + 16 * i, 0), which, y);
  };

  // The Q residuals of this thread's two output rows (read at the chunk head, so
  // that the next chunk's Q tile can load under the chain).
  uint32_t qres[2][8];

  // Chunk head: wait for the tiles; issue S, X, Y; the prefix scans (warp 2) and the
  // coefficient table (warp 3); every thread's row of the coefficient-weighted Gram
  // (the fp16 A operand) and of P = rho X + kappa Y; the Q residuals.
  auto chunk_head = [&](int c) {
    const int ntok = chunk_tokens(c);
    const uint32_t par = (uint32_t)c & 1u;
    wait_or_abort(&bars[BAR_LOAD], par, abort);
#pragma unroll
    for (int w = 0; w < 4; ++w) wait_or_abort(&bars[BAR_LOADQ + w], par, abort);
    if (warp == 0) {
      __syncwarp();
      tc_fence_after_sync();
#pragma unroll
      for (int k = 0; k < 4; ++k)
        umma_ss_w(tS, smem_desc_sw128(aA + 32 * k, 16, 1024), smem_desc_sw128(aA + 32 * k, 16, 2048), ID_S,
                  k > 0);
      umma_commit_w(&bars[BAR_S]);
      // X | Y = [K;Q] [W | S] as N = 128 products into adjacent accumulators: the
      // W and S operands are the two 64-column atoms of B, 16 KB apart (lbo).
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint64_t ak = smem_desc_sw128(aA + 32 * k, 16, 1024);
        umma_ss_w(tX, ak, smem_desc_sw128(aWhi + 2048 * k, OFF_SHI - OFF_WHI, 1024), ID_P2, k > 0);
        umma_ss_w(tX, ak, smem_desc_sw128(aWlo + 2048 * k, OFF_SLO - OFF_WLO, 1024), ID_P2, true);
      }
      umma_commit_w(&bars[BAR_P]);
      __syncwarp();
    }
    if (ntok < CHUNK) {  // ragged last chunk: absent tokens contribute nothing
      for (int x = tid; x < (CHUNK - ntok) * 32; x += THREADS) {
        const int row = ntok + x / 32, col = 2 * (x % 32);
        *reinterpret_cast<uint32_t *>(sm + OFF_G + sw128_offset(row, col)) = 0u;
      }
    }
    const int L = ntok - 1;  // the chunk's last token
    if (warp == 2) {
      // Lam_t = prod (1 - lambda), A_t = prod alpha and C_t = (1 - lambda_t) C_{t-1} + A_t;
      // absent tokens of a ragged chunk act as identities.
      float dl[2], da[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int t = lane + 32 * h;
        const bool in = t < ntok;
        dl[h] = in ? 1.f - lam_s[t] : 1.f;
        da[h] = in ? alpha_s[t] : 1.f;
      }
      // A product x_t = d_t x_{t-1} (x_{-1} = 1) is the scan's composed d.
      float pl[2] = {dl[0], dl[1]}, pa[2] = {da[0], da[1]};
      float e0[2] = {0.f, 0.f}, e1[2] = {0.f, 0.f};
      affine_scan64(pl, e0, lane);
      affine_scan64(pa, e1, lane);
      float dc[2] = {dl[0], dl[1]}, ec[2] = {pa[0], pa[1]};
      affine_scan64(dc, ec, lane);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        PL[lane + 32 * h] = pl[h];
        CC[lane + 32 * h] = ec[h];
      }
      if (lane == (L & 31)) {  // the lane that holds token L in half L / 32
        const int h = L >> 5;
        FIN[0] = pl[h];
        FIN[1] = ec[h];
        FIN[2] = pa[h];
      }
    } else if (warp == 3) {
      // The coefficient table, column sigma walked up from tau = sigma:
      // a_{tau,sigma} = alpha_tau a_{tau-1,sigma}, c_{tau,sigma} = (1 - lambda_tau)
      // c_{tau-1,sigma} + a_{tau,sigma}, both 1 at tau = sigma and 0 above the
      // diagonal.  Lane l walks columns l and 63 - l (65 steps each lane); the row
      // tau = L is c_{L,.} and a_{L,.} of the state update.  Both start at 0 and the
      // step a = alpha a + [tau = sigma] gives the 1 on the diagonal.  alpha and
      // lambda are read four tokens at a time, a group ahead (ntok is a multiple of
      // 16), so that no read waits behind the table's stores.
      const int s0 = lane, s1 = CHUNK - 1 - lane;
      float a0 = 0.f, c0 = 0.f, a1 = 0.f, c1 = 0.f;
      auto step = [&](int t, float al, float la) {
        const float om = 1.f - la;
        a0 = fmaf(al, a0, t == s0 ? 1.f : 0.f);
        c0 = fmaf(om, c0, a0);
        a1 = fmaf(al, a1, t == s1 ? 1.f : 0.f);
        c1 = fmaf(om, c1, a1);
        COEF[t * COEF_LD + s0] = c0;
        COEF[t * COEF_LD + s1] = c1;
      };
      float4 al4 = *reinterpret_cast<const float4 *>(alpha_s);
      float4 la4 = *reinterpret_cast<const float4 *>(lam_s);
      for (int t = 0; t < ntok; t += 4) {
        const float4 al = al4, la = la4;
        if (t + 4 < ntok) {
          al4 = *reinterpret_cast<const float4 *>(alpha_s + t + 4);
          la4 = *reinterpret_cast<const float4 *>(lam_s + t + 4);
        }
        step(t, al.x, la.x);
        step(t + 1, al.y, la.y);
        step(t + 2, al.z, la.z);
        step(t + 3, al.w, la.w);
      }
      CW[s0] = c0;
      AW[s0] = a0;
      CW[s1] = c1;
      AW[s1] = a1;
    }
    __syncthreads();  // coefficients, Lam, C visible
    {
      // This thread's row of [K;Q]: group 4 warp + lane / 8.  Its coefficient row
      // tau*: 16 m - 1 for a K row of mini-batch m (none for m = 0), its token for
      // a Q row (none for an absent token of a ragged chunk); column sigma gets
      // c_{tau*,sigma} S (0 above the diagonal).
      const bool qrow = (lane >> 3) & 1;
      const int mrow = mb0 + (lane >> 4);
      const int t = MB * mrow + 8 * hh + (lane & 7);
      const int tstar = t >= ntok ? -1 : (qrow ? t : MB * mrow - 1);
      const float *crow = COEF + (tstar < 0 ? 0 : tstar) * COEF_LD;
      wait_or_abort(&bars[BAR_S], par, abort);
      tc_fence_after_sync();
      __syncwarp();
      // Block j: tokens 16 j .. 16 j + 15 in S columns 8 j .. (the first eight) and
      // 32 + 8 j .. (the second), written back as fp16 pairs over the first.
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t pk[8];
        if (j <= mb0 + 1) {
          uint32_t v0[8], v1[8];
          tmem_ld_32x32b_x8(tmem_addr(tS, 32 * warp, 8 * j), v0);
          tmem_ld_32x32b_x8(tmem_addr(tS, 32 * warp, 32 + 8 * j), v1);
          float cf[16];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float4 c4 = *reinterpret_cast<const float4 *>(crow + MB * j + 4 * q);
            cf[4 * q] = c4.x;
            cf[4 * q + 1] = c4.y;
            cf[4 * q + 2] = c4.z;
            cf[4 * q + 3] = c4.w;
          }
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float x0 = tstar < 0 ? 0.f : cf[2 * e] * __uint_as_float(2 * e < 8 ? v0[2 * e] : v1[2 * e - 8]);
            const float x1 =
                tstar < 0 ? 0.f : cf[2 * e + 1] * __uint_as_float(2 * e + 1 < 8 ? v0[2 * e + 1] : v1[2 * e - 7]);
            pk[e] = pack_f16x2(x0, x1);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) pk[e] = 0u;
        }
        tmem_st_32x32b_x8(tmem_addr(tS, 32 * warp, 8 * j), pk);
      }
      // P = rho X + kappa Y over this thread's row: (Lam, C) at the row's base,
      // token 16 m - 1 for a K row of mini-batch m (Lam = 1, C = 0 for m = 0), the
      // row's own token for a Q row.
      const int tb_row = qrow ? t : MB * mrow - 1;
      const float rho = tb_row < 0 ? 1.f : PL[tb_row], kap = tb_row < 0 ? 0.f : CC[tb_row];
      wait_or_abort(&bars[BAR_P], par, abort);
      tc_fence_after_sync();
      __syncwarp();
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t xr[16], yr[16];
        tmem_ld_32x32b_x16(tmem_addr(tX, 32 * warp, 16 * q), xr);
        tmem_ld_32x32b_x16(tmem_addr(tY, 32 * warp, 16 * q), yr);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e)
          xr[e] = __float_as_uint(fmaf(kap, __uint_as_float(yr[e]), rho * __uint_as_float(xr[e])));
        tmem_st_32x32b_x16(tmem_addr(tX, 32 * warp, 16 * q), xr);
      }
      tmem_wait_st();
    }
    // Every MMA that reads this chunk's Q tile is complete (BAR_S, BAR_P): this
    // warp takes its residuals (with LN) and loads its part of the next chunk's Q.
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

    // ---- the chain: mini-batch m on warps m/2 and 2 + m/2 ------------------------
    // (u of the warp's second mini-batch first: it would otherwise sit between the
    // two updates.)
    float2 u1[8];
    float um1 = 0.f;
    if (mb0 + 1 < nmb) {
      load_kv(MB * (mb0 + 1) + 8 * hh + fr);
      make_u();
#pragma unroll
      for (int j = 0; j < 8; ++j) u1[j] = u[j];
      um1 = um;
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int m = mb0 + i;
      if (m >= nmb) break;
      const int tk = MB * m + 8 * hh + fr;
      const float e0 = eta_s[tk];
      const float cwk = CW[tk], awk = AW[tk];
      load_kv(tk);
      if (i == 0) {
        make_u();
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) u[j] = u1[j];
        um = um1;
      }
      wait_or_abort(&bars[m == 0 ? BAR_P : BAR_C0 + m - 1], par, abort);
      tc_fence_after_sync();
      __syncwarp();
      float2 y[8];
      read_p(i, 0, y);
      if (!LN) {
        // dl/dy = 2 (y - v)
        const float2 f = make_float2(2.f * e0, 2.f * e0);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float2 g = __fmul2_rn(f, fsub2(y[j], u[j]));
          *reinterpret_cast<uint32_t *>(sm + OFF_G + sw128_offset(tk, 8 * j + 2 * q4)) = pack_f16x2(g.x, g.y);
        }
      } else {
        // LN backward of ||k + gamma xhat + beta - v||^2 w.r.t. y (as in the
        // linear kernel: one reduction round for the mean, one for four sums).
        const float mean = quad_sum(sum8(y)) * (1.f / D);
        const float2 nm = make_float2(-mean, -mean);
        float2 w2[8];
        float2 sdd = make_float2(0.f, 0.f), swd = sdd, swdd = sdd, sud = sdd;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          w2[j] = *reinterpret_cast<const float2 *>(sm + OFF_W2 + 4 * (8 * j + 2 * q4));
          y[j] = __fadd2_rn(y[j], nm);
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
          const float2 g = __fmul2_rn(f, __fadd2_rn(__ffma2_rn(xh, __fadd2_rn(w2[j], nB), u[j]), nA));
          *reinterpret_cast<uint32_t *>(sm + OFF_G + sw128_offset(tk, 8 * j + 2 * q4)) = pack_f16x2(g.x, g.y);
        }
      }
      // The weighted K rows of the end-of-chunk update, fp16: c_{L,.} k in place
      // of K (X, Y and S, its bf16 readers, are complete), a_{L,.} k over the V
      // cells this thread has read (natural token order).
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float2 k2 = unpack_bf16x2(kr[j]);
        *reinterpret_cast<uint32_t *>(sm + kq_offset(tk, 0, 8 * j + 2 * q4)) = pack_f16x2(cwk * k2.x, cwk * k2.y);
        *reinterpret_cast<uint32_t *>(sm + OFF_V + sw128_offset(tk, 8 * j + 2 * q4)) =
            pack_f16x2(awk * k2.x, awk * k2.y);
      }
      fence_proxy_async_smem();
      tc_fence_before_sync();
      named_barrier_sync(1 + (warp & 1), 64);
      if (hh == 0) {
        __syncwarp();
        tc_fence_after_sync();
        umma_ts_w(tX, tS + 8 * m, smem_desc_sw128(aG + 2048 * m, 8192, 1024), ID_CORR, true);
        umma_commit_w(&bars[m == nmb - 1 ? BAR_LAST : BAR_C0 + m]);
        if (m == nmb - 1) {
          // Every eta G row and weighted K row of the chunk is written (each step's
          // writers fenced them before the barrier that its issue followed): the
          // state update's MMAs go now, under the last outputs.  dW = (c-weighted
          // K)^T (eta G): the K rows of groups 4k, 4k + 2 read twice (lbo 0) against
          // the eta G rows of the same tokens (two 8-row groups 2 KB apart); dS =
          // (a-weighted K, natural order in the V buffer)^T (eta G).
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint32_t gk = 4096u * (k & 1) + 1024u * (k >> 1);
            umma_ss_w(tC, smem_desc_sw128(aA + 4096 * k, 0, 2048), smem_desc_sw128(aG + gk, 8192, 2048), ID_DW,
                      k > 0);
          }
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_ss_w(tY, smem_desc_sw128(aV + 2048 * k, 0, 1024), smem_desc_sw128(aG + 2048 * k, 8192, 1024),
                      ID_DW, k > 0);
          umma_commit_w(&bars[BAR_DW]);
        }
        __syncwarp();
      }
    }

    // ---- outputs of this warp's Q rows (final once their mini-batch's update is in)
    float *Zc = p.Z + (tok_base + (size_t)c * CHUNK) * D;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int m = mb0 + i;
      if (m >= nmb) break;
      const int tq = MB * m + 8 * hh + fr;
      wait_or_abort(&bars[m == nmb - 1 ? BAR_LAST : BAR_C0 + m], par, abort);
      tc_fence_after_sync();
      __syncwarp();
      float2 z[8];
      read_p(i, 1, z);
      float *zrow = Zc + tq * D;
      if (!LN) {
#pragma unroll
        for (int j = 0; j < 8; ++j) *reinterpret_cast<float2 *>(zrow + 8 * j + 2 * q4) = z[j];
      } else {
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
          const float2 q = unpack_bf16x2(qres[i][j]);
          *reinterpret_cast<float2 *>(zrow + col) =
              __fadd2_rn(q, __ffma2_rn(make_float2(gb.x, gb.y), __fmul2_rn(z[j], rs), make_float2(gb.z, gb.w)));
        }
      }
    }

    // ---- the end-of-chunk state --------------------------------------------------
    wait_or_abort(&bars[BAR_DW], par, abort);
    tc_fence_after_sync();
    __syncwarp();
    if (tid == 0 && c + 1 < nchunks && !*abort) issue_loads_kv(c + 1);
    {
      const float lamL = FIN[0], cL = FIN[1], aL = FIN[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t dw[16], ds[16];
        tmem_ld_32x32b_x16(tmem_addr(tC, 32 * warp, wc0 + 16 * h), dw);
        tmem_ld_32x32b_x16(tmem_addr(tY, 32 * warp, wc0 + 16 * h), ds);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float w = wm[16 * h + e], s = sv[16 * h + e];
          wm[16 * h + e] = fmaf(lamL, w, fmaf(cL, s, -__uint_as_float(dw[e])));
          sv[16 * h + e] = fmaf(aL, s, -__uint_as_float(ds[e]));
        }
      }
      write_operands();
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (*abort) break;
    if (c + 1 < nchunks) chunk_head(c + 1);
  }

  __syncthreads();
  if (*abort) {
    if (tid == 0 && kv_last >= 0) mbar_wait(&bars[BAR_LOAD], (uint32_t)kv_last & 1u, WAIT_LIMIT);
    if (lane == 0 && q_last >= 0) mbar_wait(&bars[BAR_LOADQ + warp], (uint32_t)q_last & 1u, WAIT_LIMIT);
    if (warp < 2) umma_commit(&bars[BAR_DRAIN]);
    mbar_wait(&bars[BAR_DRAIN], 0, WAIT_LIMIT);
    tc_fence_after_sync();
  }

  {
    float4 *dw = reinterpret_cast<float4 *>(p.W_out + (size_t)unit * D * D + wi * D + wc0);
    float4 *ds = reinterpret_cast<float4 *>(p.S_out + (size_t)unit * D * D + wi * D + wc0);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      dw[q] = make_float4(wm[4 * q], wm[4 * q + 1], wm[4 * q + 2], wm[4 * q + 3]);
      ds[q] = make_float4(sv[4 * q], sv[4 * q + 1], sv[4 * q + 2], sv[4 * q + 3]);
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tb, TMEM_COLS);
  }
}

}  // namespace tcmom
}  // namespace ttt
