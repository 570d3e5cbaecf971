// momentum.cuh - forward over whole sequences of TTT-Linear and TTT-Linear + LN
// with the momentum and decay update (the Titans article's memory update,
// §二.1(2), kept to the TTT mini-batch rule, §03.6):
//   S_t = alpha_t S_{t-1} - eta_t k_t^T G_t,   W_t = (1 - lambda_t) W_{t-1} + S_t,
//   z_t = q_t W_t  (or q_t + LN(q_t W_t)),     G_t = dl/dy at y = k_t W_base,
// S_0 = 0, W_base the state at the start of token t's mini-batch.
//
// One CTA of 256 threads per (batch, head) unit.  Thread (rq, j) keeps rows
// 16 rq .. 16 rq + 15 of column j of W, W_base and S in registers for the whole
// sequence, so the state never leaves the SM.  Per mini-batch of b <= 16 tokens:
//   1. the tiles q, k, v [b][64] and eta, alpha, lambda [b] are staged in shared memory;
//   2. every y_t = k_t W_base as partial column sums over the row quarters, and
//      G_t from them (a warp per token, plain or through LN + residual) - all
//      gradients of a mini-batch are taken at its base, so this is parallel;
//   3. the token loop: each thread updates its own S and W elements and writes
//      its partial sum of q_t W_t; no barrier inside the loop (the tiles are
//      read-only there and every thread owns its state);
//   4. z_t from the partial sums (a warp per token, with the output LN).
// The per-element arithmetic is that of the momentum decode step, so a sequence
// of decode calls and this kernel agree to rounding.  HBM traffic is the inputs
// and outputs once (about 650 B per token with bf16 q, k, v); the time is the
// per-mini-batch chain of barriers.
//
// With MOMENTUM = false the same kernel runs the plain TTT rule
// (W_t = W_{t-1} - eta_t k_t^T G_t, no S, alpha, lambda): the exact-fp32
// CUDA-core forward of TTT-Linear (+ LN) for b <= 16.  Per token it computes
// z_t = q_t W_t from the state itself rather than through the dual form's
// masked Gram (the two are equal; see the mini-batch rule above).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "simt.cuh"

namespace ttt {
namespace mom {

constexpr int D = simt::D;
constexpr int MAXB = 16;
constexpr int THREADS = 256;

struct Params {
  const void *Q, *K, *V;                    // [units][T][D]
  const float *eta, *alpha, *lambda;        // [units][T] (alpha, lambda: MOMENTUM only)
  const float *W0;                          // [H][D][D]
  const float *gamma, *beta;                // [H][D] (LN)
  float eps;
  int H, T, b;
  float *Z;                                 // [units][T][D]
  float *W_out, *S_out;                     // [units][D][D] (S_out: MOMENTUM only)
};

struct Smem {
  float q[MAXB][D], k[MAXB][D], v[MAXB][D];
  float eta[MAXB], alpha[MAXB], lambda[MAXB];
  float g[MAXB][D];          // eta_t G_t
  float part[MAXB][4][D];    // per-quarter partial column sums: k_t W_base, then q_t W_t
};

// MINB: CTAs per SM the registers are capped for (4: 64 registers and a few
// spills, so that 4 x 148 units run in one wave; 1: no cap, 2-3 CTAs per SM).
template <bool LN, typename InT, bool MOMENTUM = true, int MINB = 1>
__global__ void __launch_bounds__(THREADS, MINB) momentum_fwd_kernel(const Params p) {
  __shared__ Smem s;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int j = tid & (D - 1), rq = tid >> 6;
  const long unit = blockIdx.x;
  const int head = (int)(unit % p.H);
  const int b = p.b, N = p.T / b;
  const long tok0 = unit * (long)p.T;
  const InT *Qg = static_cast<const InT *>(p.Q);
  const InT *Kg = static_cast<const InT *>(p.K);
  const InT *Vg = static_cast<const InT *>(p.V);

  float gam0 = 0.f, gam1 = 0.f, bet0 = 0.f, bet1 = 0.f;
  if (LN) {
    gam0 = p.gamma[head * D + lane];
    gam1 = p.gamma[head * D + lane + 32];
    bet0 = p.beta[head * D + lane];
    bet1 = p.beta[head * D + lane + 32];
  }
  float wb[16], w[16], sm[MOMENTUM ? 16 : 1];
#pragma unroll
  for (int r = 0; r < 16; ++r) {
    wb[r] = p.W0[(long)head * D * D + (16 * rq + r) * D + j];
    w[r] = wb[r];
    if (MOMENTUM) sm[r] = 0.f;
  }

  for (int n = 0; n < N; ++n) {
    const long row0 = tok0 + (long)n * b;
    for (int x = tid; x < b * D; x += THREADS) {
      const int t = x / D, c = x % D;
      s.q[t][c] = simt::load_in(Qg, (row0 + t) * D + c);
      s.k[t][c] = simt::load_in(Kg, (row0 + t) * D + c);
      s.v[t][c] = simt::load_in(Vg, (row0 + t) * D + c);
    }
    if (tid < b) {
      s.eta[tid] = p.eta[row0 + tid];
      if (MOMENTUM) {
        s.alpha[tid] = p.alpha[row0 + tid];
        s.lambda[tid] = p.lambda[row0 + tid];
      }
    }
    __syncthreads();

    // y_t = k_t W_base: this thread's partial sum over its 16 rows.
#pragma unroll 1
    for (int t = 0; t < b; ++t) {
      float acc = 0.f;
#pragma unroll
      for (int r = 0; r < 16; ++r) acc = fmaf(s.k[t][16 * rq + r], wb[r], acc);
      s.part[t][rq][j] = acc;
    }
    __syncthreads();

    // G_t (a warp per token), scaled by eta_t.
    for (int t = warp; t < b; t += 8) {
      const float y0 = (s.part[t][0][lane] + s.part[t][1][lane]) + (s.part[t][2][lane] + s.part[t][3][lane]);
      const float y1 = (s.part[t][0][lane + 32] + s.part[t][1][lane + 32]) +
                       (s.part[t][2][lane + 32] + s.part[t][3][lane + 32]);
      float g0, g1;
      if (LN) {
        simt::ln_residual_grad(y0, y1, s.k[t][lane], s.k[t][lane + 32], s.v[t][lane], s.v[t][lane + 32],
                               gam0, gam1, bet0, bet1, p.eps, g0, g1);
      } else {
        g0 = 2.f * (y0 - s.v[t][lane]);
        g1 = 2.f * (y1 - s.v[t][lane + 32]);
      }
      const float e = s.eta[t];
      s.g[t][lane] = e * g0;
      s.g[t][lane + 32] = e * g1;
    }
    __syncthreads();

    // The token loop: S, W of this thread's elements, and its partial of q_t W_t.
#pragma unroll 1
    for (int t = 0; t < b; ++t) {
      const float gj = s.g[t][j];
      const float al = MOMENTUM ? s.alpha[t] : 0.f;
      const float keep = MOMENTUM ? 1.f - s.lambda[t] : 1.f;
      float zacc = 0.f;
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        const int i = 16 * rq + r;
        if (MOMENTUM) {
          sm[r] = fmaf(al, sm[r], -s.k[t][i] * gj);
          w[r] = fmaf(keep, w[r], sm[r]);
        } else {
          w[r] = fmaf(-s.k[t][i], gj, w[r]);
        }
        zacc = fmaf(s.q[t][i], w[r], zacc);
      }
      s.part[t][rq][j] = zacc;
    }
    // The next mini-batch takes its gradients at the state this one ends in.
#pragma unroll
    for (int r = 0; r < 16; ++r) wb[r] = w[r];
    __syncthreads();

    // z_t (a warp per token), with the output LN and residual.
    for (int t = warp; t < b; t += 8) {
      const float z0 = (s.part[t][0][lane] + s.part[t][1][lane]) + (s.part[t][2][lane] + s.part[t][3][lane]);
      const float z1 = (s.part[t][0][lane + 32] + s.part[t][1][lane + 32]) +
                       (s.part[t][2][lane + 32] + s.part[t][3][lane + 32]);
      float o0 = z0, o1 = z1;
      if (LN)
        simt::ln_residual_fwd(z0, z1, s.q[t][lane], s.q[t][lane + 32], gam0, gam1, bet0, bet1, p.eps, o0,
                              o1);
      p.Z[(row0 + t) * D + lane] = o0;
      p.Z[(row0 + t) * D + lane + 32] = o1;
    }
    __syncthreads();
  }

#pragma unroll
  for (int r = 0; r < 16; ++r) {
    p.W_out[unit * D * D + (16 * rq + r) * D + j] = w[r];
    if (MOMENTUM) p.S_out[unit * D * D + (16 * rq + r) * D + j] = sm[r];
  }
}

}  // namespace mom
}  // namespace ttt
