// decode.cuh - primal-form decode step of TTT-Linear and TTT-Linear + LN: one
// token per (batch, head) and call, the state carried in HBM.  Decoding is
// sequential, so it takes the primal form rather than the dual one (TTT
// write-up §04.3, generation).
//
// Mini-batch semantics (§03.6): every gradient of a mini-batch is taken at the
// state W_base the mini-batch started from, so token t at position pos of its
// mini-batch sees W_t = W_base - sum_{s <= t} eta_s k_s^T G_s.  One call:
//   G       = dl/d(k W_base)   2 (k W_base - v), or through LN + residual (§03.9)
//   W      <- W - eta k^T G
//   z       = q W              (or q + LN(q W))
//   W_base <- W                only when pos == b - 1 (the next mini-batch
//                              starts from the state this one ends in)
// Per (batch, head) a call reads W_base and W (32 KB) and writes W (16 KB, and
// W_base once per mini-batch): HBM-bound, 48 KB against ~16 kFLOP.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "simt.cuh"

namespace ttt {
namespace decode {

using simt::D;
constexpr int THREADS = 256;  // thread (row quarter rq, column j) owns W[16 rq .. 16 rq + 15][j]

struct Params {
  const void *q, *k, *v;  // [units][D]
  const float *eta;       // [units]
  float *W, *W_base;      // [units][D][D], in place
  const float *gamma, *beta;
  float eps;
  int H, pos, b;
  float *z;               // [units][D]
};

template <bool LN, typename InT>
__global__ void __launch_bounds__(THREADS) decode_kernel(const Params p) {
  __shared__ float qs[D], ks[D], vs[D], part[4][D], g[D];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long unit = blockIdx.x;
  const int head = (int)(unit % p.H);
  const int j = tid & (D - 1), rq = tid >> 6;
  if (tid < D) {
    qs[tid] = simt::load_in(static_cast<const InT *>(p.q), unit * D + tid);
    ks[tid] = simt::load_in(static_cast<const InT *>(p.k), unit * D + tid);
    vs[tid] = simt::load_in(static_cast<const InT *>(p.v), unit * D + tid);
  }
  float *Wu = p.W + unit * D * D;
  float *Wb = p.W_base + unit * D * D;
  // Both state rows of this thread are read up front (one coalesced 128-byte
  // line per warp and row).
  float wb[16], w[16];
#pragma unroll
  for (int r = 0; r < 16; ++r) {
    wb[r] = Wb[(16 * rq + r) * D + j];
    w[r] = Wu[(16 * rq + r) * D + j];
  }
  __syncthreads();

  // y = k W_base: partial sum over this thread's 16 rows, then over the quarters.
  float acc = 0.f;
#pragma unroll
  for (int r = 0; r < 16; ++r) acc = fmaf(ks[16 * rq + r], wb[r], acc);
  part[rq][j] = acc;
  __syncthreads();
  if (warp == 0) {
    const float y0 = (part[0][lane] + part[1][lane]) + (part[2][lane] + part[3][lane]);
    const float y1 = (part[0][lane + 32] + part[1][lane + 32]) + (part[2][lane + 32] + part[3][lane + 32]);
    float g0, g1;
    if (LN) {
      simt::ln_residual_grad(y0, y1, ks[lane], ks[lane + 32], vs[lane], vs[lane + 32],
                             p.gamma[head * D + lane], p.gamma[head * D + lane + 32],
                             p.beta[head * D + lane], p.beta[head * D + lane + 32], p.eps, g0, g1);
    } else {
      g0 = 2.f * (y0 - vs[lane]);
      g1 = 2.f * (y1 - vs[lane + 32]);
    }
    const float e = p.eta[unit];
    g[lane] = e * g0;
    g[lane + 32] = e * g1;
  }
  __syncthreads();

  // W -= k^T (eta G); z = q W with the updated state.
  const float gj = g[j];
  const bool last = p.pos == p.b - 1;
  float zacc = 0.f;
#pragma unroll
  for (int r = 0; r < 16; ++r) {
    const int i = 16 * rq + r;
    w[r] = fmaf(-ks[i], gj, w[r]);
    zacc = fmaf(qs[i], w[r], zacc);
    Wu[i * D + j] = w[r];
    if (last) Wb[i * D + j] = w[r];
  }
  part[rq][j] = zacc;
  __syncthreads();
  if (warp == 0) {
    const float z0 = (part[0][lane] + part[1][lane]) + (part[2][lane] + part[3][lane]);
    const float z1 = (part[0][lane + 32] + part[1][lane + 32]) + (part[2][lane + 32] + part[3][lane + 32]);
    float o0 = z0, o1 = z1;
    if (LN)
      simt::ln_residual_fwd(z0, z1, qs[lane], qs[lane + 32], p.gamma[head * D + lane],
                            p.gamma[head * D + lane + 32], p.beta[head * D + lane],
                            p.beta[head * D + lane + 32], p.eps, o0, o1);
    p.z[unit * D + lane] = o0;
    p.z[unit * D + lane + 32] = o1;
  }
}

}  // namespace decode
}  // namespace ttt
