// decode.cuh - primal-form decode step of TTT-Linear, TTT-Linear + LN and
// TTT-MLP: one token per (batch, head) and call, the state carried in HBM.  Decoding is
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
//
// The momentum and decay variant of the linear kernels (the Titans article's
// memory update, §二.1(2), kept to the mini-batch base above) carries a third
// state S, zero at the start:
//   S <- alpha S - eta k^T G,   W <- (1 - lambda) W + S
// and otherwise runs the same call: 80 KB per (batch, head) and call.
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
  // Momentum and decay variant (Titans-style memory update) when S != nullptr:
  //   S <- alpha S - eta k^T G,  W <- (1 - lambda) W + S   (S [units][D][D], in place)
  const float *alpha, *lambda;  // [units]
  float *S;
};

template <bool LN, typename InT, bool MOMENTUM = false>
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
  float wb[16], w[16], sm_[MOMENTUM ? 16 : 1];
  float *Su = MOMENTUM ? p.S + unit * D * D : nullptr;
#pragma unroll
  for (int r = 0; r < 16; ++r) {
    wb[r] = Wb[(16 * rq + r) * D + j];
    w[r] = Wu[(16 * rq + r) * D + j];
    if (MOMENTUM) sm_[r] = Su[(16 * rq + r) * D + j];
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

  // W -= k^T (eta G) (or the momentum and decay update); z = q W with the
  // updated state.
  const float gj = g[j];
  const bool last = p.pos == p.b - 1;
  const float al = MOMENTUM ? p.alpha[unit] : 0.f;
  const float keep = MOMENTUM ? 1.f - p.lambda[unit] : 1.f;
  float zacc = 0.f;
#pragma unroll
  for (int r = 0; r < 16; ++r) {
    const int i = 16 * rq + r;
    if (MOMENTUM) {
      sm_[r] = fmaf(al, sm_[r], -ks[i] * gj);
      w[r] = fmaf(keep, w[r], sm_[r]);
      Su[i * D + j] = sm_[r];
    } else {
      w[r] = fmaf(-ks[i], gj, w[r]);
    }
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

// TTT-MLP, f(x) = x + LN(GELU(x W1) W2) (§03.9): the same step with two state
// matrices, W1 [D][HID] and W2 [HID][D], each with its mini-batch base.  With
// X1 = k W1b, X2 = GELU(X1), X3 = X2 W2b and G3 = dl/dX3 (LN backward), the
// gradient w.r.t. X1 is G2 = (G3 W2b^T) * GELU'(X1), and
//   W1 <- W1 - eta k^T G2,  W2 <- W2 - eta X2^T G3,
//   z   = q + LN(GELU(q W1) W2)   with the updated W1, W2.
// Per (batch, head) a call reads the four matrices (256 KB) and writes W1, W2
// (128 KB, and the bases once per mini-batch).  Thread i of the CTA owns hidden
// unit i: column i of W1 (and W1b) and row i of W2 (and W2b).
//
// The momentum and decay variant (the Titans article's MLP memory, §二.1) adds
// the momenta S1, S2 (the shapes of W1, W2, zero at the start):
//   S1 <- alpha S1 - eta k^T G2,   W1 <- (1 - lambda) W1 + S1   (and so for W2)
// 640 KB of state traffic per (batch, head) and call.
struct MlpParams {
  const void *q, *k, *v;
  const float *eta;
  float *W1, *W2, *W1_base, *W2_base;  // [units][D][HID], [units][HID][D]
  const float *gamma, *beta;
  float eps;
  int H, pos, b;
  float *z;
  const float *alpha, *lambda;  // [units], momentum variant only
  float *S1, *S2;               // like W1, W2, momentum variant only
};
constexpr int HID = simt::HID;
constexpr int MLP_THREADS = HID;

template <typename InT, bool MOMENTUM = false>
__global__ void __launch_bounds__(MLP_THREADS) mlp_decode_kernel(const MlpParams p) {
  __shared__ float qs[D], ks[D], vs[D], x2s[HID], z2s[HID], g3[D], part[8][D];
  const int i = threadIdx.x, lane = i & 31, warp = i >> 5;
  const long unit = blockIdx.x;
  const int head = (int)(unit % p.H);
  if (i < D) {
    qs[i] = simt::load_in(static_cast<const InT *>(p.q), unit * D + i);
    ks[i] = simt::load_in(static_cast<const InT *>(p.k), unit * D + i);
    vs[i] = simt::load_in(static_cast<const InT *>(p.v), unit * D + i);
  }
  float *W1 = p.W1 + unit * D * HID, *W1b = p.W1_base + unit * D * HID;
  float *W2 = p.W2 + unit * HID * D, *W2b = p.W2_base + unit * HID * D;
  __syncthreads();

  // X1 = k W1b (column i), X2 = GELU(X1).
  float x1 = 0.f;
#pragma unroll 8
  for (int pp = 0; pp < D; ++pp) x1 = fmaf(ks[pp], W1b[pp * HID + i], x1);
  const float x2 = simt::gelu(x1);
  x2s[i] = x2;
  __syncthreads();
  // X3 = X2 W2b: warp w sums hidden rows 32w .. 32w + 31 for columns lane, lane + 32.
  {
    float a0 = 0.f, a1 = 0.f;
#pragma unroll 8
    for (int r = 0; r < 32; ++r) {
      const int ii = 32 * warp + r;
      a0 = fmaf(x2s[ii], W2b[ii * D + lane], a0);
      a1 = fmaf(x2s[ii], W2b[ii * D + lane + 32], a1);
    }
    part[warp][lane] = a0;
    part[warp][lane + 32] = a1;
  }
  __syncthreads();
  if (warp == 0) {
    float y0 = 0.f, y1 = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      y0 += part[w][lane];
      y1 += part[w][lane + 32];
    }
    float d0, d1;
    simt::ln_residual_grad(y0, y1, ks[lane], ks[lane + 32], vs[lane], vs[lane + 32],
                           p.gamma[head * D + lane], p.gamma[head * D + lane + 32], p.beta[head * D + lane],
                           p.beta[head * D + lane + 32], p.eps, d0, d1);
    g3[lane] = d0;
    g3[lane + 32] = d1;
  }
  __syncthreads();
  // G2 = (G3 W2b^T) * GELU'(X1) for hidden unit i (row i of W2b).
  float g2 = 0.f;
  {
    const float4 *row = reinterpret_cast<const float4 *>(W2b + i * D);
#pragma unroll
    for (int c = 0; c < D / 4; ++c) {
      const float4 w = row[c];
      g2 = fmaf(g3[4 * c], w.x, g2);
      g2 = fmaf(g3[4 * c + 1], w.y, g2);
      g2 = fmaf(g3[4 * c + 2], w.z, g2);
      g2 = fmaf(g3[4 * c + 3], w.w, g2);
    }
  }
  const float e = p.eta[unit];
  g2 *= simt::gelu_deriv(x1) * e;
  const bool last = p.pos == p.b - 1;
  const float al = MOMENTUM ? p.alpha[unit] : 0.f;
  const float keep = MOMENTUM ? 1.f - p.lambda[unit] : 1.f;
  float *S1 = MOMENTUM ? p.S1 + unit * D * HID : nullptr;
  float *S2 = MOMENTUM ? p.S2 + unit * HID * D : nullptr;
  // W1 -= eta k^T G2 (column i; or the momentum and decay update) and Z1 = q W1
  // with the updated W1.
  // Rows in blocks of RB: every load of a block is issued before its stores, which
  // the compiler could not otherwise move past (W1, W1b and S1 are distinct
  // buffers, but nothing tells it so), keeping 2 RB loads per thread in flight.
  constexpr int RB = 16;
  float z1 = 0.f;
  for (int p0 = 0; p0 < D; p0 += RB) {
    float wv[RB], sv[MOMENTUM ? RB : 1];
#pragma unroll
    for (int u = 0; u < RB; ++u) {
      wv[u] = W1[(p0 + u) * HID + i];
      if (MOMENTUM) sv[u] = S1[(p0 + u) * HID + i];
    }
#pragma unroll
    for (int u = 0; u < RB; ++u) {
      const int pp = p0 + u;
      float w;
      if (MOMENTUM) {
        const float sm = fmaf(al, sv[u], -ks[pp] * g2);
        S1[pp * HID + i] = sm;
        w = fmaf(keep, wv[u], sm);
      } else {
        w = fmaf(-ks[pp], g2, wv[u]);
      }
      W1[pp * HID + i] = w;
      if (last) W1b[pp * HID + i] = w;
      z1 = fmaf(qs[pp], w, z1);
    }
  }
  z2s[i] = simt::gelu(z1);
  __syncthreads();
  // W2 -= eta X2^T G3 (rows 32w .. 32w + 31) and Z3 = Z2 W2 with the updated W2.
  {
    const float eg0 = e * g3[lane], eg1 = e * g3[lane + 32];
    float a0 = 0.f, a1 = 0.f;
    constexpr int R2 = 8;  // rows per block, loads first (as for W1 above)
    for (int r0 = 0; r0 < 32; r0 += R2) {
      float wv0[R2], wv1[R2], sv0[MOMENTUM ? R2 : 1], sv1[MOMENTUM ? R2 : 1];
#pragma unroll
      for (int u = 0; u < R2; ++u) {
        const int ii = 32 * warp + r0 + u;
        wv0[u] = W2[ii * D + lane];
        wv1[u] = W2[ii * D + lane + 32];
        if (MOMENTUM) {
          sv0[u] = S2[ii * D + lane];
          sv1[u] = S2[ii * D + lane + 32];
        }
      }
#pragma unroll
      for (int u = 0; u < R2; ++u) {
        const int ii = 32 * warp + r0 + u;
        float w0, w1;
        if (MOMENTUM) {
          const float s0 = fmaf(al, sv0[u], -x2s[ii] * eg0);
          const float s1 = fmaf(al, sv1[u], -x2s[ii] * eg1);
          S2[ii * D + lane] = s0;
          S2[ii * D + lane + 32] = s1;
          w0 = fmaf(keep, wv0[u], s0);
          w1 = fmaf(keep, wv1[u], s1);
        } else {
          w0 = fmaf(-x2s[ii], eg0, wv0[u]);
          w1 = fmaf(-x2s[ii], eg1, wv1[u]);
        }
        W2[ii * D + lane] = w0;
        W2[ii * D + lane + 32] = w1;
        if (last) {
          W2b[ii * D + lane] = w0;
          W2b[ii * D + lane + 32] = w1;
        }
        a0 = fmaf(z2s[ii], w0, a0);
        a1 = fmaf(z2s[ii], w1, a1);
      }
    }
    __syncthreads();  // every warp has read part[] of the X3 pass long before; reuse it
    part[warp][lane] = a0;
    part[warp][lane + 32] = a1;
  }
  __syncthreads();
  if (warp == 0) {
    float y0 = 0.f, y1 = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      y0 += part[w][lane];
      y1 += part[w][lane + 32];
    }
    float o0, o1;
    simt::ln_residual_fwd(y0, y1, qs[lane], qs[lane + 32], p.gamma[head * D + lane],
                          p.gamma[head * D + lane + 32], p.beta[head * D + lane],
                          p.beta[head * D + lane + 32], p.eps, o0, o1);
    p.z[unit * D + lane] = o0;
    p.z[unit * D + lane + 32] = o1;
  }
}

}  // namespace decode
}  // namespace ttt
