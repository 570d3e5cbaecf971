// simt.cuh - exact-fp32 CUDA-core kernels of the TTT layer forward (dual form).
//
// One CTA of 256 threads owns one (batch, head) sequence for its whole length
// and keeps the fp32 state in shared memory; mini-batches are processed in
// order, each as the dual form of the TTT write-up §03.7 (whole mini-batch as
// masked matrix products, per-token gradients never materialised).  Every
// product is an fp32 FMA chain, so these kernels serve the fp32 inputs (where
// the tolerance is 1e-5) and any size the tensor-core kernels do not cover.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace ttt {
namespace simt {

constexpr int D = 64;         // head dimension
constexpr int HID = 4 * D;    // TTT-MLP hidden width
constexpr int THREADS = 256;
constexpr int W2_LD = D + 1;  // padded row stride of W2 in shared memory

__device__ __forceinline__ float load_in(const float *p, long i) { return p[i]; }
__device__ __forceinline__ float load_in(const __nv_bfloat16 *p, long i) {
  return __bfloat162float(p[i]);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Exact GELU x * Phi(x) and its derivative Phi(x) + x phi(x), through CUDA's
// normcdff / expf.
__device__ __forceinline__ float gelu(float x) { return x * normcdff(x); }
__device__ __forceinline__ float gelu_deriv(float x) {
  return normcdff(x) + x * (0.3989422804014327f * expf(-0.5f * x * x));
}

struct Params {
  const void *Q, *K, *V;
  const float *eta;
  const float *W0;  // linear: [H][D][D]; MLP: W1_0 [H][D][HID]
  const float *W2_0;
  const float *gamma, *beta;
  float eps;
  int H, T, b;
  float *Z;
  float *W_out;  // linear: [B][H][D][D]; MLP: W1_out
  float *W2_out;
};

// LN backward for one row held by one warp (lane owns columns lane, lane+32):
// y = pre-activation, the loss is ||x + gamma*xhat + beta - v||^2.  Returns dl/dy.
__device__ __forceinline__ void ln_residual_grad(float y0, float y1, float x0, float x1, float v0,
                                                 float v1, float g0, float g1, float b0, float b1,
                                                 float eps, float &dy0, float &dy1) {
  const float mean = warp_sum(y0 + y1) * (1.0f / D);
  const float c0 = y0 - mean, c1 = y1 - mean;
  const float var = warp_sum(c0 * c0 + c1 * c1) * (1.0f / D);
  const float rstd = rsqrtf(var + eps);
  const float xh0 = c0 * rstd, xh1 = c1 * rstd;
  const float r0 = x0 + g0 * xh0 + b0 - v0, r1 = x1 + g1 * xh1 + b1 - v1;
  const float gx0 = 2.0f * r0 * g0, gx1 = 2.0f * r1 * g1;  // dl/dxhat
  const float mg = warp_sum(gx0 + gx1) * (1.0f / D);
  const float mgx = warp_sum(gx0 * xh0 + gx1 * xh1) * (1.0f / D);
  dy0 = rstd * (gx0 - mg - xh0 * mgx);
  dy1 = rstd * (gx1 - mg - xh1 * mgx);
}

// x + gamma * LN-normalise(y) + beta for one warp-held row.
__device__ __forceinline__ void ln_residual_fwd(float y0, float y1, float x0, float x1, float g0,
                                                float g1, float b0, float b1, float eps, float &z0,
                                                float &z1) {
  const float mean = warp_sum(y0 + y1) * (1.0f / D);
  const float c0 = y0 - mean, c1 = y1 - mean;
  const float var = warp_sum(c0 * c0 + c1 * c1) * (1.0f / D);
  const float rstd = rsqrtf(var + eps);
  z0 = x0 + g0 * (c0 * rstd) + b0;
  z1 = x1 + g1 * (c1 * rstd) + b1;
}

inline size_t linear_smem_bytes(int b) {
  return sizeof(float) * ((size_t)D * D + 5 * (size_t)b * D + (size_t)b * b + b);
}

template <bool LN, typename InT>
__global__ void __launch_bounds__(THREADS) linear_kernel(const Params p) {
  extern __shared__ __align__(16) float sm[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long unit = blockIdx.x;
  const int head = (int)(unit % p.H);
  const int b = p.b;
  float *W = sm;           // [D][D]
  float *Qs = W + D * D;   // [b][D]
  float *Ks = Qs + b * D;  // [b][D]
  float *Vs = Ks + b * D;  // [b][D]
  float *G = Vs + b * D;   // [b][D]: K W, then the gradient
  float *P = G + b * D;    // [b][D]: Q W, then the pre-LN output
  float *A = P + b * D;    // [b][b]: tril(Q K^T) diag(eta)
  float *es = A + b * b;   // [b]

  const float *W0 = p.W0 + (long)head * D * D;
  for (int x = tid; x < D * D; x += THREADS) W[x] = W0[x];
  float gam0 = 0.f, gam1 = 0.f, bet0 = 0.f, bet1 = 0.f;
  if (LN) {
    gam0 = p.gamma[head * D + lane];
    gam1 = p.gamma[head * D + lane + 32];
    bet0 = p.beta[head * D + lane];
    bet1 = p.beta[head * D + lane + 32];
  }
  const long tok0 = unit * (long)p.T;
  const InT *Qg = (const InT *)p.Q + tok0 * D;
  const InT *Kg = (const InT *)p.K + tok0 * D;
  const InT *Vg = (const InT *)p.V + tok0 * D;
  float *Zg = p.Z + tok0 * D;
  const int nmb = p.T / b;
  const int j = tid & (D - 1), rg = tid >> 6;  // column and row group of this thread

  for (int n = 0; n < nmb; ++n) {
    __syncthreads();  // previous mini-batch done with the tiles and W
    const long off = (long)n * b * D;
    for (int x = tid; x < b * D; x += THREADS) {
      Qs[x] = load_in(Qg, off + x);
      Ks[x] = load_in(Kg, off + x);
      Vs[x] = load_in(Vg, off + x);
    }
    if (tid < b) es[tid] = p.eta[tok0 + (long)n * b + tid];
    __syncthreads();

    // K W and Q W at the mini-batch base.
    for (int r0 = 0; r0 < b; r0 += 16) {
      float ak[4] = {0.f, 0.f, 0.f, 0.f}, aq[4] = {0.f, 0.f, 0.f, 0.f};
      for (int i = 0; i < D; ++i) {
        const float w = W[i * D + j];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int r = r0 + rg + 4 * k;
          if (r < b) {
            ak[k] = fmaf(Ks[r * D + i], w, ak[k]);
            aq[k] = fmaf(Qs[r * D + i], w, aq[k]);
          }
        }
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int r = r0 + rg + 4 * k;
        if (r < b) {
          G[r * D + j] = ak[k];
          P[r * D + j] = aq[k];
        }
      }
    }
    // Causal eta-masked Gram: A[t][s] = (q_t . k_s) eta_s for s <= t, else 0.
    for (int pr = warp; pr < b * b; pr += THREADS / 32) {
      const int t = pr / b, s = pr % b;
      float acc = 0.f;
      if (s <= t) {
        acc = Qs[t * D + lane] * Ks[s * D + lane];
        acc = fmaf(Qs[t * D + lane + 32], Ks[s * D + lane + 32], acc);
        acc = warp_sum(acc) * es[s];
      }
      if (lane == 0) A[pr] = acc;
    }
    __syncthreads();

    // Gradient of the loss with respect to K W.
    if (!LN) {
      for (int x = tid; x < b * D; x += THREADS) G[x] = 2.0f * (G[x] - Vs[x]);
    } else {
      for (int r = warp; r < b; r += THREADS / 32) {
        float dy0, dy1;
        ln_residual_grad(G[r * D + lane], G[r * D + lane + 32], Ks[r * D + lane],
                         Ks[r * D + lane + 32], Vs[r * D + lane], Vs[r * D + lane + 32], gam0,
                         gam1, bet0, bet1, p.eps, dy0, dy1);
        G[r * D + lane] = dy0;
        G[r * D + lane + 32] = dy1;
      }
    }
    __syncthreads();

    // Pre-LN output Q W - A G.
    for (int t = rg; t < b; t += 4) {
      float acc = P[t * D + j];
      for (int s = 0; s <= t; ++s) acc = fmaf(-A[t * b + s], G[s * D + j], acc);
      P[t * D + j] = acc;
    }
    // State update W -= K^T diag(eta) G (W is no longer read this mini-batch).
    for (int x = tid; x < D * D; x += THREADS) {
      const int i = x / D, jj = x % D;
      float acc = 0.f;
      for (int t = 0; t < b; ++t) acc = fmaf(Ks[t * D + i] * es[t], G[t * D + jj], acc);
      W[x] -= acc;
    }
    __syncthreads();

    // Output.
    if (!LN) {
      for (int x = tid; x < b * D; x += THREADS) Zg[off + x] = P[x];
    } else {
      for (int r = warp; r < b; r += THREADS / 32) {
        float z0, z1;
        ln_residual_fwd(P[r * D + lane], P[r * D + lane + 32], Qs[r * D + lane],
                        Qs[r * D + lane + 32], gam0, gam1, bet0, bet1, p.eps, z0, z1);
        Zg[off + r * D + lane] = z0;
        Zg[off + r * D + lane + 32] = z1;
      }
    }
  }
  __syncthreads();
  float *Wo = p.W_out + unit * D * D;
  for (int x = tid; x < D * D; x += THREADS) Wo[x] = W[x];
}

inline size_t mlp_smem_bytes(int b) {
  return sizeof(float) * ((size_t)D * HID + (size_t)HID * W2_LD + 3 * (size_t)b * D +
                          4 * (size_t)b * HID + 2 * (size_t)b * D + 2 * (size_t)b * b + b);
}

template <typename InT>
__global__ void __launch_bounds__(THREADS) mlp_kernel(const Params p) {
  extern __shared__ __align__(16) float sm[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long unit = blockIdx.x;
  const int head = (int)(unit % p.H);
  const int b = p.b;  // <= 16
  float *W1 = sm;                 // [D][HID]
  float *W2 = W1 + D * HID;       // [HID][W2_LD]
  float *Qs = W2 + HID * W2_LD;   // [b][D]
  float *Ks = Qs + b * D;
  float *Vs = Ks + b * D;
  float *X1 = Vs + b * D;         // [b][HID]  K W1
  float *X2 = X1 + b * HID;       // [b][HID]  GELU(X1)
  float *G2 = X2 + b * HID;       // [b][HID]  dl/dX1
  float *ZQ = G2 + b * HID;       // [b][HID]  Q W1 -> Z1 -> GELU(Z1)
  float *G3 = ZQ + b * HID;       // [b][D]    X2 W2 -> dl/d(X2 W2)
  float *Z3 = G3 + b * D;         // [b][D]    pre-LN output
  float *A = Z3 + b * D;          // [b][b]    tril(Q K^T) diag(eta)
  float *A2 = A + b * b;          // [b][b]    tril(Z2 X2^T) diag(eta)
  float *es = A2 + b * b;         // [b]

  {
    const float *w1 = p.W0 + (long)head * D * HID;
    const float *w2 = p.W2_0 + (long)head * HID * D;
    for (int x = tid; x < D * HID; x += THREADS) W1[x] = w1[x];
    for (int x = tid; x < HID * D; x += THREADS) W2[(x / D) * W2_LD + x % D] = w2[x];
  }
  const float gam0 = p.gamma[head * D + lane], gam1 = p.gamma[head * D + lane + 32];
  const float bet0 = p.beta[head * D + lane], bet1 = p.beta[head * D + lane + 32];
  const long tok0 = unit * (long)p.T;
  const InT *Qg = (const InT *)p.Q + tok0 * D;
  const InT *Kg = (const InT *)p.K + tok0 * D;
  const InT *Vg = (const InT *)p.V + tok0 * D;
  float *Zg = p.Z + tok0 * D;
  const int nmb = p.T / b;
  const int i = tid;                           // hidden unit owned in [.][HID] passes
  const int j = tid & (D - 1), rg = tid >> 6;  // column / row group in [.][D] passes

  for (int n = 0; n < nmb; ++n) {
    __syncthreads();
    const long off = (long)n * b * D;
    for (int x = tid; x < b * D; x += THREADS) {
      Qs[x] = load_in(Qg, off + x);
      Ks[x] = load_in(Kg, off + x);
      Vs[x] = load_in(Vg, off + x);
    }
    if (tid < b) es[tid] = p.eta[tok0 + (long)n * b + tid];
    __syncthreads();

    // X1 = K W1, ZQ = Q W1 (column i of both).
    {
      float ak[16], aq[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) ak[r] = aq[r] = 0.f;
      for (int pp = 0; pp < D; ++pp) {
        const float w = W1[pp * HID + i];
#pragma unroll
        for (int r = 0; r < 16; ++r)
          if (r < b) {
            ak[r] = fmaf(Ks[r * D + pp], w, ak[r]);
            aq[r] = fmaf(Qs[r * D + pp], w, aq[r]);
          }
      }
#pragma unroll
      for (int r = 0; r < 16; ++r)
        if (r < b) {
          X1[r * HID + i] = ak[r];
          X2[r * HID + i] = gelu(ak[r]);
          ZQ[r * HID + i] = aq[r];
        }
    }
    for (int pr = warp; pr < b * b; pr += THREADS / 32) {
      const int t = pr / b, s = pr % b;
      float acc = 0.f;
      if (s <= t) {
        acc = fmaf(Qs[t * D + lane + 32], Ks[s * D + lane + 32], Qs[t * D + lane] * Ks[s * D + lane]);
        acc = warp_sum(acc) * es[s];
      }
      if (lane == 0) A[pr] = acc;
    }
    __syncthreads();

    // X3 = X2 W2 into G3.
    for (int t = rg; t < b; t += 4) {
      float acc = 0.f;
      for (int ii = 0; ii < HID; ++ii) acc = fmaf(X2[t * HID + ii], W2[ii * W2_LD + j], acc);
      G3[t * D + j] = acc;
    }
    __syncthreads();
    // G3 = dl / d X3 through LN and the residual.
    for (int r = warp; r < b; r += THREADS / 32) {
      float dy0, dy1;
      ln_residual_grad(G3[r * D + lane], G3[r * D + lane + 32], Ks[r * D + lane],
                       Ks[r * D + lane + 32], Vs[r * D + lane], Vs[r * D + lane + 32], gam0, gam1,
                       bet0, bet1, p.eps, dy0, dy1);
      G3[r * D + lane] = dy0;
      G3[r * D + lane + 32] = dy1;
    }
    __syncthreads();
    // G2 = (G3 W2^T) * GELU'(X1); then Z1 = Q W1 - A G2 and Z2 = GELU(Z1).
    {
      float acc[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) acc[r] = 0.f;
      for (int jj = 0; jj < D; ++jj) {
        const float w = W2[i * W2_LD + jj];
#pragma unroll
        for (int r = 0; r < 16; ++r)
          if (r < b) acc[r] = fmaf(G3[r * D + jj], w, acc[r]);
      }
#pragma unroll
      for (int r = 0; r < 16; ++r)
        if (r < b) acc[r] *= gelu_deriv(X1[r * HID + i]);
#pragma unroll
      for (int r = 0; r < 16; ++r)
        if (r < b) G2[r * HID + i] = acc[r];
#pragma unroll
      for (int t = 0; t < 16; ++t)
        if (t < b) {
          float z = ZQ[t * HID + i];
          for (int s = 0; s <= t; ++s) z = fmaf(-A[t * b + s], acc[s], z);
          ZQ[t * HID + i] = gelu(z);
        }
    }
    __syncthreads();
    // A2 = tril(Z2 X2^T) diag(eta).
    for (int pr = warp; pr < b * b; pr += THREADS / 32) {
      const int t = pr / b, s = pr % b;
      float acc = 0.f;
      if (s <= t) {
        for (int ii = lane; ii < HID; ii += 32) acc = fmaf(ZQ[t * HID + ii], X2[s * HID + ii], acc);
        acc = warp_sum(acc) * es[s];
      }
      if (lane == 0) A2[pr] = acc;
    }
    __syncthreads();
    // Z3 = Z2 W2 - A2 G3.
    for (int t = rg; t < b; t += 4) {
      float acc = 0.f;
      for (int ii = 0; ii < HID; ++ii) acc = fmaf(ZQ[t * HID + ii], W2[ii * W2_LD + j], acc);
      for (int s = 0; s <= t; ++s) acc = fmaf(-A2[t * b + s], G3[s * D + j], acc);
      Z3[t * D + j] = acc;
    }
    __syncthreads();
    // Output Z = Q + LN(Z3); state updates (W1, W2 are no longer read this mini-batch).
    for (int r = warp; r < b; r += THREADS / 32) {
      float z0, z1;
      ln_residual_fwd(Z3[r * D + lane], Z3[r * D + lane + 32], Qs[r * D + lane],
                      Qs[r * D + lane + 32], gam0, gam1, bet0, bet1, p.eps, z0, z1);
      Zg[off + r * D + lane] = z0;
      Zg[off + r * D + lane + 32] = z1;
    }
    {
      // W1[pp][i] -= sum_t K[t][pp] eta_t G2[t][i]
      float g[16];
#pragma unroll
      for (int t = 0; t < 16; ++t) g[t] = t < b ? es[t] * G2[t * HID + i] : 0.f;
      for (int pp = 0; pp < D; ++pp) {
        float acc = 0.f;
#pragma unroll
        for (int t = 0; t < 16; ++t)
          if (t < b) acc = fmaf(Ks[t * D + pp], g[t], acc);
        W1[pp * HID + i] -= acc;
      }
      // W2[ii][j] -= sum_t X2[t][ii] eta_t G3[t][j]
#pragma unroll
      for (int t = 0; t < 16; ++t) g[t] = t < b ? es[t] * G3[t * D + j] : 0.f;
      for (int ii = rg; ii < HID; ii += 4) {
        float acc = 0.f;
#pragma unroll
        for (int t = 0; t < 16; ++t)
          if (t < b) acc = fmaf(X2[t * HID + ii], g[t], acc);
        W2[ii * W2_LD + j] -= acc;
      }
    }
  }
  __syncthreads();
  float *w1o = p.W_out + unit * D * HID;
  float *w2o = p.W2_out + unit * HID * D;
  for (int x = tid; x < D * HID; x += THREADS) w1o[x] = W1[x];
  for (int x = tid; x < HID * D; x += THREADS) w2o[x] = W2[(x / D) * W2_LD + x % D];
}

}  // namespace simt
}  // namespace ttt
