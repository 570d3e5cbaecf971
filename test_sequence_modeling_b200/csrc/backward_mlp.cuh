// backward_mlp.cuh - backward pass of TTT-MLP, f(x) = x + LN(GELU(x W1) W2),
// through the mini-batch chain in the dual form (the TTT write-up computes the
// backward in the dual form too, §04.3), fp32 on the CUDA cores.
//
// Forward at the base (W1, W2) of mini-batch n, E = diag(eta):
//   X1 = K W1, X2 = GELU(X1), G3 = dl/dX3 at X3 = X2 W2, H = G3 W2^T,
//   G2 = H * GELU'(X1), E2 = E G2, E3 = E G3,
//   Z1 = Q W1 - A1 E2 (A1 = tril(Q K^T)), Z2 = GELU(Z1),
//   Z3 = Z2 W2 - A2 E3 (A2 = tril(Z2 X2^T)), Z = Q + LN(Z3),
//   W1' = W1 - K^T E2, W2' = W2 - X2^T E3.
// Reverse, given dZ and the cotangents dW1', dW2' of the next base: P3 = the
// output LN backward of dZ;
//   M2 = tril(P3 E3^T): dZ2 = P3 W2^T - M2 X2, dX2 = -M2^T Z2 - E3 dW2'^T,
//   dE3 = -A2^T P3 - X2 dW2',  dW2 = dW2' + Z2^T P3;
//   dZ1 = dZ2 * GELU'(Z1), M1 = tril(dZ1 E2^T): dQ = dZ + dZ1 W1^T - M1 K,
//   dK = -M1^T Q - E2 dW1'^T, dE2 = -A1^T dZ1 - K dW1', dW1 = dW1' + Q^T dZ1;
//   deta = rowsum(dE2 * G2 + dE3 * G3), dG2 = E dE2, dG3 = E dE3;
//   dH = dG2 * GELU'(X1), dX1 = dG2 * H * GELU''(X1), GELU''(x) = phi(x)(2 - x^2);
//   dG3 += dH W2, dW2 += dH^T G3;
//   (dX3, dr) = VJP of the LN loss gradient at dG3 (the LN of the gradient
//   differentiated once more): dK += dr, dV = -dr;
//   dX2 += dX3 W2^T, dW2 += X2^T dX3;  dX1 += dX2 * GELU'(X1);
//   dK += dX1 W1^T, dW1 += K^T dX1.
// (The VJP of the LN loss gradient, with xhat, rstd of X3's row, r = k + gamma
// xhat + beta - v, gx = 2 gamma r, m2 = mean(gx xhat), u = rstd dG3:
//   dgx = u - mean(u) - xhat mean(u xhat),  dr = 2 gamma dgx,
//   dxhat = -m2 u - gx mean(u xhat) + gamma dr,  dsig = -sum(u G3),
//   dX3 = rstd (dxhat - mean(dxhat) - xhat mean(dxhat xhat)) + xhat dsig / d,
//   dgamma += 2 r dgx + xhat dr, dbeta += dr.)
//
// One CTA of 16 warps per (batch, head) unit.  A forward pass writes the state
// at every mini-batch start to the caller's checkpoint buffers (the reverse pass
// reads them back instead of recomputing the chain); the reverse pass keeps the
// [b x hidden] and [b x d] tiles of one mini-batch in shared memory, reads the
// state from its checkpoint (L2) and accumulates the state cotangents in place
// in the caller's dW1, dW2 outputs.  Products stream the [d x hidden] matrices
// from global memory with coalesced loads; the tiles' operand reads are
// warp-wide broadcasts.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "mlp_tiles.cuh"

namespace ttt {
namespace bwdmlp {

using namespace ::ttt::mlptile;

struct Params {
  const void *Q, *K, *V;          // [units][T][D]
  const float *eta;               // [units][T]
  const float *W1_0, *W2_0;       // [H][D][HID], [H][HID][D]
  const float *gamma, *beta;      // [H][D]
  float eps;
  const float *dZ;                // [units][T][D]
  const float *dW1_T, *dW2_T;     // [units][D][HID], [units][HID][D] or nullptr (zero)
  int H, T, b;
  float *dQ, *dK, *dV;            // [units][T][D]
  float *deta;                    // [units][T]
  float *dW1, *dW2;               // [units][D][HID], [units][HID][D]
  float *dgamma, *dbeta;          // [units][D]
  float *W1_ckpt, *W2_ckpt;       // [units][T / b][D][HID], [units][T / b][HID][D]
};

struct Smem {
  // [b][d] tiles
  float Q[MAXB * LDD], K[MAXB * LDD], V[MAXB * LDD], dZ[MAXB * LDD];
  float X3[MAXB * LDD];    // X3, then its normalised row xhat
  float R[MAXB * LDD];     // r = k + gamma xhat + beta - v
  float GX[MAXB * LDD];    // gx = 2 gamma r
  float G3[MAXB * LDD], E3[MAXB * LDD], Z3[MAXB * LDD], P3[MAXB * LDD];
  float dE3[MAXB * LDD], dG3[MAXB * LDD], dX3[MAXB * LDD], dQ[MAXB * LDD], dK[MAXB * LDD];
  // [b][hidden] tiles
  float T1[MAXB * LDH];  // X1
  float T2[MAXB * LDH];  // X2
  float T3[MAXB * LDH];  // H
  float T4[MAXB * LDH];  // E2, then dX1
  float T5[MAXB * LDH];  // Z1, then dX2
  float T6[MAXB * LDH];  // Z2, then dE2 / dG2
  float T7[MAXB * LDH];  // dZ2 / dZ1, then dH
  // [b][b] masked Grams
  float A1[MAXB * LDB], A2[MAXB * LDB], M1[MAXB * LDB], M2[MAXB * LDB];
  float eta[MAXB], rs[MAXB], m2[MAXB];
  float gam[D], bet[D];
  float red[2 * 16 * D];   // per-warp dgamma / dbeta partials
};

inline size_t smem_bytes() { return sizeof(Smem); }

// The forward quantities of one mini-batch at the base (W1, W2): X1, X2, X3's
// LN loss gradient G3 (with its context), E3, H and E2.  Tiles Q, K, V, eta loaded.
__device__ void forward_grads(Smem &s, const float *W1, const float *W2, int b, float eps, int tid,
                              int warp, int lane) {
  mm_W<HID>(s.T1, LDH, s.K, LDD, W1, D, b, 1.f, false, tid);  // X1 = K W1
  __syncthreads();
  for (int x = tid; x < b * HID; x += THREADS) s.T2[(x / HID) * LDH + x % HID] = gelu(s.T1[(x / HID) * LDH + x % HID]);
  __syncthreads();
  mm_W<D>(s.X3, LDD, s.T2, LDH, W2, HID, b, 1.f, false, tid);  // X3 = X2 W2
  __syncthreads();
  if (warp < b) {  // the LN loss gradient of token `warp`
    const int t = warp, c0 = 2 * lane;
    const float x0 = s.X3[t * LDD + c0], x1 = s.X3[t * LDD + c0 + 1];
    const float mean = wsum(x0 + x1) * (1.f / D);
    const float d0 = x0 - mean, d1 = x1 - mean;
    const float rs = rsqrtf(wsum(d0 * d0 + d1 * d1) * (1.f / D) + eps);
    const float h0 = d0 * rs, h1 = d1 * rs;
    const float r0 = s.K[t * LDD + c0] + s.gam[c0] * h0 + s.bet[c0] - s.V[t * LDD + c0];
    const float r1 = s.K[t * LDD + c0 + 1] + s.gam[c0 + 1] * h1 + s.bet[c0 + 1] - s.V[t * LDD + c0 + 1];
    const float gx0 = 2.f * s.gam[c0] * r0, gx1 = 2.f * s.gam[c0 + 1] * r1;
    const float m1 = wsum(gx0 + gx1) * (1.f / D);
    const float m2 = wsum(gx0 * h0 + gx1 * h1) * (1.f / D);
    const float g0 = rs * (gx0 - m1 - h0 * m2), g1 = rs * (gx1 - m1 - h1 * m2);
    s.X3[t * LDD + c0] = h0;
    s.X3[t * LDD + c0 + 1] = h1;
    s.R[t * LDD + c0] = r0;
    s.R[t * LDD + c0 + 1] = r1;
    s.GX[t * LDD + c0] = gx0;
    s.GX[t * LDD + c0 + 1] = gx1;
    s.G3[t * LDD + c0] = g0;
    s.G3[t * LDD + c0 + 1] = g1;
    s.E3[t * LDD + c0] = s.eta[t] * g0;
    s.E3[t * LDD + c0 + 1] = s.eta[t] * g1;
    if (lane == 0) {
      s.rs[t] = rs;
      s.m2[t] = m2;
    }
  }
  __syncthreads();
  mm_WT<HID>(s.T3, LDH, s.G3, LDD, W2, D, b, 1.f, false, tid);  // H = G3 W2^T
  __syncthreads();
  for (int x = tid; x < b * HID; x += THREADS) {
    const int t = x / HID, j = x % HID;
    s.T4[t * LDH + j] = s.eta[t] * s.T3[t * LDH + j] * gelu_d(s.T1[t * LDH + j]);  // E2
  }
  __syncthreads();
}

template <typename InT>
__global__ void __launch_bounds__(THREADS, 1) mlp_bwd_kernel(const Params p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Smem &s = *reinterpret_cast<Smem *>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long unit = blockIdx.x;
  const int head = (int)(unit % p.H);
  const int b = p.b, T = p.T, N = T / b;
  const long tok0 = unit * (long)T;
  const InT *Qg = static_cast<const InT *>(p.Q) + tok0 * D;
  const InT *Kg = static_cast<const InT *>(p.K) + tok0 * D;
  const InT *Vg = static_cast<const InT *>(p.V) + tok0 * D;
  const float *etag = p.eta + tok0;
  const float *dZg = p.dZ + tok0 * D;
  float *ck1 = p.W1_ckpt + unit * (long)N * D * HID;
  float *ck2 = p.W2_ckpt + unit * (long)N * HID * D;
  float *dW1 = p.dW1 + unit * (long)D * HID;
  float *dW2 = p.dW2 + unit * (long)HID * D;

  for (int x = tid; x < (int)(sizeof(Smem) / 4); x += THREADS) reinterpret_cast<float *>(smem_raw)[x] = 0.f;
  __syncthreads();
  if (tid < D) {
    s.gam[tid] = p.gamma[head * D + tid];
    s.bet[tid] = p.beta[head * D + tid];
  }
  for (int x = tid; x < D * HID; x += THREADS) {
    dW1[x] = p.dW1_T ? p.dW1_T[unit * (long)D * HID + x] : 0.f;
    dW2[x] = p.dW2_T ? p.dW2_T[unit * (long)HID * D + x] : 0.f;
  }
  if (N > 0) {
    for (int x = tid; x < D * HID; x += THREADS) {
      ck1[x] = p.W1_0[(long)head * D * HID + x];
      ck2[x] = p.W2_0[(long)head * HID * D + x];
    }
  }
  __syncthreads();

  // Forward over the mini-batches: the state at each mini-batch start.
  for (int n = 0; n + 1 < N; ++n) {
    const long row0 = (long)n * b;
    load_rows(s.K, Kg, row0, b, tid);
    load_rows(s.V, Vg, row0, b, tid);
    if (tid < b) s.eta[tid] = etag[row0 + tid];
    __syncthreads();
    const float *W1 = ck1 + (long)n * D * HID, *W2 = ck2 + (long)n * HID * D;
    forward_grads(s, W1, W2, b, p.eps, tid, warp, lane);
    outer<D, HID>(ck1 + (long)(n + 1) * D * HID, W1, s.K, LDD, s.T4, LDH, b, -1.f, tid);   // W1 - K^T E2
    outer<HID, D>(ck2 + (long)(n + 1) * HID * D, W2, s.T2, LDH, s.E3, LDD, b, -1.f, tid);  // W2 - X2^T E3
    __syncthreads();
  }

  float dg0 = 0.f, dg1 = 0.f, db0 = 0.f, db1 = 0.f;  // this lane's dgamma / dbeta partials
  for (int n = N - 1; n >= 0; --n) {
    const long row0 = (long)n * b;
    const float *W1 = ck1 + (long)n * D * HID, *W2 = ck2 + (long)n * HID * D;
    load_rows(s.Q, Qg, row0, b, tid);
    load_rows(s.K, Kg, row0, b, tid);
    load_rows(s.V, Vg, row0, b, tid);
    for (int x = tid; x < b * D; x += THREADS) s.dZ[(x / D) * LDD + x % D] = dZg[(row0 + x / D) * D + x % D];
    if (tid < b) s.eta[tid] = etag[row0 + tid];
    __syncthreads();
    forward_grads(s, W1, W2, b, p.eps, tid, warp, lane);

    // Outputs of the mini-batch, recomputed.
    gram_tril(s.A1, s.Q, LDD, s.K, LDD, D, b, tid);  // A1 = tril(Q K^T)
    __syncthreads();
    mm_W<HID>(s.T5, LDH, s.Q, LDD, W1, D, b, 1.f, false, tid);  // Z1 = Q W1 - A1 E2
    small_corr<HID>(s.T5, LDH, s.A1, false, s.T4, LDH, b, -1.f, tid);
    __syncthreads();
    for (int x = tid; x < b * HID; x += THREADS) s.T6[(x / HID) * LDH + x % HID] = gelu(s.T5[(x / HID) * LDH + x % HID]);
    __syncthreads();
    gram_tril(s.A2, s.T6, LDH, s.T2, LDH, HID, b, tid);  // A2 = tril(Z2 X2^T)
    __syncthreads();
    mm_W<D>(s.Z3, LDD, s.T6, LDH, W2, HID, b, 1.f, false, tid);  // Z3 = Z2 W2 - A2 E3
    small_corr<D>(s.Z3, LDD, s.A2, false, s.E3, LDD, b, -1.f, tid);
    __syncthreads();
    if (warp < b) {  // output LN backward: P3, and the LN parameters' gradients
      const int t = warp, c0 = 2 * lane;
      const float z0 = s.Z3[t * LDD + c0], z1 = s.Z3[t * LDD + c0 + 1];
      const float mean = wsum(z0 + z1) * (1.f / D);
      const float e0 = z0 - mean, e1 = z1 - mean;
      const float rz = rsqrtf(wsum(e0 * e0 + e1 * e1) * (1.f / D) + p.eps);
      const float zh0 = e0 * rz, zh1 = e1 * rz;
      const float dz0 = s.dZ[t * LDD + c0], dz1 = s.dZ[t * LDD + c0 + 1];
      const float gz0 = dz0 * s.gam[c0], gz1 = dz1 * s.gam[c0 + 1];
      const float ma = wsum(gz0 + gz1) * (1.f / D), mb = wsum(gz0 * zh0 + gz1 * zh1) * (1.f / D);
      s.P3[t * LDD + c0] = rz * (gz0 - ma - zh0 * mb);
      s.P3[t * LDD + c0 + 1] = rz * (gz1 - ma - zh1 * mb);
      dg0 += dz0 * zh0;
      dg1 += dz1 * zh1;
      db0 += dz0;
      db1 += dz1;
    }
    __syncthreads();

    // Reverse step.
    gram_tril(s.M2, s.P3, LDD, s.E3, LDD, D, b, tid);  // M2 = tril(P3 E3^T)
    __syncthreads();
    mm_WT<HID>(s.T7, LDH, s.P3, LDD, W2, D, b, 1.f, false, tid);  // dZ2 = P3 W2^T - M2 X2
    small_corr<HID>(s.T7, LDH, s.M2, false, s.T2, LDH, b, -1.f, tid);
    {  // dZ1 = dZ2 * GELU'(Z1), for this thread's entries
      constexpr int RPT = MAXB / (THREADS / HID);
      const int j = tid % HID, g = tid / HID;
      for (int r = 0; r < RPT; ++r) {
        const int t = g * RPT + r;
        if (t < b) s.T7[t * LDH + j] *= gelu_d(s.T5[t * LDH + j]);
      }
    }
    __syncthreads();
    mm_WT<HID>(s.T5, LDH, s.E3, LDD, dW2, D, b, -1.f, false, tid);  // dX2 = -M2^T Z2 - E3 dW2'^T
    small_corr<HID>(s.T5, LDH, s.M2, true, s.T6, LDH, b, -1.f, tid);
    mm_W<D>(s.dE3, LDD, s.T2, LDH, dW2, HID, b, -1.f, false, tid);  // dE3 = -A2^T P3 - X2 dW2'
    small_corr<D>(s.dE3, LDD, s.A2, true, s.P3, LDD, b, -1.f, tid);
    gram_tril(s.M1, s.T7, LDH, s.T4, LDH, HID, b, tid);            // M1 = tril(dZ1 E2^T)
    __syncthreads();
    outer<HID, D>(dW2, dW2, s.T6, LDH, s.P3, LDD, b, 1.f, tid);    // dW2 += Z2^T P3
    mm_WT<D>(s.dQ, LDD, s.T7, LDH, W1, HID, b, 1.f, false, tid);   // dQ = dZ + dZ1 W1^T - M1 K
    small_corr<D>(s.dQ, LDD, s.M1, false, s.K, LDD, b, -1.f, tid);
    mm_WT<D>(s.dK, LDD, s.T4, LDH, dW1, HID, b, -1.f, false, tid); // dK = -M1^T Q - E2 dW1'^T
    small_corr<D>(s.dK, LDD, s.M1, true, s.Q, LDD, b, -1.f, tid);
    __syncthreads();
    mm_W<HID>(s.T6, LDH, s.K, LDD, dW1, D, b, -1.f, false, tid);   // dE2 = -A1^T dZ1 - K dW1'
    small_corr<HID>(s.T6, LDH, s.A1, true, s.T7, LDH, b, -1.f, tid);
    __syncthreads();
    outer<D, HID>(dW1, dW1, s.Q, LDD, s.T7, LDH, b, 1.f, tid);     // dW1 += Q^T dZ1
    if (warp < b) {  // deta = rowsum(dE2 G2 + dE3 G3); dG2 = eta dE2, dG3 = eta dE3
      const int t = warp;
      float v = 0.f;
      for (int j = lane; j < HID; j += 32)
        v = fmaf(s.T6[t * LDH + j], s.T3[t * LDH + j] * gelu_d(s.T1[t * LDH + j]), v);
      v = fmaf(s.dE3[t * LDD + 2 * lane], s.G3[t * LDD + 2 * lane], v);
      v = fmaf(s.dE3[t * LDD + 2 * lane + 1], s.G3[t * LDD + 2 * lane + 1], v);
      v = wsum(v);
      if (lane == 0) p.deta[tok0 + row0 + t] = v;
      s.dG3[t * LDD + 2 * lane] = s.eta[t] * s.dE3[t * LDD + 2 * lane];
      s.dG3[t * LDD + 2 * lane + 1] = s.eta[t] * s.dE3[t * LDD + 2 * lane + 1];
    }
    __syncthreads();
    for (int x = tid; x < b * HID; x += THREADS) {  // dH = dG2 GELU'(X1), dX1 = dG2 H GELU''(X1)
      const int t = x / HID, j = x % HID;
      const float x1 = s.T1[t * LDH + j], dg2 = s.eta[t] * s.T6[t * LDH + j];
      const float ph = phi(x1);
      s.T7[t * LDH + j] = dg2 * (normcdff(x1) + x1 * ph);
      s.T4[t * LDH + j] = dg2 * s.T3[t * LDH + j] * ph * (2.f - x1 * x1);
    }
    __syncthreads();
    mm_W<D>(s.dG3, LDD, s.T7, LDH, W2, HID, b, 1.f, true, tid);  // dG3 += dH W2
    outer<HID, D>(dW2, dW2, s.T7, LDH, s.G3, LDD, b, 1.f, tid);  // dW2 += dH^T G3
    __syncthreads();
    if (warp < b) {  // VJP of the LN loss gradient at dG3: dX3, dr
      const int t = warp, c0 = 2 * lane;
      const float rs = s.rs[t], m2 = s.m2[t];
      const float xh0 = s.X3[t * LDD + c0], xh1 = s.X3[t * LDD + c0 + 1];
      const float u0 = rs * s.dG3[t * LDD + c0], u1 = rs * s.dG3[t * LDD + c0 + 1];
      const float mu = wsum(u0 + u1) * (1.f / D), mux = wsum(u0 * xh0 + u1 * xh1) * (1.f / D);
      const float dsig = -wsum(u0 * s.G3[t * LDD + c0] + u1 * s.G3[t * LDD + c0 + 1]);
      const float dgx0 = u0 - mu - xh0 * mux, dgx1 = u1 - mu - xh1 * mux;
      const float g0 = s.gam[c0], g1 = s.gam[c0 + 1];
      const float dr0 = 2.f * g0 * dgx0, dr1 = 2.f * g1 * dgx1;
      dg0 += 2.f * s.R[t * LDD + c0] * dgx0 + xh0 * dr0;
      dg1 += 2.f * s.R[t * LDD + c0 + 1] * dgx1 + xh1 * dr1;
      db0 += dr0;
      db1 += dr1;
      const float dx0 = -m2 * u0 - s.GX[t * LDD + c0] * mux + g0 * dr0;
      const float dx1 = -m2 * u1 - s.GX[t * LDD + c0 + 1] * mux + g1 * dr1;
      const float mdx = wsum(dx0 + dx1) * (1.f / D), mdxh = wsum(dx0 * xh0 + dx1 * xh1) * (1.f / D);
      s.dX3[t * LDD + c0] = rs * (dx0 - mdx - xh0 * mdxh) + xh0 * dsig * (1.f / D);
      s.dX3[t * LDD + c0 + 1] = rs * (dx1 - mdx - xh1 * mdxh) + xh1 * dsig * (1.f / D);
      s.dK[t * LDD + c0] += dr0;
      s.dK[t * LDD + c0 + 1] += dr1;
      p.dV[(tok0 + row0 + t) * D + c0] = -dr0;
      p.dV[(tok0 + row0 + t) * D + c0 + 1] = -dr1;
    }
    __syncthreads();
    mm_WT<HID>(s.T5, LDH, s.dX3, LDD, W2, D, b, 1.f, true, tid);  // dX2 += dX3 W2^T
    outer<HID, D>(dW2, dW2, s.T2, LDH, s.dX3, LDD, b, 1.f, tid);  // dW2 += X2^T dX3
    __syncthreads();
    for (int x = tid; x < b * HID; x += THREADS) {  // dX1 += dX2 GELU'(X1)
      const int t = x / HID, j = x % HID;
      s.T4[t * LDH + j] += s.T5[t * LDH + j] * gelu_d(s.T1[t * LDH + j]);
    }
    __syncthreads();
    mm_WT<D>(s.dK, LDD, s.T4, LDH, W1, HID, b, 1.f, true, tid);   // dK += dX1 W1^T
    outer<D, HID>(dW1, dW1, s.K, LDD, s.T4, LDH, b, 1.f, tid);    // dW1 += K^T dX1
    __syncthreads();
    for (int x = tid; x < b * D; x += THREADS) {
      const int t = x / D, c = x % D;
      p.dQ[(tok0 + row0 + t) * D + c] = s.dQ[t * LDD + c] + s.dZ[t * LDD + c];
      p.dK[(tok0 + row0 + t) * D + c] = s.dK[t * LDD + c];
    }
    __syncthreads();
  }

  // dgamma, dbeta: this unit's sums over its tokens.
  s.red[warp * D + 2 * lane] = dg0;
  s.red[warp * D + 2 * lane + 1] = dg1;
  s.red[16 * D + warp * D + 2 * lane] = db0;
  s.red[16 * D + warp * D + 2 * lane + 1] = db1;
  __syncthreads();
  if (tid < D) {
    float a = 0.f, c = 0.f;
    for (int w = 0; w < 16; ++w) {
      a += s.red[w * D + tid];
      c += s.red[16 * D + w * D + tid];
    }
    p.dgamma[unit * D + tid] = a;
    p.dbeta[unit * D + tid] = c;
  }
}

}  // namespace bwdmlp
}  // namespace ttt
