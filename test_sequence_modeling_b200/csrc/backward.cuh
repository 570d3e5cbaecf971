// backward.cuh - backward pass of TTT-Linear and TTT-Linear + LN through the
// mini-batch chain, in the dual form (the TTT write-up computes the backward in
// the dual form too, §04.3), fp32 on the CUDA cores.
//
// Forward, per (batch, head) unit and mini-batch n with base state W = W_n
// (rows s, t = tokens of the mini-batch, A = tril(Q K^T) with the diagonal):
//   Y = K W,  G = dl/dY  (2 (Y - V), or through LN + residual, §03.9),  E = diag(eta) G
//   Zpre = Q W - A E,  Z = Zpre  (or Q + LN(Zpre))
//   W_{n+1} = W - K^T E
// Given dZ and dW_{n+1} (the cotangent of the next base; of W_T for the last),
// the reverse step is, with P = dL/dZpre (dZ, or through the output LN) and
// M = tril(P E^T):
//   dQ = P W^T - M K (+ dZ)              dE = -A^T P - K dW_{n+1}
//   deta_s = <dE_s, G_s>,  dG = diag(eta) dE,  (dY, dr) = VJP of G at dG
//   dK = -M^T Q - E dW_{n+1}^T + dY W^T (+ dr)
//   dW_n = dW_{n+1} + Q^T P + K^T dY
// where dY = 2 dG and dV = -2 dG for the plain loss, and with LN dV = -dr, dr
// being the cotangent of the residual r = k + LN(y) - v.  The LN of the
// gradient is differentiated once more (the VJP of G w.r.t. y, k, v, gamma,
// beta): with xhat, rstd the
// row's normalised y and 1/sigma, gx = 2 gamma r, m2 = mean(gx xhat) and
// u = rstd dG:
//   dgx   = u - mean(u) - xhat mean(u xhat)
//   dxhat = -m2 u - gx mean(u xhat) + gamma dr,   dr = 2 gamma dgx
//   dsig  = -sum(u G)
//   dY    = rstd (dxhat - mean(dxhat) - xhat mean(dxhat xhat)) + xhat dsig / D
//   dgamma += 2 r dgx + xhat dr,  dbeta += dr.
//
// Two passes per unit: the forward over the mini-batches writes W_n to the
// caller's W_ckpt (so the reverse pass needs no recomputation chain), then the
// reverse pass recomputes G, E (and the output LN) from W_n and applies the
// step above.  One CTA of 256 threads per unit; every [row][D] tile, W and dW
// live in shared memory with rows of D + 4 floats: 16-byte aligned, so that the
// products read four consecutive elements per load, and a row stride of 17
// 16-byte units, so that 16-byte walks down a column (one row per lane) are free
// of bank conflicts.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "simt.cuh"

namespace ttt {
namespace bwd {

constexpr int D = simt::D;
constexpr int MAXB = 16;     // largest mini-batch of this kernel
constexpr int LD = D + 4;    // row stride of every tile (16-byte rows, 17 x 16 bytes)
constexpr int BLD = MAXB + 1;
constexpr int THREADS = 256;

struct Params {
  const void *Q, *K, *V;       // [units][T][D]
  const float *eta;            // [units][T]
  const float *W0;             // [H][D][D]
  const float *gamma, *beta;   // [H][D] (LN)
  float eps;
  const float *dZ;             // [units][T][D]
  const float *dW_T;           // [units][D][D] or nullptr (zero)
  int H, T, b;
  float *dQ, *dK, *dV;         // [units][T][D]
  float *deta;                 // [units][T]
  float *dW0;                  // [units][D][D]
  float *dgamma, *dbeta;       // [units][D] (LN)
  float *W_ckpt;               // [units][T / b][D][D]
};

struct Smem {
  float W[D * LD], dW[D * LD];
  float Q[MAXB * LD], K[MAXB * LD], V[MAXB * LD], dZ[MAXB * LD];
  float G[MAXB * LD], E[MAXB * LD], P[MAXB * LD], dE[MAXB * LD], dY[MAXB * LD];
  float X[MAXB * LD];   // Y = K W, then (LN) its normalised value xhat
  float R[MAXB * LD];   // LN: r = k + gamma xhat + beta - v, then dr
  float Zh[MAXB * LD];  // LN: Zpre
  float A[MAXB * BLD], M[MAXB * BLD];
  float eta[MAXB], rstd[MAXB], m2[MAXB];
  float red[2][8][D];   // cross-warp sums of dgamma, dbeta
};

inline size_t smem_bytes() { return sizeof(Smem); }

// Four consecutive floats of a tile (16-byte aligned: rows are LD = D + 4 floats).
__device__ __forceinline__ float4 ld4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ float dot4(float4 a, float4 b, float acc) {
  return fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, fmaf(a.w, b.w, acc))));
}

// The [row][D] products are register-blocked over the four rows rq + 4k of a
// thread and four steps of the inner index: the row operands are warp-wide
// broadcasts read four elements at a time, so one column-operand load serves
// four FMAs and one row-operand load four more.  Rows at or beyond b hold stale
// values; their sums are computed and dropped.
//
// acc[k] += sum_i in[rq + 4k][i] W[i][c]
__device__ __forceinline__ void rows_W(const float *in, const float *W, int rq, int c,
                                       float (&acc)[4]) {
#pragma unroll 2
  for (int i = 0; i < D; i += 4) {
    const float4 w = make_float4(W[i * LD + c], W[(i + 1) * LD + c], W[(i + 2) * LD + c], W[(i + 3) * LD + c]);
#pragma unroll
    for (int k = 0; k < 4; ++k) acc[k] = dot4(ld4(in + (rq + 4 * k) * LD + i), w, acc[k]);
  }
}

// out[r][c] = sum_i in[r][i] W[i][c] for the rows r = rq, rq + 4, ... < b.
__device__ __forceinline__ void rows_times_W(const float *in, const float *W, float *out, int b,
                                             int rq, int c) {
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  rows_W(in, W, rq, c, acc);
#pragma unroll
  for (int k = 0; k < 4; ++k)
    if (rq + 4 * k < b) out[(rq + 4 * k) * LD + c] = acc[k];
}

// G (and E = eta G) of the rows warp, warp + 8 < b, from Y in s.X.  With LN the
// row's xhat replaces Y in s.X, r goes to s.R, and rstd, m2 are kept per row.
template <bool LN>
__device__ __forceinline__ void grad_rows(Smem &s, int b, int warp, int lane, float g0, float g1,
                                          float be0, float be1, float eps) {
  for (int r = warp; r < b; r += 8) {
    const int o = r * LD;
    const float y0 = s.X[o + lane], y1 = s.X[o + lane + 32];
    const float v0 = s.V[o + lane], v1 = s.V[o + lane + 32];
    float G0, G1;
    if (LN) {
      const float k0 = s.K[o + lane], k1 = s.K[o + lane + 32];
      const float mean = simt::warp_sum(y0 + y1) * (1.f / D);
      const float c0 = y0 - mean, c1 = y1 - mean;
      const float var = simt::warp_sum(c0 * c0 + c1 * c1) * (1.f / D);
      const float rs = rsqrtf(var + eps);
      const float xh0 = c0 * rs, xh1 = c1 * rs;
      const float r0 = k0 + g0 * xh0 + be0 - v0, r1 = k1 + g1 * xh1 + be1 - v1;
      const float gx0 = 2.f * g0 * r0, gx1 = 2.f * g1 * r1;
      const float m1 = simt::warp_sum(gx0 + gx1) * (1.f / D);
      const float m2 = simt::warp_sum(gx0 * xh0 + gx1 * xh1) * (1.f / D);
      G0 = rs * (gx0 - m1 - xh0 * m2);
      G1 = rs * (gx1 - m1 - xh1 * m2);
      s.X[o + lane] = xh0;
      s.X[o + lane + 32] = xh1;
      s.R[o + lane] = r0;
      s.R[o + lane + 32] = r1;
      if (lane == 0) {
        s.rstd[r] = rs;
        s.m2[r] = m2;
      }
    } else {
      G0 = 2.f * (y0 - v0);
      G1 = 2.f * (y1 - v1);
    }
    const float e = s.eta[r];
    s.G[o + lane] = G0;
    s.G[o + lane + 32] = G1;
    s.E[o + lane] = e * G0;
    s.E[o + lane + 32] = e * G1;
  }
}

template <typename InT>
__device__ __forceinline__ void load_tile(float *dst, const InT *src, long row0, int b, int tid) {
  for (int x = tid; x < b * D; x += THREADS) {
    const int r = x / D, c = x % D;
    dst[r * LD + c] = simt::load_in(src, (row0 + r) * D + c);
  }
}

template <bool LN, typename InT>
__global__ void __launch_bounds__(THREADS) linear_bwd_kernel(const Params p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Smem &s = *reinterpret_cast<Smem *>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int col = tid & (D - 1), rq = tid >> 6;  // [row][D] outputs: rows rq, rq + 4, ...
  const long unit = blockIdx.x;
  const int head = (int)(unit % p.H);
  const int b = p.b, T = p.T, N = T / b;
  const long tok0 = unit * (long)T;
  const InT *Qg = static_cast<const InT *>(p.Q) + tok0 * D;
  const InT *Kg = static_cast<const InT *>(p.K) + tok0 * D;
  const InT *Vg = static_cast<const InT *>(p.V) + tok0 * D;
  const float *etag = p.eta + tok0;
  const float *dZg = p.dZ + tok0 * D;
  float *ck = p.W_ckpt + unit * (long)N * D * D;

  float g0 = 0.f, g1 = 0.f, be0 = 0.f, be1 = 0.f;
  if (LN) {
    g0 = p.gamma[head * D + lane];
    g1 = p.gamma[head * D + lane + 32];
    be0 = p.beta[head * D + lane];
    be1 = p.beta[head * D + lane + 32];
  }
  float dg0 = 0.f, dg1 = 0.f, db0 = 0.f, db1 = 0.f;  // this lane's dgamma, dbeta partial sums

  for (int x = tid; x < D * D; x += THREADS) s.W[(x / D) * LD + x % D] = p.W0[(long)head * D * D + x];
  __syncthreads();

  // Forward over the mini-batches; W_n is checkpointed at each base.
  for (int n = 0; n < N; ++n) {
    float *ckn = ck + (long)n * D * D;
    for (int x = tid; x < D * D; x += THREADS) ckn[x] = s.W[(x / D) * LD + x % D];
    const long row0 = (long)n * b;
    load_tile(s.K, Kg, row0, b, tid);
    load_tile(s.V, Vg, row0, b, tid);
    if (tid < b) s.eta[tid] = etag[row0 + tid];
    __syncthreads();
    rows_times_W(s.K, s.W, s.X, b, rq, col);
    __syncthreads();
    grad_rows<LN>(s, b, warp, lane, g0, g1, be0, be1, p.eps);
    __syncthreads();
    // W -= K^T E; this thread's rows i = 16 rq + k of column col.
    {
      float acc[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) acc[k] = 0.f;
      for (int r = 0; r < b; ++r) {
        const float e = s.E[r * LD + col];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 kv = ld4(s.K + r * LD + 16 * rq + 4 * q);
          acc[4 * q] = fmaf(kv.x, e, acc[4 * q]);
          acc[4 * q + 1] = fmaf(kv.y, e, acc[4 * q + 1]);
          acc[4 * q + 2] = fmaf(kv.z, e, acc[4 * q + 2]);
          acc[4 * q + 3] = fmaf(kv.w, e, acc[4 * q + 3]);
        }
      }
#pragma unroll
      for (int k = 0; k < 16; ++k) s.W[(16 * rq + k) * LD + col] -= acc[k];
    }
    __syncthreads();
  }

  // Reverse pass.  dW holds the cotangent of the next mini-batch's base.
  for (int x = tid; x < D * D; x += THREADS)
    s.dW[(x / D) * LD + x % D] = p.dW_T ? p.dW_T[unit * D * D + x] : 0.f;
  __syncthreads();
  for (int n = N - 1; n >= 0; --n) {
    const long row0 = (long)n * b;
    const float *ckn = ck + (long)n * D * D;
    for (int x = tid; x < D * D; x += THREADS) s.W[(x / D) * LD + x % D] = ckn[x];
    load_tile(s.Q, Qg, row0, b, tid);
    load_tile(s.K, Kg, row0, b, tid);
    load_tile(s.V, Vg, row0, b, tid);
    load_tile(s.dZ, dZg, row0, b, tid);
    if (tid < b) s.eta[tid] = etag[row0 + tid];
    __syncthreads();

    // Y = K W and A = tril(Q K^T).
    rows_times_W(s.K, s.W, s.X, b, rq, col);
    {
      const int t = tid >> 4, u = tid & 15;
      if (t < b && u < b) {
        float a = 0.f;
        if (u <= t) {
#pragma unroll 4
          for (int i = 0; i < D; i += 4) a = dot4(ld4(s.Q + t * LD + i), ld4(s.K + u * LD + i), a);
        }
        s.A[t * BLD + u] = a;
      }
    }
    __syncthreads();
    grad_rows<LN>(s, b, warp, lane, g0, g1, be0, be1, p.eps);
    __syncthreads();

    if (LN) {
      // Zpre = Q W - A E, then P = dL/dZpre through the output LN.
      {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        rows_W(s.Q, s.W, rq, col, acc);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int r = rq + 4 * k;
          if (r < b) {
            float z = acc[k];
            for (int u = 0; u <= r; ++u) z = fmaf(-s.A[r * BLD + u], s.E[u * LD + col], z);
            s.Zh[r * LD + col] = z;
          }
        }
      }
      __syncthreads();
      for (int r = warp; r < b; r += 8) {
        const int o = r * LD;
        const float z0 = s.Zh[o + lane], z1 = s.Zh[o + lane + 32];
        const float mean = simt::warp_sum(z0 + z1) * (1.f / D);
        const float c0 = z0 - mean, c1 = z1 - mean;
        const float var = simt::warp_sum(c0 * c0 + c1 * c1) * (1.f / D);
        const float rs = rsqrtf(var + p.eps);
        const float zh0 = c0 * rs, zh1 = c1 * rs;
        const float dz0 = s.dZ[o + lane], dz1 = s.dZ[o + lane + 32];
        const float gz0 = dz0 * g0, gz1 = dz1 * g1;
        const float mg = simt::warp_sum(gz0 + gz1) * (1.f / D);
        const float mgx = simt::warp_sum(gz0 * zh0 + gz1 * zh1) * (1.f / D);
        s.P[o + lane] = rs * (gz0 - mg - zh0 * mgx);
        s.P[o + lane + 32] = rs * (gz1 - mg - zh1 * mgx);
        dg0 = fmaf(dz0, zh0, dg0);
        dg1 = fmaf(dz1, zh1, dg1);
        db0 += dz0;
        db1 += dz1;
      }
      __syncthreads();
    }
    const float *P = LN ? s.P : s.dZ;

    // M = tril(P E^T).
    {
      const int t = tid >> 4, u = tid & 15;
      if (t < b && u < b) {
        float m = 0.f;
        if (u <= t) {
#pragma unroll 4
          for (int j = 0; j < D; j += 4) m = dot4(ld4(P + t * LD + j), ld4(s.E + u * LD + j), m);
        }
        s.M[t * BLD + u] = m;
      }
    }
    __syncthreads();

    // dQ (to global) and dE.  Here col is the output column (i for dQ, j for dE).
    {
      float q[4] = {0.f, 0.f, 0.f, 0.f}, e[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 2
      for (int j = 0; j < D; j += 4) {
        const float4 w = ld4(s.W + col * LD + j);
        const float4 dw = make_float4(-s.dW[j * LD + col], -s.dW[(j + 1) * LD + col], -s.dW[(j + 2) * LD + col],
                                      -s.dW[(j + 3) * LD + col]);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          q[k] = dot4(ld4(P + (rq + 4 * k) * LD + j), w, q[k]);
          e[k] = dot4(ld4(s.K + (rq + 4 * k) * LD + j), dw, e[k]);
        }
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int r = rq + 4 * k;
        if (r < b) {
          float qq = LN ? q[k] + s.dZ[r * LD + col] : q[k];
          for (int u = 0; u <= r; ++u) qq = fmaf(-s.M[r * BLD + u], s.K[u * LD + col], qq);
          p.dQ[(tok0 + row0 + r) * D + col] = qq;
          float ee = e[k];
          for (int t = r; t < b; ++t) ee = fmaf(-s.A[t * BLD + r], P[t * LD + col], ee);
          s.dE[r * LD + col] = ee;
        }
      }
    }
    __syncthreads();

    // Per row: deta, dG, the VJP of G -> dY (and dr), dV.
    for (int r = warp; r < b; r += 8) {
      const int o = r * LD;
      const float de0 = s.dE[o + lane], de1 = s.dE[o + lane + 32];
      const float G0 = s.G[o + lane], G1 = s.G[o + lane + 32];
      const float de = simt::warp_sum(de0 * G0 + de1 * G1);
      if (lane == 0) p.deta[tok0 + row0 + r] = de;
      const float e = s.eta[r];
      const float dG0 = e * de0, dG1 = e * de1;
      float dY0, dY1, dV0, dV1;
      if (LN) {
        const float rs = s.rstd[r], m2 = s.m2[r];
        const float xh0 = s.X[o + lane], xh1 = s.X[o + lane + 32];
        const float r0 = s.R[o + lane], r1 = s.R[o + lane + 32];
        const float gx0 = 2.f * g0 * r0, gx1 = 2.f * g1 * r1;
        const float u0 = rs * dG0, u1 = rs * dG1;
        const float mu = simt::warp_sum(u0 + u1) * (1.f / D);
        const float mux = simt::warp_sum(u0 * xh0 + u1 * xh1) * (1.f / D);
        const float dsig = -simt::warp_sum(u0 * G0 + u1 * G1);
        const float dgx0 = u0 - mu - xh0 * mux, dgx1 = u1 - mu - xh1 * mux;
        const float dr0 = 2.f * g0 * dgx0, dr1 = 2.f * g1 * dgx1;
        dg0 += 2.f * r0 * dgx0 + xh0 * dr0;
        dg1 += 2.f * r1 * dgx1 + xh1 * dr1;
        db0 += dr0;
        db1 += dr1;
        const float dx0 = -m2 * u0 - gx0 * mux + g0 * dr0;
        const float dx1 = -m2 * u1 - gx1 * mux + g1 * dr1;
        const float mdx = simt::warp_sum(dx0 + dx1) * (1.f / D);
        const float mdxx = simt::warp_sum(dx0 * xh0 + dx1 * xh1) * (1.f / D);
        dY0 = rs * (dx0 - mdx - xh0 * mdxx) + xh0 * dsig * (1.f / D);
        dY1 = rs * (dx1 - mdx - xh1 * mdxx) + xh1 * dsig * (1.f / D);
        s.R[o + lane] = dr0;  // r is no longer needed: keep dr for dK
        s.R[o + lane + 32] = dr1;
        dV0 = -dr0;
        dV1 = -dr1;
      } else {
        dY0 = 2.f * dG0;
        dY1 = 2.f * dG1;
        dV0 = -dY0;
        dV1 = -dY1;
      }
      s.dY[o + lane] = dY0;
      s.dY[o + lane + 32] = dY1;
      p.dV[(tok0 + row0 + r) * D + lane] = dV0;
      p.dV[(tok0 + row0 + r) * D + lane + 32] = dV1;
    }
    __syncthreads();

    // dK (to global); col is the output column i.
    {
      float kk[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 2
      for (int j = 0; j < D; j += 4) {
        const float4 dw = ld4(s.dW + col * LD + j), w = ld4(s.W + col * LD + j);
        const float4 ndw = make_float4(-dw.x, -dw.y, -dw.z, -dw.w);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          kk[k] = dot4(ld4(s.E + (rq + 4 * k) * LD + j), ndw, kk[k]);
          kk[k] = dot4(ld4(s.dY + (rq + 4 * k) * LD + j), w, kk[k]);
        }
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int r = rq + 4 * k;
        if (r < b) {
          float v = LN ? kk[k] + s.R[r * LD + col] : kk[k];
          for (int t = r; t < b; ++t) v = fmaf(-s.M[t * BLD + r], s.Q[t * LD + col], v);
          p.dK[(tok0 + row0 + r) * D + col] = v;
        }
      }
    }
    __syncthreads();

    // dW_n = dW_{n+1} + Q^T P + K^T dY; this thread's rows i = 16 rq + k of column col.
    {
      float acc[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) acc[k] = 0.f;
      for (int r = 0; r < b; ++r) {
        const float pr = P[r * LD + col], dyr = s.dY[r * LD + col];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 qv = ld4(s.Q + r * LD + 16 * rq + 4 * q), kv = ld4(s.K + r * LD + 16 * rq + 4 * q);
          acc[4 * q] = fmaf(kv.x, dyr, fmaf(qv.x, pr, acc[4 * q]));
          acc[4 * q + 1] = fmaf(kv.y, dyr, fmaf(qv.y, pr, acc[4 * q + 1]));
          acc[4 * q + 2] = fmaf(kv.z, dyr, fmaf(qv.z, pr, acc[4 * q + 2]));
          acc[4 * q + 3] = fmaf(kv.w, dyr, fmaf(qv.w, pr, acc[4 * q + 3]));
        }
      }
#pragma unroll
      for (int k = 0; k < 16; ++k) s.dW[(16 * rq + k) * LD + col] += acc[k];
    }
    __syncthreads();
  }

  for (int x = tid; x < D * D; x += THREADS) p.dW0[unit * D * D + x] = s.dW[(x / D) * LD + x % D];
  if (LN) {
    s.red[0][warp][lane] = dg0;
    s.red[0][warp][lane + 32] = dg1;
    s.red[1][warp][lane] = db0;
    s.red[1][warp][lane + 32] = db1;
    __syncthreads();
    if (tid < 2 * D) {
      const int which = tid / D, c = tid % D;
      float acc = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) acc += s.red[which][w][c];
      (which ? p.dbeta : p.dgamma)[unit * D + c] = acc;
    }
  }
}

}  // namespace bwd
}  // namespace ttt
