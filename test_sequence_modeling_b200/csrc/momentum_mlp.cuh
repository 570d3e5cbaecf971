// momentum_mlp.cuh - whole-sequence forward of TTT-MLP, f(x) = x + LN(GELU(x W1) W2),
// with the momentum and decay update of the Titans article (§二.1(2): momentum on
// past surprise, a forget gate that decays the memory; its memory is an MLP,
// §二.1(3)), kept to the TTT mini-batch rule: with S_0 = 0 and g_t the loss
// gradient at the state the mini-batch of token t started from,
//   S_t = alpha_t S_{t-1} - eta_t g_t,   W_t = (1 - lambda_t) W_{t-1} + S_t,
//   z_t = f(q_t; W_t),
// for both layers.  fp32 on the CUDA cores.
//
// Dual form.  Inside a mini-batch with base state (W_b, S_b) and local tokens
// t, s = 0 .. b-1, the recursion is linear in the base and in the gradients:
//   S_t = A_t S_b - sum_{s<=t} a_{t,s} eta_s g_s
//   W_t = Lam_t W_b + C_t S_b - sum_{s<=t} c_{t,s} eta_s g_s
// with A_t = prod_{r<=t} alpha_r, Lam_t = prod_{r<=t} (1 - lambda_r),
// C_t = (1 - lambda_t) C_{t-1} + A_t, a_{t,s} = prod_{s<r<=t} alpha_r and
// c_{t,s} = (1 - lambda_t) c_{t-1,s} + a_{t,s} (c_{s,s} = a_{s,s} = 1).  The
// layer-1 gradient of token s is k_s^T G2_s and the layer-2 one X2_s^T G3_s,
// all taken at the base (X1 = K W1_b, X2 = GELU(X1), G3 through the LN loss,
// G2 = (G3 W2_b^T) GELU'(X1)), so
//   Zq1 = diag(Lam) Q W1_b + diag(C) Q S1_b - (c o tril(Q K^T)) diag(eta) G2,
//   Zq2 = GELU(Zq1),
//   Zq3 = diag(Lam) Zq2 W2_b + diag(C) Zq2 S2_b - (c o tril(Zq2 X2^T)) diag(eta) G3,
//   Z = Q + LN(Zq3),
// and at the end of the mini-batch (t = b - 1) both states follow from the
// last row of the coefficients.  alpha = lambda = 0 gives A = C = 0, Lam = 1 and
// c = a = tril(1): the TTT-MLP dual form.
//
// One CTA of 16 warps per (batch, head) unit; the state (W1, W2, S1, S2) lives
// in the caller's outputs in global memory (L2) for the whole sequence and the
// mini-batch's tiles in shared memory (mlp_tiles.cuh).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "mlp_tiles.cuh"

namespace ttt {
namespace mommlp {

using namespace ::ttt::mlptile;

struct Params {
  const void *Q, *K, *V;              // [units][T][D]
  const float *eta, *alpha, *lambda;  // [units][T]
  const float *W1_0, *W2_0;           // [H][D][HID], [H][HID][D]
  const float *gamma, *beta;          // [H][D]
  float eps;
  int H, T, b;
  float *Z;                           // [units][T][D]
  float *W1, *W2, *S1, *S2;           // [units][D][HID], [units][HID][D] (x2): the running state
};

struct Smem {
  float Q[MAXB * LDD], K[MAXB * LDD], V[MAXB * LDD];
  float X3[MAXB * LDD], G3[MAXB * LDD], Z3[MAXB * LDD];
  float X1[MAXB * LDH], X2[MAXB * LDH], G2[MAXB * LDH], Z1[MAXB * LDH], Z2[MAXB * LDH];
  float A1[MAXB * LDB], A2[MAXB * LDB];  // coefficient-weighted masked Grams (with eta)
  float cW[MAXB * LDB], cS[MAXB * LDB];  // c_{t,s}, a_{t,s}
  float eta[MAXB], alpha[MAXB], keep[MAXB], lam[MAXB], cb[MAXB];
  float wW[MAXB], wS[MAXB];              // c_{b-1,s} eta_s, a_{b-1,s} eta_s
  float fin[4];                          // Lam, C, A at the last token
  float gam[D], bet[D];
};

inline size_t smem_bytes() { return sizeof(Smem); }

// out[t][j] = Lam_t sum_k A[t][k] W[k][j] + C_t sum_k A[t][k] S[k][j]  (W, S global [Kd][N]).
template <int N>
__device__ void mm_two(float *out, int ldo, const float *A, int lda, const float *W, const float *S,
                       const float *lam, const float *cb, int Kd, int b, int tid) {
  constexpr int TPC = THREADS / N, RPT = MAXB / TPC;
  const int j = tid % N, g = tid / N;
  float a[RPT], c[RPT];
#pragma unroll
  for (int r = 0; r < RPT; ++r) a[r] = c[r] = 0.f;
#pragma unroll 2
  for (int k = 0; k < Kd; k += 4) {
    float w[4], sv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      w[u] = W[(size_t)(k + u) * N + j];
      sv[u] = S[(size_t)(k + u) * N + j];
    }
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
      const float4 x = ld4(A + (g * RPT + r) * lda + k);
      a[r] = fmaf(x.w, w[3], fmaf(x.z, w[2], fmaf(x.y, w[1], fmaf(x.x, w[0], a[r]))));
      c[r] = fmaf(x.w, sv[3], fmaf(x.z, sv[2], fmaf(x.y, sv[1], fmaf(x.x, sv[0], c[r]))));
    }
  }
#pragma unroll
  for (int r = 0; r < RPT; ++r) {
    const int t = g * RPT + r;
    if (t < b) out[t * ldo + j] = lam[t] * a[r] + cb[t] * c[r];
  }
}

// The end-of-mini-batch state of one layer, element by element:
//   W <- Lam W + C S - sum_t L[t][r] wW_t Rt[t][c],   S <- A S - sum_t L[t][r] wS_t Rt[t][c]
// (W, S global [R][C]; each thread reads and writes only its own elements).
template <int R, int C>
__device__ void update_state(float *W, float *S, const float *L, int ldl, const float *Rt, int ldr,
                             const float *wW, const float *wS, const float *fin, int b, int tid) {
  constexpr int GROUPS = THREADS / C, RPG = R / GROUPS;
  const int c = tid % C, g = tid / C;
  const float lam = fin[0], cc = fin[1], aa = fin[2];
  float rw[MAXB], rs[MAXB];
#pragma unroll
  for (int t = 0; t < MAXB; ++t) {
    const float v = t < b ? Rt[t * ldr + c] : 0.f;
    rw[t] = v * wW[t];
    rs[t] = v * wS[t];
  }
  static_assert(RPG % ROW_BLOCK == 0, "rows per thread group must fill whole blocks");
  for (int i0 = 0; i0 < RPG; i0 += ROW_BLOCK) {
    float wv[ROW_BLOCK], sv[ROW_BLOCK];
#pragma unroll
    for (int u = 0; u < ROW_BLOCK; ++u) {
      const size_t e = (size_t)(g * RPG + i0 + u) * C + c;
      wv[u] = W[e];
      sv[u] = S[e];
    }
    const int r0 = g * RPG + i0;
    float gw[ROW_BLOCK], gs[ROW_BLOCK];
#pragma unroll
    for (int u = 0; u < ROW_BLOCK; ++u) gw[u] = gs[u] = 0.f;
#pragma unroll
    for (int t = 0; t < MAXB; ++t)
      if (t < b) {
        const float4 l0 = ld4(L + t * ldl + r0), l1 = ld4(L + t * ldl + r0 + 4);
        const float l[ROW_BLOCK] = {l0.x, l0.y, l0.z, l0.w, l1.x, l1.y, l1.z, l1.w};
#pragma unroll
        for (int u = 0; u < ROW_BLOCK; ++u) {
          gw[u] = fmaf(l[u], rw[t], gw[u]);
          gs[u] = fmaf(l[u], rs[t], gs[u]);
        }
      }
#pragma unroll
    for (int u = 0; u < ROW_BLOCK; ++u) {
      const size_t e = (size_t)(r0 + u) * C + c;
      W[e] = lam * wv[u] + cc * sv[u] - gw[u];
      S[e] = aa * sv[u] - gs[u];
    }
  }
}

template <typename InT>
__global__ void __launch_bounds__(THREADS, 1) mlp_momentum_fwd_kernel(const Params p) {
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
  float *W1 = p.W1 + unit * (long)D * HID, *S1 = p.S1 + unit * (long)D * HID;
  float *W2 = p.W2 + unit * (long)HID * D, *S2 = p.S2 + unit * (long)HID * D;

  for (int x = tid; x < (int)(sizeof(Smem) / 4); x += THREADS) reinterpret_cast<float *>(smem_raw)[x] = 0.f;
  if (tid < D) {
    s.gam[tid] = p.gamma[head * D + tid];
    s.bet[tid] = p.beta[head * D + tid];
  }
  for (int x = tid; x < D * HID; x += THREADS) {
    W1[x] = p.W1_0[(long)head * D * HID + x];
    W2[x] = p.W2_0[(long)head * HID * D + x];
    S1[x] = 0.f;
    S2[x] = 0.f;
  }
  __syncthreads();

  for (int n = 0; n < N; ++n) {
    const long row0 = (long)n * b;
    load_rows(s.Q, Qg, row0, b, tid);
    load_rows(s.K, Kg, row0, b, tid);
    load_rows(s.V, Vg, row0, b, tid);
    if (tid < b) {
      s.eta[tid] = p.eta[tok0 + row0 + tid];
      s.alpha[tid] = p.alpha[tok0 + row0 + tid];
      s.keep[tid] = 1.f - p.lambda[tok0 + row0 + tid];
    }
    __syncthreads();
    // Coefficients: column s of c and a (thread s), and Lam_t, C_t (thread 32).
    if (tid < b) {
      const int sc = tid;
      float a = 1.f, c = 1.f;
      for (int t = 0; t < b; ++t) {
        if (t > sc) {
          a *= s.alpha[t];
          c = s.keep[t] * c + a;
        }
        s.cS[t * LDB + sc] = t >= sc ? a : 0.f;
        s.cW[t * LDB + sc] = t >= sc ? c : 0.f;
      }
      s.wS[sc] = a * s.eta[sc];
      s.wW[sc] = c * s.eta[sc];
    } else if (tid == 32) {
      float lam = 1.f, A = 1.f, C = 0.f;
      for (int t = 0; t < b; ++t) {
        lam *= s.keep[t];
        A *= s.alpha[t];
        C = s.keep[t] * C + A;
        s.lam[t] = lam;
        s.cb[t] = C;
      }
      s.fin[0] = lam;
      s.fin[1] = C;
      s.fin[2] = A;
    }
    // Gradients at the base.
    mm_W<HID>(s.X1, LDH, s.K, LDD, W1, D, b, 1.f, false, tid);  // X1 = K W1_b
    __syncthreads();
    for (int x = tid; x < b * HID; x += THREADS) s.X2[(x / HID) * LDH + x % HID] = gelu(s.X1[(x / HID) * LDH + x % HID]);
    __syncthreads();
    mm_W<D>(s.X3, LDD, s.X2, LDH, W2, HID, b, 1.f, false, tid);  // X3 = X2 W2_b
    __syncthreads();
    if (warp < b) {  // G3: the LN loss gradient of token `warp`
      const int t = warp, c0 = 2 * lane;
      const float x0 = s.X3[t * LDD + c0], x1 = s.X3[t * LDD + c0 + 1];
      const float mean = wsum(x0 + x1) * (1.f / D);
      const float d0 = x0 - mean, d1 = x1 - mean;
      const float rs = rsqrtf(wsum(d0 * d0 + d1 * d1) * (1.f / D) + p.eps);
      const float h0 = d0 * rs, h1 = d1 * rs;
      const float gx0 = 2.f * s.gam[c0] * (s.K[t * LDD + c0] + s.gam[c0] * h0 + s.bet[c0] - s.V[t * LDD + c0]);
      const float gx1 = 2.f * s.gam[c0 + 1] *
                        (s.K[t * LDD + c0 + 1] + s.gam[c0 + 1] * h1 + s.bet[c0 + 1] - s.V[t * LDD + c0 + 1]);
      const float m1 = wsum(gx0 + gx1) * (1.f / D), m2 = wsum(gx0 * h0 + gx1 * h1) * (1.f / D);
      s.G3[t * LDD + c0] = rs * (gx0 - m1 - h0 * m2);
      s.G3[t * LDD + c0 + 1] = rs * (gx1 - m1 - h1 * m2);
    }
    __syncthreads();
    mm_WT<HID>(s.G2, LDH, s.G3, LDD, W2, D, b, 1.f, false, tid);  // G3 W2_b^T
    gram_tril(s.A1, s.Q, LDD, s.K, LDD, D, b, tid);                // tril(Q K^T)
    __syncthreads();
    for (int x = tid; x < b * HID; x += THREADS) {
      const int t = x / HID, j = x % HID;
      s.G2[t * LDH + j] *= gelu_d(s.X1[t * LDH + j]);  // G2
    }
    if (tid < b * b) {  // (c o tril(Q K^T)) diag(eta)
      const int t = tid / b, sc = tid % b;
      s.A1[t * LDB + sc] *= s.cW[t * LDB + sc] * s.eta[sc];
    }
    __syncthreads();
    // Outputs.
    mm_two<HID>(s.Z1, LDH, s.Q, LDD, W1, S1, s.lam, s.cb, D, b, tid);
    small_corr<HID>(s.Z1, LDH, s.A1, false, s.G2, LDH, b, -1.f, tid);
    __syncthreads();
    for (int x = tid; x < b * HID; x += THREADS) s.Z2[(x / HID) * LDH + x % HID] = gelu(s.Z1[(x / HID) * LDH + x % HID]);
    __syncthreads();
    gram_tril(s.A2, s.Z2, LDH, s.X2, LDH, HID, b, tid);  // tril(Zq2 X2^T)
    __syncthreads();
    if (tid < b * b) {
      const int t = tid / b, sc = tid % b;
      s.A2[t * LDB + sc] *= s.cW[t * LDB + sc] * s.eta[sc];
    }
    __syncthreads();
    mm_two<D>(s.Z3, LDD, s.Z2, LDH, W2, S2, s.lam, s.cb, HID, b, tid);
    small_corr<D>(s.Z3, LDD, s.A2, false, s.G3, LDD, b, -1.f, tid);
    __syncthreads();
    if (warp < b) {  // Z = Q + LN(Zq3)
      const int t = warp, c0 = 2 * lane;
      const float z0 = s.Z3[t * LDD + c0], z1 = s.Z3[t * LDD + c0 + 1];
      const float mean = wsum(z0 + z1) * (1.f / D);
      const float e0 = z0 - mean, e1 = z1 - mean;
      const float rz = rsqrtf(wsum(e0 * e0 + e1 * e1) * (1.f / D) + p.eps);
      float *zr = p.Z + (tok0 + row0 + t) * D + c0;
      zr[0] = s.Q[t * LDD + c0] + s.gam[c0] * e0 * rz + s.bet[c0];
      zr[1] = s.Q[t * LDD + c0 + 1] + s.gam[c0 + 1] * e1 * rz + s.bet[c0 + 1];
    }
    // The next base: every read of the state above is complete after this barrier.
    __syncthreads();
    update_state<D, HID>(W1, S1, s.K, LDD, s.G2, LDH, s.wW, s.wS, s.fin, b, tid);
    update_state<HID, D>(W2, S2, s.X2, LDH, s.G3, LDD, s.wW, s.wS, s.fin, b, tid);
    __syncthreads();
  }
}

}  // namespace mommlp
}  // namespace ttt
