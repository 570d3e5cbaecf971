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

// TTT-MLP: b <= 16 rows per mini-batch, padded to MBR = 16 (padded rows are
// zero and carry eta = 0, so they touch neither the state nor any output).
// Row tiles that are contracted over their columns are kept transposed,
// [column][16 rows] (`t` suffix), so that one 16-byte shared load serves four
// rows and every product runs as f32x2 FMAs over row pairs; hidden-width tiles
// get a padded stride (20 floats) so that a thread's rows of one column are
// written without bank conflicts.  512 threads: in the [.][HID] passes thread
// (i, rh) owns hidden unit i and rows 8 rh .. 8 rh + 7; in the [.][D] passes
// thread (j, e) owns column j and hidden eighth e.
constexpr int MBR = 16;
constexpr int HT_LD = 20;
constexpr int DT_LD = 20;  // padded stride of the [D][16] transposed tiles
constexpr int MLP_THREADS = 512;

struct MlpSmem {
  float W1[D * HID];          // [D][HID] state
  float W2[HID * W2_LD];      // [HID][W2_LD] state
  float Qt[D * DT_LD], Kt[D * DT_LD];
  float V[MBR * D];           // [16][D]
  float X2t[HID * HT_LD];     // GELU(K W1), [HID][16]
  float Z2t[HID * HT_LD];     // GELU(Z1), [HID][16]
  float G3[MBR * D];          // X2 W2, then dl/d(X2 W2), [16][D]
  float G3t[D * DT_LD];       // G3 transposed
  union {
    float part[4 * MBR * D];  // partial sums over hidden parts
    float G2t[HID * HT_LD];   // dl/dX1, [HID][16] (between the X3 and A2 passes)
  };
  float A[MBR * MBR], A2[MBR * MBR];
  float eta[MBR];
};

inline size_t mlp_smem_bytes(int) { return sizeof(MlpSmem) + 16; }

__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

// Rows 8 h .. 8 h + 7 (h = 0, 1) or all 16 rows of column c of a transposed
// tile, as row pairs.
template <int N>
__device__ __forceinline__ void load_rows(const float *t, float2 (&v)[N]) {
  const float4 *q = reinterpret_cast<const float4 *>(t);
#pragma unroll
  for (int k = 0; k < N / 2; ++k) {
    const float4 x = q[k];
    v[2 * k] = make_float2(x.x, x.y);
    v[2 * k + 1] = make_float2(x.z, x.w);
  }
}
template <int N>
__device__ __forceinline__ void store_rows(float *t, const float2 (&v)[N]) {
  float4 *q = reinterpret_cast<float4 *>(t);
#pragma unroll
  for (int k = 0; k < N / 2; ++k) q[k] = make_float4(v[2 * k].x, v[2 * k].y, v[2 * k + 1].x, v[2 * k + 1].y);
}

template <typename InT>
__global__ void __launch_bounds__(MLP_THREADS) mlp_kernel(const Params p) {
  extern __shared__ __align__(16) float smem_f[];
  MlpSmem &S = *reinterpret_cast<MlpSmem *>(smem_f);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long unit = blockIdx.x;
  const int head = (int)(unit % p.H);
  const int b = p.b;  // <= 16

  {
    const float *w1 = p.W0 + (long)head * D * HID;
    const float *w2 = p.W2_0 + (long)head * HID * D;
    for (int x = tid; x < D * HID; x += MLP_THREADS) S.W1[x] = w1[x];
    for (int x = tid; x < HID * D; x += MLP_THREADS) S.W2[(x / D) * W2_LD + x % D] = w2[x];
  }
  const float gam0 = p.gamma[head * D + lane], gam1 = p.gamma[head * D + lane + 32];
  const float bet0 = p.beta[head * D + lane], bet1 = p.beta[head * D + lane + 32];
  const long tok0 = unit * (long)p.T;
  const InT *Qg = (const InT *)p.Q + tok0 * D;
  const InT *Kg = (const InT *)p.K + tok0 * D;
  const InT *Vg = (const InT *)p.V + tok0 * D;
  float *Zg = p.Z + tok0 * D;
  const int nmb = p.T / b;
  const int i = tid & (HID - 1), rh = tid >> 8;  // hidden unit, row half
  const int r0 = 8 * rh;
  const int j = tid & (D - 1), e = tid >> 6;     // column, hidden eighth
  const int ilo = HID / 8 * e, ihi = ilo + HID / 8;

  for (int n = 0; n < nmb; ++n) {
    __syncthreads();
    const long off = (long)n * b * D;
    for (int x = tid; x < MBR * D; x += MLP_THREADS) {
      const int r = x / D, c = x % D;
      const bool in = r < b;
      S.Qt[c * DT_LD + r] = in ? load_in(Qg, off + r * D + c) : 0.f;
      S.Kt[c * DT_LD + r] = in ? load_in(Kg, off + r * D + c) : 0.f;
      S.V[x] = in ? load_in(Vg, off + x) : 0.f;
    }
    if (tid < MBR) S.eta[tid] = tid < b ? p.eta[tok0 + (long)n * b + tid] : 0.f;
    __syncthreads();

    // X1 = K W1 and Z1 = Q W1: column i, this thread's 8 rows.
    float2 x1[4], zq[4];
    {
#pragma unroll
      for (int k = 0; k < 4; ++k) x1[k] = zq[k] = make_float2(0.f, 0.f);
#pragma unroll 8
      for (int pp = 0; pp < D; ++pp) {
        const float w = S.W1[pp * HID + i];
        const float2 ww = make_float2(w, w);
        float2 kv[4], qv[4];
        load_rows(&S.Kt[pp * DT_LD + r0], kv);
        load_rows(&S.Qt[pp * DT_LD + r0], qv);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          x1[k] = ffma2(kv[k], ww, x1[k]);
          zq[k] = ffma2(qv[k], ww, zq[k]);
        }
      }
      float2 x2[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) x2[k] = make_float2(gelu(x1[k].x), gelu(x1[k].y));
      store_rows(&S.X2t[i * HT_LD + r0], x2);
    }
    // A = tril(Q K^T) diag(eta), one entry per thread of the first 256.
    if (tid < MBR * MBR) {
      const int t = tid >> 4, s0 = tid & 15;
      float acc = 0.f;
      if (s0 <= t) {
#pragma unroll 8
        for (int pp = 0; pp < D; ++pp) acc = fmaf(S.Qt[pp * DT_LD + t], S.Kt[pp * DT_LD + s0], acc);
        acc *= S.eta[s0];
      }
      S.A[tid] = acc;
    }
    __syncthreads();

    // X3 = X2 W2: partial sums over hidden eighth e for column j, all 16 rows;
    // eighths 2q and 2q+1 meet in part[q].
    auto hidden_product = [&](const float *Xt) {
      float2 acc[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) acc[k] = make_float2(0.f, 0.f);
#pragma unroll 4
      for (int ii = ilo; ii < ihi; ++ii) {
        const float w = S.W2[ii * W2_LD + j];
        const float2 ww = make_float2(w, w);
        float2 xv[8];
        load_rows(&Xt[ii * HT_LD], xv);
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] = ffma2(xv[k], ww, acc[k]);
      }
      // Two passes through part[]: odd eighths add onto what even eighths wrote.
      float *dst = &S.part[(e >> 1) * MBR * D + j];
      if ((e & 1) == 0) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          dst[(2 * k) * D] = acc[k].x;
          dst[(2 * k + 1) * D] = acc[k].y;
        }
      }
      __syncthreads();
      if (e & 1) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          dst[(2 * k) * D] += acc[k].x;
          dst[(2 * k + 1) * D] += acc[k].y;
        }
      }
      __syncthreads();
    };
    hidden_product(S.X2t);
    for (int x = tid; x < MBR * D; x += MLP_THREADS)
      S.G3[x] = (S.part[x] + S.part[MBR * D + x]) + (S.part[2 * MBR * D + x] + S.part[3 * MBR * D + x]);
    __syncthreads();
    // G3 = dl / d X3 through LN and the residual (a warp per row).
    {
      const int r = warp;
      float dy0, dy1;
      ln_residual_grad(S.G3[r * D + lane], S.G3[r * D + lane + 32], S.Kt[lane * DT_LD + r],
                       S.Kt[(lane + 32) * DT_LD + r], S.V[r * D + lane], S.V[r * D + lane + 32], gam0,
                       gam1, bet0, bet1, p.eps, dy0, dy1);
      S.G3[r * D + lane] = dy0;
      S.G3[r * D + lane + 32] = dy1;
      S.G3t[lane * DT_LD + r] = dy0;
      S.G3t[(lane + 32) * DT_LD + r] = dy1;
    }
    __syncthreads();

    // G2 = (G3 W2^T) * GELU'(X1): column i, this thread's 8 rows.
    {
      float2 g2[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) g2[k] = make_float2(0.f, 0.f);
#pragma unroll 8
      for (int jj = 0; jj < D; ++jj) {
        const float w = S.W2[i * W2_LD + jj];
        const float2 ww = make_float2(w, w);
        float2 gv[4];
        load_rows(&S.G3t[jj * DT_LD + r0], gv);
#pragma unroll
        for (int k = 0; k < 4; ++k) g2[k] = ffma2(gv[k], ww, g2[k]);
      }
#pragma unroll
      for (int k = 0; k < 4; ++k)
        g2[k] = make_float2(g2[k].x * gelu_deriv(x1[k].x), g2[k].y * gelu_deriv(x1[k].y));
      store_rows(&S.G2t[i * HT_LD + r0], g2);
    }
    __syncthreads();
    // Z1 = Q W1 - A G2 and Z2 = GELU(Z1): column i, this thread's 8 rows.
    {
      float g2s[MBR];
      {
        float2 gv[8];
        load_rows(&S.G2t[i * HT_LD], gv);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          g2s[2 * k] = gv[k].x;
          g2s[2 * k + 1] = gv[k].y;
        }
      }
      float2 z2[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float za = zq[k].x, zb = zq[k].y;
        const int t0 = r0 + 2 * k, t1 = t0 + 1;
#pragma unroll
        for (int s0 = 0; s0 < MBR; ++s0) {
          if (s0 <= t0) za = fmaf(-S.A[t0 * MBR + s0], g2s[s0], za);
          if (s0 <= t1) zb = fmaf(-S.A[t1 * MBR + s0], g2s[s0], zb);
        }
        z2[k] = make_float2(gelu(za), gelu(zb));
      }
      store_rows(&S.Z2t[i * HT_LD + r0], z2);
    }
    {
      // W1[pp][i] -= sum_t K[t][pp] eta_t G2[t][i], pp in this thread's half.
      float2 g[8];
      {
        float2 gv[8];
        load_rows(&S.G2t[i * HT_LD], gv);
#pragma unroll
        for (int k = 0; k < 8; ++k) g[k] = make_float2(S.eta[2 * k] * gv[k].x, S.eta[2 * k + 1] * gv[k].y);
      }
#pragma unroll 4
      for (int pp = D / 2 * rh; pp < D / 2 * (rh + 1); ++pp) {
        float2 kv[8];
        load_rows(&S.Kt[pp * DT_LD], kv);
        float2 acc = make_float2(0.f, 0.f);
#pragma unroll
        for (int k = 0; k < 8; ++k) acc = ffma2(kv[k], g[k], acc);
        S.W1[pp * HID + i] -= acc.x + acc.y;
      }
    }
    __syncthreads();

    // A2 = tril(Z2 X2^T) diag(eta): entry (t, 4 s4 .. 4 s4 + 3), hidden eighth q.
    {
      const int q = tid >> 6, t = (tid >> 2) & 15, s4 = tid & 3;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      if (4 * s4 <= t) {
#pragma unroll 4
        for (int ii = HID / 8 * q; ii < HID / 8 * (q + 1); ++ii) {
          const float z = S.Z2t[ii * HT_LD + t];
          const float4 x = *reinterpret_cast<const float4 *>(&S.X2t[ii * HT_LD + 4 * s4]);
          acc.x = fmaf(z, x.x, acc.x);
          acc.y = fmaf(z, x.y, acc.y);
          acc.z = fmaf(z, x.z, acc.z);
          acc.w = fmaf(z, x.w, acc.w);
        }
      }
      *reinterpret_cast<float4 *>(&S.part[(q * MBR + t) * MBR + 4 * s4]) = acc;
    }
    __syncthreads();
    if (tid < MBR * MBR) {
      const int t = tid >> 4, s0 = tid & 15;
      float a = 0.f;
#pragma unroll
      for (int q = 0; q < 8; ++q) a += S.part[q * MBR * MBR + tid];
      S.A2[tid] = s0 <= t ? a * S.eta[s0] : 0.f;
    }
    __syncthreads();

    // Z3 = Z2 W2 - A2 G3.
    hidden_product(S.Z2t);
    // Output Z = Q + LN(Z3) (a warp per row).
    {
      const int r = warp;
      if (r < b) {
        float y[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int x = r * D + lane + 32 * h;
          float acc = (S.part[x] + S.part[MBR * D + x]) + (S.part[2 * MBR * D + x] + S.part[3 * MBR * D + x]);
          for (int s0 = 0; s0 <= r; ++s0) acc = fmaf(-S.A2[r * MBR + s0], S.G3[s0 * D + lane + 32 * h], acc);
          y[h] = acc;
        }
        float z0, z1;
        ln_residual_fwd(y[0], y[1], S.Qt[lane * DT_LD + r], S.Qt[(lane + 32) * DT_LD + r], gam0, gam1, bet0,
                        bet1, p.eps, z0, z1);
        Zg[off + r * D + lane] = z0;
        Zg[off + r * D + lane + 32] = z1;
      }
    }
    // W2 update (no product of this mini-batch reads W2 any more).
    {
      float2 g[8];
      // W2[ii][j] -= sum_t X2[t][ii] eta_t G3[t][j], ii in hidden eighth e.
#pragma unroll
      for (int k = 0; k < 8; ++k)
        g[k] = make_float2(S.eta[2 * k] * S.G3[(2 * k) * D + j], S.eta[2 * k + 1] * S.G3[(2 * k + 1) * D + j]);
#pragma unroll 4
      for (int ii = ilo; ii < ihi; ++ii) {
        float2 xv[8];
        load_rows(&S.X2t[ii * HT_LD], xv);
        float2 acc = make_float2(0.f, 0.f);
#pragma unroll
        for (int k = 0; k < 8; ++k) acc = ffma2(xv[k], g[k], acc);
        S.W2[ii * W2_LD + j] -= acc.x + acc.y;
      }
    }
  }
  __syncthreads();
  float *w1o = p.W_out + unit * D * HID;
  float *w2o = p.W2_out + unit * HID * D;
  for (int x = tid; x < D * HID; x += MLP_THREADS) w1o[x] = S.W1[x];
  for (int x = tid; x < HID * D; x += MLP_THREADS) w2o[x] = S.W2[(x / D) * W2_LD + x % D];
}

}  // namespace simt
}  // namespace ttt
