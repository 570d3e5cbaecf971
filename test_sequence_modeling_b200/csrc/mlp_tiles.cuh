// mlp_tiles.cuh - fp32 CUDA-core building blocks of the TTT-MLP kernels that
// keep one mini-batch's [b x hidden] and [b x d] tiles in shared memory and
// stream the [d x hidden] matrices (state, cotangents, momenta) from global
// memory: products of a tile with such a matrix (coalesced matrix loads,
// warp-wide broadcast tile reads), rank-b updates of a matrix, masked b x b
// Grams and their products, for a CTA of 16 warps and b <= 16.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace ttt {
namespace mlptile {

constexpr int D = 64;
constexpr int HID = 256;
constexpr int MAXB = 16;     // largest mini-batch of this kernel
constexpr int THREADS = 512;
constexpr int LDD = D + 4;   // row stride of the [b][d] tiles (16-byte aligned rows)
constexpr int LDH = HID + 4; // row stride of the [b][hidden] tiles
constexpr int LDB = MAXB + 1;

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

// Four consecutive floats of a tile: every tile row (LDD, LDH floats) and every
// tile base is 16-byte aligned, and the callers index in steps of 4.
__device__ __forceinline__ float4 ld4(const float *p) { return *reinterpret_cast<const float4 *>(p); }

__device__ __forceinline__ float wsum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ float phi(float x) { return 0.398942280401432678f * expf(-0.5f * x * x); }
__device__ __forceinline__ float gelu(float x) { return x * normcdff(x); }
__device__ __forceinline__ float gelu_d(float x) { return normcdff(x) + x * phi(x); }

// out[t][j] (+/-)= sum_k A[t][k] W[k][j]   (W global, row-major [Kd][N], written
// earlier in this kernel or by the caller: plain loads, not the read-only path).
template <int N>
__device__ void mm_W(float *out, int ldo, const float *A, int lda, const float *W, int Kd, int b,
                     float sign, bool acc, int tid) {
  constexpr int TPC = THREADS / N, RPT = MAXB / TPC;
  const int j = tid % N, g = tid / N;
  float a[RPT];
#pragma unroll
  for (int r = 0; r < RPT; ++r) a[r] = 0.f;
#pragma unroll 2
  for (int k = 0; k < Kd; k += 4) {
    const float w0 = W[(size_t)k * N + j], w1 = W[(size_t)(k + 1) * N + j];
    const float w2 = W[(size_t)(k + 2) * N + j], w3 = W[(size_t)(k + 3) * N + j];
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
      const float4 x = ld4(A + (g * RPT + r) * lda + k);
      a[r] = fmaf(x.w, w3, fmaf(x.z, w2, fmaf(x.y, w1, fmaf(x.x, w0, a[r]))));
    }
  }
#pragma unroll
  for (int r = 0; r < RPT; ++r) {
    const int t = g * RPT + r;
    if (t < b) out[t * ldo + j] = (acc ? out[t * ldo + j] : 0.f) + sign * a[r];
  }
}

// out[t][j] (+/-)= sum_k A[t][k] W[j][k]   (W global, row-major [N][Kd]).
template <int N>
__device__ void mm_WT(float *out, int ldo, const float *A, int lda, const float *W, int Kd, int b,
                      float sign, bool acc, int tid) {
  constexpr int TPC = THREADS / N, RPT = MAXB / TPC;
  const int j = tid % N, g = tid / N;
  float a[RPT];
#pragma unroll
  for (int r = 0; r < RPT; ++r) a[r] = 0.f;
  const float4 *wr = reinterpret_cast<const float4 *>(W + (size_t)j * Kd);
#pragma unroll 4
  for (int k = 0; k < Kd; k += 4) {
    const float4 w = wr[k >> 2];
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
      const float4 x = *reinterpret_cast<const float4 *>(A + (g * RPT + r) * lda + k);
      a[r] = fmaf(x.x, w.x, fmaf(x.y, w.y, fmaf(x.z, w.z, fmaf(x.w, w.w, a[r]))));
    }
  }
#pragma unroll
  for (int r = 0; r < RPT; ++r) {
    const int t = g * RPT + r;
    if (t < b) out[t * ldo + j] = (acc ? out[t * ldo + j] : 0.f) + sign * a[r];
  }
}

// out[t][j] += sign sum_{s<b} S[t][s] B[s][j]  (or S[s][t] when trans); the same
// (t, j) ownership as mm_W / mm_WT with this N, so it may follow them without a
// barrier.
template <int N>
__device__ void small_corr(float *out, int ldo, const float *S, bool trans, const float *B, int ldb,
                           int b, float sign, int tid) {
  constexpr int TPC = THREADS / N, RPT = MAXB / TPC;
  const int j = tid % N, g = tid / N;
#pragma unroll
  for (int r = 0; r < RPT; ++r) {
    const int t = g * RPT + r;
    if (t >= b) continue;
    float v = 0.f;
    for (int s = 0; s < b; ++s) v = fmaf(trans ? S[s * LDB + t] : S[t * LDB + s], B[s * ldb + j], v);
    out[t * ldo + j] += sign * v;
  }
}

// Rows per block of the element-wise state passes: every load of a block is
// issued before its stores, which the compiler cannot otherwise move a load past
// (the destination may be the source, or another buffer it cannot tell apart).
constexpr int ROW_BLOCK = 8;

// dst[r][c] = src[r][c] + sign sum_{t<b} L[t][r] Rt[t][c]   (dst, src global [R][C];
// dst may be src: each thread reads and writes only its own entries).
template <int R, int C>
__device__ void outer(float *dst, const float *src, const float *L, int ldl, const float *Rt, int ldr,
                      int b, float sign, int tid) {
  constexpr int GROUPS = THREADS / C, RPG = R / GROUPS;
  static_assert(RPG % ROW_BLOCK == 0 && ROW_BLOCK == 8, "rows per thread group must fill whole 8-row blocks");
  const int c = tid % C, g = tid / C;
  float rt[MAXB];
#pragma unroll
  for (int t = 0; t < MAXB; ++t) rt[t] = t < b ? Rt[t * ldr + c] : 0.f;
  for (int i0 = 0; i0 < RPG; i0 += ROW_BLOCK) {
    const int r0 = g * RPG + i0;
    float sv[ROW_BLOCK], a[ROW_BLOCK];
#pragma unroll
    for (int u = 0; u < ROW_BLOCK; ++u) {
      sv[u] = src[(size_t)(r0 + u) * C + c];
      a[u] = 0.f;
    }
    // L[t][r0 .. r0 + 7]: two 16-byte loads per token (warp-wide broadcasts).
#pragma unroll
    for (int t = 0; t < MAXB; ++t)
      if (t < b) {
        const float4 l0 = ld4(L + t * ldl + r0), l1 = ld4(L + t * ldl + r0 + 4);
        const float x = rt[t];
        a[0] = fmaf(l0.x, x, a[0]);
        a[1] = fmaf(l0.y, x, a[1]);
        a[2] = fmaf(l0.z, x, a[2]);
        a[3] = fmaf(l0.w, x, a[3]);
        a[4] = fmaf(l1.x, x, a[4]);
        a[5] = fmaf(l1.y, x, a[5]);
        a[6] = fmaf(l1.z, x, a[6]);
        a[7] = fmaf(l1.w, x, a[7]);
      }
#pragma unroll
    for (int u = 0; u < ROW_BLOCK; ++u) dst[(size_t)(r0 + u) * C + c] = sv[u] + sign * a[u];
  }
}

// S[t][s] = sum_k A[t][k] B[s][k] for s <= t < b (zero elsewhere).
__device__ void gram_tril(float *S, const float *A, int lda, const float *B, int ldb, int Kd, int b,
                          int tid) {
  const int p = tid >> 1, hf = tid & 1;
  const int t = p >> 4, s = p & 15;
  float v = 0.f;
  if (t < b && s <= t) {
    const int k0 = hf * (Kd / 2);
    for (int k = k0; k < k0 + Kd / 2; k += 4) {
      const float4 x = *reinterpret_cast<const float4 *>(A + t * lda + k);
      const float4 y = *reinterpret_cast<const float4 *>(B + s * ldb + k);
      v = fmaf(x.x, y.x, fmaf(x.y, y.y, fmaf(x.z, y.z, fmaf(x.w, y.w, v))));
    }
  }
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  if (hf == 0) S[t * LDB + s] = (t < b && s <= t) ? v : 0.f;
}

template <typename InT>
__device__ void load_rows(float *dst, const InT *src, long row0, int b, int tid) {
  for (int x = tid; x < b * D; x += THREADS) dst[(x / D) * LDD + x % D] = to_f(src[(row0 + x / D) * D + x % D]);
}

}  // namespace mlptile
}  // namespace ttt
