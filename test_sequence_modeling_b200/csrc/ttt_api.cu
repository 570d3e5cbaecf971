// ttt_api.cu - C ABI of the TTT layer forward: argument checks, kernel
// selection and launch.  Everything the ABI promises about errors is decided
// here on the host before any CUDA call.  The kernels live in the headers this
// file includes, so that the library is one translation unit and one device
// status word.
#include <atomic>
#include <cmath>
#include <cstdint>
#include <algorithm>
#include <mutex>
#include <vector>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "ttt.h"
#include "device_status.cuh"
#include "backward.cuh"
#include "backward_mlp.cuh"
#include "decode.cuh"
#include "momentum.cuh"
#include "momentum_mlp.cuh"
#include "simt.cuh"
#include "tc_linear.cuh"
#include "tc_momentum.cuh"
#include "tc_mlp.cuh"

namespace simt = ttt::simt;
namespace tc = ttt::tc;
namespace tcmlp = ttt::tcmlp;
namespace decode = ttt::decode;
namespace bwd = ttt::bwd;
namespace bwdmlp = ttt::bwdmlp;
namespace mom = ttt::mom;
namespace mommlp = ttt::mommlp;
namespace tcmom = ttt::tcmom;

namespace {

std::atomic<int> g_path{TTT_PATH_AUTO};
std::atomic<long long> g_launches{0};
std::atomic<int> g_inject_timeout{0};

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Range {
  uintptr_t lo, hi;
};
Range range_of(const void *p, size_t bytes) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(p);
  return {a, a + bytes};
}
bool overlap(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi; }

enum Kind { LINEAR = 0, LINEAR_LN = 1, MLP_LN = 2 };

struct Call {
  Kind kind;
  const void *Q, *K, *V;
  int qkv_dtype;
  const float *eta, *W0, *W2_0, *gamma, *beta;
  float eps;
  int B, H, T, d, hidden, b;
  float *Z, *W_out, *W2_out;
  void *stream;
};

// Host-side checks shared by every entry point.  Returns TTT_OK or the status
// to return without launching.
int validate(const Call &c) {
  if (c.qkv_dtype != TTT_F32 && c.qkv_dtype != TTT_BF16) return TTT_ERR_ARG;
  if (c.B < 0 || c.H < 0 || c.T < 0 || c.d <= 0 || c.b <= 0) return TTT_ERR_ARG;
  if (c.T % c.b != 0) return TTT_ERR_ARG;
  if (c.kind != LINEAR && !(std::isfinite(c.eps) && c.eps > 0.f)) return TTT_ERR_ARG;
  if (c.kind == MLP_LN && c.hidden <= 0) return TTT_ERR_ARG;
  if (c.d != simt::D) return TTT_ERR_UNSUPPORTED;
  if (c.kind == MLP_LN && c.hidden != simt::HID) return TTT_ERR_UNSUPPORTED;
  if (c.b > (c.kind == MLP_LN ? 16 : 64)) return TTT_ERR_UNSUPPORTED;
  const long long units = (long long)c.B * c.H;
  if (units == 0) return TTT_OK;
  if (units > 0x7fffffffLL) return TTT_ERR_UNSUPPORTED;
  const long long elems = units * c.T * c.d;
  if (elems >= (1LL << 40)) return TTT_ERR_UNSUPPORTED;

  // Pointers: required ones non-null and 16-byte aligned.
  const bool has_tokens = c.T > 0;
  const void *req[] = {c.W0, c.W_out, c.kind == MLP_LN ? (const void *)c.W2_0 : c.W0,
                       c.kind == MLP_LN ? (const void *)c.W2_out : c.W_out,
                       c.kind != LINEAR ? (const void *)c.gamma : c.W0,
                       c.kind != LINEAR ? (const void *)c.beta : c.W0};
  for (const void *p : req)
    if (!p) return TTT_ERR_ARG;
  if (has_tokens && (!c.Q || !c.K || !c.V || !c.eta || !c.Z)) return TTT_ERR_ARG;
  for (const void *p : req)
    if (!aligned16(p)) return TTT_ERR_ALIGN;
  if (has_tokens) {
    const void *tok[] = {c.Q, c.K, c.V, c.eta, c.Z};
    for (const void *p : tok)
      if (!aligned16(p)) return TTT_ERR_ALIGN;
  }

  // Outputs must not overlap inputs or each other.
  const size_t in_elt = c.qkv_dtype == TTT_BF16 ? 2 : 4;
  const size_t P1 = c.kind == MLP_LN ? (size_t)c.d * c.hidden : (size_t)c.d * c.d;
  Range ins[8];
  int nin = 0;
  if (has_tokens) {
    ins[nin++] = range_of(c.Q, (size_t)elems * in_elt);
    ins[nin++] = range_of(c.K, (size_t)elems * in_elt);
    ins[nin++] = range_of(c.V, (size_t)elems * in_elt);
    ins[nin++] = range_of(c.eta, (size_t)units * c.T * 4);
  }
  ins[nin++] = range_of(c.W0, (size_t)c.H * P1 * 4);
  if (c.kind == MLP_LN) ins[nin++] = range_of(c.W2_0, (size_t)c.H * P1 * 4);
  if (c.kind != LINEAR) {
    ins[nin++] = range_of(c.gamma, (size_t)c.H * c.d * 4);
    ins[nin++] = range_of(c.beta, (size_t)c.H * c.d * 4);
  }
  Range outs[3];
  int nout = 0;
  if (has_tokens) outs[nout++] = range_of(c.Z, (size_t)elems * 4);
  outs[nout++] = range_of(c.W_out, (size_t)units * P1 * 4);
  if (c.kind == MLP_LN) outs[nout++] = range_of(c.W2_out, (size_t)units * P1 * 4);
  for (int o = 0; o < nout; ++o) {
    for (int i = 0; i < nin; ++i)
      if (overlap(outs[o], ins[i])) return TTT_ERR_ARG;
    for (int o2 = o + 1; o2 < nout; ++o2)
      if (overlap(outs[o], outs[o2])) return TTT_ERR_ARG;
  }
  return TTT_OK;
}

// Launches the register-state kernel (b <= 16) in whichever register budget runs
// `grid` CTAs in fewer waves on this device: capped for 4 CTAs per SM (a few
// spills) or uncapped (2-3 CTAs per SM); a tie keeps the uncapped one.
template <bool LN, typename InT, bool MOMENTUM>
int launch_register_state(unsigned grid, cudaStream_t s, const mom::Params &p) {
  auto k1 = mom::momentum_fwd_kernel<LN, InT, MOMENTUM, 1>;
  auto k4 = mom::momentum_fwd_kernel<LN, InT, MOMENTUM, 4>;
  int dev = 0, sms = 0, occ1 = 0, occ4 = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ1, k1, mom::THREADS, 0) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ4, k4, mom::THREADS, 0) != cudaSuccess)
    return TTT_ERR_CUDA;
  auto waves = [&](int occ) {
    const long long slots = (long long)sms * occ;
    return slots > 0 ? ((long long)grid + slots - 1) / slots : (1LL << 62);
  };
  if (waves(occ4) < waves(occ1)) k4<<<grid, mom::THREADS, 0, s>>>(p);
  else k1<<<grid, mom::THREADS, 0, s>>>(p);
  if (cudaGetLastError() != cudaSuccess) return TTT_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return TTT_OK;
}

template <typename KernelT>
int launch(KernelT kernel, int grid, size_t smem, cudaStream_t stream,
           const simt::Params &p, int threads = simt::THREADS) {
  if (smem > 48 * 1024) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      return TTT_ERR_CUDA;
  }
  kernel<<<grid, threads, smem, stream>>>(p);
  if (cudaGetLastError() != cudaSuccess) return TTT_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return TTT_OK;
}

int run_simt(const Call &c) {
  simt::Params p;
  p.Q = c.Q;
  p.K = c.K;
  p.V = c.V;
  p.eta = c.eta;
  p.W0 = c.W0;
  p.W2_0 = c.W2_0;
  p.gamma = c.gamma;
  p.beta = c.beta;
  p.eps = c.eps;
  p.H = c.H;
  p.T = c.T;
  p.b = c.b;
  p.Z = c.Z;
  p.W_out = c.W_out;
  p.W2_out = c.W2_out;
  const int grid = c.B * c.H;
  cudaStream_t s = static_cast<cudaStream_t>(c.stream);
  const bool bf16 = c.qkv_dtype == TTT_BF16;
  if (c.kind == MLP_LN) {
    const size_t smem = simt::mlp_smem_bytes(c.b);
    return bf16 ? launch(simt::mlp_kernel<__nv_bfloat16>, grid, smem, s, p, simt::MLP_THREADS)
                : launch(simt::mlp_kernel<float>, grid, smem, s, p, simt::MLP_THREADS);
  }
  if (c.b <= mom::MAXB) {
    // b <= 16: the state stays in registers for the whole sequence (the plain
    // instantiation of the momentum kernel).
    mom::Params q{c.Q, c.K, c.V, c.eta, nullptr, nullptr, c.W0, c.gamma, c.beta, c.eps,
                  c.H, c.T, c.b, c.Z, c.W_out, nullptr};
    if (c.kind == LINEAR_LN)
      return bf16 ? launch_register_state<true, __nv_bfloat16, false>(grid, s, q)
                  : launch_register_state<true, float, false>(grid, s, q);
    return bf16 ? launch_register_state<false, __nv_bfloat16, false>(grid, s, q)
                : launch_register_state<false, float, false>(grid, s, q);
  }
  const size_t smem = simt::linear_smem_bytes(c.b);
  if (c.kind == LINEAR_LN)
    return bf16 ? launch(simt::linear_kernel<true, __nv_bfloat16>, grid, smem, s, p)
                : launch(simt::linear_kernel<true, float>, grid, smem, s, p);
  return bf16 ? launch(simt::linear_kernel<false, __nv_bfloat16>, grid, smem, s, p)
              : launch(simt::linear_kernel<false, float>, grid, smem, s, p);
}

// cuTensorMapEncodeTiled through the runtime's driver entry point, so that the
// library does not link against libcuda.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// [units][T][64] bf16 viewed as a 3-D tensor; boxes of `box_rows` tokens x 64
// features with the 128-byte swizzle.  Rows past T read as zeros.
bool make_qkv_map(CUtensorMap *map, const void *base, int T, long long units, int box_rows) {
  auto encode = tensor_map_encoder();
  if (!encode) return false;
  cuuint64_t dims[3] = {64, (cuuint64_t)T, (cuuint64_t)units};
  cuuint64_t strides[2] = {64 * 2, (cuuint64_t)T * 64 * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
                box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool tc_supported(const Call &c) {
  if (c.qkv_dtype != TTT_BF16 || c.T <= 0) return false;
  return c.kind == MLP_LN ? c.b == tcmlp::MB : c.b == tc::MB;
}

template <bool LN>
int launch_linear_tc(const Call &c) {
  const long long units = (long long)c.B * c.H;
  CUtensorMap mq, mk, mv;
  // Q and K arrive as 8-token boxes (the row groups of the [K;Q] operand), V as
  // one 64-token box per chunk.
  if (!make_qkv_map(&mq, c.Q, c.T, units, 8) || !make_qkv_map(&mk, c.K, c.T, units, 8) ||
      !make_qkv_map(&mv, c.V, c.T, units, tc::CHUNK))
    return TTT_ERR_CUDA;
  tc::Params p;
  p.eta = c.eta;
  p.W0 = c.W0;
  p.gamma = c.gamma;
  p.beta = c.beta;
  p.eps = c.eps;
  p.H = c.H;
  p.T = c.T;
  p.Z = c.Z;
  p.W_out = c.W_out;
  p.inject_timeout = g_inject_timeout.load();
  // Two register budgets: 4 CTAs per SM (128 registers) or 2 (the compiler's
  // choice, ~200).  The roomier one runs a CTA's chain faster (-6 to -8 % on
  // grids of 32 and 192 units) but holds half the CTAs per SM: it is taken
  // unless the capped one runs the grid in fewer waves.
  auto k4 = tc::linear_tc_kernel<LN, 4>;
  auto k2 = tc::linear_tc_kernel<LN, 2>;
  for (auto k : {k4, k2})
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tc::SMEM_BYTES) !=
            cudaSuccess ||
        cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared) != cudaSuccess)
      return TTT_ERR_CUDA;
  // CTAs per SM from registers, shared memory and TMEM (128 of 512 columns).  The
  // occupancy query is not used: it returns 1 for these kernels (their barrier
  // count, all 16 reserved by the pair barrier's computed id, misleads it),
  // while the SM runs 4 (2 for the roomier budget).
  int dev = 0, sms = 0, regs_sm = 0, smem_sm = 0, reserved = 0;
  cudaFuncAttributes a4, a2;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess ||
      cudaFuncGetAttributes(&a4, k4) != cudaSuccess || cudaFuncGetAttributes(&a2, k2) != cudaSuccess)
    return TTT_ERR_CUDA;
  auto per_sm = [&](const cudaFuncAttributes &a) {
    const long long regs = (long long)((a.numRegs + 7) / 8 * 8) * tc::THREADS;
    const long long smem = (long long)tc::SMEM_BYTES + reserved;
    long long n = 512 / tc::TMEM_COLS;
    if (regs > 0) n = std::min(n, (long long)regs_sm / regs);
    return (int)std::min(n, (long long)smem_sm / smem);
  };
  const int occ4 = per_sm(a4), occ2 = per_sm(a2);
  auto waves = [&](int occ) {
    const long long slots = (long long)sms * occ;
    return slots > 0 ? (units + slots - 1) / slots : (1LL << 62);
  };
  auto kernel = waves(occ4) < waves(occ2) ? k4 : k2;
  kernel<<<(unsigned)units, tc::THREADS, tc::SMEM_BYTES, static_cast<cudaStream_t>(c.stream)>>>(
      mq, mk, mv, p);
  if (cudaGetLastError() != cudaSuccess) return TTT_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return TTT_OK;
}

int launch_mlp_tc(const Call &c) {
  const long long units = (long long)c.B * c.H;
  CUtensorMap mq, mk, mv;
  if (!make_qkv_map(&mq, c.Q, c.T, units, tcmlp::CHUNK) ||
      !make_qkv_map(&mk, c.K, c.T, units, tcmlp::CHUNK) ||
      !make_qkv_map(&mv, c.V, c.T, units, tcmlp::CHUNK))
    return TTT_ERR_CUDA;
  tcmlp::Params p;
  p.eta = c.eta;
  p.W1_0 = c.W0;
  p.W2_0 = c.W2_0;
  p.gamma = c.gamma;
  p.beta = c.beta;
  p.eps = c.eps;
  p.H = c.H;
  p.T = c.T;
  p.Z = c.Z;
  p.W1_out = c.W_out;
  p.W2_out = c.W2_out;
  p.inject_timeout = g_inject_timeout.load();
  auto kernel = tcmlp::mlp_tc_kernel;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)tcmlp::SMEM_BYTES) != cudaSuccess)
    return TTT_ERR_CUDA;
  kernel<<<(unsigned)units, tcmlp::THREADS, tcmlp::SMEM_BYTES,
           static_cast<cudaStream_t>(c.stream)>>>(mq, mk, mv, p);
  if (cudaGetLastError() != cudaSuccess) return TTT_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return TTT_OK;
}

// One primal-form decode step (decode.cuh).  Checks on the host first, as the
// forward entry points do.
int run_decode(bool ln, const void *q, const void *k, const void *v, int qkv_dtype, const float *eta,
               float *W, float *W_base, const float *gamma, const float *beta, float eps, int B,
               int H, int d, int b, int pos, float *z, void *stream, bool momentum = false,
               const float *alpha = nullptr, const float *lambda = nullptr, float *S = nullptr) {
  if (qkv_dtype != TTT_F32 && qkv_dtype != TTT_BF16) return TTT_ERR_ARG;
  if (B < 0 || H < 0 || d <= 0 || b <= 0 || pos < 0 || pos >= b) return TTT_ERR_ARG;
  if (ln && !(std::isfinite(eps) && eps > 0.f)) return TTT_ERR_ARG;
  if (d != decode::D) return TTT_ERR_UNSUPPORTED;
  const long long units = (long long)B * H;
  if (units == 0) return TTT_OK;
  if (units > 0x7fffffffLL) return TTT_ERR_UNSUPPORTED;
  const void *req[] = {q, k, v, eta, W, W_base, z, ln ? (const void *)gamma : q,
                       ln ? (const void *)beta : q, momentum ? (const void *)alpha : q,
                       momentum ? (const void *)lambda : q, momentum ? (const void *)S : q};
  for (const void *x : req)
    if (!x) return TTT_ERR_ARG;
  for (const void *x : req)
    if (!aligned16(x)) return TTT_ERR_ALIGN;
  const size_t in_elt = qkv_dtype == TTT_BF16 ? 2 : 4;
  Range ins[8] = {range_of(q, units * d * in_elt), range_of(k, units * d * in_elt),
                  range_of(v, units * d * in_elt), range_of(eta, units * 4),
                  range_of(ln ? (const void *)gamma : q, ln ? (size_t)H * d * 4 : 0),
                  range_of(ln ? (const void *)beta : q, ln ? (size_t)H * d * 4 : 0),
                  range_of(momentum ? (const void *)alpha : q, momentum ? units * 4 : 0),
                  range_of(momentum ? (const void *)lambda : q, momentum ? units * 4 : 0)};
  Range outs[4] = {range_of(W, units * d * d * 4), range_of(W_base, units * d * d * 4),
                   range_of(z, units * d * 4),
                   range_of(momentum ? (const void *)S : z, momentum ? units * d * d * 4 : 0)};
  for (int o = 0; o < 4; ++o) {
    for (int i = 0; i < 8; ++i)
      if (overlap(outs[o], ins[i])) return TTT_ERR_ARG;
    for (int o2 = o + 1; o2 < 4; ++o2)
      if (overlap(outs[o], outs[o2])) return TTT_ERR_ARG;
  }
  decode::Params p{q, k, v, eta, W, W_base, gamma, beta, eps, H, pos, b, z, alpha, lambda, S};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool bf16 = qkv_dtype == TTT_BF16;
  const unsigned grid = (unsigned)units;
  if (momentum) {
    if (ln) {
      if (bf16) decode::decode_kernel<true, __nv_bfloat16, true><<<grid, decode::THREADS, 0, s>>>(p);
      else decode::decode_kernel<true, float, true><<<grid, decode::THREADS, 0, s>>>(p);
    } else {
      if (bf16) decode::decode_kernel<false, __nv_bfloat16, true><<<grid, decode::THREADS, 0, s>>>(p);
      else decode::decode_kernel<false, float, true><<<grid, decode::THREADS, 0, s>>>(p);
    }
  } else if (ln) {
    if (bf16) decode::decode_kernel<true, __nv_bfloat16><<<grid, decode::THREADS, 0, s>>>(p);
    else decode::decode_kernel<true, float><<<grid, decode::THREADS, 0, s>>>(p);
  } else {
    if (bf16) decode::decode_kernel<false, __nv_bfloat16><<<grid, decode::THREADS, 0, s>>>(p);
    else decode::decode_kernel<false, float><<<grid, decode::THREADS, 0, s>>>(p);
  }
  if (cudaGetLastError() != cudaSuccess) return TTT_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return TTT_OK;
}

// One primal-form decode step of TTT-MLP (decode.cuh), host checks first.
int run_mlp_decode(const void *q, const void *k, const void *v, int qkv_dtype, const float *eta,
                   float *W1, float *W2, float *W1_base, float *W2_base, const float *gamma,
                   const float *beta, float eps, int B, int H, int d, int hidden, int b, int pos,
                   float *z, void *stream, bool momentum = false, const float *alpha = nullptr,
                   const float *lambda = nullptr, float *S1 = nullptr, float *S2 = nullptr) {
  if (qkv_dtype != TTT_F32 && qkv_dtype != TTT_BF16) return TTT_ERR_ARG;
  if (B < 0 || H < 0 || d <= 0 || hidden <= 0 || b <= 0 || pos < 0 || pos >= b) return TTT_ERR_ARG;
  if (!(std::isfinite(eps) && eps > 0.f)) return TTT_ERR_ARG;
  if (d != decode::D || hidden != decode::HID) return TTT_ERR_UNSUPPORTED;
  const long long units = (long long)B * H;
  if (units == 0) return TTT_OK;
  if (units > 0x7fffffffLL) return TTT_ERR_UNSUPPORTED;
  const void *req[] = {q, k, v, eta, W1, W2, W1_base, W2_base, z, gamma, beta,
                       momentum ? (const void *)alpha : q, momentum ? (const void *)lambda : q,
                       momentum ? (const void *)S1 : q, momentum ? (const void *)S2 : q};
  for (const void *x : req)
    if (!x) return TTT_ERR_ARG;
  for (const void *x : req)
    if (!aligned16(x)) return TTT_ERR_ALIGN;
  const size_t in_elt = qkv_dtype == TTT_BF16 ? 2 : 4;
  const size_t wbytes = (size_t)units * d * hidden * 4;
  const size_t sbytes = momentum ? wbytes : 0, rbytes = momentum ? units * 4 : 0;
  Range ins[8] = {range_of(q, units * d * in_elt), range_of(k, units * d * in_elt),
                  range_of(v, units * d * in_elt), range_of(eta, units * 4),
                  range_of(gamma, (size_t)H * d * 4), range_of(beta, (size_t)H * d * 4),
                  range_of(momentum ? (const void *)alpha : q, rbytes),
                  range_of(momentum ? (const void *)lambda : q, rbytes)};
  Range outs[7] = {range_of(W1, wbytes), range_of(W2, wbytes), range_of(W1_base, wbytes),
                   range_of(W2_base, wbytes), range_of(z, units * d * 4),
                   range_of(momentum ? (const void *)S1 : z, sbytes),
                   range_of(momentum ? (const void *)S2 : z, sbytes)};
  for (int o = 0; o < 7; ++o) {
    for (int i = 0; i < 8; ++i)
      if (overlap(outs[o], ins[i])) return TTT_ERR_ARG;
    for (int o2 = o + 1; o2 < 7; ++o2)
      if (overlap(outs[o], outs[o2])) return TTT_ERR_ARG;
  }
  decode::MlpParams p{q, k, v, eta, W1, W2, W1_base, W2_base, gamma, beta, eps, H, pos, b, z,
                      alpha, lambda, S1, S2};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const unsigned grid = (unsigned)units;
  const bool bf16 = qkv_dtype == TTT_BF16;
  if (momentum) {
    if (bf16) decode::mlp_decode_kernel<__nv_bfloat16, true><<<grid, decode::MLP_THREADS, 0, s>>>(p);
    else decode::mlp_decode_kernel<float, true><<<grid, decode::MLP_THREADS, 0, s>>>(p);
  } else {
    if (bf16) decode::mlp_decode_kernel<__nv_bfloat16><<<grid, decode::MLP_THREADS, 0, s>>>(p);
    else decode::mlp_decode_kernel<float><<<grid, decode::MLP_THREADS, 0, s>>>(p);
  }
  if (cudaGetLastError() != cudaSuccess) return TTT_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return TTT_OK;
}

int run_bwd(bool ln, const void *Q, const void *K, const void *V, int qkv_dtype, const float *eta,
            const float *W0, const float *gamma, const float *beta, float eps, const float *dZ,
            const float *dW_T, int B, int H, int T, int d, int b, float *dQ, float *dK, float *dV,
            float *deta, float *dW0, float *dgamma, float *dbeta, float *W_ckpt, void *stream) {
  if (qkv_dtype != TTT_F32 && qkv_dtype != TTT_BF16) return TTT_ERR_ARG;
  if (B < 0 || H < 0 || T < 0 || d <= 0 || b <= 0) return TTT_ERR_ARG;
  if (T % b != 0) return TTT_ERR_ARG;
  if (ln && !(std::isfinite(eps) && eps > 0.f)) return TTT_ERR_ARG;
  if (d != bwd::D || b > bwd::MAXB) return TTT_ERR_UNSUPPORTED;
  const long long units = (long long)B * H;
  if (units == 0) return TTT_OK;
  if (units > 0x7fffffffLL) return TTT_ERR_UNSUPPORTED;
  const long long elems = units * T * d;
  if (elems >= (1LL << 40)) return TTT_ERR_UNSUPPORTED;
  const bool tok = T > 0;
  // Required pointers (a stand-in that passes the checks where one is not needed).
  const void *req[] = {W0, dW0, ln ? (const void *)gamma : W0, ln ? (const void *)beta : W0,
                       ln ? (const void *)dgamma : dW0, ln ? (const void *)dbeta : dW0,
                       tok ? Q : W0, tok ? K : W0, tok ? V : W0, tok ? (const void *)eta : W0,
                       tok ? (const void *)dZ : W0, tok ? (const void *)dQ : dW0,
                       tok ? (const void *)dK : dW0, tok ? (const void *)dV : dW0,
                       tok ? (const void *)deta : dW0, tok ? (const void *)W_ckpt : dW0};
  for (const void *x : req)
    if (!x) return TTT_ERR_ARG;
  for (const void *x : req)
    if (!aligned16(x)) return TTT_ERR_ALIGN;
  if (dW_T && !aligned16(dW_T)) return TTT_ERR_ALIGN;
  const size_t in_elt = qkv_dtype == TTT_BF16 ? 2 : 4;
  const size_t tbytes = tok ? (size_t)elems * 4 : 0, ibytes = tok ? (size_t)elems * in_elt : 0;
  const size_t ebytes = tok ? (size_t)units * T * 4 : 0, wbytes = (size_t)units * d * d * 4;
  const size_t vbytes = ln ? (size_t)units * d * 4 : 0, pbytes = ln ? (size_t)H * d * 4 : 0;
  const size_t cbytes = tok ? (size_t)units * (T / b) * d * d * 4 : 0;
  Range ins[9] = {range_of(Q, ibytes), range_of(K, ibytes), range_of(V, ibytes),
                  range_of(eta, ebytes), range_of(W0, (size_t)H * d * d * 4),
                  range_of(gamma, pbytes), range_of(beta, pbytes), range_of(dZ, tbytes),
                  range_of(dW_T, dW_T ? wbytes : 0)};
  Range outs[8] = {range_of(dQ, tbytes),   range_of(dK, tbytes),     range_of(dV, tbytes),
                   range_of(deta, ebytes), range_of(dW0, wbytes),    range_of(dgamma, vbytes),
                   range_of(dbeta, vbytes), range_of(W_ckpt, cbytes)};
  for (int o = 0; o < 8; ++o) {
    for (int i = 0; i < 9; ++i)
      if (overlap(outs[o], ins[i])) return TTT_ERR_ARG;
    for (int o2 = o + 1; o2 < 8; ++o2)
      if (overlap(outs[o], outs[o2])) return TTT_ERR_ARG;
  }
  bwd::Params p{Q, K, V, eta, W0, gamma, beta, eps, dZ, dW_T, H, T, b,
                dQ, dK, dV, deta, dW0, dgamma, dbeta, W_ckpt};
  auto kernel = ln ? (qkv_dtype == TTT_BF16 ? bwd::linear_bwd_kernel<true, __nv_bfloat16>
                                            : bwd::linear_bwd_kernel<true, float>)
                   : (qkv_dtype == TTT_BF16 ? bwd::linear_bwd_kernel<false, __nv_bfloat16>
                                            : bwd::linear_bwd_kernel<false, float>);
  const size_t smem = bwd::smem_bytes();
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return TTT_ERR_CUDA;
  kernel<<<(unsigned)units, bwd::THREADS, smem, static_cast<cudaStream_t>(stream)>>>(p);
  if (cudaGetLastError() != cudaSuccess) return TTT_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return TTT_OK;
}

int run_mlp_bwd(const void *Q, const void *K, const void *V, int qkv_dtype, const float *eta,
                const float *W1_0, const float *W2_0, const float *gamma, const float *beta, float eps,
                const float *dZ, const float *dW1_T, const float *dW2_T, int B, int H, int T, int d,
                int hidden, int b, float *dQ, float *dK, float *dV, float *deta, float *dW1,
                float *dW2, float *dgamma, float *dbeta, float *W1_ckpt, float *W2_ckpt,
                void *stream) {
  if (qkv_dtype != TTT_F32 && qkv_dtype != TTT_BF16) return TTT_ERR_ARG;
  if (B < 0 || H < 0 || T < 0 || d <= 0 || hidden <= 0 || b <= 0) return TTT_ERR_ARG;
  if (T % b != 0) return TTT_ERR_ARG;
  if (!(std::isfinite(eps) && eps > 0.f)) return TTT_ERR_ARG;
  if (d != bwdmlp::D || hidden != bwdmlp::HID || b > bwdmlp::MAXB) return TTT_ERR_UNSUPPORTED;
  const long long units = (long long)B * H;
  if (units == 0) return TTT_OK;
  if (units > 0x7fffffffLL) return TTT_ERR_UNSUPPORTED;
  const long long elems = units * T * d;
  if (elems >= (1LL << 40)) return TTT_ERR_UNSUPPORTED;
  const bool tok = T > 0;
  const void *req[] = {W1_0, W2_0, gamma, beta, dW1, dW2, dgamma, dbeta,
                       tok ? Q : W1_0, tok ? K : W1_0, tok ? V : W1_0, tok ? (const void *)eta : W1_0,
                       tok ? (const void *)dZ : W1_0, tok ? (const void *)dQ : dW1,
                       tok ? (const void *)dK : dW1, tok ? (const void *)dV : dW1,
                       tok ? (const void *)deta : dW1, tok ? (const void *)W1_ckpt : dW1,
                       tok ? (const void *)W2_ckpt : dW1};
  for (const void *x : req)
    if (!x) return TTT_ERR_ARG;
  for (const void *x : req)
    if (!aligned16(x)) return TTT_ERR_ALIGN;
  if ((dW1_T && !aligned16(dW1_T)) || (dW2_T && !aligned16(dW2_T))) return TTT_ERR_ALIGN;
  const size_t in_elt = qkv_dtype == TTT_BF16 ? 2 : 4;
  const size_t tbytes = tok ? (size_t)elems * 4 : 0, ibytes = tok ? (size_t)elems * in_elt : 0;
  const size_t ebytes = tok ? (size_t)units * T * 4 : 0, wbytes = (size_t)units * d * hidden * 4;
  const size_t hbytes = (size_t)H * d * hidden * 4, pbytes = (size_t)H * d * 4;
  const size_t vbytes = (size_t)units * d * 4;
  const size_t cbytes = tok ? (size_t)units * (T / b) * d * hidden * 4 : 0;
  Range ins[11] = {range_of(Q, ibytes),   range_of(K, ibytes),   range_of(V, ibytes),
                   range_of(eta, ebytes), range_of(W1_0, hbytes), range_of(W2_0, hbytes),
                   range_of(gamma, pbytes), range_of(beta, pbytes), range_of(dZ, tbytes),
                   range_of(dW1_T, dW1_T ? wbytes : 0), range_of(dW2_T, dW2_T ? wbytes : 0)};
  Range outs[10] = {range_of(dQ, tbytes),      range_of(dK, tbytes),      range_of(dV, tbytes),
                    range_of(deta, ebytes),    range_of(dW1, wbytes),     range_of(dW2, wbytes),
                    range_of(dgamma, vbytes),  range_of(dbeta, vbytes),   range_of(W1_ckpt, cbytes),
                    range_of(W2_ckpt, cbytes)};
  for (int o = 0; o < 10; ++o) {
    for (int i = 0; i < 11; ++i)
      if (overlap(outs[o], ins[i])) return TTT_ERR_ARG;
    for (int o2 = o + 1; o2 < 10; ++o2)
      if (overlap(outs[o], outs[o2])) return TTT_ERR_ARG;
  }
  bwdmlp::Params p{Q,  K,  V,    eta,  W1_0, W2_0, gamma,  beta,  eps,     dZ,     dW1_T,
                   dW2_T, H, T, b, dQ,   dK,   dV,    deta,  dW1,    dW2,   dgamma,  dbeta,
                   W1_ckpt, W2_ckpt};
  auto kernel = qkv_dtype == TTT_BF16 ? bwdmlp::mlp_bwd_kernel<__nv_bfloat16> : bwdmlp::mlp_bwd_kernel<float>;
  const size_t smem = bwdmlp::smem_bytes();
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return TTT_ERR_CUDA;
  kernel<<<(unsigned)units, bwdmlp::THREADS, smem, static_cast<cudaStream_t>(stream)>>>(p);
  if (cudaGetLastError() != cudaSuccess) return TTT_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return TTT_OK;
}

int run_momentum_fwd(bool ln, const void *Q, const void *K, const void *V, int qkv_dtype,
                     const float *eta, const float *alpha, const float *lambda, const float *W0,
                     const float *gamma, const float *beta, float eps, int B, int H, int T, int d,
                     int b, float *Z, float *W_out, float *S_out, void *stream) {
  if (qkv_dtype != TTT_F32 && qkv_dtype != TTT_BF16) return TTT_ERR_ARG;
  if (B < 0 || H < 0 || T < 0 || d <= 0 || b <= 0) return TTT_ERR_ARG;
  if (T % b != 0) return TTT_ERR_ARG;
  if (ln && !(std::isfinite(eps) && eps > 0.f)) return TTT_ERR_ARG;
  if (d != mom::D || b > mom::MAXB) return TTT_ERR_UNSUPPORTED;
  const long long units = (long long)B * H;
  if (units == 0) return TTT_OK;
  if (units > 0x7fffffffLL) return TTT_ERR_UNSUPPORTED;
  const long long elems = units * T * d;
  if (elems >= (1LL << 40)) return TTT_ERR_UNSUPPORTED;
  const bool tok = T > 0;
  const void *req[] = {W0, W_out, S_out, ln ? (const void *)gamma : W0, ln ? (const void *)beta : W0,
                       tok ? Q : W0, tok ? K : W0, tok ? V : W0, tok ? (const void *)eta : W0,
                       tok ? (const void *)alpha : W0, tok ? (const void *)lambda : W0,
                       tok ? (const void *)Z : W_out};
  for (const void *x : req)
    if (!x) return TTT_ERR_ARG;
  for (const void *x : req)
    if (!aligned16(x)) return TTT_ERR_ALIGN;
  const size_t in_elt = qkv_dtype == TTT_BF16 ? 2 : 4;
  const size_t ibytes = tok ? (size_t)elems * in_elt : 0, ebytes = tok ? (size_t)units * T * 4 : 0;
  const size_t pbytes = ln ? (size_t)H * d * 4 : 0, wbytes = (size_t)units * d * d * 4;
  Range ins[9] = {range_of(Q, ibytes),     range_of(K, ibytes),      range_of(V, ibytes),
                  range_of(eta, ebytes),   range_of(alpha, ebytes),  range_of(lambda, ebytes),
                  range_of(W0, (size_t)H * d * d * 4), range_of(gamma, pbytes), range_of(beta, pbytes)};
  Range outs[3] = {range_of(Z, tok ? (size_t)elems * 4 : 0), range_of(W_out, wbytes),
                   range_of(S_out, wbytes)};
  for (int o = 0; o < 3; ++o) {
    for (int i = 0; i < 9; ++i)
      if (overlap(outs[o], ins[i])) return TTT_ERR_ARG;
    for (int o2 = o + 1; o2 < 3; ++o2)
      if (overlap(outs[o], outs[o2])) return TTT_ERR_ARG;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const unsigned grid = (unsigned)units;
  const bool bf16 = qkv_dtype == TTT_BF16;
  // bf16 inputs and b = 16: the tensor-core dual form (unless the CUDA-core path
  // is selected).
  const int path = g_path.load();
  const bool tc_ok = bf16 && b == tcmom::MB;
  if (path == TTT_PATH_TC && !tc_ok) return TTT_ERR_UNSUPPORTED;
  if (tc_ok && T > 0 && path != TTT_PATH_SIMT) {
    CUtensorMap mq, mk, mv;
    if (!make_qkv_map(&mq, Q, T, units, 8) || !make_qkv_map(&mk, K, T, units, 8) ||
        !make_qkv_map(&mv, V, T, units, tcmom::CHUNK))
      return TTT_ERR_CUDA;
    tcmom::Params tp{eta, alpha, lambda, W0, gamma, beta, eps, H, T, Z, W_out, S_out, g_inject_timeout.load()};
    auto kernel = ln ? tcmom::momentum_tc_kernel<true> : tcmom::momentum_tc_kernel<false>;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tcmom::SMEM_BYTES) !=
            cudaSuccess ||
        cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared) != cudaSuccess)
      return TTT_ERR_CUDA;
    kernel<<<grid, tcmom::THREADS, tcmom::SMEM_BYTES, s>>>(mq, mk, mv, tp);
    if (cudaGetLastError() != cudaSuccess) return TTT_ERR_CUDA;
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return TTT_OK;
  }
  mom::Params p{Q, K, V, eta, alpha, lambda, W0, gamma, beta, eps, H, T, b, Z, W_out, S_out};
  if (ln)
    return bf16 ? launch_register_state<true, __nv_bfloat16, true>(grid, s, p)
                : launch_register_state<true, float, true>(grid, s, p);
  return bf16 ? launch_register_state<false, __nv_bfloat16, true>(grid, s, p)
              : launch_register_state<false, float, true>(grid, s, p);
}

int run_mlp_momentum_fwd(const void *Q, const void *K, const void *V, int qkv_dtype,
                         const float *eta, const float *alpha, const float *lambda,
                         const float *W1_0, const float *W2_0, const float *gamma, const float *beta,
                         float eps, int B, int H, int T, int d, int hidden, int b, float *Z,
                         float *W1, float *W2, float *S1, float *S2, void *stream) {
  if (qkv_dtype != TTT_F32 && qkv_dtype != TTT_BF16) return TTT_ERR_ARG;
  if (B < 0 || H < 0 || T < 0 || d <= 0 || hidden <= 0 || b <= 0) return TTT_ERR_ARG;
  if (T % b != 0) return TTT_ERR_ARG;
  if (!(std::isfinite(eps) && eps > 0.f)) return TTT_ERR_ARG;
  if (d != mommlp::D || hidden != mommlp::HID || b > mommlp::MAXB) return TTT_ERR_UNSUPPORTED;
  const long long units = (long long)B * H;
  if (units == 0) return TTT_OK;
  if (units > 0x7fffffffLL) return TTT_ERR_UNSUPPORTED;
  const long long elems = units * T * d;
  if (elems >= (1LL << 40)) return TTT_ERR_UNSUPPORTED;
  const bool tok = T > 0;
  const void *req[] = {W1_0, W2_0, gamma, beta, W1, W2, S1, S2,
                       tok ? Q : W1_0, tok ? K : W1_0, tok ? V : W1_0, tok ? (const void *)eta : W1_0,
                       tok ? (const void *)alpha : W1_0, tok ? (const void *)lambda : W1_0,
                       tok ? (const void *)Z : W1};
  for (const void *x : req)
    if (!x) return TTT_ERR_ARG;
  for (const void *x : req)
    if (!aligned16(x)) return TTT_ERR_ALIGN;
  const size_t in_elt = qkv_dtype == TTT_BF16 ? 2 : 4;
  const size_t ibytes = tok ? (size_t)elems * in_elt : 0, ebytes = tok ? (size_t)units * T * 4 : 0;
  const size_t hbytes = (size_t)H * d * hidden * 4, pbytes = (size_t)H * d * 4;
  const size_t wbytes = (size_t)units * d * hidden * 4;
  Range ins[10] = {range_of(Q, ibytes),    range_of(K, ibytes),      range_of(V, ibytes),
                   range_of(eta, ebytes),  range_of(alpha, ebytes),  range_of(lambda, ebytes),
                   range_of(W1_0, hbytes), range_of(W2_0, hbytes),   range_of(gamma, pbytes),
                   range_of(beta, pbytes)};
  Range outs[5] = {range_of(Z, tok ? (size_t)elems * 4 : 0), range_of(W1, wbytes), range_of(W2, wbytes),
                   range_of(S1, wbytes), range_of(S2, wbytes)};
  for (int o = 0; o < 5; ++o) {
    for (int i = 0; i < 10; ++i)
      if (overlap(outs[o], ins[i])) return TTT_ERR_ARG;
    for (int o2 = o + 1; o2 < 5; ++o2)
      if (overlap(outs[o], outs[o2])) return TTT_ERR_ARG;
  }
  mommlp::Params p{Q, K, V, eta, alpha, lambda, W1_0, W2_0, gamma, beta, eps, H, T, b, Z, W1, W2, S1, S2};
  auto kernel = qkv_dtype == TTT_BF16 ? mommlp::mlp_momentum_fwd_kernel<__nv_bfloat16>
                                      : mommlp::mlp_momentum_fwd_kernel<float>;
  const size_t smem = mommlp::smem_bytes();
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return TTT_ERR_CUDA;
  kernel<<<(unsigned)units, mommlp::THREADS, smem, static_cast<cudaStream_t>(stream)>>>(p);
  if (cudaGetLastError() != cudaSuccess) return TTT_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return TTT_OK;
}

int run(const Call &c) {
  const int st = validate(c);
  if (st != TTT_OK) return st;
  if ((long long)c.B * c.H == 0) return TTT_OK;
  const int path = g_path.load();
  const bool tc_ok = tc_supported(c);
  if (path == TTT_PATH_TC && !tc_ok) return TTT_ERR_UNSUPPORTED;
  if (path != TTT_PATH_SIMT && tc_ok) {
    if (c.kind == MLP_LN) return launch_mlp_tc(c);
    return c.kind == LINEAR_LN ? launch_linear_tc<true>(c) : launch_linear_tc<false>(c);
  }
  return run_simt(c);
}

// ---- the forward with inputs and outputs in host memory -----------------------------

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Byte offsets of the device copies in the caller's workspace (each 256-byte aligned).
struct HostLayout {
  size_t q, k, v, eta, z, w, w2, p0, p1, p2, p3, total;
};

HostLayout host_layout(Kind kind, int qkv_dtype, long long B, long long H, long long T, long long d,
                       long long hidden) {
  const size_t in_elt = qkv_dtype == TTT_BF16 ? 2 : 4;
  const size_t units = (size_t)(B * H), elems = units * (size_t)(T * d);
  const size_t P1 = (size_t)(kind == MLP_LN ? d * hidden : d * d);
  HostLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align256(bytes);
    return o;
  };
  L.q = take(elems * in_elt);
  L.k = take(elems * in_elt);
  L.v = take(elems * in_elt);
  L.eta = take(units * (size_t)T * 4);
  L.z = take(elems * 4);
  L.w = take(units * P1 * 4);
  L.w2 = take(kind == MLP_LN ? units * P1 * 4 : 0);
  L.p0 = take((size_t)H * P1 * 4);
  L.p1 = take(kind == MLP_LN ? (size_t)H * P1 * 4 : 0);
  L.p2 = take(kind != LINEAR ? (size_t)(H * d) * 4 : 0);
  L.p3 = take(kind != LINEAR ? (size_t)(H * d) * 4 : 0);
  L.total = off;
  return L;
}

// Streams and events of one host-memory call, released on every return path (a
// stream or event with work still pending is released once that work is done).
struct HostCallResources {
  cudaStream_t s_in = nullptr, s_out = nullptr;
  std::vector<cudaEvent_t> events;
  ~HostCallResources() {
    for (cudaEvent_t e : events) cudaEventDestroy(e);
    if (s_in) cudaStreamDestroy(s_in);
    if (s_out) cudaStreamDestroy(s_out);
  }
  cudaEvent_t event() {
    cudaEvent_t e = nullptr;
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return nullptr;
    events.push_back(e);
    return e;
  }
};

// The batch is split into `chunks` contiguous slices; slice i is copied in on s_in,
// computed on the caller's stream and copied out on s_out, so that the copy in of
// slice i + 1, the forward of slice i and the copy out of slice i - 1 overlap.
// Every step is ordered after the work already on the caller's stream, and the
// caller's stream waits for the last copy out.
int run_host(const Call &h, void *workspace, size_t workspace_bytes, int chunks) {
  const int st = validate(h);
  if (st != TTT_OK) return st;
  if (chunks < 1) return TTT_ERR_ARG;
  const long long units = (long long)h.B * h.H;
  if (units == 0) return TTT_OK;
  const HostLayout L = host_layout(h.kind, h.qkv_dtype, h.B, h.H, h.T, h.d, h.hidden);
  if (!workspace || workspace_bytes < L.total) return TTT_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return TTT_ERR_ALIGN;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  cudaStream_t s_run = static_cast<cudaStream_t>(h.stream);

  HostCallResources r;
  if (cudaStreamCreateWithFlags(&r.s_in, cudaStreamNonBlocking) != cudaSuccess ||
      cudaStreamCreateWithFlags(&r.s_out, cudaStreamNonBlocking) != cudaSuccess)
    return TTT_ERR_CUDA;
  cudaEvent_t fork = r.event();
  if (!fork || cudaEventRecord(fork, s_run) != cudaSuccess || cudaStreamWaitEvent(r.s_in, fork, 0) != cudaSuccess ||
      cudaStreamWaitEvent(r.s_out, fork, 0) != cudaSuccess)
    return TTT_ERR_CUDA;

  auto h2d = [&](size_t off, const void *src, size_t bytes) {
    return bytes == 0 || cudaMemcpyAsync(ws + off, src, bytes, cudaMemcpyHostToDevice, r.s_in) == cudaSuccess;
  };
  auto d2h = [&](void *dst, size_t off, size_t bytes) {
    return bytes == 0 || cudaMemcpyAsync(dst, ws + off, bytes, cudaMemcpyDeviceToHost, r.s_out) == cudaSuccess;
  };

  const size_t in_elt = h.qkv_dtype == TTT_BF16 ? 2 : 4;
  const size_t P1 = (size_t)(h.kind == MLP_LN ? (size_t)h.d * h.hidden : (size_t)h.d * h.d);
  const size_t tok_per_b = (size_t)h.H * h.T, elem_per_b = tok_per_b * h.d, state_per_b = (size_t)h.H * P1;
  // Per-head inputs first.
  if (!h2d(L.p0, h.W0, (size_t)h.H * P1 * 4)) return TTT_ERR_CUDA;
  if (h.kind == MLP_LN && !h2d(L.p1, h.W2_0, (size_t)h.H * P1 * 4)) return TTT_ERR_CUDA;
  if (h.kind != LINEAR && (!h2d(L.p2, h.gamma, (size_t)h.H * h.d * 4) || !h2d(L.p3, h.beta, (size_t)h.H * h.d * 4)))
    return TTT_ERR_CUDA;

  const int n = (int)std::min<long long>(chunks, h.B);
  for (int i = 0; i < n; ++i) {
    const size_t b0 = (size_t)((long long)h.B * i / n), b1 = (size_t)((long long)h.B * (i + 1) / n);
    const size_t nb = b1 - b0;
    if (nb == 0) continue;
    const size_t qo = b0 * elem_per_b * in_elt, qn = nb * elem_per_b * in_elt;
    const size_t eo = b0 * tok_per_b * 4, en = nb * tok_per_b * 4;
    const size_t zo = b0 * elem_per_b * 4, zn = nb * elem_per_b * 4;
    const size_t wo = b0 * state_per_b * 4, wn = nb * state_per_b * 4;
    if (h.T > 0) {
      const uint8_t *q = static_cast<const uint8_t *>(h.Q), *k = static_cast<const uint8_t *>(h.K),
                    *v = static_cast<const uint8_t *>(h.V);
      if (!h2d(L.q + qo, q + qo, qn) || !h2d(L.k + qo, k + qo, qn) || !h2d(L.v + qo, v + qo, qn) ||
          !h2d(L.eta + eo, reinterpret_cast<const uint8_t *>(h.eta) + eo, en))
        return TTT_ERR_CUDA;
    }
    cudaEvent_t loaded = r.event(), computed = r.event();
    if (!loaded || !computed || cudaEventRecord(loaded, r.s_in) != cudaSuccess ||
        cudaStreamWaitEvent(s_run, loaded, 0) != cudaSuccess)
      return TTT_ERR_CUDA;
    Call c = h;
    c.B = (int)nb;
    c.Q = ws + L.q + qo;
    c.K = ws + L.k + qo;
    c.V = ws + L.v + qo;
    c.eta = reinterpret_cast<const float *>(ws + L.eta + eo);
    c.Z = reinterpret_cast<float *>(ws + L.z + zo);
    c.W_out = reinterpret_cast<float *>(ws + L.w + wo);
    c.W2_out = h.kind == MLP_LN ? reinterpret_cast<float *>(ws + L.w2 + wo) : nullptr;
    c.W0 = reinterpret_cast<const float *>(ws + L.p0);
    c.W2_0 = h.kind == MLP_LN ? reinterpret_cast<const float *>(ws + L.p1) : nullptr;
    c.gamma = h.kind != LINEAR ? reinterpret_cast<const float *>(ws + L.p2) : nullptr;
    c.beta = h.kind != LINEAR ? reinterpret_cast<const float *>(ws + L.p3) : nullptr;
    c.stream = s_run;
    if (h.T == 0) c.Q = c.K = c.V = nullptr, c.eta = nullptr, c.Z = nullptr;
    const int rs = run(c);
    if (rs != TTT_OK) return rs;
    if (cudaEventRecord(computed, s_run) != cudaSuccess || cudaStreamWaitEvent(r.s_out, computed, 0) != cudaSuccess)
      return TTT_ERR_CUDA;
    if ((h.T > 0 && !d2h(reinterpret_cast<uint8_t *>(h.Z) + zo, L.z + zo, zn)) ||
        !d2h(reinterpret_cast<uint8_t *>(h.W_out) + wo, L.w + wo, wn) ||
        (h.kind == MLP_LN && !d2h(reinterpret_cast<uint8_t *>(h.W2_out) + wo, L.w2 + wo, wn)))
      return TTT_ERR_CUDA;
  }
  cudaEvent_t joined = r.event();
  if (!joined || cudaEventRecord(joined, r.s_out) != cudaSuccess || cudaStreamWaitEvent(s_run, joined, 0) != cudaSuccess)
    return TTT_ERR_CUDA;
  return TTT_OK;
}

Kind host_kind(int variant, bool *ok) {
  *ok = true;
  switch (variant) {
    case TTT_VARIANT_LINEAR: return LINEAR;
    case TTT_VARIANT_LINEAR_LN: return LINEAR_LN;
    case TTT_VARIANT_MLP: return MLP_LN;
    default: *ok = false; return LINEAR;
  }
}

}  // namespace

extern "C" {

size_t ttt_fwd_host_workspace_bytes(int variant, int qkv_dtype, int B, int H, int T, int d, int hidden) {
  bool ok = false;
  const Kind kind = host_kind(variant, &ok);
  if (!ok || (qkv_dtype != TTT_F32 && qkv_dtype != TTT_BF16) || B < 0 || H < 0 || T < 0 || d <= 0 ||
      (kind == MLP_LN && hidden <= 0))
    return 0;
  return host_layout(kind, qkv_dtype, B, H, T, d, hidden).total;
}

int ttt_fwd_host(int variant, const void *Q, const void *K, const void *V, int qkv_dtype, const float *eta,
                 const float *W0, const float *W2_0, const float *ln_gamma, const float *ln_beta, float ln_eps,
                 int B, int H, int T, int d, int hidden, int b, float *Z, float *W_out, float *W2_out,
                 void *workspace, size_t workspace_bytes, int chunks, void *stream) {
  bool ok = false;
  const Kind kind = host_kind(variant, &ok);
  if (!ok) return TTT_ERR_ARG;
  Call c{kind,
         Q,
         K,
         V,
         qkv_dtype,
         eta,
         W0,
         kind == MLP_LN ? W2_0 : nullptr,
         kind != LINEAR ? ln_gamma : nullptr,
         kind != LINEAR ? ln_beta : nullptr,
         kind != LINEAR ? ln_eps : 0.f,
         B,
         H,
         T,
         d,
         kind == MLP_LN ? hidden : 0,
         b,
         Z,
         W_out,
         kind == MLP_LN ? W2_out : nullptr,
         stream};
  return run_host(c, workspace, workspace_bytes, chunks);
}


int ttt_linear_fwd(const void *Q, const void *K, const void *V, int qkv_dtype, const float *eta,
                   const float *W0, int B, int H, int T, int d, int b, float *Z, float *W_out,
                   void *stream) {
  Call c{LINEAR, Q, K, V, qkv_dtype, eta, W0, nullptr, nullptr, nullptr, 0.f,
         B,      H, T, d, 0,         b,   Z,  W_out,   nullptr, stream};
  return run(c);
}

int ttt_linear_ln_fwd(const void *Q, const void *K, const void *V, int qkv_dtype, const float *eta,
                      const float *W0, const float *ln_gamma, const float *ln_beta, float ln_eps,
                      int B, int H, int T, int d, int b, float *Z, float *W_out, void *stream) {
  Call c{LINEAR_LN, Q, K, V, qkv_dtype, eta, W0, nullptr, ln_gamma, ln_beta, ln_eps,
         B,         H, T, d, 0,         b,   Z,  W_out,   nullptr,  stream};
  return run(c);
}

int ttt_mlp_fwd(const void *Q, const void *K, const void *V, int qkv_dtype, const float *eta,
                const float *W1_0, const float *W2_0, const float *ln_gamma, const float *ln_beta,
                float ln_eps, int B, int H, int T, int d, int hidden, int b, float *Z,
                float *W1_out, float *W2_out, void *stream) {
  Call c{MLP_LN, Q, K, V, qkv_dtype, eta, W1_0, W2_0, ln_gamma, ln_beta, ln_eps,
         B,      H, T, d, hidden,    b,   Z,    W1_out, W2_out, stream};
  return run(c);
}

const char *ttt_status_string(int status) {
  switch (status) {
    case TTT_OK: return "success";
    case TTT_ERR_ARG: return "invalid argument (null pointer, negative size, bad dtype, T % b != 0 or overlapping buffers)";
    case TTT_ERR_ALIGN: return "pointer not 16-byte aligned";
    case TTT_ERR_UNSUPPORTED: return "unsupported size (d, b or hidden) for this library";
    case TTT_ERR_CUDA: return "CUDA runtime call or kernel launch failed";
    case TTT_ERR_TIMEOUT: return "a bounded device-side wait expired";
    default: return "unknown status";
  }
}

int ttt_last_device_status(void *stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return TTT_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, ttt::g_device_status, sizeof(int)) != cudaSuccess) return TTT_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(ttt::g_device_status, &zero, sizeof(int)) != cudaSuccess) return TTT_ERR_CUDA;
  return v;
}

int ttt_set_path(int path) {
  if (path != TTT_PATH_AUTO && path != TTT_PATH_SIMT && path != TTT_PATH_TC) return TTT_ERR_ARG;
  return g_path.exchange(path);
}

long long ttt_launch_count(void) { return g_launches.load(); }

int ttt_debug_inject_timeout(int on) { return g_inject_timeout.exchange(on ? 1 : 0); }

int ttt_linear_decode(const void *q, const void *k, const void *v, int qkv_dtype, const float *eta,
                      float *W, float *W_base, int B, int H, int d, int b, int pos, float *z,
                      void *stream) {
  return run_decode(false, q, k, v, qkv_dtype, eta, W, W_base, nullptr, nullptr, 1.f, B, H, d, b,
                    pos, z, stream);
}

int ttt_linear_momentum_decode(const void *q, const void *k, const void *v, int qkv_dtype,
                               const float *eta, const float *alpha, const float *lambda, float *W,
                               float *W_base, float *S, int B, int H, int d, int b, int pos, float *z,
                               void *stream) {
  return run_decode(false, q, k, v, qkv_dtype, eta, W, W_base, nullptr, nullptr, 1.f, B, H, d, b,
                    pos, z, stream, true, alpha, lambda, S);
}

int ttt_linear_ln_momentum_decode(const void *q, const void *k, const void *v, int qkv_dtype,
                                  const float *eta, const float *alpha, const float *lambda,
                                  float *W, float *W_base, float *S, const float *ln_gamma,
                                  const float *ln_beta, float ln_eps, int B, int H, int d, int b,
                                  int pos, float *z, void *stream) {
  return run_decode(true, q, k, v, qkv_dtype, eta, W, W_base, ln_gamma, ln_beta, ln_eps, B, H, d, b,
                    pos, z, stream, true, alpha, lambda, S);
}

int ttt_mlp_decode(const void *q, const void *k, const void *v, int qkv_dtype, const float *eta,
                   float *W1, float *W2, float *W1_base, float *W2_base, const float *ln_gamma,
                   const float *ln_beta, float ln_eps, int B, int H, int d, int hidden, int b, int pos,
                   float *z, void *stream) {
  return run_mlp_decode(q, k, v, qkv_dtype, eta, W1, W2, W1_base, W2_base, ln_gamma, ln_beta, ln_eps,
                        B, H, d, hidden, b, pos, z, stream);
}

int ttt_mlp_momentum_decode(const void *q, const void *k, const void *v, int qkv_dtype,
                            const float *eta, const float *alpha, const float *lambda, float *W1,
                            float *W2, float *W1_base, float *W2_base, float *S1, float *S2,
                            const float *ln_gamma, const float *ln_beta, float ln_eps, int B, int H,
                            int d, int hidden, int b, int pos, float *z, void *stream) {
  return run_mlp_decode(q, k, v, qkv_dtype, eta, W1, W2, W1_base, W2_base, ln_gamma, ln_beta, ln_eps,
                        B, H, d, hidden, b, pos, z, stream, true, alpha, lambda, S1, S2);
}

int ttt_linear_momentum_fwd(const void *Q, const void *K, const void *V, int qkv_dtype,
                            const float *eta, const float *alpha, const float *lambda,
                            const float *W0, int B, int H, int T, int d, int b, float *Z,
                            float *W_out, float *S_out, void *stream) {
  return run_momentum_fwd(false, Q, K, V, qkv_dtype, eta, alpha, lambda, W0, nullptr, nullptr, 1.f, B,
                          H, T, d, b, Z, W_out, S_out, stream);
}

int ttt_linear_ln_momentum_fwd(const void *Q, const void *K, const void *V, int qkv_dtype,
                               const float *eta, const float *alpha, const float *lambda,
                               const float *W0, const float *ln_gamma, const float *ln_beta,
                               float ln_eps, int B, int H, int T, int d, int b, float *Z,
                               float *W_out, float *S_out, void *stream) {
  return run_momentum_fwd(true, Q, K, V, qkv_dtype, eta, alpha, lambda, W0, ln_gamma, ln_beta, ln_eps,
                          B, H, T, d, b, Z, W_out, S_out, stream);
}

int ttt_linear_bwd(const void *Q, const void *K, const void *V, int qkv_dtype, const float *eta,
                   const float *W0, const float *dZ, const float *dW_T, int B, int H, int T, int d,
                   int b, float *dQ, float *dK, float *dV, float *deta, float *dW0, float *W_ckpt,
                   void *stream) {
  return run_bwd(false, Q, K, V, qkv_dtype, eta, W0, nullptr, nullptr, 1.f, dZ, dW_T, B, H, T, d, b,
                 dQ, dK, dV, deta, dW0, nullptr, nullptr, W_ckpt, stream);
}

int ttt_linear_ln_bwd(const void *Q, const void *K, const void *V, int qkv_dtype, const float *eta,
                      const float *W0, const float *ln_gamma, const float *ln_beta, float ln_eps,
                      const float *dZ, const float *dW_T, int B, int H, int T, int d, int b,
                      float *dQ, float *dK, float *dV, float *deta, float *dW0, float *dgamma,
                      float *dbeta, float *W_ckpt, void *stream) {
  return run_bwd(true, Q, K, V, qkv_dtype, eta, W0, ln_gamma, ln_beta, ln_eps, dZ, dW_T, B, H, T, d,
                 b, dQ, dK, dV, deta, dW0, dgamma, dbeta, W_ckpt, stream);
}

int ttt_mlp_momentum_fwd(const void *Q, const void *K, const void *V, int qkv_dtype,
                         const float *eta, const float *alpha, const float *lambda,
                         const float *W1_0, const float *W2_0, const float *ln_gamma,
                         const float *ln_beta, float ln_eps, int B, int H, int T, int d, int hidden,
                         int b, float *Z, float *W1_out, float *W2_out, float *S1_out, float *S2_out,
                         void *stream) {
  return run_mlp_momentum_fwd(Q, K, V, qkv_dtype, eta, alpha, lambda, W1_0, W2_0, ln_gamma, ln_beta,
                              ln_eps, B, H, T, d, hidden, b, Z, W1_out, W2_out, S1_out, S2_out, stream);
}

int ttt_mlp_bwd(const void *Q, const void *K, const void *V, int qkv_dtype, const float *eta,
                const float *W1_0, const float *W2_0, const float *ln_gamma, const float *ln_beta,
                float ln_eps, const float *dZ, const float *dW1_T, const float *dW2_T, int B, int H,
                int T, int d, int hidden, int b, float *dQ, float *dK, float *dV, float *deta,
                float *dW1_0, float *dW2_0, float *dgamma, float *dbeta, float *W1_ckpt,
                float *W2_ckpt, void *stream) {
  return run_mlp_bwd(Q, K, V, qkv_dtype, eta, W1_0, W2_0, ln_gamma, ln_beta, ln_eps, dZ, dW1_T, dW2_T,
                     B, H, T, d, hidden, b, dQ, dK, dV, deta, dW1_0, dW2_0, dgamma, dbeta, W1_ckpt,
                     W2_ckpt, stream);
}

int ttt_linear_ln_decode(const void *q, const void *k, const void *v, int qkv_dtype,
                         const float *eta, float *W, float *W_base, const float *ln_gamma,
                         const float *ln_beta, float ln_eps, int B, int H, int d, int b, int pos,
                         float *z, void *stream) {
  return run_decode(true, q, k, v, qkv_dtype, eta, W, W_base, ln_gamma, ln_beta, ln_eps, B, H, d,
                    b, pos, z, stream);
}

}  // extern "C"

// ---- Backward of TTT-Linear + LN without any allocation -------------------------
//
// For callers that cannot call cudaMalloc (an operator hosted by a framework
// that owns the device allocator, or a process that reserves all device memory
// up front): the per-mini-batch states that the backward's reverse pass reads
// back live in one fixed device array of this library instead of a caller
// workspace.  Every device that loads the library holds the array (64 MiB)
// until the process exits; calls on a device share it, so calls that overlap
// on the GPU race on it.  A call writes each state before reading it, so the
// array never needs clearing.
namespace ttt {
namespace noalloc {

constexpr long long MAX_STATES = TTT_NOALLOC_BWD_MAX_STATES;  // d x d fp32 states
static __device__ __align__(256) float g_bwd_states[MAX_STATES * 64 * 64];

}  // namespace noalloc
}  // namespace ttt

namespace {

constexpr int kNoAllocMaxDevices = 256;
std::mutex g_noalloc_mu;
std::atomic<float *> g_noalloc_states[kNoAllocMaxDevices];

// The device address of the state array on the current device, looked up once
// per device.  In host code the array's name denotes a host-side stand-in, not
// device memory, so only this address may be handed to a kernel.
int noalloc_states(float **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return TTT_ERR_CUDA;
  if (dev >= kNoAllocMaxDevices) return TTT_ERR_UNSUPPORTED;
  float *ptr = g_noalloc_states[dev].load(std::memory_order_acquire);
  if (!ptr) {
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    ptr = g_noalloc_states[dev].load(std::memory_order_relaxed);
    if (!ptr) {
      void *addr = nullptr;
      if (cudaGetSymbolAddress(&addr, ttt::noalloc::g_bwd_states) != cudaSuccess || !addr)
        return TTT_ERR_CUDA;
      ptr = static_cast<float *>(addr);
      g_noalloc_states[dev].store(ptr, std::memory_order_release);
    }
  }
  *out = ptr;
  return TTT_OK;
}

}  // namespace

extern "C" int ttt_linear_ln_bwd_noalloc(const void *Q, const void *K, const void *V,
                                         int qkv_dtype, const float *eta, const float *W0,
                                         const float *ln_gamma, const float *ln_beta, float ln_eps,
                                         const float *dZ, const float *dW_T, int B, int H, int T,
                                         int d, int b, float *dQ, float *dK, float *dV,
                                         float *deta, float *dW0, float *dgamma, float *dbeta,
                                         void *stream) {
  // The size checks of the backward, then the array's capacity, all before the
  // one-time address lookup; the pointer checks follow in run_bwd.
  if (qkv_dtype != TTT_F32 && qkv_dtype != TTT_BF16) return TTT_ERR_ARG;
  if (B < 0 || H < 0 || T < 0 || d <= 0 || b <= 0 || T % b != 0) return TTT_ERR_ARG;
  if (!(std::isfinite(ln_eps) && ln_eps > 0.f)) return TTT_ERR_ARG;
  if (d != bwd::D || b > bwd::MAXB) return TTT_ERR_UNSUPPORTED;
  const long long units = (long long)B * H;
  if (units == 0) return TTT_OK;
  if (units > ttt::noalloc::MAX_STATES || units * (T / b) > ttt::noalloc::MAX_STATES)
    return TTT_ERR_UNSUPPORTED;
  float *states = nullptr;
  const int st = noalloc_states(&states);
  if (st != TTT_OK) return st;
  return run_bwd(true, Q, K, V, qkv_dtype, eta, W0, ln_gamma, ln_beta, ln_eps, dZ, dW_T, B, H, T, d,
                 b, dQ, dK, dV, deta, dW0, dgamma, dbeta, states, stream);
}
