// Exact-flow step size (EFLA) for the delta rule, as a reparametrisation of
// beta in front of the chunked forward pass and the decode step.
//
// The delta rule's token update S <- S - beta k (S^T k - v)^T is one explicit
// Euler step of length beta of the flow dS/dtau = -k k^T S + k v^T (the
// gradient flow of 1/2 ||S^T k - v||^2); EFLA replaces the Euler step by the
// exact flow, whose rank-1 dynamics make the matrix exponential and the input
// integral collapse to the same update form ("Delta-Rule Linear Attention"
// topic page, EFLA card).  With lambda = ||k||^2, exp(-beta k k^T) =
// I - (1 - e^{-beta lambda}) / lambda k k^T and the input integral is
// (1 - e^{-beta lambda}) / lambda k v^T, so the exact step is the delta rule
// with
//   beta' = (1 - e^{-beta lambda}) / lambda      (-> beta as lambda -> 0).
// The decay (D S) applies before the flow, as for the delta rule.
//
// One warp per (token, head): the squared key norm by a warp reduction, then
// beta' from expm1 (accurate for small beta lambda).

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "gdr_internal.h"

namespace gdr {
namespace {

template <typename T>
__device__ __forceinline__ float efla_ld(const T *p);
template <>
__device__ __forceinline__ float efla_ld<float>(const float *p) {
  return *p;
}
template <>
__device__ __forceinline__ float efla_ld<__nv_bfloat16>(
    const __nv_bfloat16 *p) {
  return __bfloat162float(*p);
}

template <typename T>
__global__ void __launch_bounds__(256)
    gdr_efla_beta_kernel(const T *k, const float *beta, float *beta_out,
                         long long rows, int dk) {
  const long long row =
      (long long)blockIdx.x * 8 + (threadIdx.x >> 5);   // (token, head)
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const T *kr = k + row * dk;
  float s = 0.f;
  for (int c = lane; c < dk; c += 32) {
    const float x = efla_ld(kr + c);
    s = fmaf(x, x, s);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1)
    s += __shfl_xor_sync(0xffffffffu, s, off);
  if (lane == 0) {
    const float b = beta[row];
    // (1 - e^{-b s}) / s, and its limit b for s -> 0
    beta_out[row] = s > 0.f ? -expm1f(-b * s) / s : b;
  }
}

// Chain rule through beta' = (1 - e^{-x}) / s, x = beta s, s = |k|^2:
//   d beta = d beta' e^{-x},
//   dk    += d beta' (d beta' / d s) 2 k,
//   d beta' / d s = (x e^{-x} + e^{-x} - 1) / s^2 = beta^2 f(x) / x^2,
// with f(x) / x^2 = -1/2 + x/3 - x^2/8 + x^3/30 - x^4/144 + ... (its Taylor
// series below x = 0.25, where the closed form cancels; the next term is
// under 1e-6 of the sum there).  One warp per (token, head).
template <typename T>
__global__ void __launch_bounds__(256)
    gdr_efla_beta_bwd_kernel(const T *k, const float *beta, const float *dbp,
                             float *dbeta, float *dk, long long rows,
                             int dkd) {
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const T *kr = k + row * dkd;
  float s = 0.f;
  for (int c = lane; c < dkd; c += 32) {
    const float x = efla_ld(kr + c);
    s = fmaf(x, x, s);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1)
    s += __shfl_xor_sync(0xffffffffu, s, off);
  const float b = beta[row], g = dbp[row];
  const float x = b * s;
  float fx;   // f(x) / x^2
  if (x < 0.25f) {
    fx = -0.5f + x * (1.f / 3.f + x * (-0.125f + x * (1.f / 30.f -
                                                      x * (1.f / 144.f))));
  } else {
    const float e = __expf(-x);
    fx = (x * e + expm1f(-x)) / (x * x);
  }
  const float dbeta_ds = b * b * fx;
  if (lane == 0) dbeta[row] = g * __expf(-x);
  const float sc = 2.f * g * dbeta_ds;
  for (int c = lane; c < dkd; c += 32) dk[row * dkd + c] += sc * efla_ld(kr + c);
}

}  // namespace
}  // namespace gdr

extern "C" gdr_status gdr_efla_beta_backward(const void *k, const float *beta,
                                             const float *d_beta_prime,
                                             float *d_beta, float *dk,
                                             int ntok, int H, int dk_,
                                             gdr_dtype dtype,
                                             cudaStream_t stream) {
  if (ntok < 0 || H < 0) return GDR_ERR_INVALID_ARGUMENT;
  if (dtype != GDR_BF16 && dtype != GDR_FP32) return GDR_ERR_INVALID_ARGUMENT;
  if (dk_ != 16 && dk_ != 32 && dk_ != 64 && dk_ != 128)
    return GDR_ERR_UNSUPPORTED;
  const long long rows = (long long)ntok * H;
  if (rows == 0) return GDR_OK;
  if (rows > (1ll << 33)) return GDR_ERR_UNSUPPORTED;   // grid.x bound
  if (!k || !beta || !d_beta_prime || !d_beta || !dk)
    return GDR_ERR_INVALID_ARGUMENT;
  const void *ptrs[] = {k, beta, d_beta_prime, d_beta, dk};
  for (const void *p : ptrs)
    if (reinterpret_cast<uintptr_t>(p) & 15u) return GDR_ERR_INVALID_ARGUMENT;
  const long long blocks = (rows + 7) / 8;
  if (dtype == GDR_BF16)
    gdr::gdr_efla_beta_bwd_kernel<__nv_bfloat16>
        <<<(unsigned)blocks, 256, 0, stream>>>(
            static_cast<const __nv_bfloat16 *>(k), beta, d_beta_prime, d_beta,
            dk, rows, dk_);
  else
    gdr::gdr_efla_beta_bwd_kernel<float><<<(unsigned)blocks, 256, 0, stream>>>(
        static_cast<const float *>(k), beta, d_beta_prime, d_beta, dk, rows,
        dk_);
  return cudaGetLastError() == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

extern "C" gdr_status gdr_efla_beta(const void *k, const float *beta,
                                    float *beta_out, int ntok, int H, int dk,
                                    gdr_dtype dtype, cudaStream_t stream) {
  if (ntok < 0 || H < 0) return GDR_ERR_INVALID_ARGUMENT;
  if (dtype != GDR_BF16 && dtype != GDR_FP32) return GDR_ERR_INVALID_ARGUMENT;
  if (dk != 16 && dk != 32 && dk != 64 && dk != 128) return GDR_ERR_UNSUPPORTED;
  const long long rows = (long long)ntok * H;
  if (rows == 0) return GDR_OK;
  if (rows > (1ll << 33)) return GDR_ERR_UNSUPPORTED;   // grid.x bound
  if (!k || !beta || !beta_out) return GDR_ERR_INVALID_ARGUMENT;
  const void *ptrs[] = {k, beta, beta_out};
  for (const void *p : ptrs)
    if (reinterpret_cast<uintptr_t>(p) & 15u) return GDR_ERR_INVALID_ARGUMENT;
  // beta_out may be beta itself (in place); otherwise they must not overlap
  if (beta_out != beta) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(beta);
    const uintptr_t b = reinterpret_cast<uintptr_t>(beta_out);
    const size_t bytes = (size_t)rows * sizeof(float);
    if (a < b + bytes && b < a + bytes) return GDR_ERR_INVALID_ARGUMENT;
  }
  const long long blocks = (rows + 7) / 8;
  if (dtype == GDR_BF16)
    gdr::gdr_efla_beta_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(k), beta, beta_out, rows, dk);
  else
    gdr::gdr_efla_beta_kernel<float><<<(unsigned)blocks, 256, 0, stream>>>(
        static_cast<const float *>(k), beta, beta_out, rows, dk);
  return cudaGetLastError() == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}
