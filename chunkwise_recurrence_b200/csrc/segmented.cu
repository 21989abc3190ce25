// Context-parallel state passing: the sequential combine of segment maps.
//
// The recurrence is affine in the state ("DeltaTTT: Layerwise Optimization
// for Nonlinear Recurrent Memory", §2 Background: the update is affine in the
// preceding memory), so over a segment of a sequence the state map is
//   S_out = M S_in + N,
// with M (dk x dk) the segment's state transition (the recurrence run from
// S_in = I with v = 0) and N (dk x dv) its offset (run from S_in = 0).
// gdr_chunk_fwd_segmented computes M and N of every segment in parallel with
// the ordinary forward kernels; this kernel then walks each sequence's
// segments in order,
//   S_in(s) = S,   S <- M_s S + N_s,
// and hands every segment its true initial state for the final pass.
//
// One CTA per (sequence, head); S (dk x dv) and M_s (dk x dk) in shared
// memory, fp32 throughout.  Thread (warp w, lane l) owns rows
// [w dk/8, (w+1) dk/8) and columns [4l, 4l+4) of S.

#include <cuda_runtime.h>

#include <cstdint>

#include "gdr_internal.h"

namespace gdr {
namespace {

constexpr int kCombThreads = 256;

__global__ void __launch_bounds__(kCombThreads)
    segment_combine_kernel(const float *s0, const float *Ms, const float *Ns,
                           float *Sin, const int32_t *seg_first, int H,
                           int dk, int dv) {
  extern __shared__ __align__(16) float sm[];
  float *S = sm;                 // [dk][dv]
  float *M = sm + dk * dv;       // [dk][dk]
  const int n = blockIdx.x / H, h = blockIdx.x % H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int R = dk / 8, j0 = 4 * lane;
  const bool act = j0 < dv;
  const size_t ss = (size_t)dk * dv, sm2 = (size_t)dk * dk;
  for (int i = threadIdx.x; i < dk * dv; i += kCombThreads)
    S[i] = s0 ? s0[((size_t)n * H + h) * ss + i] : 0.f;
  const int f0 = seg_first[n], f1 = seg_first[n + 1];
  for (int sg = f0; sg < f1; ++sg) {
    const size_t base = (size_t)sg * H + h;
    __syncthreads();   // S complete
    for (int i = threadIdx.x; i < dk * dv; i += kCombThreads)
      Sin[base * ss + i] = S[i];
    for (int i = threadIdx.x; i < dk * dk; i += kCombThreads)
      M[i] = Ms[base * sm2 + i];
    __syncthreads();   // M loaded
    float4 acc[16];   // rows r < R of this thread (R <= 16)
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      const int c = warp * R + r;
      acc[r] = (act && r < R) ? *reinterpret_cast<const float4 *>(
                                    Ns + base * ss + (size_t)c * dv + j0)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (act) {
      for (int e = 0; e < dk; ++e) {
        const float4 se = *reinterpret_cast<const float4 *>(S + e * dv + j0);
#pragma unroll
        for (int r = 0; r < 16; ++r) {
          if (r < R) {
            const float m = M[(warp * R + r) * dk + e];
            acc[r].x = fmaf(m, se.x, acc[r].x);
            acc[r].y = fmaf(m, se.y, acc[r].y);
            acc[r].z = fmaf(m, se.z, acc[r].z);
            acc[r].w = fmaf(m, se.w, acc[r].w);
          }
        }
      }
    }
    __syncthreads();   // every thread has read S and M
    if (act) {
#pragma unroll
      for (int r = 0; r < 16; ++r)
        if (r < R)
          *reinterpret_cast<float4 *>(S + (warp * R + r) * dv + j0) = acc[r];
    }
  }
}

__global__ void fill_identity_kernel(float *eye, long long nstates, int dk) {
  const long long total = nstates * dk * dk;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
       i < total; i += (long long)gridDim.x * blockDim.x) {
    const int rc = (int)(i % ((long long)dk * dk));
    eye[i] = (rc / dk == rc % dk) ? 1.f : 0.f;
  }
}

}  // namespace

cudaError_t fill_identity(float *eye, long long nstates, int dk,
                          cudaStream_t s) {
  if (nstates == 0) return cudaSuccess;
  fill_identity_kernel<<<592, 256, 0, s>>>(eye, nstates, dk);
  return cudaGetLastError();
}

cudaError_t segment_combine(const float *s0, const float *Ms, const float *Ns,
                            float *Sin, const int32_t *seg_first, int nseq,
                            int H, int dk, int dv, cudaStream_t s) {
  if (nseq == 0 || H == 0) return cudaSuccess;
  const int smem = (dk * dv + dk * dk) * (int)sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(
      segment_combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
      smem);
  if (e != cudaSuccess) return e;
  segment_combine_kernel<<<nseq * H, kCombThreads, smem, s>>>(
      s0, Ms, Ns, Sin, seg_first, H, dk, dv);
  return cudaGetLastError();
}

}  // namespace gdr
