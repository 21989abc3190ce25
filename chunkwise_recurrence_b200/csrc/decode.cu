// Single-token decode step of libgdr: the recurrent update of a resident
// state, one token per (sequence, head).
//
// Per (sequence, head), with the state S (dk x dv, fp32) and one token:
//   S~ = D S                   D = I, alpha I or diag(alpha)
//   r  = S~^T k,  u = beta (v - r)
//   S' = S~ + k u^T            (= (I - beta k k^T) D S + beta k v^T)
//   o  = S'^T q = S~^T q + u (k . q)
// This is the delta rule's one-token step ("DeltaTTT: Layerwise Optimization
// for Nonlinear Recurrent Memory", §2 Background and §4.1); decoding runs it
// once per generated token with the state read and written back each time
// ("Delta-Rule Linear Attention" topic page, GDN decode-accelerator card: one
// state read and one state write per token, under 1 FLOP per byte).
//
// The step moves 2 dk dv 4 bytes of state per (sequence, head) against about
// 6 dk dv flops, so it is bound by HBM bandwidth.  One CTA of 256 threads per
// (sequence, head).  The state tile (contiguous, dk dv 4 bytes) comes into
// shared memory with one bulk asynchronous copy (cp.async.bulk, completion on
// an mbarrier) and leaves with one bulk store, so three CTAs per SM keep
// up to 3 x 64 KB of state in flight with a handful of instructions.  In
// shared memory warp w owns rows [w dk/8, (w+1) dk/8) of S and lane l
// columns [4l, 4l+4) (16-byte accesses, whole 512-byte rows per warp); the
// two column reductions (S~^T k, S~^T q) meet in shared memory; S' overwrites
// the tile in place before the store.  state_in == state_out is safe: the
// tile is read in full before any of it is written back.  The copy wait is
// bounded; on expiry the CTA skips its step and raises the library's device
// error word (gdr_device_error: GDR_ERR_TIMEOUT).
//
// With Gated DeltaNet-2's gates (erase != nullptr) the read key is b . k
// (erase gate b, per key channel) and the target w . v (write gate w, per
// value channel), without beta:  u = w . v - S~^T (b . k),  S' = S~ + k u^T,
// o = S~^T q + u (k . q)  (gdr_decode_step_gdn2).  With FG^2-GDN's rate
// (wkey != nullptr) the write key is a . k (rate a, per key channel) and the
// target (c .) v:  u = (c .) v - S~^T k,  S' = S~ + (a . k) u^T,
// o = S~^T q + u ((a . k) . q)  (gdr_decode_step_fg2).

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdlib>

#include "gdr_internal.h"
#include "sm100.cuh"

namespace gdr {

__device__ unsigned g_decode_error;

namespace {

using namespace sm100;

constexpr int kDecThreads = 256;
constexpr long long kDecWaitCycles = 1ll << 31;   // ~1 s: never reached
// GDR_FAULT_INJECT_DECODE_TIMEOUT=1: the state copy is never issued and the
// wait gives up after this many cycles (tests of the timeout path)
constexpr long long kDecInjectWaitCycles = 1ll << 20;

__device__ __forceinline__ void bulk_load(void *dst, const void *src,
                                          uint32_t bytes, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1], %2, [%3];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void bulk_store(void *dst, const void *src,
                                           uint32_t bytes) {
  asm volatile(
      "cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(
          reinterpret_cast<uint64_t>(dst)),
      "r"(smem_u32(src)), "r"(bytes)
      : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
  // the source tile must stay in place until the copy has read it
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

struct DecodeParams {
  const void *q, *k, *v;
  const float *log_alpha, *beta, *s_in;
  float *s_out;
  void *out;
  int dv;
  // Gated DeltaNet-2 gates [N*H][dk] and [N*H][dv], or nullptr
  const float *erase, *write;
  // FG^2-GDN's key-side rate [N*H][dk], or nullptr (`write` is then the
  // optional value-side scaling)
  const float *wkey;
  // failure injection (host hook): the state copy is not issued, so the
  // CTA's wait runs out after wait_cycles and reports a timeout
  int inject_timeout;
  long long wait_cycles;
};

template <typename T>
__device__ __forceinline__ float ld1(const T *p);
template <>
__device__ __forceinline__ float ld1<float>(const float *p) {
  return *p;
}
template <>
__device__ __forceinline__ float ld1<__nv_bfloat16>(const __nv_bfloat16 *p) {
  return __bfloat162float(*p);
}
// four consecutive elements (8- or 16-byte aligned)
__device__ __forceinline__ float4 ld4(const float *p) {
  return *reinterpret_cast<const float4 *>(p);
}
__device__ __forceinline__ float4 ld4(const __nv_bfloat16 *p) {
  const uint2 w = *reinterpret_cast<const uint2 *>(p);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w.y));
  return make_float4(a.x, a.y, b.x, b.y);
}
__device__ __forceinline__ void st4(float *p, float4 x) {
  *reinterpret_cast<float4 *>(p) = x;
}
__device__ __forceinline__ void st4(__nv_bfloat16 *p, float4 x) {
  const __nv_bfloat162 a = __floats2bfloat162_rn(x.x, x.y);
  const __nv_bfloat162 b = __floats2bfloat162_rn(x.z, x.w);
  uint2 w;
  w.x = *reinterpret_cast<const uint32_t *>(&a);
  w.y = *reinterpret_cast<const uint32_t *>(&b);
  *reinterpret_cast<uint2 *>(p) = w;
}
__device__ __forceinline__ float4 fma4(float s, float4 a, float4 b) {
  return make_float4(fmaf(s, a.x, b.x), fmaf(s, a.y, b.y), fmaf(s, a.z, b.z),
                     fmaf(s, a.w, b.w));
}

template <int DK, typename T, int GATE>
__global__ void __launch_bounds__(kDecThreads)
    gdr_decode_kernel(DecodeParams p) {
  constexpr int R = DK / 8;   // rows of S per warp
  extern __shared__ __align__(128) float tile[];   // the state, [DK][dv]
  // sr: read key; sw: write key
  __shared__ float sk[DK], sq[DK], sa[DK], sr[DK], sw[DK];
  __shared__ float4 red[2][8][32];   // per warp: partial S~^T k, S~^T q
  __shared__ float kq_s;
  __shared__ __align__(8) uint64_t bar;
  __shared__ int copy_ok;
  const int nh = blockIdx.x;         // (sequence, head), flattened
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int dv = p.dv, j0 = 4 * lane;
  const bool act = j0 < dv;
  const size_t sb = (size_t)nh * DK * dv;
  const uint32_t bytes = (uint32_t)(DK * dv * 4);
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    copy_ok = 1;
    if (p.s_in) {
      mbar_arrive_expect_tx(&bar, bytes);
      if (!p.inject_timeout) bulk_load(tile, p.s_in + sb, bytes, &bar);
    }
  }
  const T *q = static_cast<const T *>(p.q) + (size_t)nh * DK;
  const T *k = static_cast<const T *>(p.k) + (size_t)nh * DK;
  for (int c = threadIdx.x; c < DK; c += kDecThreads) {
    sk[c] = ld1(k + c);
    sq[c] = ld1(q + c);
    sa[c] = GATE == 0   ? 1.f
            : GATE == 1 ? __expf(p.log_alpha[nh])
                        : __expf(p.log_alpha[(size_t)nh * DK + c]);
    sr[c] = p.erase ? p.erase[(size_t)nh * DK + c] * sk[c] : sk[c];
    sw[c] = p.wkey ? p.wkey[(size_t)nh * DK + c] * sk[c] : sk[c];
  }
  if (threadIdx.x == 0 && p.s_in) {
    const long long t0 = clock64();
    while (!mbar_try_wait(&bar, 0)) {
      if (clock64() - t0 > p.wait_cycles) {
        copy_ok = 0;
        atomicOr(&g_decode_error, 1u);
        break;
      }
    }
    // After an expired wait the tile is not used, but the CTA stays until
    // the copy it issued has landed (a second bounded wait), so that a late
    // copy never writes into shared memory another CTA has since been
    // given.  (An injected expiry issued no copy.)  A copy still in flight
    // after that leaves the context suspect: see GDR_ERR_TIMEOUT.
    if (!copy_ok && !p.inject_timeout) {
      const long long t1 = clock64();
      while (!mbar_try_wait(&bar, 0) && clock64() - t1 < 4 * p.wait_cycles) {
      }
    }
  }
  __syncthreads();
  if (!copy_ok) return;   // uniform: the tile never arrived
  // S~ = D S for this thread's rows and columns; partial column reductions
  float4 pk = make_float4(0.f, 0.f, 0.f, 0.f), pq = pk;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int c = warp * R + r;
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    if (act && p.s_in) x = ld4(tile + c * dv + j0);
    const float a = sa[c];
    x = make_float4(a * x.x, a * x.y, a * x.z, a * x.w);
    if (act) st4(tile + c * dv + j0, x);   // S~, kept for the update
    pk = fma4(sr[c], x, pk);
    pq = fma4(sq[c], x, pq);
  }
  red[0][warp][lane] = pk;
  red[1][warp][lane] = pq;
  if (warp == 0) {
    float t = 0.f;
    for (int c = lane; c < DK; c += 32) t = fmaf(sw[c], sq[c], t);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
      t += __shfl_xor_sync(0xffffffffu, t, off);
    if (lane == 0) kq_s = t;
  }
  __syncthreads();
  float4 rk = red[0][0][lane], rq = red[1][0][lane];
#pragma unroll
  for (int w = 1; w < 8; ++w) {
    const float4 a = red[0][w][lane], b = red[1][w][lane];
    rk = make_float4(rk.x + a.x, rk.y + a.y, rk.z + a.z, rk.w + a.w);
    rq = make_float4(rq.x + b.x, rq.y + b.y, rq.z + b.z, rq.w + b.w);
  }
  if (act) {
    // u = beta (v - S~^T k) (Gated DeltaNet-2: w . v - S~^T (b . k);
    // FG^2-GDN: (c .) v - S~^T k);  o = S~^T q + u (write key . q)
    const float4 vv = ld4(static_cast<const T *>(p.v) + (size_t)nh * dv + j0);
    float4 u;
    if (p.erase || p.wkey) {
      const float4 wg = p.write ? ld4(p.write + (size_t)nh * dv + j0)
                                : make_float4(1.f, 1.f, 1.f, 1.f);
      u = make_float4(wg.x * vv.x - rk.x, wg.y * vv.y - rk.y,
                      wg.z * vv.z - rk.z, wg.w * vv.w - rk.w);
    } else {
      const float bt = p.beta[nh];
      u = make_float4(bt * (vv.x - rk.x), bt * (vv.y - rk.y),
                      bt * (vv.z - rk.z), bt * (vv.w - rk.w));
    }
    if (warp == 0)
      st4(static_cast<T *>(p.out) + (size_t)nh * dv + j0, fma4(kq_s, u, rq));
    // S' = S~ + (write key) u^T, in place in the tile
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int c = warp * R + r;
      float *e = tile + c * dv + j0;
      st4(e, fma4(sw[c], u, ld4(e)));
    }
  }
  // the tile's generic-proxy writes, visible to the bulk store
  fence_proxy_async_smem();
  __syncthreads();
  if (threadIdx.x == 0) bulk_store(p.s_out + sb, tile, bytes);
}

template <int DK, typename T, int GATE>
cudaError_t launch_g(const DecodeParams &dp, int nblocks, cudaStream_t s) {
  const int smem = DK * dp.dv * 4;
  cudaError_t e = cudaFuncSetAttribute(
      gdr_decode_kernel<DK, T, GATE>,
      cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  gdr_decode_kernel<DK, T, GATE><<<nblocks, kDecThreads, smem, s>>>(dp);
  return cudaGetLastError();
}

template <int DK, typename T>
cudaError_t launch_dk(const DecodeParams &dp, int gate, int nblocks,
                      cudaStream_t s) {
  switch (gate) {
    case 0: return launch_g<DK, T, 0>(dp, nblocks, s);
    case 1: return launch_g<DK, T, 1>(dp, nblocks, s);
    default: return launch_g<DK, T, 2>(dp, nblocks, s);
  }
}

template <typename T>
cudaError_t launch_t(const DecodeParams &dp, int dk, int gate, int nblocks,
                     cudaStream_t s) {
  switch (dk) {
    case 16: return launch_dk<16, T>(dp, gate, nblocks, s);
    case 32: return launch_dk<32, T>(dp, gate, nblocks, s);
    case 64: return launch_dk<64, T>(dp, gate, nblocks, s);
    default: return launch_dk<128, T>(dp, gate, nblocks, s);
  }
}

}  // namespace

cudaError_t decode_read_error(unsigned *word, bool clear) {
  cudaError_t e = cudaMemcpyFromSymbol(word, g_decode_error, sizeof(unsigned));
  if (e != cudaSuccess) return e;
  if (clear && *word) {
    const unsigned zero = 0;
    e = cudaMemcpyToSymbol(g_decode_error, &zero, sizeof(unsigned));
  }
  return e;
}

namespace {

bool aligned16(const void *p) {
  return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}
bool dim_ok(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }

}  // namespace
}  // namespace gdr

namespace gdr {
namespace {

// The gate form follows from which of beta, erase, wkey is given: exactly
// one of them (erase with write, wkey with an optional write).
gdr_status decode_entry(const void *q, const void *k, const void *v,
                        const float *log_alpha, const float *beta,
                        const float *erase, const float *write,
                        const float *wkey,
                        const float *state_in, float *state_out, void *out,
                        int N, int H, int dk, int dv, cudaStream_t stream,
                        const gdr_opts *opts) {
  gdr_opts o;
  o.dtype = GDR_BF16;
  o.gate = GDR_GATE_SCALAR;
  o.cu_seqlens = nullptr;
  o.num_seqs = 0;
  o.algo = GDR_ALGO_AUTO;
  if (opts) o = *opts;
  if (N < 0 || H < 0) return GDR_ERR_INVALID_ARGUMENT;
  if (o.dtype != GDR_BF16 && o.dtype != GDR_FP32) return GDR_ERR_INVALID_ARGUMENT;
  if (o.gate != GDR_GATE_NONE && o.gate != GDR_GATE_SCALAR &&
      o.gate != GDR_GATE_CHANNEL)
    return GDR_ERR_INVALID_ARGUMENT;
  if (o.cu_seqlens != nullptr || o.num_seqs != 0)
    return GDR_ERR_INVALID_ARGUMENT;   // one token per sequence: no packing
  if (o.algo != GDR_ALGO_AUTO) return GDR_ERR_UNSUPPORTED;
  if (!dim_ok(dk) || !dim_ok(dv)) return GDR_ERR_UNSUPPORTED;
  if ((o.gate == GDR_GATE_NONE) != (log_alpha == nullptr))
    return GDR_ERR_INVALID_ARGUMENT;
  const long long nh = (long long)N * H;
  if (nh > 0x7fffffffLL) return GDR_ERR_UNSUPPORTED;
  if (nh == 0) return GDR_OK;
  if (!q || !k || !v || !state_out || !out) return GDR_ERR_INVALID_ARGUMENT;
  if ((beta != nullptr) + (erase != nullptr) + (wkey != nullptr) != 1)
    return GDR_ERR_INVALID_ARGUMENT;
  if (beta && write) return GDR_ERR_INVALID_ARGUMENT;
  if (erase && !write) return GDR_ERR_INVALID_ARGUMENT;
  const void *ptrs[] = {q, k, v, log_alpha, beta, erase, write, wkey,
                        state_in, state_out, out};
  for (const void *ptr : ptrs)
    if (ptr && !aligned16(ptr)) return GDR_ERR_INVALID_ARGUMENT;
  // state_in and state_out: the same buffer (in-place update) or disjoint
  if (state_in && state_in != state_out) {
    const size_t bytes = (size_t)nh * dk * dv * sizeof(float);
    const uintptr_t a = reinterpret_cast<uintptr_t>(state_in);
    const uintptr_t b = reinterpret_cast<uintptr_t>(state_out);
    if (a < b + bytes && b < a + bytes) return GDR_ERR_INVALID_ARGUMENT;
  }
  DecodeParams dp;
  dp.q = q;
  dp.k = k;
  dp.v = v;
  dp.log_alpha = log_alpha;
  dp.beta = beta;
  dp.s_in = state_in;
  dp.s_out = state_out;
  dp.out = out;
  dp.dv = dv;
  dp.erase = erase;
  dp.write = write;
  dp.wkey = wkey;
  const char *inj = std::getenv("GDR_FAULT_INJECT_DECODE_TIMEOUT");
  dp.inject_timeout = (inj && inj[0] == '1') ? 1 : 0;
  dp.wait_cycles = dp.inject_timeout ? kDecInjectWaitCycles : kDecWaitCycles;
  const int nb = (int)nh;
  const cudaError_t e =
      o.dtype == GDR_BF16
          ? launch_t<__nv_bfloat16>(dp, dk, o.gate, nb, stream)
          : launch_t<float>(dp, dk, o.gate, nb, stream);
  return e == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

}  // namespace
}  // namespace gdr

extern "C" gdr_status gdr_decode_step(const void *q, const void *k,
                                      const void *v, const float *log_alpha,
                                      const float *beta,
                                      const float *state_in, float *state_out,
                                      void *out, int N, int H, int dk, int dv,
                                      cudaStream_t stream,
                                      const gdr_opts *opts) {
  return gdr::decode_entry(q, k, v, log_alpha, beta, nullptr, nullptr,
                           nullptr, state_in, state_out, out, N, H, dk, dv,
                           stream, opts);
}

extern "C" gdr_status gdr_decode_step_gdn2(
    const void *q, const void *k, const void *v, const float *log_alpha,
    const float *erase_gate, const float *write_gate, const float *state_in,
    float *state_out, void *out, int N, int H, int dk, int dv,
    cudaStream_t stream, const gdr_opts *opts) {
  if (!erase_gate || !write_gate) return GDR_ERR_INVALID_ARGUMENT;
  return gdr::decode_entry(q, k, v, log_alpha, nullptr, erase_gate,
                           write_gate, nullptr, state_in, state_out, out, N, H,
                           dk, dv, stream, opts);
}

extern "C" gdr_status gdr_decode_step_fg2(
    const void *q, const void *k, const void *v, const float *log_alpha,
    const float *beta_k, const float *beta_v, const float *state_in,
    float *state_out, void *out, int N, int H, int dk, int dv,
    cudaStream_t stream, const gdr_opts *opts) {
  if (!beta_k) return GDR_ERR_INVALID_ARGUMENT;
  return gdr::decode_entry(q, k, v, log_alpha, nullptr, nullptr, beta_v,
                           beta_k, state_in, state_out, out, N, H, dk, dv,
                           stream, opts);
}
