// Backward pass of the gated delta rule (gradients of the forward pass with
// respect to q, k, v, beta, log_alpha and the initial state), as a reverse
// token recurrence in fp32.
//
// Forward, per sequence and head, token t (the definition the chunked kernels
// evaluate; "DeltaTTT: Layerwise Optimization for Nonlinear Recurrent Memory",
// §2 Background and §4.1):
//   S~_t = D_t S_{t-1},  r_t = S~_t^T k_t,  u_t = beta_t (v_t - r_t),
//   S_t = S~_t + k_t u_t^T,  o_t = S_t^T q_t.
// Reverse, with G = dL/dS_t (starting from dL/dS_T, the final-state
// gradient, or zero) and dO_t = dL/do_t:
//   G     += q_t dO_t^T                    dq_t = S_t dO_t
//   du_t   = G^T k_t                       dk_t = G u_t - beta_t S~_t du_t
//   dbeta_t = du_t . (v_t - r_t)           dv_t = beta_t du_t
//   G~     = G - beta_t k_t du_t^T         (= dL/dS~_t)
//   dlog_alpha_t = sum_j G~ . S~_t         (per key row c for the channel
//                                           gate, over all of S for scalar)
//   G      = D_t G~                        (= dL/dS_{t-1});  dS_0 = G at t = 1.
//
// The reverse sweep needs S~_t in reverse order.  One CTA per (sequence,
// head) first runs the forward recurrence and checkpoints the state at every
// kWin-th token in scratch; then, window by window from the end, it replays
// the window from its checkpoint (keeping S~_t of each token of the window in
// scratch) and runs the reverse steps over it.  The state tile lives in
// registers as in the decode step: warp w owns rows [w dk/8, (w+1) dk/8),
// lane l owns columns [4l, 4l+4); column sums (over key rows) meet in shared
// memory, row sums (over value columns) are warp shuffles.
//
// This is a reference-grade kernel: each token is a chain of dependent
// reductions, so it is latency-bound (see the measurement notes); a chunked
// tensor-core backward is the next step.

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "gdr_internal.h"

namespace gdr {
namespace {

constexpr int kBwThreads = 256;
constexpr int kWin = 16;   // tokens per checkpoint window

struct BwParams {
  const void *q, *k, *v, *dout;
  const float *log_alpha, *beta, *s0, *dsT;
  float *gq, *gk, *gv, *gla, *gbeta, *gs0;   // gradients (written)
  // scratch: checkpoints [H][total_win][dk*dv] (sequence n's windows start
  // at the sum of the earlier sequences' window counts), then one window of
  // S~ states per (sequence, head) [nseq*H][kWin][dk*dv]
  float *scratch;
  const int32_t *cu;
  int T, ntok, H, dv, nseq;
  long long total_win;
};

template <typename T>
__device__ __forceinline__ float bld(const T *p);
template <>
__device__ __forceinline__ float bld<float>(const float *p) {
  return *p;
}
template <>
__device__ __forceinline__ float bld<__nv_bfloat16>(const __nv_bfloat16 *p) {
  return __bfloat162float(*p);
}

__device__ __forceinline__ float4 f4(float a) { return make_float4(a, a, a, a); }
__device__ __forceinline__ float4 add4(float4 a, float4 b) {
  return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}
__device__ __forceinline__ float4 fma4(float s, float4 a, float4 b) {
  return make_float4(fmaf(s, a.x, b.x), fmaf(s, a.y, b.y), fmaf(s, a.z, b.z),
                     fmaf(s, a.w, b.w));
}
__device__ __forceinline__ float dot4(float4 a, float4 b) {
  return a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1)
    x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

// Per-token vectors staged in shared memory for the whole CTA.
template <int DK>
struct alignas(16) TokVec {
  float k[DK], q[DK], a[DK];   // key, query, decay per key row
  float v[128], dO[128];
  float beta;
};

// A token's vectors, one element of each per thread (thread i holds key row
// i and value column i): fetched from global memory one token ahead, then
// published to shared memory at the token boundary.
struct TokReg {
  float k, q, la, v, dO, beta;
};

template <int DK, typename T, int GATE>
__device__ __forceinline__ TokReg fetch_tok(const BwParams &p, size_t row,
                                            bool with_grad) {
  TokReg r{0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  const int i = threadIdx.x;
  if (i < DK) {
    r.k = bld(static_cast<const T *>(p.k) + row * DK + i);
    r.q = bld(static_cast<const T *>(p.q) + row * DK + i);
    if (GATE == 1) r.la = p.log_alpha[row];
    if (GATE == 2) r.la = p.log_alpha[row * DK + i];
  }
  if (i < p.dv) {
    r.v = bld(static_cast<const T *>(p.v) + row * p.dv + i);
    if (with_grad) r.dO = bld(static_cast<const T *>(p.dout) + row * p.dv + i);
  }
  if (i == 0) r.beta = p.beta[row];
  return r;
}

template <int DK, int GATE>
__device__ __forceinline__ void publish_tok(TokVec<DK> &tv, const TokReg &r,
                                            int dv) {
  const int i = threadIdx.x;
  if (i < DK) {
    tv.k[i] = r.k;
    tv.q[i] = r.q;
    tv.a[i] = GATE == 0 ? 1.f : __expf(r.la);
  }
  if (i < dv) {
    tv.v[i] = r.v;
    tv.dO[i] = r.dO;
  }
  if (i == 0) tv.beta = r.beta;
}

template <int DK, typename T, int GATE>
__global__ void __launch_bounds__(kBwThreads, 1) gdr_bwd_kernel(BwParams p) {
  constexpr int R = DK / 8;
  __shared__ TokVec<DK> tv;
  __shared__ float4 red[2][2][8][32];   // [parity][quantity][warp][lane]
  __shared__ float bsum[8];
  const int n = blockIdx.x / p.H, h = blockIdx.x % p.H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int dv = p.dv, j0 = 4 * lane;
  const bool act = j0 < dv;
  int start = p.cu ? p.cu[n] : n * p.T;
  int end = p.cu ? p.cu[n + 1] : (n + 1) * p.T;
  start = min(max(start, 0), p.ntok);
  end = min(max(end, start), p.ntok);
  const int L = end - start;
  const int nwin = (L + kWin - 1) / kWin;
  const size_t ss = (size_t)DK * dv;                  // floats per state
  long long woff = 0;   // windows of the sequences before this one
  if (p.cu) {
    for (int m = 0; m < n; ++m) {
      const int a = min(max(p.cu[m], 0), p.ntok);
      const int e = min(max(p.cu[m + 1], a), p.ntok);
      woff += (e - a + kWin - 1) / kWin;
    }
  } else {
    woff = (long long)n * ((p.T + kWin - 1) / kWin);
  }
  float *ckpt = p.scratch + ((size_t)h * p.total_win + woff) * ss;
  float *winb = p.scratch + (size_t)p.H * p.total_win * ss +
                (size_t)blockIdx.x * kWin * ss;
  const size_t sb = ((size_t)n * p.H + h) * ss;
  auto idx = [&](int r) { return (size_t)(warp * R + r) * dv + j0; };
  auto ld = [&](const float *base, int r) {
    return act ? *reinterpret_cast<const float4 *>(base + idx(r)) : f4(0.f);
  };
  auto st = [&](float *base, int r, float4 x) {
    if (act) *reinterpret_cast<float4 *>(base + idx(r)) = x;
  };
  auto row_of = [&](int t) { return (size_t)(start + t) * p.H + h; };

  // one forward token on the register tile S: S <- D S (S~ saved if asked),
  // then S <- S~ + k u^T; returns nothing (u is not needed later)
  float4 S[R];
  int par = 0;
  TokReg nx{0.f, 0.f, 0.f, 0.f, 0.f, 0.f};   // the next token's vectors
  // forward token t (its vectors in nx); prefetches token tn (if >= 0)
  auto fwd_token = [&](int t, float *save, int tn) {
    publish_tok<DK, GATE>(tv, nx, dv);
    if (tn >= 0) nx = fetch_tok<DK, T, GATE>(p, row_of(tn), false);
    __syncthreads();
    float4 pr = f4(0.f);
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int c = warp * R + r;
      const float a = tv.a[c];
      S[r] = make_float4(a * S[r].x, a * S[r].y, a * S[r].z, a * S[r].w);
      if (save) st(save, r, S[r]);
      pr = fma4(tv.k[c], S[r], pr);
    }
    red[par][0][warp][lane] = pr;
    __syncthreads();
    float4 rk = red[par][0][0][lane];
#pragma unroll
    for (int w = 1; w < 8; ++w) rk = add4(rk, red[par][0][w][lane]);
    const float b = tv.beta;
    const float4 vv = act ? *reinterpret_cast<const float4 *>(&tv.v[j0]) : f4(0.f);
    const float4 u = make_float4(b * (vv.x - rk.x), b * (vv.y - rk.y),
                                 b * (vv.z - rk.z), b * (vv.w - rk.w));
#pragma unroll
    for (int r = 0; r < R; ++r) S[r] = fma4(tv.k[warp * R + r], u, S[r]);
    par ^= 1;
    __syncthreads();   // tv is reloaded by the next token
  };

  // ---- forward sweep: checkpoint the state before every window
#pragma unroll
  for (int r = 0; r < R; ++r) S[r] = p.s0 ? ld(p.s0 + sb, r) : f4(0.f);
  if (L > 0) nx = fetch_tok<DK, T, GATE>(p, row_of(0), false);
  for (int t = 0; t < L; ++t) {
    if (t % kWin == 0) {
#pragma unroll
      for (int r = 0; r < R; ++r) st(ckpt + (size_t)(t / kWin) * ss, r, S[r]);
    }
    fwd_token(t, nullptr, t + 1 < L ? t + 1 : -1);
  }
  // ---- reverse sweep
  float4 G[R];
#pragma unroll
  for (int r = 0; r < R; ++r) G[r] = p.dsT ? ld(p.dsT + sb, r) : f4(0.f);
  for (int w = nwin - 1; w >= 0; --w) {
    const int t0 = w * kWin, t1 = min(L, t0 + kWin);
    // replay the window from its checkpoint, keeping each token's S~
#pragma unroll
    for (int r = 0; r < R; ++r) S[r] = ld(ckpt + (size_t)w * ss, r);
    nx = fetch_tok<DK, T, GATE>(p, row_of(t0), false);
    for (int t = t0; t < t1; ++t)
      fwd_token(t, winb + (size_t)(t - t0) * ss, t + 1 < t1 ? t + 1 : -1);
    nx = fetch_tok<DK, T, GATE>(p, row_of(t1 - 1), true);
    for (int t = t1 - 1; t >= t0; --t) {
      const size_t row = row_of(t);
      publish_tok<DK, GATE>(tv, nx, dv);
      if (t > t0) nx = fetch_tok<DK, T, GATE>(p, row_of(t - 1), true);
      float4 Sm[R];   // S~_t
#pragma unroll
      for (int r = 0; r < R; ++r) Sm[r] = ld(winb + (size_t)(t - t0) * ss, r);
      __syncthreads();
      const float4 dO = act ? *reinterpret_cast<const float4 *>(&tv.dO[j0]) : f4(0.f);
      // G += q dO^T; column partials of S~^T k and G^T k
      float4 pr = f4(0.f), pd = f4(0.f);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int c = warp * R + r;
        G[r] = fma4(tv.q[c], dO, G[r]);
        pr = fma4(tv.k[c], Sm[r], pr);
        pd = fma4(tv.k[c], G[r], pd);
      }
      red[par][0][warp][lane] = pr;
      red[par][1][warp][lane] = pd;
      __syncthreads();
      float4 rk = red[par][0][0][lane], du = red[par][1][0][lane];
#pragma unroll
      for (int ww = 1; ww < 8; ++ww) {
        rk = add4(rk, red[par][0][ww][lane]);
        du = add4(du, red[par][1][ww][lane]);
      }
      par ^= 1;
      const float b = tv.beta;
      const float4 vv = act ? *reinterpret_cast<const float4 *>(&tv.v[j0]) : f4(0.f);
      const float4 vr = make_float4(vv.x - rk.x, vv.y - rk.y, vv.z - rk.z,
                                    vv.w - rk.w);
      const float4 u = make_float4(b * vr.x, b * vr.y, b * vr.z, b * vr.w);
      if (!act) {
        du = f4(0.f);
      }
      // dbeta = du . (v - r): warp 0's lanes cover every column once
      if (warp == 0) {
        const float db = warp_sum(dot4(du, vr));
        if (lane == 0) p.gbeta[row] = db;
        if (act) {
          float *dvp = p.gv + row * dv + j0;
          *reinterpret_cast<float4 *>(dvp) =
              make_float4(b * du.x, b * du.y, b * du.z, b * du.w);
        }
      }
      // per key row: dq = S_t dO, dk = G u - beta S~ du, dla = G~ . S~
      float dla_tot = 0.f;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int c = warp * R + r;
        const float kc = tv.k[c];
        const float4 St = fma4(kc, u, Sm[r]);
        float dqc = warp_sum(dot4(St, dO));
        float dkc = warp_sum(dot4(G[r], u) - b * dot4(Sm[r], du));
        const float4 Gt = fma4(-b * kc, du, G[r]);   // G~
        const float dl = dot4(Gt, Sm[r]);
        if (GATE == 2) {
          const float dlc = warp_sum(dl);
          if (lane == 0) p.gla[row * DK + c] = dlc;
        } else {
          dla_tot += dl;
        }
        if (lane == 0) {
          p.gq[row * DK + c] = dqc;
          p.gk[row * DK + c] = dkc;
        }
        const float a = tv.a[c];
        G[r] = make_float4(a * Gt.x, a * Gt.y, a * Gt.z, a * Gt.w);
      }
      if (GATE == 1) {
        dla_tot = warp_sum(dla_tot);
        if (lane == 0) bsum[warp] = dla_tot;
      }
      __syncthreads();   // bsum complete; tv reloaded next token
      if (GATE == 1 && threadIdx.x == 0) {
        float s = 0.f;
#pragma unroll
        for (int ww = 0; ww < 8; ++ww) s += bsum[ww];
        p.gla[row] = s;
      }
    }
  }
  if (p.gs0) {
#pragma unroll
    for (int r = 0; r < R; ++r) st(p.gs0 + sb, r, G[r]);
  }
}

template <int DK, typename T>
cudaError_t bw_launch_dk(const BwParams &bp, int gate, int nblocks,
                         cudaStream_t s) {
  switch (gate) {
    case 0: gdr_bwd_kernel<DK, T, 0><<<nblocks, kBwThreads, 0, s>>>(bp); break;
    case 1: gdr_bwd_kernel<DK, T, 1><<<nblocks, kBwThreads, 0, s>>>(bp); break;
    default: gdr_bwd_kernel<DK, T, 2><<<nblocks, kBwThreads, 0, s>>>(bp); break;
  }
  return cudaGetLastError();
}

template <typename T>
cudaError_t bw_launch_t(const BwParams &bp, int dk, int gate, int nblocks,
                        cudaStream_t s) {
  switch (dk) {
    case 16: return bw_launch_dk<16, T>(bp, gate, nblocks, s);
    case 32: return bw_launch_dk<32, T>(bp, gate, nblocks, s);
    case 64: return bw_launch_dk<64, T>(bp, gate, nblocks, s);
    default: return bw_launch_dk<128, T>(bp, gate, nblocks, s);
  }
}

}  // namespace

size_t backward_scratch_bytes(const Problem &p, long long *total_win) {
  // windows over all sequences: exactly nseq * ceil(T / kWin) for fixed
  // length; at most ntok / kWin + nseq for a packed batch
  const long long tw =
      p.cu ? (long long)p.ntok / kWin + p.nseq
           : (long long)p.nseq * ((p.T + kWin - 1) / kWin);
  *total_win = tw;
  const long long ss = (long long)p.dk * p.dv;
  return (size_t)(((long long)p.H * tw + (long long)p.nseq * p.H * kWin) * ss) *
         sizeof(float);
}

cudaError_t backward_run(const Problem &p, const BackwardIO &io,
                         float *scratch, long long total_win, cudaStream_t s) {
  BwParams bp;
  bp.q = p.q;
  bp.k = p.k;
  bp.v = p.v;
  bp.dout = io.dout;
  bp.log_alpha = p.log_alpha;
  bp.beta = p.beta;
  bp.s0 = p.s0;
  bp.dsT = io.dsT;
  bp.gq = io.dq;
  bp.gk = io.dk;
  bp.gv = io.dv;
  bp.gla = io.dla;
  bp.gbeta = io.dbeta;
  bp.gs0 = io.ds0;
  bp.scratch = scratch;
  bp.cu = p.cu;
  bp.T = p.T;
  bp.ntok = p.ntok;
  bp.H = p.H;
  bp.dv = p.dv;
  bp.nseq = p.nseq;
  bp.total_win = total_win;
  const int nb = p.nseq * p.H;
  return p.dtype == GDR_BF16
             ? bw_launch_t<__nv_bfloat16>(bp, p.dk, p.gate, nb, s)
             : bw_launch_t<float>(bp, p.dk, p.gate, nb, s);
}

}  // namespace gdr
