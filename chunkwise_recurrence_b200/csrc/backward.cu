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
// That single-CTA kernel serves dk or dv = 16; for dk, dv >= 32 the
// column-split kernel further down runs the same three sweeps on dv / 32
// CTAs per (sequence, head).  Both evaluate every token's rank-one products
// on CUDA cores (about 29 dk dv flops per token and head over the three
// sweeps), so they are bound by fp32 issue, not by HBM.  gdr_backward runs
// them as its RECURRENT algorithm; the chunked backward
// (backward_chunked.cu) is the default.

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
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


// ---------------------------------------------------------------------------
// Column-split variant (dk, dv in {32, 64, 128}).  The recurrence acts on
// every value column j of S independently (S~_t = D_t S_{t-1} and the delta
// update read and write column j alone, with r_t[j] = k_t . S~_t[:, j]), so a
// (sequence, head) chain is split over dv / 32 CTAs of 32 columns each; only
// the row sums dq, dk, dlog_alpha and dbeta cross the split.  Each CTA writes
// its share of those per token into a partial array of its own, and a
// reduction kernel adds the groups in a fixed order (deterministic).
//
// Thread (warp w, lane l) of a 128-thread CTA holds rows c_i = 16 i + 4 w +
// (l >> 3), i < dk / 16, and the four columns 32 g + 4 (l & 7) .. +3 of its
// group g: a column sum over rows is a shuffle over l >> 3 plus one exchange
// of four warp partials in shared memory (one CTA barrier per token); a row
// sum over the CTA's columns is a shuffle over l & 7, done for all rows at
// once by a transposing reduction.
constexpr int kBcThreads = 128;
constexpr int kCW = 32;      // value columns per CTA
constexpr int kBcWin = 8;    // tokens per checkpoint window

struct BcParams {
  const void *q, *k, *v, *dout;
  const float *log_alpha, *beta, *s0, *dsT;
  float *gv, *gs0;
  float *ckpt;   // [H][total_win][ng][dk * kCW], thread-private tile layout
  float *winb;   // [nblocks][kBcWin][dk * kCW]
  float *pq, *pk, *pla, *pb;   // partials, group-major
  const int32_t *cu;
  int T, ntok, H, dv, nseq, ng;
  long long total_win;
};

template <int DK>
struct alignas(16) BcTok {
  float k[DK], q[DK], a[DK];   // a: channel gate's per-row decay
  float v[kCW], dO[kCW];
  float beta, a_s;             // a_s: scalar decay (1 without a gate)
};

// Reduces x[0..V) over the 8 lanes that share l >> 3 (xor 4, 2, 1),
// halving the values each lane keeps: afterwards this lane holds the sums
// of indices [base, base + n), n = max(V / 8, 1).  Where fewer than 8
// values remain, lanes pair up and hold equal sums (dup_mask picks one).
template <int V>
__device__ __forceinline__ int xreduce8(float *x, int cq) {
  int base = 0;
  int n = V;
#pragma unroll
  for (int d = 4; d >= 1; d >>= 1) {
    if (n > 1) {
      const int half = n / 2;
      const bool hi = (cq & d) != 0;
#pragma unroll
      for (int j = 0; j < half; ++j) {
        const float send = hi ? x[j] : x[j + half];
        const float keep = hi ? x[j + half] : x[j];
        x[j] = keep + __shfl_xor_sync(0xffffffffu, send, d);
      }
      if (hi) base += half;
      n = half;
    } else {
      x[0] += __shfl_xor_sync(0xffffffffu, x[0], d);
    }
  }
  return base;
}
template <int V>
constexpr int xreduce8_dup_mask() {
  return (V < 2 ? 4 : 0) | (V < 4 ? 2 : 0) | (V < 8 ? 1 : 0);
}

template <int DK, typename T, int GATE>
__global__ void __launch_bounds__(kBcThreads, 4)
    gdr_bwd_cols_kernel(BcParams p) {
  constexpr int R = DK / 16;       // rows per thread
  constexpr int NW = kBcThreads / 32;
  constexpr int TILE = DK * kCW;   // floats of one CTA's state tile
  __shared__ BcTok<DK> tv[3];
  __shared__ float4 red[2][2][NW][8];   // [parity][quantity][warp][cq]
  const int chain = blockIdx.x / p.ng, g = blockIdx.x % p.ng;
  const int n = chain / p.H, h = chain % p.H;
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int cq = lane & 7, rl = lane >> 3;
  const int dv = p.dv, jc = g * kCW + 4 * cq;   // first column of this thread
  int start = p.cu ? p.cu[n] : n * p.T;
  int end = p.cu ? p.cu[n + 1] : (n + 1) * p.T;
  start = min(max(start, 0), p.ntok);
  end = min(max(end, start), p.ntok);
  const int L = end - start;
  const int nwin = (L + kBcWin - 1) / kBcWin;
  long long woff = 0;
  if (p.cu) {
    for (int m = 0; m < n; ++m) {
      const int a = min(max(p.cu[m], 0), p.ntok);
      const int e = min(max(p.cu[m + 1], a), p.ntok);
      woff += (e - a + kBcWin - 1) / kBcWin;
    }
  } else {
    woff = (long long)n * ((p.T + kBcWin - 1) / kBcWin);
  }
  const size_t X = (size_t)p.ntok * p.H;
  auto ckpt_of = [&](int win) {
    return p.ckpt + (((size_t)h * p.total_win + woff + win) * p.ng + g) * TILE;
  };
  float *winb = p.winb + (size_t)blockIdx.x * kBcWin * TILE;
  const size_t sb = ((size_t)n * p.H + h) * DK * dv;
  auto row_c = [&](int i) { return 16 * i + 4 * w + rl; };
  // thread-private tile layout: element group i of thread tid at float4
  // index i * kBcThreads + tid (coalesced, read back by the same thread)
  auto tl = [&](float *base, int i) {
    return reinterpret_cast<float4 *>(base) + i * kBcThreads + tid;
  };
  auto row_of = [&](int t) { return (size_t)(start + t) * p.H + h; };

  // token vectors: fetched into registers two tokens ahead, published to
  // shared memory (three slots) one token ahead
  struct Reg {
    float k, q, la, v, dO, beta;
  };
  auto fetch = [&](int t, bool grad) {
    Reg r{0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    const size_t row = row_of(t);
    if (tid < DK) {
      r.k = bld(static_cast<const T *>(p.k) + row * DK + tid);
      r.q = bld(static_cast<const T *>(p.q) + row * DK + tid);
      if (GATE == 2) r.la = p.log_alpha[row * DK + tid];
    }
    if (tid < kCW) {
      r.v = bld(static_cast<const T *>(p.v) + row * dv + g * kCW + tid);
      if (grad)
        r.dO = bld(static_cast<const T *>(p.dout) + row * dv + g * kCW + tid);
    }
    if (tid == 0) {
      r.beta = p.beta[row];
      if (GATE == 1) r.la = p.log_alpha[row];
    }
    return r;
  };
  auto publish = [&](BcTok<DK> &b, const Reg &r) {
    if (tid < DK) {
      b.k[tid] = r.k;
      b.q[tid] = r.q;
      if (GATE == 2) b.a[tid] = __expf(r.la);
    }
    if (tid < kCW) {
      b.v[tid] = r.v;
      b.dO[tid] = r.dO;
    }
    if (tid == 0) {
      b.beta = r.beta;
      b.a_s = GATE == 1 ? __expf(r.la) : 1.f;
    }
  };
  auto decay = [&](const BcTok<DK> &b, int c) {
    return GATE == 2 ? b.a[c] : b.a_s;
  };
  // a stream of tokens tok(0), tok(1), ...: slot s % 3 holds tok(s)
  Reg nx;
  int par = 0;
  auto stream_begin = [&](int t_first, int t_second, bool grad) {
    nx = fetch(t_first, grad);
    __syncthreads();   // every reader of the slots is done
    publish(tv[0], nx);
    if (t_second >= 0) nx = fetch(t_second, grad);
    __syncthreads();
  };
  // before step s's barrier: publish tok(s+1), fetch tok(s+2)
  auto stream_advance = [&](int s, int t_next, int t_after, bool grad) {
    if (t_next >= 0) publish(tv[(s + 1) % 3], nx);
    if (t_after >= 0) nx = fetch(t_after, grad);
  };
  // column sums over the CTA's rows: over the 4 row lanes of a warp, then
  // over the warps' partials in shared memory (after the barrier)
  auto colsum_warp = [&](float4 &x) {
#pragma unroll
    for (int d = 8; d <= 16; d <<= 1) {
      x.x += __shfl_xor_sync(0xffffffffu, x.x, d);
      x.y += __shfl_xor_sync(0xffffffffu, x.y, d);
      x.z += __shfl_xor_sync(0xffffffffu, x.z, d);
      x.w += __shfl_xor_sync(0xffffffffu, x.w, d);
    }
  };
  auto colsum_cta = [&](int q) {
    float4 x = red[par][q][0][cq];
#pragma unroll
    for (int ww = 1; ww < NW; ++ww) x = add4(x, red[par][q][ww][cq]);
    return x;
  };

  float4 S[R];
  // forward token (stream step s, token vectors in slot s % 3); S~ saved
  // to `save` (thread-private layout) if given
  auto fwd_step = [&](int s, float *save, int t_next, int t_after) {
    const BcTok<DK> &b = tv[s % 3];
    float4 pr = f4(0.f);
#pragma unroll
    for (int i = 0; i < R; ++i) {
      const int c = row_c(i);
      const float a = decay(b, c);
      S[i] = make_float4(a * S[i].x, a * S[i].y, a * S[i].z, a * S[i].w);
      if (save) *tl(save, i) = S[i];
      pr = fma4(b.k[c], S[i], pr);
    }
    colsum_warp(pr);
    if (rl == 0) red[par][0][w][cq] = pr;
    stream_advance(s, t_next, t_after, false);
    __syncthreads();
    const float4 rk = colsum_cta(0);
    const float bb = b.beta;
    const float4 vv = *reinterpret_cast<const float4 *>(&b.v[4 * cq]);
    const float4 u = make_float4(bb * (vv.x - rk.x), bb * (vv.y - rk.y),
                                 bb * (vv.z - rk.z), bb * (vv.w - rk.w));
#pragma unroll
    for (int i = 0; i < R; ++i) S[i] = fma4(b.k[row_c(i)], u, S[i]);
    par ^= 1;
  };

  // ---- forward sweep: checkpoint before every window
#pragma unroll
  for (int i = 0; i < R; ++i)
    S[i] = p.s0 ? *reinterpret_cast<const float4 *>(p.s0 + sb +
                                                     (size_t)row_c(i) * dv + jc)
                : f4(0.f);
  if (L > 0) {
    stream_begin(0, L > 1 ? 1 : -1, false);
    for (int t = 0; t < L; ++t) {
      if (t % kBcWin == 0) {
#pragma unroll
        for (int i = 0; i < R; ++i) *tl(ckpt_of(t / kBcWin), i) = S[i];
      }
      fwd_step(t, nullptr, t + 1 < L ? t + 1 : -1, t + 2 < L ? t + 2 : -1);
    }
  }

  // ---- reverse sweep, window by window from the end
  float4 G[R];
#pragma unroll
  for (int i = 0; i < R; ++i)
    G[i] = p.dsT ? *reinterpret_cast<const float4 *>(p.dsT + sb +
                                                      (size_t)row_c(i) * dv + jc)
                 : f4(0.f);
  for (int win = nwin - 1; win >= 0; --win) {
    const int t0 = win * kBcWin, t1 = min(L, t0 + kBcWin), nt = t1 - t0;
    // replay the window from its checkpoint, keeping each token's S~
#pragma unroll
    for (int i = 0; i < R; ++i) S[i] = *tl(ckpt_of(win), i);
    stream_begin(t0, nt > 1 ? t0 + 1 : -1, false);
    for (int s = 0; s < nt; ++s)
      fwd_step(s, winb + (size_t)s * TILE, s + 1 < nt ? t0 + s + 1 : -1,
               s + 2 < nt ? t0 + s + 2 : -1);
    // reverse steps t1-1 .. t0 (stream step s = t1-1-t)
    stream_begin(t1 - 1, nt > 1 ? t1 - 2 : -1, true);
    for (int s = 0; s < nt; ++s) {
      const int t = t1 - 1 - s;
      const size_t row = row_of(t);
      const BcTok<DK> &b = tv[s % 3];
      // S~_t (L2-resident: written by the replay just above); the loads
      // are issued first and overlap the G update below
      float4 Sm[R];
#pragma unroll
      for (int i = 0; i < R; ++i) Sm[i] = *tl(winb + (size_t)(t - t0) * TILE, i);
      const float4 dO = *reinterpret_cast<const float4 *>(&b.dO[4 * cq]);
      // G += q dO^T; column partials of S~^T k and G^T k
      float4 pr = f4(0.f), pd = f4(0.f);
#pragma unroll
      for (int i = 0; i < R; ++i) {
        const int c = row_c(i);
        G[i] = fma4(b.q[c], dO, G[i]);
        pr = fma4(b.k[c], Sm[i], pr);
        pd = fma4(b.k[c], G[i], pd);
      }
      colsum_warp(pr);
      colsum_warp(pd);
      if (rl == 0) {
        red[par][0][w][cq] = pr;
        red[par][1][w][cq] = pd;
      }
      stream_advance(s, s + 1 < nt ? t - 1 : -1, s + 2 < nt ? t - 2 : -1,
                     true);
      __syncthreads();
      const float4 rk = colsum_cta(0);
      const float4 du = colsum_cta(1);
      par ^= 1;
      const float bb = b.beta;
      const float4 vv = *reinterpret_cast<const float4 *>(&b.v[4 * cq]);
      const float4 vr = make_float4(vv.x - rk.x, vv.y - rk.y, vv.z - rk.z,
                                    vv.w - rk.w);
      const float4 u = make_float4(bb * vr.x, bb * vr.y, bb * vr.z, bb * vr.w);
      // dv = beta du (this group's columns), dbeta partial = du . (v - r)
      if (w == 0 && rl == 0) {
        *reinterpret_cast<float4 *>(p.gv + row * dv + jc) =
            make_float4(bb * du.x, bb * du.y, bb * du.z, bb * du.w);
        float db = dot4(du, vr);
        db += __shfl_xor_sync(0xffu, db, 1);
        db += __shfl_xor_sync(0xffu, db, 2);
        db += __shfl_xor_sync(0xffu, db, 4);
        if (cq == 0) p.pb[(size_t)g * X + row] = db;
      }
      // per row c: dq = S_t dO, dk = G u - beta S~ du, dla = G~ . S~ over
      // this group's columns; then G = D G~
      // S_t dO = S~ dO + k (u . dO); G~ . S~ = G . S~ - beta k (S~ du)
      float qk[2 * R], dl[R];
      float dl_tot = 0.f;
      const float udo = dot4(u, dO);
#pragma unroll
      for (int i = 0; i < R; ++i) {
        const int c = row_c(i);
        const float kc = b.k[c], a = decay(b, c), sk = -bb * kc;
        const float sdu = dot4(Sm[i], du);
        qk[i] = fmaf(kc, udo, dot4(Sm[i], dO));
        qk[R + i] = fmaf(-bb, sdu, dot4(G[i], u));
        dl[i] = fmaf(sk, sdu, dot4(G[i], Sm[i]));
        dl_tot += dl[i];
        G[i] = make_float4(a * fmaf(sk, du.x, G[i].x), a * fmaf(sk, du.y, G[i].y),
                           a * fmaf(sk, du.z, G[i].z), a * fmaf(sk, du.w, G[i].w));
      }
      {
        const int base = xreduce8<2 * R>(qk, cq);
        constexpr int cnt = (2 * R) / 8 > 0 ? (2 * R) / 8 : 1;
        if ((cq & xreduce8_dup_mask<2 * R>()) == 0) {
#pragma unroll
          for (int e = 0; e < cnt; ++e) {
            const int idx = base + e;
            float *dst = idx < R ? p.pq : p.pk;
            dst[((size_t)g * X + row) * DK + row_c(idx % R)] = qk[e];
          }
        }
      }
      if (GATE == 2) {
        const int base = xreduce8<R>(dl, cq);
        constexpr int cnt = R / 8 > 0 ? R / 8 : 1;
        if ((cq & xreduce8_dup_mask<R>()) == 0) {
#pragma unroll
          for (int e = 0; e < cnt; ++e)
            p.pla[((size_t)g * X + row) * DK + row_c(base + e)] = dl[e];
        }
      } else if (GATE == 1) {
        // scalar gate: one partial per (group, warp)
        dl_tot = warp_sum(dl_tot);
        if (lane == 0) p.pla[((size_t)g * NW + w) * X + row] = dl_tot;
      }
    }
  }
  if (p.gs0) {
#pragma unroll
    for (int i = 0; i < R; ++i)
      *reinterpret_cast<float4 *>(p.gs0 + sb + (size_t)row_c(i) * dv + jc) =
          G[i];
  }
}

// gq, gk (and the channel gate's dlog_alpha) = sum over groups of the
// partials, [X][DK]; dbeta and the scalar gate's dlog_alpha, [X]
__global__ void gdr_bwd_reduce_kernel(const float *pq, const float *pk,
                                      const float *pla, const float *pb,
                                      float *gq, float *gk, float *gla,
                                      float *gbeta, long long X, int DK,
                                      int ng, int gate) {
  const long long nv = X * DK / 4;
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
       i < nv; i += stride) {
    float4 a = f4(0.f), b = f4(0.f), c = f4(0.f);
    for (int g = 0; g < ng; ++g) {
      a = add4(a, reinterpret_cast<const float4 *>(pq)[g * nv + i]);
      b = add4(b, reinterpret_cast<const float4 *>(pk)[g * nv + i]);
      if (gate == 2)
        c = add4(c, reinterpret_cast<const float4 *>(pla)[g * nv + i]);
    }
    reinterpret_cast<float4 *>(gq)[i] = a;
    reinterpret_cast<float4 *>(gk)[i] = b;
    if (gate == 2) reinterpret_cast<float4 *>(gla)[i] = c;
  }
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < X;
       i += stride) {
    float sb = 0.f, sl = 0.f;
    for (int g = 0; g < ng; ++g) sb += pb[g * X + i];
    gbeta[i] = sb;
    if (gate == 1) {
      for (int g = 0; g < kBcThreads / 32 * ng; ++g) sl += pla[g * X + i];
      gla[i] = sl;
    }
  }
}

template <int DK, typename T>
cudaError_t bc_launch_dk(const BcParams &bp, int gate, int nblocks,
                         cudaStream_t s) {
  switch (gate) {
    case 0: gdr_bwd_cols_kernel<DK, T, 0><<<nblocks, kBcThreads, 0, s>>>(bp); break;
    case 1: gdr_bwd_cols_kernel<DK, T, 1><<<nblocks, kBcThreads, 0, s>>>(bp); break;
    default: gdr_bwd_cols_kernel<DK, T, 2><<<nblocks, kBcThreads, 0, s>>>(bp); break;
  }
  return cudaGetLastError();
}

template <typename T>
cudaError_t bc_launch_t(const BcParams &bp, int dk, int gate, int nblocks,
                        cudaStream_t s) {
  switch (dk) {
    case 32: return bc_launch_dk<32, T>(bp, gate, nblocks, s);
    case 64: return bc_launch_dk<64, T>(bp, gate, nblocks, s);
    default: return bc_launch_dk<128, T>(bp, gate, nblocks, s);
  }
}

bool cols_path(const Problem &p) { return p.dk >= 32 && p.dv >= kCW; }

// float counts of the column-split scratch regions, each rounded up to 64
struct BcLayout {
  size_t ckpt, winb, pq, pk, pla, pb;
  size_t total() const { return ckpt + winb + pq + pk + pla + pb; }
};
size_t up64(size_t x) { return (x + 63) / 64 * 64; }
BcLayout bc_layout(const Problem &p, long long tw) {
  const size_t X = (size_t)p.ntok * p.H, ng = (size_t)(p.dv / kCW);
  const size_t nb = (size_t)p.nseq * p.H * ng;
  BcLayout l;
  l.ckpt = up64((size_t)p.H * tw * p.dk * p.dv);
  l.winb = up64(nb * kBcWin * p.dk * kCW);
  l.pq = up64(ng * X * p.dk);
  l.pk = l.pq;
  l.pla = p.gate == GDR_GATE_CHANNEL ? l.pq
          : p.gate == GDR_GATE_SCALAR ? up64(kBcThreads / 32 * ng * X) : 0;
  l.pb = up64(ng * X);
  return l;
}

}  // namespace

size_t backward_scratch_bytes(const Problem &p, long long *total_win) {
  if (cols_path(p)) {
    const long long tw =
        p.cu ? (long long)p.ntok / kBcWin + p.nseq
             : (long long)p.nseq * ((p.T + kBcWin - 1) / kBcWin);
    *total_win = tw;
    return bc_layout(p, tw).total() * sizeof(float);
  }
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
  if (cols_path(p)) {
    const BcLayout l = bc_layout(p, total_win);
    BcParams bc;
    bc.q = p.q;
    bc.k = p.k;
    bc.v = p.v;
    bc.dout = io.dout;
    bc.log_alpha = p.log_alpha;
    bc.beta = p.beta;
    bc.s0 = p.s0;
    bc.dsT = io.dsT;
    bc.gv = io.dv;
    bc.gs0 = io.ds0;
    bc.ckpt = scratch;
    bc.winb = bc.ckpt + l.ckpt;
    bc.pq = bc.winb + l.winb;
    bc.pk = bc.pq + l.pq;
    bc.pla = bc.pk + l.pk;
    bc.pb = bc.pla + l.pla;
    bc.cu = p.cu;
    bc.T = p.T;
    bc.ntok = p.ntok;
    bc.H = p.H;
    bc.dv = p.dv;
    bc.nseq = p.nseq;
    bc.ng = p.dv / kCW;
    bc.total_win = total_win;
    const int nb = p.nseq * p.H * bc.ng;
    cudaError_t e = p.dtype == GDR_BF16
                        ? bc_launch_t<__nv_bfloat16>(bc, p.dk, p.gate, nb, s)
                        : bc_launch_t<float>(bc, p.dk, p.gate, nb, s);
    if (e != cudaSuccess) return e;
    const long long X = (long long)p.ntok * p.H;
    if (X == 0) return cudaSuccess;
    const long long work = X * p.dk / 4;
    const int grid = (int)std::min<long long>((work + 255) / 256, 148 * 16);
    gdr_bwd_reduce_kernel<<<grid, 256, 0, s>>>(
        bc.pq, bc.pk, bc.pla, bc.pb, io.dq, io.dk, io.dla, io.dbeta, X, p.dk,
        bc.ng, p.gate == GDR_GATE_NONE ? 0 : p.gate == GDR_GATE_SCALAR ? 1 : 2);
    return cudaGetLastError();
  }
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
