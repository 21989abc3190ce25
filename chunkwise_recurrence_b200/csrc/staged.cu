// Staged path of libgdr: the chunkwise gated delta rule as four kernels with
// fp32 CUDA-core arithmetic and the intermediates in scratch memory.
//
//   (a) cumsum_kernel  : in-chunk cumulative log-decay g_r = sum_{s<=r} log a_s
//   (b) wy_kernel      : A = strictly-lower beta_r k_r^T Gamma_r Gamma_i^-1 k_i,
//                        T = (I + A)^-1 by forward substitution,
//                        W = T diag(beta) (K . e^g),  U = T diag(beta) V
//   (c) state_kernel   : sequential over the chunks of one (sequence, head,
//                        dv tile): V_new = U - W S_n,
//                        S_{n+1} = Gamma_C S_n + (K . e^{g_C - g})^T V_new
//   (d) output_kernel  : O = (Q . e^g) S_n + mask_{i<=r}[(Q . e^g)(K . e^-g)^T] V_new
//
// The gate variants change only which vectors enter these products.  Each
// token has a read key (the key the state is read with before the write), a
// write key (the key its correction is written along) and a target:
//   delta rule         : read k,      write k,      target v,     rows x beta
//   Gated DeltaNet-2   : read b . k,  write k,      target w . v
//   FG^2-GDN (+)       : read k,      write a . k,  target (c .) v
// A[r][i] pairs the read key of r with the write key of i, W is built from
// the read keys, U from the targets, and the state update and the
// intra-chunk output use the write keys.
//
// The chunkwise form rests on the update being affine in the preceding memory
// ("DeltaTTT: Layerwise Optimization for Nonlinear Recurrent Memory",
// §2 Background) and on the WY form with the decay folded into the erase
// factors (Gated DeltaNet-2 abstract, comparative-study page 2607.07953).
// Decay ratios exp(g_r - g_i) are always formed as one exponential of a
// difference with i <= r, so they never exceed 1 for log-decays <= 0.
//
// This path serves every supported shape and both dtypes; it is the fp32
// path (tensor-core TF32 cannot hold a 1e-4 relative error) and the reference
// layout for the fused tensor-core kernel.

#include <cuda_bf16.h>

#include "gdr_internal.h"

namespace gdr {
namespace {

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) {
  return __bfloat162float(x);
}
template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) {
  return x;
}
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Builds the chunk table from the sequence boundaries.  Boundaries are
// clamped to [previous end, ntok] so that the table never exceeds
// ntok / C + nseq entries, whatever the device-side contents of cu.
__global__ void chunk_table_kernel(const int32_t *cu, int nseq, int T,
                                   int ntok, int C, ChunkInfo *table,
                                   int *seq_first) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  int j = 0, prev_end = 0;
  for (int n = 0; n < nseq; ++n) {
    int s0 = cu ? cu[n] : n * T;
    int e0 = cu ? cu[n + 1] : (n + 1) * T;
    s0 = min(max(s0, prev_end), ntok);
    e0 = min(max(e0, s0), ntok);
    prev_end = e0;
    seq_first[n] = j;
    for (int s = s0; s < e0; s += C) {
      ChunkInfo ci;
      ci.tok0 = s;
      ci.len = min(C, e0 - s);
      ci.seq = n;
      ci.pad = 0;
      table[j++] = ci;
    }
  }
  seq_first[nseq] = j;
}

// (a) segmented cumulative log-decay, restarting at every chunk start.
__global__ void cumsum_kernel(const float *__restrict__ log_alpha,
                              float *__restrict__ g,
                              const ChunkInfo *__restrict__ table,
                              const int *__restrict__ nchunks, int H,
                              int gdim) {
  const int j = blockIdx.x, h = blockIdx.y;
  if (j >= *nchunks) return;
  const ChunkInfo ci = table[j];
  for (int c = threadIdx.x; c < gdim; c += blockDim.x) {
    float acc = 0.f;
    for (int r = 0; r < ci.len; ++r) {
      const size_t idx = ((size_t)(ci.tok0 + r) * H + h) * gdim + c;
      acc += log_alpha[idx];
      g[idx] = acc;
    }
  }
}

// Cumulative log-decay of row r, channel c (0 when there is no gate).
__device__ __forceinline__ float gval(const float *Gs, int gdim, int r,
                                      int c) {
  if (gdim == 0) return 0.f;
  return gdim == 1 ? Gs[r] : Gs[r * gdim + c];
}

// (b) intra-chunk WY/UT transform of one (chunk, head).
// With the Gated DeltaNet-2 gates (erase != nullptr), the read key of token
// r is b_r . k_r (erase gate b_r, per key channel) and its target w_r . v_r
// (write gate w_r, per value channel), and beta is not used:
//   A[r][i] = (b_r . k_r)^T Gamma_r Gamma_i^-1 k_i,  W = T ((B . K) . e^g),
//   U = T (Wg . V).
// With FG^2-GDN's rate (wkey != nullptr) the write key of token i is
// a_i . k_i and the target (c_r .) v_r, with write = c or nullptr:
//   A[r][i] = k_r^T Gamma_r Gamma_i^-1 (a_i . k_i),  W = T (K . e^g),
//   U = T ((C .) V).
// Shared memory: the key rows are padded to dk + 1 floats so that the A
// products, whose lanes walk rows, read distinct banks; the factors of W and
// U (beta_i (read key) e^{g_i} and beta_i (target)) are formed once per
// chunk, not once per (row, column) of the product.
template <typename Tin>
__global__ void wy_kernel(const Tin *__restrict__ k, const Tin *__restrict__ v,
                          const float *__restrict__ beta,
                          const float *__restrict__ erase,
                          const float *__restrict__ write,
                          const float *__restrict__ wkey,
                          const float *__restrict__ g, float *__restrict__ W,
                          float *__restrict__ U,
                          const ChunkInfo *__restrict__ table,
                          const int *__restrict__ nchunks, int H, int dk,
                          int dv, int C, int gdim) {
  const int j = blockIdx.x, h = blockIdx.y;
  if (j >= *nchunks) return;
  const ChunkInfo ci = table[j];
  const int L = ci.len;
  const int gd = gdim == 0 ? 1 : gdim;
  const int dkp = dk + 1;
  const bool g2 = erase != nullptr;
  // a read key that differs from the write key needs a tile of its own
  const bool split = g2 || wkey != nullptr;
  extern __shared__ __align__(16) float sm[];
  float *Ks = sm;                  // [C][dkp], the write keys
  float *Gs = Ks + C * dkp;        // [C][gd]
  float *As = Gs + C * gd;         // [C][C+1]
  float *Ts = As + C * (C + 1);    // [C][C+1]
  float *bs = Ts + C * (C + 1);    // [C]
  float *Vs = bs + C;              // [C][dv], the targets (times beta_i)
  float *Es = Vs + C * dv;         // [C][dkp], the read keys when split
  // the read keys: b_r . k_r (Gated DeltaNet-2), k_r (FG^2-GDN; the write
  // keys are then a_r . k_r) or the write keys themselves; the row factor
  // bs[r] is beta_r for the delta rule and 1 otherwise
  float *Rs = split ? Es : Ks;
  const int tid = threadIdx.x, nt = blockDim.x;

  for (int idx = tid; idx < L * dk; idx += nt) {
    const int r = idx / dk, c = idx % dk;
    const size_t off = ((size_t)(ci.tok0 + r) * H + h) * dk + c;
    const float kv = to_f(k[off]);
    Ks[r * dkp + c] = wkey ? wkey[off] * kv : kv;
    if (split) Es[r * dkp + c] = g2 ? erase[off] * kv : kv;
  }
  if (gdim)
    for (int idx = tid; idx < L * gdim; idx += nt) {
      const int r = idx / gdim, c = idx % gdim;
      Gs[r * gdim + c] = g[((size_t)(ci.tok0 + r) * H + h) * gdim + c];
    }
  for (int r = tid; r < L; r += nt)
    bs[r] = split ? 1.f : beta[(size_t)(ci.tok0 + r) * H + h];
  __syncthreads();
  for (int idx = tid; idx < L * dv; idx += nt) {
    const int r = idx / dv, c = idx % dv;
    const size_t e = ((size_t)(ci.tok0 + r) * H + h) * dv + c;
    Vs[r * dv + c] = bs[r] * (write ? write[e] * to_f(v[e]) : to_f(v[e]));
  }

  // A[r][i] = beta_r sum_c rk_r[c] wk_i[c] exp(g_r[c] - g_i[c]),  i < r
  for (int idx = tid; idx < L * L; idx += nt) {
    const int r = idx / L, i = idx % L;
    float a = 0.f;
    if (i < r) {
      const float *rr = Rs + r * dkp, *ki = Ks + i * dkp;
      if (gdim <= 1) {
        for (int c = 0; c < dk; ++c) a += rr[c] * ki[c];
        if (gdim == 1) a *= __expf(Gs[r] - Gs[i]);
      } else {
        const float *gr = Gs + r * gdim, *gi = Gs + i * gdim;
        for (int c = 0; c < dk; ++c)
          a += rr[c] * ki[c] * __expf(gr[c] - gi[c]);
      }
      a *= bs[r];
    }
    As[r * (C + 1) + i] = a;
    Ts[r * (C + 1) + i] = (r == i) ? 1.f : 0.f;
  }
  __syncthreads();

  // the factor of W, in place of the read keys (A no longer needs them):
  // X[i][c] = beta_i rk_i[c] e^{g_i[c]}
  for (int idx = tid; idx < L * dk; idx += nt) {
    const int i = idx / dk, c = idx % dk;
    Rs[i * dkp + c] = bs[i] * Rs[i * dkp + c] * __expf(gval(Gs, gdim, i, c));
  }

  // T = (I + A)^-1, row by row: T[r][j] = -sum_{j<=i<r} A[r][i] T[i][j]
  for (int r = 1; r < L; ++r) {
    for (int jj = tid; jj < r; jj += nt) {
      float acc = 0.f;
      for (int i = jj; i < r; ++i) acc += As[r * (C + 1) + i] * Ts[i * (C + 1) + jj];
      Ts[r * (C + 1) + jj] = -acc;
    }
    __syncthreads();
  }
  if (L <= 1) __syncthreads();   // the X and Vs writes before their reads

  // W = T X,  U = T Vs
  for (int idx = tid; idx < L * dk; idx += nt) {
    const int r = idx / dk, c = idx % dk;
    const float *tr = Ts + r * (C + 1);
    float acc = 0.f;
    for (int i = 0; i <= r; ++i) acc += tr[i] * Rs[i * dkp + c];
    W[((size_t)(ci.tok0 + r) * H + h) * dk + c] = acc;
  }
  for (int idx = tid; idx < L * dv; idx += nt) {
    const int r = idx / dv, c = idx % dv;
    const float *tr = Ts + r * (C + 1);
    float acc = 0.f;
    for (int i = 0; i <= r; ++i) acc += tr[i] * Vs[i * dv + c];
    U[((size_t)(ci.tok0 + r) * H + h) * dv + c] = acc;
  }
}

// (c) sequential state passing for one (sequence, head, dv tile).
// Per chunk the rows k_r . e^{g_C - g_r} are formed once in shared memory
// (one exponential per row and channel) before the state update reads them.
template <typename Tin>
__global__ void state_kernel(const Tin *__restrict__ k,
                             const float *__restrict__ wkey,
                             const float *__restrict__ g,
                             const float *__restrict__ W,
                             const float *__restrict__ U,
                             const float *__restrict__ s0,
                             float *__restrict__ sT, float *__restrict__ Sbuf,
                             float *__restrict__ Vn,
                             const ChunkInfo *__restrict__ table,
                             const int *__restrict__ seq_first, int H, int dk,
                             int dv, int C, int gdim, int DVT) {
  const int n = blockIdx.x, h = blockIdx.y, j0 = blockIdx.z * DVT;
  extern __shared__ __align__(16) float sm[];
  float *S = sm;              // [dk][DVT]
  float *V = S + dk * DVT;    // [C][DVT]
  float *gl = V + C * DVT;    // [dk]
  float *Kt = gl + dk;        // [C][dk], (write key)_r . e^{g_C - g_r}
  const int tid = threadIdx.x, nt = blockDim.x;
  const size_t sbase = ((size_t)n * H + h) * dk * dv;

  for (int idx = tid; idx < dk * DVT; idx += nt) {
    const int c = idx / DVT, jj = idx % DVT;
    S[idx] = s0 ? s0[sbase + (size_t)c * dv + j0 + jj] : 0.f;
  }
  __syncthreads();

  const int jb = seq_first[n], je = seq_first[n + 1];
  for (int j = jb; j < je; ++j) {
    const ChunkInfo ci = table[j];
    const int L = ci.len;
    float *Sn = Sbuf + ((size_t)j * H + h) * dk * dv;
    for (int idx = tid; idx < dk * DVT; idx += nt) {
      const int c = idx / DVT, jj = idx % DVT;
      Sn[(size_t)c * dv + j0 + jj] = S[idx];
    }
    // V_new = U - W S
    for (int idx = tid; idx < L * DVT; idx += nt) {
      const int r = idx / DVT, jj = idx % DVT;
      const size_t row = (size_t)(ci.tok0 + r) * H + h;
      float acc = U[row * dv + j0 + jj];
      for (int c = 0; c < dk; ++c) acc -= W[row * dk + c] * S[c * DVT + jj];
      V[r * DVT + jj] = acc;
      Vn[row * dv + j0 + jj] = acc;
    }
    for (int c = tid; c < dk; c += nt)
      gl[c] = gdim == 0 ? 0.f
                        : g[((size_t)(ci.tok0 + L - 1) * H + h) * gdim +
                            (gdim == 1 ? 0 : c)];
    __syncthreads();
    for (int idx = tid; idx < L * dk; idx += nt) {
      const int r = idx / dk, c = idx % dk;
      const size_t row = (size_t)(ci.tok0 + r) * H + h;
      const float gr = gdim == 0 ? 0.f : g[row * gdim + (gdim == 1 ? 0 : c)];
      const float kw = to_f(k[row * dk + c]) * (wkey ? wkey[row * dk + c] : 1.f);
      Kt[idx] = kw * __expf(gl[c] - gr);
    }
    __syncthreads();
    // S <- Gamma_C S + (K . e^{g_C - g})^T V_new
    for (int idx = tid; idx < dk * DVT; idx += nt) {
      const int c = idx / DVT, jj = idx % DVT;
      float acc = __expf(gl[c]) * S[idx];
      for (int r = 0; r < L; ++r) acc += Kt[r * dk + c] * V[r * DVT + jj];
      S[idx] = acc;
    }
    __syncthreads();
  }
  if (sT)
    for (int idx = tid; idx < dk * DVT; idx += nt) {
      const int c = idx / DVT, jj = idx % DVT;
      sT[sbase + (size_t)c * dv + j0 + jj] = S[idx];
    }
}

// (d) chunk output for one (chunk, head).  After the masked products P, the
// rows of Q are scaled in place to Q . e^g; each thread then owns one value
// column and blocks of kOutRows rows, so that a state element read from
// memory serves kOutRows outputs.
constexpr int kOutRows = 8;

template <typename Tin>
__global__ void output_kernel(const Tin *__restrict__ q,
                              const Tin *__restrict__ k,
                              const float *__restrict__ wkey,
                              const float *__restrict__ g,
                              const float *__restrict__ Sbuf,
                              const float *__restrict__ Vn,
                              Tin *__restrict__ out,
                              const ChunkInfo *__restrict__ table,
                              const int *__restrict__ nchunks, int H, int dk,
                              int dv, int C, int gdim) {
  const int j = blockIdx.x, h = blockIdx.y;
  if (j >= *nchunks) return;
  const ChunkInfo ci = table[j];
  const int L = ci.len;
  const int gd = gdim == 0 ? 1 : gdim;
  const int dkp = dk + 1;
  extern __shared__ __align__(16) float sm[];
  float *Qs = sm;               // [C][dk]
  float *Ks = Qs + C * dk;      // [C][dkp], the write keys
  float *Gs = Ks + C * dkp;     // [C][gd]
  float *Ps = Gs + C * gd;      // [C][C+1]
  const int tid = threadIdx.x, nt = blockDim.x;
  for (int idx = tid; idx < L * dk; idx += nt) {
    const int r = idx / dk, c = idx % dk;
    const size_t off = ((size_t)(ci.tok0 + r) * H + h) * dk + c;
    Qs[r * dk + c] = to_f(q[off]);
    Ks[r * dkp + c] = to_f(k[off]) * (wkey ? wkey[off] : 1.f);
  }
  if (gdim)
    for (int idx = tid; idx < L * gdim; idx += nt) {
      const int r = idx / gdim, c = idx % gdim;
      Gs[r * gdim + c] = g[((size_t)(ci.tok0 + r) * H + h) * gdim + c];
    }
  __syncthreads();
  // P[r][i] = sum_c q_r[c] k_i[c] exp(g_r[c] - g_i[c]),  i <= r
  for (int idx = tid; idx < L * L; idx += nt) {
    const int r = idx / L, i = idx % L;
    float a = 0.f;
    if (i <= r) {
      const float *qr = Qs + r * dk, *ki = Ks + i * dkp;
      if (gdim <= 1) {
        for (int c = 0; c < dk; ++c) a += qr[c] * ki[c];
        if (gdim == 1) a *= __expf(Gs[r] - Gs[i]);
      } else {
        const float *gr = Gs + r * gdim, *gi = Gs + i * gdim;
        for (int c = 0; c < dk; ++c)
          a += qr[c] * ki[c] * __expf(gr[c] - gi[c]);
      }
    }
    Ps[r * (C + 1) + i] = a;
  }
  __syncthreads();
  for (int idx = tid; idx < L * dk; idx += nt) {
    const int r = idx / dk, c = idx % dk;
    Qs[idx] = Qs[idx] * __expf(gval(Gs, gdim, r, c));
  }
  __syncthreads();
  const float *Sn = Sbuf + ((size_t)j * H + h) * dk * dv;
  const int groups = nt / dv;   // dv divides the block size
  const int c = tid % dv;
  for (int r0 = (tid / dv) * kOutRows; r0 < L; r0 += groups * kOutRows) {
    // rows r0 .. r0 + kOutRows - 1 lie inside the C-row tiles (C is a
    // multiple of kOutRows); rows >= L hold stale values and are not stored
    float acc[kOutRows];
#pragma unroll
    for (int i = 0; i < kOutRows; ++i) acc[i] = 0.f;
    for (int e = 0; e < dk; e += 4) {
      const float s0 = Sn[(size_t)e * dv + c];
      const float s1 = Sn[(size_t)(e + 1) * dv + c];
      const float s2 = Sn[(size_t)(e + 2) * dv + c];
      const float s3 = Sn[(size_t)(e + 3) * dv + c];
#pragma unroll
      for (int i = 0; i < kOutRows; ++i) {
        const float4 qv =
            *reinterpret_cast<const float4 *>(Qs + (r0 + i) * dk + e);
        acc[i] += qv.x * s0;
        acc[i] += qv.y * s1;
        acc[i] += qv.z * s2;
        acc[i] += qv.w * s3;
      }
    }
    const int iend = min(L, r0 + kOutRows);
    for (int i2 = 0; i2 < iend; ++i2) {
      const float vn = Vn[((size_t)(ci.tok0 + i2) * H + h) * dv + c];
#pragma unroll
      for (int i = 0; i < kOutRows; ++i)
        if (i2 <= r0 + i) acc[i] += Ps[(r0 + i) * (C + 1) + i2] * vn;
    }
#pragma unroll
    for (int i = 0; i < kOutRows; ++i)
      if (r0 + i < L)
        out[((size_t)(ci.tok0 + r0 + i) * H + h) * dv + c] =
            from_f<Tin>(acc[i]);
  }
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct StagedLayout {
  size_t table, seq_first, g, W, U, Vn, Sbuf, total;
};

StagedLayout layout(const Problem &p) {
  const int gdim = p.gate == GDR_GATE_NONE ? 0
                   : p.gate == GDR_GATE_SCALAR ? 1
                                               : p.dk;
  const size_t th = (size_t)p.ntok * p.H;
  StagedLayout L;
  size_t o = 0;
  L.table = o;     o += align256(sizeof(ChunkInfo) * (size_t)p.max_chunks);
  L.seq_first = o; o += align256(sizeof(int) * ((size_t)p.nseq + 1));
  L.g = o;         o += align256(sizeof(float) * th * (size_t)gdim);
  L.W = o;         o += align256(sizeof(float) * th * p.dk);
  L.U = o;         o += align256(sizeof(float) * th * p.dv);
  L.Vn = o;        o += align256(sizeof(float) * th * p.dv);
  L.Sbuf = o;
  o += align256(sizeof(float) * (size_t)p.max_chunks * p.H * p.dk * p.dv);
  L.total = o;
  return L;
}

template <typename Tin>
cudaError_t run_typed(const Problem &p, char *ws, cudaStream_t s) {
  const StagedLayout L = layout(p);
  const int gdim = p.gate == GDR_GATE_NONE ? 0
                   : p.gate == GDR_GATE_SCALAR ? 1
                                               : p.dk;
  const int gd = gdim == 0 ? 1 : gdim;
  const int C = p.chunk;
  ChunkInfo *table = reinterpret_cast<ChunkInfo *>(ws + L.table);
  int *seq_first = reinterpret_cast<int *>(ws + L.seq_first);
  int *nchunks = seq_first + p.nseq;
  float *g = gdim ? reinterpret_cast<float *>(ws + L.g) : nullptr;
  float *W = reinterpret_cast<float *>(ws + L.W);
  float *U = reinterpret_cast<float *>(ws + L.U);
  float *Vn = reinterpret_cast<float *>(ws + L.Vn);
  float *Sbuf = reinterpret_cast<float *>(ws + L.Sbuf);
  const Tin *q = static_cast<const Tin *>(p.q);
  const Tin *k = static_cast<const Tin *>(p.k);
  const Tin *v = static_cast<const Tin *>(p.v);
  Tin *out = static_cast<Tin *>(p.out);

  chunk_table_kernel<<<1, 32, 0, s>>>(p.cu, p.nseq, p.T, p.ntok, C, table,
                                      seq_first);
  if (p.max_chunks > 0) {
    const dim3 grid(p.max_chunks, p.H);
    if (gdim)
      cumsum_kernel<<<grid, 128, 0, s>>>(p.log_alpha, g, table, nchunks, p.H,
                                         gdim);
    const size_t dkp = (size_t)p.dk + 1;
    const size_t wy_smem =
        sizeof(float) * ((size_t)C * dkp + (size_t)C * gd +
                         2 * (size_t)C * (C + 1) + C + (size_t)C * p.dv +
                         ((p.erase || p.wkey) ? (size_t)C * dkp : 0));
    cudaError_t e = cudaFuncSetAttribute(
        wy_kernel<Tin>, cudaFuncAttributeMaxDynamicSharedMemorySize,
        (int)wy_smem);
    if (e != cudaSuccess) return e;
    wy_kernel<Tin><<<grid, 256, wy_smem, s>>>(k, v, p.beta, p.erase, p.write,
                                             p.wkey, g, W, U, table, nchunks,
                                             p.H, p.dk, p.dv, C, gdim);
  }
  const int DVT = p.dv < 64 ? p.dv : 64;
  const size_t st_smem =
      sizeof(float) * ((size_t)p.dk * DVT + (size_t)C * DVT + p.dk +
                       (size_t)C * p.dk);
  {
    cudaError_t e = cudaFuncSetAttribute(
        state_kernel<Tin>, cudaFuncAttributeMaxDynamicSharedMemorySize,
        (int)st_smem);
    if (e != cudaSuccess) return e;
  }
  state_kernel<Tin><<<dim3(p.nseq, p.H, p.dv / DVT), 256, st_smem, s>>>(
      k, p.wkey, g, W, U, p.s0, p.sT, Sbuf, Vn, table, seq_first, p.H, p.dk,
      p.dv, C, gdim, DVT);
  if (p.max_chunks > 0) {
    const size_t o_smem =
        sizeof(float) * ((size_t)C * p.dk + (size_t)C * (p.dk + 1) +
                         (size_t)C * gd + (size_t)C * (C + 1));
    cudaError_t e = cudaFuncSetAttribute(
        output_kernel<Tin>, cudaFuncAttributeMaxDynamicSharedMemorySize,
        (int)o_smem);
    if (e != cudaSuccess) return e;
    output_kernel<Tin><<<dim3(p.max_chunks, p.H), 256, o_smem, s>>>(
        q, k, p.wkey, g, Sbuf, Vn, out, table, nchunks, p.H, p.dk, p.dv, C,
        gdim);
  }
  return cudaGetLastError();
}

}  // namespace

size_t staged_workspace_bytes(const Problem &p) { return layout(p).total; }

StagedBufs staged_bufs(const Problem &p, void *workspace) {
  char *ws = static_cast<char *>(workspace);
  const StagedLayout L = layout(p);
  StagedBufs b;
  b.table = reinterpret_cast<ChunkInfo *>(ws + L.table);
  b.seq_first = reinterpret_cast<int *>(ws + L.seq_first);
  b.nchunks = b.seq_first + p.nseq;
  b.g = reinterpret_cast<float *>(ws + L.g);
  b.W = reinterpret_cast<float *>(ws + L.W);
  b.U = reinterpret_cast<float *>(ws + L.U);
  b.Vn = reinterpret_cast<float *>(ws + L.Vn);
  b.Sbuf = reinterpret_cast<float *>(ws + L.Sbuf);
  return b;
}

cudaError_t staged_chunks_run(const Problem &p, void *workspace,
                              cudaStream_t s) {
  const StagedBufs b = staged_bufs(p, workspace);
  const int gdim = p.gate == GDR_GATE_NONE ? 0
                   : p.gate == GDR_GATE_SCALAR ? 1
                                               : p.dk;
  chunk_table_kernel<<<1, 32, 0, s>>>(p.cu, p.nseq, p.T, p.ntok, p.chunk,
                                      b.table, b.seq_first);
  if (gdim && p.max_chunks > 0)
    cumsum_kernel<<<dim3(p.max_chunks, p.H), 128, 0, s>>>(
        p.log_alpha, b.g, b.table, b.nchunks, p.H, gdim);
  return cudaGetLastError();
}

cudaError_t staged_run(const Problem &p, void *workspace, cudaStream_t s) {
  char *ws = static_cast<char *>(workspace);
  if (p.dtype == GDR_FP32) return run_typed<float>(p, ws, s);
  return run_typed<__nv_bfloat16>(p, ws, s);
}

}  // namespace gdr
