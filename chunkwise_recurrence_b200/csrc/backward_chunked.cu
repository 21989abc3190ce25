// Chunked backward pass of the gated delta rule: the gradients of the
// chunkwise forward (its WY form, chunk by chunk) taken product by product,
// in fp32 on CUDA cores.
//
// Per chunk (C = 64 tokens, rows past the sequence end zero), with S the
// state at the chunk start, Lambda = dL/dS at the chunk end, g the in-chunk
// cumulative log-decay, Gamma-weights e^{g_r - g_i}:
//   forward   A = strict-lower(beta_r k_r^T Gamma k_i),  T = (I + A)^-1,
//             Y = V - (K . e^g) S,  V_new = T diag(beta) Y,
//             O = (Q . e^g) S + P V_new,  P = lower(q_r^T Gamma k_i),
//             S' = e^{g_C} S + (K . e^{g_C - g})^T V_new
//   reverse   dV_new = (K . e^{g_C - g}) Lambda + P^T dO
//             dL/dS = e^{g_C} Lambda + (Q . e^g)^T dO
//                     - (K . e^g)^T diag(beta) T^T dV_new
//   gradients Z = T^T dV_new,  dv = beta . Z,  dbeta += rowsum(Z . Y),
//             dT = dV_new (beta . Y)^T,  dA = -T^T dT T^T (strictly lower),
//             dP = lower(dO V_new^T),  and the key, query and decay
//             gradients of A, P and of the factors e^g, e^{g_C - g}.
// The update is affine in the preceding memory ("DeltaTTT: Layerwise
// Optimization for Nonlinear Recurrent Memory", §2 Background), which is
// what makes the chunk-level scans below exact; the WY form with the decay in
// the erase factors is the one the Gated DeltaNet-2 abstract (comparative-
// study page 2607.07953) names.
//
// Kernels (per call): the staged path's chunk table and cumsum, then
//   bw_wy_kernel     per (chunk, head), in parallel: A, P, T = (I + A)^-1,
//                    W and U;
//   bw_prep_kernel   per (chunk, head), in parallel: the chunk's state map
//                    S' = Cm S + Dm and the adjoint's input Bm;
//   bw_scan_kernel   per (sequence, head): the chunk-start states (forward),
//                    then dL/dS at every chunk end and dL/dS_0 (reverse, on
//                    the transposed maps), one dk x dk x dv product a chunk;
//   bw_vn_kernel     per (chunk, head, 64 value columns), in parallel: V_new
//                    and dV_new from those states;
//   bw_grad_kernel   per (chunk, head), in parallel: every input gradient of
//                    the chunk from S, Lambda, V_new and dV_new.
// The products run on the tensor cores over shared-memory tiles (gemm_tc).

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "gdr_internal.h"

namespace gdr {
namespace {

constexpr int kBC = 64;      // chunk length
constexpr int kNT = 512;     // threads per CTA
constexpr int kSl = 16;      // key rows per slice in bw_grad_kernel
// shared-memory row strides: d-wide rows (d <= 128) and C-wide rows, each
// 4 (mod 32) floats, so that an MMA fragment's 8 rows x 4 columns fall in 32
// distinct banks (and its 4 rows x 8 columns, the transposed walk, in at
// most two per bank)
constexpr int kP = 132, kCP = kBC + 4;
// largest in-chunk spread |g - g_ref| of a channel-wise decay for which the
// gradient kernel factors e^{g_r - g_i} as e^{g_r - g_ref} e^{g_ref - g_i}
// (both stay far inside fp32 for normalised keys); wider chunks take one
// exponential per element
constexpr float kFactRange = 60.f;

__device__ __forceinline__ float ldf(const float *p) { return *p; }
__device__ __forceinline__ float ldf(const __nv_bfloat16 *p) {
  return __bfloat162float(*p);
}

// ---- products on the tensor cores: mma.sync m16n8k8 tf32 with each fp32
// operand split into a tf32 high part and the (tf32-truncated) remainder,
// C += A_hi B_lo + A_lo B_hi + A_hi B_hi.  The dropped
// A_lo B_lo and the truncation of the remainders leave a relative error near
// 2^-21 per product, fp32-like; one tf32 product alone would leave 2^-11.
__device__ __forceinline__ void tf32_split(float x, uint32_t &hi,
                                           uint32_t &lo) {
  const uint32_t h = __float_as_uint(x) & 0xffffe000u;
  hi = h;
  lo = __float_as_uint(x - __uint_as_float(h));
}

__device__ __forceinline__ void mma_tf32(float (&c)[4], const uint32_t (&a)[4],
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// The split-tf32 fragments of A rows m0 + g, m0 + g + 8 and columns k0 + t,
// k0 + t + 4 (g = lane / 4, t = lane % 4: the m16n8k8 A layout).
template <class FA>
__device__ __forceinline__ void load_a(FA A, int m0, int k0, int g, int t,
                                       uint32_t (&ah)[4], uint32_t (&al)[4]) {
  tf32_split(A(m0 + g, k0 + t), ah[0], al[0]);
  tf32_split(A(m0 + g + 8, k0 + t), ah[1], al[1]);
  tf32_split(A(m0 + g, k0 + t + 4), ah[2], al[2]);
  tf32_split(A(m0 + g + 8, k0 + t + 4), ah[3], al[3]);
}

// out(m, n, value) for every element of the M x N product sum_k A(m, k)
// B(k, n), M a multiple of 16, N of 8, K of 8: warp w takes the blocks of
// 16 rows x 8 NT columns w, w + 8, ... (A's fragment is loaded once per
// block row and k step and reused over the NT column tiles).
template <int NT, class FA, class FB, class FO>
__device__ __forceinline__ void gemm_tc(int M, int N, int K, FA A, FB B,
                                        FO out) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int nb = N / (8 * NT), total = (M / 16) * nb;
  for (int blk = warp; blk < total; blk += kNT / 32) {
    const int m0 = (blk / nb) * 16, n0 = (blk % nb) * 8 * NT;
    // the main products and the two correction products in accumulators of
    // their own, so that consecutive MMAs do not wait on one another
    float c[NT][4], e[NT][4];
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int x = 0; x < 4; ++x) c[j][x] = e[j][x] = 0.f;
    for (int k0 = 0; k0 < K; k0 += 8) {
      uint32_t ah[4], al[4], bh[NT][2], bl[NT][2];
      load_a(A, m0, k0, g, t, ah, al);
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        tf32_split(B(k0 + t, n0 + 8 * j + g), bh[j][0], bl[j][0]);
        tf32_split(B(k0 + t + 4, n0 + 8 * j + g), bh[j][1], bl[j][1]);
      }
#pragma unroll
      for (int j = 0; j < NT; ++j) mma_tf32(c[j], ah, bh[j][0], bh[j][1]);
#pragma unroll
      for (int j = 0; j < NT; ++j) mma_tf32(e[j], al, bh[j][0], bh[j][1]);
#pragma unroll
      for (int j = 0; j < NT; ++j) mma_tf32(e[j], ah, bl[j][0], bl[j][1]);
    }
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      const int n = n0 + 8 * j + 2 * t;
      out(m0 + g, n, c[j][0] + e[j][0]);
      out(m0 + g, n + 1, c[j][1] + e[j][1]);
      out(m0 + g + 8, n, c[j][2] + e[j][2]);
      out(m0 + g + 8, n + 1, c[j][3] + e[j][3]);
    }
  }
}

// Four products over the same M x N x K shape, each of its own A and B,
// handed to out(m, n, v1, v2, v3, v4) together (one output mapping for all).
template <int NT, class FA1, class FB1, class FA2, class FB2, class FA3,
          class FB3, class FA4, class FB4, class FO>
__device__ __forceinline__ void gemm_tc4(int M, int N, int K, FA1 A1, FB1 B1,
                                         FA2 A2, FB2 B2, FA3 A3, FB3 B3,
                                         FA4 A4, FB4 B4, FO out) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int nb = N / (8 * NT), total = (M / 16) * nb;
  for (int blk = warp; blk < total; blk += kNT / 32) {
    const int m0 = (blk / nb) * 16, n0 = (blk % nb) * 8 * NT;
    float c[4][NT][4];
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
      for (int j = 0; j < NT; ++j)
        c[p][j][0] = c[p][j][1] = c[p][j][2] = c[p][j][3] = 0.f;
    for (int k0 = 0; k0 < K; k0 += 8) {
      auto step = [&](int p, auto A, auto B) {
        uint32_t ah[4], al[4];
        load_a(A, m0, k0, g, t, ah, al);
#pragma unroll
        for (int j = 0; j < NT; ++j) {
          uint32_t bh0, bl0, bh1, bl1;
          tf32_split(B(k0 + t, n0 + 8 * j + g), bh0, bl0);
          tf32_split(B(k0 + t + 4, n0 + 8 * j + g), bh1, bl1);
          mma_tf32(c[p][j], al, bh0, bh1);
          mma_tf32(c[p][j], ah, bl0, bl1);
          mma_tf32(c[p][j], ah, bh0, bh1);
        }
      };
      step(0, A1, B1);
      step(1, A2, B2);
      step(2, A3, B3);
      step(3, A4, B4);
    }
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      const int n = n0 + 8 * j + 2 * t;
#pragma unroll
      for (int e = 0; e < 4; ++e)
        out(m0 + g + (e >> 1) * 8, n + (e & 1), c[0][j][e], c[1][j][e],
            c[2][j][e], c[3][j][e]);
    }
  }
}

// gemm_tc with the widest column block that divides N (N is a runtime
// multiple of 8)
// (but narrower when that leaves warps without a block: the products here
// are latency-bound, and a block per warp matters more than fragment reuse)
template <class FA, class FB, class FO>
__device__ __forceinline__ void gemm_tcn(int M, int N, int K, FA A, FB B,
                                         FO out) {
  const int rows = M / 16, warps = kNT / 32;
  if (N % 32 == 0 && rows * (N / 32) >= warps) gemm_tc<4>(M, N, K, A, B, out);
  else if (N % 16 == 0 && rows * (N / 16) >= warps)
    gemm_tc<2>(M, N, K, A, B, out);
  else gemm_tc<1>(M, N, K, A, B, out);
}

__device__ __forceinline__ float block_max(float x, float *red) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1)
    x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, off));
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = x;
  __syncthreads();
  float r = red[0];
  for (int w = 1; w < kNT / 32; ++w) r = fmaxf(r, red[w]);
  __syncthreads();
  return r;
}

// g of token row r (< L) and key channel c; 0 without a gate
__device__ __forceinline__ float gv(const float *g, int gdim, size_t row,
                                    int c) {
  return gdim == 0 ? 0.f : g[row * gdim + (gdim == 1 ? 0 : c)];
}

// ---------------------------------------------------------------------------
// T = (I + A)^-1 for the strictly lower 64 x 64 A (rows kCP floats apart), in
// fp32, by 16 x 16 blocks: the diagonal blocks D_b = (I + A_bb)^-1 by forward
// substitution in registers (one thread per block column), then the blocks
// below them level by level, T_bc = -D_b sum_{c <= e < b} A_be T_ec, each
// level's sum (into Mt) and its product with D_b as independent dot
// products.  Six barriers in all.  Ts must not alias As; Mt is [3][16][16].
__device__ __forceinline__ void invert_unit_lower(const float *As, float *Ts,
                                                  float *Mt) {
  const int tid = threadIdx.x;
  for (int idx = tid; idx < kBC * kBC; idx += kNT)
    Ts[(idx / kBC) * kCP + idx % kBC] = 0.f;
  __syncthreads();
  if (tid < 64) {
    const int b = tid >> 4, jc = tid & 15, o = 16 * b;
    float x[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      float a0 = (r == jc) ? 1.f : 0.f, a1 = 0.f;
#pragma unroll
      for (int i = 0; i < r; ++i) {
        const float a = As[(o + r) * kCP + o + i];
        if (i & 1) a1 -= a * x[i];
        else a0 -= a * x[i];
      }
      x[r] = a0 + a1;
    }
#pragma unroll
    for (int r = 0; r < 16; ++r) Ts[(o + r) * kCP + o + jc] = x[r];
  }
  __syncthreads();
  // level d = b - c: blocks (c + d, c), c = 0 .. 3 - d
  for (int d = 1; d < 4; ++d) {
    const int nblk = 4 - d;
    for (int idx = tid; idx < nblk * 256; idx += kNT) {
      const int c = idx >> 8, r = (idx >> 4) & 15, col = idx & 15;
      const int bb = c + d;
      // M = sum_{c <= e < b} A_{b e} T_{e c}
      float acc = 0.f;
      for (int e = c; e < bb; ++e)
#pragma unroll
        for (int i = 0; i < 16; ++i)
          acc += As[(16 * bb + r) * kCP + 16 * e + i] *
                 Ts[(16 * e + i) * kCP + 16 * c + col];
      Mt[idx] = acc;
    }
    __syncthreads();
    for (int idx = tid; idx < nblk * 256; idx += kNT) {
      const int c = idx >> 8, r = (idx >> 4) & 15, col = idx & 15;
      const int bb = c + d;
      float acc = 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i)
        acc += Ts[(16 * bb + r) * kCP + 16 * bb + i] * Mt[c * 256 + i * 16 + col];
      Ts[(16 * bb + r) * kCP + 16 * c + col] = -acc;
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// The WY quantities of one (chunk, head), in parallel over all chunks:
//   A[r][i] = beta_r sum_c k_r[c] k_i[c] e^{g_r[c] - g_i[c]}   (i < r < L)
//   P[t][i] =        sum_c q_t[c] k_i[c] e^{g_t[c] - g_i[c]}   (i <= t < L)
//   T = (I + A)^-1,  W = T diag(beta) (K . e^g),  U = T diag(beta) V.
// A and P share their key operand; for the channel-wise decay the weights
// are factored around the chunk's middle row (e^{g - g_ref} on the row side,
// e^{g_ref - g} on the column side) while the chunk's spread allows it, else
// formed one exponential per element; the scalar decay multiplies the
// products by the C x C matrix e^{g_r - g_i}.  T, P go to [chunks][H][C][C];
// W, U to the staged path's [ntok][H][d] buffers.
template <typename Tin, int GATE>
__global__ void __launch_bounds__(kNT)
    bw_wy_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k,
                 const Tin *__restrict__ v, const float *__restrict__ beta,
                 const float *__restrict__ erase,
                 const float *__restrict__ write,
                 const float *__restrict__ wkey,
                 const float *__restrict__ g, float *__restrict__ Tout,
                 float *__restrict__ Pout, float *__restrict__ Wout,
                 float *__restrict__ Uout, const ChunkInfo *__restrict__ table,
                 const int *__restrict__ nchunks, int H, int dk, int dv) {
  const int j = blockIdx.x, h = blockIdx.y;
  if (j >= *nchunks) return;
  const ChunkInfo ci = table[j];
  const int L = ci.len;
  const int gdim = GATE == 0 ? 0 : GATE == 1 ? 1 : dk;
  extern __shared__ float sm[];
  float *Qu = sm;                    // [C][kP]: q e^{g - g_ref}; then the
                                     //   W operand beta k e^g
  float *Ku = Qu + kBC * kP;         // [C][kP]: k e^{g - g_ref}; then beta v
  float *Kd = Ku + kBC * kP;         // [C][kP]: k e^{g_ref - g}
  float *As = Kd + kBC * kP;         // [C][kCP]: A
  float *Ts = As + kBC * kCP;        // [C][kCP]: T
  float *Gh = Ts + kBC * kCP;        // [C][kCP]: e^{g_r - g_i} (scalar gate)
  float *bs = Gh + kBC * kCP;        // [C]
  float *red = bs + kBC;             // [kNT / 32]
  const int tid = threadIdx.x;
  const size_t base = (size_t)ci.tok0 * H + h;
  auto row = [&](int t) { return base + (size_t)t * H; };
  auto gt = [&](int t, int c) { return gv(g, gdim, row(t), c); };
  const int ref = (L - 1) / 2;
  bool fact = true;
  if (GATE == 2) {
    float spread = 0.f;
    for (int idx = tid; idx < L * dk; idx += kNT) {
      const int t = idx / dk, c = idx % dk;
      spread = fmaxf(spread, fabsf(gt(t, c) - gt(ref, c)));
    }
    fact = block_max(spread, red) <= kFactRange;
  }
  for (int idx = tid; idx < kBC * dk; idx += kNT) {
    const int t = idx / dk, c = idx % dk;
    float kv = 0.f, qv = 0.f, d = 0.f, rv = 0.f;
    if (t < L) {
      kv = ldf(k + row(t) * dk + c);
      qv = ldf(q + row(t) * dk + c);
      rv = erase ? erase[row(t) * dk + c] * kv : kv;   // the read key
      if (wkey) kv *= wkey[row(t) * dk + c];            // the write key
      if (GATE == 2 && fact) d = gt(t, c) - gt(ref, c);
    }
    const float up = __expf(d), dn = __expf(-d);
    Qu[t * kP + c] = qv * up;
    Ku[t * kP + c] = rv * up;
    Kd[t * kP + c] = kv * dn;
  }
  // beta, or 1 with the gate variants (0 past the sequence end)
  for (int t = tid; t < kBC; t += kNT)
    bs[t] = t < L ? ((erase || wkey) ? 1.f : beta[row(t)]) : 0.f;
  if (GATE == 1)
    for (int idx = tid; idx < kBC * kBC; idx += kNT) {
      const int r = idx / kBC, i = idx % kBC;
      Gh[r * kCP + i] =
          (i <= r && r < L) ? __expf(gt(r, 0) - gt(i, 0)) : 0.f;
    }
  __syncthreads();
  float *Pg = Pout + ((size_t)j * H + h) * kBC * kBC;
  if (GATE != 2 || fact) {
    gemm_tcn(
        kBC, kBC, dk, [&](int r, int c) { return Ku[r * kP + c]; },
        [&](int c, int i) { return Kd[i * kP + c]; },
        [&](int r, int i, float x) {
          float a = (i < r && r < L) ? bs[r] * x : 0.f;
          if (GATE == 1) a *= Gh[r * kCP + i];
          As[r * kCP + i] = a;
        });
    gemm_tcn(
        kBC, kBC, dk, [&](int t, int c) { return Qu[t * kP + c]; },
        [&](int c, int i) { return Kd[i * kP + c]; },
        [&](int t, int i, float x) {
          float w = (i <= t && t < L) ? x : 0.f;
          if (GATE == 1) w *= Gh[t * kCP + i];
          Pg[t * kBC + i] = w;
        });
  } else {
    // the chunk's channel-wise decay is too wide to factor
    for (int idx = tid; idx < kBC * kBC; idx += kNT) {
      const int r = idx / kBC, i = idx % kBC;
      float a = 0.f, pp = 0.f;
      if (i <= r && r < L)
        for (int c = 0; c < dk; ++c) {
          const float e = Kd[i * kP + c] * __expf(gt(r, c) - gt(i, c));
          a += Ku[r * kP + c] * e;
          pp += Qu[r * kP + c] * e;
        }
      As[r * kCP + i] = i < r ? bs[r] * a : 0.f;
      Pg[idx] = pp;
    }
  }
  __syncthreads();
  invert_unit_lower(As, Ts, Gh);   // Gh (no longer needed) as the scratch
  float *Tg = Tout + ((size_t)j * H + h) * kBC * kBC;
  for (int idx = tid; idx < kBC * kBC; idx += kNT)
    Tg[idx] = Ts[(idx / kBC) * kCP + idx % kBC];
  // the W and U operands: beta (read key) e^g over Qu, beta (target) over Ku
  for (int idx = tid; idx < kBC * dk; idx += kNT) {
    const int t = idx / dk, c = idx % dk;
    float x = 0.f;
    if (t < L) {
      x = bs[t] * ldf(k + row(t) * dk + c) * __expf(gt(t, c));
      if (erase) x *= erase[row(t) * dk + c];
    }
    Qu[t * kP + c] = x;
  }
  for (int idx = tid; idx < kBC * dv; idx += kNT) {
    const int t = idx / dv, c = idx % dv;
    float x = 0.f;
    if (t < L) {
      x = bs[t] * ldf(v + row(t) * dv + c);
      if (write) x *= write[row(t) * dv + c];
    }
    Ku[t * kP + c] = x;
  }
  __syncthreads();
  gemm_tcn(
      kBC, dk, kBC, [&](int r, int s2) { return Ts[r * kCP + s2]; },
      [&](int s2, int c) { return Qu[s2 * kP + c]; },
      [&](int r, int c, float x) {
        if (r < L) Wout[row(r) * dk + c] = x;
      });
  gemm_tcn(
      kBC, dv, kBC, [&](int r, int s2) { return Ts[r * kCP + s2]; },
      [&](int s2, int c) { return Ku[s2 * kP + c]; },
      [&](int r, int c, float x) {
        if (r < L) Uout[row(r) * dv + c] = x;
      });
}

// ---------------------------------------------------------------------------
// Per (chunk, head), in parallel: the chunk's state map and its adjoint's
// input.  With Kc = K . e^{g_C - g}, Qd = Q . e^g, the forward step is
//   S' = Cm S + Dm,   Cm = diag(e^{g_C}) - Kc^T W  [dk x dk],  Dm = Kc^T U,
// and the reverse step (the adjoint runs on the transposed map)
//   Lambda = Cm^T Lambda' + Bm,   Bm = (Qd - P W)^T dO  [dk x dv].
template <typename Tin>
__global__ void __launch_bounds__(kNT)
    bw_prep_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k,
                   const Tin *__restrict__ dout, const float *__restrict__ wkey,
                   const float *__restrict__ g,
                   const float *__restrict__ W, const float *__restrict__ U,
                   const float *__restrict__ Pbuf, float *__restrict__ Cm,
                   float *__restrict__ Dm, float *__restrict__ Bm,
                   const ChunkInfo *__restrict__ table,
                   const int *__restrict__ nchunks, int H, int dk, int dv,
                   int gdim) {
  const int j = blockIdx.x, h = blockIdx.y;
  if (j >= *nchunks) return;
  const ChunkInfo ci = table[j];
  const int L = ci.len;
  extern __shared__ float sm[];
  float *Ws = sm;                    // [C][kP]: W
  float *Ks = Ws + kBC * kP;         // [C][kP]: Kc
  float *Qs = Ks + kBC * kP;         // [C][kP]: Qd, then Qd - P W
  float *Us = Qs + kBC * kP;         // [C][kP]: U, then dO
  float *Ps = Us + kBC * kP;         // [C][kCP]
  float *gl = Ps + kBC * kCP;        // [dk]: g_C
  const int tid = threadIdx.x;
  const size_t base = (size_t)ci.tok0 * H + h;
  for (int c = tid; c < dk; c += kNT)
    gl[c] = gv(g, gdim, base + (size_t)(L - 1) * H, c);
  __syncthreads();
  for (int idx = tid; idx < kBC * dk; idx += kNT) {
    const int r = idx / dk, c = idx % dk;
    const size_t row = base + (size_t)r * H;
    const bool live = r < L;
    const float gr = live ? gv(g, gdim, row, c) : 0.f;
    Ws[r * kP + c] = live ? W[row * dk + c] : 0.f;
    Ks[r * kP + c] = live ? ldf(k + row * dk + c) * __expf(gl[c] - gr) *
                                (wkey ? wkey[row * dk + c] : 1.f)
                          : 0.f;
    Qs[r * kP + c] = live ? ldf(q + row * dk + c) * __expf(gr) : 0.f;
  }
  for (int idx = tid; idx < kBC * dv; idx += kNT) {
    const int r = idx / dv, c = idx % dv;
    Us[r * kP + c] = r < L ? U[(base + (size_t)r * H) * dv + c] : 0.f;
  }
  const float *Pg = Pbuf + ((size_t)j * H + h) * kBC * kBC;
  for (int idx = tid; idx < kBC * kBC; idx += kNT)
    Ps[(idx / kBC) * kCP + idx % kBC] = Pg[idx];
  __syncthreads();
  const size_t mo = ((size_t)j * H + h);
  float *Cg = Cm + mo * dk * dk, *Dg = Dm + mo * dk * dv,
        *Bg = Bm + mo * dk * dv;
  gemm_tcn(
      dk, dk, kBC, [&](int a, int t) { return Ks[t * kP + a]; },
      [&](int t, int b) { return Ws[t * kP + b]; },
      [&](int a, int b, float x) {
        Cg[(size_t)a * dk + b] = (a == b ? __expf(gl[a]) : 0.f) - x;
      });
  gemm_tcn(
      dk, dv, kBC, [&](int a, int t) { return Ks[t * kP + a]; },
      [&](int t, int b) { return Us[t * kP + b]; },
      [&](int a, int b, float x) { Dg[(size_t)a * dv + b] = x; });
  // Qd - P W, in place (own elements)
  gemm_tcn(
      kBC, dk, kBC, [&](int t, int s) { return Ps[t * kCP + s]; },
      [&](int s, int c) { return Ws[s * kP + c]; },
      [&](int t, int c, float x) { Qs[t * kP + c] -= x; });
  __syncthreads();
  for (int idx = tid; idx < kBC * dv; idx += kNT) {
    const int r = idx / dv, c = idx % dv;
    Us[r * kP + c] =
        r < L ? ldf(dout + (base + (size_t)r * H) * dv + c) : 0.f;
  }
  __syncthreads();
  gemm_tcn(
      dk, dv, kBC, [&](int a, int t) { return Qs[t * kP + a]; },
      [&](int t, int b) { return Us[t * kP + b]; },
      [&](int a, int b, float x) { Bg[(size_t)a * dv + b] = x; });
}

// ---------------------------------------------------------------------------
// The two scans over the chunk boundaries, one (sequence, head) per CTA, the
// whole [dk][dv] carried in shared memory: forward (REV = 0) from the initial
// state, X <- Cm X + Dm, storing the state at every chunk start into Xout;
// reverse (REV = 1) from dL/d final_state, X <- Cm^T X + Bm from the last
// chunk, storing dL/dS at every chunk end into Xout and dL/dS_0 into xfin.
template <int REV>
__global__ void __launch_bounds__(kNT)
    bw_scan_kernel(const float *__restrict__ Cm, const float *__restrict__ Nm,
                   const float *__restrict__ x0, float *__restrict__ Xout,
                   float *__restrict__ xfin,
                   const int *__restrict__ seq_first, int H, int dk, int dv) {
  const int n = blockIdx.x, h = blockIdx.y;
  extern __shared__ float sm[];
  float *Ms = sm;                    // [dk][kP]: Cm
  float *Xa = Ms + 128 * kP;         // [dk][kP]: X
  float *Xb = Xa + 128 * kP;         // [dk][kP]: the next X
  const int tid = threadIdx.x;
  const size_t sbase = ((size_t)n * H + h) * dk * dv;
  for (int idx = tid; idx < dk * dv; idx += kNT)
    Xa[(idx / dv) * kP + idx % dv] = x0 ? x0[sbase + idx] : 0.f;
  const int jb = seq_first[n], je = seq_first[n + 1];
  for (int s = 0; s < je - jb; ++s) {
    const int j = REV ? je - 1 - s : jb + s;
    const size_t mo = ((size_t)j * H + h);
    const float *Cg = Cm + mo * dk * dk, *Ng = Nm + mo * dk * dv;
    float *Og = Xout + mo * dk * dv;
    __syncthreads();   // X of the previous step
    for (int idx = tid; idx < dk * dv; idx += kNT) {
      const int a = idx / dv, b = idx % dv;
      Og[idx] = Xa[a * kP + b];
      Xb[a * kP + b] = Ng[idx];
    }
    for (int idx = tid; idx < dk * dk; idx += kNT)
      Ms[(idx / dk) * kP + idx % dk] = Cg[idx];
    __syncthreads();
    gemm_tcn(
        dk, dv, dk,
        [&](int a, int c) { return REV ? Ms[c * kP + a] : Ms[a * kP + c]; },
        [&](int c, int b) { return Xa[c * kP + b]; },
        [&](int a, int b, float x) { Xb[a * kP + b] += x; });
    float *t = Xa;
    Xa = Xb;
    Xb = t;
  }
  __syncthreads();
  if (xfin)
    for (int idx = tid; idx < dk * dv; idx += kNT)
      xfin[sbase + idx] = Xa[(idx / dv) * kP + idx % dv];
}

// ---------------------------------------------------------------------------
// Per (chunk, head, kVH value columns), in parallel: V_new = U - W S and
// dV_new = Kc Lambda + P^T dO, from the scans' S (chunk start) and Lambda
// (chunk end).
constexpr int kVH = 64;
template <typename Tin>
__global__ void __launch_bounds__(kNT)
    bw_vn_kernel(const Tin *__restrict__ k, const Tin *__restrict__ dout,
                 const float *__restrict__ wkey,
                 const float *__restrict__ g, const float *__restrict__ W,
                 const float *__restrict__ U, const float *__restrict__ Pbuf,
                 const float *__restrict__ Sbuf,
                 const float *__restrict__ Lam, float *__restrict__ Vn,
                 float *__restrict__ dVn, const ChunkInfo *__restrict__ table,
                 const int *__restrict__ nchunks, int H, int dk, int dv,
                 int gdim) {
  const int j = blockIdx.x, h = blockIdx.y, j0 = blockIdx.z * kVH;
  if (j >= *nchunks) return;
  const ChunkInfo ci = table[j];
  const int L = ci.len, DV = min(kVH, dv), vp = kVH + 4;
  extern __shared__ float sm[];
  float *Ws = sm;                    // [C][kP]: W
  float *Ks = Ws + kBC * kP;         // [C][kP]: Kc
  float *Ps = Ks + kBC * kP;         // [C][kCP]
  float *Ss = Ps + kBC * kCP;        // [dk][vp]: S columns j0..
  float *Ls = Ss + 128 * vp;         // [dk][vp]: Lambda columns
  float *Os = Ls + 128 * vp;         // [C][vp]: dO columns
  float *gl = Os + kBC * vp;         // [dk]
  const int tid = threadIdx.x;
  const size_t base = (size_t)ci.tok0 * H + h;
  const size_t mo = ((size_t)j * H + h) * dk * dv;
  for (int c = tid; c < dk; c += kNT)
    gl[c] = gv(g, gdim, base + (size_t)(L - 1) * H, c);
  __syncthreads();
  for (int idx = tid; idx < kBC * dk; idx += kNT) {
    const int r = idx / dk, c = idx % dk;
    const size_t row = base + (size_t)r * H;
    const bool live = r < L;
    Ws[r * kP + c] = live ? W[row * dk + c] : 0.f;
    Ks[r * kP + c] = live ? ldf(k + row * dk + c) *
                                __expf(gl[c] - gv(g, gdim, row, c)) *
                                (wkey ? wkey[row * dk + c] : 1.f)
                          : 0.f;
  }
  const float *Pg = Pbuf + ((size_t)j * H + h) * kBC * kBC;
  for (int idx = tid; idx < kBC * kBC; idx += kNT)
    Ps[(idx / kBC) * kCP + idx % kBC] = Pg[idx];
  for (int idx = tid; idx < dk * DV; idx += kNT) {
    const int a = idx / DV, b = idx % DV;
    Ss[a * vp + b] = Sbuf[mo + (size_t)a * dv + j0 + b];
    Ls[a * vp + b] = Lam[mo + (size_t)a * dv + j0 + b];
  }
  for (int idx = tid; idx < kBC * DV; idx += kNT) {
    const int r = idx / DV, b = idx % DV;
    Os[r * vp + b] =
        r < L ? ldf(dout + (base + (size_t)r * H) * dv + j0 + b) : 0.f;
  }
  __syncthreads();
  gemm_tcn(
      kBC, DV, dk, [&](int t, int c) { return Ws[t * kP + c]; },
      [&](int c, int b) { return Ss[c * vp + b]; },
      [&](int t, int b, float x) {
        if (t < L) {
          const size_t o = (base + (size_t)t * H) * dv + j0 + b;
          Vn[o] = U[o] - x;
        }
      });
  gemm_tcn(
      kBC, DV, dk + kBC,
      [&](int t, int x) {
        return x < dk ? Ks[t * kP + x] : Ps[(x - dk) * kCP + t];
      },
      [&](int x, int b) {
        return x < dk ? Ls[x * vp + b] : Os[(x - dk) * vp + b];
      },
      [&](int t, int b, float x) {
        if (t < L) dVn[(base + (size_t)t * H) * dv + j0 + b] = x;
      });
}

// ---------------------------------------------------------------------------
// Gradients of one (chunk, head).  Shared memory (floats), for dk, dv <= 128:
//   TS  T [C][65]
//   BIG five [C][129] tiles: dV_new, V_new, dO, Z, Y (phase 1); then K e^d,
//       K e^-d, Q e^d [C][129] and dT / dA, Xi, M [C][65] (phase 2)
//   SL  the slice tiles S, Lambda [16][129] and (K . e^g) [C][17]; then dP
//   XT  the slice products X1, X2, X3 [3][C][16]
//   small per-row and per-channel sums
constexpr int kRS = kSl + 4;
constexpr int kTS = 0;
constexpr int kBIG = kTS + kBC * kCP;
constexpr int kSLo = kBIG + 5 * kBC * kP;
constexpr int kXT = kSLo + 2 * kSl * kP + kBC * kRS;
constexpr int kSM = kXT + 3 * kBC * kSl;
constexpr int kSmall = 64 * 3 + 128 * 3 + 16;
static_assert(kBC * kSl <= 2 * kNT, "two slice elements per thread");
constexpr int kGradSmemFloats = kSM + kSmall;
static_assert(kBIG + 3 * kBC * kP + 3 * kBC * kCP <= kSLo, "phase-2 tiles");
static_assert(kGradSmemFloats * 4 <= 232448, "shared memory");
static_assert(kBC * kCP <= 2 * kSl * kP + kBC * kRS, "dP tile");

template <typename Tin, int GATE>
__global__ void __launch_bounds__(kNT)
    bw_grad_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k,
                   const Tin *__restrict__ v, const Tin *__restrict__ dout,
                   const float *__restrict__ beta, const float *__restrict__ g,
                   const float *__restrict__ erase,
                   const float *__restrict__ write,
                   const float *__restrict__ wkey,
                   const float *__restrict__ Tbuf,
                   const float *__restrict__ Sbuf,
                   const float *__restrict__ Lam,
                   const float *__restrict__ Vnb,
                   const float *__restrict__ dVnb, float *__restrict__ dq,
                   float *__restrict__ dkg, float *__restrict__ dvg,
                   float *__restrict__ dbeta, float *__restrict__ dla,
                   float *__restrict__ derase, float *__restrict__ dwrite,
                   float *__restrict__ dwkey,
                   const ChunkInfo *__restrict__ table,
                   const int *__restrict__ nchunks, int H, int dk, int dv) {
  const int j = blockIdx.x, h = blockIdx.y;
  if (j >= *nchunks) return;
  const ChunkInfo ci = table[j];
  const int L = ci.len;
  const int gdim = GATE == 0 ? 0 : GATE == 1 ? 1 : dk;
  extern __shared__ float sm[];
  float *Ts = sm + kTS;
  float *Ds = sm + kBIG, *Vs = Ds + kBC * kP, *Os = Vs + kBC * kP,
        *Zs = Os + kBC * kP, *Ys = Zs + kBC * kP;
  float *Ss = sm + kSLo, *Ls = Ss + kSl * kP, *Rs = Ls + kSl * kP;
  float *X1 = sm + kXT, *X2 = X1 + kBC * kSl, *X3 = X2 + kBC * kSl;
  float *bs = sm + kSM, *dbs = bs + 64, *dgs = dbs + 64, *dgC = dgs + 64,
        *gC = dgC + 128, *gR = gC + 128, *red = gR + 128;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t base = (size_t)ci.tok0 * H + h;   // row of token 0
  auto row = [&](int t) { return base + (size_t)t * H; };
  auto gt = [&](int t, int c) { return gv(g, gdim, row(t), c); };
  const float *Sg = Sbuf + ((size_t)j * H + h) * dk * dv;
  const float *Lg = Lam + ((size_t)j * H + h) * dk * dv;

  // ---- phase 1: the value side
  {
    const float *Tg = Tbuf + ((size_t)j * H + h) * kBC * kBC;
    for (int idx = tid; idx < kBC * kBC; idx += kNT)
      Ts[(idx / kBC) * kCP + idx % kBC] = Tg[idx];
  }
  for (int idx = tid; idx < kBC * dv; idx += kNT) {
    const int t = idx / dv, c = idx % dv;
    const bool live = t < L;
    const size_t o = row(t) * dv + c;
    Ds[t * kP + c] = live ? dVnb[o] : 0.f;
    Vs[t * kP + c] = live ? Vnb[o] : 0.f;
    Os[t * kP + c] = live ? ldf(dout + o) : 0.f;
    // Y starts from the target (v, or w . v with Gated DeltaNet-2's gates)
    Ys[t * kP + c] = live ? ldf(v + o) * (write ? write[o] : 1.f) : 0.f;
  }
  for (int t = tid; t < 64; t += kNT) {
    bs[t] = t < L ? ((erase || wkey) ? 1.f : beta[row(t)]) : 0.f;
    dbs[t] = 0.f;
    dgs[t] = 0.f;
  }
  for (int c = tid; c < 128; c += kNT) {
    dgC[c] = 0.f;
    gC[c] = c < dk ? gt(L - 1, c) : 0.f;
  }
  __syncthreads();
  // Z = T^T dV_new
  gemm_tcn(
      kBC, dv, kBC, [&](int r, int s) { return Ts[s * kCP + r]; },
      [&](int s, int c) { return Ds[s * kP + c]; },
      [&](int r, int c, float x) { Zs[r * kP + c] = x; });
  __syncthreads();
  for (int c0 = 0; c0 < dk; c0 += kSl) {
    for (int idx = tid; idx < kSl * dv; idx += kNT) {
      const int cc = idx / dv, c = idx % dv;
      Ss[cc * kP + c] = Sg[(size_t)(c0 + cc) * dv + c];
      Ls[cc * kP + c] = Lg[(size_t)(c0 + cc) * dv + c];
    }
    // the elementwise pass's inputs (two elements per thread), fetched
    // before the products so that their latency hides behind them
    float pg[2], pq[2], pk[2], pb[2], pa[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int idx = tid + u * kNT;
      pg[u] = pq[u] = pk[u] = 0.f;
      pb[u] = pa[u] = 1.f;
      if (idx < L * kSl) {
        const int t = idx / kSl, c = c0 + idx % kSl;
        const size_t o = row(t) * dk + c;
        pg[u] = gt(t, c);
        pq[u] = ldf(q + o);
        pk[u] = ldf(k + o);
        if (erase) pb[u] = erase[o];
        if (wkey) pa[u] = wkey[o];
      }
    }
    for (int idx = tid; idx < kBC * kSl; idx += kNT) {
      const int t = idx / kSl, cc = idx % kSl;
      // the read key times e^g
      float x = 0.f;
      if (t < L) {
        const size_t o = row(t) * dk + c0 + cc;
        x = ldf(k + o) * __expf(gt(t, c0 + cc));
        if (erase) x *= erase[o];
      }
      Rs[t * kRS + cc] = x;
    }
    __syncthreads();
    // Y -= (K . e^g)[:, slice] S[slice, :]
    gemm_tcn(
        kBC, dv, kSl, [&](int t, int cc) { return Rs[t * kRS + cc]; },
        [&](int cc, int c) { return Ss[cc * kP + c]; },
        [&](int t, int c, float x) { Ys[t * kP + c] -= x; });
    // X1 = dO S^T, X2 = (beta . Z) S^T, X3 = V_new Lambda^T (slice columns)
    gemm_tcn(
        kBC, kSl, dv, [&](int t, int c) { return Os[t * kP + c]; },
        [&](int c, int cc) { return Ss[cc * kP + c]; },
        [&](int t, int cc, float x) { X1[t * kSl + cc] = x; });
    gemm_tcn(
        kBC, kSl, dv, [&](int t, int c) { return bs[t] * Zs[t * kP + c]; },
        [&](int c, int cc) { return Ss[cc * kP + c]; },
        [&](int t, int cc, float x) { X2[t * kSl + cc] = x; });
    gemm_tcn(
        kBC, kSl, dv, [&](int t, int c) { return Vs[t * kP + c]; },
        [&](int c, int cc) { return Ls[cc * kP + c]; },
        [&](int t, int cc, float x) { X3[t * kSl + cc] = x; });
    // e^{g_C} sum_j Lambda[c][j] S[c][j]: the decay of the carried state
    for (int cc = warp; cc < kSl; cc += kNT / 32) {
      float s = 0.f;
      for (int c = lane; c < dv; c += 32) s += Ls[cc * kP + c] * Ss[cc * kP + c];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1)
        s += __shfl_xor_sync(0xffffffffu, s, off);
      if (lane == 0) dgC[c0 + cc] += __expf(gC[c0 + cc]) * s;
    }
    __syncthreads();
    // elementwise: dq = X1 e^g; dk = -X2 e^g + X3 e^{g_C - g}; the decay
    // gradient of the factors e^g (on q and on the read key) and
    // e^{g_C - g} (on the update key)
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int idx = tid + u * kNT;
      if (idx >= L * kSl) continue;
      const int t = idx / kSl, cc = idx % kSl, c = c0 + cc;
      const float gg = pg[u], e = __expf(gg), ec = __expf(gC[c] - gg);
      const size_t o = row(t) * dk + c;
      const float qv = pq[u], kv = pk[u];
      const float bv = pb[u], av = pa[u];   // read key bv kv, write key av kv
      const float x1 = X1[t * kSl + cc], x2 = X2[t * kSl + cc],
                  x3 = X3[t * kSl + cc];
      // read-key gradient -x2 e^g, write-key gradient x3 e^{g_C - g}
      dq[o] = x1 * e;
      dkg[o] = -x2 * e * bv + av * x3 * ec;
      if (erase) derase[o] = -x2 * e * kv;
      if (wkey) dwkey[o] = kv * x3 * ec;
      const float dgv = (x1 * qv - x2 * bv * kv) * e - x3 * av * kv * ec;
      if (GATE == 2) dla[row(t) * dk + c] = dgv;
      if (GATE == 1) atomicAdd(&dgs[t], dgv);
      if (GATE != 0) atomicAdd(&dgC[c], x3 * av * kv * ec);
    }
    __syncthreads();
  }
  // dbeta (value side) and dv
  for (int t = warp; t < L; t += kNT / 32) {
    float s = 0.f;
    for (int c = lane; c < dv; c += 32) s += Zs[t * kP + c] * Ys[t * kP + c];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
      s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) dbs[t] = s;
  }
  for (int idx = tid; idx < L * dv; idx += kNT) {
    const int t = idx / dv, c = idx % dv;
    const size_t o = row(t) * dv + c;
    // the target's gradient beta Z, through w . v with the gates
    const float dt = bs[t] * Zs[t * kP + c];
    dvg[o] = write ? write[o] * dt : dt;
    if (write) dwrite[o] = ldf(v + o) * dt;
  }
  __syncthreads();
  float *dTs = sm + kBIG + 3 * kBC * kP;   // over Z (phase 2: then dA)
  float *Xi = dTs + kBC * kCP;
  float *Ms = Xi + kBC * kCP;
  float *dPs = sm + kSLo;                  // over the slice tiles
  // dT = dV_new (beta . Y)^T;  dP = lower(dO V_new^T)
  gemm_tcn(
      kBC, kBC, dv, [&](int r, int c) { return Ds[r * kP + c]; },
      [&](int c, int i) { return bs[i] * Ys[i * kP + c]; },
      [&](int r, int i, float x) { dTs[r * kCP + i] = x; });
  gemm_tcn(
      kBC, kBC, dv, [&](int t, int c) { return Os[t * kP + c]; },
      [&](int c, int i) { return Vs[i * kP + c]; },
      [&](int t, int i, float x) {
        dPs[t * kCP + i] = (i <= t && t < L) ? x : 0.f;
      });
  __syncthreads();

  // ---- phase 2: the key side of A and P
  float *Ku = sm + kBIG, *Kd = Ku + kBC * kP, *Qu = Kd + kBC * kP;
  // Xi = T^T dT
  gemm_tcn(
      kBC, kBC, kBC, [&](int r, int s) { return Ts[s * kCP + r]; },
      [&](int s, int i) { return dTs[s * kCP + i]; },
      [&](int r, int i, float x) { Xi[r * kCP + i] = x; });
  // keys and queries, with e^{+-(g - g_ref)} for the channel gate when the
  // chunk's spread allows the factoring
  const int ref = (L - 1) / 2;
  bool fact = true;
  if (GATE == 2) {
    for (int c = tid; c < dk; c += kNT) gR[c] = gt(ref, c);
    float spread = 0.f;
    for (int idx = tid; idx < L * dk; idx += kNT) {
      const int t = idx / dk, c = idx % dk;
      spread = fmaxf(spread, fabsf(gt(t, c) - gt(ref, c)));
    }
    fact = block_max(spread, red) <= kFactRange;   // (its barriers publish gR)
  }
  for (int idx = tid; idx < kBC * dk; idx += kNT) {
    const int t = idx / dk, c = idx % dk;
    float kv = 0.f, qv = 0.f, d = 0.f, rv = 0.f;
    if (t < L) {
      kv = ldf(k + row(t) * dk + c);
      qv = ldf(q + row(t) * dk + c);
      rv = erase ? erase[row(t) * dk + c] * kv : kv;   // the read key
      if (wkey) kv *= wkey[row(t) * dk + c];            // the write key
      if (GATE == 2 && fact) d = gt(t, c) - gt(ref, c);
    }
    const float up = __expf(d), dn = __expf(-d);
    Ku[t * kP + c] = rv * up;
    Kd[t * kP + c] = kv * dn;
    Qu[t * kP + c] = qv * up;
  }
  __syncthreads();
  // dA = -Xi T^T, strictly lower (over dT)
  gemm_tcn(
      kBC, kBC, kBC, [&](int r, int s) { return Xi[r * kCP + s]; },
      [&](int s, int i) { return Ts[i * kCP + s]; },
      [&](int r, int i, float x) {
        dTs[r * kCP + i] = (i < r && r < L) ? -x : 0.f;
      });
  // M = the A matrix without beta: k_r^T Gamma k_i, i < r
  if (GATE != 2 || fact) {
    gemm_tcn(
        kBC, kBC, dk, [&](int r, int c) { return Ku[r * kP + c]; },
        [&](int c, int i) { return Kd[i * kP + c]; },
        [&](int r, int i, float x) {
          float w = (i < r && r < L) ? x : 0.f;
          if (GATE == 1 && i < r && r < L) w *= __expf(gt(r, 0) - gt(i, 0));
          Ms[r * kCP + i] = w;
        });
  } else {
    for (int idx = tid; idx < kBC * kBC; idx += kNT) {
      const int r = idx / kBC, i = idx % kBC;
      float a = 0.f;
      if (i < r && r < L)
        for (int c = 0; c < dk; ++c)
          a += Ku[r * kP + c] * Kd[i * kP + c] * __expf(gt(r, c) - gt(i, c));
      Ms[r * kCP + i] = a;
    }
  }
  __syncthreads();
  // dbeta += rowsum(dA . M); then dA -> beta_r dA (times e^{g_r - g_i} for
  // the scalar gate), dP -> dP e^{g_t - g_i} (scalar gate)
  for (int r = warp; r < L; r += kNT / 32) {
    float s = 0.f;
    for (int i = lane; i < r; i += 32) s += dTs[r * kCP + i] * Ms[r * kCP + i];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
      s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) dbs[r] += s;
  }
  __syncthreads();
  for (int idx = tid; idx < kBC * kBC; idx += kNT) {
    const int r = idx / kBC, i = idx % kBC;
    const float gw =
        (GATE == 1 && i <= r && r < L) ? __expf(gt(r, 0) - gt(i, 0)) : 1.f;
    dTs[r * kCP + i] *= bs[r] * gw;
    dPs[r * kCP + i] *= gw;
  }
  __syncthreads();
  // the key and query gradients of A and P:
  //   drho = dM Kd, dkap = dM^T Ku, dqP = dP Kd, dkP = dP^T Qu
  // (times e^{+-(g - g_ref)} for the factored channel gate)
  if (GATE != 2 || fact) {
    auto pair_out = [&](int t, int c, float r1, float r2, float r3, float r4) {
      if (t >= L) return;
      const float d = (GATE == 2) ? gt(t, c) - gR[c] : 0.f;
      const float up = __expf(d), dn = __expf(-d);
      const float drho = up * r1, dkap = dn * r2, dqP = up * r3, dkP = dn * r4;
      const size_t o = row(t) * dk + c;
      // the write key, query and read key back from their rescaled tiles
      // (the raw key is the write key with the erase gate, the read key
      // with FG^2-GDN's rate)
      const float kv = Kd[t * kP + c] * up, qv = Qu[t * kP + c] * dn,
                  rv = Ku[t * kP + c] * dn;
      dq[o] += dqP;
      dkg[o] += (erase ? erase[o] : 1.f) * drho +
                (wkey ? wkey[o] : 1.f) * (dkap + dkP);
      if (erase) derase[o] += kv * drho;
      if (wkey) dwkey[o] += rv * (dkap + dkP);
      const float dgv = rv * drho - kv * (dkap + dkP) + qv * dqP;
      if (GATE == 2) dla[o] += dgv;
      if (GATE == 1) atomicAdd(&dgs[t], dgv);
    };
    // rows and columns of dA and dP past L are zero, so K = C
    auto a1 = [&](int t, int i) { return dTs[t * kCP + i]; };
    auto a2 = [&](int t, int i) { return dTs[i * kCP + t]; };
    auto a3 = [&](int t, int i) { return dPs[t * kCP + i]; };
    auto a4 = [&](int t, int i) { return dPs[i * kCP + t]; };
    auto bk = [&](int i, int c) { return Kd[i * kP + c]; };
    auto bu = [&](int i, int c) { return Ku[i * kP + c]; };
    auto bq = [&](int i, int c) { return Qu[i * kP + c]; };
    if (dk % 16 == 0 && (kBC / 16) * (dk / 16) >= kNT / 32)
      gemm_tc4<2>(kBC, dk, kBC, a1, bk, a2, bu, a3, bk, a4, bq, pair_out);
    else
      gemm_tc4<1>(kBC, dk, kBC, a1, bk, a2, bu, a3, bk, a4, bq, pair_out);
  } else {
    // channel-wise decay too wide to factor: one exponential per element
    for (int idx = tid; idx < L * dk; idx += kNT) {
      const int t = idx / dk, c = idx % dk;
      const float gtc = gt(t, c);
      float drho = 0.f, dkap = 0.f, dqP = 0.f, dkP = 0.f;
      for (int i = 0; i < L; ++i) {
        const float e = __expf(i <= t ? gtc - gt(i, c) : gt(i, c) - gtc);
        if (i < t) drho += dTs[t * kCP + i] * Kd[i * kP + c] * e;
        if (i > t) dkap += dTs[i * kCP + t] * Ku[i * kP + c] * e;
        if (i <= t) dqP += dPs[t * kCP + i] * Kd[i * kP + c] * e;
        if (i >= t) dkP += dPs[i * kCP + t] * Qu[i * kP + c] * e;
      }
      const size_t o = row(t) * dk + c;
      // (unfactored: Ku holds the read key, Kd the write key, Qu the query)
      const float rv = Ku[t * kP + c], kv = Kd[t * kP + c],
                  qv = Qu[t * kP + c];
      dq[o] += dqP;
      dkg[o] += (erase ? erase[o] : 1.f) * drho +
                (wkey ? wkey[o] : 1.f) * (dkap + dkP);
      if (erase) derase[o] += kv * drho;
      if (wkey) dwkey[o] += rv * (dkap + dkP);
      dla[o] += rv * drho - kv * (dkap + dkP) + qv * dqP;
    }
  }
  __syncthreads();
  // the last row carries g_C; then d log_alpha = reverse cumsum of dg
  if (GATE == 2) {
    for (int c = tid; c < dk; c += kNT) {
      float acc = dgC[c];
      for (int t = L - 1; t >= 0; --t) {
        const size_t o = row(t) * dk + c;
        acc += dla[o];
        dla[o] = acc;
      }
    }
  } else if (GATE == 1) {
    if (warp == 0) {
      float s = 0.f;
      for (int c = lane; c < dk; c += 32) s += dgC[c];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1)
        s += __shfl_xor_sync(0xffffffffu, s, off);
      if (lane == 0) {
        float acc = s;
        for (int t = L - 1; t >= 0; --t) {
          acc += dgs[t];
          dla[row(t)] = acc;
        }
      }
    }
  }
  if (dbeta)
    for (int t = tid; t < L; t += kNT) dbeta[row(t)] = dbs[t];
}

// ---------------------------------------------------------------------------
// host side

size_t al256(size_t x) { return (x + 255) & ~size_t(255); }

struct ChunkedLayout {
  size_t staged, T, P, Lam, dVn, Cm, Dm, Bm, total;
};

ChunkedLayout chunked_layout(const Problem &p) {
  ChunkedLayout l;
  const size_t cc = (size_t)p.max_chunks * p.H;
  size_t o = 0;
  l.staged = o;  o += al256(staged_workspace_bytes(p));
  l.T = o;       o += al256(sizeof(float) * cc * kBC * kBC);
  l.P = o;       o += al256(sizeof(float) * cc * kBC * kBC);
  l.Lam = o;     o += al256(sizeof(float) * cc * p.dk * p.dv);
  l.dVn = o;     o += al256(sizeof(float) * (size_t)p.ntok * p.H * p.dv);
  l.Cm = o;      o += al256(sizeof(float) * cc * p.dk * p.dk);
  l.Dm = o;      o += al256(sizeof(float) * cc * p.dk * p.dv);
  l.Bm = o;      o += al256(sizeof(float) * cc * p.dk * p.dv);
  l.total = o;
  return l;
}

template <typename Tin, int GATE>
cudaError_t run_grad(const Problem &p, const BackwardIO &io,
                     const StagedBufs &b, const float *Tb, const float *Lam,
                     const float *dVn, cudaStream_t s) {
  const int smem = kGradSmemFloats * (int)sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(
      bw_grad_kernel<Tin, GATE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
      smem);
  if (e != cudaSuccess) return e;
  bw_grad_kernel<Tin, GATE><<<dim3(p.max_chunks, p.H), kNT, smem, s>>>(
      static_cast<const Tin *>(p.q), static_cast<const Tin *>(p.k),
      static_cast<const Tin *>(p.v), static_cast<const Tin *>(io.dout),
      p.beta, b.g, p.erase, p.write, p.wkey, Tb, b.Sbuf, Lam, b.Vn, dVn,
      io.dq, io.dk, io.dv, io.dbeta, io.dla, io.derase, io.dwrite, io.dwkey,
      b.table, b.nchunks, p.H, p.dk, p.dv);
  return cudaGetLastError();
}

template <typename Tin, int GATE>
cudaError_t run_wy(const Problem &p, const StagedBufs &b, float *Tb, float *Pb,
                   cudaStream_t s) {
  const int smem =
      (int)sizeof(float) * (3 * kBC * kP + 3 * kBC * kCP + kBC + kNT / 32);
  cudaError_t e = cudaFuncSetAttribute(
      bw_wy_kernel<Tin, GATE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
      smem);
  if (e != cudaSuccess) return e;
  bw_wy_kernel<Tin, GATE><<<dim3(p.max_chunks, p.H), kNT, smem, s>>>(
      static_cast<const Tin *>(p.q), static_cast<const Tin *>(p.k),
      static_cast<const Tin *>(p.v), p.beta, p.erase, p.write, p.wkey, b.g,
      Tb, Pb, b.W, b.U, b.table, b.nchunks, p.H, p.dk, p.dv);
  return cudaGetLastError();
}

template <typename Tin>
cudaError_t run_typed(const Problem &p, const BackwardIO &io, char *ws,
                      cudaStream_t s) {
  const ChunkedLayout l = chunked_layout(p);
  float *Tb = reinterpret_cast<float *>(ws + l.T);
  float *Pb = reinterpret_cast<float *>(ws + l.P);
  float *Lam = reinterpret_cast<float *>(ws + l.Lam);
  float *dVn = reinterpret_cast<float *>(ws + l.dVn);
  cudaError_t e = staged_chunks_run(p, ws + l.staged, s);
  if (e != cudaSuccess) return e;
  const StagedBufs b = staged_bufs(p, ws + l.staged);
  const int gdim = p.gate == GDR_GATE_NONE ? 0
                   : p.gate == GDR_GATE_SCALAR ? 1
                                               : p.dk;
  const Tin *q = static_cast<const Tin *>(p.q);
  const Tin *k = static_cast<const Tin *>(p.k);
  if (p.max_chunks > 0) {
    e = p.gate == GDR_GATE_NONE
            ? run_wy<Tin, 0>(p, b, Tb, Pb, s)
            : p.gate == GDR_GATE_SCALAR ? run_wy<Tin, 1>(p, b, Tb, Pb, s)
                                        : run_wy<Tin, 2>(p, b, Tb, Pb, s);
    if (e != cudaSuccess) return e;
  }
  float *Cm = reinterpret_cast<float *>(ws + l.Cm);
  float *Dm = reinterpret_cast<float *>(ws + l.Dm);
  float *Bm = reinterpret_cast<float *>(ws + l.Bm);
  const Tin *dout = static_cast<const Tin *>(io.dout);
  if (p.max_chunks > 0) {
    const int smem = (int)sizeof(float) * (4 * kBC * kP + kBC * kCP + p.dk);
    e = cudaFuncSetAttribute(bw_prep_kernel<Tin>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    bw_prep_kernel<Tin><<<dim3(p.max_chunks, p.H), kNT, smem, s>>>(
        q, k, dout, p.wkey, b.g, b.W, b.U, Pb, Cm, Dm, Bm, b.table,
        b.nchunks, p.H, p.dk, p.dv, gdim);
  }
  {
    const int smem = (int)sizeof(float) * 3 * 128 * kP;
    e = cudaFuncSetAttribute(bw_scan_kernel<0>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(bw_scan_kernel<1>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const dim3 sgrid(p.nseq, p.H);
    bw_scan_kernel<0><<<sgrid, kNT, smem, s>>>(Cm, Dm, p.s0, b.Sbuf, nullptr,
                                               b.seq_first, p.H, p.dk, p.dv);
    bw_scan_kernel<1><<<sgrid, kNT, smem, s>>>(Cm, Bm, io.dsT, Lam, io.ds0,
                                               b.seq_first, p.H, p.dk, p.dv);
  }
  if (p.max_chunks > 0) {
    const int vp = kVH + 4;
    const int smem = (int)sizeof(float) *
                     (2 * kBC * kP + kBC * kCP + 2 * 128 * vp + kBC * vp +
                      p.dk);
    e = cudaFuncSetAttribute(bw_vn_kernel<Tin>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int dvh = p.dv < kVH ? p.dv : kVH;
    bw_vn_kernel<Tin><<<dim3(p.max_chunks, p.H, p.dv / dvh), kNT, smem, s>>>(
        k, dout, p.wkey, b.g, b.W, b.U, Pb, b.Sbuf, Lam, b.Vn, dVn, b.table,
        b.nchunks, p.H, p.dk, p.dv, gdim);
  }
  if (p.max_chunks == 0) return cudaGetLastError();
  switch (p.gate) {
    case GDR_GATE_NONE: return run_grad<Tin, 0>(p, io, b, Tb, Lam, dVn, s);
    case GDR_GATE_SCALAR: return run_grad<Tin, 1>(p, io, b, Tb, Lam, dVn, s);
    default: return run_grad<Tin, 2>(p, io, b, Tb, Lam, dVn, s);
  }
}

}  // namespace

bool backward_chunked_applies(const Problem &p) {
  return p.chunk == kBC && p.dk <= 128 && p.dv <= 128 && p.dk % kSl == 0 &&
         p.dv % 16 == 0;
}

size_t backward_chunked_bytes(const Problem &p) {
  return chunked_layout(p).total;
}

cudaError_t backward_chunked_run(const Problem &p, const BackwardIO &io,
                                 void *workspace, cudaStream_t s) {
  char *ws = static_cast<char *>(workspace);
  if (p.dtype == GDR_FP32) return run_typed<float>(p, io, ws, s);
  return run_typed<__nv_bfloat16>(p, io, ws, s);
}

}  // namespace gdr
