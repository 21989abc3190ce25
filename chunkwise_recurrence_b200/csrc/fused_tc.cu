// Fused tensor-core path of libgdr: one persistent CTA per (sequence, head)
// runs the whole chunkwise gated delta rule chunk after chunk, with every
// intermediate on chip, on sm_100a tcgen05 tensor cores.
//
// Per chunk of C = 64 tokens (dk = dv = 128), with g the in-chunk cumulative
// log-decay (per key channel for KDA), S the state at the chunk start:
//   A  = strictly-lower beta_r k_r^T Gamma_r Gamma_i^-1 k_i      (K K^T on TC)
//   T  = (I + A)^-1                          (blocked forward substitution)
//   W  = T diag(beta) (K . e^g),  U = T diag(beta) V              (TC)
//   V_new = U - W S                                               (TC)
//   O  = (Q . e^g) S + mask_{i<=r}[(Q . e^g)(K . e^-g)^T] V_new   (TC)
//   S <- Gamma_C S + (K . e^{g_C - g})^T V_new                    (TC)
// This is the WY form of the delta rule with the decay absorbed into the
// erase factors (Gated DeltaNet-2 abstract, comparative-study page
// 2607.07953), which rests on the update being affine in the preceding memory
// ("DeltaTTT: Layerwise Optimization for Nonlinear Recurrent Memory",
// §2 Background).
//
// Everything that does not depend on S (A, T, W, U, the output mask P) for
// chunk n+1 is computed while the S-dependent chain of chunk n runs:
//   warp 0      TMA producer: Q, K (two stages) and V tiles, 128-B swizzle;
//               channel gate, the fp32 log-decay tile one chunk ahead
//   warp 1      tensor-memory allocation and the single MMA-issuing thread
//   warps 2..5  "state" warps: S -> fp16 operand and decay, V_new -> fp16
//               operand, output tile -> global (thread = tensor-memory lane
//               = one value channel)
//   warps 6..13 "prep" warps (two per scheduler): gates, cumsum and per-row
//               decay factors (channel gate: per-channel running sums and
//               Q, K rescaled by e^{+-(g - g_m)}, fp16 or bf16 per chunk),
//               A and P from K K^T / Q K^T, T = (I+A)^-1, T-factor
//               operands, -W operand, in-place Q . e^g and K . e^{g_C - g}
//               (fp16; channel gate: K~ only)
//   warps 14,15 "convert" warps: channel gate, V tile bf16 -> fp16 in place
//               for the fp16 U product, then K . e^g (for W) and Q . e^g
//               (for X) in place; the scalar / no gate U and W read the raw
//               bf16 V and K
// The channel gate also runs the per-channel gate variants (template GV):
//   GV = 1  Gated DeltaNet-2: the read key is b . k (erase gate b, per key
//           channel) and the target w . v (write gate w, per value channel);
//   GV = 2  FG^2-GDN: the write key is a . k (rate a, per key channel) and
//           the target (c .) v (FG^2-GDN+'s value scaling c, optional).
// beta is then 1 (0 past the sequence end, which masks those rows as
// before).  The prep warps fold b into the M-side key block or a into the
// write-key tile when they rescale them (one fp32 product, one rounding);
// the convert warps fold w or c into V when they convert it to fp16.  The
// TMA producer prefetches each chunk's gate rows into L2 one chunk ahead.
// Waiting threads ask to be suspended until their phase completes, so that
// they leave issue slots to the working warps (the MMA thread above all).
// All state lives in tensor memory as S^T (lane = value channel, column =
// key channel) in fp32; fp16 / bf16 appear only as tensor-core operands.
//
// Tensor memory (512 columns x 128 lanes, fp32):
//   [0,128) S^T   [128,256) V_new^T x2   [256,384) O^T x2
//   [384,448) [K;Q] K^T   [448,512) W^T
//
// Every mbarrier wait is bounded; on expiry the kernel raises a sticky error
// word (read by gdr_device_error) and every role winds down.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <mutex>
#include <type_traits>

#include "gdr_internal.h"
#include "sm100.cuh"

namespace gdr {
namespace {

using namespace sm100;

constexpr int kC = 64;         // chunk length
constexpr int kD = 128;        // dk = dv
constexpr int kThreads = 512;  // 16 warps
constexpr int kPrep = 256;     // prep threads (warps 6..13)
constexpr int kConv = 64;      // convert threads (warps 14, 15)
// fp32 16x16 blocks: rows kRS floats apart, blocks kBS floats apart.  The
// padding spreads eight consecutive rows (16-byte accesses) and the tf32
// fragment rows over distinct banks, and puts neighbouring blocks on
// opposite bank halves.
constexpr int kRS = 20;
constexpr int kBS = 16 * kRS + 16;

// ---- shared memory layout (bytes from a 1024-aligned base) ----------------
// A stage holds one chunk's K and Q as four 8 KB [64 rows][64 cols] blocks:
// [K cols 0..63 | Q cols 0..63 | K cols 64..127 | Q cols 64..127], so that
// rows 0..63 (K) and 64..127 (Q) of a 16 KB block form one M=128 operand.
constexpr uint32_t kStageBytes = 32768;
constexpr uint32_t OFF_STAGE = 0;                        // 2 stages
constexpr uint32_t OFF_V = OFF_STAGE + 2 * kStageBytes;  // [2][64][64] bf16
constexpr uint32_t OFF_NW = OFF_V + 16384;               // -W^T [128][64]
constexpr uint32_t OFF_OS = OFF_NW + 16384;              // output staging
constexpr uint32_t OFF_P = OFF_OS + 16384;               // P [2][64][64]
constexpr uint32_t OFF_TP = OFF_P + 16384;               // T-factor tiles
template <int GATE>
struct Layout {
  // fp16 T-factor tiles: scalar / no gate T diag(b e^g) (TPG) and
  // T diag(b) (TPB); channel gate T diag(b) only, plus K e^{g_m - g} (bf16)
  // T-factor tiles.  Scalar / no gate, bf16 against the raw bf16 V and K:
  // T diag(b) for U as a hi + lo pair (TPB, TPB_LO: the lo tile holds the
  // bf16 rounding residual, so U carries about 16 significant bits of the
  // factor; a single bf16 factor there quadruples the final-state error),
  // and T diag(b e^g) for W as one tile (TPG).  Channel gate: T diag(b) in
  // fp16 (TPB) for both, against fp16 V and K e^g.
  // Scalar / no gate: one set per chunk parity, so that chunk m+1's factors
  // are written while U of chunk m may still read its own (W done of chunk
  // m+1 is waited for later and covers U of chunk m, issued before it).  The
  // channel gate has no room for a second set: its prep warps wait for V
  // free (U done) instead.
  static constexpr uint32_t TP_PAR = (GATE == 2) ? 0 : 24576;
  static constexpr uint32_t TP_BYTES = (GATE == 2) ? 8192 : 2 * 24576;
  static constexpr uint32_t TPB = OFF_TP, TPG = OFF_TP + 8192,
                            TPB_LO = OFF_TP + 16384;
  static constexpr uint32_t KN = OFF_TP + TP_BYTES;
  static constexpr uint32_t KN_BYTES = (GATE == 2) ? 16384 : 0;
  static constexpr uint32_t AC = KN + KN_BYTES;   // A blocks fp32 [10][kBS]
  static constexpr uint32_t TC = AC + 40 * kBS;   // T blocks fp32 [10][kBS]
  // per-chunk gate arrays, three buffers (chunk m uses buffer m % 3): a
  // chunk's gates are written while the two before it may still be read
  static constexpr uint32_t GS = TC + 40 * kBS;   // g [3][64]
  static constexpr uint32_t FT = GS + 768;        // row factors [3][6][64]
  static constexpr uint32_t GC = FT + 4608;       // g_C [3][128]
  // channel gate, per key channel, for the chunk in progress: e^{g_m}
  // (g_m = g at row 31) and e^{g_C - g_m}
  static constexpr uint32_t GM = GC + 1536;       // [2][128]
  // channel gate: each half-chunk's log-decay total per key channel [2][128]
  // followed by the prep warps' decay-range maxima [8] and, per chunk
  // parity, whether the chunk's rescaled Q, K use fp16 (else bf16) [2]
  static constexpr uint32_t TT = GM + 1024;
  static constexpr uint32_t TT_BYTES = (GATE == 2) ? 1024 + 64 : 0;
  static constexpr uint32_t TT_WMAX = TT + 1024, TT_F16 = TT + 1024 + 32;
  // channel gate: the chunk's log-decays, fp32 [2][64 rows][64 channels]
  // (channels 0..63, then 64..127), loaded by TMA one chunk ahead; turned
  // into running sums in place
  static constexpr uint32_t LA = (TT + TT_BYTES + 127) & ~127u;
  static constexpr uint32_t LA_BYTES = (GATE == 2) ? 32768 : 0;
  static constexpr uint32_t MISC = LA + LA_BYTES; // barriers, tmem base, flags
  static constexpr uint32_t BYTES = MISC + 256;
  static_assert(BYTES + 1024 <= 232448, "shared memory budget");
};
// per-row factor arrays inside FT (each [64] fp32), for one chunk buffer
enum { F_B, F_BG, F_E, F_F, F_EG, F_EK, F_COUNT };

// tensor-memory columns
constexpr uint32_t ACC_S = 0, ACC_V = 128, ACC_O = 256, ACC_KK = 384,
                   ACC_W = 448;

// mbarrier indices
// (pairs indexed by chunk parity complete every other chunk, so a waiter
// that falls one chunk behind cannot mistake a later phase for its own)
enum {
  B_FULL0, B_FULL1, B_EMPTY0, B_EMPTY1, B_VFREE, B_KKREADY,
  B_KKDONE0, B_KKDONE1,  // K K^T of the chunk done (MMA commit)
  B_TREADY, B_WDONE, B_WREADY, B_SREADY, B_XDONE, B_VNREADY, B_SDONE,
  B_ODONE, B_DRAIN, B_FULLV,
  B_CONV,                // channel gate: V, Q, K fp16 (convert warps)
  B_LAFULL, B_LAFREE,    // channel gate: log-decay tile landed / read
  B_QCONV,               // channel gate: Q e^g fp16 (convert warps)
  B_COUNT
};

// Instruction descriptors (M = 128 everywhere).  Operands built on chip are
// fp16 (11-bit significand: 8x finer than bf16 at the same tensor-core rate).
// Products that read raw bf16 input tiles stay bf16: K K^T, and for the
// scalar / no gate U and W (their T factors are bf16; U's as a hi + lo
// pair).  The channel gate's K K^T reads keys scaled by e^{+-(g - g_m)}:
// fp16 when the chunk's decay keeps those factors within e^{+-9}, else bf16
// for its exponent range; its U and W are fp16.
constexpr uint32_t ID_KK_B = idesc_f16kind(128, 64, false, false, true);
constexpr uint32_t ID_KK_H = idesc_f16kind(128, 64, false, false, false);
// largest |g - g_m| for which the channel gate's rescaled operands use fp16
// (e^9 = 8103: normalised keys stay far below fp16's 65504)
constexpr float kF16Range = 9.f;
constexpr uint32_t ID_UW_H = idesc_f16kind(128, 64, true, false, false);
constexpr uint32_t ID_UW_B = idesc_f16kind(128, 64, true, false, true);
constexpr uint32_t ID_XV = idesc_f16kind(128, 64, false, true, false);
constexpr uint32_t ID_XO = idesc_f16kind(128, 64, false, false, false);
constexpr uint32_t ID_SU = idesc_f16kind(128, 128, false, true, false);
constexpr uint32_t ID_OI = idesc_f16kind(128, 64, false, false, false);

// error word bits: 0..23 = the mbarrier whose wait expired; range errors
constexpr unsigned kErrRange = 1u << 24;      // input beyond fp16 range
constexpr unsigned kErrNonFinite = 1u << 25;  // non-finite output or state
constexpr float kF16Max = 65504.f;

constexpr long long kWaitCycles = 1ll << 32;   // ~2 s: a wait never lasts this

__device__ unsigned g_fused_error;

struct Params {
  const float *beta;
  // per-channel gate variants (GV != 0): the key-side gate [ntok][H][128]
  // (erase gate b or rate a) and the value-side gate (write gate w or
  // scaling c; nullptr for none)
  const float *gk, *gv;
  const float *log_alpha;
  const float *s0;
  __nv_bfloat16 *out;
  float *sT;
  const int32_t *cu;
  int nseq, T, ntok, H;
};

struct Ctx {
  uint64_t *bar;
  volatile int *abort_flag;
};

// Bounded wait: true when the phase completed, false on abort or timeout.
// While the phase is incomplete the thread asks to be suspended (it resumes
// when the phase completes), so that waiting warps leave their scheduler's
// issue slots to the warps that work -- the MMA-issuing thread above all.
constexpr uint32_t kSuspendNs = 20000;
__device__ __forceinline__ bool wait_bar(const Ctx &cx, int b,
                                         uint32_t parity) {
  if (mbar_try_wait(&cx.bar[b], parity)) return true;
  const long long t0 = clock64();
  for (;;) {
    if (mbar_try_wait_sleep(&cx.bar[b], parity, kSuspendNs)) return true;
    if (*cx.abort_flag) return false;
    if (clock64() - t0 > kWaitCycles) {
      *cx.abort_flag = 1;
      atomicOr(&g_fused_error, 1u << b);
      return false;
    }
  }
}

// AND of `pred` over the `count` threads of named barrier `id` (a barrier):
// a role group takes every wait decision together, so no thread is left
// behind at a later named barrier when another one gives up.
__device__ __forceinline__ bool group_all(bool pred, int id, int count) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}\n"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}
__device__ __forceinline__ void unpack_bf16(uint32_t w, float &lo, float &hi) {
  __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162 *>(&w);
  float2 f = __bfloat1622float2(v);
  lo = f.x;
  hi = f.y;
}
__device__ __forceinline__ void unpack_f16(uint32_t w, float &lo, float &hi) {
  __half2 v = *reinterpret_cast<__half2 *>(&w);
  float2 f = __half22float2(v);
  lo = f.x;
  hi = f.y;
}
// 8 values in place (16 bytes of shared memory): bf16 -> fp16 times sc
// 8 values in place (16 bytes of shared memory): bf16 -> fp16 times sc[e]
__device__ __forceinline__ void bf16_to_f16_16B_each(uint8_t *ptr,
                                                     const float *sc) {
  uint4 x = *reinterpret_cast<uint4 *>(ptr);
  uint32_t *w = reinterpret_cast<uint32_t *>(&x);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162 *>(&w[e]);
    float2 f = __bfloat1622float2(b);
    __half2 hv = __floats2half2_rn(f.x * sc[2 * e], f.y * sc[2 * e + 1]);
    w[e] = *reinterpret_cast<uint32_t *>(&hv);
  }
  *reinterpret_cast<uint4 *>(ptr) = x;
}
// 8 consecutive fp32 gate values of row `row` (two 16-byte loads); zeros for
// a row past the chunk's last token, whose token may lie beyond the tensor
__device__ __forceinline__ void load_gate8(float *g8, const float *base,
                                           size_t row, int ch, bool live) {
  if (live) {
    const float4 *gp =
        reinterpret_cast<const float4 *>(base + row * kD + ch);
    const float4 a = __ldg(gp), b = __ldg(gp + 1);
    g8[0] = a.x; g8[1] = a.y; g8[2] = a.z; g8[3] = a.w;
    g8[4] = b.x; g8[5] = b.y; g8[6] = b.z; g8[7] = b.w;
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) g8[e] = 0.f;
  }
}
__device__ __forceinline__ void bf16_to_f16_16B(uint8_t *ptr, float sc) {
  uint4 x = *reinterpret_cast<uint4 *>(ptr);
  uint32_t *w = reinterpret_cast<uint32_t *>(&x);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162 *>(&w[e]);
    float2 f = __bfloat1622float2(b);
    __half2 hv = __floats2half2_rn(f.x * sc, f.y * sc);
    w[e] = *reinterpret_cast<uint32_t *>(&hv);
  }
  *reinterpret_cast<uint4 *>(ptr) = x;
}
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}
__device__ __forceinline__ void st_smem_v4(uint8_t *p, uint32_t a, uint32_t b,
                                           uint32_t c, uint32_t d) {
  *reinterpret_cast<uint4 *>(p) = make_uint4(a, b, c, d);
}

// index of the 16x16 block (rb, cb), cb <= rb, in the compact lower storage
__device__ __forceinline__ int blk(int rb, int cb) {
  return rb * (rb + 1) / 2 + cb;
}

// tf32 operand: the fp32 bit pattern as is (the tensor core reads the top
// 19 bits, i.e. truncates; a rounding cvt would cost an ALU op per operand)
__device__ __forceinline__ uint32_t to_tf32(float x) { return __float_as_uint(x); }

// acc (2 n-tiles of m16n8 C fragments) += X (16x16) * Z (16x16), both
// row-major fp32 in shared memory, on mma.sync m16n8k8 tf32.
__device__ __forceinline__ void mma16(const float *X, const float *Z,
                                      float acc[8], int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int ks = 0; ks < 2; ++ks) {
    const uint32_t a0 = to_tf32(X[g * kRS + 8 * ks + t]);
    const uint32_t a1 = to_tf32(X[(g + 8) * kRS + 8 * ks + t]);
    const uint32_t a2 = to_tf32(X[g * kRS + 8 * ks + t + 4]);
    const uint32_t a3 = to_tf32(X[(g + 8) * kRS + 8 * ks + t + 4]);
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const uint32_t b0 = to_tf32(Z[(8 * ks + t) * kRS + 8 * nt + g]);
      const uint32_t b1 = to_tf32(Z[(8 * ks + t + 4) * kRS + 8 * nt + g]);
      float *c = acc + 4 * nt;
      asm volatile(
          "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 "
          "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
          "{%0, %1, %2, %3};"
          : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
          : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    }
  }
}

// acc (one m16n8 C fragment: columns 8 nt .. 8 nt + 7) += X * Z
__device__ __forceinline__ void mma16_nt(const float *X, const float *Z,
                                         float acc[4], int lane, int nt) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int ks = 0; ks < 2; ++ks) {
    const uint32_t a0 = to_tf32(X[g * kRS + 8 * ks + t]);
    const uint32_t a1 = to_tf32(X[(g + 8) * kRS + 8 * ks + t]);
    const uint32_t a2 = to_tf32(X[g * kRS + 8 * ks + t + 4]);
    const uint32_t a3 = to_tf32(X[(g + 8) * kRS + 8 * ks + t + 4]);
    const uint32_t b0 = to_tf32(Z[(8 * ks + t) * kRS + 8 * nt + g]);
    const uint32_t b1 = to_tf32(Z[(8 * ks + t + 4) * kRS + 8 * nt + g]);
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(acc[0]), "+f"(acc[1]), "+f"(acc[2]), "+f"(acc[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
}
__device__ __forceinline__ void store16_nt(float *Y, const float acc[4],
                                           float s, int lane, int nt) {
  const int g = lane >> 2, t = lane & 3;
  Y[g * kRS + 8 * nt + 2 * t] = s * acc[0];
  Y[g * kRS + 8 * nt + 2 * t + 1] = s * acc[1];
  Y[(g + 8) * kRS + 8 * nt + 2 * t] = s * acc[2];
  Y[(g + 8) * kRS + 8 * nt + 2 * t + 1] = s * acc[3];
}

// store C fragments (scaled by s) to a row-major 16x16 fp32 block
__device__ __forceinline__ void load16_nt(const float *Y, float acc[4],
                                          int lane, int nt) {
  const int g = lane >> 2, t = lane & 3;
  acc[0] = Y[g * kRS + 8 * nt + 2 * t];
  acc[1] = Y[g * kRS + 8 * nt + 2 * t + 1];
  acc[2] = Y[(g + 8) * kRS + 8 * nt + 2 * t];
  acc[3] = Y[(g + 8) * kRS + 8 * nt + 2 * t + 1];
}
__device__ __forceinline__ void store16(float *Y, const float acc[8], float s,
                                        int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    Y[g * kRS + 8 * nt + 2 * t] = s * acc[4 * nt + 0];
    Y[g * kRS + 8 * nt + 2 * t + 1] = s * acc[4 * nt + 1];
    Y[(g + 8) * kRS + 8 * nt + 2 * t] = s * acc[4 * nt + 2];
    Y[(g + 8) * kRS + 8 * nt + 2 * t + 1] = s * acc[4 * nt + 3];
  }
}

template <int GATE, int GV>
__global__ void __launch_bounds__(kThreads, 1)
    gdr_fused_tc_kernel(const __grid_constant__ CUtensorMap tmq,
                        const __grid_constant__ CUtensorMap tmk,
                        const __grid_constant__ CUtensorMap tmv,
                        const __grid_constant__ CUtensorMap tmla,
                        const __grid_constant__ CUtensorMap tmgk,
                        const __grid_constant__ CUtensorMap tmgv, Params p) {
  static_assert(GV == 0 || GATE == 2, "gate variants need the channel gate");
  using Lay = Layout<GATE>;
  extern __shared__ uint8_t smem_raw[];
  // 1024-aligned base, derived by pointer arithmetic on the shared array so
  // that the compiler keeps every access in the shared address space
  uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t *bar = reinterpret_cast<uint64_t *>(sm + Lay::MISC);
  uint32_t *tmem_base_slot = reinterpret_cast<uint32_t *>(sm + Lay::MISC + 8 * B_COUNT);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + Lay::MISC + 8 * B_COUNT + 4);
  float *scan_tmp = reinterpret_cast<float *>(sm + Lay::MISC + 8 * B_COUNT + 8);
  float *AC = reinterpret_cast<float *>(sm + Lay::AC);
  float *TC = reinterpret_cast<float *>(sm + Lay::TC);
  const Ctx cx{bar, abort_flag};

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = blockIdx.x / p.H, h = blockIdx.x % p.H;
  int start = p.cu ? p.cu[n] : n * p.T;
  int end = p.cu ? p.cu[n + 1] : (n + 1) * p.T;
  start = min(max(start, 0), p.ntok);
  end = min(max(end, start), p.ntok);
  const int NC = (end - start + kC - 1) / kC;
  const size_t sbase = ((size_t)n * p.H + h) * kD * kD;

  if (threadIdx.x == 0) {
    const uint32_t counts[B_COUNT] = {
        1, 1, 1, 1, 1, kPrep, 1, 1, kPrep, 1, kPrep, 128, 1, 128, 1, 1, 1, 1,
        kConv, 1, kPrep, kConv};
    for (int i = 0; i < B_COUNT; ++i) mbar_init(&bar[i], counts[i]);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_base_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_slot;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_map(&tmq);
      tma_prefetch_map(&tmk);
      tma_prefetch_map(&tmv);
      if (GATE == 2) tma_prefetch_map(&tmla);
      if (GV != 0) {
        tma_prefetch_map(&tmgk);
        if (p.gv) tma_prefetch_map(&tmgv);
      }
      int issued = 0, issued_v = 0, issued_la = 0;
      for (int m = 0; m < NC; ++m) {
        const int s = m & 1;
        if (GATE == 2) {
          // log-decays of chunk m, once the prep warps have read chunk m-1's
          if (m >= 1 && !wait_bar(cx, B_LAFREE, (m - 1) & 1)) break;
          mbar_arrive_expect_tx(&bar[B_LAFULL], 2 * 16384);
          for (int kb = 0; kb < 2; ++kb)
            tma_load_3d(sm + Lay::LA + kb * 16384, &tmla, &bar[B_LAFULL],
                        kb * 64, h, start + m * kC);
          issued_la = m + 1;
          // the gate rows of chunk m into L2, a chunk before they are read
          if (GV != 0) {
            for (int kb = 0; kb < 2; ++kb) {
              tma_prefetch_l2_3d(&tmgk, kb * 64, h, start + m * kC);
              if (p.gv) tma_prefetch_l2_3d(&tmgv, kb * 64, h, start + m * kC);
            }
          }
        }
        if (m >= 2 && !wait_bar(cx, B_EMPTY0 + s, ((m - 2) >> 1) & 1)) break;
        const int tok0 = start + m * kC;
        uint8_t *stg = sm + OFF_STAGE + s * kStageBytes;
        // Q, K of chunk m -> stage m % 2 (full[s]); V -> its one buffer
        // (fullv) once U of chunk m-1 has read the previous V
        mbar_arrive_expect_tx(&bar[B_FULL0 + s], 4 * 8192);
        for (int kb = 0; kb < 2; ++kb) {
          tma_load_3d(stg + kb * 16384, &tmk, &bar[B_FULL0 + s], kb * 64, h,
                      tok0);
          tma_load_3d(stg + kb * 16384 + 8192, &tmq, &bar[B_FULL0 + s],
                      kb * 64, h, tok0);
        }
        issued = m + 1;
        if (m >= 1 && !wait_bar(cx, B_VFREE, (m - 1) & 1)) break;
        mbar_arrive_expect_tx(&bar[B_FULLV], 2 * 8192);
        for (int kb = 0; kb < 2; ++kb)
          tma_load_3d(sm + OFF_V + kb * 8192, &tmv, &bar[B_FULLV], kb * 64, h,
                      tok0);
        issued_v = m + 1;
      }
      if (*abort_flag) {
        // let in-flight copies land before the CTA exits (bounded)
        for (int m = max(0, issued - 2); m < issued; ++m) {
          const long long t0 = clock64();
          while (!mbar_try_wait(&bar[B_FULL0 + (m & 1)], (m >> 1) & 1) &&
                 clock64() - t0 < (1ll << 28)) {
          }
        }
        if (issued_v > 0) {
          const long long t0 = clock64();
          while (!mbar_try_wait(&bar[B_FULLV], (issued_v - 1) & 1) &&
                 clock64() - t0 < (1ll << 28)) {
          }
        }
        if (issued_la > 0) {
          const long long t0 = clock64();
          while (!mbar_try_wait(&bar[B_LAFULL], (issued_la - 1) & 1) &&
                 clock64() - t0 < (1ll << 28)) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t nw = smem_u32(sm + OFF_NW), vt = smem_u32(sm + OFF_V),
                     kn = smem_u32(sm + Lay::KN), sm_base_u32 = smem_u32(sm);
      // Shared-memory descriptors are built once; a K step or sub-tile
      // only adds its byte offset / 16 to the start-address field (shared
      // addresses stay below 256 KB, so the 14-bit field never carries).
      auto dadd = [](uint64_t d, uint32_t bytes) { return d + (bytes >> 4); };
      const uint64_t st16[2] = {sdesc_sw128(sm_base_u32 + OFF_STAGE, 16, 1024),
                                sdesc_sw128(sm_base_u32 + OFF_STAGE + kStageBytes,
                                            16, 1024)};
      const uint64_t stmn[2] = {
          sdesc_sw128(sm_base_u32 + OFF_STAGE, 16384, 1024),
          sdesc_sw128(sm_base_u32 + OFF_STAGE + kStageBytes, 16384, 1024)};
      auto st_k = [&](int m) { return (m & 1) ? st16[1] : st16[0]; };
      auto st_mn = [&](int m) { return (m & 1) ? stmn[1] : stmn[0]; };
      const uint64_t d_kn = sdesc_sw128(kn, 16, 1024);
      const uint64_t d_vt = sdesc_sw128(vt, 8192, 1024);
      const uint64_t d_nw = sdesc_sw128(nw, 8192, 1024);
      const uint64_t d_tpb = sdesc_sw128(smem_u32(sm + Lay::TPB), 16, 1024);
      const uint64_t d_tpw = sdesc_sw128(
          smem_u32(sm + (GATE == 2 ? Lay::TPB : Lay::TPG)), 16, 1024);
      const uint64_t d_tplo = sdesc_sw128(smem_u32(sm + Lay::TPB_LO), 16, 1024);
      const uint64_t d_p[2] = {sdesc_sw128(smem_u32(sm + OFF_P), 16, 1024),
                               sdesc_sw128(smem_u32(sm + OFF_P + 8192), 16, 1024)};
      // channel gate: the prep warps rescale Q, K in place first (kk_ready);
      // otherwise K K^T runs straight on the landed bf16 tiles
      auto kk_inputs_ready = [&](int m) {
        return GATE == 2 ? wait_bar(cx, B_KKREADY, m & 1)
                         : wait_bar(cx, B_FULL0 + (m & 1), (m >> 1) & 1);
      };
      auto issue_kk = [&](int m) {
        const uint64_t base = st_k(m);
        // channel gate: the prep warps chose fp16 or bf16 for this chunk
        const uint32_t kk_id =
            (GATE == 2 &&
             reinterpret_cast<const volatile int *>(sm + Lay::TT_F16)[m & 1])
                ? ID_KK_H
                : ID_KK_B;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t koff = (ks >> 2) * 16384 + (ks & 3) * 32;
          const uint64_t a = dadd(base, koff);
          const uint64_t b =
              GATE == 2 ? dadd(d_kn, (ks >> 2) * 8192 + (ks & 3) * 32) : a;
          mma_f16kind(tmem + ACC_KK, a, b, kk_id, ks > 0);
        }
        mma_commit(&bar[B_KKDONE0 + (m & 1)]);
      };
      // U^T = V^T (T diag b)^T and W^T = (K e^g)^T (T diag(b e^g))^T, all
      // fp16: V and K are converted in place by the convert warps (for the
      // channel gate K already holds K e^g, and the factor is T diag(b))
      // scalar / no gate: raw bf16 V and K against bf16 T factors; channel
      // gate: fp16 (V converted, K e^g written by the prep warps)
      constexpr uint32_t kIdUW = (GATE == 2) ? ID_UW_H : ID_UW_B;
      auto issue_uw = [&](int m) {
        if (!wait_bar(cx, B_CONV, m & 1)) return false;
        tc_fence_after();
        const uint64_t base = st_mn(m);
        const uint32_t accv = tmem + ACC_V + (m & 1) * 64;
        const uint32_t tpo = (m & 1) * Lay::TP_PAR;   // T-factor set
        // W first: its commit (W done) lets the prep warps start P5 while
        // the U products still run.  X, which accumulates onto U, is issued
        // later by this thread, and one thread's MMAs complete in order.
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma_f16kind(tmem + ACC_W, dadd(base, ks * 2048),
                      dadd(d_tpw, tpo + ks * 32), kIdUW, ks > 0);
        mma_commit(&bar[B_WDONE]);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma_f16kind(accv, dadd(d_vt, ks * 2048), dadd(d_tpb, tpo + ks * 32),
                      kIdUW, ks > 0);
        if (GATE != 2) {
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            mma_f16kind(accv, dadd(d_vt, ks * 2048),
                        dadd(d_tplo, tpo + ks * 32), kIdUW, 1);
        }
        mma_commit(&bar[B_VFREE]);
        return true;
      };
      // K K^T of chunk j may run as soon as its tiles are in and the prep
      // warps have read K K^T of chunk j-1 (t_ready(j-1)); after each U/W
      // issue the next one is tried without blocking, else it is issued at
      // its place in the loop below
      int kk_next = 0;
      auto try_kk_early = [&](int j) {
        if (kk_next != j || j >= NC) return;
        const bool ready =
            GATE == 2 ? mbar_try_wait(&bar[B_KKREADY], j & 1)
                      : mbar_try_wait(&bar[B_FULL0 + (j & 1)], (j >> 1) & 1);
        if (ready) {
          tc_fence_after();
          issue_kk(j);
          ++kk_next;
        }
      };
      bool ok = true;
      if (NC > 0) {
        ok = kk_inputs_ready(0);
        if (ok) {
          tc_fence_after();
          issue_kk(0);
          kk_next = 1;
          ok = wait_bar(cx, B_TREADY, 0);
        }
        if (ok) {
          tc_fence_after();
          ok = issue_uw(0);
          try_kk_early(1);
        }
      }
      for (int m = 0; m < NC && ok; ++m) {
        const uint64_t qbase = dadd(st_k(m), 8192), kbase = st_mn(m);
        // X(m): V_new^T = U^T + S^T (-W)^T ; O^T = S^T (Q e^g)^T
        if (!wait_bar(cx, B_SREADY, m & 1) || !wait_bar(cx, B_WREADY, m & 1) ||
            (GATE == 2 && !wait_bar(cx, B_QCONV, m & 1)))
          break;
        tc_fence_after();
        // A = S^T, fp16 pairs in tensor memory (8 columns per K step)
        const uint32_t st_op = tmem + ACC_V + ((m + 1) & 1) * 64;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_f16kind_ts(tmem + ACC_V + (m & 1) * 64, st_op + 8 * ks,
                         dadd(d_nw, ks * 2048), ID_XV, 1);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_f16kind_ts(tmem + ACC_O + (m & 1) * 64, st_op + 8 * ks,
                         dadd(qbase, (ks >> 2) * 16384 + (ks & 3) * 32), ID_XO,
                         ks > 0);
        mma_commit(&bar[B_XDONE]);
        // K K^T of chunk m+1 while the state warps turn V_new into an
        // operand, if its inputs are in (the channel gate's rescaling may
        // still be running: the S update must not wait for it)
        try_kk_early(m + 1);
        // S update and intra-chunk output
        if (!wait_bar(cx, B_VNREADY, m & 1)) break;
        tc_fence_after();
        // A = V_new^T, fp16 pairs in tensor memory; B = K e^{g_C - g}
        const uint32_t vn_op = tmem + ACC_V + (m & 1) * 64;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma_f16kind_ts(tmem + ACC_S, vn_op + 8 * ks, dadd(kbase, ks * 2048),
                         ID_SU, 1);
        const uint64_t pbase = (m & 1) ? d_p[1] : d_p[0];
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma_f16kind_ts(tmem + ACC_O + (m & 1) * 64, vn_op + 8 * ks,
                         dadd(pbase, ks * 32), ID_OI, 1);
        // S done also covers the intra-chunk output: both read V_new(m),
        // whose columns S^T(m+1) reuses
        mma_commit(&bar[B_SDONE]);
        mma_commit(&bar[B_ODONE]);
        mma_commit(&bar[B_EMPTY0 + (m & 1)]);
        // K K^T of chunk m+1 now at the latest: its T factors depend on it
        if (m + 1 < NC && kk_next == m + 1) {
          if (!kk_inputs_ready(m + 1)) break;
          tc_fence_after();
          issue_kk(m + 1);
          ++kk_next;
        }
        // U, W of chunk m+1
        if (m + 1 < NC) {
          if (!wait_bar(cx, B_TREADY, (m + 1) & 1)) break;
          tc_fence_after();
          if (!issue_uw(m + 1)) break;
          try_kk_early(m + 2);
        }
      }
      // every MMA issued has completed before tensor memory is released
      mma_commit(&bar[B_DRAIN]);
      const long long t0 = clock64();
      while (!mbar_try_wait(&bar[B_DRAIN], 0) && clock64() - t0 < kWaitCycles) {
      }
    }
  } else if (warp < 6) {
    // ------------------------------------------------------ state warps
    const int q4 = warp & 3;
    const int l = q4 * 32 + lane;                  // value channel
    const uint32_t trow = tmem + ((uint32_t)(q4 * 32) << 16);
    float v[32];
    // initial state -> S^T in tensor memory
    for (int c0 = 0; c0 < kD; c0 += 32) {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        v[j] = p.s0 ? p.s0[sbase + (size_t)(c0 + j) * kD + l] : 0.f;
      tmem_st32(trow + ACC_S + c0, v);
    }
    tmem_wait_st();
    bool ok = true;
    // O^T of chunk m (lane = value channel, column = row) -> out rows, via
    // a [64 rows][128 channels] bf16 staging tile in shared memory.
    // Neighbouring lanes swap values so each writes two adjacent channels.
    auto store_output = [&](int m) {
      const int tok0 = start + m * kC, L = min(kC, end - tok0);
      uint8_t *stg = sm + OFF_OS;
      float osum = 0.f;   // a non-finite output shows up in this sum
      for (int c0 = 0; c0 < kC; c0 += 32) {
        tmem_ld32(trow + ACC_O + (m & 1) * 64 + c0, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) osum += (c0 + j < L) ? v[j] : 0.f;
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const float send = (l & 1) ? v[j] : v[j + 1];
          const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
          const int r = c0 + j + (l & 1);
          const float lo = (l & 1) ? recv : v[j];
          const float hi = (l & 1) ? v[j + 1] : recv;
          *reinterpret_cast<uint32_t *>(stg + r * 256 + (l & ~1) * 2) =
              pack_bf16(lo, hi);
        }
      }
      if (!isfinite(osum)) atomicOr(&g_fused_error, kErrNonFinite);
      named_bar_sync(1, 128);
      for (int i = l; i < kC * 16; i += 128) {
        const int r = i >> 4, ch = i & 15;
        if (r < L) {
          const uint4 x = *reinterpret_cast<const uint4 *>(stg + r * 256 + ch * 16);
          *reinterpret_cast<uint4 *>(p.out + ((size_t)(tok0 + r) * p.H + h) * kD +
                                     ch * 8) = x;
        }
      }
      named_bar_sync(1, 128);
    };
    float *gC = reinterpret_cast<float *>(sm + Lay::GC);
    for (int m = 0; m < NC; ++m) {
      // S (chunk start) -> fp16 operand; decayed S back to tensor memory
      if (m > 0 && !(ok = group_all(wait_bar(cx, B_SDONE, (m - 1) & 1), 1, 128)))
        break;
      if (!(ok = group_all(wait_bar(cx, B_TREADY, m & 1), 1, 128))) break;
      tc_fence_after();
      const float *gcm = gC + (m % 3) * 128;
      const float dscal = GATE == 1 ? __expf(gcm[0]) : 1.f;
      // S^T as fp16 pairs (key channels 2j, 2j+1 in column j) into the
      // V_new^T region of the other chunk parity, free from S done(m-1)
      // (whose commit follows the last reader of V_new(m-1)) until U(m+1)
      const uint32_t st_op = trow + ACC_V + ((m + 1) & 1) * 64;
      for (int c0 = 0; c0 < kD; c0 += 32) {
        tmem_ld32(trow + ACC_S + c0, v);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) pk[j] = pack_f16(v[2 * j], v[2 * j + 1]);
        tmem_st16(st_op + (c0 >> 1), pk);
        if (GATE != 0) {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            v[j] *= (GATE == 1) ? dscal : gcm[c0 + j];   // KDA: e^{g_C}
          tmem_st32(trow + ACC_S + c0, v);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar[B_SREADY]);
      // output of the previous chunk while X(m) runs
      if (m > 0) {
        if (!(ok = group_all(wait_bar(cx, B_ODONE, (m - 1) & 1), 1, 128))) break;
        tc_fence_after();
        store_output(m - 1);
      }
      // V_new^T -> fp16 pairs (tokens 2j, 2j+1 in column j) in place, in
      // the first 32 columns of its own region
      if (!(ok = group_all(wait_bar(cx, B_XDONE, m & 1), 1, 128))) break;
      tc_fence_after();
      {
        // both halves are loaded before the first store overwrites
        // columns 0..15
        const uint32_t vreg = trow + ACC_V + (m & 1) * 64;
        uint32_t pk[16];
        tmem_ld32(vreg, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) pk[j] = pack_f16(v[2 * j], v[2 * j + 1]);
        tmem_ld32(vreg + 32, v);
        tmem_wait_ld();
        tmem_st16(vreg, pk);
#pragma unroll
        for (int j = 0; j < 16; ++j) pk[j] = pack_f16(v[2 * j], v[2 * j + 1]);
        tmem_st16(vreg + 16, pk);
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(&bar[B_VNREADY]);
    }
    if (ok && NC > 0) {
      ok = group_all(wait_bar(cx, B_ODONE, (NC - 1) & 1), 1, 128);
      if (ok) {
        tc_fence_after();
        store_output(NC - 1);
        ok = group_all(wait_bar(cx, B_SDONE, (NC - 1) & 1), 1, 128);
      }
    }
    if (ok) {
      tc_fence_after();
      bool finite = true;
      for (int c0 = 0; c0 < kD; c0 += 32) {
        tmem_ld32(trow + ACC_S + c0, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          finite = finite && isfinite(v[j]);
          if (p.sT) p.sT[sbase + (size_t)(c0 + j) * kD + l] = v[j];
        }
      }
      if (!finite) atomicOr(&g_fused_error, kErrNonFinite);
    }
  } else if (warp >= 14) {
    // ------------------------------------------------------ convert warps
    // Channel gate: V -> fp16 in place for U = (T diag b) V, once V has
    // landed, and Q, K -> fp16 Q e^g, K e^g once K K^T has read them.
    // Scalar / no gate: U and W read the raw bf16 tiles, and these warps
    // only pass the V arrival on.
    const int ct = threadIdx.x - 14 * 32;
    const float *gM = reinterpret_cast<const float *>(sm + Lay::GM);
    for (int m = 0; m < NC; ++m) {
      if (!group_all(wait_bar(cx, B_FULLV, m & 1), 3, kConv)) break;
      if (GATE == 2) {
        if (GV != 0 && p.gv) {
          // V . (write gate or value scaling): item i is row r and the
          // physical 16-byte chunk i & 7 of block i >> 9, i.e. channels
          // 64 (i >> 9) + 8 ((i & 7) ^ (r & 7)) .. + 7 (128-B swizzle)
          const int tok0 = start + m * kC, L = min(kC, end - tok0);
#pragma unroll 4
          for (int i = ct; i < 1024; i += kConv) {
            const int r = (i >> 3) & 63;
            const int c = (i >> 9) * 64 + (((i & 7) ^ (r & 7)) << 3);
            float gw[8];
            load_gate8(gw, p.gv, (size_t)(tok0 + r) * p.H + h, c, r < L);
            bf16_to_f16_16B_each(sm + OFF_V + i * 16, gw);
          }
        } else {
#pragma unroll 4
          for (int i = ct; i < 1024; i += kConv)
            bf16_to_f16_16B(sm + OFF_V + i * 16, 1.f);
        }
        // once K K^T has read them: K e^{g-g_m}, then Q e^{g-g_m} (bf16)
        // -> K e^g for W (conv), then Q e^g for X (qconv), fp16 in place.
        // Item = row, 8 channels; the 8 factors e^{g_m} are two vector loads.
        if (!group_all(wait_bar(cx, B_KKDONE0 + (m & 1), (m >> 1) & 1), 3,
                       kConv))
          break;
        uint8_t *stg = sm + OFF_STAGE + (m & 1) * kStageBytes;
        const bool src16 =
            reinterpret_cast<const volatile int *>(sm + Lay::TT_F16)[m & 1] != 0;
        auto to_f16_ge = [&](uint32_t part, auto h16) {
          constexpr bool kH = decltype(h16)::value;
#pragma unroll 4
          for (int idx = ct; idx < kC * 16; idx += kConv) {
            const int r = idx >> 4, cc = idx & 15, kb = cc >> 3;
            const float4 *fp = reinterpret_cast<const float4 *>(gM + cc * 8);
            const float4 f0 = fp[0], f1 = fp[1];
            const float f[8] = {f0.x, f0.y, f0.z, f0.w,
                                f1.x, f1.y, f1.z, f1.w};
            uint4 *xp = reinterpret_cast<uint4 *>(
                stg + kb * 16384 + part + sw128_chunk(r, cc & 7));
            uint4 xv = *xp;
            uint32_t *xw = reinterpret_cast<uint32_t *>(&xv);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              float a0, a1;
              if (kH) unpack_f16(xw[e], a0, a1);
              else unpack_bf16(xw[e], a0, a1);
              xw[e] = pack_f16(a0 * f[2 * e], a1 * f[2 * e + 1]);
            }
            *xp = xv;
          }
          fence_proxy_async_smem();
        };
        if (src16) to_f16_ge(0, std::true_type{});
        else to_f16_ge(0, std::false_type{});
        mbar_arrive(&bar[B_CONV]);
        if (src16) to_f16_ge(8192, std::true_type{});
        else to_f16_ge(8192, std::false_type{});
        mbar_arrive(&bar[B_QCONV]);
      } else {
        mbar_arrive(&bar[B_CONV]);
      }
    }
  } else {
    // ------------------------------------------------------ prep warps
    // 8 warps, two per scheduler.  pt = 0..255; TMEM lane l (two threads per
    // lane: hf selects which 32 of a 64-column accumulator each one reads).
    const int pt = threadIdx.x - 6 * 32;
    const int q4 = warp & 3;
    const int l = q4 * 32 + lane;
    const int hf = (warp - 6) >> 2;
    const int pw = warp - 6;                       // 0..7
    const uint32_t trow = tmem + ((uint32_t)(q4 * 32) << 16);
    float *gS = reinterpret_cast<float *>(sm + Lay::GS);
    float *FT = reinterpret_cast<float *>(sm + Lay::FT);
    float *gC = reinterpret_cast<float *>(sm + Lay::GC);
    float *gM = reinterpret_cast<float *>(sm + Lay::GM);
    float v[32];
    // gates of the next chunk are loaded one chunk ahead (threads pt < 64)
    float nb = 0.f, na = 0.f;
    auto load_gates = [&](int m) {
      nb = 0.f;
      na = 0.f;
      const int tok0 = start + m * kC, L = min(kC, end - tok0);
      if (m < NC && pt < L) {
        nb = GV != 0 ? 1.f : p.beta[(size_t)(tok0 + pt) * p.H + h];
        if (GATE == 1) na = p.log_alpha[(size_t)(tok0 + pt) * p.H + h];
      }
    };
    // ---- P1 of chunk j: beta, in-chunk cumulative log-decay, per-row
    // factors, into gate buffer j % 3; prefetches the gates of chunk j+1
    auto p1 = [&](int j) {
      float *g = gS + (j % 3) * 64, *gc = gC + (j % 3) * 128;
      float *F = FT + (j % 3) * (F_COUNT * 64);
      float x = na, bb = nb;
      if (pt < 64) load_gates(j + 1);
      if (GATE != 2) {
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const float y = __shfl_up_sync(0xffffffffu, x, off);
          if (lane >= off) x += y;
        }
        if (pt == 31) *scan_tmp = x;
      }
      named_bar_sync(2, kPrep);
      if (pt < 64) {
        if (GATE != 2 && pt >= 32) x += *scan_tmp;
        if (GATE != 2) g[pt] = x;
        F[F_B * 64 + pt] = bb;
      }
      if (GATE != 2 && pt == 63) gc[0] = x;
      named_bar_sync(2, kPrep);
      // factors: E_r = e^{g_r - g_31}, F_r = e^{g_31 - g_r} (so that
      // e^{g_r - g_i} = E_r F_i without a per-element exponential; used
      // when the chunk's decay range keeps both within fp32), b e^g, e^g,
      // e^{g_C - g}
      if (GATE != 2 && pt < 64) {
        const float gr = x, gref = g[31], gcv = g[63];
        F[F_BG * 64 + pt] = bb * __expf(gr);
        F[F_E * 64 + pt] = __expf(gr - gref);
        F[F_F * 64 + pt] = __expf(gref - gr);
        F[F_EG * 64 + pt] = __expf(gr);
        F[F_EK * 64 + pt] = __expf(gcv - gr);
      }
    };
    if (pt < 64) load_gates(0);
    if (NC > 0) p1(0);
    for (int m = 0; m < NC; ++m) {
      const int s = m & 1, tok0 = start + m * kC, L = min(kC, end - tok0);
      uint8_t *stg = sm + OFF_STAGE + s * kStageBytes;
      float *g = gS + (m % 3) * 64, *gc = gC + (m % 3) * 128;
      float *F = FT + (m % 3) * (F_COUNT * 64);
      // ---- P2 (channel gate only): per key channel c, with g_m = g at row
      // 31: Q e^{g-g_m}, K e^{g-g_m}, K e^{g_m-g} (bf16)
      float amax = 0.f;
      if (GATE == 2) {
        if (!group_all(wait_bar(cx, B_FULL0 + s, (m >> 1) & 1) &&
                           wait_bar(cx, B_LAFULL, m & 1),
                       2, kPrep))
          break;
        // (a) per key channel c and half of the chunk, the running sum of
        // the log-decays over the half's rows, in place; each half's total
        // in TT (rows past the sequence end add nothing)
        {
          const int c = pt & 127, half = pt >> 7;
          float *la = reinterpret_cast<float *>(sm + Lay::LA) +
                      (c >> 6) * 4096 + (c & 63);
          float lv[32];   // all loads first: one latency, not 32
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int r = half * 32 + j;
            lv[j] = (r < L) ? la[r * 64] : 0.f;
          }
          float run = 0.f, lo = 0.f, hi = 0.f;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            run += lv[j];
            la[(half * 32 + j) * 64] = run;
            lo = fminf(lo, run);
            hi = fmaxf(hi, run);
          }
          reinterpret_cast<float *>(sm + Lay::TT)[half * 128 + c] = run;
          // largest |g - g_m| of this half: g - g_m = running sum - g_m in
          // the first half (g_m = its total), the running sum in the second
          const float ref = half ? 0.f : run;
          float bnd = fmaxf(fabsf(lo - ref), fabsf(hi - ref));
#pragma unroll
          for (int off = 16; off > 0; off >>= 1)
            bnd = fmaxf(bnd, __shfl_xor_sync(0xffffffffu, bnd, off));
          if (lane == 0)
            reinterpret_cast<float *>(sm + Lay::TT_WMAX)[warp - 6] = bnd;
        }
        named_bar_sync(2, kPrep);
        bool use16;
        {
          const float *wm = reinterpret_cast<const float *>(sm + Lay::TT_WMAX);
          float b = wm[0];
#pragma unroll
          for (int w8 = 1; w8 < 8; ++w8) b = fmaxf(b, wm[w8]);
          use16 = b <= kF16Range;   // same decision in every prep thread
          if (pt == 0) {
            reinterpret_cast<int *>(sm + Lay::TT_F16)[m & 1] = use16 ? 1 : 0;
            // beyond the fp16 window the rescaled operands fall back to
            // bf16, whose 8-bit significand does not keep the result within
            // the accuracy of the fp16 path: the call says so
            if (!use16) atomicOr(&g_fused_error, kErrRange);
          }
        }
        // (b) with g_m = g at row 31 (the first half's total): row r's
        // g_r - g_m is its running sum minus g_m in the first half, and its
        // running sum in the second.  Item = row r, 8 channels (16 bytes of
        // Q, K and K e^{g_m-g}); thread pt takes items pt + 256 u.
        // one loop per operand format (the choice is uniform per chunk)
        auto rescale = [&](auto h16) {
          constexpr bool kH = decltype(h16)::value;
          const float *gl = reinterpret_cast<const float *>(sm + Lay::LA);
          const float *T0 = reinterpret_cast<const float *>(sm + Lay::TT);
#pragma unroll 2
          for (int u = 0; u < 4; ++u) {
            const int item = pt + 256 * u, r = item >> 4, ch = item & 15;
            const int kb = ch >> 3, cc = ch & 7;
            const float4 *gp = reinterpret_cast<const float4 *>(
                gl + kb * 4096 + r * 64 + cc * 8);
            const float4 g0 = gp[0], g1 = gp[1];
            float x[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
            if (r < 32) {
              const float4 *tp = reinterpret_cast<const float4 *>(T0 + ch * 8);
              const float4 t0 = tp[0], t1 = tp[1];
              x[0] -= t0.x; x[1] -= t0.y; x[2] -= t0.z; x[3] -= t0.w;
              x[4] -= t1.x; x[5] -= t1.y; x[6] -= t1.z; x[7] -= t1.w;
            }
            const uint32_t off = kb * 16384 + sw128_chunk(r, cc);
            uint4 *qp = reinterpret_cast<uint4 *>(stg + off + 8192);
            uint4 *kp = reinterpret_cast<uint4 *>(stg + off);
            uint4 qv = *qp, kv = *kp, nv;
            uint32_t *qw = reinterpret_cast<uint32_t *>(&qv);
            uint32_t *kw = reinterpret_cast<uint32_t *>(&kv);
            uint32_t *knw = reinterpret_cast<uint32_t *>(&nv);
            // the key-side gate: erase gate on the read key (GV 1, the
            // M-side block) or rate on the write key (GV 2, K e^{g_m-g})
            float gk[8];
            if (GV != 0)
              load_gate8(gk, p.gk, (size_t)(tok0 + r) * p.H + h,
                         kb * 64 + cc * 8, r < L);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float ep0 = __expf(x[2 * e]), ep1 = __expf(x[2 * e + 1]);
              const float en0 = __expf(-x[2 * e]), en1 = __expf(-x[2 * e + 1]);
              float q0, q1, k0, k1;
              unpack_bf16(qw[e], q0, q1);
              unpack_bf16(kw[e], k0, k1);
              float kr0 = k0, kr1 = k1, kn0 = k0, kn1 = k1;
              if (GV == 1) {
                kr0 *= gk[2 * e];
                kr1 *= gk[2 * e + 1];
              } else if (GV == 2) {
                kn0 *= gk[2 * e];
                kn1 *= gk[2 * e + 1];
              }
              amax = fmaxf(amax, fmaxf(fmaxf(fabsf(q0), fabsf(q1)),
                                       fmaxf(fabsf(k0), fabsf(k1))));
              if (GV != 0)
                amax = fmaxf(amax, fmaxf(fmaxf(fabsf(kr0), fabsf(kr1)),
                                         fmaxf(fabsf(kn0), fabsf(kn1))));
              qw[e] = kH ? pack_f16(q0 * ep0, q1 * ep1)
                         : pack_bf16(q0 * ep0, q1 * ep1);
              kw[e] = kH ? pack_f16(kr0 * ep0, kr1 * ep1)
                         : pack_bf16(kr0 * ep0, kr1 * ep1);
              knw[e] = kH ? pack_f16(kn0 * en0, kn1 * en1)
                          : pack_bf16(kn0 * en0, kn1 * en1);
            }
            *qp = qv;
            *kp = kv;
            *reinterpret_cast<uint4 *>(sm + Lay::KN + kb * 8192 +
                                       sw128_chunk(r, cc)) = nv;
          }
        };
        if (use16) rescale(std::true_type{});
        else rescale(std::false_type{});
        {
          const float *T0 = reinterpret_cast<const float *>(sm + Lay::TT);
          // per-channel factors, one exponential each per chunk: e^{g_m};
          // e^{g_C} (decay of S) in gc; e^{g_C - g_m} in gM + 128
          if (pt < 128) {
            const float t0 = T0[pt], t1 = T0[128 + pt];
            gM[pt] = __expf(t0);
            gc[pt] = __expf(t0 + t1);
            gM[128 + pt] = __expf(t1);
          }
        }
        // the log-decay tile has been read: the next chunk's may land
        mbar_arrive(&bar[B_LAFREE]);
        fence_proxy_async_smem();
        mbar_arrive(&bar[B_KKREADY]);
      }
      // ---- P3: A (strictly lower, fp32 blocks) and P (lower, fp16 operand)
      if (!group_all(wait_bar(cx, B_KKDONE0 + s, (m >> 1) & 1), 2, kPrep))
        break;
      tc_fence_after();
      const bool fact = (GATE != 1) || (g[0] - g[63] < 80.f);
      {
        const int c0 = hf * 32;
        tmem_ld32(trow + ACC_KK + c0, v);
        tmem_wait_ld();
        const bool arow = (l < 64);
        const int r = arow ? l : l - 64;
        // A row: beta_r e^{g_r - g_i} (K K^T)_ri, i < r;
        // P row: e^{g_r - g_i} (Q K^T)_ri, i <= r
        const float br = arow ? ((r < L) ? F[F_B * 64 + r] : 0.f) : 1.f;
        const float gr = (GATE == 1) ? g[r] : 0.f;
        const bool use_f = (GATE == 1) && fact;
        const float sc = use_f ? br * F[F_E * 64 + r] : br;
        if (GATE == 1 && !fact) {
          // decay range too wide to factor: one exponential per element
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int i = c0 + j;
            const bool keep = arow ? (i < r) : (i <= r);
            v[j] = keep ? v[j] * __expf(gr - g[i]) * sc : 0.f;
          }
        } else {
#pragma unroll
          for (int j4 = 0; j4 < 8; ++j4) {
            const float4 f4 = use_f
                ? *reinterpret_cast<const float4 *>(F + F_F * 64 + c0 + 4 * j4)
                : make_float4(1.f, 1.f, 1.f, 1.f);
            const float fi[4] = {f4.x, f4.y, f4.z, f4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int j = 4 * j4 + e, i = c0 + j;
              // A rows are used below the diagonal only (the inverse never
              // reads i >= r), so only the P rows need the causal mask
              v[j] = (arow || i <= r) ? v[j] * fi[e] * sc : 0.f;
            }
          }
        }
        if (arow) {
#pragma unroll
          for (int half2 = 0; half2 < 2; ++half2) {
            const int cb = (c0 >> 4) + half2;
            if (cb <= (r >> 4)) {
              float4 *dst = reinterpret_cast<float4 *>(
                  AC + blk(r >> 4, cb) * kBS + (r & 15) * kRS);
#pragma unroll
              for (int e = 0; e < 4; ++e)
                dst[e] = make_float4(v[16 * half2 + 4 * e], v[16 * half2 + 4 * e + 1],
                                     v[16 * half2 + 4 * e + 2], v[16 * half2 + 4 * e + 3]);
            }
          }
        } else {
          uint8_t *ptl = sm + OFF_P + s * 8192;
#pragma unroll
          for (int ch = 0; ch < 4; ++ch)
            st_smem_v4(ptl + sw128_chunk(r, (c0 >> 3) + ch),
                       pack_f16(v[8 * ch + 0], v[8 * ch + 1]),
                       pack_f16(v[8 * ch + 2], v[8 * ch + 3]),
                       pack_f16(v[8 * ch + 4], v[8 * ch + 5]),
                       pack_f16(v[8 * ch + 6], v[8 * ch + 7]));
        }
      }
      named_bar_sync(2, kPrep);
      // ---- P4: T = (I + A)^-1.  Diagonal 16x16 blocks by forward
      // substitution (one thread per column), then the off-diagonal blocks
      // T_bc = -D_b sum_{c<=e<b} A_be T_ec on mma.sync (tf32), level by level.
      if (pt < 64) {
        const int bb = pt >> 4, j = pt & 15;
        const float *Ab = AC + blk(bb, bb) * kBS;
        float xs[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
          float acc0 = (r == j) ? 1.f : 0.f, acc1 = 0.f;
#pragma unroll
          for (int i = 0; i < r; ++i) {
            if (i & 1) acc1 -= Ab[r * kRS + i] * xs[i];
            else acc0 -= Ab[r * kRS + i] * xs[i];
          }
          xs[r] = acc0 + acc1;
        }
        float *Tb = TC + blk(bb, bb) * kBS;
#pragma unroll
        for (int r = 0; r < 16; ++r) Tb[r * kRS + j] = xs[r];
      }
      named_bar_sync(2, kPrep);
      // M_be = D_b A_be for the six blocks below the diagonal, in place
      if (pw < 6) {
        const int bb = (pw < 1) ? 1 : (pw < 3) ? 2 : 3;
        const int e = (pw < 1) ? 0 : (pw < 3) ? pw - 1 : pw - 3;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        mma16(TC + blk(bb, bb) * kBS, AC + blk(bb, e) * kBS, acc, lane);
        __syncwarp();
        store16(AC + blk(bb, e) * kBS, acc, 1.f, lane);
      }
      named_bar_sync(2, kPrep);
      // T_bc = -sum_{c<=e<b} M_be T_ec (T_cc = D_c), scheduled on the
      // dependency depth with partial sums kept in the T blocks:
      //   step 1: T10, T21, T32 = -M D, and P20 = M20 D0, P31 = M31 D1,
      //           P30 = M30 D0
      //   step 2: T20 = -(P20 + M21 T10), T31 = -(P31 + M32 T21),
      //           P30 += M31 T10
      //   step 3: T30 = -(P30 + M32 T20)
      // One task = one 8-column half of one block; a task reads only the
      // half it writes, and inputs that no task of its step writes.
      {
        // task (rb, cb, e): block T_{rb,cb} (or its partial sum) from
        // M_{rb,e} T_{e,cb}, negated or not, added to the stored partial
        auto run = [&](int rb, int cb, int e, bool neg, bool accum, int nt) {
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
          float *dst = TC + blk(rb, cb) * kBS;
          if (accum) load16_nt(dst, acc, lane, nt);
          mma16_nt(AC + blk(rb, e) * kBS, TC + blk(e, cb) * kBS, acc, lane,
                   nt);
          store16_nt(dst, acc, neg ? -1.f : 1.f, lane, nt);
        };
        const int b2 = pw >> 1, nt = pw & 1;
        // step 1: 12 half-tasks, T10, T21, T32 first
        if (b2 < 3) run(b2 + 1, b2, b2, true, false, nt);   // T_{b+1,b}
        else run(2, 0, 0, false, false, nt);                 // P20
        if (pw < 2) run(3, 1, 1, false, false, nt);          // P31
        else if (pw < 4) run(3, 0, 0, false, false, nt);     // P30
        named_bar_sync(2, kPrep);
        // step 2
        if (b2 == 0) run(2, 0, 1, true, true, nt);           // T20
        else if (b2 == 1) run(3, 1, 2, true, true, nt);      // T31
        else if (b2 == 2) run(3, 0, 1, false, true, nt);     // P30 += M31 T10
        named_bar_sync(2, kPrep);
        // step 3
        if (b2 == 0) run(3, 0, 2, true, true, nt);           // T30
      }
      // Channel gate: its single T-factor tile is rewritten only once U of
      // the previous chunk, its last reader, has completed (V free); U is
      // issued after W, so W done does not imply it.  Scalar / no gate: the
      // tiles alternate by chunk parity.
      if (GATE == 2) {
        if (!group_all(m == 0 || pt != 0 || wait_bar(cx, B_VFREE, (m - 1) & 1),
                       2, kPrep))
          break;
      } else {
        named_bar_sync(2, kPrep);
      }
      const uint32_t tpo = (m & 1) * Lay::TP_PAR;   // T-factor set
      // ---- T-factor operands: T diag(b e^g) (scalar / no gate) and
      // T diag(b), with T diag(b)'s bf16 residual tile (scalar / no gate).
      // Item (tile, row r, 16-byte chunk ch); consecutive threads take
      // consecutive rows.
      {
        if (GATE != 2) {
          // Thread = row r and two 8-column chunks; each T value feeds both
          // tiles.  All loads are issued before the first store.
          const int r = pt & 63, rb = r >> 4;
          float4 t[2][2], fg[2][2], fb[2][2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int ch = (pt >> 6) + 4 * u;
            if ((ch >> 1) <= rb) {
              const float4 *tsrc = reinterpret_cast<const float4 *>(
                  TC + blk(rb, ch >> 1) * kBS + (r & 15) * kRS + ((8 * ch) & 15));
              t[u][0] = tsrc[0];
              t[u][1] = tsrc[1];
            } else {
              t[u][0] = t[u][1] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
            fg[u][0] = *reinterpret_cast<const float4 *>(F + F_BG * 64 + 8 * ch);
            fg[u][1] = *reinterpret_cast<const float4 *>(F + F_BG * 64 + 8 * ch + 4);
            fb[u][0] = *reinterpret_cast<const float4 *>(F + F_B * 64 + 8 * ch);
            fb[u][1] = *reinterpret_cast<const float4 *>(F + F_B * 64 + 8 * ch + 4);
          }
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int ch = (pt >> 6) + 4 * u;
            const float tv[8] = {t[u][0].x, t[u][0].y, t[u][0].z, t[u][0].w,
                                 t[u][1].x, t[u][1].y, t[u][1].z, t[u][1].w};
            const float gv[8] = {fg[u][0].x, fg[u][0].y, fg[u][0].z, fg[u][0].w,
                                 fg[u][1].x, fg[u][1].y, fg[u][1].z, fg[u][1].w};
            const float bv[8] = {fb[u][0].x, fb[u][0].y, fb[u][0].z, fb[u][0].w,
                                 fb[u][1].x, fb[u][1].y, fb[u][1].z, fb[u][1].w};
            uint32_t gw[4], hw[4], lw[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              gw[e] = pack_bf16(tv[2 * e] * gv[2 * e], tv[2 * e + 1] * gv[2 * e + 1]);
              const float b0 = tv[2 * e] * bv[2 * e], b1 = tv[2 * e + 1] * bv[2 * e + 1];
              hw[e] = pack_bf16(b0, b1);
              float h0, h1;
              unpack_bf16(hw[e], h0, h1);
              lw[e] = pack_bf16(b0 - h0, b1 - h1);
            }
            const uint32_t o = sw128_chunk(r, ch);
            st_smem_v4(sm + Lay::TPG + tpo + o, gw[0], gw[1], gw[2], gw[3]);
            st_smem_v4(sm + Lay::TPB + tpo + o, hw[0], hw[1], hw[2], hw[3]);
            st_smem_v4(sm + Lay::TPB_LO + tpo + o, lw[0], lw[1], lw[2], lw[3]);
          }
        }
        constexpr int kTiles = 1;
#pragma unroll
        for (int it = pt; GATE == 2 && it < kTiles * 512; it += kPrep) {
          const int r = it & 63, rb = r >> 4, ch = (it >> 6) & 7;
          const bool tb = (GATE == 2) || (it >> 9) == 1;   // T diag(b)
          const float *fac = F + (tb ? F_B : F_BG) * 64;
          const int cb = ch >> 1;
          float t8[8];
          if (cb <= rb) {
            const float4 *tsrc = reinterpret_cast<const float4 *>(
                TC + blk(rb, cb) * kBS + (r & 15) * kRS + ((8 * ch) & 15));
            const float4 t0 = tsrc[0], t1 = tsrc[1];
            const float4 f0 = *reinterpret_cast<const float4 *>(fac + 8 * ch);
            const float4 f1 = *reinterpret_cast<const float4 *>(fac + 8 * ch + 4);
            t8[0] = t0.x * f0.x; t8[1] = t0.y * f0.y; t8[2] = t0.z * f0.z;
            t8[3] = t0.w * f0.w; t8[4] = t1.x * f1.x; t8[5] = t1.y * f1.y;
            t8[6] = t1.z * f1.z; t8[7] = t1.w * f1.w;
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) t8[e] = 0.f;
          }
          auto pk = [](float a, float b) {
            return GATE == 2 ? pack_f16(a, b) : pack_bf16(a, b);
          };
          uint32_t hw[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) hw[e] = pk(t8[2 * e], t8[2 * e + 1]);
          st_smem_v4(sm + (tb ? Lay::TPB : Lay::TPG) + tpo + sw128_chunk(r, ch),
                     hw[0], hw[1], hw[2], hw[3]);
          if (GATE != 2 && tb) {
            uint32_t lw[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              float h0, h1;
              unpack_bf16(hw[e], h0, h1);
              lw[e] = pack_bf16(t8[2 * e] - h0, t8[2 * e + 1] - h1);
            }
            st_smem_v4(sm + Lay::TPB_LO + sw128_chunk(r, ch), lw[0], lw[1],
                       lw[2], lw[3]);
          }
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&bar[B_TREADY]);
      // P1 of the next chunk while U and W run
      if (m + 1 < NC) p1(m + 1);
      // Q e^g (fp16, in place) while U and W run: K K^T of this chunk has
      // read the raw tile (P3 waited for it)
      if (GATE != 2) {
        constexpr int kIq = kC * 16 / kPrep;   // 4
        uint4 xq[kIq];
        float eq[kIq];
        uint32_t offq[kIq];
#pragma unroll
        for (int u = 0; u < kIq; ++u) {
          const int idx = pt + u * kPrep;
          const int r = idx >> 4, cc = idx & 15;
          offq[u] = (cc >> 3) * 16384 + 8192 + sw128_chunk(r, cc & 7);
          eq[u] = (GATE == 1) ? F[F_EG * 64 + r] : 1.f;
          xq[u] = *reinterpret_cast<const uint4 *>(stg + offq[u]);
        }
#pragma unroll
        for (int u = 0; u < kIq; ++u) {
          uint32_t *wq = reinterpret_cast<uint32_t *>(&xq[u]);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float a0, a1;
            unpack_bf16(wq[e], a0, a1);
            wq[e] = pack_f16(a0 * eq[u], a1 * eq[u]);
          }
          *reinterpret_cast<uint4 *>(stg + offq[u]) = xq[u];
        }
      }
      // ---- P5: -W^T operand; K e^{g_C - g} in place (fp16).  The tensor-
      // memory load of W is in flight while K is converted: v is read only
      // after the load's wait.
      if (!group_all(wait_bar(cx, B_WDONE, m & 1), 2, kPrep)) break;
      tc_fence_after();
      {
        const int c0 = hf * 32;
        tmem_ld32(trow + ACC_W + c0, v);
        if (GATE != 2) {
          // K e^{g_C - g}, fp16 in place: all four 16-byte chunks of a thread
          // are loaded before any is stored
          constexpr int kIt = kC * 16 / kPrep;   // 4
          uint4 xk[kIt];
          float ek[kIt];
          uint32_t off[kIt];
#pragma unroll
          for (int u = 0; u < kIt; ++u) {
            const int idx = pt + u * kPrep;
            const int r = idx >> 4, cc = idx & 15;
            off[u] = (cc >> 3) * 16384 + sw128_chunk(r, cc & 7);
            ek[u] = (GATE == 1) ? F[F_EK * 64 + r] : 1.f;
            xk[u] = *reinterpret_cast<const uint4 *>(stg + off[u]);
          }
#pragma unroll
          for (int u = 0; u < kIt; ++u) {
            uint32_t *wk = reinterpret_cast<uint32_t *>(&xk[u]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              float a0, a1;
              unpack_bf16(wk[e], a0, a1);
              wk[e] = pack_f16(a0 * ek[u], a1 * ek[u]);
            }
            *reinterpret_cast<uint4 *>(stg + off[u]) = xk[u];
          }
        }
        tmem_wait_ld();
#pragma unroll
        for (int ch = 0; ch < 4; ++ch)
          st_smem_v4(sm + OFF_NW + sw128_chunk(l, (c0 >> 3) + ch),
                     pack_f16(-v[8 * ch + 0], -v[8 * ch + 1]),
                     pack_f16(-v[8 * ch + 2], -v[8 * ch + 3]),
                     pack_f16(-v[8 * ch + 4], -v[8 * ch + 5]),
                     pack_f16(-v[8 * ch + 6], -v[8 * ch + 7]));
      }
      const bool kn16 =
          GATE == 2 && reinterpret_cast<const int *>(sm + Lay::TT_F16)[m & 1];
      auto ktilde = [&](auto h16) {
        constexpr bool kH = decltype(h16)::value;
#pragma unroll 2
        for (int idx = pt; GATE == 2 && idx < kC * 16; idx += kPrep) {
          const int r = idx >> 4, cc = idx & 15, kb = cc >> 3;
          uint8_t *kp = stg + kb * 16384 + sw128_chunk(r, cc & 7);
          // K~ = (K e^{g_m-g}) e^{g_C-g_m}, per channel (8 factors, two
          // vector loads)
          const float4 *fp = reinterpret_cast<const float4 *>(gM + 128 + cc * 8);
          const float4 f0 = fp[0], f1 = fp[1];
          const float f[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
          uint4 kv = *reinterpret_cast<const uint4 *>(
              sm + Lay::KN + kb * 8192 + sw128_chunk(r, cc & 7));
          uint32_t *kw = reinterpret_cast<uint32_t *>(&kv);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float a0, a1;
            if (kH) unpack_f16(kw[e], a0, a1);
            else unpack_bf16(kw[e], a0, a1);
            kw[e] = pack_f16(a0 * f[2 * e], a1 * f[2 * e + 1]);
          }
          *reinterpret_cast<uint4 *>(kp) = kv;
        }
      };
      if (kn16) ktilde(std::true_type{});
      else ktilde(std::false_type{});
      if (!(amax <= kF16Max)) atomicOr(&g_fused_error, kErrRange);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bar[B_WREADY]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType,
                                  cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr,
                                cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// [ntok][H][128], box of 64 channels x 1 head x 64 tokens: bf16 with the
// 128-B swizzle (q, k, v), or fp32 unswizzled (per-channel log-decays)
bool make_map(CUtensorMap *map, const void *base, int ntok, int H,
              bool f32 = false) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t es_bytes = f32 ? 4 : 2;
  const cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)H,
                              (cuuint64_t)(ntok > 0 ? ntok : 1)};
  const cuuint64_t strides[2] = {(cuuint64_t)kD * es_bytes,
                                 (cuuint64_t)H * kD * es_bytes};
  const cuuint32_t box[3] = {64, 1, (cuuint32_t)kC};
  const cuuint32_t es[3] = {1, 1, 1};
  return enc(map,
             f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
             3, const_cast<void *>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE,
             f32 ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int GATE, int GV>
cudaError_t launch(const Problem &pr, const float *gk, const float *gv,
                   cudaStream_t s) {
  CUtensorMap mq, mk, mv, mla, mgk, mgv;
  if (!make_map(&mq, pr.q, pr.ntok, pr.H) || !make_map(&mk, pr.k, pr.ntok, pr.H) ||
      !make_map(&mv, pr.v, pr.ntok, pr.H))
    return cudaErrorInvalidValue;
  // the channel gate's log-decays; the other gates never read this map
  if (GATE == 2 ? !make_map(&mla, pr.log_alpha, pr.ntok, pr.H, true)
                : !make_map(&mla, pr.q, pr.ntok, pr.H))
    return cudaErrorInvalidValue;
  // the gate variants' gate tensors (fp32, the layout of the log-decays);
  // a map the kernel never reads describes q
  if (!(GV != 0 ? make_map(&mgk, gk, pr.ntok, pr.H, true)
                : make_map(&mgk, pr.q, pr.ntok, pr.H)) ||
      !(GV != 0 && gv ? make_map(&mgv, gv, pr.ntok, pr.H, true)
                      : make_map(&mgv, pr.q, pr.ntok, pr.H)))
    return cudaErrorInvalidValue;
  Params p;
  p.beta = pr.beta;
  p.gk = gk;
  p.gv = gv;
  p.log_alpha = pr.log_alpha;
  p.s0 = pr.s0;
  p.out = static_cast<__nv_bfloat16 *>(pr.out);
  p.sT = pr.sT;
  p.cu = pr.cu;
  p.nseq = pr.nseq;
  p.T = pr.T;
  p.ntok = pr.ntok;
  p.H = pr.H;
  const int smem = Layout<GATE>::BYTES + 1024;
  cudaError_t e = cudaFuncSetAttribute(
      gdr_fused_tc_kernel<GATE, GV>,
      cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  gdr_fused_tc_kernel<GATE, GV><<<pr.nseq * pr.H, kThreads, smem, s>>>(
      mq, mk, mv, mla, mgk, mgv, p);
  return cudaGetLastError();
}

// The per-channel gate variants run on the channel-gate kernel; a scalar or
// absent decay is handed to it as the channel-wise decay with every channel
// equal (log-decays expanded into scratch, [ntok][H][128] fp32).
__global__ void expand_log_decay_kernel(const float *__restrict__ la,
                                        float *__restrict__ out, long long n4) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n4) return;
  const long long row = i / (kD / 4);   // (token, head)
  const float x = la ? la[row] : 0.f;
  reinterpret_cast<float4 *>(out)[i] = make_float4(x, x, x, x);
}

bool variant_needs_expand(const Problem &p) {
  return (p.erase || p.write || p.wkey) && p.gate != GDR_GATE_CHANNEL;
}

}  // namespace

bool fused_tc_applies(const Problem &p) {
  return p.dtype == GDR_BF16 && p.dk == kD && p.dv == kD && p.chunk == kC &&
         (long long)p.nseq * p.H < (1ll << 31);
}

size_t fused_tc_scratch_bytes(const Problem &p) {
  return variant_needs_expand(p) ? (size_t)p.ntok * p.H * kD * sizeof(float)
                                 : 0;
}

cudaError_t fused_tc_run(const Problem &p, void *scratch, cudaStream_t s) {
  if (variant_needs_expand(p)) {
    if (!scratch) return cudaErrorInvalidValue;
    float *la = static_cast<float *>(scratch);
    const long long n4 = (long long)p.ntok * p.H * (kD / 4);
    if (n4 > 0) {
      const int bs = 256;
      expand_log_decay_kernel<<<(unsigned)((n4 + bs - 1) / bs), bs, 0, s>>>(
          p.gate == GDR_GATE_SCALAR ? p.log_alpha : nullptr, la, n4);
    }
    Problem pc = p;
    pc.gate = GDR_GATE_CHANNEL;
    pc.log_alpha = la;
    return fused_tc_run(pc, nullptr, s);
  }
  if (p.erase) return launch<2, 1>(p, p.erase, p.write, s);
  if (p.wkey) return launch<2, 2>(p, p.wkey, p.write, s);
  switch (p.gate) {
    case GDR_GATE_NONE: return launch<0, 0>(p, nullptr, nullptr, s);
    case GDR_GATE_SCALAR: return launch<1, 0>(p, nullptr, nullptr, s);
    default: return launch<2, 0>(p, nullptr, nullptr, s);
  }
}

cudaError_t fused_tc_read_error(unsigned *word, bool clear) {
  cudaError_t e = cudaMemcpyFromSymbol(word, g_fused_error, sizeof(unsigned));
  if (e != cudaSuccess) return e;
  if (clear && *word) {
    const unsigned zero = 0;
    e = cudaMemcpyToSymbol(g_fused_error, &zero, sizeof(unsigned));
  }
  return e;
}

}  // namespace gdr
