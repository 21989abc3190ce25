// Host side of libgdr's C ABI: argument checks, scratch management, dispatch
// to the staged or the fused tensor-core kernels, and the host-buffer entry.
//
// Every check runs before the first CUDA call, so a rejected call has no side
// effect and the checks can be exercised on a machine without a GPU.

#include <climits>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "gdr_internal.h"

namespace {

using gdr::Problem;

bool aligned16(const void *p) {
  return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

bool pow2_in(int x, int lo, int hi) {
  return x >= lo && x <= hi && (x & (x - 1)) == 0;
}

gdr_opts default_opts() {
  gdr_opts o;
  o.dtype = GDR_BF16;
  o.gate = GDR_GATE_SCALAR;
  o.cu_seqlens = nullptr;
  o.num_seqs = 0;
  o.algo = GDR_ALGO_AUTO;
  return o;
}

// Fills `p` from the arguments, or returns the reason they are rejected.
gdr_status validate(const void *q, const void *k, const void *v,
                    const float *log_alpha, const float *beta,
                    const float *initial_state, const void *out,
                    const float *final_state, int B, int T, int H, int dk,
                    int dv, int chunk, const gdr_opts &o, Problem *p) {
  if (B < 0 || T < 0 || H < 0) return GDR_ERR_INVALID_ARGUMENT;
  if (o.dtype != GDR_BF16 && o.dtype != GDR_FP32)
    return GDR_ERR_INVALID_ARGUMENT;
  if (o.gate != GDR_GATE_NONE && o.gate != GDR_GATE_SCALAR &&
      o.gate != GDR_GATE_CHANNEL)
    return GDR_ERR_INVALID_ARGUMENT;
  if (o.algo != GDR_ALGO_AUTO && o.algo != GDR_ALGO_STAGED &&
      o.algo != GDR_ALGO_FUSED_TC && o.algo != GDR_ALGO_RECURRENT)
    return GDR_ERR_INVALID_ARGUMENT;
  // the reverse token recurrence is a backward algorithm only
  if (o.algo == GDR_ALGO_RECURRENT) return GDR_ERR_UNSUPPORTED;
  if (!pow2_in(dk, 16, 128) || !pow2_in(dv, 16, 128) ||
      !pow2_in(chunk, 16, 64))
    return GDR_ERR_UNSUPPORTED;
  const bool varlen = o.cu_seqlens != nullptr;
  if (varlen && (B != 1 || o.num_seqs < 0)) return GDR_ERR_INVALID_ARGUMENT;
  if (!varlen && o.num_seqs != 0) return GDR_ERR_INVALID_ARGUMENT;
  // sizes: every flat index must fit comfortably in 64 bits and the token
  // count in an int
  const long long ntok = varlen ? (long long)T : (long long)B * T;
  if (ntok > INT_MAX / 2) return GDR_ERR_UNSUPPORTED;
  if (H > 65535) return GDR_ERR_UNSUPPORTED;       // grid.y limit
  const int nseq = varlen ? o.num_seqs : B;
  if ((o.gate == GDR_GATE_NONE) != (log_alpha == nullptr))
    return GDR_ERR_INVALID_ARGUMENT;
  const bool empty = (nseq == 0 || H == 0);
  if (!empty) {
    if (!q || !k || !v || !beta || !out) return GDR_ERR_INVALID_ARGUMENT;
    const void *ptrs[] = {q, k, v, log_alpha, beta, initial_state, out,
                          final_state, o.cu_seqlens};
    for (const void *ptr : ptrs)
      if (ptr && !aligned16(ptr)) return GDR_ERR_INVALID_ARGUMENT;
  }
  p->q = q;
  p->k = k;
  p->v = v;
  p->log_alpha = log_alpha;
  p->beta = beta;
  p->s0 = initial_state;
  p->out = const_cast<void *>(out);
  p->sT = const_cast<float *>(final_state);
  p->cu = o.cu_seqlens;
  p->nseq = nseq;
  p->T = T;
  p->ntok = (int)ntok;
  p->H = H;
  p->dk = dk;
  p->dv = dv;
  p->chunk = chunk;
  p->dtype = o.dtype;
  p->gate = o.gate;
  // upper bound on the chunk count: B * ceil(T / C) for fixed length; for
  // varlen sum_n ceil(L_n / C) <= floor(ntok / C) + nseq
  p->max_chunks = varlen ? (int)(ntok / chunk) + nseq
                         : B * ((T + chunk - 1) / chunk);
  return GDR_OK;
}

// Scratch allocation with a host-side failure hook: GDR_FAULT_INJECT_ALLOC=1
// in the environment makes every scratch allocation fail before any CUDA
// call (used by the failure-handling tests).
bool alloc_fault_injected() {
  const char *inj = std::getenv("GDR_FAULT_INJECT_ALLOC");
  return inj && inj[0] == '1';
}

gdr_status scratch_alloc(void **ptr, size_t bytes, cudaStream_t s) {
  *ptr = nullptr;
  if (alloc_fault_injected()) return GDR_ERR_OUT_OF_MEMORY;
  if (bytes == 0) return GDR_OK;
  cudaError_t e = cudaMallocAsync(ptr, bytes, s);
  if (e == cudaErrorMemoryAllocation) {
    (void)cudaGetLastError();
    return GDR_ERR_OUT_OF_MEMORY;
  }
  return e == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

gdr_status run(const Problem &p, gdr_algo algo, cudaStream_t stream) {
  if (p.nseq == 0 || p.H == 0) return GDR_OK;
  const bool tc = gdr::fused_tc_applies(p);
  if (algo == GDR_ALGO_FUSED_TC && !tc) return GDR_ERR_UNSUPPORTED;
  if (tc && algo != GDR_ALGO_STAGED) {
    // (the gate variants with a scalar or no decay take their log-decays
    // expanded per channel, in scratch)
    const size_t bytes = gdr::fused_tc_scratch_bytes(p);
    void *ws = nullptr;
    if (bytes) {
      gdr_status st = scratch_alloc(&ws, bytes, stream);
      if (st != GDR_OK) return st;
    }
    cudaError_t e = gdr::fused_tc_run(p, ws, stream);
    cudaError_t f = ws ? cudaFreeAsync(ws, stream) : cudaSuccess;
    return (e == cudaSuccess && f == cudaSuccess) ? GDR_OK : GDR_ERR_CUDA;
  }
  void *ws = nullptr;
  gdr_status st = scratch_alloc(&ws, gdr::staged_workspace_bytes(p), stream);
  if (st != GDR_OK) return st;
  cudaError_t e = gdr::staged_run(p, ws, stream);
  cudaError_t f = cudaFreeAsync(ws, stream);
  if (e != cudaSuccess || f != cudaSuccess) return GDR_ERR_CUDA;
  return GDR_OK;
}

}  // namespace

extern "C" gdr_status gdr_chunk_fwd(const void *q, const void *k,
                                    const void *v, const float *log_alpha,
                                    const float *beta,
                                    const float *initial_state, void *out,
                                    float *final_state, int B, int T, int H,
                                    int dk, int dv, int chunk,
                                    cudaStream_t stream,
                                    const gdr_opts *opts) {
  const gdr_opts o = opts ? *opts : default_opts();
  Problem p;
  gdr_status st = validate(q, k, v, log_alpha, beta, initial_state, out,
                           final_state, B, T, H, dk, dv, chunk, o, &p);
  if (st != GDR_OK) return st;
  return run(p, o.algo, stream);
}

// Gated DeltaNet-2 gates (erase on the read key, write on the target), on
// the staged path: see gdr.h.
extern "C" gdr_status gdr_chunk_fwd_gdn2(const void *q, const void *k,
                                         const void *v, const float *log_alpha,
                                         const float *erase_gate,
                                         const float *write_gate,
                                         const float *initial_state, void *out,
                                         float *final_state, int B, int T,
                                         int H, int dk, int dv, int chunk,
                                         cudaStream_t stream,
                                         const gdr_opts *opts) {
  const gdr_opts o = opts ? *opts : default_opts();
  Problem p;
  // the erase gate stands in for beta in the common checks (presence,
  // alignment); the write gate is checked here
  gdr_status st = validate(q, k, v, log_alpha, erase_gate, initial_state, out,
                           final_state, B, T, H, dk, dv, chunk, o, &p);
  if (st != GDR_OK) return st;
  if (p.nseq == 0 || p.H == 0) return GDR_OK;
  if (!write_gate || !aligned16(write_gate)) return GDR_ERR_INVALID_ARGUMENT;
  p.beta = nullptr;
  p.erase = erase_gate;
  p.write = write_gate;
  return run(p, o.algo, stream);
}

// FG^2-GDN's per-key-channel rate on the write key (and FG^2-GDN+'s
// per-value-channel target scaling), on the staged path: see gdr.h.
extern "C" gdr_status gdr_chunk_fwd_fg2(const void *q, const void *k,
                                        const void *v, const float *log_alpha,
                                        const float *beta_k,
                                        const float *beta_v,
                                        const float *initial_state, void *out,
                                        float *final_state, int B, int T,
                                        int H, int dk, int dv, int chunk,
                                        cudaStream_t stream,
                                        const gdr_opts *opts) {
  const gdr_opts o = opts ? *opts : default_opts();
  Problem p;
  // the key-side rate stands in for beta in the common checks (presence,
  // alignment); the optional value-side scaling is checked here
  gdr_status st = validate(q, k, v, log_alpha, beta_k, initial_state, out,
                           final_state, B, T, H, dk, dv, chunk, o, &p);
  if (st != GDR_OK) return st;
  if (p.nseq == 0 || p.H == 0) return GDR_OK;
  if (beta_v && !aligned16(beta_v)) return GDR_ERR_INVALID_ARGUMENT;
  p.beta = nullptr;
  p.wkey = beta_k;
  p.write = beta_v;
  return run(p, o.algo, stream);
}

// ---------------------------------------------------------------------------
// Host-buffer entry.  The work is cut into up to kHostPieces pieces, each
// with its own device buffers.  Three streams overlap the pieces: the
// host-to-device copies of piece i+1 (upload stream) run while piece i
// computes (the caller's stream) and the results of piece i-1 come back
// (download stream), so the host link carries both directions at once and
// the kernels hide behind the copies.  Fixed-length batches are cut by time,
// at chunk boundaries: a piece holds the same token range of every sequence
// and starts from the state the previous piece ended with (kept on the
// device), so the last piece -- the part that cannot hide behind an upload --
// is a few chunks long.  The results are those of one call: the state passes
// from piece to piece in fp32, exactly as from chunk to chunk.  Packed
// batches are cut into pieces of whole sequences.
namespace {

constexpr int kHostPieces = 8;

// Per-device resources of the host entry, created on first use and kept for
// the life of the process: a memory pool that keeps its memory between calls
// (repeated calls then reuse it instead of mapping and unmapping device
// memory every time), and the two copy streams.
struct HostCtx {
  cudaMemPool_t pool = nullptr;
  cudaStream_t up = nullptr, down = nullptr;
};
constexpr int kMaxHostDevices = 64;
std::mutex g_host_mu;
HostCtx g_host_ctx[kMaxHostDevices];

gdr_status host_ctx(HostCtx *out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return GDR_ERR_CUDA;
  if (dev < 0 || dev >= kMaxHostDevices) return GDR_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_host_mu);
  HostCtx &c = g_host_ctx[dev];
  if (!c.pool) {
    cudaMemPoolProps props;
    std::memset(&props, 0, sizeof(props));
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t pool = nullptr;
    if (cudaMemPoolCreate(&pool, &props) != cudaSuccess) return GDR_ERR_CUDA;
    uint64_t keep = UINT64_MAX;
    cudaStream_t up = nullptr, down = nullptr;
    if (cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold,
                                &keep) != cudaSuccess ||
        cudaStreamCreateWithFlags(&up, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&down, cudaStreamNonBlocking) !=
            cudaSuccess) {
      if (up) cudaStreamDestroy(up);
      cudaMemPoolDestroy(pool);
      return GDR_ERR_CUDA;
    }
    c.pool = pool;
    c.up = up;
    c.down = down;
  }
  *out = c;
  return GDR_OK;
}

// Token offsets of one piece, relative to its first sequence.
__global__ void rebase_offsets_kernel(const int32_t *src, int32_t *dst,
                                      int nseq) {
  const int32_t base = src[0];
  for (int j = threadIdx.x; j <= nseq; j += blockDim.x) dst[j] = src[j] - base;
}

// Events of one call, destroyed when the call returns (a destroyed event
// that is still pending is released by the runtime once it completes).
struct EventSet {
  cudaEvent_t ev[2 * kHostPieces + 3] = {};
  int n = 0;
  cudaEvent_t make() {
    cudaEvent_t e = nullptr;
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess)
      return nullptr;
    ev[n++] = e;
    return e;
  }
  ~EventSet() {
    for (int i = 0; i < n; ++i) cudaEventDestroy(ev[i]);
  }
};

}  // namespace

namespace {

// Fixed-length host entry, cut by time (see above).
gdr_status host_by_time(const Problem &p, const gdr_opts &o, const void *q,
                        const void *k, const void *v, const float *log_alpha,
                        const float *beta, const float *initial_state,
                        void *out, float *final_state, cudaStream_t stream) {
  const int B = p.nseq, T = p.T, C = p.chunk;
  const int nck = (T + C - 1) / C;
  const int P = nck < kHostPieces ? nck : kHostPieces;
  int tb[kHostPieces + 1];   // token boundaries, multiples of C
  for (int i = 0; i < P; ++i) tb[i] = (int)((long long)nck * i / P) * C;
  tb[P] = T;
  const size_t esz = o.dtype == GDR_FP32 ? 4 : 2;
  const size_t gdim = o.gate == GDR_GATE_NONE     ? 0
                      : o.gate == GDR_GATE_SCALAR ? 1
                                                  : (size_t)p.dk;
  const size_t state1 = (size_t)p.H * p.dk * p.dv * sizeof(float);
  // per-token bytes, in the order q k v log_alpha beta out
  const size_t tok_bytes[6] = {
      (size_t)p.H * p.dk * esz, (size_t)p.H * p.dk * esz,
      (size_t)p.H * p.dv * esz,
      log_alpha ? (size_t)p.H * gdim * sizeof(float) : 0,
      (size_t)p.H * sizeof(float), (size_t)p.H * p.dv * esz};
  const void *host_in[5] = {q, k, v, log_alpha, beta};
  auto up256 = [](size_t x) { return (x + 255) & ~size_t(255); };
  enum { BQ, BK, BV, BLA, BB, BOUT, NBUF };
  size_t off[kHostPieces][NBUF];
  // the initial state, then two states that the pieces pass on in turn
  size_t total = 0;
  const size_t off_s0 = total;
  total += initial_state ? up256((size_t)B * state1) : 0;
  const size_t off_st[2] = {total, total + up256((size_t)B * state1)};
  total += 2 * up256((size_t)B * state1);
  for (int i = 0; i < P; ++i) {
    const size_t nt = (size_t)B * (tb[i + 1] - tb[i]);
    for (int b = 0; b < NBUF; ++b) {
      off[i][b] = total;
      total += up256(nt * tok_bytes[b]);
    }
  }

  if (alloc_fault_injected()) return GDR_ERR_OUT_OF_MEMORY;
  HostCtx hc;
  gdr_status st = host_ctx(&hc);
  if (st != GDR_OK) return st;
  EventSet evs;
  cudaEvent_t ev_start = evs.make(), ev_up_end = evs.make(),
              ev_down_end = evs.make();
  cudaEvent_t ev_in[kHostPieces], ev_run[kHostPieces];
  for (int i = 0; i < P; ++i) {
    ev_in[i] = evs.make();
    ev_run[i] = evs.make();
  }
  if (evs.n != 3 + 2 * P) return GDR_ERR_CUDA;
  void *block = nullptr;
  {
    cudaError_t e = cudaMallocFromPoolAsync(&block, total, hc.pool, stream);
    if (e == cudaErrorMemoryAllocation) {
      (void)cudaGetLastError();
      return GDR_ERR_OUT_OF_MEMORY;
    }
    if (e != cudaSuccess) return GDR_ERR_CUDA;
  }
  char *base = static_cast<char *>(block);
  auto ok = [&](cudaError_t e) {
    if (e != cudaSuccess && st == GDR_OK) st = GDR_ERR_CUDA;
    return st == GDR_OK;
  };
  ok(cudaEventRecord(ev_start, stream));
  ok(cudaStreamWaitEvent(hc.up, ev_start, 0));
  if (initial_state)
    ok(cudaMemcpyAsync(base + off_s0, initial_state, (size_t)B * state1,
                       cudaMemcpyHostToDevice, hc.up));
  for (int i = 0; i < P && st == GDR_OK; ++i) {
    const size_t t0 = tb[i], tp = tb[i + 1] - tb[i];
    char *pb[NBUF];
    for (int b = 0; b < NBUF; ++b) pb[b] = base + off[i][b];
    // inputs of piece i: tokens [t0, t0 + tp) of every sequence
    for (int b = BQ; b <= BB; ++b)
      if (host_in[b] && tok_bytes[b])
        ok(cudaMemcpy2DAsync(pb[b], tp * tok_bytes[b],
                             static_cast<const char *>(host_in[b]) +
                                 t0 * tok_bytes[b],
                             (size_t)T * tok_bytes[b], tp * tok_bytes[b], B,
                             cudaMemcpyHostToDevice, hc.up));
    ok(cudaEventRecord(ev_in[i], hc.up));
    if (st != GDR_OK) break;
    ok(cudaStreamWaitEvent(stream, ev_in[i], 0));
    Problem pp = p;
    pp.q = pb[BQ];
    pp.k = pb[BK];
    pp.v = pb[BV];
    pp.log_alpha = log_alpha ? reinterpret_cast<const float *>(pb[BLA])
                             : nullptr;
    pp.beta = reinterpret_cast<const float *>(pb[BB]);
    pp.s0 = i == 0 ? (initial_state
                          ? reinterpret_cast<const float *>(base + off_s0)
                          : nullptr)
                   : reinterpret_cast<const float *>(base + off_st[(i - 1) & 1]);
    pp.sT = reinterpret_cast<float *>(base + off_st[i & 1]);
    pp.out = pb[BOUT];
    pp.T = (int)tp;
    pp.ntok = (int)(B * tp);
    pp.cu = nullptr;
    pp.max_chunks = B * (int)((tp + C - 1) / C);
    const gdr_status rs = run(pp, o.algo, stream);
    if (rs != GDR_OK) {
      st = rs;
      break;
    }
    ok(cudaEventRecord(ev_run[i], stream));
    // results of piece i
    ok(cudaStreamWaitEvent(hc.down, ev_run[i], 0));
    ok(cudaMemcpy2DAsync(static_cast<char *>(out) + t0 * tok_bytes[BOUT],
                         (size_t)T * tok_bytes[BOUT], pb[BOUT],
                         tp * tok_bytes[BOUT], tp * tok_bytes[BOUT], B,
                         cudaMemcpyDeviceToHost, hc.down));
    if (final_state && i == P - 1)
      ok(cudaMemcpyAsync(final_state, base + off_st[i & 1], (size_t)B * state1,
                         cudaMemcpyDeviceToHost, hc.down));
  }
  gdr_status fin = GDR_OK;
  auto fin_ok = [&](cudaError_t e) {
    if (e != cudaSuccess) fin = GDR_ERR_CUDA;
  };
  fin_ok(cudaEventRecord(ev_up_end, hc.up));
  fin_ok(cudaEventRecord(ev_down_end, hc.down));
  fin_ok(cudaStreamWaitEvent(stream, ev_up_end, 0));
  fin_ok(cudaStreamWaitEvent(stream, ev_down_end, 0));
  fin_ok(cudaFreeAsync(block, stream));
  return st != GDR_OK ? st : fin;
}

}  // namespace

extern "C" gdr_status gdr_chunk_fwd_host(const void *q, const void *k,
                                         const void *v, const float *log_alpha,
                                         const float *beta,
                                         const float *initial_state, void *out,
                                         float *final_state, int B, int T,
                                         int H, int dk, int dv, int chunk,
                                         cudaStream_t stream,
                                         const gdr_opts *opts) {
  const gdr_opts o = opts ? *opts : default_opts();
  Problem p;
  gdr_status st = validate(q, k, v, log_alpha, beta, initial_state, out,
                           final_state, B, T, H, dk, dv, chunk, o, &p);
  if (st != GDR_OK) return st;
  if (p.nseq == 0 || p.H == 0) return GDR_OK;
  if (o.cu_seqlens == nullptr && p.T > chunk)
    return host_by_time(p, o, q, k, v, log_alpha, beta, initial_state, out,
                        final_state, stream);

  // host offsets are read here, so that every piece is exact
  const bool varlen = o.cu_seqlens != nullptr;
  const int32_t *hcu = o.cu_seqlens;
  if (varlen) {
    if (hcu[0] != 0 || hcu[p.nseq] != p.ntok) return GDR_ERR_INVALID_ARGUMENT;
    for (int n = 0; n < p.nseq; ++n)
      if (hcu[n + 1] < hcu[n]) return GDR_ERR_INVALID_ARGUMENT;
  }
  auto first_token = [&](int n) -> long long {
    return varlen ? hcu[n] : (long long)n * p.T;
  };

  // pieces: sequence boundaries sb[], about ntok / P tokens each, at least
  // one sequence each
  const int P = p.nseq < kHostPieces ? p.nseq : kHostPieces;
  int sb[kHostPieces + 1];
  sb[0] = 0;
  sb[P] = p.nseq;
  for (int i = 1; i < P; ++i) {
    const long long target = (long long)p.ntok * i / P;
    int n = sb[i - 1] + 1;
    while (n < p.nseq - (P - i) && first_token(n) < target) ++n;
    sb[i] = n;
  }

  // device layout: the caller's offsets (varlen), then per piece its inputs
  // and outputs, every buffer 256-byte aligned
  const size_t esz = o.dtype == GDR_FP32 ? 4 : 2;
  const size_t gdim = o.gate == GDR_GATE_NONE     ? 0
                      : o.gate == GDR_GATE_SCALAR ? 1
                                                  : (size_t)dk;
  const size_t state1 = (size_t)H * dk * dv * sizeof(float);
  // per-token bytes of each tensor, in the order q k v log_alpha beta out
  const size_t tok_bytes[6] = {
      (size_t)H * dk * esz, (size_t)H * dk * esz, (size_t)H * dv * esz,
      log_alpha ? (size_t)H * gdim * sizeof(float) : 0,
      (size_t)H * sizeof(float), (size_t)H * dv * esz};
  const void *host_in[5] = {q, k, v, log_alpha, beta};
  auto up256 = [](size_t x) { return (x + 255) & ~size_t(255); };
  enum { BQ, BK, BV, BLA, BB, BOUT, BS0, BST, BCU, NBUF };
  size_t off[kHostPieces][NBUF];
  size_t total = varlen ? up256(((size_t)p.nseq + 1) * sizeof(int32_t)) : 0;
  for (int i = 0; i < P; ++i) {
    const size_t nt = first_token(sb[i + 1]) - first_token(sb[i]);
    const size_t ns = sb[i + 1] - sb[i];
    const size_t bytes[NBUF] = {
        nt * tok_bytes[0], nt * tok_bytes[1], nt * tok_bytes[2],
        nt * tok_bytes[3], nt * tok_bytes[4], nt * tok_bytes[5],
        initial_state ? ns * state1 : 0, final_state ? ns * state1 : 0,
        varlen ? (ns + 1) * sizeof(int32_t) : 0};
    for (int b = 0; b < NBUF; ++b) {
      off[i][b] = total;
      total += up256(bytes[b]);
    }
  }

  if (alloc_fault_injected()) return GDR_ERR_OUT_OF_MEMORY;
  HostCtx hc;
  st = host_ctx(&hc);
  if (st != GDR_OK) return st;
  EventSet evs;
  cudaEvent_t ev_start = evs.make(), ev_up_end = evs.make(),
              ev_down_end = evs.make();
  cudaEvent_t ev_in[kHostPieces], ev_run[kHostPieces];
  for (int i = 0; i < P; ++i) {
    ev_in[i] = evs.make();
    ev_run[i] = evs.make();
  }
  if (evs.n != 3 + 2 * P) return GDR_ERR_CUDA;
  void *block = nullptr;
  {
    cudaError_t e = cudaMallocFromPoolAsync(&block, total, hc.pool, stream);
    if (e == cudaErrorMemoryAllocation) {
      (void)cudaGetLastError();
      return GDR_ERR_OUT_OF_MEMORY;
    }
    if (e != cudaSuccess) return GDR_ERR_CUDA;
  }
  char *base = static_cast<char *>(block);
  auto ok = [&](cudaError_t e) {
    if (e != cudaSuccess && st == GDR_OK) st = GDR_ERR_CUDA;
    return st == GDR_OK;
  };

  // the upload stream starts after the caller's earlier work (and the
  // allocation) on `stream`
  ok(cudaEventRecord(ev_start, stream));
  ok(cudaStreamWaitEvent(hc.up, ev_start, 0));
  if (varlen)
    ok(cudaMemcpyAsync(base, hcu, ((size_t)p.nseq + 1) * sizeof(int32_t),
                       cudaMemcpyHostToDevice, hc.up));
  for (int i = 0; i < P && st == GDR_OK; ++i) {
    const long long t0 = first_token(sb[i]), t1 = first_token(sb[i + 1]);
    const int s0 = sb[i], ns = sb[i + 1] - sb[i];
    char *pb[NBUF];
    for (int b = 0; b < NBUF; ++b) pb[b] = base + off[i][b];
    // inputs of piece i
    for (int b = BQ; b <= BB; ++b)
      if (host_in[b] && tok_bytes[b])
        ok(cudaMemcpyAsync(pb[b],
                           static_cast<const char *>(host_in[b]) +
                               t0 * tok_bytes[b],
                           (t1 - t0) * tok_bytes[b], cudaMemcpyHostToDevice,
                           hc.up));
    if (initial_state)
      ok(cudaMemcpyAsync(pb[BS0],
                         reinterpret_cast<const char *>(initial_state) +
                             s0 * state1,
                         ns * state1, cudaMemcpyHostToDevice, hc.up));
    ok(cudaEventRecord(ev_in[i], hc.up));
    if (st != GDR_OK) break;
    // compute on the caller's stream
    ok(cudaStreamWaitEvent(stream, ev_in[i], 0));
    Problem pp = p;
    pp.q = pb[BQ];
    pp.k = pb[BK];
    pp.v = pb[BV];
    pp.log_alpha = log_alpha ? reinterpret_cast<const float *>(pb[BLA])
                             : nullptr;
    pp.beta = reinterpret_cast<const float *>(pb[BB]);
    pp.s0 = initial_state ? reinterpret_cast<const float *>(pb[BS0]) : nullptr;
    pp.out = pb[BOUT];
    pp.sT = final_state ? reinterpret_cast<float *>(pb[BST]) : nullptr;
    pp.nseq = ns;
    pp.ntok = (int)(t1 - t0);
    if (varlen) {
      int32_t *cu = reinterpret_cast<int32_t *>(pb[BCU]);
      rebase_offsets_kernel<<<1, 256, 0, stream>>>(
          reinterpret_cast<const int32_t *>(base) + s0, cu, ns);
      if (!ok(cudaGetLastError())) break;
      pp.cu = cu;
      pp.T = pp.ntok;
      pp.max_chunks = pp.ntok / p.chunk + ns;
    } else {
      pp.cu = nullptr;
      pp.max_chunks = ns * ((p.T + p.chunk - 1) / p.chunk);
    }
    const gdr_status rs = run(pp, o.algo, stream);
    if (rs != GDR_OK) {
      st = rs;
      break;
    }
    ok(cudaEventRecord(ev_run[i], stream));
    // results of piece i
    ok(cudaStreamWaitEvent(hc.down, ev_run[i], 0));
    ok(cudaMemcpyAsync(static_cast<char *>(out) + t0 * tok_bytes[BOUT],
                       pb[BOUT], (t1 - t0) * tok_bytes[BOUT],
                       cudaMemcpyDeviceToHost, hc.down));
    if (final_state)
      ok(cudaMemcpyAsync(reinterpret_cast<char *>(final_state) + s0 * state1,
                         pb[BST], ns * state1, cudaMemcpyDeviceToHost,
                         hc.down));
  }
  // the caller's stream waits for both copy streams, then releases the
  // block; this runs on every path once the allocation has succeeded
  gdr_status fin = GDR_OK;
  auto fin_ok = [&](cudaError_t e) {
    if (e != cudaSuccess) fin = GDR_ERR_CUDA;
  };
  fin_ok(cudaEventRecord(ev_up_end, hc.up));
  fin_ok(cudaEventRecord(ev_down_end, hc.down));
  fin_ok(cudaStreamWaitEvent(stream, ev_up_end, 0));
  fin_ok(cudaStreamWaitEvent(stream, ev_down_end, 0));
  fin_ok(cudaFreeAsync(block, stream));
  return st != GDR_OK ? st : fin;
}

// ---------------------------------------------------------------------------
// No-allocation entry: the staged kernels with their scratch in a static
// device array instead of a stream-ordered allocation.  Host code cannot use
// the array's name as a device address (in host code it names a host-side
// stand-in), so each device's address is looked up once with
// cudaGetSymbolAddress while that device is current, and cached.
static __device__ __align__(256) unsigned char
    g_noalloc_scratch[GDR_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[kMaxDevices];

gdr_status noalloc_scratch(void **ptr) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return GDR_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return GDR_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p)
      return GDR_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *ptr = g_noalloc_ptr[dev];
  return GDR_OK;
}

}  // namespace

extern "C" gdr_status gdr_chunk_fwd_noalloc(
    const void *q, const void *k, const void *v, const float *log_alpha,
    const float *beta, const float *initial_state, void *out,
    float *final_state, int B, int T, int H, int dk, int dv, int chunk,
    cudaStream_t stream, const gdr_opts *opts) {
  const gdr_opts o = opts ? *opts : default_opts();
  Problem p;
  gdr_status st = validate(q, k, v, log_alpha, beta, initial_state, out,
                           final_state, B, T, H, dk, dv, chunk, o, &p);
  if (st != GDR_OK) return st;
  if (o.algo == GDR_ALGO_FUSED_TC) return GDR_ERR_UNSUPPORTED;
  if (p.nseq == 0 || p.H == 0) return GDR_OK;
  if (gdr::staged_workspace_bytes(p) > GDR_NOALLOC_SCRATCH_BYTES)
    return GDR_ERR_UNSUPPORTED;
  void *scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st != GDR_OK) return st;
  return gdr::staged_run(p, scratch, stream) == cudaSuccess ? GDR_OK
                                                            : GDR_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Context-parallel forward pass: every sequence is cut into segments of whole
// chunks; the segments' state maps (M, N) are computed in parallel, combined
// in order per sequence, and a final pass runs every segment from its true
// initial state.
extern "C" gdr_status gdr_chunk_fwd_segmented(
    const void *q, const void *k, const void *v, const float *log_alpha,
    const float *beta, const float *initial_state, void *out,
    float *final_state, int B, int T, int H, int dk, int dv, int chunk,
    int segments, cudaStream_t stream, const gdr_opts *opts) {
  const gdr_opts o = opts ? *opts : default_opts();
  if (segments < 1) return GDR_ERR_INVALID_ARGUMENT;
  Problem p;
  gdr_status st = validate(q, k, v, log_alpha, beta, initial_state, out,
                           final_state, B, T, H, dk, dv, chunk, o, &p);
  if (st != GDR_OK) return st;
  if (p.nseq == 0 || p.H == 0) return GDR_OK;
  const int nseq = p.nseq;
  // sequence offsets on the host (packed batches: one synchronous read)
  std::vector<int64_t> cu(nseq + 1);
  if (p.cu) {
    std::vector<int32_t> hcu(nseq + 1);
    if (cudaMemcpyAsync(hcu.data(), p.cu, (nseq + 1) * sizeof(int32_t),
                        cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess)
      return GDR_ERR_CUDA;
    if (hcu[0] != 0 || hcu[nseq] != p.ntok) return GDR_ERR_INVALID_ARGUMENT;
    for (int i = 0; i <= nseq; ++i) {
      if (i > 0 && hcu[i] < hcu[i - 1]) return GDR_ERR_INVALID_ARGUMENT;
      cu[i] = hcu[i];
    }
  } else {
    for (int i = 0; i <= nseq; ++i) cu[i] = (int64_t)i * T;
  }
  // the plan: sequence n of L tokens = ceil(L / chunk) chunks, cut into at
  // most `segments` pieces of equally many whole chunks
  std::vector<int32_t> seg_cu(1, 0), seg_first(nseq + 1, 0), seg_last(nseq);
  int nseg = 0;
  for (int n = 0; n < nseq; ++n) {
    seg_first[n] = nseg;
    const int64_t L = cu[n + 1] - cu[n];
    const int64_t nch = (L + chunk - 1) / chunk;
    const int64_t pieces = nch < segments ? nch : segments;
    const int64_t per = pieces > 0 ? (nch + pieces - 1) / pieces : 0;
    for (int64_t a = 0; a < L; a += per * chunk) {
      const int64_t e = a + per * chunk < L ? a + per * chunk : L;
      seg_cu.back() = (int32_t)(cu[n] + a);
      seg_cu.push_back((int32_t)(cu[n] + e));
      ++nseg;
    }
    seg_last[n] = nseg - 1;
  }
  seg_first[nseq] = nseg;
  // seg_cu holds nseg + 1 offsets; consecutive segments share boundaries
  // except across empty sequences, where the next start equals the end
  const size_t ss = (size_t)dk * dv, sk2 = (size_t)dk * dk;
  const size_t esz = p.dtype == GDR_FP32 ? 4 : 2;
  auto up256 = [](size_t x) { return (x + 255) & ~(size_t)255; };
  const size_t b_cu = up256((size_t)(nseg + 1) * 4);
  const size_t b_first = up256((size_t)(nseq + 1) * 4);
  const size_t b_zero = up256((size_t)p.ntok * H * dk * esz);
  const size_t b_otmp = up256((size_t)p.ntok * H * (dk > dv ? dk : dv) * esz);
  const size_t b_sq = up256((size_t)nseg * H * sk2 * 4);   // eye, Ms
  const size_t b_st = up256((size_t)nseg * H * ss * 4);    // Ns, Sin, Sfin
  const size_t total = b_cu + b_first + b_zero + b_otmp + 2 * b_sq + 3 * b_st;
  if (alloc_fault_injected()) return GDR_ERR_OUT_OF_MEMORY;
  HostCtx hc;
  st = host_ctx(&hc);
  if (st != GDR_OK) return st;
  void *block = nullptr;
  {
    cudaError_t e = cudaMallocFromPoolAsync(&block, total, hc.pool, stream);
    if (e == cudaErrorMemoryAllocation) {
      (void)cudaGetLastError();
      return GDR_ERR_OUT_OF_MEMORY;
    }
    if (e != cudaSuccess) return GDR_ERR_CUDA;
  }
  char *c = static_cast<char *>(block);
  int32_t *d_cu = reinterpret_cast<int32_t *>(c); c += b_cu;
  int32_t *d_first = reinterpret_cast<int32_t *>(c); c += b_first;
  void *zero_v = c; c += b_zero;
  void *otmp = c; c += b_otmp;
  float *eye = reinterpret_cast<float *>(c); c += b_sq;
  float *Ms = reinterpret_cast<float *>(c); c += b_sq;
  float *Ns = reinterpret_cast<float *>(c); c += b_st;
  float *Sin = reinterpret_cast<float *>(c); c += b_st;
  float *Sfin = reinterpret_cast<float *>(c);
  auto ok = [&](cudaError_t e) {
    if (e != cudaSuccess && st == GDR_OK) st = GDR_ERR_CUDA;
    return st == GDR_OK;
  };
  // the host vectors are pageable: these copies complete before returning
  ok(cudaMemcpyAsync(d_cu, seg_cu.data(), (nseg + 1) * sizeof(int32_t),
                     cudaMemcpyHostToDevice, stream));
  ok(cudaMemcpyAsync(d_first, seg_first.data(), (nseq + 1) * sizeof(int32_t),
                     cudaMemcpyHostToDevice, stream));
  if (nseg > 0 && st == GDR_OK) {
    // the segment problem: the same token axis, segments as sequences
    Problem sp = p;
    sp.cu = d_cu;
    sp.nseq = nseg;
    sp.T = p.ntok;
    sp.max_chunks = p.ntok / chunk + nseg;
    // pass M: transitions, from S = I with v = 0 (dv' = dk)
    Problem pm = sp;
    pm.v = zero_v;
    pm.dv = dk;
    pm.s0 = eye;
    pm.out = otmp;
    pm.sT = Ms;
    ok(cudaMemsetAsync(zero_v, 0, (size_t)p.ntok * H * dk * esz, stream));
    ok(gdr::fill_identity(eye, (long long)nseg * H, dk, stream));
    if (st == GDR_OK) st = run(pm, o.algo, stream);
    // pass N: offsets, from S = 0
    Problem pn = sp;
    pn.s0 = nullptr;
    pn.out = otmp;
    pn.sT = Ns;
    if (st == GDR_OK) st = run(pn, o.algo, stream);
    // in order per sequence: each segment's initial state
    if (st == GDR_OK)
      ok(gdr::segment_combine(p.s0, Ms, Ns, Sin, d_first, nseq, H, dk, dv,
                              stream));
    // pass C: every segment from its initial state: out, segment finals
    Problem pc = sp;
    pc.s0 = Sin;
    pc.sT = Sfin;
    if (st == GDR_OK) st = run(pc, o.algo, stream);
  }
  // final states: the last segment's, or the initial state of an empty
  // sequence
  if (final_state && st == GDR_OK) {
    const size_t bytes = (size_t)H * ss * sizeof(float);
    for (int n = 0; n < nseq && st == GDR_OK; ++n) {
      float *dst = final_state + (size_t)n * H * ss;
      if (seg_first[n + 1] > seg_first[n])
        ok(cudaMemcpyAsync(dst, Sfin + (size_t)seg_last[n] * H * ss, bytes,
                           cudaMemcpyDeviceToDevice, stream));
      else if (p.s0)
        ok(cudaMemcpyAsync(dst, p.s0 + (size_t)n * H * ss, bytes,
                           cudaMemcpyDeviceToDevice, stream));
      else
        ok(cudaMemsetAsync(dst, 0, bytes, stream));
    }
  }
  const cudaError_t f = cudaFreeAsync(block, stream);
  if (st == GDR_OK && f != cudaSuccess) st = GDR_ERR_CUDA;
  return st;
}

namespace {

// gdr_backward, gdr_backward_gdn2 and gdr_backward_fg2: with erase the
// Gated DeltaNet-2 gates (erase, write) replace beta, with wkey FG^2-GDN's
// rate (and, when write is given, FG^2-GDN+'s value scaling); their
// gradients go to d_erase / d_wkey and d_write (the chunked backward only).
gdr_status backward_entry(const void *q, const void *k, const void *v,
                          const float *log_alpha, const float *beta,
                          const float *erase, const float *write,
                          const float *wkey, const float *initial_state,
                          const void *d_out, const float *d_final_state,
                          float *dq, float *dk, float *dv, float *d_log_alpha,
                          float *d_beta, float *d_erase, float *d_write,
                          float *d_wkey, float *d_initial_state, int B, int T,
                          int H, int dk_, int dv_, cudaStream_t stream,
                          const gdr_opts *opts) {
  const gdr_opts o = opts ? *opts : default_opts();
  const bool gates = erase != nullptr || wkey != nullptr;
  const float *key_gate = erase ? erase : wkey;
  if (o.algo == GDR_ALGO_FUSED_TC) return GDR_ERR_UNSUPPORTED;
  const bool recurrent = o.algo == GDR_ALGO_RECURRENT;
  if (recurrent && gates) return GDR_ERR_UNSUPPORTED;
  gdr_opts ov = o;
  if (recurrent) ov.algo = GDR_ALGO_AUTO;
  Problem p;
  // the forward pass's checks, with d_out in the place of out and
  // d_final_state in the place of final_state (the chunked backward runs
  // chunks of 64 tokens whatever the forward used); the erase gate stands in
  // for beta with the gates
  gdr_status st = validate(q, k, v, log_alpha, gates ? key_gate : beta,
                           initial_state, d_out, d_final_state, B, T, H, dk_,
                           dv_, 64, ov, &p);
  if (st != GDR_OK) return st;
  if (p.nseq == 0 || p.H == 0) return GDR_OK;
  if (!dq || !dk || !dv) return GDR_ERR_INVALID_ARGUMENT;
  if (!gates && !d_beta) return GDR_ERR_INVALID_ARGUMENT;
  if (erase && (!write || !d_erase || !d_write))
    return GDR_ERR_INVALID_ARGUMENT;
  if (wkey && (!d_wkey || (write != nullptr) != (d_write != nullptr)))
    return GDR_ERR_INVALID_ARGUMENT;
  if ((o.gate == GDR_GATE_NONE) != (d_log_alpha == nullptr))
    return GDR_ERR_INVALID_ARGUMENT;
  const void *ptrs[] = {dq, dk, dv, d_log_alpha, d_beta, d_initial_state,
                        write, d_erase, d_write, d_wkey};
  for (const void *ptr : ptrs)
    if (ptr && !aligned16(ptr)) return GDR_ERR_INVALID_ARGUMENT;
  // AUTO and STAGED: the chunked backward (the faster of the two on every
  // measured shape); RECURRENT: the reverse token recurrence
  const bool chunked = !recurrent && gdr::backward_chunked_applies(p);
  if (gates && !chunked) return GDR_ERR_UNSUPPORTED;
  if (gates) {
    p.beta = nullptr;
    p.erase = erase;
    p.write = write;
    p.wkey = wkey;
  }
  long long total_win = 0;
  const size_t bytes = chunked ? gdr::backward_chunked_bytes(p)
                               : gdr::backward_scratch_bytes(p, &total_win);
  // the scratch comes from the library's per-device pool, which keeps its
  // memory between calls (hundreds of MB at training sizes: mapping it anew
  // every call would cost more than the copies it saves)
  if (alloc_fault_injected()) return GDR_ERR_OUT_OF_MEMORY;
  HostCtx hc;
  st = host_ctx(&hc);
  if (st != GDR_OK) return st;
  void *ws = nullptr;
  {
    cudaError_t e = cudaMallocFromPoolAsync(&ws, bytes, hc.pool, stream);
    if (e == cudaErrorMemoryAllocation) {
      (void)cudaGetLastError();
      return GDR_ERR_OUT_OF_MEMORY;
    }
    if (e != cudaSuccess) return GDR_ERR_CUDA;
  }
  gdr::BackwardIO io;
  io.dout = d_out;
  io.dsT = d_final_state;
  io.dq = dq;
  io.dk = dk;
  io.dv = dv;
  io.dla = d_log_alpha;
  io.dbeta = gates ? nullptr : d_beta;
  io.ds0 = d_initial_state;
  io.derase = erase ? d_erase : nullptr;
  io.dwrite = write ? d_write : nullptr;
  io.dwkey = wkey ? d_wkey : nullptr;
  cudaError_t e =
      chunked ? gdr::backward_chunked_run(p, io, ws, stream)
              : gdr::backward_run(p, io, static_cast<float *>(ws), total_win,
                                  stream);
  cudaError_t f = cudaFreeAsync(ws, stream);
  return (e == cudaSuccess && f == cudaSuccess) ? GDR_OK : GDR_ERR_CUDA;
}

}  // namespace

extern "C" gdr_status gdr_backward(
    const void *q, const void *k, const void *v, const float *log_alpha,
    const float *beta, const float *initial_state, const void *d_out,
    const float *d_final_state, float *dq, float *dk, float *dv,
    float *d_log_alpha, float *d_beta, float *d_initial_state, int B, int T,
    int H, int dk_, int dv_, cudaStream_t stream, const gdr_opts *opts) {
  return backward_entry(q, k, v, log_alpha, beta, nullptr, nullptr, nullptr,
                        initial_state, d_out, d_final_state, dq, dk, dv,
                        d_log_alpha, d_beta, nullptr, nullptr, nullptr,
                        d_initial_state, B, T, H, dk_, dv_, stream, opts);
}

extern "C" gdr_status gdr_backward_gdn2(
    const void *q, const void *k, const void *v, const float *log_alpha,
    const float *erase_gate, const float *write_gate,
    const float *initial_state, const void *d_out,
    const float *d_final_state, float *dq, float *dk, float *dv,
    float *d_log_alpha, float *d_erase, float *d_write,
    float *d_initial_state, int B, int T, int H, int dk_, int dv_,
    cudaStream_t stream, const gdr_opts *opts) {
  if (!erase_gate || !write_gate) return GDR_ERR_INVALID_ARGUMENT;
  return backward_entry(q, k, v, log_alpha, nullptr, erase_gate, write_gate,
                        nullptr, initial_state, d_out, d_final_state, dq, dk,
                        dv, d_log_alpha, nullptr, d_erase, d_write, nullptr,
                        d_initial_state, B, T, H, dk_, dv_, stream, opts);
}

extern "C" gdr_status gdr_backward_fg2(
    const void *q, const void *k, const void *v, const float *log_alpha,
    const float *beta_k, const float *beta_v, const float *initial_state,
    const void *d_out, const float *d_final_state, float *dq, float *dk,
    float *dv, float *d_log_alpha, float *d_beta_k, float *d_beta_v,
    float *d_initial_state, int B, int T, int H, int dk_, int dv_,
    cudaStream_t stream, const gdr_opts *opts) {
  if (!beta_k) return GDR_ERR_INVALID_ARGUMENT;
  return backward_entry(q, k, v, log_alpha, nullptr, nullptr, beta_v, beta_k,
                        initial_state, d_out, d_final_state, dq, dk, dv,
                        d_log_alpha, nullptr, nullptr, d_beta_v, d_beta_k,
                        d_initial_state, B, T, H, dk_, dv_, stream, opts);
}

extern "C" gdr_status gdr_device_error(cudaStream_t stream, int clear) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return GDR_ERR_CUDA;
  unsigned word = 0;
  if (gdr::fused_tc_read_error(&word, clear != 0) != cudaSuccess)
    return GDR_ERR_CUDA;
  unsigned dword = 0;   // the decode step's bulk copy never completed
  if (gdr::decode_read_error(&dword, clear != 0) != cudaSuccess)
    return GDR_ERR_CUDA;
  if ((word & 0xFFFFFFu) || dword) return GDR_ERR_TIMEOUT;  // a wait expired
  return word ? GDR_ERR_RANGE : GDR_OK;
}

extern "C" int gdr_algo_applies(gdr_algo algo, gdr_dtype dtype,
                                gdr_gate gate, int dk, int dv, int chunk) {
  if (!pow2_in(dk, 16, 128) || !pow2_in(dv, 16, 128) ||
      !pow2_in(chunk, 16, 64))
    return 0;
  if (dtype != GDR_BF16 && dtype != GDR_FP32) return 0;
  if (gate != GDR_GATE_NONE && gate != GDR_GATE_SCALAR &&
      gate != GDR_GATE_CHANNEL)
    return 0;
  if (algo == GDR_ALGO_AUTO || algo == GDR_ALGO_STAGED) return 1;
  if (algo != GDR_ALGO_FUSED_TC) return 0;
  Problem p;
  std::memset(&p, 0, sizeof(p));
  p.dtype = dtype;
  p.gate = gate;
  p.dk = dk;
  p.dv = dv;
  p.chunk = chunk;
  return gdr::fused_tc_applies(p) ? 1 : 0;
}

extern "C" const char *gdr_status_string(gdr_status s) {
  switch (s) {
    case GDR_OK: return "GDR_OK";
    case GDR_ERR_INVALID_ARGUMENT: return "GDR_ERR_INVALID_ARGUMENT";
    case GDR_ERR_UNSUPPORTED: return "GDR_ERR_UNSUPPORTED";
    case GDR_ERR_CUDA: return "GDR_ERR_CUDA";
    case GDR_ERR_OUT_OF_MEMORY: return "GDR_ERR_OUT_OF_MEMORY";
    case GDR_ERR_TIMEOUT: return "GDR_ERR_TIMEOUT";
    case GDR_ERR_RANGE: return "GDR_ERR_RANGE";
  }
  return "GDR_ERR_UNKNOWN";
}
