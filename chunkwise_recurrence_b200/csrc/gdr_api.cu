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
      o.algo != GDR_ALGO_FUSED_TC)
    return GDR_ERR_INVALID_ARGUMENT;
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
gdr_status scratch_alloc(void **ptr, size_t bytes, cudaStream_t s) {
  *ptr = nullptr;
  const char *inj = std::getenv("GDR_FAULT_INJECT_ALLOC");
  if (inj && inj[0] == '1') return GDR_ERR_OUT_OF_MEMORY;
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
    cudaError_t e = gdr::fused_tc_run(p, stream);
    return e == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
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

  const size_t esz = o.dtype == GDR_FP32 ? 4 : 2;
  const size_t th = (size_t)p.ntok * p.H;
  const size_t gdim = o.gate == GDR_GATE_NONE     ? 0
                      : o.gate == GDR_GATE_SCALAR ? 1
                                                  : (size_t)dk;
  const size_t state = (size_t)p.nseq * H * dk * dv * sizeof(float);
  struct Buf {
    const void *host;
    void *dev;
    size_t bytes;
    bool in, out;
  } bufs[] = {
      {q, nullptr, th * dk * esz, true, false},
      {k, nullptr, th * dk * esz, true, false},
      {v, nullptr, th * dv * esz, true, false},
      {log_alpha, nullptr, log_alpha ? th * gdim * sizeof(float) : 0, true,
       false},
      {beta, nullptr, th * sizeof(float), true, false},
      {initial_state, nullptr, initial_state ? state : 0, true, false},
      {o.cu_seqlens, nullptr,
       o.cu_seqlens ? ((size_t)p.nseq + 1) * sizeof(int32_t) : 0, true,
       false},
      {out, nullptr, th * dv * esz, false, true},
      {final_state, nullptr, final_state ? state : 0, false, true},
  };
  const int nb = sizeof(bufs) / sizeof(bufs[0]);
  size_t total = 0, offs[nb];
  for (int i = 0; i < nb; ++i) {
    offs[i] = total;
    total += (bufs[i].bytes + 255) & ~size_t(255);
  }
  void *block = nullptr;
  st = scratch_alloc(&block, total, stream);
  if (st != GDR_OK) return st;
  char *base = static_cast<char *>(block);
  for (int i = 0; i < nb; ++i) {
    if (!bufs[i].host || bufs[i].bytes == 0) continue;
    bufs[i].dev = base + offs[i];
    if (bufs[i].in &&
        cudaMemcpyAsync(bufs[i].dev, bufs[i].host, bufs[i].bytes,
                        cudaMemcpyHostToDevice, stream) != cudaSuccess) {
      cudaFreeAsync(block, stream);
      return GDR_ERR_CUDA;
    }
  }
  Problem pd = p;
  pd.q = bufs[0].dev;
  pd.k = bufs[1].dev;
  pd.v = bufs[2].dev;
  pd.log_alpha = static_cast<const float *>(bufs[3].dev);
  pd.beta = static_cast<const float *>(bufs[4].dev);
  pd.s0 = static_cast<const float *>(bufs[5].dev);
  pd.cu = static_cast<const int32_t *>(bufs[6].dev);
  pd.out = bufs[7].dev;
  pd.sT = static_cast<float *>(bufs[8].dev);
  st = run(pd, o.algo, stream);
  if (st == GDR_OK) {
    for (int i = 0; i < nb; ++i) {
      if (!bufs[i].out || !bufs[i].dev) continue;
      if (cudaMemcpyAsync(const_cast<void *>(bufs[i].host), bufs[i].dev,
                          bufs[i].bytes, cudaMemcpyDeviceToHost,
                          stream) != cudaSuccess) {
        st = GDR_ERR_CUDA;
        break;
      }
    }
  }
  if (cudaFreeAsync(block, stream) != cudaSuccess && st == GDR_OK)
    st = GDR_ERR_CUDA;
  return st;
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

extern "C" gdr_status gdr_device_error(cudaStream_t stream, int clear) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return GDR_ERR_CUDA;
  unsigned word = 0;
  if (gdr::fused_tc_read_error(&word, clear != 0) != cudaSuccess)
    return GDR_ERR_CUDA;
  if (word & 0xFFFFu) return GDR_ERR_TIMEOUT;   // an mbarrier wait expired
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
