// Internal declarations shared by the host API and the kernel files of libgdr.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "gdr.h"

namespace gdr {

// One chunk of one sequence: tokens [tok0, tok0 + len), sequence `seq`.
struct ChunkInfo {
  int tok0;
  int len;
  int seq;
  int pad;
};

// Problem description after host validation.  Token index tok runs over the
// flattened [B*T] (fixed length) or packed [T] (varlen) token axis; element
// (tok, h, c) of a [.., H, d] tensor sits at (tok * H + h) * d + c.
struct Problem {
  const void *q, *k, *v;
  const float *log_alpha, *beta, *s0;
  void *out;
  float *sT;
  const int32_t *cu;  // device, nseq+1 entries, or nullptr (fixed length)
  int nseq;           // number of sequences (B, or num_seqs)
  int T;              // per-sequence length (fixed) / packed total (varlen)
  int ntok;           // total tokens
  int H, dk, dv, chunk;
  gdr_dtype dtype;
  gdr_gate gate;
  int max_chunks;     // upper bound on the number of chunks over all sequences
  // Gated DeltaNet-2 gates (staged path, the fused channel-gate kernel, the
  // chunked backward; nullptr otherwise): the per-key-channel erase gate
  // [ntok][H][dk] and per-value-channel write gate [ntok][H][dv] that
  // replace beta
  const float *erase = nullptr, *write = nullptr;
  // FG^2-GDN's per-key-channel rate [ntok][H][dk] (staged path, the fused
  // channel-gate kernel; nullptr otherwise): the write key of token t is
  // wkey_t . k_t and the read key k_t; `write` (or nullptr for ones) then
  // scales the target
  const float *wkey = nullptr;
};

// Staged path: four kernels + a chunk-table kernel, fp32 CUDA-core math.
size_t staged_workspace_bytes(const Problem &p);
cudaError_t staged_run(const Problem &p, void *workspace, cudaStream_t s);
// The staged path's scratch regions inside a workspace of
// staged_workspace_bytes(p) bytes: the chunk table, per-sequence first chunk
// (nseq + 1 entries; the last is the chunk count), in-chunk cumulative
// log-decays g [ntok][H][gdim], W [ntok][H][dk], U and V_new [ntok][H][dv],
// chunk-start states [max_chunks][H][dk][dv].
struct StagedBufs {
  ChunkInfo *table;
  int *seq_first, *nchunks;
  float *g, *W, *U, *Vn, *Sbuf;
};
StagedBufs staged_bufs(const Problem &p, void *workspace);
// The staged path's chunk table and in-chunk cumulative log-decays g only.
cudaError_t staged_chunks_run(const Problem &p, void *workspace,
                              cudaStream_t s);

// Fused tensor-core path.
bool fused_tc_applies(const Problem &p);
// scratch fused_tc_run needs (bytes; 0 for most problems: the gate variants
// with a scalar or no decay take their log-decays expanded per channel)
size_t fused_tc_scratch_bytes(const Problem &p);
cudaError_t fused_tc_run(const Problem &p, void *scratch, cudaStream_t s);
// Reads (and optionally clears) the fused kernel's sticky device error word.
cudaError_t fused_tc_read_error(unsigned *word, bool clear);

// Context-parallel state passing (csrc/segmented.cu): for each sequence n,
// walk its segments seg_first[n] .. seg_first[n+1]-1 in order, writing each
// segment's initial state into Sin and advancing S <- M_s S + N_s; S starts
// from s0[n] (or zero).  Ms [nseg][H][dk][dk], Ns and Sin [nseg][H][dk][dv].
cudaError_t segment_combine(const float *s0, const float *Ms, const float *Ns,
                            float *Sin, const int32_t *seg_first, int nseq,
                            int H, int dk, int dv, cudaStream_t s);
// eye[i] = I (dk x dk) for nstates consecutive states.
cudaError_t fill_identity(float *eye, long long nstates, int dk,
                          cudaStream_t s);

// Decode step: reads (and optionally clears) its sticky device error word
// (a bulk copy that never completed).
cudaError_t decode_read_error(unsigned *word, bool clear);

// Backward pass (csrc/backward.cu): upstream gradients in, gradients out.
struct BackwardIO {
  const void *dout;      // dL/d out, layout of out, dtype of the problem
  const float *dsT;      // dL/d final_state [N][H][dk][dv], or nullptr
  float *dq, *dk, *dv;   // fp32, layouts of q, k, v
  float *dla;            // fp32, layout of log_alpha (nullptr for no gate)
  float *dbeta;          // fp32 [ntok][H]
  float *ds0;            // fp32 [N][H][dk][dv], or nullptr
  // Gated DeltaNet-2 gates' gradients (chunked backward; the gates are the
  // Problem's erase / write): layouts of k and v, or nullptr
  float *derase = nullptr, *dwrite = nullptr;
  // FG^2-GDN's rate gradient (the Problem's wkey): layout of k, or nullptr
  float *dwkey = nullptr;
};
// Chunked backward pass (csrc/backward_chunked.cu): the gradients of the
// chunked forward product by product, fp32, chunk-parallel except for one
// forward and one reverse scan over the chunk boundaries.  p.chunk must be 64.
bool backward_chunked_applies(const Problem &p);
size_t backward_chunked_bytes(const Problem &p);
cudaError_t backward_chunked_run(const Problem &p, const BackwardIO &io,
                                 void *workspace, cudaStream_t s);
// Scratch the backward pass needs (bytes); *total_win = the number of
// checkpoint windows per head, to pass on to backward_run.
size_t backward_scratch_bytes(const Problem &p, long long *total_win);
cudaError_t backward_run(const Problem &p, const BackwardIO &io,
                         float *scratch, long long total_win, cudaStream_t s);

}  // namespace gdr
