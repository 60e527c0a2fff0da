// Launch-side interface between the C ABI (api.cu) and the kernels. Host-only declarations.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "compkv.h"

namespace compkv {

constexpr int kBlockTokensHost = 16;  // the only supported block size

struct SummariesArgs {
  bool bf16;
  bool fp16_summ;  // mean_k / mean_v stored as fp16
  int B, Hkv, T, D, Nb, r;
  const void* K;
  const void* V;
  const int32_t* ctx_lens;
  void* mean_k;
  float* var_g;
  void* mean_v;
  int32_t* count;
};

struct AppendArgs {
  bool bf16;
  bool fp16_summ;  // mean_k / mean_v stored as fp16
  int pairs, Hkv, T, D, Nb, r;
  const void* k_new;
  const void* v_new;
  const int32_t* positions;
  void* K;
  void* V;
  void* mean_k;
  float* var_g;
  void* mean_v;
  int32_t* count;
  int32_t* status;
};

// A Mean-compensation partial per query head: [m, l, acc[D]] with m a reference logit,
// l = sum n e^{lbar - m} and acc = sum n e^{lbar - m} nu over the blocks it covers.
inline size_t comp_partial_floats(int G, int D) { return static_cast<size_t>(G) * (D + 2); }

constexpr int kStepMaxRanks = 16;  // largest cluster of the decode-step kernel

// Problem shape of the decode-step kernel (decode_step.cu).
struct StepShape {
  bool bf16;       // q, K, V in bf16 (else fp32)
  bool fp16_summ;  // mean_k / mean_v stored as fp16
  int pairs, G, D, T, Nb, Kb, r;
};

// One launch of the decode-step kernel. do_stream: phases A and B (the pass over every block's
// summaries); do_select: Zhat exchange and Top-K_b (writes sel_idx, scores; without do_attend
// also the per-block records xrec and the ranks' compensation partials cpart); do_attend:
// attention over the selection (with do_select the one just made, without it sel_idx, xrec and
// cpart as a select-only launch left them) and the outputs.
struct StepArgs {
  StepShape s;
  int mode;
  bool do_select, do_attend, do_stream;
  float scale;
  const void* q;
  const void* K;
  const void* V;
  const void* mean_k;
  const float* var_g;
  const void* mean_v;
  const int32_t* count;
  float* ug;          // [pairs][Nb][G] log scores (used when they do not fit in shared memory)
  float* xrec;        // [pairs][Nb][G] x = s q_h . mu_j + log n_j
  float* cpart;       // [pairs][kStepMaxRanks][G][D+2] the ranks' compensation partials
  int32_t* sel_idx;   // [pairs][Kb]
  float* scores;      // [pairs][Nb] or null
  float* out;         // [pairs][G][D]
  int32_t* status;
};

struct FullArgs {
  bool bf16;
  int B, Hkv, G, D, T;
  float scale;
  const void* q;
  const void* K;
  const void* V;
  const int32_t* ctx_lens;
  float* out;
  float* part;        // [B*Hkv][nsplit][G][D+2]
  uint32_t* counters; // [B*Hkv]
  int nsplit;
  int32_t* status;
};

inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
constexpr size_t kWsHeader = 256;

// Workspace of the sparse step: a 256-byte header whose first int32 is the device status word,
// then 256-aligned sections.
struct StepWorkspace {
  size_t ug, xrec, cpart, total;
  void build(int pairs, int Nb, int G, int D) {
    size_t o = kWsHeader;
    ug = o;    o += align256(sizeof(float) * static_cast<size_t>(pairs) * Nb * G);
    xrec = o;  o += align256(sizeof(float) * static_cast<size_t>(pairs) * Nb * G);
    cpart = o; o += align256(sizeof(float) * static_cast<size_t>(pairs) * kStepMaxRanks * comp_partial_floats(G, D));
    total = o;
  }
};

// Cluster size, blocks per rank and shared-memory bytes the decode-step kernel uses for this
// shape (bf16 selects the kernel instantiation; the plan does not depend on it otherwise).
cudaError_t step_plan(const StepShape& a, int* C, int* chunk, size_t* smem);
// Splits per kv-head of full_decode (<= max_full_splits(T)).
int full_splits(int B, int Hkv, int T);
inline int max_full_splits(int T) { return (T + 511) / 512; }

cudaError_t launch_build_summaries(const SummariesArgs& a, cudaStream_t st);
cudaError_t launch_append(const AppendArgs& a, cudaStream_t st);
cudaError_t launch_decode_step(const StepArgs& a, cudaStream_t st);
cudaError_t launch_full_decode(const FullArgs& a, cudaStream_t st);

}  // namespace compkv
