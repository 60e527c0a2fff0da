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
  int B, Hkv, T, D, Nb, r;
  const void* K;
  const void* V;
  const int32_t* ctx_lens;
  float* mean_k;
  float* var_g;
  float* mean_v;
  int32_t* count;
};

// Per-kv-head Mean-compensation partial, merged over all blocks: [m, l, acc[D]] per query head.
// m is the running max of (lbar + log n), l = sum n e^{lbar - m}, acc = sum n e^{lbar - m} nu.
inline size_t comp_partial_floats(int G, int D) { return static_cast<size_t>(G) * (D + 2); }

struct ScoreSelectArgs {
  bool bf16;
  int mode;
  int B, Hkv, G, D, Nb, r, Kb;
  float scale;
  const void* q;
  const float* mean_k;
  const float* var_g;
  const float* mean_v;
  const int32_t* count;
  int32_t* sel_idx;
  float* scores;
  float* comp;        // [B*Hkv][G][D+2]
  int32_t* status;    // device status word
};

struct SparseArgs {
  bool bf16;
  int mode;
  int B, Hkv, G, D, T, Nb, Kb;
  float scale;
  const void* q;
  const void* K;
  const void* V;
  const float* mean_k;
  const float* mean_v;
  const int32_t* count;
  const int32_t* sel_idx;
  const float* comp;  // [B*Hkv][G][D+2] from score_select
  float* out;
  int32_t* status;
  bool pdl;           // launched right after score_select: use programmatic dependent launch
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

// Workspace layout (bytes, 256-aligned sections):
//   [0, 256)            int32 status word
//   comp partials       B*Hkv*G*(D+2) floats
constexpr size_t kWsHeader = 256;
inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Cluster size used by score_select for this shape on the current device (1..16).
int score_select_cluster(int B, int Hkv, int G, int D, int r, int Nb, int Kb, bool bf16,
                         size_t* smem_bytes);
// Blocks per CTA and the CTA count per kv-head (a cluster) of sparse_decode.
void sparse_split(int B, int Hkv, int Kb, int* blocks_per_cta, int* nsplit);
// Splits per kv-head of full_decode (<= max_full_splits(T)).
int full_splits(int B, int Hkv, int T);
inline int max_full_splits(int T) { return (T + 511) / 512; }

cudaError_t launch_build_summaries(const SummariesArgs& a, cudaStream_t st);
cudaError_t launch_score_select(const ScoreSelectArgs& a, cudaStream_t st);
cudaError_t launch_sparse_decode(const SparseArgs& a, cudaStream_t st);
cudaError_t launch_full_decode(const FullArgs& a, cudaStream_t st);

}  // namespace compkv
