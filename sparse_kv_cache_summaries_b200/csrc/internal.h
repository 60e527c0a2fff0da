// Launch-side interface between the C ABI (api.cu) and the kernels. Host-only declarations.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "compkv.h"

namespace compkv {

constexpr int kBlockTokensHost = 16;  // the only supported block size
constexpr int kStreamTile = 32;       // blocks per tile of the streaming score kernel
constexpr int kStreamMaxCtas = 384;   // grid cap of the streaming score kernel

// Floats per block of the record {x_0..x_{G-1}, n} the streaming kernel writes for the attention
// kernel (x_h = s q_h . mu_j + log n_j; n as int bits), padded to 16 bytes.
__host__ __device__ constexpr int xrec_stride(int G) { return ((G + 1 + 3) / 4) * 4; }

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

struct StreamArgs {
  bool bf16;
  bool fp16_summ;  // mean_k / mean_v stored as fp16
  int mode;
  int pairs, G, D, Nb, r, slots;
  float scale;
  const void* q;
  const void* mean_k;
  const float* var_g;
  const void* mean_v;
  const int32_t* count;
  float* u;          // [pairs][Nb][G]   per-block log scores
  float* xrec;       // [pairs][Nb][xrec_stride(G)]
  float* zpart;      // [pairs][slots][G][2]   log-sum-exp partials of the mass estimate
  float* comp_seg;   // [pairs][slots][G][D+2] compensation partials per segment
  int32_t* status;
  int* nctas_out;    // grid size used (host), may be null
};

// The select-and-attend kernel (decode_fused.cu). do_select: Top-K_b from the streaming
// kernel's outputs (writes sel_idx; without do_attend also the merged compensation partial
// `comp`). do_attend: attention over the selection (with do_select, the one just made; without,
// sel_idx and `comp` as given).
struct FusedArgs {
  bool bf16;
  bool fp16_summ;  // mean_k / mean_v stored as fp16
  int mode;
  bool do_select, do_attend;
  int pairs, G, D, T, Nb, Kb, slots, nctas_stream;
  float scale;
  const void* q;
  const void* K;
  const void* V;
  const void* mean_v;
  const float* u;
  const float* xrec;      // [pairs][Nb][xrec_stride(G)] from the streaming kernel
  const float* zpart;
  const float* comp_seg;
  float* comp;            // [pairs][G][D+2] merged compensation partial
  int32_t* sel_idx;       // [pairs][Kb]
  float* scores;          // [pairs][Nb] or null
  float* out;             // [pairs][G][D]
  int32_t* status;
  bool pdl;               // launched right after the streaming kernel: programmatic dependent launch
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

// Segment records per (sequence, kv-head) the streaming kernel may write: the tiles_per_pair
// tiles of a pair meet at most ceil(tiles_per_pair / min_tiles_per_cta) + 1 CTA ranges, and a
// grid of at most kStreamMaxCtas CTAs gives every CTA at least floor(F / kStreamMaxCtas) tiles.
inline int stream_slots(int pairs, int Nb) {
  const long long tp = (Nb + kStreamTile - 1) / kStreamTile;
  const long long F = tp * pairs;
  long long min_tiles = F / kStreamMaxCtas;
  if (min_tiles < 1) min_tiles = 1;
  return static_cast<int>((tp + min_tiles - 1) / min_tiles + 1);
}

// Workspace of the sparse step: a 256-byte header whose first int32 is the device status word,
// then 256-aligned sections.
struct StepWorkspace {
  size_t u, xrec, zpart, comp_seg, comp, total;
  int slots;
  void build(int pairs, int Nb, int G, int D) {
    slots = stream_slots(pairs, Nb);
    size_t o = kWsHeader;
    u = o;        o += align256(sizeof(float) * static_cast<size_t>(pairs) * Nb * G);
    xrec = o;     o += align256(sizeof(float) * static_cast<size_t>(pairs) * Nb * xrec_stride(G));
    zpart = o;    o += align256(sizeof(float) * static_cast<size_t>(pairs) * slots * G * 2);
    comp_seg = o; o += align256(sizeof(float) * static_cast<size_t>(pairs) * slots * G * (D + 2));
    comp = o;     o += align256(sizeof(float) * static_cast<size_t>(pairs) * comp_partial_floats(G, D));
    total = o;
  }
};

// Grid size of the streaming score kernel for this shape on the current device.
int stream_grid_ctas(bool bf16, bool fp16_summ, int D, int G, int r, int total_tiles);
// Splits per kv-head of full_decode (<= max_full_splits(T)).
int full_splits(int B, int Hkv, int T);
inline int max_full_splits(int T) { return (T + 511) / 512; }

cudaError_t launch_build_summaries(const SummariesArgs& a, cudaStream_t st);
cudaError_t launch_append(const AppendArgs& a, cudaStream_t st);
cudaError_t launch_score_stream(const StreamArgs& a, cudaStream_t st);
cudaError_t launch_decode_fused(const FusedArgs& a, cudaStream_t st);
cudaError_t launch_full_decode(const FullArgs& a, cudaStream_t st);

}  // namespace compkv
