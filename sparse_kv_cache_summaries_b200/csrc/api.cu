// C ABI of the CompKV decode hot path: argument validation, workspace layout and kernel
// dispatch. No allocation, no host synchronisation (except compkv_read_device_status).
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>

#include "compkv.h"
#include "internal.h"

namespace {

thread_local char g_last_cuda_error[256] = "";

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return COMPKV_OK;
  std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s: %s", cudaGetErrorName(e),
                cudaGetErrorString(e));
  return COMPKV_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

int check_shape(const compkv_shape* s) {
  if (s == nullptr) return COMPKV_ERR_INVALID_ARG;
  if (s->batch < 1 || s->n_q_heads < 1 || s->n_kv_heads < 1 || s->ctx_len < 1 || s->head_dim < 1 ||
      s->n_groups < 1)
    return COMPKV_ERR_INVALID_ARG;
  if (s->n_q_heads % s->n_kv_heads != 0) return COMPKV_ERR_UNSUPPORTED_SHAPE;
  const int G = s->n_q_heads / s->n_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return COMPKV_ERR_UNSUPPORTED_SHAPE;
  if (s->head_dim != 64 && s->head_dim != 128) return COMPKV_ERR_UNSUPPORTED_SHAPE;
  if (s->block_size != compkv::kBlockTokensHost) return COMPKV_ERR_UNSUPPORTED_SHAPE;
  const int r = s->n_groups;
  if ((r & (r - 1)) != 0 || r > s->head_dim) return COMPKV_ERR_UNSUPPORTED_SHAPE;
  if (s->summary_dtype != COMPKV_SUMMARY_FP32 && s->summary_dtype != COMPKV_SUMMARY_FP16)
    return COMPKV_ERR_INVALID_ARG;
  // grid and index limits of the kernels
  const long long nb = (s->ctx_len + 15) / 16;
  if (static_cast<long long>(s->batch) * s->n_kv_heads * nb > (1LL << 30)) return COMPKV_ERR_UNSUPPORTED_SHAPE;
  return COMPKV_OK;
}

int check_dtype(int dtype) {
  return (dtype == COMPKV_BF16 || dtype == COMPKV_FP32) ? COMPKV_OK : COMPKV_ERR_INVALID_ARG;
}

int check_mode(int mode) {
  return (mode == COMPKV_MODE_COMPKV || mode == COMPKV_MODE_MASS || mode == COMPKV_MODE_MASS_COMP)
             ? COMPKV_OK
             : COMPKV_ERR_INVALID_ARG;
}

int n_blocks(const compkv_shape* s) { return (s->ctx_len + 15) / 16; }

int kb_of(const compkv_shape* s, int budget) {
  const int nb = n_blocks(s);
  const int k = budget / 16;
  return k < nb ? k : nb;
}

float scale_of(const compkv_shape* s, float softmax_scale) {
  return softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(s->head_dim));
}

compkv::StepWorkspace step_ws(const compkv_shape* s) {
  compkv::StepWorkspace w;
  w.build(s->batch * s->n_kv_heads, n_blocks(s), s->n_q_heads / s->n_kv_heads, s->head_dim);
  return w;
}

int32_t* status_word(void* ws) { return static_cast<int32_t*>(ws); }
float* ws_at(void* ws, size_t off) { return reinterpret_cast<float*>(static_cast<char*>(ws) + off); }

struct Common {
  int G, Nb, Kb;
  float scale;
};

int check_step_args(const compkv_shape* shape, int dtype, int mode, int budget, void* ws,
                    size_t ws_bytes, Common* c) {
  int st = check_shape(shape);
  if (st) return st;
  if ((st = check_dtype(dtype)) || (st = check_mode(mode))) return st;
  if (budget < 0) return COMPKV_ERR_INVALID_ARG;
  c->G = shape->n_q_heads / shape->n_kv_heads;
  c->Nb = n_blocks(shape);
  c->Kb = kb_of(shape, budget);
  if (c->Kb == 0 && mode == COMPKV_MODE_MASS) return COMPKV_ERR_INVALID_ARG;
  if (ws == nullptr) return COMPKV_ERR_INVALID_ARG;
  if (!aligned16(ws)) return COMPKV_ERR_BAD_ALIGNMENT;
  if (ws_bytes < compkv_workspace_bytes(shape, budget)) return COMPKV_ERR_WORKSPACE_TOO_SMALL;
  return COMPKV_OK;
}

}  // namespace

extern "C" {

int32_t compkv_num_selected(const compkv_shape* shape, int32_t budget_tokens) {
  const int st = check_shape(shape);
  if (st) return st;
  if (budget_tokens < 0) return COMPKV_ERR_INVALID_ARG;
  return kb_of(shape, budget_tokens);
}

size_t compkv_workspace_bytes(const compkv_shape* shape, int32_t budget_tokens) {
  if (check_shape(shape) != COMPKV_OK || budget_tokens < 0) return 0;
  return step_ws(shape).total;
}

size_t compkv_full_workspace_bytes(const compkv_shape* shape) {
  if (check_shape(shape) != COMPKV_OK) return 0;
  const int G = shape->n_q_heads / shape->n_kv_heads;
  const size_t pairs = static_cast<size_t>(shape->batch) * shape->n_kv_heads;
  const size_t counters = compkv::align256(sizeof(uint32_t) * pairs);
  const size_t parts = compkv::align256(sizeof(float) * pairs * compkv::max_full_splits(shape->ctx_len) *
                                        compkv::comp_partial_floats(G, shape->head_dim));
  return compkv::kWsHeader + counters + parts;
}

int compkv_build_summaries(const compkv_shape* shape, compkv_dtype dtype, const void* K,
                           const void* V, const int32_t* ctx_lens, void* mean_k, float* var_g,
                           void* mean_v, int32_t* count, void* stream) {
  int st = check_shape(shape);
  if (st) return st;
  if ((st = check_dtype(dtype))) return st;
  if (!K || !V || !mean_k || !var_g || !mean_v || !count) return COMPKV_ERR_INVALID_ARG;
  if (!aligned16(K) || !aligned16(V) || !aligned16(mean_k) || !aligned16(mean_v) || !aligned4(var_g) ||
      !aligned4(count) || (ctx_lens && !aligned4(ctx_lens)))
    return COMPKV_ERR_BAD_ALIGNMENT;
  compkv::SummariesArgs a;
  a.bf16 = dtype == COMPKV_BF16;
  a.fp16_summ = shape->summary_dtype == COMPKV_SUMMARY_FP16;
  a.B = shape->batch;
  a.Hkv = shape->n_kv_heads;
  a.T = shape->ctx_len;
  a.D = shape->head_dim;
  a.Nb = n_blocks(shape);
  a.r = shape->n_groups;
  a.K = K;
  a.V = V;
  a.ctx_lens = ctx_lens;
  a.mean_k = mean_k;
  a.var_g = var_g;
  a.mean_v = mean_v;
  a.count = count;
  return cuda_status(compkv::launch_build_summaries(a, static_cast<cudaStream_t>(stream)));
}

int compkv_append(const compkv_shape* shape, compkv_dtype dtype, const void* k_new,
                  const void* v_new, const int32_t* positions, void* K, void* V, void* mean_k,
                  float* var_g, void* mean_v, int32_t* count, int32_t* status, void* stream) {
  int st = check_shape(shape);
  if (st) return st;
  if ((st = check_dtype(dtype))) return st;
  if (!k_new || !v_new || !positions || !mean_k || !var_g || !mean_v || !count || (!K) != (!V))
    return COMPKV_ERR_INVALID_ARG;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned4(positions) || (K && !aligned16(K)) ||
      (V && !aligned16(V)) || !aligned16(mean_k) || !aligned16(mean_v) || !aligned4(var_g) ||
      !aligned4(count) || (status && !aligned4(status)))
    return COMPKV_ERR_BAD_ALIGNMENT;
  compkv::AppendArgs a;
  a.bf16 = dtype == COMPKV_BF16;
  a.fp16_summ = shape->summary_dtype == COMPKV_SUMMARY_FP16;
  a.pairs = shape->batch * shape->n_kv_heads;
  a.Hkv = shape->n_kv_heads;
  a.T = shape->ctx_len;
  a.D = shape->head_dim;
  a.Nb = n_blocks(shape);
  a.r = shape->n_groups;
  a.k_new = k_new;
  a.v_new = v_new;
  a.positions = positions;
  a.K = K;
  a.V = V;
  a.mean_k = mean_k;
  a.var_g = var_g;
  a.mean_v = mean_v;
  a.count = count;
  a.status = status;
  return cuda_status(compkv::launch_append(a, static_cast<cudaStream_t>(stream)));
}

enum class Upto { kStream, kSelect, kAttend };

// Streaming score kernel, then (unless `upto` is kStream) the select kernel, or with kAttend the
// select-and-attend kernel, launched with programmatic dependent launch.
static int score_select_impl(const compkv_shape* shape, compkv_dtype dtype, compkv_mode mode,
                             const void* q, const void* mean_k, const float* var_g,
                             const void* mean_v, const int32_t* count, int32_t budget_tokens,
                             float softmax_scale, int32_t* sel_idx, float* scores, void* workspace,
                             size_t workspace_bytes, void* stream, Upto upto, const void* K,
                             const void* V, float* out) {
  Common c;
  int st = check_step_args(shape, dtype, mode, budget_tokens, workspace, workspace_bytes, &c);
  if (st) return st;
  const bool comp = mode != COMPKV_MODE_MASS;
  if (!q || !mean_k || !var_g || !count || (comp && !mean_v) ||
      (upto != Upto::kStream && c.Kb > 0 && !sel_idx))
    return COMPKV_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(mean_k) || (comp && !aligned16(mean_v)) || !aligned4(var_g) ||
      !aligned4(count) || (sel_idx && !aligned4(sel_idx)) || (scores && !aligned4(scores)))
    return COMPKV_ERR_BAD_ALIGNMENT;
  const compkv::StepWorkspace W = step_ws(shape);
  const int pairs = shape->batch * shape->n_kv_heads;
  int nctas = 0;
  compkv::StreamArgs a;
  a.bf16 = dtype == COMPKV_BF16;
  a.fp16_summ = shape->summary_dtype == COMPKV_SUMMARY_FP16;
  a.mode = mode;
  a.pairs = pairs;
  a.G = c.G;
  a.D = shape->head_dim;
  a.Nb = c.Nb;
  a.r = shape->n_groups;
  a.slots = W.slots;
  a.scale = scale_of(shape, softmax_scale);
  a.q = q;
  a.mean_k = mean_k;
  a.var_g = var_g;
  a.mean_v = mean_v;
  a.count = count;
  a.u = ws_at(workspace, W.u);
  a.xrec = ws_at(workspace, W.xrec);
  a.zpart = ws_at(workspace, W.zpart);
  a.comp_seg = ws_at(workspace, W.comp_seg);
  a.status = status_word(workspace);
  a.nctas_out = &nctas;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  int rc = cuda_status(compkv::launch_score_stream(a, cs));
  if (rc || upto == Upto::kStream) return rc;
  compkv::FusedArgs b;
  b.bf16 = a.bf16;
  b.fp16_summ = a.fp16_summ;
  b.mode = mode;
  b.do_select = true;
  b.do_attend = upto == Upto::kAttend;
  b.pairs = pairs;
  b.G = c.G;
  b.D = shape->head_dim;
  b.T = shape->ctx_len;
  b.Nb = c.Nb;
  b.Kb = c.Kb;
  b.slots = W.slots;
  b.nctas_stream = nctas;
  b.scale = a.scale;
  b.q = q;
  b.K = K;
  b.V = V;
  b.mean_v = mean_v;
  b.u = a.u;
  b.xrec = a.xrec;
  b.zpart = a.zpart;
  b.comp_seg = a.comp_seg;
  b.comp = ws_at(workspace, W.comp);
  b.sel_idx = sel_idx;
  b.scores = scores;
  b.out = out;
  b.status = a.status;
  b.pdl = true;
  return cuda_status(compkv::launch_decode_fused(b, cs));
}

int compkv_score_select(const compkv_shape* shape, compkv_dtype dtype, compkv_mode mode,
                        const void* q, const void* mean_k, const float* var_g,
                        const void* mean_v, const int32_t* count, int32_t budget_tokens,
                        float softmax_scale, int32_t* sel_idx, float* scores, void* workspace,
                        size_t workspace_bytes, void* stream) {
  return score_select_impl(shape, dtype, mode, q, mean_k, var_g, mean_v, count, budget_tokens,
                           softmax_scale, sel_idx, scores, workspace, workspace_bytes, stream,
                           Upto::kSelect, nullptr, nullptr, nullptr);
}

int compkv_score_stream(const compkv_shape* shape, compkv_dtype dtype, compkv_mode mode,
                        const void* q, const void* mean_k, const float* var_g,
                        const void* mean_v, const int32_t* count, int32_t budget_tokens,
                        float softmax_scale, void* workspace, size_t workspace_bytes,
                        void* stream) {
  return score_select_impl(shape, dtype, mode, q, mean_k, var_g, mean_v, count, budget_tokens,
                           softmax_scale, nullptr, nullptr, workspace, workspace_bytes, stream,
                           Upto::kStream, nullptr, nullptr, nullptr);
}

int compkv_sparse_decode(const compkv_shape* shape, compkv_dtype dtype, compkv_mode mode,
                         const void* q, const void* K, const void* V, const void* mean_k,
                         const void* mean_v, const int32_t* count, const int32_t* sel_idx,
                         int32_t budget_tokens, float softmax_scale, float* out, void* workspace,
                         size_t workspace_bytes, void* stream) {
  Common c;
  int st = check_step_args(shape, dtype, mode, budget_tokens, workspace, workspace_bytes, &c);
  if (st) return st;
  const bool comp = mode != COMPKV_MODE_MASS;
  if (!q || !K || !V || !count || !out || (comp && (!mean_k || !mean_v)) || (c.Kb > 0 && !sel_idx))
    return COMPKV_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(K) || !aligned16(V) || (comp && (!aligned16(mean_k) || !aligned16(mean_v))) ||
      !aligned4(count) || (sel_idx && !aligned4(sel_idx)) || !aligned4(out))
    return COMPKV_ERR_BAD_ALIGNMENT;
  const compkv::StepWorkspace W = step_ws(shape);
  compkv::FusedArgs b;
  b.bf16 = dtype == COMPKV_BF16;
  b.fp16_summ = shape->summary_dtype == COMPKV_SUMMARY_FP16;
  b.mode = mode;
  b.do_select = false;
  b.do_attend = true;
  b.pairs = shape->batch * shape->n_kv_heads;
  b.G = c.G;
  b.D = shape->head_dim;
  b.T = shape->ctx_len;
  b.Nb = c.Nb;
  b.Kb = c.Kb;
  b.slots = W.slots;
  b.nctas_stream = 0;
  b.scale = scale_of(shape, softmax_scale);
  b.q = q;
  b.K = K;
  b.V = V;
  b.mean_v = mean_v;
  b.u = nullptr;
  b.xrec = ws_at(workspace, W.xrec);
  b.zpart = nullptr;
  b.comp_seg = nullptr;
  b.comp = ws_at(workspace, W.comp);
  b.sel_idx = const_cast<int32_t*>(sel_idx);  // read only when do_select is false
  b.scores = nullptr;
  b.out = out;
  b.status = status_word(workspace);
  b.pdl = false;
  return cuda_status(compkv::launch_decode_fused(b, static_cast<cudaStream_t>(stream)));
}

int compkv_decode_step(const compkv_shape* shape, compkv_dtype dtype, compkv_mode mode,
                       const void* q, const void* K, const void* V, const void* mean_k,
                       const float* var_g, const void* mean_v, const int32_t* count,
                       int32_t budget_tokens, float softmax_scale, int32_t* sel_idx,
                       float* scores, float* out, void* workspace, size_t workspace_bytes,
                       void* stream) {
  if (!K || !V || !out) return COMPKV_ERR_INVALID_ARG;
  if (!aligned16(K) || !aligned16(V) || !aligned4(out)) return COMPKV_ERR_BAD_ALIGNMENT;
  return score_select_impl(shape, dtype, mode, q, mean_k, var_g, mean_v, count, budget_tokens,
                           softmax_scale, sel_idx, scores, workspace, workspace_bytes, stream,
                           Upto::kAttend, K, V, out);
}

int compkv_full_decode(const compkv_shape* shape, compkv_dtype dtype, const void* q,
                       const void* K, const void* V, const int32_t* ctx_lens, float softmax_scale,
                       float* out, void* workspace, size_t workspace_bytes, void* stream) {
  int st = check_shape(shape);
  if (st) return st;
  if ((st = check_dtype(dtype))) return st;
  if (!q || !K || !V || !out || !workspace) return COMPKV_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(K) || !aligned16(V) || !aligned4(out) || !aligned16(workspace) ||
      (ctx_lens && !aligned4(ctx_lens)))
    return COMPKV_ERR_BAD_ALIGNMENT;
  if (workspace_bytes < compkv_full_workspace_bytes(shape)) return COMPKV_ERR_WORKSPACE_TOO_SMALL;
  const size_t pairs = static_cast<size_t>(shape->batch) * shape->n_kv_heads;
  char* ws = static_cast<char*>(workspace);
  compkv::FullArgs a;
  a.bf16 = dtype == COMPKV_BF16;
  a.B = shape->batch;
  a.Hkv = shape->n_kv_heads;
  a.G = shape->n_q_heads / shape->n_kv_heads;
  a.D = shape->head_dim;
  a.T = shape->ctx_len;
  a.scale = scale_of(shape, softmax_scale);
  a.q = q;
  a.K = K;
  a.V = V;
  a.ctx_lens = ctx_lens;
  a.out = out;
  a.counters = reinterpret_cast<uint32_t*>(ws + compkv::kWsHeader);
  a.part = reinterpret_cast<float*>(ws + compkv::kWsHeader + compkv::align256(sizeof(uint32_t) * pairs));
  a.nsplit = compkv::full_splits(a.B, a.Hkv, a.T);
  a.status = status_word(workspace);
  return cuda_status(compkv::launch_full_decode(a, static_cast<cudaStream_t>(stream)));
}

int compkv_read_device_status(void* workspace, void* stream, int32_t* status) {
  if (!workspace || !status) return COMPKV_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(status, workspace, sizeof(int32_t), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemsetAsync(workspace, 0, sizeof(int32_t), s);
  return cuda_status(e);
}

const char* compkv_status_string(int status) {
  switch (status) {
    case COMPKV_OK: return "ok";
    case COMPKV_ERR_INVALID_ARG: return "invalid argument";
    case COMPKV_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case COMPKV_ERR_BAD_ALIGNMENT: return "pointer not 16-byte aligned";
    case COMPKV_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case COMPKV_ERR_CUDA: return "CUDA error";
    default: return "unknown status";
  }
}

const char* compkv_last_cuda_error(void) { return g_last_cuda_error; }

int compkv_version(void) { return COMPKV_VERSION; }

}  // extern "C"
