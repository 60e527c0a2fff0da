// a4. Dense decode attention over all cached tokens: the full attention that the sparse step is
// measured against (CompKV review, Key claims and FAQ: speedup over full attention, Table 4).
//
// Split-K flash decode: the tokens of each (sequence, kv-head) are cut into `nsplit` contiguous
// ranges, one CTA each, sized so the grid covers the SMs about three times. A CTA streams its
// range in 32-token tiles of K and V through a 3-stage ring of bulk copies tracked by mbarriers,
// computes the logits of the G query heads of the kv-head (transpose-reduced dot products),
// updates an online softmax per head and accumulates P.V. Split partials (max, sum, acc) go to
// the workspace; the last CTA of a kv-head to finish (atomic ticket, no waiting) merges them and
// resets the ticket to zero for the next call.
#include "attend.cuh"
#include "common.cuh"
#include "internal.h"

namespace compkv {
namespace {

constexpr int kTT = 32;      // tokens per tile
constexpr int kStages = 3;

struct FParams {
  int Hkv, T, nsplit;
  float scale;
  const void* q;
  const void* K;
  const void* V;
  const int32_t* ctx_lens;
  float* out;
  float* part;
  uint32_t* counters;
  int32_t* status;
};

template <typename T, int D, int G>
struct FLayout {
  static constexpr size_t tile_bytes = sizeof(T) * kTT * D;
  static constexpr size_t off_k = 0;                                        // [S][kTT][D]
  static constexpr size_t off_v = off_k + kStages * tile_bytes;             // [S][kTT][D]
  static constexpr size_t off_lg = off_v + kStages * tile_bytes;            // [G][kTT]
  static constexpr size_t off_p = off_lg + sizeof(float) * G * kTT;         // [kTT][G]
  static constexpr size_t off_q = off_p + sizeof(float) * G * kTT;          // [G][D]
  static constexpr size_t off_red = off_q + sizeof(float) * G * D;          // [kSub][G][D]
  static constexpr size_t off_ml = off_red + sizeof(float) * PV<T, D, G>::kSub * G * D;
  static constexpr size_t off_sc = off_ml + sizeof(float) * 2 * 8;
  static constexpr size_t off_flag = off_sc + sizeof(float) * 8;
  static constexpr size_t off_mbar = (off_flag + 16 + 15) & ~size_t(15);
  static constexpr size_t total = off_mbar + 8 * kStages;
};

template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreads) full_decode_kernel(const __grid_constant__ FParams p) {
  using LY = FLayout<T, D, G>;
  using RG = RowGeom<T, D>;
  using PVt = PV<T, D, G>;
  constexpr int EPV = RG::kEpv, VEC = PVt::kVec;
  extern __shared__ __align__(128) unsigned char sm[];
  T* kt = reinterpret_cast<T*>(sm + LY::off_k);
  T* vt = reinterpret_cast<T*>(sm + LY::off_v);
  float* lg = reinterpret_cast<float*>(sm + LY::off_lg);
  float* pT = reinterpret_cast<float*>(sm + LY::off_p);
  float* q_s = reinterpret_cast<float*>(sm + LY::off_q);
  float* red = reinterpret_cast<float*>(sm + LY::off_red);
  float* ml_s = reinterpret_cast<float*>(sm + LY::off_ml);
  float* sc_s = reinterpret_cast<float*>(sm + LY::off_sc);
  int* flag = reinterpret_cast<int*>(sm + LY::off_flag);
  uint64_t* mbar = reinterpret_cast<uint64_t*>(sm + LY::off_mbar);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bk = blockIdx.x / p.nsplit, split = blockIdx.x % p.nsplit;
  const int b = bk / p.Hkv;
  int Tb = p.ctx_lens ? p.ctx_lens[b] : p.T;
  Tb = max(0, min(Tb, p.T));
  const int per = ((Tb + p.nsplit - 1) / p.nsplit + kTT - 1) / kTT * kTT;
  const int t0 = min(Tb, split * per), t1 = min(Tb, t0 + per);
  const int ntiles = (t1 - t0 + kTT - 1) / kTT;
  const T* Kb = static_cast<const T*>(p.K) + (static_cast<size_t>(bk) * p.T + t0) * D;
  const T* Vb = static_cast<const T*>(p.V) + (static_cast<size_t>(bk) * p.T + t0) * D;
  const uint64_t policy = l2_evict_first_policy();

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&mbar[s], 1);
    mbar_init_fence();
  }
  {
    const T* qp = static_cast<const T*>(p.q) + static_cast<size_t>(bk) * G * D;
    for (int i = tid; i < G * D; i += kThreads) q_s[i] = to_float(qp[i]);
  }
  __syncthreads();
  auto issue = [&](int i) {
    const int st = i % kStages;
    const int rows = min(kTT, t1 - t0 - i * kTT);
    const uint32_t bytes = static_cast<uint32_t>(rows) * D * sizeof(T);
    mbar_arrive_expect_tx(&mbar[st], 2 * bytes);
    bulk_g2s_stream(kt + static_cast<size_t>(st) * kTT * D, Kb + static_cast<size_t>(i) * kTT * D, bytes, &mbar[st], policy);
    bulk_g2s_stream(vt + static_cast<size_t>(st) * kTT * D, Vb + static_cast<size_t>(i) * kTT * D, bytes, &mbar[st], policy);
  };
  if (tid == 0)
    for (int i = 0; i < min(ntiles, kStages - 1); ++i) issue(i);
  int issued = min(ntiles, kStages - 1), waited = ntiles;

  const int li = lane % RG::kLpr;
  float qr[G][EPV];
  load_q_regs<T, D, G>(q_s, li, qr);
  const int cv = tid % PVt::kCols, sub = tid / PVt::kCols;
  float acc[G][VEC];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < VEC; ++e) acc[h][e] = 0.f;
  float m_run = -CUDART_INF_F, l_run = 0.f;
  bool ok = true;

#pragma unroll 1
  for (int i = 0; i < ntiles; ++i) {
    const int st = i % kStages;
    const int rows = min(kTT, t1 - t0 - i * kTT);
    T* ks = kt + static_cast<size_t>(st) * kTT * D;
    T* vs = vt + static_cast<size_t>(st) * kTT * D;
    const bool got = mbar_wait(&mbar[st], (i / kStages) & 1, p.status);
    if (rows < kTT) {  // ragged last tile: zero the V rows no copy wrote (their weight is 0)
      for (int e = tid; e < (kTT - rows) * D; e += kThreads) vs[static_cast<size_t>(rows) * D + e] = T(0);
    }
    tile_logits<T, D, G>(ks, kTT, qr, p.scale, lg, kTT, [&](int row) { return row < rows; });
    ok = __syncthreads_and(got) != 0;
    if (!ok) {
      waited = i;
      break;
    }
    if (tid == 0 && i + kStages - 1 < ntiles) issue(i + kStages - 1);
    if (i + kStages - 1 < ntiles) ++issued;
    if (warp < G) {
      const int h = warp;
      const float x = lg[h * kTT + lane];
      const float m_new = fmaxf(m_run, warp_max(x));
      const float w = (x == -CUDART_INF_F) ? 0.f : __expf(x - m_new);
      pT[lane * G + h] = w;
      const float sc = (m_run == -CUDART_INF_F) ? 0.f : __expf(m_run - m_new);
      l_run = l_run * sc + warp_sum(w);
      m_run = m_new;
      if (lane == 0) sc_s[h] = sc;
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float sc = sc_s[h];
#pragma unroll
      for (int e = 0; e < VEC; ++e) acc[h][e] *= sc;
    }
    PVt::accumulate(vs, pT, kTT, sub, cv, acc);
  }
  if (!ok) {
    for (int i = waited; i < issued; ++i) mbar_wait(&mbar[i % kStages], (i / kStages) & 1, nullptr);
  }
  __syncthreads();

  // ---- split partial -> workspace
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < VEC; ++e) red[(sub * G + h) * D + cv * VEC + e] = acc[h][e];
  if (warp < G && lane == 0) {
    ml_s[2 * warp] = m_run;
    ml_s[2 * warp + 1] = l_run;
  }
  __syncthreads();
  float* mine = p.part + (static_cast<size_t>(bk) * p.nsplit + split) * G * (D + 2);
  for (int i = tid; i < G * D; i += kThreads) {
    float s = 0.f;
    for (int k = 0; k < PVt::kSub; ++k) s += red[k * G * D + i];
    mine[(i / D) * (D + 2) + 2 + (i % D)] = s;
  }
  if (tid < G) {
    mine[tid * (D + 2)] = ml_s[2 * tid];
    mine[tid * (D + 2) + 1] = ml_s[2 * tid + 1];
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) flag[0] = (atomicAdd(&p.counters[bk], 1u) == static_cast<uint32_t>(p.nsplit - 1));
  __syncthreads();
  if (!flag[0]) return;

  // ---- last CTA of this kv-head: merge the splits
  __threadfence();
  const float* parts = p.part + static_cast<size_t>(bk) * p.nsplit * G * (D + 2);
  if (tid < G) {
    float M = -CUDART_INF_F;
    for (int s = 0; s < p.nsplit; ++s) M = fmaxf(M, __ldcg(parts + (static_cast<size_t>(s) * G + tid) * (D + 2)));
    float den = 0.f;
    for (int s = 0; s < p.nsplit; ++s) {
      const float* ps = parts + (static_cast<size_t>(s) * G + tid) * (D + 2);
      const float ms = __ldcg(ps);
      if (ms != -CUDART_INF_F) den = fmaf(__expf(ms - M), __ldcg(ps + 1), den);
    }
    ml_s[2 * tid] = M;
    ml_s[2 * tid + 1] = den > 0.f ? 1.f / den : 0.f;
  }
  __syncthreads();
  float* o = p.out + static_cast<size_t>(bk) * G * D;
  for (int i = tid; i < G * D; i += kThreads) {
    const int h = i / D, c = i % D;
    const float M = ml_s[2 * h];
    float a = 0.f;
    for (int s = 0; s < p.nsplit; ++s) {
      const float* ps = parts + (static_cast<size_t>(s) * G + h) * (D + 2);
      const float ms = __ldcg(ps);
      if (ms != -CUDART_INF_F) a = fmaf(__expf(ms - M), __ldcg(ps + 2 + c), a);
    }
    o[i] = a * ml_s[2 * h + 1];
  }
  if (tid == 0) p.counters[bk] = 0u;
}

template <typename T, int D, int G>
cudaError_t launch_t(const FullArgs& a, cudaStream_t st) {
  auto kern = full_decode_kernel<T, D, G>;
  const size_t smem = FLayout<T, D, G>::total;
  static bool attrs_set = false;  // set once, so a launch inside stream capture only launches
  if (!attrs_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    attrs_set = true;
  }
  FParams p;
  p.Hkv = a.Hkv;
  p.T = a.T;
  p.nsplit = a.nsplit;
  p.scale = a.scale;
  p.q = a.q;
  p.K = a.K;
  p.V = a.V;
  p.ctx_lens = a.ctx_lens;
  p.out = a.out;
  p.part = a.part;
  p.counters = a.counters;
  p.status = a.status;
  full_decode_kernel<T, D, G><<<a.B * a.Hkv * a.nsplit, kThreads, smem, st>>>(p);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t dispatch_g(const FullArgs& a, cudaStream_t st) {
  switch (a.G) {
    case 1: return launch_t<T, D, 1>(a, st);
    case 2: return launch_t<T, D, 2>(a, st);
    case 4: return launch_t<T, D, 4>(a, st);
    case 8: return launch_t<T, D, 8>(a, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

int full_splits(int B, int Hkv, int T) {
  int sms = 0, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (sms <= 0) sms = 148;
  const int pairs = B * Hkv;
  int ns = (3 * sms + pairs - 1) / pairs;
  ns = ns < 1 ? 1 : ns;
  const int mx = max_full_splits(T);
  return ns > mx ? mx : ns;
}

cudaError_t launch_full_decode(const FullArgs& a, cudaStream_t st) {
  if (a.bf16) return a.D == 128 ? dispatch_g<uint16_t, 128>(a, st) : dispatch_g<uint16_t, 64>(a, st);
  return a.D == 128 ? dispatch_g<float, 128>(a, st) : dispatch_g<float, 64>(a, st);
}

}  // namespace compkv
