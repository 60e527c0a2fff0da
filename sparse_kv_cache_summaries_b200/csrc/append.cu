// a0, incremental: one new token per sequence updates the summaries of the block it enters
// (CompKV review, Frequently asked questions: per-block summaries "updated incrementally as new
// tokens enter the cache"). Welford's running mean and per-channel sum of squared deviations,
// summed over each channel group, keep the grouped population variance exact from the stored
// (n, mu, var_g) alone.
//
// One warp per (sequence, kv-head): lane l holds channels [l VW, l VW + VW) (VW = d / 32).
#include "common.cuh"
#include "internal.h"

namespace compkv {
namespace {

template <typename T, int D, typename S>
__global__ void __launch_bounds__(kThreads) append_kernel(const __grid_constant__ AppendArgs p) {
  constexpr int VW = D / 32;
  __shared__ float dev_s[kWarps][D];  // per-channel (k - mu)(k - mu') of each warp's pair
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int pair = blockIdx.x * kWarps + warp;
  if (pair >= p.pairs) return;
  const int b = pair / p.Hkv;
  const int t = p.positions[b];
  if (t < 0 || t >= p.T) {
    if (lane == 0 && p.status) atomicOr(p.status, COMPKV_DEVERR_BAD_POSITION);
    return;
  }
  const int j = t / kBlockTokens;
  const T* kp = static_cast<const T*>(p.k_new) + static_cast<size_t>(pair) * D + lane * VW;
  const T* vp = static_cast<const T*>(p.v_new) + static_cast<size_t>(pair) * D + lane * VW;
  float k[VW], v[VW];
#pragma unroll
  for (int e = 0; e < VW; ++e) {
    k[e] = to_float(kp[e]);
    v[e] = to_float(vp[e]);
  }
  if (p.K != nullptr && p.V != nullptr) {  // the token also enters the caches at row t
    const size_t off = (static_cast<size_t>(pair) * p.T + t) * D + lane * VW;
#pragma unroll
    for (int e = 0; e < VW; ++e) {
      static_cast<T*>(p.K)[off + e] = kp[e];
      static_cast<T*>(p.V)[off + e] = vp[e];
    }
  }
  const size_t row = static_cast<size_t>(pair) * p.Nb + j;
  const int n = p.count[row];
  const float n1 = static_cast<float>(n + 1);
  S* mk = static_cast<S*>(p.mean_k) + row * D + lane * VW;
  S* mv = static_cast<S*>(p.mean_v) + row * D + lane * VW;
#pragma unroll
  for (int e = 0; e < VW; ++e) {
    const float mu = sload(mk + e);  // the stored mean (fp16 storage: already rounded)
    const float mu1 = mu + (k[e] - mu) / n1;
    dev_s[warp][lane * VW + e] = (k[e] - mu) * (k[e] - mu1);
    sstore(mk + e, mu1);
    const float nu = sload(mv + e);
    sstore(mv + e, nu + (v[e] - nu) / n1);
  }
  __syncwarp();
  const int gs = D / p.r;
  for (int g = lane; g < p.r; g += 32) {
    float sdev = 0.f;
    for (int c = 0; c < gs; ++c) sdev += dev_s[warp][g * gs + c];
    float* vg = p.var_g + row * p.r + g;
    *vg = (*vg * static_cast<float>(n * gs) + sdev) / (n1 * static_cast<float>(gs));
  }
  __syncwarp();  // every lane has read the old count
  if (lane == 0) p.count[row] = n + 1;
}

template <typename T, typename S>
cudaError_t launch_t(const AppendArgs& a, cudaStream_t st) {
  const dim3 grid((a.pairs + kWarps - 1) / kWarps);
  if (a.D == 128) append_kernel<T, 128, S><<<grid, kThreads, 0, st>>>(a);
  else append_kernel<T, 64, S><<<grid, kThreads, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_append(const AppendArgs& a, cudaStream_t st) {
  if (a.D != 64 && a.D != 128) return cudaErrorInvalidValue;
  if (a.fp16_summ) return a.bf16 ? launch_t<uint16_t, __half>(a, st) : launch_t<float, __half>(a, st);
  return a.bf16 ? launch_t<uint16_t, float>(a, st) : launch_t<float, float>(a, st);
}

}  // namespace compkv
