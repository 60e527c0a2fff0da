// a0. Per-block summaries of the KV cache: token count, mean key, grouped key variance, mean
// value (CompKV review, Summary and FAQ: "mean key, grouped key variances (4 groups by default),
// and mean value, i.e., 2d+r+1 scalars per block").
//
// One warp per 16-token block. The block's K rows (and V rows) are contiguous in [B, Hkv, T, d],
// so the warp reads them with 16-byte coalesced loads, K and V issued together (up to 16 loads
// in flight per lane). Each lane owns a fixed 16-byte channel slice of some rows; per-channel
// sums are finished with xor-shuffles across the lanes that share a slice. The variance is the
// two-pass population form on the register-resident values. Group variances reduce across the
// lanes (or within the lane) that hold the group's channels.
#include "common.cuh"
#include "internal.h"

namespace compkv {
namespace {

template <typename T, int D>
struct Geom {
  static constexpr int kEpv = 16 / static_cast<int>(sizeof(T));  // elements per 16-byte vector
  static constexpr int kLpr = D / kEpv;                          // lanes per token row
  static constexpr int kRpl = 32 / kLpr;                         // rows per warp-wide load
  static constexpr int kLoads = kBlockTokens / kRpl;             // loads per block and tensor
  static_assert(kLpr <= 32 && 32 % kLpr == 0, "unsupported head_dim / dtype");
};

template <typename T, int EPV>
__device__ __forceinline__ void to_floats(const uint4& w, float (&f)[EPV]);

template <>
__device__ __forceinline__ void to_floats<uint16_t, 8>(const uint4& w, float (&f)[8]) {
  unpack8_bf16(w, f);
}
template <>
__device__ __forceinline__ void to_floats<float, 4>(const uint4& w, float (&f)[4]) {
  f[0] = __uint_as_float(w.x);
  f[1] = __uint_as_float(w.y);
  f[2] = __uint_as_float(w.z);
  f[3] = __uint_as_float(w.w);
}

template <typename T, int D, typename S>
__global__ void __launch_bounds__(kThreads)
    build_summaries_kernel(const T* __restrict__ K, const T* __restrict__ V,
                           const int32_t* __restrict__ ctx_lens, int n_blk_total, int Hkv, int T_cap,
                           int Nb, int r, S* __restrict__ mean_k, float* __restrict__ var_g,
                           S* __restrict__ mean_v, int32_t* __restrict__ count) {
  using Gm = Geom<T, D>;
  constexpr int EPV = Gm::kEpv, LPR = Gm::kLpr, RPL = Gm::kRpl, NL = Gm::kLoads;
  const int lane = threadIdx.x & 31;
  const int w = blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (w >= n_blk_total) return;
  const int j = w % Nb;
  const int bg = w / Nb;  // b * Hkv + g
  const int b = bg / Hkv;
  int Tb = ctx_lens ? ctx_lens[b] : T_cap;
  Tb = max(0, min(Tb, T_cap));
  const int n = max(0, min(kBlockTokens, Tb - j * kBlockTokens));
  const int li = lane % LPR, rs = lane / LPR;
  const size_t base = (static_cast<size_t>(bg) * T_cap + static_cast<size_t>(j) * kBlockTokens) * D;
  const uint4* kp = reinterpret_cast<const uint4*>(K + base) + li;
  const uint4* vp = reinterpret_cast<const uint4*>(V + base) + li;

  uint4 kraw[NL], vraw[NL];
#pragma unroll
  for (int i = 0; i < NL; ++i) {
    const int row = i * RPL + rs;
    if (row < n) {
      kraw[i] = __ldcs(kp + row * (D / EPV));
      vraw[i] = __ldcs(vp + row * (D / EPV));
    } else {
      kraw[i] = make_uint4(0, 0, 0, 0);
      vraw[i] = make_uint4(0, 0, 0, 0);
    }
  }
  const float inv_n = n > 0 ? 1.f / static_cast<float>(n) : 0.f;

  // means
  float ks[EPV], vs[EPV];
#pragma unroll
  for (int e = 0; e < EPV; ++e) ks[e] = vs[e] = 0.f;
#pragma unroll
  for (int i = 0; i < NL; ++i) {
    float kf[EPV], vf[EPV];
    to_floats<T, EPV>(kraw[i], kf);
    to_floats<T, EPV>(vraw[i], vf);
#pragma unroll
    for (int e = 0; e < EPV; ++e) {
      ks[e] += kf[e];
      vs[e] += vf[e];
    }
  }
#pragma unroll
  for (int o = LPR; o < 32; o <<= 1) {
#pragma unroll
    for (int e = 0; e < EPV; ++e) {
      ks[e] += __shfl_xor_sync(0xffffffffu, ks[e], o);
      vs[e] += __shfl_xor_sync(0xffffffffu, vs[e], o);
    }
  }
  float mu[EPV];
#pragma unroll
  for (int e = 0; e < EPV; ++e) mu[e] = ks[e] * inv_n;

  // per-channel population variance (two-pass on registers)
  float dv[EPV];
#pragma unroll
  for (int e = 0; e < EPV; ++e) dv[e] = 0.f;
#pragma unroll
  for (int i = 0; i < NL; ++i) {
    if (i * RPL + rs < n) {
      float kf[EPV];
      to_floats<T, EPV>(kraw[i], kf);
#pragma unroll
      for (int e = 0; e < EPV; ++e) {
        const float x = kf[e] - mu[e];
        dv[e] = fmaf(x, x, dv[e]);
      }
    }
  }
#pragma unroll
  for (int o = LPR; o < 32; o <<= 1) {
#pragma unroll
    for (int e = 0; e < EPV; ++e) dv[e] += __shfl_xor_sync(0xffffffffu, dv[e], o);
  }

  const size_t row_out = static_cast<size_t>(w);
  if (rs == 0) {
    if constexpr (sizeof(S) == 4) {
      float4* mk = reinterpret_cast<float4*>(mean_k + row_out * D + li * EPV);
      float4* mv = reinterpret_cast<float4*>(mean_v + row_out * D + li * EPV);
#pragma unroll
      for (int e = 0; e < EPV; e += 4) {
        mk[e / 4] = make_float4(mu[e], mu[e + 1], mu[e + 2], mu[e + 3]);
        mv[e / 4] = make_float4(vs[e] * inv_n, vs[e + 1] * inv_n, vs[e + 2] * inv_n, vs[e + 3] * inv_n);
      }
    } else {  // fp16 storage: pairs rounded to nearest even
      __half2* mk = reinterpret_cast<__half2*>(mean_k + row_out * D + li * EPV);
      __half2* mv = reinterpret_cast<__half2*>(mean_v + row_out * D + li * EPV);
#pragma unroll
      for (int e = 0; e < EPV; e += 2) {
        mk[e / 2] = __floats2half2_rn(mu[e], mu[e + 1]);
        mv[e / 2] = __floats2half2_rn(vs[e] * inv_n, vs[e + 1] * inv_n);
      }
    }
  }
  if (lane == 0) count[row_out] = n;

  // group variances: group size gs = D / r channels, contiguous
  const int gs = D / r;
  float* vg = var_g + row_out * r;
  if (gs >= EPV) {
    float part = 0.f;
#pragma unroll
    for (int e = 0; e < EPV; ++e) part += dv[e];
    const int lanes_per_group = gs / EPV;  // power of two <= LPR
    for (int o = 1; o < lanes_per_group; o <<= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (rs == 0 && (li % lanes_per_group) == 0) vg[(li * EPV) / gs] = part * inv_n / gs;
  } else if (rs == 0) {
    const int groups_per_lane = EPV / gs;
    for (int q = 0; q < groups_per_lane; ++q) {
      float part = 0.f;
      for (int e = 0; e < gs; ++e) part += dv[q * gs + e];
      vg[(li * EPV) / gs + q] = part * inv_n / gs;
    }
  }
}

template <typename T, int D, typename S>
cudaError_t launch_t(const SummariesArgs& a, cudaStream_t st) {
  const int total = a.B * a.Hkv * a.Nb;
  const int grid = (total + kWarps - 1) / kWarps;
  build_summaries_kernel<T, D, S><<<grid, kThreads, 0, st>>>(
      static_cast<const T*>(a.K), static_cast<const T*>(a.V), a.ctx_lens, total, a.Hkv, a.T, a.Nb,
      a.r, static_cast<S*>(a.mean_k), a.var_g, static_cast<S*>(a.mean_v), a.count);
  return cudaGetLastError();
}

template <typename S>
cudaError_t launch_s(const SummariesArgs& a, cudaStream_t st) {
  if (a.bf16) return a.D == 128 ? launch_t<uint16_t, 128, S>(a, st) : launch_t<uint16_t, 64, S>(a, st);
  return a.D == 128 ? launch_t<float, 128, S>(a, st) : launch_t<float, 64, S>(a, st);
}

}  // namespace

cudaError_t launch_build_summaries(const SummariesArgs& a, cudaStream_t st) {
  return a.fp16_summ ? launch_s<__half>(a, st) : launch_s<float>(a, st);
}

}  // namespace compkv
