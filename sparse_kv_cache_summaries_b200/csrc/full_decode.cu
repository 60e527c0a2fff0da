// a4. Dense decode attention over all cached tokens: the full attention that the sparse step is
// measured against (CompKV review, Key claims and FAQ: speedup over full attention, Table 4).
//
// Split-K flash decode: the tokens of each (sequence, kv-head) are cut into `nsplit` contiguous
// ranges, one CTA each, about two CTAs per SM. A producer warp streams the range in 32-token
// tiles of K and V (bulk copies into a ring of shared-memory stages with a "full" and an "empty"
// mbarrier each); eight consumer warps in two groups of four take alternate tiles, each warp 8
// rows of its group's tile (as groups of 8 rows, 4 for 8 query heads per kv-head), and keep their
// own online softmax per query head, so no CTA barrier is needed until the end: logits of the rows
// against the G query heads of the kv-head (each lane holds D / 32 channels of a row, paired fp32
// arithmetic; one transpose-reduce gives every lane one (row, head) logit), the running max and
// sum, and P.V into per-lane accumulators. The 8 warps' partials merge in
// shared memory into the split's partial (max, sum, acc) in the workspace; the last CTA of a
// kv-head to finish (atomic ticket, no waiting) merges the splits and resets the ticket to zero
// for the next call.
#include "attend.cuh"
#include "common.cuh"
#include "internal.h"

namespace compkv {
namespace {

constexpr int kTT = 32;                      // tokens per tile
constexpr int kCons = 8;                     // consumer warps
constexpr int kGroupW = 4;                   // consumer warps that share a tile
constexpr int kGroups = kCons / kGroupW;     // tiles in work at once
constexpr int kFThreads = (kCons + 1) * 32;  // + the producer warp
constexpr int kMaxStages = 8;

struct FParams {
  int Hkv, T, nsplit, stages;
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
  static constexpr size_t tile_bytes = sizeof(T) * kTT * D;           // K (or V) rows of a tile
  static constexpr size_t stage_bytes = 2 * tile_bytes;               // K, then V
  static constexpr size_t off_q = 0;                                  // [G][D] fp32
  static constexpr size_t off_wacc = off_q + sizeof(float) * G * D;   // [kCons][G][D]
  static constexpr size_t off_wml = off_wacc + sizeof(float) * kCons * G * D;  // [kCons][G][2]
  static constexpr size_t off_fac = off_wml + sizeof(float) * kCons * G * 2;   // [kCons][G], [G][2]
  static constexpr size_t off_flag = off_fac + sizeof(float) * (kCons * G + 2 * G);
  static constexpr size_t off_bar = (off_flag + 16 + 15) & ~size_t(15);        // full, empty
  static constexpr size_t off_ring = (off_bar + 8 * 2 * kMaxStages + 127) & ~size_t(127);
  static size_t total(int stages) { return off_ring + stage_bytes * stages; }
};

// One lane's VEP channels of a K or V row (bf16 or fp32) in shared memory, as VEP / 2 float pairs.
template <typename T, int VEP>
__device__ __forceinline__ void load_pairs(const T* row, int lane, float2 (&f)[VEP / 2]) {
  if constexpr (sizeof(T) == 2) {
    if constexpr (VEP == 4) {
      const uint2 w = reinterpret_cast<const uint2*>(row)[lane];
      f[0] = make_float2(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xffff0000u));
      f[1] = make_float2(__uint_as_float(w.y << 16), __uint_as_float(w.y & 0xffff0000u));
    } else {
      const uint32_t w = reinterpret_cast<const uint32_t*>(row)[lane];
      f[0] = make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
    }
  } else {
    if constexpr (VEP == 4) {
      const float4 w = reinterpret_cast<const float4*>(row)[lane];
      f[0] = make_float2(w.x, w.y);
      f[1] = make_float2(w.z, w.w);
    } else {
      f[0] = reinterpret_cast<const float2*>(row)[lane];
    }
  }
}

template <int G>
__device__ __forceinline__ float pick_head(const float (&a)[G], int h) {
  float v = a[0];
#pragma unroll
  for (int i = 1; i < G; ++i) v = (h == i) ? a[i] : v;
  return v;
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kFThreads, 2) full_decode_kernel(const __grid_constant__ FParams p) {
  using LY = FLayout<T, D, G>;
  constexpr int VEP = D / 32;                // channels per lane
  constexpr int RPW = kTT / kGroupW;         // rows of a tile per consumer warp: 8
  constexpr int GR = (32 / G < RPW) ? 32 / G : RPW;  // rows per group: 8 (4 for 8 heads)
  constexpr int NV = GR * G;                 // (row, head) logits of a group
  constexpr int LPV = 32 / NV;               // lanes per (row, head) after the reduce
  static_assert(NV <= 32 && RPW % GR == 0, "unsupported head layout");
  extern __shared__ __align__(128) unsigned char sm[];
  float* q_s = reinterpret_cast<float*>(sm + LY::off_q);
  float* wacc = reinterpret_cast<float*>(sm + LY::off_wacc);
  float* wml = reinterpret_cast<float*>(sm + LY::off_wml);
  float* fac = reinterpret_cast<float*>(sm + LY::off_fac);
  int* flag = reinterpret_cast<int*>(sm + LY::off_flag);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + LY::off_bar);
  uint64_t* empty = full + kMaxStages;
  unsigned char* ring = sm + LY::off_ring;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int NS = p.stages;
  const int bk = blockIdx.x / p.nsplit, split = blockIdx.x % p.nsplit;
  const int b = bk / p.Hkv;
  int Tb = p.ctx_lens ? p.ctx_lens[b] : p.T;
  Tb = max(0, min(Tb, p.T));
  const int per = ((Tb + p.nsplit - 1) / p.nsplit + kTT - 1) / kTT * kTT;
  const int t0 = min(Tb, split * per), t1 = min(Tb, t0 + per);
  const int ntiles = (t1 - t0 + kTT - 1) / kTT;
  const T* Kb = static_cast<const T*>(p.K) + (static_cast<size_t>(bk) * p.T + t0) * D;
  const T* Vb = static_cast<const T*>(p.V) + (static_cast<size_t>(bk) * p.T + t0) * D;

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kGroupW);
    }
    flag[1] = 0;
    mbar_init_fence();
  }
  {
    const T* qp = static_cast<const T*>(p.q) + static_cast<size_t>(bk) * G * D;
    for (int i = tid; i < G * D; i += kFThreads) q_s[i] = to_float(qp[i]);
  }
  __syncthreads();

  if (warp == kCons) {  // ---- producer: tile i into stage i % NS once its last use is released
    const uint64_t policy = l2_evict_first_policy();
    int issued = 0;
    for (int i = 0; i < ntiles; ++i) {
      const int st = i % NS;
      if (i >= NS) {
        bool got = mbar_wait(&empty[st], static_cast<uint32_t>((i / NS - 1) & 1), p.status);
        got = __all_sync(0xffffffffu, got);
        if (!got) {
          if (lane == 0) flag[1] = 1;
          break;
        }
        fence_proxy_async();
      }
      if (lane == 0) {
        const int rows = min(kTT, t1 - t0 - i * kTT);
        const uint32_t bytes = static_cast<uint32_t>(rows) * D * sizeof(T);
        unsigned char* sb = ring + LY::stage_bytes * st;
        mbar_arrive_expect_tx(&full[st], 2 * bytes);
        bulk_g2s_stream(sb, Kb + static_cast<size_t>(i) * kTT * D, bytes, &full[st], policy);
        bulk_g2s_stream(sb + LY::tile_bytes, Vb + static_cast<size_t>(i) * kTT * D, bytes, &full[st], policy);
      }
      ++issued;
    }
    if (*reinterpret_cast<volatile int*>(&flag[1]) != 0) {  // gave up: drain the copies in flight
      for (int i = max(0, issued - NS); i < issued; ++i)
        mbar_wait(&full[i % NS], static_cast<uint32_t>((i / NS) & 1), nullptr);
    }
  } else {  // ---- consumers: warp w takes rows [8 (w % 4), 8 (w % 4) + 8) of the tiles i = w / 4 mod 2
    constexpr int VP = VEP / 2;               // channel pairs per lane
    float2 qv[G][VP];
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int e = 0; e < VP; ++e) qv[h][e] = make_float2(q_s[h * D + lane * VEP + 2 * e], q_s[h * D + lane * VEP + 2 * e + 1]);
    float2 acc[G][VP];
    float mw[G], lw[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      mw[h] = -CUDART_INF_F;
      lw[h] = 0.f;
#pragma unroll
      for (int e = 0; e < VP; ++e) acc[h][e] = make_float2(0.f, 0.f);
    }
    const int my_v = lane / LPV, my_r = my_v / G, my_h = my_v % G;
    const int grp = warp / kGroupW, wi = warp % kGroupW;
    bool ok = true;
#pragma unroll 1
    for (int i = grp; i < ntiles; i += kGroups) {
      const int st = i % NS;
      ok = __all_sync(0xffffffffu, ok && mbar_wait(&full[st], static_cast<uint32_t>((i / NS) & 1), p.status));
      const int rows = ok ? min(kTT, t1 - t0 - i * kTT) : 0;
      const T* kt = reinterpret_cast<const T*>(ring + LY::stage_bytes * st);
      const T* vt = reinterpret_cast<const T*>(ring + LY::stage_bytes * st + LY::tile_bytes);
#pragma unroll
      for (int g0 = 0; g0 < RPW; g0 += GR) {
        const int r0 = wi * RPW + g0;  // the group's first row in the tile
        if (r0 >= rows) break;
        float v[NV];
#pragma unroll
        for (int r = 0; r < GR; ++r) {
          float2 kf[VP];
          if (r0 + r < rows) {
            load_pairs<T, VEP>(kt + (r0 + r) * D, lane, kf);
          } else {
#pragma unroll
            for (int e = 0; e < VP; ++e) kf[e] = make_float2(0.f, 0.f);
          }
#pragma unroll
          for (int h = 0; h < G; ++h) {
            float2 s2 = __fmul2_rn(qv[h][0], kf[0]);
#pragma unroll
            for (int e = 1; e < VP; ++e) s2 = __ffma2_rn(qv[h][e], kf[e], s2);
            v[r * G + h] = s2.x + s2.y;
          }
        }
        TransposeReduce<NV, 16>::run(v, lane);  // lane holds (row my_r, head my_h)
        const float lg = (r0 + my_r < rows) ? p.scale * v[0] : -CUDART_INF_F;
        float gm = lg;
#pragma unroll
        for (int o = LPV * G; o < 32; o <<= 1) gm = fmaxf(gm, __shfl_xor_sync(0xffffffffu, gm, o));
        float mn[G], sc[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float gh = __shfl_sync(0xffffffffu, gm, h * LPV);
          mn[h] = fmaxf(mw[h], gh);
          sc[h] = (mw[h] == -CUDART_INF_F) ? 0.f : __expf(mw[h] - mn[h]);
        }
        const float pe = (lg == -CUDART_INF_F) ? 0.f : __expf(lg - pick_head<G>(mn, my_h));
        float ps = pe;
#pragma unroll
        for (int o = LPV * G; o < 32; o <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
#pragma unroll
        for (int h = 0; h < G; ++h) {
          lw[h] = lw[h] * sc[h] + __shfl_sync(0xffffffffu, ps, h * LPV);
          mw[h] = mn[h];
          const float2 s2 = make_float2(sc[h], sc[h]);
#pragma unroll
          for (int e = 0; e < VP; ++e) acc[h][e] = __fmul2_rn(acc[h][e], s2);
        }
#pragma unroll
        for (int r = 0; r < GR; ++r) {
          if (r0 + r < rows) {  // rows past the range carry weight 0 and are skipped
            float2 vf[VP];
            load_pairs<T, VEP>(vt + (r0 + r) * D, lane, vf);
#pragma unroll
            for (int h = 0; h < G; ++h) {
              const float prh = __shfl_sync(0xffffffffu, pe, (r * G + h) * LPV);
              const float2 p2 = make_float2(prh, prh);
#pragma unroll
              for (int e = 0; e < VP; ++e) acc[h][e] = __ffma2_rn(p2, vf[e], acc[h][e]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
    }
    // this warp's partial
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int e = 0; e < VP; ++e)
        *reinterpret_cast<float2*>(wacc + (warp * G + h) * D + lane * VEP + 2 * e) = acc[h][e];
    if (lane == 0) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        wml[(warp * G + h) * 2] = mw[h];
        wml[(warp * G + h) * 2 + 1] = lw[h];
      }
    }
  }
  __syncthreads();

  // ---- the 8 warps' partials -> this split's partial in the workspace
  float* mine = p.part + (static_cast<size_t>(bk) * p.nsplit + split) * G * (D + 2);
  float* wf = fac;                 // [kCons][G] factors
  float* sml = fac + kCons * G;    // [G][2] the split's (max, sum)
  if (warp < G) {
    const int h = warp;
    const float mwv = lane < kCons ? wml[(lane * G + h) * 2] : -CUDART_INF_F;
    const float M = warp_max(mwv);
    const float f = exp_diff(mwv, M);
    const float Ls = warp_sum(lane < kCons ? f * wml[(lane * G + h) * 2 + 1] : 0.f);
    if (lane < kCons) wf[lane * G + h] = f;
    if (lane == 0) {
      sml[2 * h] = M;
      sml[2 * h + 1] = Ls;
    }
  }
  __syncthreads();
  for (int i = tid; i < G * D; i += kFThreads) {
    const int h = i / D;
    float a = 0.f;
#pragma unroll
    for (int w = 0; w < kCons; ++w) a = fmaf(wf[w * G + h], wacc[(w * G + h) * D + (i % D)], a);
    mine[h * (D + 2) + 2 + (i % D)] = a;
  }
  if (tid < G) {
    mine[tid * (D + 2)] = sml[2 * tid];
    mine[tid * (D + 2) + 1] = sml[2 * tid + 1];
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) flag[0] = (atomicAdd(&p.counters[bk], 1u) == static_cast<uint32_t>(p.nsplit - 1));
  __syncthreads();
  if (!flag[0]) return;

  // ---- last CTA of this kv-head: merge the splits
  __threadfence();
  const float* parts = p.part + static_cast<size_t>(bk) * p.nsplit * G * (D + 2);
  float* ml_s = sml;
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
  for (int i = tid; i < G * D; i += kFThreads) {
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

// Stages that keep two CTAs per SM (the tile ring is the bulk of the shared memory).
template <typename T, int D, int G>
int stages_for() {
  using LY = FLayout<T, D, G>;
  int s = kMaxStages;
  while (s > 2 && LY::total(s) > (113u << 10)) --s;
  return s;
}

template <typename T, int D, int G>
cudaError_t launch_t(const FullArgs& a, cudaStream_t st) {
  auto kern = full_decode_kernel<T, D, G>;
  const int stages = stages_for<T, D, G>();
  const size_t smem = FLayout<T, D, G>::total(stages);
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
  p.stages = stages;
  p.scale = a.scale;
  p.q = a.q;
  p.K = a.K;
  p.V = a.V;
  p.ctx_lens = a.ctx_lens;
  p.out = a.out;
  p.part = a.part;
  p.counters = a.counters;
  p.status = a.status;
  full_decode_kernel<T, D, G><<<a.B * a.Hkv * a.nsplit, kFThreads, smem, st>>>(p);
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
  int ns = (2 * sms + pairs - 1) / pairs;  // about two CTAs per SM over all kv-heads
  ns = ns < 1 ? 1 : ns;
  const int mx = max_full_splits(T);
  return ns > mx ? mx : ns;
}

cudaError_t launch_full_decode(const FullArgs& a, cudaStream_t st) {
  if (a.bf16) return a.D == 128 ? dispatch_g<uint16_t, 128>(a, st) : dispatch_g<uint16_t, 64>(a, st);
  return a.D == 128 ? dispatch_g<float, 128>(a, st) : dispatch_g<float, 64>(a, st);
}

}  // namespace compkv
