// a1 (first half). Streams the block summaries once and computes, per block and query head, the
// log of the compensation-aware score, together with the per-head partial sums the selection and
// the attention need (CompKV review, Summary: residual of an omitted block governed by its mass
// and within-block logit variance, Section 3 Eq. 4-7; second-order mass estimate):
//
//   lbar = s q_h . mu_j          V = s^2 sum_g |q_{h,C_g}|^2 var_{j,g}       x = lbar + log n_j
//   log m = x + log(1 + V/2)     u = log m + log(V/2)   (mass modes: u = log m)
//   Zhat partial:  (max, sum) of exp(log m) over the segment
//   compensation:  (m_ref, sum n e^{lbar - m_ref}, sum n e^{lbar - m_ref} nu) over the segment
//
// Work split (B200): the (sequence, kv-head) tiles of 32 blocks are laid end to end and cut into
// equal contiguous ranges, one per CTA, two CTAs per SM, so every SM streams the same number of
// bytes whatever B and Hkv are. A CTA's range crosses at most a few (sequence, kv-head) pairs; it
// writes one partial record per pair it touches ("segment"). The mean keys and mean values of a
// tile arrive by bulk copy and the grouped variances and counts by 4-byte cp.async, on one
// mbarrier per stage of a 3-deep ring.
//
// Per tile there is one CTA barrier. The D/8 lanes of a block dot its mean key with the G heads
// (transpose-reduce); the lane that ends up holding head h's dot does the scalar work for that
// (block, head) and keeps its own running Zhat and compensation sums. Compensation weights use a
// reference m_ref per head that only moves up when a logit would exceed it by 64 (e^64 keeps
// every sum finite in fp32), so the common tile needs no max-reduction; the rare tile that moves
// it takes one extra barrier. Weights go through a double-buffered shared array to the
// accumulation, where each thread owns 4 channels of all G heads, so each mean value is read
// from shared memory once.
#include <mutex>

#include "attend.cuh"
#include "common.cuh"
#include "internal.h"

namespace compkv {
namespace {

constexpr int kTile = kStreamTile;
constexpr int kStages = 3;
constexpr float kRefSlack = 64.f;

struct StreamParams {
  int mode, Nb, tiles_per_pair, total_tiles, nctas, slots, r;
  float scale;
  const void* q;
  const float* mean_k;
  const float* var_g;
  const float* mean_v;
  const int32_t* count;
  float* u;        // [pairs][Nb][G]
  float* zpart;    // [pairs][slots][G][2]
  float* comp;     // [pairs][slots][G][D+2]
  int32_t* status;
};

__host__ __device__ inline size_t a16(size_t x) { return (x + 15) & ~static_cast<size_t>(15); }

struct SLay {
  size_t stage_bytes, off_mu, off_nu, off_var, off_cnt, stage0, mbar, ws, q, qn, comp, red, misc, total;
  __host__ __device__ void build(int D, int G, int r) {
    off_mu = 0;
    off_nu = a16(sizeof(float) * kTile * D);
    off_var = a16(off_nu + sizeof(float) * kTile * D);
    off_cnt = a16(off_var + sizeof(float) * kTile * r);
    stage_bytes = a16(off_cnt + sizeof(int) * kTile);
    size_t o = 0;
    mbar = o;   o = a16(o + 8 * kStages);
    stage0 = o; o = a16(o + stage_bytes * kStages);
    ws = o;     o = a16(o + sizeof(float) * 2 * kTile * G);   // double-buffered weights [2][kTile][G]
    q = o;      o = a16(o + sizeof(float) * G * D);
    qn = o;     o = a16(o + sizeof(float) * G * r);
    comp = o;   o = a16(o + sizeof(float) * G * D);
    red = o;    o = a16(o + sizeof(float) * 3 * G * 64);      // per-head lane-slot reductions
    misc = o;   o = a16(o + sizeof(float) * 64);   // mref[8] sc[8] tmax[3][8] flag[3] logn[17]
    total = o;
  }
};

// Ordered int of a float (monotone), for shared-memory atomicMax.
__device__ __forceinline__ int ord_float(float f) {
  const int i = __float_as_int(f);
  return i >= 0 ? i : i ^ 0x7fffffff;
}
__device__ __forceinline__ float unord_float(int i) { return __int_as_float(i >= 0 ? i : i ^ 0x7fffffff); }

template <typename TQ, int D, int G>
__global__ void __launch_bounds__(kThreads, 2) score_stream_kernel(const __grid_constant__ StreamParams p) {
  extern __shared__ __align__(128) unsigned char sm[];
  SLay L;
  L.build(D, G, p.r);
  const int r = p.r;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool compensate = p.mode != COMPKV_MODE_MASS;
  const int F = p.total_tiles, TP = p.tiles_per_pair;
  const int f0 = static_cast<int>((static_cast<long long>(blockIdx.x) * F) / p.nctas);
  const int f1 = static_cast<int>((static_cast<long long>(blockIdx.x + 1) * F) / p.nctas);
  const int nt = f1 - f0;

  uint64_t* mbar = reinterpret_cast<uint64_t*>(sm + L.mbar);
  float* ws_s = reinterpret_cast<float*>(sm + L.ws);
  float* q_s = reinterpret_cast<float*>(sm + L.q);
  float* qn_s = reinterpret_cast<float*>(sm + L.qn);
  float* comp_s = reinterpret_cast<float*>(sm + L.comp);
  float* red_s = reinterpret_cast<float*>(sm + L.red);
  float* mref_s = reinterpret_cast<float*>(sm + L.misc);        // [8] compensation reference
  float* sc_s = mref_s + 8;                                       // [8] rescale factors
  int* tmax_s = reinterpret_cast<int*>(mref_s + 16);              // [3][8] tile max (ordered)
  int* flag_s = tmax_s + 24;                                      // [3]
  float* logn_s = mref_s + 44;                                    // [17]
  const uint64_t policy = l2_evict_first_policy();

  auto tile_pair = [&](int f) { return f / TP; };
  auto issue = [&](int k) {  // local tile k -> stage k % kStages
    const int f = f0 + k;
    const int pr = f / TP, t = f % TP;
    const int jt0 = t * kTile;
    const int tn = min(kTile, p.Nb - jt0);
    const size_t row0 = static_cast<size_t>(pr) * p.Nb + jt0;
    const int st = k % kStages;
    unsigned char* sb = sm + L.stage0 + L.stage_bytes * st;
    float* var_d = reinterpret_cast<float*>(sb + L.off_var);
    int* cnt_d = reinterpret_cast<int*>(sb + L.off_cnt);
    for (int i = tid; i < tn * r; i += kThreads) cp_async4(var_d + i, p.var_g + row0 * r + i);
    for (int i = tid; i < tn; i += kThreads) cp_async4(cnt_d + i, p.count + row0 + i);
    if (tid == 0) {
      const uint32_t bytes = static_cast<uint32_t>(tn) * D * sizeof(float);
      mbar_arrive_expect_tx(&mbar[st], compensate ? 2 * bytes : bytes);
      bulk_g2s_stream(sb + L.off_mu, p.mean_k + row0 * D, bytes, &mbar[st], policy);
      if (compensate) bulk_g2s_stream(sb + L.off_nu, p.mean_v + row0 * D, bytes, &mbar[st], policy);
    }
    cp_async_arrive(&mbar[st]);
  };

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&mbar[s], kThreads + 1);
    mbar_init_fence();
  }
  if (tid < 17) logn_s[tid] = tid > 0 ? logf(static_cast<float>(tid)) : -CUDART_INF_F;
  __syncthreads();
  for (int k = 0; k < min(nt, kStages - 1); ++k) issue(k);
  pdl_launch_dependents();

  constexpr int LPB = D / 8;           // lanes per block in the dot phase
  constexpr int BPP = 32 / LPB;        // blocks per warp per pass
  constexpr int PASSES = kTile / (kWarps * BPP);
  constexpr int LPH = LPB / G;         // lanes per head after the transpose-reduce
  constexpr int NC4 = D / 4;
  constexpr int NJS = kThreads / NC4;  // block subsets of the accumulation phase
  const int li = lane % LPB, bsub = lane / LPB;
  const bool head_lane = (li % LPH) == 0;
  const int my_h = li / LPH;
  const int c4 = tid % NC4, js = tid / NC4;
  // lane-slot index of this head lane among all head lanes of head my_h (for reductions)
  const int slot = warp * BPP + bsub;  // < kWarps * BPP <= 32

  float qreg[G][8];
  float acc[G][4];
  float zmax = -CUDART_INF_F, zsum = 0.f, lsum = 0.f;
  int cur = -1;
  int issued = min(nt, kStages - 1);

  // Writes the partials of the current segment (pair `cur`) and clears the running state.
  auto finish_segment = [&]() {
    if (head_lane) {
      red_s[(0 * G + my_h) * 64 + slot] = zmax;
      red_s[(1 * G + my_h) * 64 + slot] = zsum;
      red_s[(2 * G + my_h) * 64 + slot] = lsum;
    }
    if (compensate) {  // fixed order over the block subsets, so results are deterministic
      for (int w = 0; w < NJS; ++w) {
        if (js == w) {
#pragma unroll
          for (int h = 0; h < G; ++h)
#pragma unroll
            for (int e = 0; e < 4; ++e) comp_s[h * D + c4 * 4 + e] += acc[h][e];
        }
        __syncthreads();
      }
    }
    __syncthreads();
    const int k = blockIdx.x - static_cast<int>(((static_cast<long long>(cur) * TP + 1) * p.nctas - 1) / F);
    const size_t rec = static_cast<size_t>(cur) * p.slots + k;
    constexpr int NSL = kWarps * BPP;
    if (tid < G) {
      float zm = -CUDART_INF_F, zs = 0.f, ls = 0.f;
      for (int s = 0; s < NSL; ++s) {
        lse_merge(zm, zs, red_s[(0 * G + tid) * 64 + s], red_s[(1 * G + tid) * 64 + s]);
        ls += red_s[(2 * G + tid) * 64 + s];
      }
      p.zpart[(rec * G + tid) * 2] = zm;
      p.zpart[(rec * G + tid) * 2 + 1] = zs;
      if (compensate) {
        p.comp[(rec * G + tid) * (D + 2)] = mref_s[tid];
        p.comp[(rec * G + tid) * (D + 2) + 1] = ls;
      }
    }
    if (compensate)
      for (int i = tid; i < G * D; i += kThreads) p.comp[(rec * G + i / D) * (D + 2) + 2 + (i % D)] = comp_s[i];
    __syncthreads();
  };

  // Loads the query heads of pair `pr` and resets the running state.
  auto start_segment = [&](int pr) {
    const TQ* qp = static_cast<const TQ*>(p.q) + static_cast<size_t>(pr) * G * D;
    for (int i = tid; i < G * D; i += kThreads) {
      q_s[i] = to_float(qp[i]);
      comp_s[i] = 0.f;
    }
    if (tid < 8) mref_s[tid] = -CUDART_INF_F;
    if (tid < 24) tmax_s[tid] = ord_float(-CUDART_INF_F);
    if (tid < 3) flag_s[tid] = 0;
    __syncthreads();
    const int gsz = D / r;
    for (int i = tid; i < G * r; i += kThreads) {
      const int h = i / r, g = i % r;
      float s = 0.f;
      for (int c = 0; c < gsz; ++c) {
        const float x = q_s[h * D + g * gsz + c];
        s = fmaf(x, x, s);
      }
      qn_s[i] = p.scale * p.scale * s;
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        qreg[h][e] = q_s[h * D + li * 4 + e];
        qreg[h][4 + e] = q_s[h * D + D / 2 + li * 4 + e];
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[h][e] = 0.f;
    }
    zmax = -CUDART_INF_F;
    zsum = lsum = 0.f;
    __syncthreads();
  };

  bool ok = true;
  int waited = nt;
#pragma unroll 1
  for (int k = 0; k < nt; ++k) {
    const int f = f0 + k;
    const int pr = tile_pair(f);
    if (pr != cur) {
      if (cur >= 0) finish_segment();
      start_segment(pr);
      cur = pr;
    }
    const int jt0 = (f % TP) * kTile;
    const int tn = min(kTile, p.Nb - jt0);
    const int st = k % kStages;
    const unsigned char* sb = sm + L.stage0 + L.stage_bytes * st;
    const float* mu_t = reinterpret_cast<const float*>(sb + L.off_mu);
    const float* nu_t = reinterpret_cast<const float*>(sb + L.off_nu);
    const float* var_t = reinterpret_cast<const float*>(sb + L.off_var);
    const int* cnt_t = reinterpret_cast<const int*>(sb + L.off_cnt);
    // weights: double buffer (written in phase 1 of tile k, read after its barrier). Tile max and
    // the reference flag: 3-deep ring; thread 0 clears tile k+1's entry here, which lies after
    // the barrier that ends tile k-2's readers and before the barrier that starts tile k+1.
    float* ws_b = ws_s + (k & 1) * kTile * G;
    const int buf = k % 3;
    if (tid == 0) {
      const int nb3 = (k + 1) % 3;
#pragma unroll
      for (int h = 0; h < 8; ++h) tmax_s[nb3 * 8 + h] = ord_float(-CUDART_INF_F);
      flag_s[nb3] = 0;
    }
    const bool got = mbar_wait(&mbar[st], (k / kStages) & 1, p.status);

    // ---- (1) dots, scalars, log scores, running Zhat and compensation sums
    float xs[PASSES], wv[PASSES];
    const float mref = compensate ? mref_s[my_h] : 0.f;
    const float lprev = lsum;
#pragma unroll
    for (int pass = 0; pass < PASSES; ++pass) {
      const int jt = pass * kWarps * BPP + warp * BPP + bsub;
      const float4 a = reinterpret_cast<const float4*>(mu_t + jt * D)[li];
      const float4 b = reinterpret_cast<const float4*>(mu_t + jt * D + D / 2)[li];
      float v[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float s = qreg[h][0] * a.x;
        s = fmaf(qreg[h][1], a.y, s);
        s = fmaf(qreg[h][2], a.z, s);
        s = fmaf(qreg[h][3], a.w, s);
        s = fmaf(qreg[h][4], b.x, s);
        s = fmaf(qreg[h][5], b.y, s);
        s = fmaf(qreg[h][6], b.z, s);
        s = fmaf(qreg[h][7], b.w, s);
        v[h] = s;
      }
      TransposeReduce<G, LPB / 2>::run(v, li);
      xs[pass] = -CUDART_INF_F;
      wv[pass] = 0.f;
      if (head_lane && jt < tn) {
        const int n = cnt_t[jt];
        float vh = 0.f;
        for (int g = 0; g < r; ++g) vh = fmaf(qn_s[my_h * r + g], var_t[jt * r + g], vh);
        const float lbar = p.scale * v[0];
        float uu;
        if (n > 0) {
          const float x = lbar + logn_s[min(n, 16)];
          const float lm = x + __logf(1.f + 0.5f * vh);
          uu = (p.mode == COMPKV_MODE_COMPKV) ? lm + __logf(0.5f * vh) : lm;
          xs[pass] = x;
          if (lm > zmax) {
            zsum = zsum * __expf(zmax - lm) + 1.f;
            zmax = lm;
          } else {
            zsum += __expf(lm - zmax);
          }
          if (compensate) {
            atomicMax(&tmax_s[buf * 8 + my_h], ord_float(x));
            if (x > mref + kRefSlack) flag_s[buf] = 1;
            else wv[pass] = __expf(x - mref);
          }
        } else {
          uu = __int_as_float(0x7fffffff);  // NaN marks an empty block
        }
        p.u[((static_cast<size_t>(pr) * p.Nb) + jt0 + jt) * G + my_h] = uu;
      }
      if (compensate && head_lane) {
        ws_b[jt * G + my_h] = wv[pass];
        lsum += wv[pass];
      }
    }
    ok = __syncthreads_and(got) != 0;
    if (!ok) {
      waited = k;
      break;
    }
    if (k + kStages - 1 < nt) {
      issue(k + kStages - 1);
      ++issued;
    }
    if (compensate) {
      if (flag_s[buf]) {  // rare: move the reference of the heads that need it and rescale
        if (tid < G) {
          const float old = mref_s[tid];
          const float tm = unord_float(tmax_s[buf * 8 + tid]);
          const float nm = (tm > old + kRefSlack) ? tm : old;
          sc_s[tid] = (old == -CUDART_INF_F) ? 0.f : __expf(old - nm);
          mref_s[tid] = nm;
        }
        __syncthreads();
        const float nref = mref_s[my_h];
        lsum = lprev * sc_s[my_h];
#pragma unroll
        for (int pass = 0; pass < PASSES; ++pass) {
          const int jt = pass * kWarps * BPP + warp * BPP + bsub;
          const float w = (xs[pass] == -CUDART_INF_F) ? 0.f : __expf(xs[pass] - nref);
          if (head_lane) {
            ws_b[jt * G + my_h] = w;
            lsum += w;
          }
        }
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float sc = sc_s[h];
          acc[h][0] *= sc; acc[h][1] *= sc; acc[h][2] *= sc; acc[h][3] *= sc;
        }
        __syncthreads();
      }
      // ---- (2) acc_h += w_{j,h} nu_j: 4 channels x G heads per thread
      for (int jt = js; jt < tn; jt += NJS) {
        const float4 nv = reinterpret_cast<const float4*>(nu_t + jt * D)[c4];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float w = ws_b[jt * G + h];
          acc[h][0] = fmaf(w, nv.x, acc[h][0]);
          acc[h][1] = fmaf(w, nv.y, acc[h][1]);
          acc[h][2] = fmaf(w, nv.z, acc[h][2]);
          acc[h][3] = fmaf(w, nv.w, acc[h][3]);
        }
      }
    }
  }
  if (!ok) {
    for (int k = waited; k < issued; ++k) mbar_wait(&mbar[k % kStages], (k / kStages) & 1, nullptr);
  } else if (cur >= 0) {
    finish_segment();
  }
}

template <typename TQ, int D, int G>
const void* kptr() {
  return reinterpret_cast<const void*>(&score_stream_kernel<TQ, D, G>);
}

const void* pick(bool bf16, int D, int G) {
#define COMPKV_PICK(T, DD)                  \
  switch (G) {                              \
    case 1: return kptr<T, DD, 1>();        \
    case 2: return kptr<T, DD, 2>();        \
    case 4: return kptr<T, DD, 4>();        \
    case 8: return kptr<T, DD, 8>();        \
  }
  if (bf16) {
    if (D == 128) { COMPKV_PICK(uint16_t, 128) } else { COMPKV_PICK(uint16_t, 64) }
  } else {
    if (D == 128) { COMPKV_PICK(float, 128) } else { COMPKV_PICK(float, 64) }
  }
#undef COMPKV_PICK
  return nullptr;
}

struct Grid {
  const void* kern = nullptr;
  int dev = -1, D = 0, G = 0, r = 0;
  int ctas_per_sm = 0, sms = 0;
  size_t smem = 0;
};
Grid g_grids[16];
int g_ngrids = 0;
std::mutex g_mu;

cudaError_t grid_for(const void* kern, int D, int G, int r, Grid* out) {
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(g_mu);
  for (int i = 0; i < g_ngrids; ++i)
    if (g_grids[i].kern == kern && g_grids[i].dev == dev && g_grids[i].r == r) {
      *out = g_grids[i];
      return cudaSuccess;
    }
  Grid g;
  g.kern = kern;
  g.dev = dev;
  g.D = D;
  g.G = G;
  g.r = r;
  SLay L;
  L.build(D, G, r);
  g.smem = L.total;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(g.smem));
  if (e != cudaSuccess) return e;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&g.ctas_per_sm, kern, kThreads, g.smem);
  if (e != cudaSuccess) return e;
  if (g.ctas_per_sm < 1) return cudaErrorInvalidConfiguration;
  cudaDeviceGetAttribute(&g.sms, cudaDevAttrMultiProcessorCount, dev);
  if (g_ngrids < 16) g_grids[g_ngrids++] = g;
  *out = g;
  return cudaSuccess;
}

}  // namespace

int stream_ctas(int total_tiles, int sms, int ctas_per_sm) {
  int n = sms * (ctas_per_sm < 2 ? ctas_per_sm : 2);
  if (n > kStreamMaxCtas) n = kStreamMaxCtas;
  if (n > total_tiles) n = total_tiles;
  return n < 1 ? 1 : n;
}

cudaError_t launch_score_stream(const StreamArgs& a, cudaStream_t st) {
  const void* kern = pick(a.bf16, a.D, a.G);
  if (!kern) return cudaErrorInvalidValue;
  Grid g;
  cudaError_t e = grid_for(kern, a.D, a.G, a.r, &g);
  if (e != cudaSuccess) return e;
  StreamParams p;
  p.mode = a.mode;
  p.Nb = a.Nb;
  p.tiles_per_pair = (a.Nb + kTile - 1) / kTile;
  p.total_tiles = a.pairs * p.tiles_per_pair;
  p.nctas = stream_ctas(p.total_tiles, g.sms, g.ctas_per_sm);
  p.slots = a.slots;
  p.r = a.r;
  p.scale = a.scale;
  p.q = a.q;
  p.mean_k = a.mean_k;
  p.var_g = a.var_g;
  p.mean_v = a.mean_v;
  p.count = a.count;
  p.u = a.u;
  p.zpart = a.zpart;
  p.comp = a.comp_seg;
  p.status = a.status;
  if (a.nctas_out) *a.nctas_out = p.nctas;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.nctas, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = g.smem;
  cfg.stream = st;
  cfg.numAttrs = 0;
  void* args[] = {&p};
  return cudaLaunchKernelExC(&cfg, kern, args);
}

int stream_grid_ctas(bool bf16, int D, int G, int r, int total_tiles) {
  const void* kern = pick(bf16, D, G);
  Grid g;
  if (!kern || grid_for(kern, D, G, r, &g) != cudaSuccess) return -1;
  return stream_ctas(total_tiles, g.sms, g.ctas_per_sm);
}

}  // namespace compkv
