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
// writes one partial record per pair it touches ("segment").
//
// Pipeline: a 3-stage shared-memory ring with a "full" and an "empty" mbarrier per stage. Warp 0
// refills a stage (bulk copies of the tile's mean keys and mean values, 4-byte cp.async of its
// grouped variances and counts) once all 8 warps have released it. Each warp owns 4 blocks of
// every tile and works through the ring on its own, with no CTA barrier in steady state: its
// lanes dot the mean keys with the G heads (transpose-reduce), the lane left holding head h's dot
// does that (block, head)'s scalar work, and the warp accumulates its blocks' weighted mean
// values for all G heads (4 channels per lane). Compensation weights are taken against a
// per-warp reference logit per head that only moves up when a logit would exceed it by 64 (e^64
// keeps every sum finite in fp32). Warps meet only where a segment ends, to merge their partials
// in a fixed order (deterministic results).
//
// Besides the log scores u it writes, per block, the record {x_h (h < G), n_j} that lets the
// attention kernel add and remove the block's compensation term without re-reading its summary.
#include <mutex>

#include "attend.cuh"
#include "common.cuh"
#include "internal.h"

namespace compkv {
namespace {

constexpr int kTile = kStreamTile;
constexpr int kStages = 3;
constexpr int kBlocksPerWarp = kTile / kWarps;  // 4
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
  float* xrec;     // [pairs][Nb][xrec_stride(G)]  {x_0..x_{G-1}, n}
  float* zpart;    // [pairs][slots][G][2]
  float* comp;     // [pairs][slots][G][D+2]
  int32_t* status;
};

__host__ __device__ inline size_t a16(size_t x) { return (x + 15) & ~static_cast<size_t>(15); }

struct SLay {
  size_t stage_bytes, off_mu, off_nu, off_var, off_cnt, stage0, full, empty, wsw, q, qn, comp, refw, red, logn, total;
  __host__ __device__ void build(int D, int G, int r) {
    off_mu = 0;
    off_nu = a16(sizeof(float) * kTile * D);
    off_var = a16(off_nu + sizeof(float) * kTile * D);
    off_cnt = a16(off_var + sizeof(float) * kTile * r);
    stage_bytes = a16(off_cnt + sizeof(int) * kTile);
    size_t o = 0;
    full = o;   o = a16(o + 8 * kStages);
    empty = o;  o = a16(o + 8 * kStages);
    stage0 = o; o = a16(o + stage_bytes * kStages);
    wsw = o;    o = a16(o + sizeof(float) * kWarps * kBlocksPerWarp * G);   // per-warp weights
    q = o;      o = a16(o + sizeof(float) * G * D);
    qn = o;     o = a16(o + sizeof(float) * G * r);
    comp = o;   o = a16(o + sizeof(float) * G * D);
    refw = o;   o = a16(o + sizeof(float) * kWarps * G);
    red = o;    o = a16(o + sizeof(float) * 3 * G * 32);
    logn = o;   o = a16(o + sizeof(float) * 17);
    total = o;
  }
};

template <int G>
__device__ __forceinline__ float pick_h(const float (&a)[G], int h) {
  float v = a[0];
#pragma unroll
  for (int i = 1; i < G; ++i) v = (h == i) ? a[i] : v;
  return v;
}

// R = 4 specialises the default group count (grouped variances as one float4); R = 0 is any r.
template <typename TQ, int D, int G, int R>
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
  constexpr int XS = xrec_stride(G);

  uint64_t* full = reinterpret_cast<uint64_t*>(sm + L.full);
  uint64_t* empty = reinterpret_cast<uint64_t*>(sm + L.empty);
  float* wsw = reinterpret_cast<float*>(sm + L.wsw) + warp * kBlocksPerWarp * G;
  float* q_s = reinterpret_cast<float*>(sm + L.q);
  float* qn_s = reinterpret_cast<float*>(sm + L.qn);
  float* comp_s = reinterpret_cast<float*>(sm + L.comp);
  float* refw_s = reinterpret_cast<float*>(sm + L.refw);
  float* red_s = reinterpret_cast<float*>(sm + L.red);
  float* logn_s = reinterpret_cast<float*>(sm + L.logn);
  const uint64_t policy = l2_evict_first_policy();

  // Refills the stage of local tile k (warp 0 only; all 32 lanes).
  auto issue = [&](int k) {
    const int f = f0 + k;
    const int pr = f / TP, t = f % TP;
    const int jt0 = t * kTile;
    const int tn = min(kTile, p.Nb - jt0);
    const size_t row0 = static_cast<size_t>(pr) * p.Nb + jt0;
    const int st = k % kStages;
    unsigned char* sb = sm + L.stage0 + L.stage_bytes * st;
    float* var_d = reinterpret_cast<float*>(sb + L.off_var);
    int* cnt_d = reinterpret_cast<int*>(sb + L.off_cnt);
    for (int i = lane; i < tn * r; i += 32) cp_async4(var_d + i, p.var_g + row0 * r + i);
    for (int i = lane; i < tn; i += 32) cp_async4(cnt_d + i, p.count + row0 + i);
    if (lane == 0) {
      const uint32_t bytes = static_cast<uint32_t>(tn) * D * sizeof(float);
      mbar_arrive_expect_tx(&full[st], compensate ? 2 * bytes : bytes);
      bulk_g2s_stream(sb + L.off_mu, p.mean_k + row0 * D, bytes, &full[st], policy);
      if (compensate) bulk_g2s_stream(sb + L.off_nu, p.mean_v + row0 * D, bytes, &full[st], policy);
    }
    cp_async_arrive(&full[st]);
  };

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 32 + 1);
      mbar_init(&empty[s], kWarps);
    }
    mbar_init_fence();
  }
  if (tid < 17) logn_s[tid] = tid > 0 ? logf(static_cast<float>(tid)) : -CUDART_INF_F;
  __syncthreads();
  int issued = min(nt, kStages);
  if (warp == 0)
    for (int k = 0; k < issued; ++k) issue(k);
  pdl_launch_dependents();

  constexpr int LPB = D / 8;            // lanes per block in the dot phase
  constexpr int BPP = 32 / LPB;         // blocks per warp per pass
  constexpr int PASSES = kBlocksPerWarp / BPP;
  constexpr int LPH = LPB / G;          // lanes per head after the transpose-reduce
  constexpr int LR = D / 4;             // lanes per mean-value row (4 channels per lane)
  constexpr int RS = 32 / LR;           // mean-value rows per warp step
  constexpr int NSL = kWarps * BPP * PASSES;  // scalar lanes per head in the CTA
  static_assert(PASSES <= LPH, "scalar lanes of a block must cover its passes");
  const int li = lane % LPB, bsub = lane / LPB;
  // after the transpose-reduce, lane li of a block group holds head li / LPH; the pass-p value is
  // moved p lanes up, so lane (h * LPH + p) does the scalar work of (pass p, head h)
  const int my_pass = li % LPH;
  const bool head_lane = my_pass < PASSES;
  const int my_h = li / LPH;
  const int my_bl = my_pass * BPP + bsub;  // block of this scalar lane within the warp's 4
  const int c4 = lane % LR, rsub = lane / LR;
  const int slot = (warp * BPP + bsub) * PASSES + my_pass;

  float2 qreg[G][4];
  float qnr[4];
  float acc[G][4];
  float mref[G];
  float zmax = -CUDART_INF_F, zsum = 0.f, lsum = 0.f;
  int cur = -1;

  // Merges the 8 warps' partials of the current segment (pair `cur`) in a fixed order.
  auto finish_segment = [&]() {
    if (RS > 1 && compensate) {  // fold the row subsets of each warp (D < 128)
#pragma unroll
      for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < 4; ++e)
#pragma unroll
          for (int o = LR; o < 32; o <<= 1) acc[h][e] += __shfl_xor_sync(0xffffffffu, acc[h][e], o);
    }
    if (lane == 0) {
#pragma unroll
      for (int h = 0; h < G; ++h) refw_s[warp * G + h] = mref[h];
    }
    if (head_lane) {
      red_s[(0 * G + my_h) * 32 + slot] = zmax;
      red_s[(1 * G + my_h) * 32 + slot] = zsum;
    }
    for (int i = tid; i < G * D; i += kThreads) comp_s[i] = 0.f;
    __syncthreads();
    float M[G], fw[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      M[h] = -CUDART_INF_F;
      for (int w = 0; w < kWarps; ++w) M[h] = fmaxf(M[h], refw_s[w * G + h]);
      fw[h] = (mref[h] == -CUDART_INF_F) ? 0.f : __expf(mref[h] - M[h]);
    }
    if (head_lane) red_s[(2 * G + my_h) * 32 + slot] = lsum * pick_h<G>(fw, my_h);
    if (compensate) {
      for (int w = 0; w < kWarps; ++w) {
        if (warp == w && rsub == 0) {
#pragma unroll
          for (int h = 0; h < G; ++h)
#pragma unroll
            for (int e = 0; e < 4; ++e) comp_s[h * D + c4 * 4 + e] += fw[h] * acc[h][e];
        }
        __syncthreads();
      }
    } else {
      __syncthreads();
    }
    const int k = blockIdx.x - static_cast<int>(((static_cast<long long>(cur) * TP + 1) * p.nctas - 1) / F);
    const size_t rec = static_cast<size_t>(cur) * p.slots + k;
    if (tid < G) {
      float zm = -CUDART_INF_F, zs = 0.f, ls = 0.f;
      for (int s = 0; s < NSL; ++s) {
        lse_merge(zm, zs, red_s[(0 * G + tid) * 32 + s], red_s[(1 * G + tid) * 32 + s]);
        ls += red_s[(2 * G + tid) * 32 + s];
      }
      p.zpart[(rec * G + tid) * 2] = zm;
      p.zpart[(rec * G + tid) * 2 + 1] = zs;
      if (compensate) {
        p.comp[(rec * G + tid) * (D + 2)] = pick_h<G>(M, tid);
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
    for (int i = tid; i < G * D; i += kThreads) q_s[i] = to_float(qp[i]);
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
    __syncthreads();
#pragma unroll
    for (int h = 0; h < G; ++h) {
      qreg[h][0] = make_float2(q_s[h * D + li * 4 + 0], q_s[h * D + li * 4 + 1]);
      qreg[h][1] = make_float2(q_s[h * D + li * 4 + 2], q_s[h * D + li * 4 + 3]);
      qreg[h][2] = make_float2(q_s[h * D + D / 2 + li * 4 + 0], q_s[h * D + D / 2 + li * 4 + 1]);
      qreg[h][3] = make_float2(q_s[h * D + D / 2 + li * 4 + 2], q_s[h * D + D / 2 + li * 4 + 3]);
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[h][e] = 0.f;
      mref[h] = -CUDART_INF_F;
    }
    if constexpr (R == 4) {
#pragma unroll
      for (int g = 0; g < 4; ++g) qnr[g] = qn_s[my_h * 4 + g];
    }
    zmax = -CUDART_INF_F;
    zsum = lsum = 0.f;
    __syncthreads();
  };

  // `ok` goes false (for this warp) once a wait gives up; the warp then stops waiting and
  // computing but keeps the loop's structure, so every CTA barrier stays matched.
  bool ok = true;
  int first_unwaited = nt;
#pragma unroll 1
  for (int k = 0; k < nt; ++k) {
    const int f = f0 + k;
    const int pr = f / TP;
    if (pr != cur) {  // every warp reaches this at the same tile
      __syncthreads();
      if (cur >= 0) finish_segment();
      start_segment(pr);
      cur = pr;
    }
    const int st = k % kStages;
    // warp 0 refills the stage of tile k + kStages - 1 once every warp has released tile k - 1
    if (warp == 0 && k >= 1 && k + kStages - 1 < nt) {
      const int kk = k + kStages - 1;
      bool freed = ok && mbar_wait(&empty[kk % kStages], ((kk / kStages) - 1) & 1, p.status);
      freed = __all_sync(0xffffffffu, freed);
      if (freed) {
        issue(kk);
        ++issued;
      } else {
        ok = false;
      }
    }
    bool got = ok && mbar_wait(&full[st], (k / kStages) & 1, p.status);
    got = __all_sync(0xffffffffu, got);
    if (!got && ok) {
      ok = false;
      first_unwaited = k;
    }
    const int jt0 = (f % TP) * kTile;
    const int tn = ok ? min(kTile, p.Nb - jt0) : 0;
    const unsigned char* sb = sm + L.stage0 + L.stage_bytes * st;
    const float* mu_t = reinterpret_cast<const float*>(sb + L.off_mu);
    const float* nu_t = reinterpret_cast<const float*>(sb + L.off_nu);
    const float* var_t = reinterpret_cast<const float*>(sb + L.off_var);
    const int* cnt_t = reinterpret_cast<const int*>(sb + L.off_cnt);

    // ---- (1) dots of this warp's blocks with the G heads
    float v[PASSES][G];
#pragma unroll
    for (int pass = 0; pass < PASSES; ++pass) {
      const int jt = warp * kBlocksPerWarp + pass * BPP + bsub;
      const float4 a = reinterpret_cast<const float4*>(mu_t + jt * D)[li];
      const float4 b = reinterpret_cast<const float4*>(mu_t + jt * D + D / 2)[li];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float2 s2 = __fmul2_rn(qreg[h][0], make_float2(a.x, a.y));
        s2 = __ffma2_rn(qreg[h][1], make_float2(a.z, a.w), s2);
        s2 = __ffma2_rn(qreg[h][2], make_float2(b.x, b.y), s2);
        s2 = __ffma2_rn(qreg[h][3], make_float2(b.z, b.w), s2);
        v[pass][h] = s2.x + s2.y;
      }
    }
#pragma unroll
    for (int pass = 0; pass < PASSES; ++pass) TransposeReduce<G, LPB / 2>::run(v[pass], li);
    float dot = v[0][0];
#pragma unroll
    for (int pass = 1; pass < PASSES; ++pass) {
      const float t = __shfl_up_sync(0xffffffffu, v[pass][0], pass);
      if (my_pass == pass) dot = t;
    }

    // ---- (2) per (block, head) scalars, one (block, head) per scalar lane
    float xs = -CUDART_INF_F;
    bool need = false;
    {
      const int jt = warp * kBlocksPerWarp + my_bl;
      if (head_lane && jt < tn) {
        const int n = cnt_t[jt];
        float vh;
        if constexpr (R == 4) {
          const float4 vv = reinterpret_cast<const float4*>(var_t)[jt];
          vh = qnr[0] * vv.x;
          vh = fmaf(qnr[1], vv.y, vh);
          vh = fmaf(qnr[2], vv.z, vh);
          vh = fmaf(qnr[3], vv.w, vh);
        } else {
          vh = 0.f;
          for (int g = 0; g < r; ++g) vh = fmaf(qn_s[my_h * r + g], var_t[jt * r + g], vh);
        }
        const float lbar = p.scale * dot;
        const size_t row = static_cast<size_t>(pr) * p.Nb + jt0 + jt;
        float uu;
        if (n > 0) {
          xs = lbar + logn_s[min(n, 16)];
          const float lm = xs + __logf(1.f + 0.5f * vh);
          uu = (p.mode == COMPKV_MODE_COMPKV) ? lm + __logf(0.5f * vh) : lm;
          if (lm > zmax) {
            zsum = zsum * __expf(zmax - lm) + 1.f;
            zmax = lm;
          } else {
            zsum += __expf(lm - zmax);
          }
          need = xs > pick_h<G>(mref, my_h) + kRefSlack;
        } else {
          uu = __int_as_float(0x7fffffff);  // NaN marks an empty block
        }
        p.u[row * G + my_h] = uu;
        p.xrec[row * XS + my_h] = xs;
        if (my_h == 0) p.xrec[row * XS + G] = __int_as_float(n);
      }
    }
    if (compensate) {
      if (__any_sync(0xffffffffu, need)) {  // rare: move this warp's reference up
        float sc_mine = 1.f;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float tm = warp_max((head_lane && my_h == h) ? xs : -CUDART_INF_F);
          const float nm = (tm > mref[h] + kRefSlack) ? tm : mref[h];
          const float sc = (mref[h] == -CUDART_INF_F) ? 0.f : __expf(mref[h] - nm);
          acc[h][0] *= sc; acc[h][1] *= sc; acc[h][2] *= sc; acc[h][3] *= sc;
          if (my_h == h) sc_mine = sc;
          mref[h] = nm;
        }
        lsum *= sc_mine;
      }
      if (head_lane) {
        const float w = (xs == -CUDART_INF_F) ? 0.f : __expf(xs - pick_h<G>(mref, my_h));
        wsw[my_bl * G + my_h] = w;
        lsum += w;
      }
      __syncwarp();
      // ---- (3) acc_h += w_{j,h} nu_j over this warp's blocks: 4 channels x G heads per lane
#pragma unroll
      for (int b0 = 0; b0 < kBlocksPerWarp; b0 += RS) {
        const int bl = b0 + rsub;
        const int jt = warp * kBlocksPerWarp + bl;
        if (jt < tn) {
          const float4 nv = reinterpret_cast<const float4*>(nu_t + jt * D)[c4];
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const float w = wsw[bl * G + h];
            const float2 w2 = make_float2(w, w);
            const float2 lo = __ffma2_rn(w2, make_float2(nv.x, nv.y), make_float2(acc[h][0], acc[h][1]));
            const float2 hi = __ffma2_rn(w2, make_float2(nv.z, nv.w), make_float2(acc[h][2], acc[h][3]));
            acc[h][0] = lo.x;
            acc[h][1] = lo.y;
            acc[h][2] = hi.x;
            acc[h][3] = hi.y;
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);  // this warp is done with the stage
  }
  if (!ok && warp == 0) {
    // a wait gave up (status recorded): wait, bounded, for the copies warp 0 issued
    for (int k = first_unwaited; k < issued; ++k) mbar_wait(&full[k % kStages], (k / kStages) & 1, nullptr);
  }
  __syncthreads();
  if (cur >= 0) finish_segment();
}

template <typename TQ, int D, int G>
const void* kptr(int r) {
  return r == 4 ? reinterpret_cast<const void*>(&score_stream_kernel<TQ, D, G, 4>)
                : reinterpret_cast<const void*>(&score_stream_kernel<TQ, D, G, 0>);
}

const void* pick(bool bf16, int D, int G, int r) {
#define COMPKV_PICK(T, DD)                  \
  switch (G) {                              \
    case 1: return kptr<T, DD, 1>(r);       \
    case 2: return kptr<T, DD, 2>(r);       \
    case 4: return kptr<T, DD, 4>(r);       \
    case 8: return kptr<T, DD, 8>(r);       \
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
  int dev = -1, r = 0;
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

int stream_ctas(int total_tiles, int sms, int ctas_per_sm) {
  int n = sms * (ctas_per_sm < 2 ? ctas_per_sm : 2);
  if (n > kStreamMaxCtas) n = kStreamMaxCtas;
  if (n > total_tiles) n = total_tiles;
  return n < 1 ? 1 : n;
}

}  // namespace

cudaError_t launch_score_stream(const StreamArgs& a, cudaStream_t st) {
  const void* kern = pick(a.bf16, a.D, a.G, a.r);
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
  p.xrec = a.xrec;
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
  const void* kern = pick(bf16, D, G, r);
  Grid g;
  if (!kern || grid_for(kern, D, G, r, &g) != cudaSuccess) return -1;
  return stream_ctas(total_tiles, g.sms, g.ctas_per_sm);
}

}  // namespace compkv
