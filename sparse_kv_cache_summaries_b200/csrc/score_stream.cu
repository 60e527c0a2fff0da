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
// equal contiguous ranges, one per CTA, two CTAs per SM (one, with a 6-stage ring, for 8 heads of
// d = 128), so every SM streams the same number of bytes whatever B and Hkv are. A CTA's range
// crosses at most a few (sequence, kv-head) pairs; it writes one partial record per pair it
// touches ("segment").
//
// Pipeline: a 3-stage (6-stage) shared-memory ring with a "full" and an "empty" mbarrier per stage. A
// producer warp fills the stages (bulk copies of the tile's mean keys and mean values, 4-byte
// cp.async of its grouped variances and counts) as soon as the 8 consumer warps have released
// them, so no consumer ever pays for issuing a copy. Each consumer warp owns 4 blocks of every
// tile and works through the ring on its own, with no CTA barrier in steady state. Lane l holds the same VW channels of
// every row for all G heads, so each mean key and mean value is read from shared memory once:
// partial dots of the 4 blocks with the G heads, one transpose-reduce over the warp that leaves
// each lane with one (block, head) dot for the scalar work, then each lane accumulates its
// channels of every head's weighted mean values. Compensation weights are taken against a
// per-warp reference logit per head that only moves up when a logit would exceed it by 64 (e^64
// keeps every sum finite in fp32). Warps meet only where a segment ends, to merge their partials
// in a fixed order (deterministic results), using the ring stage just released as scratch.
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
// Ring stages and CTAs per SM of a layout: two 9-warp CTAs per SM cap a thread at 96 registers,
// which G = 8 query heads of d = 128 exceed (their per-lane state spills); that layout runs one
// CTA per SM with a deeper ring instead, so the SM keeps as many bytes in flight.
__host__ __device__ constexpr bool stream_wide(int G, int D) { return G >= 8 && D >= 128; }
__host__ __device__ constexpr int stream_stages(int G, int D) { return stream_wide(G, D) ? 6 : 3; }
__host__ __device__ constexpr int stream_min_ctas(int G, int D) { return stream_wide(G, D) ? 1 : 2; }
constexpr int kBlocksPerWarp = kTile / kWarps;  // 4 (kWarps consumer warps)
constexpr int kStreamThreads = (kWarps + 1) * 32;  // the consumers and one producer warp
constexpr int kConsumerBar = 1;                    // named barrier of the consumer warps
constexpr float kRefSlack = 64.f;

struct StreamParams {
  int mode, Nb, tiles_per_pair, total_tiles, nctas, slots, r;
  float scale;
  const void* q;
  const void* mean_k;   // [pairs][Nb][D] of the summary type
  const float* var_g;
  const void* mean_v;
  const int32_t* count;
  float* u;        // [pairs][Nb][G]
  float* xrec;     // [pairs][Nb][xrec_stride(G)]  {x_0..x_{G-1}, n}
  float* zpart;    // [pairs][slots][G][2]
  float* comp;     // [pairs][slots][G][D+2]
  int32_t* status;
};

__host__ __device__ inline size_t a16(size_t x) { return (x + 15) & ~static_cast<size_t>(15); }

struct SLay {
  size_t stage_bytes, off_mu, off_nu, off_var, off_cnt, stage0, full, rel, wsw, q, qn, refw, red, logn, total;
  __host__ __device__ void build(int D, int G, int r, int ssz) {
    const int kStages = stream_stages(G, D);
    off_mu = 0;
    off_nu = a16(static_cast<size_t>(ssz) * kTile * D);
    off_var = a16(off_nu + static_cast<size_t>(ssz) * kTile * D);
    off_cnt = a16(off_var + sizeof(float) * kTile * r);
    stage_bytes = a16(off_cnt + sizeof(int) * kTile);
    // a released stage is the segment merge's scratch: [kWarps][G][D] floats
    const size_t scratch = sizeof(float) * kWarps * G * D;
    if (stage_bytes < scratch) stage_bytes = a16(scratch);
    size_t o = 0;
    full = o;   o = a16(o + 8 * 2 * kStages);                   // full[kStages], empty[kStages]
    rel = o;    o = a16(o + sizeof(uint32_t) * 4);              // abort flag
    wsw = o;    o = a16(o + sizeof(float) * kWarps * kBlocksPerWarp * G);   // per-warp weights
    stage0 = o; o = a16(o + stage_bytes * kStages);
    q = o;      o = a16(o + sizeof(float) * G * D);
    qn = o;     o = a16(o + sizeof(float) * G * r);
    refw = o;   o = a16(o + sizeof(float) * kWarps * G);
    red = o;    o = a16(o + sizeof(float) * 3 * G * 32);
    logn = o;   o = a16(o + sizeof(float) * 17);
    total = o;
  }
};

// R = 4 specialises the default group count (grouped variances as one float4); R = 0 is any r.
// One lane's VW channels of a summary row in shared memory, as VW / 2 float pairs.
template <int VW, typename S>
__device__ __forceinline__ void row_pairs(const S* row, float2 (&a)[VW / 2]) {
  if constexpr (sizeof(S) == 4) {
    if constexpr (VW == 4) {
      const float4 a4 = *reinterpret_cast<const float4*>(row);
      a[0] = make_float2(a4.x, a4.y);
      a[1] = make_float2(a4.z, a4.w);
    } else {
      a[0] = *reinterpret_cast<const float2*>(row);
    }
  } else {
    if constexpr (VW == 4) {
      const uint2 w = *reinterpret_cast<const uint2*>(row);
      a[0] = __half22float2(*reinterpret_cast<const __half2*>(&w.x));
      a[1] = __half22float2(*reinterpret_cast<const __half2*>(&w.y));
    } else {
      a[0] = __half22float2(*reinterpret_cast<const __half2*>(row));
    }
  }
}

// S: storage type of the mean key and mean value (float, or __half).
template <typename TQ, int D, int G, int R, typename S>
__global__ void __launch_bounds__(kStreamThreads, stream_min_ctas(G, D)) score_stream_kernel(const __grid_constant__ StreamParams p) {
  constexpr int kStages = stream_stages(G, D);
  extern __shared__ __align__(128) unsigned char sm[];
  SLay L;
  L.build(D, G, p.r, sizeof(S));
  const int r = p.r;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool compensate = p.mode != COMPKV_MODE_MASS;
  const int F = p.total_tiles, TP = p.tiles_per_pair;
  const int f0 = static_cast<int>((static_cast<long long>(blockIdx.x) * F) / p.nctas);
  const int f1 = static_cast<int>((static_cast<long long>(blockIdx.x + 1) * F) / p.nctas);
  const int nt = f1 - f0;
  constexpr int XS = xrec_stride(G);

  uint64_t* full = reinterpret_cast<uint64_t*>(sm + L.full);  // [kStages]: the tile has landed
  uint64_t* empty = full + kStages;                            // [kStages]: the 8 warps are done
  volatile uint32_t* abort_s = reinterpret_cast<uint32_t*>(sm + L.rel);  // a wait gave up
  float* q_s = reinterpret_cast<float*>(sm + L.q);
  float* qn_s = reinterpret_cast<float*>(sm + L.qn);
  float* refw_s = reinterpret_cast<float*>(sm + L.refw);
  float* red_s = reinterpret_cast<float*>(sm + L.red);
  float* logn_s = reinterpret_cast<float*>(sm + L.logn);
  const uint64_t policy = l2_evict_first_policy();

  // Refills the stage of local tile k (one whole warp).
  auto issue = [&](int k, int pr, int t) {  // tile k is tile t of pair pr
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
      const uint32_t bytes = static_cast<uint32_t>(tn) * D * sizeof(S);
      mbar_arrive_expect_tx(&full[st], compensate ? 2 * bytes : bytes);
      bulk_g2s_stream(sb + L.off_mu, static_cast<const S*>(p.mean_k) + row0 * D, bytes, &full[st], policy);
      if (compensate)
        bulk_g2s_stream(sb + L.off_nu, static_cast<const S*>(p.mean_v) + row0 * D, bytes, &full[st], policy);
    }
    cp_async_arrive(&full[st]);
  };

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 32 + 1);   // the producer's 32 lanes (cp.async) + the byte count
      mbar_init(&empty[s], kWarps);  // one arrival per consumer warp
    }
    *abort_s = 0;
    mbar_init_fence();
  }
  if (tid < 17) logn_s[tid] = tid > 0 ? logf(static_cast<float>(tid)) : -CUDART_INF_F;
  __syncthreads();
  // Launched with programmatic serialisation: everything above touches shared memory only, so it
  // overlaps the previous kernel's tail; every global read and write comes after this wait.
  pdl_wait();
  const int pr0 = f0 / TP, t0 = f0 % TP;
  pdl_launch_dependents();

  if (warp == kWarps) {
    // ---- producer: tile k goes into stage k % kStages once the consumer warps have released
    // tile k - kStages (the k / kStages - 1 th completion of that stage's empty barrier)
    int pr = pr0, tt = t0, issued = 0;
    for (int k = 0; k < nt; ++k) {
      const int st = k % kStages;
      if (k >= kStages) {
        bool got = mbar_wait(&empty[st], static_cast<uint32_t>((k / kStages - 1) & 1), p.status);
        got = __all_sync(0xffffffffu, got);
        if (!got && lane == 0) *abort_s = 1;
        if (!got || *abort_s != 0) break;
        // the consumers' generic-proxy reads (and merge scratch writes) of the stage come first
        fence_proxy_async();
      }
      issue(k, pr, tt);
      ++issued;
      if (++tt == TP) {
        tt = 0;
        ++pr;
      }
    }
    if (*abort_s != 0) {  // a wait gave up (status recorded): wait, bounded, for the copies in flight
      for (int k = max(0, issued - kStages); k < issued; ++k)
        mbar_wait(&full[k % kStages], static_cast<uint32_t>((k / kStages) & 1), nullptr);
    }
    __syncthreads();  // matched by the consumers' barrier after their loop: no copy is in flight
    return;
  }

  // Lane map: lane l holds channels [l VW, l VW + VW) of every row for all G heads (a warp-wide
  // row load is one contiguous 512 or 256 bytes: each mean key and mean value is read from
  // shared memory once). One transpose-reduce of the 4 blocks x G heads partial dots over the
  // 32 lanes leaves lane l with the full dot of one (block, head) pair: LPBK lanes per pair.
  constexpr int VW = D / 32;                // 4 (D = 128) or 2 (D = 64)
  constexpr int NVAL = kBlocksPerWarp * G;  // partial dots per lane
  constexpr int LPBK = 32 / NVAL;           // lanes per (block, head) after the reduce
  static_assert(VW == 2 || VW == 4, "head_dim must be 64 or 128");
  static_assert(NVAL <= 32, "at most 8 heads per kv-head");
  const int my_idx = lane / LPBK;           // value index b * G + h this lane ends with
  const int my_b = my_idx / G, my_h = my_idx % G;
  const bool rep = (lane % LPBK) == 0;      // one lane per (block, head) writes and is merged
  const int slot = warp * kBlocksPerWarp + my_b;  // 0..31 per head

  float2 qv[G][VW / 2];   // q_h at this lane's channels
  float2 acc[G][VW / 2];  // sum w nu at this lane's channels, per head
  float qnr[4];           // s^2 |q_{my_h, C_g}|^2 (R = 4)
  float mref[G];          // this warp's reference logit per head
  float zmax = -CUDART_INF_F, zsum = 0.f, lsum = 0.f;  // this lane's (block, head) partials
  int cur = -1;
  size_t seg_rec = 0;  // record index of the current segment
  float* wsw = reinterpret_cast<float*>(sm + L.wsw) + warp * NVAL;  // weights of the warp's pairs

  // the consumer warps' CTA barrier (the producer warp takes no part)
  auto consumer_sync = [&]() { named_bar_sync(kConsumerBar, kWarps * 32); };

  // Merges the 8 consumer warps' partials of the current segment (pair `cur`) in a fixed order,
  // with the stage `free_stage` (no copy in flight) as scratch for the warps' mean-value sums.
  auto finish_segment = [&](int free_stage) {
    // (1) each warp publishes its references, its slots' partials and its unscaled
    // compensation sums (the stage `free_stage` is the scratch: [kWarps][G][D])
    float* part = reinterpret_cast<float*>(sm + L.stage0 + L.stage_bytes * free_stage);
    if (lane == 0) {
#pragma unroll
      for (int h = 0; h < G; ++h) refw_s[warp * G + h] = mref[h];
    }
    if (rep) {
      red_s[(0 * G + my_h) * 32 + slot] = zmax;
      red_s[(1 * G + my_h) * 32 + slot] = zsum;
      red_s[(2 * G + my_h) * 32 + slot] = lsum;
    }
    if (compensate) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float* pw = part + (warp * G + h) * D + lane * VW;
        if constexpr (VW == 4) {
          reinterpret_cast<float4*>(pw)[0] = make_float4(acc[h][0].x, acc[h][0].y, acc[h][1].x, acc[h][1].y);
        } else {
          reinterpret_cast<float2*>(pw)[0] = acc[h][0];
        }
      }
    }
    consumer_sync();
    // (2) the per-head chains, spread over the warps (fixed order within each): chain c < G is
    // head c's log-partition partial (max, then the sum rescaled to it); chain G + c is head c's
    // compensation reference (the largest warp reference), the warps' rescale factors (written
    // over their references) and the weight sum. Slot l belongs to warp l / kBlocksPerWarp.
    for (int c = warp; c < 2 * G; c += kWarps) {
      if (c < G) {
        const float zm = red_s[(0 * G + c) * 32 + lane], zs = red_s[(1 * G + c) * 32 + lane];
        const float M1 = warp_max(zm);
        const float z = warp_sum(zm == -CUDART_INF_F ? 0.f : zs * __expf(zm - M1));
        if (lane == 0) {
          p.zpart[(seg_rec * G + c) * 2] = M1;
          p.zpart[(seg_rec * G + c) * 2 + 1] = z;
        }
      } else if (compensate) {
        const int h = c - G;
        const float rw = lane < kWarps ? refw_s[lane * G + h] : -CUDART_INF_F;
        const float Mh = warp_max(rw);
        const float f = (rw == -CUDART_INF_F) ? 0.f : __expf(rw - Mh);
        if (lane < kWarps) refw_s[lane * G + h] = f;
        const float fl = __shfl_sync(0xffffffffu, f, lane / kBlocksPerWarp);
        const float l = warp_sum(red_s[(2 * G + h) * 32 + lane] * fl);
        if (lane == 0) {
          p.comp[(seg_rec * G + h) * (D + 2)] = Mh;
          p.comp[(seg_rec * G + h) * (D + 2) + 1] = l;
        }
      }
    }
    if (compensate) {  // (3) the channels: sum over the warps of factor x partial
      consumer_sync();
      for (int i = tid; i < G * D; i += kThreads) {
        const int h = i / D;
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) v = fmaf(refw_s[w * G + h], part[w * G * D + i], v);
        p.comp[(seg_rec * G + h) * (D + 2) + 2 + (i % D)] = v;
      }
    }
    consumer_sync();  // the scratch stage and the slots are free again
  };

  // Loads the query heads of pair `pr` and resets the running state.
  auto start_segment = [&](int pr) {
    // this CTA's record of pair pr: slot (this CTA - the first CTA whose range reaches pr)
    seg_rec = static_cast<size_t>(pr) * p.slots + blockIdx.x -
              static_cast<int>(((static_cast<long long>(pr) * TP + 1) * p.nctas - 1) / F);
    const TQ* qp = static_cast<const TQ*>(p.q) + static_cast<size_t>(pr) * G * D;
    for (int i = tid; i < G * D; i += kThreads) q_s[i] = to_float(qp[i]);
    consumer_sync();
    const int gsz = D / r;
    for (int i = tid; i < G * r; i += kThreads) {
      const int hh = i / r, g = i % r;
      float s = 0.f;
      for (int cc = 0; cc < gsz; ++cc) {
        const float x = q_s[hh * D + g * gsz + cc];
        s = fmaf(x, x, s);
      }
      qn_s[i] = p.scale * p.scale * s;
    }
    consumer_sync();
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float* qh = q_s + h * D + lane * VW;
#pragma unroll
      for (int e = 0; e < VW / 2; ++e) {
        qv[h][e] = make_float2(qh[2 * e], qh[2 * e + 1]);
        acc[h][e] = make_float2(0.f, 0.f);
      }
      mref[h] = -CUDART_INF_F;
    }
    if constexpr (R == 4) {
#pragma unroll
      for (int g = 0; g < 4; ++g) qnr[g] = qn_s[my_h * 4 + g];
    }
    zmax = -CUDART_INF_F;
    zsum = lsum = 0.f;
    consumer_sync();
  };

  // `ok` goes false (for this warp) once a wait gives up; the warp then stops waiting and
  // computing but keeps the loop's structure, so every CTA barrier stays matched.
  bool ok = true;
  int pr = pr0, tt = t0;      // pair and tile-in-pair of tile k, kept without divisions
  int st = 0, ph = 0;         // ring stage and its phase parity for tile k
#pragma unroll 1
  for (int k = 0; k < nt; ++k) {
    if (pr != cur) {  // every consumer warp reaches this at the same tile
      consumer_sync();
      // the stage of tile k - 1 (not yet released) is the merge's scratch; released afterwards
      if (cur >= 0) finish_segment((k + kStages - 1) % kStages);
      start_segment(pr);
      cur = pr;
      if (k >= 1 && lane == 0) mbar_arrive(&empty[(k + kStages - 1) % kStages]);
    }
    bool got = ok && mbar_wait(&full[st], ph, p.status);
    got = __all_sync(0xffffffffu, got);
    if (!got && ok) {
      ok = false;
      if (lane == 0) *abort_s = 1;
    }
    const int jt0 = tt * kTile;
    const int tn = ok ? min(kTile, p.Nb - jt0) : 0;
    const unsigned char* sb = sm + L.stage0 + L.stage_bytes * st;
    const S* mu_t = reinterpret_cast<const S*>(sb + L.off_mu);
    const S* nu_t = reinterpret_cast<const S*>(sb + L.off_nu);
    const float* var_t = reinterpret_cast<const float*>(sb + L.off_var);
    const int* cnt_t = reinterpret_cast<const int*>(sb + L.off_cnt);
    const int jw = warp * kBlocksPerWarp;  // the warp's first block in the tile

    // ---- (1) partial dots over this lane's channels: 4 blocks x G heads
    float v[NVAL];
#pragma unroll
    for (int b = 0; b < kBlocksPerWarp; ++b) {
      float2 a[VW / 2];
      row_pairs<VW, S>(mu_t + (jw + b) * D + lane * VW, a);
#pragma unroll
      for (int hh = 0; hh < G; ++hh) {
        float2 s2 = __fmul2_rn(qv[hh][0], a[0]);
        if constexpr (VW == 4) s2 = __ffma2_rn(qv[hh][1], a[1], s2);
        v[b * G + hh] = s2.x + s2.y;
      }
    }
    TransposeReduce<NVAL, 16>::run(v, lane);  // lane now holds pair my_idx's dot in v[0]

    // ---- (2) scalars of (block my_b, head my_h)
    const int jm = jw + my_b;
    float xs = -CUDART_INF_F;
    float st_u = 0.f;  // stored after the stage is released (the release fence then has no
    int st_n = 0;      // global stores of this tile to wait for)
    if (jm < tn) {
      const int n = cnt_t[jm];
      float vh;
      if constexpr (R == 4) {
        const float4 vv = reinterpret_cast<const float4*>(var_t)[jm];
        vh = qnr[0] * vv.x;
        vh = fmaf(qnr[1], vv.y, vh);
        vh = fmaf(qnr[2], vv.z, vh);
        vh = fmaf(qnr[3], vv.w, vh);
      } else {
        vh = 0.f;
        for (int g = 0; g < r; ++g) vh = fmaf(qn_s[my_h * r + g], var_t[jm * r + g], vh);
      }
      float uu;
      if (n > 0) {
        xs = fmaf(p.scale, v[0], logn_s[min(n, 16)]);
        const float lm = xs + __logf(1.f + 0.5f * vh);
        uu = (p.mode == COMPKV_MODE_COMPKV) ? lm + __logf(0.5f * vh) : lm;
        if (lm > zmax) {
          zsum = zsum * __expf(zmax - lm) + 1.f;
          zmax = lm;
        } else {
          zsum += __expf(lm - zmax);
        }
      } else {
        uu = __int_as_float(0x7fffffff);  // NaN marks an empty block
      }
      st_u = uu;
      st_n = n;
    }

    // ---- (3) compensation weights and acc_h += w_{j,h} nu_j over the warp's 4 blocks
    if (compensate) {
      const float mme0 = mref[0];
      float mme = mme0;
#pragma unroll
      for (int hh = 1; hh < G; ++hh) mme = (my_h == hh) ? mref[hh] : mme;
      const bool need = xs > mme + kRefSlack;
      if (__any_sync(0xffffffffu, need)) {  // rare: move the warp's reference up
#pragma unroll
        for (int hh = 0; hh < G; ++hh) {
          const float tm = warp_max((need && my_h == hh) ? xs : -CUDART_INF_F);
          if (tm > mref[hh] + kRefSlack) {
            const float sc = (mref[hh] == -CUDART_INF_F) ? 0.f : __expf(mref[hh] - tm);
            const float2 sc2 = make_float2(sc, sc);
#pragma unroll
            for (int e = 0; e < VW / 2; ++e) acc[hh][e] = __fmul2_rn(acc[hh][e], sc2);
            if (my_h == hh) lsum *= sc;
            mref[hh] = tm;
          }
        }
        mme = mref[0];
#pragma unroll
        for (int hh = 1; hh < G; ++hh) mme = (my_h == hh) ? mref[hh] : mme;
      }
      const float w = (xs == -CUDART_INF_F) ? 0.f : __expf(xs - mme);
      lsum += w;
      if (rep) wsw[my_idx] = w;
      __syncwarp();
#pragma unroll
      for (int b = 0; b < kBlocksPerWarp; ++b) {
        if (jw + b < tn) {
          float2 a[VW / 2];
          row_pairs<VW, S>(nu_t + (jw + b) * D + lane * VW, a);
          float wb[G];
          if constexpr (G % 4 == 0) {
#pragma unroll
            for (int q4 = 0; q4 < G / 4; ++q4) {
              const float4 t = reinterpret_cast<const float4*>(wsw + b * G)[q4];
              wb[4 * q4] = t.x;
              wb[4 * q4 + 1] = t.y;
              wb[4 * q4 + 2] = t.z;
              wb[4 * q4 + 3] = t.w;
            }
          } else {
#pragma unroll
            for (int hh = 0; hh < G; ++hh) wb[hh] = wsw[b * G + hh];
          }
#pragma unroll
          for (int hh = 0; hh < G; ++hh) {
            const float2 w2 = make_float2(wb[hh], wb[hh]);
#pragma unroll
            for (int e = 0; e < VW / 2; ++e) acc[hh][e] = __ffma2_rn(w2, a[e], acc[hh][e]);
          }
        }
      }
    }

    // release the stage to the producer (unless tile k + 1 starts a new segment: the stage is
    // then the segment merge's scratch and is released after it)
    __syncwarp();
    if (lane == 0 && !(k + 1 < nt && tt + 1 == TP)) mbar_arrive(&empty[st]);
    if (rep && jm < tn) {
      const size_t row = static_cast<size_t>(pr) * p.Nb + jt0 + jm;
      p.u[row * G + my_h] = st_u;
      p.xrec[row * XS + my_h] = xs;
      if (my_h == 0) p.xrec[row * XS + G] = __int_as_float(st_n);
    }
    if (++tt == TP) {
      tt = 0;
      ++pr;
    }
    if (++st == kStages) {
      st = 0;
      ph ^= 1;
    }
  }
  __syncthreads();  // with the producer, which has drained any copy still in flight
  if (cur >= 0) finish_segment(0);
}

template <typename TQ, int D, int G, typename S>
const void* kptr(int r) {
  return r == 4 ? reinterpret_cast<const void*>(&score_stream_kernel<TQ, D, G, 4, S>)
                : reinterpret_cast<const void*>(&score_stream_kernel<TQ, D, G, 0, S>);
}

template <typename S>
const void* pick_s(bool bf16, int D, int G, int r) {
#define COMPKV_PICK(T, DD)                  \
  switch (G) {                              \
    case 1: return kptr<T, DD, 1, S>(r);    \
    case 2: return kptr<T, DD, 2, S>(r);    \
    case 4: return kptr<T, DD, 4, S>(r);    \
    case 8: return kptr<T, DD, 8, S>(r);    \
  }
  if (bf16) {
    if (D == 128) { COMPKV_PICK(uint16_t, 128) } else { COMPKV_PICK(uint16_t, 64) }
  } else {
    if (D == 128) { COMPKV_PICK(float, 128) } else { COMPKV_PICK(float, 64) }
  }
#undef COMPKV_PICK
  return nullptr;
}

const void* pick(bool bf16, int D, int G, int r, bool fp16) {
  return fp16 ? pick_s<__half>(bf16, D, G, r) : pick_s<float>(bf16, D, G, r);
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

cudaError_t grid_for(const void* kern, int D, int G, int r, bool fp16, Grid* out) {
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
  L.build(D, G, r, fp16 ? 2 : 4);
  g.smem = L.total;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(g.smem));
  if (e != cudaSuccess) return e;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&g.ctas_per_sm, kern, kStreamThreads, g.smem);
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
  const void* kern = pick(a.bf16, a.D, a.G, a.r, a.fp16_summ);
  if (!kern) return cudaErrorInvalidValue;
  Grid g;
  cudaError_t e = grid_for(kern, a.D, a.G, a.r, a.fp16_summ, &g);
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
  cfg.blockDim = dim3(kStreamThreads, 1, 1);
  cfg.dynamicSmemBytes = g.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  void* args[] = {&p};
  return cudaLaunchKernelExC(&cfg, kern, args);
}

int stream_grid_ctas(bool bf16, bool fp16_summ, int D, int G, int r, int total_tiles) {
  const void* kern = pick(bf16, D, G, r, fp16_summ);
  Grid g;
  if (!kern || grid_for(kern, D, G, r, fp16_summ, &g) != cudaSuccess) return -1;
  return stream_ctas(total_tiles, g.sms, g.ctas_per_sm);
}

}  // namespace compkv
