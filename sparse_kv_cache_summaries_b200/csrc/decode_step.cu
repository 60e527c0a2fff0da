// a1 + a2 + a3 in one clustered kernel: the whole CompKV decode step for every (sequence,
// kv-head) pair (CompKV review, Summary: blocks are scored from their summaries by the
// compensation-aware score, the top ones up to a token budget are attended exactly, and the
// omitted ones enter the same softmax through their block-mean logit; Section 3, Eq. 4-7: the
// residual of an omitted block is governed by its attention mass and within-block logit
// variance; abstract: exact attention over a selected subset, compensation of the omitted tail).
//
// One thread-block cluster of C CTAs per pair, one CTA per SM. Rank c owns the blocks
// [c chunk, c chunk + chunk) (chunk a multiple of the 32-block tile). The work of a rank:
//
//   phase A (all 16 worker warps): stream the rank's mean keys, grouped key variances and counts
//     through a ring of shared-memory stages filled by a producer warp with bulk copies; per
//     block and query head: lbar = s q_h . mu_j, V = s^2 sum_g |q_{h,C_g}|^2 var_{j,g},
//     x = lbar + log n_j, log m = x + log(1 + V/2), u = log m + log(V/2) (mass modes: u = log m);
//     u and x are kept per block, and the rank's log-sum-exp partial of m per head.
//   exchange: every rank pushes its partials of Zhat_h to every rank (st.async into the peers'
//     shared memory, counted on their mbarriers), so each rank knows log Zhat_h.
//   phase B (warps 0-7): the producer streams the rank's mean values right after the mean keys;
//     the Mean-compensation sum over all of the rank's blocks, sum_j e^{x_{j,h} - M_h} nu_j with
//     M_h the rank's largest x_h, accumulates here.
//   selection (warps 8-15, concurrently with phase B): S_j = sum_h e^{u_{j,h} - log Zhat_h} as
//     order-preserving keys; each rank's best 32 LS codes (key, then ~index: ties go to the lower
//     index) built with warp bitonic networks; every rank pushes its list to every rank; every
//     rank merges the C lists into the same global Top-K_b (exact: the global Top-K_b under this
//     strict order lies in the union of the ranks' best K_b). Budgets above 32 LS take several
//     rounds, each over the codes below the previous round's last one. The selection is marked
//     in a bitmap over the blocks, which gives it in ascending block order.
//   attention (warps 8-15): rank c attends the c-th contiguous slice of the ordered selection:
//     the blocks' K and V rows and mean values are staged into shared memory with bulk copies,
//     then exact logits, an online softmax per head, P.V, and removal of each attended block's
//     compensation term (taken against a reference at least its mean logit, so no weight
//     exceeds 1).
//   merge: the rank's attention partial and its compensation partial combine into one partial;
//     output channels are cut into C slices, every rank pushes its partial of each slice to the
//     rank that owns it, and each owner writes its slice of the outputs.
//
// Flags select parts: the score-and-select call runs phases A, B and the selection and leaves
// the records (x per block) and the ranks' compensation partials in the workspace; the
// sparse-decode call attends a given selection from those; the stream-only call runs phases A
// and B alone (for timing the bandwidth-bound part). Every wait is bounded; a wait that gives up
// records COMPKV_DEVERR_WAIT_TIMEOUT and the CTA skips the work but keeps every barrier.
#include <algorithm>
#include <mutex>

#include "attend.cuh"
#include "common.cuh"
#include "internal.h"
#include "topk_lists.cuh"

namespace compkv {
namespace {

constexpr int kTile = 32;                 // blocks per ring stage
constexpr int kWork = 16;                 // worker warps
constexpr int kHalf = 8;                  // stream warps (0..7) and select warps (8..15)
constexpr int kSelThreads = kHalf * 32;   // 256
constexpr int kNT = (kWork + 1) * 32;     // + the producer warp: 544 threads
constexpr int kBPW = kTile / kWork;       // blocks per worker warp in a phase-A tile: 2
constexpr int kBPS = kTile / kHalf;       // blocks per stream warp in a phase-B tile: 4
constexpr int kMaxC = 16;

// Named barriers (0 is __syncthreads).
constexpr int kBarWork = 1;    // the 16 worker warps
constexpr int kBarStream = 2;  // warps 0-7
constexpr int kBarSel = 3;     // warps 8-15
constexpr int kBarHand = 4;    // warps 0-15: the compensation partial is ready (0-7 arrive)
constexpr int kBarPair = 5;    // 5..11: pairwise list merges among the select warps

__host__ __device__ inline size_t al16(size_t x) { return (x + 15) & ~static_cast<size_t>(15); }

// Shared-memory layout of one plan (the same on host and device).
struct StepLay {
  int NS, KVB, LS, chunk, C, per, nbw;  // stages, K/V blocks per staging buffer, list slots,
                                        // blocks per rank, ranks, slots per rank, bitmap words
  int ux_smem;                          // u and x per block kept in shared memory (else global)
  size_t stage, s_var, s_cnt;           // ring stage bytes; offsets of var and count in a stage
  size_t kvblk, kv_v, kv_nu;            // staged block bytes; offsets of V rows and mean value
  size_t ring, bar, q, qn, red, zin, zr, u, x, keys, lin, wl, mg, bmp, bpre, slot, kv, wml, apart,
      cpl, racc, rml, fac, misc, logn, total;

  __host__ __device__ void build(int D, int G, int r, int ssz, int esz, int Kb, int Nb, int C_,
                                 int chunk_, int NS_, int KVB_, int ux) {
    NS = NS_;
    KVB = KVB_;
    C = C_;
    chunk = chunk_;
    ux_smem = ux;
    LS = Kb <= 32 ? 1 : (Kb <= 64 ? 2 : 4);
    per = (Kb + C - 1) / C;
    nbw = (Nb + 31) / 32;
    s_var = al16(static_cast<size_t>(kTile) * D * ssz);
    s_cnt = al16(s_var + sizeof(float) * kTile * r);
    stage = al16(s_cnt + sizeof(int) * kTile);
    kv_v = static_cast<size_t>(kBlockTokens) * D * esz;
    kv_nu = 2 * kv_v;
    kvblk = al16(kv_nu + static_cast<size_t>(D) * ssz);
    const int LW = 32 * LS;
    size_t o = 0;
    ring = o;  o = al16(o + stage * NS);
    {  // the ring is the stream warps' merge scratch after phase B: [kHalf][G][D] floats
      const size_t need = sizeof(float) * kHalf * G * D;
      if (o - ring < need) o = al16(ring + need);
    }
    bar = o;   o = al16(o + 8 * (2 * NS + 8));
    q = o;     o = al16(o + sizeof(float) * G * D);
    qn = o;    o = al16(o + sizeof(float) * G * r);
    red = o;   o = al16(o + sizeof(float) * 3 * kTile * G);
    zin = o;   o = al16(o + sizeof(float) * 2 * kMaxC * G);
    zr = o;    o = al16(o + sizeof(float) * 4 * G);
    u = o;     o = al16(o + (ux ? sizeof(float) * chunk * G : 0));
    x = o;     o = al16(o + (ux ? sizeof(float) * chunk * G : 0));
    keys = o;  o = al16(o + sizeof(uint32_t) * chunk);
    lin = o;   o = al16(o + sizeof(uint64_t) * 2 * C * LW);
    wl = o;    o = al16(o + sizeof(uint64_t) * kHalf * LW);
    mg = o;    o = al16(o + sizeof(uint64_t) * 2 * kHalf * LW);
    bmp = o;   o = al16(o + sizeof(uint32_t) * nbw);
    bpre = o;  o = al16(o + sizeof(int) * (kSelThreads + 1));
    slot = o;  o = al16(o + sizeof(int) * (per + 1));
    kv = o;    {
      size_t need = 2 * kvblk * KVB;
      const size_t scratch = sizeof(float) * kHalf * G * D;  // attention warps' partials
      if (need < scratch) need = scratch;
      o = al16(o + need);
    }
    wml = o;   o = al16(o + sizeof(float) * (3 * kHalf * G + 2 * G));
    apart = o; o = al16(o + sizeof(float) * G * (D + 2));
    cpl = o;   o = al16(o + sizeof(float) * G * (D + 2));
    const int E = G * D, per_o = (E + C - 1) / C;
    racc = o;  o = al16(o + sizeof(float) * C * per_o);
    rml = o;   o = al16(o + sizeof(float) * C * G * 2);
    fac = o;   o = al16(o + sizeof(float) * G * (kMaxC + 5));
    misc = o;  o = al16(o + sizeof(int) * 32);
    logn = o;  o = al16(o + sizeof(float) * (kBlockTokens + 1));
    total = o;
  }
};

struct StepParams {
  StepLay L;
  int mode, do_select, do_attend, do_stream;
  int Nb, Kb, T, r;
  float scale;
  const void* q;
  const void* K;
  const void* V;
  const void* mean_k;
  const float* var_g;
  const void* mean_v;
  const int32_t* count;
  float* ug;        // [pairs][Nb][G] log scores when they are not kept in shared memory
  float* xrec;      // [pairs][Nb][G] x = lbar + log n per block and head
  float* cpart;     // [pairs][kMaxC][G][D + 2] the ranks' compensation partials
  int32_t* sel_idx; // [pairs][Kb]
  float* scores;    // [pairs][Nb] or null
  float* out;       // [pairs][G][D]
  int32_t* status;
};

// mbarrier arrive counting `n` arrivals at once.
__device__ __forceinline__ void mbar_arrive_n(uint64_t* bar, uint32_t n) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(n) : "memory");
}

// CTA barrier over the `n` threads of named barrier `id` that also returns the AND of `pred`
// over them (so a decision taken after a bounded wait is the same in every participating warp).
__device__ __forceinline__ bool named_bar_and(int id, int n, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, %2, %3, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

// Orders this thread's earlier shared-memory writes before later accesses by other CTAs of the
// cluster that synchronise with it.
__device__ __forceinline__ void fence_cluster() { asm volatile("fence.acq_rel.cluster;" ::: "memory"); }

// The 8 select warps' descending lists merged pairwise in 3 levels through `lists` ([kHalf][L])
// and named barriers kBarPair.. shared by the two warps of a pair; select warp 0 ends with the
// CTA's best L.
template <int E>
__device__ __forceinline__ void sel_pairs_merge(uint64_t (&best)[E], uint64_t* lists, int sw) {
  const int lane = threadIdx.x & 31;
  constexpr int L = 32 * E;
  int id = kBarPair;
#pragma unroll
  for (int s = 1; s < kHalf; s <<= 1) {
    if ((sw & (2 * s - 1)) == s) {
#pragma unroll
      for (int e = 0; e < E; ++e) lists[sw * L + e * 32 + lane] = best[e];
      named_bar_arrive(id + (sw - s) / (2 * s), 64);
    } else if ((sw & (2 * s - 1)) == 0) {
      named_bar_sync(id + sw / (2 * s), 64);
      uint64_t b[E];
#pragma unroll
      for (int e = 0; e < E; ++e) b[e] = lists[(sw + s) * L + e * 32 + lane];
      list_merge_top<E>(best, b);
    }
    id += kHalf / (2 * s);
  }
}

// One lane's VW channels of a summary row in shared memory, as VW / 2 float pairs.
template <int VW, typename S>
__device__ __forceinline__ void srow_pairs(const S* row, float2 (&a)[VW / 2]) {
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

// One lane's VEP channels of a K or V row in shared memory (bf16 or fp32), as floats.
template <typename T, int VEP>
__device__ __forceinline__ void kvrow(const T* row, int lane, float (&f)[VEP]) {
  if constexpr (sizeof(T) == 2) {
    if constexpr (VEP == 4) {
      const uint2 w = reinterpret_cast<const uint2*>(row)[lane];
      f[0] = __uint_as_float(w.x << 16);
      f[1] = __uint_as_float(w.x & 0xffff0000u);
      f[2] = __uint_as_float(w.y << 16);
      f[3] = __uint_as_float(w.y & 0xffff0000u);
    } else {
      const uint32_t w = reinterpret_cast<const uint32_t*>(row)[lane];
      f[0] = __uint_as_float(w << 16);
      f[1] = __uint_as_float(w & 0xffff0000u);
    }
  } else {
    if constexpr (VEP == 4) {
      const float4 w = reinterpret_cast<const float4*>(row)[lane];
      f[0] = w.x;
      f[1] = w.y;
      f[2] = w.z;
      f[3] = w.w;
    } else {
      const float2 w = reinterpret_cast<const float2*>(row)[lane];
      f[0] = w.x;
      f[1] = w.y;
    }
  }
}

template <int G>
__device__ __forceinline__ float pick_h(const float (&a)[G], int h) {
  float v = a[0];
#pragma unroll
  for (int i = 1; i < G; ++i) v = (h == i) ? a[i] : v;
  return v;
}

// TQ: element type of q, K and V (uint16_t = bf16, or float); S: summary storage (float,
// __half); LS: list slots.
template <typename TQ, int D, int G, typename S, int LS>
__global__ void __launch_bounds__(kNT, 1) decode_step_kernel(const __grid_constant__ StepParams p) {
  extern __shared__ __align__(128) unsigned char sm[];
  const StepLay& L = p.L;
  const int C = static_cast<int>(cluster_size());
  const int rank = static_cast<int>(cluster_rank());
  const int pr = blockIdx.x / C;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int r = p.r;
  const int Nb = p.Nb, Kb = p.Kb;
  const bool compensate = p.mode != COMPKV_MODE_MASS;
  const bool stream = p.do_stream != 0;
  const int chunk = L.chunk;
  const int j0 = rank * chunk;
  const int nloc = max(0, min(chunk, Nb - j0));
  const int ntA = stream ? (nloc + kTile - 1) / kTile : 0;
  const int ntB = (stream && compensate) ? ntA : 0;
  constexpr int LW = 32 * LS;
  constexpr int E = G * D;
  const int per_o = (E + C - 1) / C;
  const int oe0 = min(E, rank * per_o), oe1 = min(E, oe0 + per_o);

  uint64_t* full = reinterpret_cast<uint64_t*>(sm + L.bar);
  uint64_t* empty = full + L.NS;
  uint64_t* zbar = empty + L.NS;     // [1] the C ranks' Zhat partials
  uint64_t* lbar = zbar + 1;         // [2] the C ranks' candidate lists, by round parity
  uint64_t* kvbar = lbar + 2;        // [2] staged K/V of the attended blocks, by buffer
  uint64_t* obar = kvbar + 2;        // [1] the C ranks' partials of this rank's output slice
  int* misc = reinterpret_cast<int*>(sm + L.misc);  // [0] abort flag of the producer
  float* q_s = reinterpret_cast<float*>(sm + L.q);
  float* qn_s = reinterpret_cast<float*>(sm + L.qn);
  float* zin = reinterpret_cast<float*>(sm + L.zin);  // [C][G][2]
  float* zr = reinterpret_cast<float*>(sm + L.zr);    // [G][2] the rank's Zhat partial, [2G..3G) M_h
  float* cpl = reinterpret_cast<float*>(sm + L.cpl);  // [G][D+2] the rank's compensation partial
  float* logn_s = reinterpret_cast<float*>(sm + L.logn);  // log n for n = 0..16
  // u and x of the rank's blocks: shared memory, or the workspace rows of this rank
  float* ub = L.ux_smem ? reinterpret_cast<float*>(sm + L.u)
                        : p.ug + (static_cast<size_t>(pr) * Nb + j0) * G;
  float* xb = L.ux_smem ? reinterpret_cast<float*>(sm + L.x)
                        : p.xrec + (static_cast<size_t>(pr) * Nb + j0) * G;
  const bool x_to_global = L.ux_smem && p.do_select && !p.do_attend;  // records for sparse_decode

  // ---------------------------------------------------------------- prologue
  if (tid == 0) {
    for (int s = 0; s < L.NS; ++s) {
      mbar_init(&full[s], 32 + 1);   // the producer's 32 lanes (cp.async) + the byte count
      mbar_init(&empty[s], kWork);   // one arrival per worker warp (stream warps arrive twice)
    }
    mbar_init(zbar, 1);
    mbar_init(&lbar[0], 1);
    mbar_init(&lbar[1], 1);
    mbar_init(&kvbar[0], 1);
    mbar_init(&kvbar[1], 1);
    mbar_init(obar, 1);
    misc[0] = 0;
    mbar_init_fence();
    if (p.do_select && stream) {
      mbar_arrive_expect_tx(zbar, static_cast<uint32_t>(C * G * 8));
      if (Kb > 0 && Kb < Nb) {
        mbar_arrive_expect_tx(&lbar[0], static_cast<uint32_t>(C * LW * 8));
        mbar_arrive_expect_tx(&lbar[1], static_cast<uint32_t>(C * LW * 8));
      }
    }
    if (p.do_attend && oe0 < oe1) {
      const int nh = (oe1 - 1) / D - oe0 / D + 1;
      mbar_arrive_expect_tx(obar, static_cast<uint32_t>(C * ((oe1 - oe0) * 4 + nh * 8)));
    }
  }
  if (tid <= kBlockTokens) logn_s[tid] = tid > 0 ? logf(static_cast<float>(tid)) : -CUDART_INF_F;
  __syncthreads();
  cluster_arrive_relaxed();  // matched by cluster_wait() before this CTA first writes a peer
  pdl_wait();                // the previous grid's writes are visible from here on

  // ---------------------------------------------------------------- producer warp
  if (warp == kWork) {
    const uint64_t policy = l2_evict_first_policy();
    const int total = ntA + ntB;
    int issued = 0;
    for (int k = 0; k < total; ++k) {
      const int st = k % L.NS;
      if (k >= L.NS) {
        bool got = mbar_wait(&empty[st], static_cast<uint32_t>((k / L.NS - 1) & 1), p.status);
        got = __all_sync(0xffffffffu, got);
        if (!got && lane == 0) misc[0] = 1;
        __syncwarp();
        if (!got || *reinterpret_cast<volatile int*>(&misc[0]) != 0) break;
        fence_proxy_async();  // the consumers' generic reads (and scratch writes) come first
      }
      const bool phaseA = k < ntA;
      const int t = phaseA ? k : k - ntA;
      const int jt0 = j0 + t * kTile;
      const int tn = min(kTile, j0 + nloc - jt0);
      const size_t row0 = static_cast<size_t>(pr) * Nb + jt0;
      unsigned char* sb = sm + L.ring + L.stage * st;
      if (phaseA) {
        float* var_d = reinterpret_cast<float*>(sb + L.s_var);
        int* cnt_d = reinterpret_cast<int*>(sb + L.s_cnt);
        for (int i = lane; i < tn * r; i += 32) cp_async4(var_d + i, p.var_g + row0 * r + i);
        for (int i = lane; i < tn; i += 32) cp_async4(cnt_d + i, p.count + row0 + i);
      }
      if (lane == 0) {
        const uint32_t bytes = static_cast<uint32_t>(tn) * D * sizeof(S);
        mbar_arrive_expect_tx(&full[st], bytes);
        const void* src = phaseA ? p.mean_k : p.mean_v;
        bulk_g2s_stream(sb, static_cast<const S*>(src) + row0 * D, bytes, &full[st], policy);
      }
      cp_async_arrive(&full[st]);
      ++issued;
    }
    if (misc[0] != 0) {  // gave up: wait (bounded) for the copies still in flight
      for (int k = max(0, issued - L.NS); k < issued; ++k)
        mbar_wait(&full[k % L.NS], static_cast<uint32_t>((k / L.NS) & 1), nullptr);
    }
    pdl_launch_dependents();
    cluster_wait();
    cluster_arrive();
    cluster_wait();
    return;
  }

  // ---------------------------------------------------------------- workers: q and phase A
  constexpr int VW = D / 32;
  static_assert(VW == 2 || VW == 4, "head_dim must be 64 or 128");
  {
    const TQ* qp = static_cast<const TQ*>(p.q) + static_cast<size_t>(pr) * G * D;
    for (int i = tid; i < G * D; i += kWork * 32) q_s[i] = to_float(qp[i]);
    named_bar_sync(kBarWork, kWork * 32);
  }
  if (stream) {
    const int gsz = D / r;
    for (int i = tid; i < G * r; i += kWork * 32) {
      const int hh = i / r, g = i % r;
      float s = 0.f;
      for (int cc = 0; cc < gsz; ++cc) {
        const float v = q_s[hh * D + g * gsz + cc];
        s = fmaf(v, v, s);
      }
      qn_s[i] = p.scale * p.scale * s;
    }
    named_bar_sync(kBarWork, kWork * 32);
  }

  constexpr int NVAL = kBPW * G;       // partial dots per lane in phase A
  constexpr int LPBK = 32 / NVAL;      // lanes per (block, head) after the transpose-reduce
  static_assert(NVAL <= 32, "at most 8 heads per kv-head");
  const int my_idx = lane / LPBK;
  const int my_b = my_idx / G, my_h = my_idx % G;
  const bool rep = (lane % LPBK) == 0;
  float zmax = -CUDART_INF_F, zsum = 0.f, xmx = -CUDART_INF_F;
  bool ok = true;  // this warp's waits have all succeeded
  if (stream) {
    float2 qv[G][VW / 2];
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int e = 0; e < VW / 2; ++e)
        qv[h][e] = make_float2(q_s[h * D + lane * VW + 2 * e], q_s[h * D + lane * VW + 2 * e + 1]);
    float qnr[4] = {0.f, 0.f, 0.f, 0.f};  // the default r = 4 takes the variances as one float4
    if (r == 4) {
#pragma unroll
      for (int g = 0; g < 4; ++g) qnr[g] = qn_s[my_h * 4 + g];
    }
    int st = 0, ph = 0;
#pragma unroll 1
    for (int k = 0; k < ntA; ++k) {
      bool got = ok && mbar_wait(&full[st], ph, p.status);
      got = __all_sync(0xffffffffu, got);
      ok = got;
      const int tn = ok ? min(kTile, nloc - k * kTile) : 0;
      const unsigned char* sb = sm + L.ring + L.stage * st;
      const S* mu_t = reinterpret_cast<const S*>(sb);
      const float* var_t = reinterpret_cast<const float*>(sb + L.s_var);
      const int* cnt_t = reinterpret_cast<const int*>(sb + L.s_cnt);
      const int jw = warp * kBPW;
      float v[NVAL];
#pragma unroll
      for (int b = 0; b < kBPW; ++b) {
        float2 a[VW / 2];
        srow_pairs<VW, S>(mu_t + (jw + b) * D + lane * VW, a);
#pragma unroll
        for (int hh = 0; hh < G; ++hh) {
          float2 s2 = __fmul2_rn(qv[hh][0], a[0]);
          if constexpr (VW == 4) s2 = __ffma2_rn(qv[hh][1], a[1], s2);
          v[b * G + hh] = s2.x + s2.y;
        }
      }
      TransposeReduce<NVAL, 16>::run(v, lane);
      const int jm = jw + my_b;
      float uu = 0.f, xs = -CUDART_INF_F;
      if (jm < tn) {
        const int n = cnt_t[jm];
        float vh;
        if (r == 4) {
          const float4 vv = reinterpret_cast<const float4*>(var_t)[jm];
          vh = qnr[0] * vv.x;
          vh = fmaf(qnr[1], vv.y, vh);
          vh = fmaf(qnr[2], vv.z, vh);
          vh = fmaf(qnr[3], vv.w, vh);
        } else {
          vh = 0.f;
          for (int g = 0; g < r; ++g) vh = fmaf(qn_s[my_h * r + g], var_t[jm * r + g], vh);
        }
        if (n > 0) {
          xs = fmaf(p.scale, v[0], logn_s[min(n, kBlockTokens)]);
          const float lm = xs + __logf(1.f + 0.5f * vh);
          uu = (p.mode == COMPKV_MODE_COMPKV) ? lm + __logf(0.5f * vh) : lm;
          if (lm > zmax) {
            zsum = zsum * __expf(zmax - lm) + 1.f;
            zmax = lm;
          } else {
            zsum += __expf(lm - zmax);
          }
          xmx = fmaxf(xmx, xs);
        } else {
          uu = __int_as_float(0x7fffffff);  // NaN marks an empty block
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
      if (rep && jm < tn) {
        const int jl = k * kTile + jm;
        ub[jl * G + my_h] = uu;
        xb[jl * G + my_h] = xs;
        if (x_to_global) p.xrec[(static_cast<size_t>(pr) * Nb + j0 + jl) * G + my_h] = xs;
      }
      if (++st == L.NS) {
        st = 0;
        ph ^= 1;
      }
    }
  }

  // ---------------------------------------------------------------- rank partials, exchange
  float* red = reinterpret_cast<float*>(sm + L.red);  // [32 entries][G][3]
  const bool exchange = stream && p.do_select;
  if (stream) {
    fence_cluster();  // x of this rank's blocks is read by the other ranks during attention
    if (rep) {
      float* e = red + ((warp * kBPW + my_b) * G + my_h) * 3;
      e[0] = zmax;
      e[1] = zsum;
      e[2] = xmx;
    }
    named_bar_sync(kBarWork, kWork * 32);
    if (warp < G) {  // warp h: head h over the 32 (warp, block) entries
      const int h = warp;
      const float* e = red + (lane * G + h) * 3;
      float m = e[0], s = e[1], xm = e[2];
      if (m == -CUDART_INF_F) s = 0.f;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
        const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
        lse_merge(m, s, m2, s2);
        xm = fmaxf(xm, __shfl_xor_sync(0xffffffffu, xm, o));
      }
      if (lane == 0) {
        zr[2 * h] = m;
        zr[2 * h + 1] = s;
        zr[2 * G + h] = xm;  // M_h: the rank's reference logit of phase B
      }
    }
    named_bar_sync(kBarWork, kWork * 32);
  }
  cluster_wait();  // every CTA of the cluster has started: peers' shared memory may be written
  if (exchange && warp == 0) {
    for (int i = lane; i < C * G; i += 32) {
      const int c = i / G, h = i % G;
      const uint64_t v = (static_cast<uint64_t>(__float_as_uint(zr[2 * h + 1])) << 32) |
                         __float_as_uint(zr[2 * h]);
      st_async_b64(cluster_smem_addr(zin + (rank * G + h) * 2, c), v, cluster_smem_addr(zbar, c));
    }
  }

  // ---------------------------------------------------------------- stream warps: phase B
  if (warp < kHalf) {
    if (ntB > 0) {
      float Mref[G];
#pragma unroll
      for (int h = 0; h < G; ++h) Mref[h] = zr[2 * G + h];
      float2 acc[G][VW / 2];
#pragma unroll
      for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < VW / 2; ++e) acc[h][e] = make_float2(0.f, 0.f);
      float lsum = 0.f;  // lane l < kBPS G: weight sum of (block l / G, head l % G)
      float* wsw = red + warp * kBPS * G;  // the red scratch is free again: weights per warp
      const int wl_b = lane / G, wl_h = lane % G;
      const float mref_l = pick_h<G>(Mref, wl_h);
      int st = ntA % L.NS, ph = (ntA / L.NS) & 1;
#pragma unroll 1
      for (int kb = 0; kb < ntB; ++kb) {
        bool got = ok && mbar_wait(&full[st], ph, p.status);
        got = __all_sync(0xffffffffu, got);
        ok = got;
        const int tn = ok ? min(kTile, nloc - kb * kTile) : 0;
        const S* nu_t = reinterpret_cast<const S*>(sm + L.ring + L.stage * st);
        const int jw = warp * kBPS;
        if (lane < kBPS * G) {
          const int jl = kb * kTile + jw + wl_b;
          const float w = (jw + wl_b < tn) ? exp_diff(xb[jl * G + wl_h], mref_l) : 0.f;
          lsum += w;
          wsw[lane] = w;
        }
        __syncwarp();
#pragma unroll
        for (int b = 0; b < kBPS; ++b) {
          if (jw + b < tn) {
            float2 a[VW / 2];
            srow_pairs<VW, S>(nu_t + (jw + b) * D + lane * VW, a);
#pragma unroll
            for (int hh = 0; hh < G; ++hh) {
              const float w = wsw[b * G + hh];
              const float2 w2 = make_float2(w, w);
#pragma unroll
              for (int e = 0; e < VW / 2; ++e) acc[hh][e] = __ffma2_rn(w2, a[e], acc[hh][e]);
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_n(&empty[st], 2);
        if (++st == L.NS) {
          st = 0;
          ph ^= 1;
        }
      }
      // the rank's compensation partial: the 8 warps' sums (same reference) in a fixed order
      if (lane < kBPS * G) wsw[lane] = lsum;
      named_bar_sync(kBarStream, kSelThreads);  // every stream warp is done with the ring
      float* part = reinterpret_cast<float*>(sm + L.ring);  // [kHalf][G][D]
#pragma unroll
      for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < VW / 2; ++e)
          *reinterpret_cast<float2*>(part + (warp * G + h) * D + lane * VW + 2 * e) = acc[h][e];
      named_bar_sync(kBarStream, kSelThreads);  // the weight sums in red are complete too
      float* cg = (p.do_select && !p.do_attend)
                      ? p.cpart + (static_cast<size_t>(pr) * kMaxC + rank) * G * (D + 2)
                      : nullptr;
      for (int i = tid; i < E; i += kSelThreads) {
        const int h = i / D, c = i % D;
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < kHalf; ++w) s += part[(w * G + h) * D + c];
        cpl[h * (D + 2) + 2 + c] = s;
        if (cg) cg[h * (D + 2) + 2 + c] = s;
      }
      if (tid < G) {
        const int h = tid;
        float s = 0.f;
        for (int w = 0; w < kHalf; ++w)
          for (int b = 0; b < kBPS; ++b) s += red[w * kBPS * G + b * G + h];
        cpl[h * (D + 2)] = Mref[h];
        cpl[h * (D + 2) + 1] = s;
        if (cg) {
          cg[h * (D + 2)] = Mref[h];
          cg[h * (D + 2) + 1] = s;
        }
      }
    }
    named_bar_arrive(kBarHand, kWork * 32);  // the compensation partial is in cpl
    pdl_launch_dependents();
    cluster_arrive();
    cluster_wait();
    return;
  }

  // ---------------------------------------------------------------- select warps
  const int sw = warp - kHalf, stid = tid - kHalf * 32;
  int* slot_s = reinterpret_cast<int*>(sm + L.slot);
  uint32_t* bmp = reinterpret_cast<uint32_t*>(sm + L.bmp);
  int* bpre = reinterpret_cast<int*>(sm + L.bpre);
  const int per = L.per;
  const int s0 = min(Kb, rank * per), s1 = min(Kb, s0 + per);
  int nsl = 0;  // this rank's attended blocks

  if (p.do_select) {
    uint32_t* keys = reinterpret_cast<uint32_t*>(sm + L.keys);
    for (int i = stid; i < L.nbw; i += kSelThreads) bmp[i] = 0u;
    // log Zhat_h from the C ranks' partials (every select warp computes it)
    float lz[G];
    const bool zok = __all_sync(0xffffffffu, mbar_wait_cluster(zbar, 0, p.status));
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float m = -CUDART_INF_F, s = 0.f;
      if (zok && lane < C) {
        m = zin[(lane * G + h) * 2];
        s = zin[(lane * G + h) * 2 + 1];
        if (m == -CUDART_INF_F) s = 0.f;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
        const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
        lse_merge(m, s, m2, s2);
      }
      lz[h] = (m == -CUDART_INF_F) ? -CUDART_INF_F : m + logf(s);
    }
    // keys of this rank's blocks: S_j = sum_h exp(u - log Zhat_h); empty blocks key 0
    const int span = ((nloc + kHalf * 32 - 1) / (kHalf * 32)) * 32;
    const int jb = sw * span;
    for (int j = jb + lane; j < min(nloc, jb + span); j += 32) {
      float Sj = 0.f;
#pragma unroll
      for (int h = 0; h < G; ++h) Sj += __expf(ub[j * G + h] - lz[h]);
      const bool emp = Sj != Sj;
      keys[j] = emp ? 0u : score_key(Sj);
      if (p.scores) p.scores[static_cast<size_t>(pr) * Nb + j0 + j] = emp ? 0.f : Sj;
    }
    named_bar_sync(kBarSel, kSelThreads);  // keys and the cleared bitmap are visible

    if (Kb >= Nb) {  // every block is selected
      for (int i = stid; i < L.nbw; i += kSelThreads) {
        const int rem = Nb - i * 32;
        bmp[i] = rem >= 32 ? 0xffffffffu : ((1u << rem) - 1u);
      }
    } else if (Kb > 0) {
      uint64_t* lin = reinterpret_cast<uint64_t*>(sm + L.lin);  // [2][C][LW]
      uint64_t* wlists = reinterpret_cast<uint64_t*>(sm + L.wl);
      uint64_t* mg = reinterpret_cast<uint64_t*>(sm + L.mg);     // [2][kHalf][LW]
      uint64_t thr = ~0ull;  // this round takes codes below thr
      int remaining = Kb;
      for (int rnd = 0; remaining > 0; ++rnd) {
        const int b2 = rnd & 1;
        // this warp's best LW codes below thr, then the rank's through the pair merges
        uint64_t best[LS];
#pragma unroll
        for (int e = 0; e < LS; ++e) best[e] = 0ull;
        for (int c0 = 0; c0 * 32 < span; c0 += LS) {
          uint64_t v[LS];
#pragma unroll
          for (int e = 0; e < LS; ++e) {
            const int j = jb + (c0 + e) * 32 + lane;
            v[e] = 0ull;
            if ((c0 + e) * 32 < span && j < nloc) {
              const uint64_t code = topk_code(keys[j], j0 + j);
              v[e] = code < thr ? code : 0ull;
            }
          }
          list_sort_desc<LS>(v);
          if (c0 == 0) {
#pragma unroll
            for (int e = 0; e < LS; ++e) best[e] = v[e];
          } else {
            list_merge_top<LS>(best, v);
          }
        }
        sel_pairs_merge<LS>(best, wlists, sw);
        if (sw == 0) {  // push the rank's list into every rank
#pragma unroll 1
          for (int c = 0; c < C; ++c) {
#pragma unroll
            for (int e = 0; e < LS; ++e)
              st_async_b64(cluster_smem_addr(lin + (static_cast<size_t>(b2) * C + rank) * LW + e * 32 + lane, c),
                           best[e], cluster_smem_addr(&lbar[b2], c));
          }
          if (rnd == 0 && p.do_attend) {
            // speculative: this rank's likeliest picks start moving from HBM to L2 while the
            // lists cross the cluster (about 2 K_b / C of them)
            const int m = min(32, max(1, (2 * Kb + C - 1) / C));
            const uint64_t code = best[0];
            if (lane < m && code != 0ull) {
              const int j = topk_index(code);
              const size_t off = (static_cast<size_t>(pr) * p.T + static_cast<size_t>(j) * kBlockTokens) * D;
              const size_t bytes = static_cast<size_t>(min(kBlockTokens, p.T - j * kBlockTokens)) * D * sizeof(TQ);
              prefetch_l2_range(static_cast<const TQ*>(p.K) + off, bytes);
              prefetch_l2_range(static_cast<const TQ*>(p.V) + off, bytes);
            }
          }
        }
        // the C lists of this round: every rank merges them into the same global list
        const bool lok = named_bar_and(kBarSel, kSelThreads, mbar_wait_cluster(&lbar[b2], (rnd >> 1) & 1, p.status));
        const uint64_t* src = lin + static_cast<size_t>(b2) * C * LW;
        int nl = C;
        int lev = 0;
        while (nl > 1) {
          const int pairs_n = nl / 2;
          uint64_t* dst = mg + static_cast<size_t>(lev & 1) * kHalf * LW;
          for (int w = sw; w < (nl + 1) / 2; w += kHalf) {
            uint64_t a[LS], b[LS];
#pragma unroll
            for (int e = 0; e < LS; ++e) {
              a[e] = lok ? src[(2 * w) * LW + e * 32 + lane] : 0ull;
              b[e] = (lok && w < pairs_n) ? src[(2 * w + 1) * LW + e * 32 + lane] : 0ull;
            }
            if (w < pairs_n) list_merge_top<LS>(a, b);
#pragma unroll
            for (int e = 0; e < LS; ++e) dst[w * LW + e * 32 + lane] = a[e];
          }
          named_bar_sync(kBarSel, kSelThreads);
          src = dst;
          nl = (nl + 1) / 2;
          ++lev;
        }
        // src[0 .. LW) is the round's global list: mark the first `take` codes
        const int take = min(LW, remaining);
        uint64_t lastc = 0ull;
        if (sw == 0) {
#pragma unroll
          for (int e = 0; e < LS; ++e) {
            const int i = e * 32 + lane;
            const uint64_t code = lok ? src[i] : 0ull;
            if (i < take && code != 0ull) {
              const int j = topk_index(code);
              atomicOr(&bmp[j >> 5], 1u << (j & 31));
            }
          }
        }
        lastc = lok ? src[take - 1] : 0ull;
        named_bar_sync(kBarSel, kSelThreads);  // every warp has read src; the bitmap is marked
        if (tid == kHalf * 32 && remaining - take > 0) {  // re-arm this parity for round rnd + 2
          mbar_arrive_expect_tx(&lbar[b2], static_cast<uint32_t>(C * LW * 8));
        }
        remaining -= take;
        thr = lastc;
        if (!lok || lastc == 0ull) break;
      }
    }
    named_bar_sync(kBarSel, kSelThreads);
    // ascending order: prefix of the bitmap's popcounts over the select threads
    {
      const int wpt = (L.nbw + kSelThreads - 1) / kSelThreads;
      const int w0 = min(L.nbw, stid * wpt), w1 = min(L.nbw, w0 + wpt);
      int cnt = 0;
      for (int w = w0; w < w1; ++w) cnt += __popc(bmp[w]);
      // exclusive scan over the 256 select threads
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      if (lane == 31) bpre[sw] = incl;
      named_bar_sync(kBarSel, kSelThreads);
      int base = 0;
#pragma unroll
      for (int w = 0; w < kHalf; ++w) base += (w < sw) ? bpre[w] : 0;
      int pos = base + incl - cnt;
      int32_t* sel_out = (p.sel_idx && rank == 0) ? p.sel_idx + static_cast<size_t>(pr) * Kb : nullptr;
      for (int w = w0; w < w1; ++w) {
        uint32_t bits = bmp[w];
        while (bits) {
          const int b = __ffs(bits) - 1;
          bits &= bits - 1;
          const int j = w * 32 + b;
          if (pos < Kb) {
            if (sel_out) sel_out[pos] = j;
            if (pos >= s0 && pos < s1) slot_s[pos - s0] = j;
          }
          ++pos;
        }
      }
    }
    nsl = s1 - s0;
    named_bar_sync(kBarSel, kSelThreads);
  } else if (p.do_attend) {
    for (int i = stid; i < s1 - s0; i += kSelThreads) slot_s[i] = p.sel_idx[static_cast<size_t>(pr) * Kb + s0 + i];
    nsl = s1 - s0;
    named_bar_sync(kBarSel, kSelThreads);
  }

  if (!p.do_attend) {  // select only: wait for phase B's hand-off, then leave with the cluster
    named_bar_sync(kBarHand, kWork * 32);
    pdl_launch_dependents();
    cluster_arrive();
    cluster_wait();
    return;
  }

  // ---------------------------------------------------------------- attention
  // Work unit: a group of 4 rows of one staged block; select warp w takes groups w, w + 8, ...
  // Each lane holds VEP = D / 32 channels of every row, with an online softmax per warp and head.
  // The group holding a block's first rows also removes the block's compensation term.
  constexpr int VEP = D / 32;
  constexpr int GR = 4;
  constexpr int GPB = kBlockTokens / GR;
  constexpr int NV = GR * G;
  constexpr int LPV = 32 / NV;
  static_assert(NV <= 32, "unsupported head layout");
  float acc[G][VEP], mw[G], lw[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    mw[h] = -CUDART_INF_F;
    lw[h] = 0.f;
#pragma unroll
    for (int e = 0; e < VEP; ++e) acc[h][e] = 0.f;
  }
  const int my_v = lane / LPV, my_r = my_v / G, my_vh = my_v % G;
  unsigned char* kvs = sm + L.kv;
  const int KVB = L.KVB;
  const int nr = (nsl + KVB - 1) / KVB;
  // staging of round rr (one thread): K and V rows up to the cache capacity, and the mean value
  auto issue = [&](int rr) {
    const int buf = rr & 1;
    const int i0 = rr * KVB, cnt = min(KVB, nsl - i0);
    uint32_t total = 0;
    for (int i = 0; i < cnt; ++i) {
      const int j = slot_s[i0 + i];
      const int rows = (j >= 0 && j < Nb) ? min(kBlockTokens, p.T - j * kBlockTokens) : 0;
      total += 2u * rows * D * sizeof(TQ) + (rows > 0 && compensate ? D * sizeof(S) : 0u);
    }
    mbar_arrive_expect_tx(&kvbar[buf], total);
    for (int i = 0; i < cnt; ++i) {
      const int j = slot_s[i0 + i];
      const int rows = (j >= 0 && j < Nb) ? min(kBlockTokens, p.T - j * kBlockTokens) : 0;
      if (rows == 0) continue;
      unsigned char* dst = kvs + (static_cast<size_t>(buf) * KVB + i) * L.kvblk;
      const size_t off = (static_cast<size_t>(pr) * p.T + static_cast<size_t>(j) * kBlockTokens) * D;
      const uint32_t bytes = static_cast<uint32_t>(rows) * D * sizeof(TQ);
      bulk_g2s(dst, static_cast<const TQ*>(p.K) + off, bytes, &kvbar[buf]);
      bulk_g2s(dst + L.kv_v, static_cast<const TQ*>(p.V) + off, bytes, &kvbar[buf]);
      if (compensate)
        bulk_g2s(dst + L.kv_nu, static_cast<const S*>(p.mean_v) + (static_cast<size_t>(pr) * Nb + j) * D,
                 D * sizeof(S), &kvbar[buf]);
    }
  };
  if (stid == 0) {
    if (nr > 0) issue(0);
    if (nr > 1) issue(1);
  }
  bool aok = true;
#pragma unroll 1
  for (int rr = 0; rr < nr; ++rr) {
    const int buf = rr & 1;
    const int i0 = rr * KVB, cnt = min(KVB, nsl - i0);
    aok = __all_sync(0xffffffffu, aok && mbar_wait(&kvbar[buf], static_cast<uint32_t>((rr >> 1) & 1), p.status));
    const int ngroups = aok ? cnt * GPB : 0;
#pragma unroll 1
    for (int g = sw; g < ngroups; g += kHalf) {
      const int i = g / GPB, t0 = (g % GPB) * GR;
      const int j = slot_s[i0 + i];
      const bool valid = j >= 0 && j < Nb;
      const bool first = (g % GPB) == 0;
      const int rows = valid ? min(kBlockTokens, p.T - j * kBlockTokens) : 0;
      const int n = valid ? max(0, min(p.count[static_cast<size_t>(pr) * Nb + j], rows)) : 0;
      float xh = -CUDART_INF_F;
      if (compensate && first && valid) {
        if (L.ux_smem && p.do_select) {
          const int owner = j / chunk, jl = j - owner * chunk;
          xh = ld_dsmem_f32(dsmem_addr(reinterpret_cast<float*>(sm + L.x) + jl * G + my_vh, owner));
        } else {
          xh = p.xrec[(static_cast<size_t>(pr) * Nb + j) * G + my_vh];
        }
      }
      const unsigned char* blk = kvs + (static_cast<size_t>(buf) * KVB + i) * L.kvblk;
      const TQ* krow = reinterpret_cast<const TQ*>(blk);
      const TQ* vrow = reinterpret_cast<const TQ*>(blk + L.kv_v);
      // logits of the group's rows (rows past the token count are masked below)
      float v[NV];
#pragma unroll
      for (int rr2 = 0; rr2 < GR; ++rr2) {
        float kf[VEP];
        if (t0 + rr2 < rows) {
          kvrow<TQ, VEP>(krow + (t0 + rr2) * D, lane, kf);
        } else {
#pragma unroll
          for (int e = 0; e < VEP; ++e) kf[e] = 0.f;
        }
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float qh[VEP];
          if constexpr (VEP == 4) {
            const float4 t = reinterpret_cast<const float4*>(q_s + h * D)[lane];
            qh[0] = t.x;
            qh[1] = t.y;
            qh[2] = t.z;
            qh[3] = t.w;
          } else {
            const float2 t = reinterpret_cast<const float2*>(q_s + h * D)[lane];
            qh[0] = t.x;
            qh[1] = t.y;
          }
          float sdot = 0.f;
#pragma unroll
          for (int e = 0; e < VEP; ++e) sdot = fmaf(qh[e], kf[e], sdot);
          v[rr2 * G + h] = sdot;
        }
      }
      TransposeReduce<NV, 16>::run(v, lane);  // lane holds (row my_r, head my_vh)
      const bool live = t0 + my_r < n;
      const float lg = live ? p.scale * v[0] : -CUDART_INF_F;
      float gm = lg;
#pragma unroll
      for (int o = LPV * G; o < 32; o <<= 1) gm = fmaxf(gm, __shfl_xor_sync(0xffffffffu, gm, o));
      gm = fmaxf(gm, xh);
      float mn[G], sc[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float gh = __shfl_sync(0xffffffffu, gm, h * LPV);
        mn[h] = fmaxf(mw[h], gh);
        sc[h] = (mw[h] == -CUDART_INF_F) ? 0.f : __expf(mw[h] - mn[h]);
      }
      const float mme = pick_h<G>(mn, my_vh);
      const float pe = (lg == -CUDART_INF_F) ? 0.f : __expf(lg - mme);
      float ps = pe;
#pragma unroll
      for (int o = LPV * G; o < 32; o <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
      const float pw = (xh == -CUDART_INF_F) ? 0.f : __expf(xh - mme);
      // the block's compensation term leaves (first group only; nu is zero otherwise)
      float nu[VEP];
#pragma unroll
      for (int e = 0; e < VEP; ++e) nu[e] = 0.f;
      if (compensate && first && valid && rows > 0) {
        const S* nrow = reinterpret_cast<const S*>(blk + L.kv_nu) + lane * VEP;
#pragma unroll
        for (int e = 0; e < VEP; ++e) nu[e] = sload(nrow + e);
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float psum = __shfl_sync(0xffffffffu, ps, h * LPV);
        const float pwh = __shfl_sync(0xffffffffu, pw, h * LPV);
        lw[h] = lw[h] * sc[h] + psum - pwh;
        mw[h] = mn[h];
#pragma unroll
        for (int e = 0; e < VEP; ++e) acc[h][e] = fmaf(-pwh, nu[e], acc[h][e] * sc[h]);
      }
      // P.V over the live rows (rows past the token count carry weight 0 and are skipped, so
      // stale shared memory never meets a zero weight)
#pragma unroll
      for (int rr2 = 0; rr2 < GR; ++rr2) {
        if (t0 + rr2 < n) {
          float vf[VEP];
          kvrow<TQ, VEP>(vrow + (t0 + rr2) * D, lane, vf);
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const float prh = __shfl_sync(0xffffffffu, pe, (rr2 * G + h) * LPV);
#pragma unroll
            for (int e = 0; e < VEP; ++e) acc[h][e] = fmaf(prh, vf[e], acc[h][e]);
          }
        }
      }
    }
    named_bar_sync(kBarSel, kSelThreads);  // every warp is done with this buffer
    if (stid == 0 && rr + 2 < nr) issue(rr + 2);
  }

  // the 8 warps' partials -> this rank's attention partial (M_h, L_h, A_h) in apart
  float* wacc = reinterpret_cast<float*>(sm + L.kv);   // [kHalf][G][D] (the staging is free)
  float* wml = reinterpret_cast<float*>(sm + L.wml);   // [kHalf][G][2], factors [kHalf][G]
  float* apart = reinterpret_cast<float*>(sm + L.apart);
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < VEP; ++e) wacc[(sw * G + h) * D + lane * VEP + e] = acc[h][e];
  if (lane == 0) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      wml[(sw * G + h) * 2] = mw[h];
      wml[(sw * G + h) * 2 + 1] = lw[h];
    }
  }
  named_bar_sync(kBarSel, kSelThreads);
  float* wf = wml + kHalf * G * 2;
  if (sw < G) {  // warp h: head h's factors over the 8 warps
    const int h = sw;
    const float mwv = lane < kHalf ? wml[(lane * G + h) * 2] : -CUDART_INF_F;
    float M = mwv;
#pragma unroll
    for (int o = kHalf / 2; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const float f = (mwv == -CUDART_INF_F) ? 0.f : __expf(mwv - M);
    float Ls = lane < kHalf ? f * wml[(lane * G + h) * 2 + 1] : 0.f;
#pragma unroll
    for (int o = kHalf / 2; o > 0; o >>= 1) Ls += __shfl_xor_sync(0xffffffffu, Ls, o);
    if (lane < kHalf) wf[lane * G + h] = f;
    if (lane == 0) {
      apart[h * (D + 2)] = M;
      apart[h * (D + 2) + 1] = Ls;
    }
  }
  named_bar_sync(kBarSel, kSelThreads);
  for (int i = stid; i < E; i += kSelThreads) {
    const int h = i / D;
    float a = 0.f;
#pragma unroll
    for (int w = 0; w < kHalf; ++w) a = fmaf(wf[w * G + h], wacc[(w * G + h) * D + (i % D)], a);
    apart[h * (D + 2) + 2 + (i % D)] = a;
  }
  // the rank's compensation partial: from phase B (fused), or from the workspace
  named_bar_sync(kBarHand, kWork * 32);  // the stream warps' hand-off (always one per launch)
  const float* cp = nullptr;
  if (compensate) cp = stream ? cpl : p.cpart + (static_cast<size_t>(pr) * kMaxC + rank) * G * (D + 2);
  named_bar_sync(kBarSel, kSelThreads);
  float* fac = reinterpret_cast<float*>(sm + L.fac);  // [G][2]: attention and compensation factors
  if (stid < G) {
    const int h = stid;
    const float ma = apart[h * (D + 2)], la = apart[h * (D + 2) + 1];
    float mc = -CUDART_INF_F, lc = 0.f;
    if (cp) {
      mc = cp[h * (D + 2)];
      lc = cp[h * (D + 2) + 1];
    }
    const float M = fmaxf(ma, mc);
    const float fa = exp_diff(ma, M), fc = exp_diff(mc, M);
    fac[2 * h] = fa;
    fac[2 * h + 1] = fc;
    fac[2 * G + 2 * h] = M;
    fac[2 * G + 2 * h + 1] = fmaf(fa, la, fc * lc);
  }
  named_bar_sync(kBarSel, kSelThreads);
  // push this rank's partial of every output slice to the rank that owns it
  float* racc = reinterpret_cast<float*>(sm + L.racc);  // [C][per_o]
  float* rml = reinterpret_cast<float*>(sm + L.rml);    // [C][G][2]
  if (sw < G) {
    const int h = sw;
    const int o_lo = (h * D) / per_o, o_hi = (h * D + D - 1) / per_o;
    const int o = o_lo + lane;
    if (o <= o_hi && o < C) {
      const uint64_t ml = (static_cast<uint64_t>(__float_as_uint(fac[2 * G + 2 * h + 1])) << 32) |
                          __float_as_uint(fac[2 * G + 2 * h]);
      st_async_b64(cluster_smem_addr(rml + (rank * G + h) * 2, o), ml, cluster_smem_addr(obar, o));
    }
  }
  for (int i = stid; i < E; i += kSelThreads) {
    const int h = i / D, c = i % D;
    float a = fac[2 * h] * apart[h * (D + 2) + 2 + c];
    if (cp) a = fmaf(fac[2 * h + 1], cp[h * (D + 2) + 2 + c], a);
    const int ow = i / per_o;
    st_async_b32(cluster_smem_addr(racc + rank * per_o + (i - ow * per_o), ow), __float_as_uint(a),
                 cluster_smem_addr(obar, ow));
  }
  pdl_launch_dependents();
  cluster_arrive();  // this rank's pushes are issued (matched by the wait before exit)

  // ---------------------------------------------------------------- outputs of this rank's slice
  const bool have = (oe0 < oe1) && __all_sync(0xffffffffu, mbar_wait_cluster(obar, 0, p.status));
  if (have) {
    const int hlo = oe0 / D, nh = (oe1 - 1) / D - hlo + 1;
    float* f2 = fac + 4 * G;  // [nh][C + 1]: per-rank factors, then 1 / denominator
    if (sw < nh) {
      const int h = hlo + sw;
      const float ms = lane < C ? rml[(lane * G + h) * 2] : -CUDART_INF_F;
      const float ls = lane < C ? rml[(lane * G + h) * 2 + 1] : 0.f;
      const float M = warp_max(ms);
      const float f = exp_diff(ms, M);
      const float den = warp_sum(f * ls);
      if (lane < C) f2[sw * (kMaxC + 1) + lane] = f;
      if (lane == 0) f2[sw * (kMaxC + 1) + kMaxC] = den > 0.f ? 1.f / den : 0.f;
    }
  }
  named_bar_sync(kBarSel, kSelThreads);
  if (have) {
    const int hlo = oe0 / D;
    const float* f2 = fac + 4 * G;
    float* o = p.out + static_cast<size_t>(pr) * E;
    for (int i = oe0 + stid; i < oe1; i += kSelThreads) {
      const int hs = i / D - hlo;
      float a = 0.f;
      for (int c = 0; c < C; ++c) a = fmaf(f2[hs * (kMaxC + 1) + c], racc[c * per_o + (i - oe0)], a);
      o[i] = a * f2[hs * (kMaxC + 1) + kMaxC];
    }
  }
  cluster_wait();  // no CTA leaves while a peer may still read or write its shared memory
}

// ------------------------------------------------------------------------------ host side

template <typename TQ, int D, typename S, int LS>
const void* kp_g(int G) {
  switch (G) {
    case 1: return reinterpret_cast<const void*>(&decode_step_kernel<TQ, D, 1, S, LS>);
    case 2: return reinterpret_cast<const void*>(&decode_step_kernel<TQ, D, 2, S, LS>);
    case 4: return reinterpret_cast<const void*>(&decode_step_kernel<TQ, D, 4, S, LS>);
    case 8: return reinterpret_cast<const void*>(&decode_step_kernel<TQ, D, 8, S, LS>);
  }
  return nullptr;
}

template <typename S, int LS>
const void* kp_t(bool bf16, int D, int G) {
  if (bf16) return D == 128 ? kp_g<uint16_t, 128, S, LS>(G) : (D == 64 ? kp_g<uint16_t, 64, S, LS>(G) : nullptr);
  return D == 128 ? kp_g<float, 128, S, LS>(G) : (D == 64 ? kp_g<float, 64, S, LS>(G) : nullptr);
}

template <typename S>
const void* kp_ls(bool bf16, int D, int G, int ls) {
  switch (ls) {
    case 1: return kp_t<S, 1>(bf16, D, G);
    case 2: return kp_t<S, 2>(bf16, D, G);
    default: return kp_t<S, 4>(bf16, D, G);
  }
}

const void* pick_kernel(bool bf16, bool fp16, int D, int G, int ls) {
  return fp16 ? kp_ls<__half>(bf16, D, G, ls) : kp_ls<float>(bf16, D, G, ls);
}

struct Plan {
  const void* kern = nullptr;
  int dev = -1, pairs = 0, Nb = 0, Kb = 0, G = 0, D = 0, r = 0, ssz = 0, esz = 0;
  StepLay L;
};
Plan g_plans[32];
int g_nplans = 0, g_next = 0;
std::mutex g_mu;

cudaLaunchConfig_t make_cfg(int pairs, int C, size_t smem, cudaStream_t st, cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pairs * C, 1, 1);
  cfg.blockDim = dim3(kNT, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cfg;
}

// Shared-memory layout for C ranks, or total = 0 if nothing fits.
StepLay layout_for(const StepShape& a, int C, size_t optin) {
  const int chunk = ((a.Nb + C - 1) / C + kTile - 1) / kTile * kTile;
  const int Kb = a.Kb;
  const int per = (Kb + C - 1) / C;
  StepLay L;
  for (int ux = 1; ux >= 0; --ux) {
    if (ux && static_cast<size_t>(2) * chunk * a.G * 4 > (64u << 10)) continue;
    for (int NS = 8; NS >= 3; --NS) {
      for (int KVB = std::min(per > 0 ? per : 1, 4); KVB >= 1; KVB /= 2) {
        L.build(a.D, a.G, a.r, a.fp16_summ ? 2 : 4, a.bf16 ? 2 : 4, Kb, a.Nb, C, chunk, NS, KVB, ux);
        if (L.total <= optin) return L;
        if (KVB == 1) break;
      }
    }
  }
  L.total = 0;
  return L;
}

cudaError_t make_plan(const void* kern, const StepShape& a, StepLay* out) {
  int dev = 0, sms = 0, optin = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e != cudaSuccess) return e;
  // ranks: as many as one wave of one CTA per SM allows (at most 16), at least 64 blocks each
  int cmax = std::max(1, std::min(kMaxC, sms / std::max(1, a.pairs)));
  while (cmax > 1 && (a.Nb + cmax - 1) / cmax < 64) --cmax;
  StepLay best;
  best.total = 0;
  long long best_score = -1;
  int last = 0;
  for (int C0 = cmax; C0 >= 1; --C0) {
    // chunks are whole 32-block tiles: C0 ranks may cover the blocks with fewer
    const int chunk0 = ((a.Nb + C0 - 1) / C0 + kTile - 1) / kTile * kTile;
    const int C = (a.Nb + chunk0 - 1) / chunk0;
    if (C == last) continue;
    last = C;
    StepLay L = layout_for(a, C, static_cast<size_t>(optin));
    if (L.total == 0 || (a.Nb + L.chunk - 1) / L.chunk != C) continue;
    cudaLaunchAttribute attr[2];
    cudaLaunchConfig_t cfg = make_cfg(a.pairs, C, L.total, nullptr, attr);
    int ncl = 0;
    if (cudaOccupancyMaxActiveClusters(&ncl, kern, &cfg) != cudaSuccess) {
      cudaGetLastError();
      ncl = 0;
    }
    if (ncl < 1) continue;
    if (ncl >= a.pairs) {  // one wave: take the largest such C
      *out = L;
      return cudaSuccess;
    }
    const long long score = static_cast<long long>(std::min(ncl, a.pairs)) * C;
    if (score > best_score) {
      best_score = score;
      best = L;
    }
  }
  if (best.total == 0) return cudaErrorInvalidConfiguration;
  *out = best;
  return cudaSuccess;
}

}  // namespace

int step_list_slots(int Kb) { return Kb <= 32 ? 1 : (Kb <= 64 ? 2 : 4); }

cudaError_t step_plan(const StepShape& a, int* C, int* chunk, size_t* smem) {
  const void* kern = pick_kernel(a.bf16, a.fp16_summ, a.D, a.G, step_list_slots(a.Kb));
  if (!kern) return cudaErrorInvalidValue;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(g_mu);
  for (int i = 0; i < g_nplans; ++i) {
    const Plan& q = g_plans[i];
    if (q.kern == kern && q.dev == dev && q.pairs == a.pairs && q.Nb == a.Nb && q.Kb == a.Kb && q.r == a.r) {
      *C = q.L.C;
      *chunk = q.L.chunk;
      *smem = q.L.total;
      return cudaSuccess;
    }
  }
  Plan pl;
  cudaError_t e = make_plan(kern, a, &pl.L);
  if (e != cudaSuccess) return e;
  pl.kern = kern;
  pl.dev = dev;
  pl.pairs = a.pairs;
  pl.Nb = a.Nb;
  pl.Kb = a.Kb;
  pl.r = a.r;
  const int slot = g_nplans < 32 ? g_nplans++ : (g_next++ % 32);
  g_plans[slot] = pl;
  *C = pl.L.C;
  *chunk = pl.L.chunk;
  *smem = pl.L.total;
  return cudaSuccess;
}

cudaError_t launch_decode_step(const StepArgs& a, cudaStream_t st) {
  const void* kern = pick_kernel(a.s.bf16, a.s.fp16_summ, a.s.D, a.s.G, step_list_slots(a.s.Kb));
  if (!kern) return cudaErrorInvalidValue;
  int dev = 0;
  cudaGetDevice(&dev);
  StepLay L;
  bool found = false;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    for (int i = 0; i < g_nplans; ++i) {
      const Plan& q = g_plans[i];
      if (q.kern == kern && q.dev == dev && q.pairs == a.s.pairs && q.Nb == a.s.Nb && q.Kb == a.s.Kb && q.r == a.s.r) {
        L = q.L;
        found = true;
      }
    }
  }
  if (!found) {
    int C = 0, chunk = 0;
    size_t smem = 0;
    cudaError_t e = step_plan(a.s, &C, &chunk, &smem);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(g_mu);
    for (int i = 0; i < g_nplans; ++i) {
      const Plan& q = g_plans[i];
      if (q.kern == kern && q.dev == dev && q.pairs == a.s.pairs && q.Nb == a.s.Nb && q.Kb == a.s.Kb && q.r == a.s.r) L = q.L;
    }
  }
  StepParams p;
  p.L = L;
  p.mode = a.mode;
  p.do_select = a.do_select ? 1 : 0;
  p.do_attend = a.do_attend ? 1 : 0;
  p.do_stream = a.do_stream ? 1 : 0;
  p.Nb = a.s.Nb;
  p.Kb = a.s.Kb;
  p.T = a.s.T;
  p.r = a.s.r;
  p.scale = a.scale;
  p.q = a.q;
  p.K = a.K;
  p.V = a.V;
  p.mean_k = a.mean_k;
  p.var_g = a.var_g;
  p.mean_v = a.mean_v;
  p.count = a.count;
  p.ug = a.ug;
  p.xrec = a.xrec;
  p.cpart = a.cpart;
  p.sel_idx = a.sel_idx;
  p.scores = a.scores;
  p.out = a.out;
  p.status = a.status;
  cudaLaunchAttribute attr[2];
  cudaLaunchConfig_t cfg = make_cfg(a.s.pairs, L.C, L.total, st, attr);
  void* args[] = {&p};
  return cudaLaunchKernelExC(&cfg, kern, args);
}

}  // namespace compkv
