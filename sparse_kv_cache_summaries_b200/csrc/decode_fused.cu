// a1 (second half) + a2 + a3. Normalised group score, Top-K selection, and exact attention over
// the selected blocks with Mean compensation of every omitted block, in one softmax (CompKV
// abstract: exact attention over a selected subset, compensation of the omitted tail; review,
// Summary: blocks selected up to a token budget by the compensation-aware score, "omitted blocks
// contribute their block-mean logit").
//
// Runs after the streaming kernel, whose outputs it reads from the workspace: per-block log
// scores u_{j,h}, per-block records {x_h = s q_h . mu_j + log n_j, n_j}, and per-segment partials
// of log Zhat and of the compensation sum over all blocks.
//
// One thread-block cluster of C CTAs per (sequence, kv-head); rank c owns the blocks
// [c*chunk, c*chunk + chunk):
//  1. log Zhat_h (log-sum-exp over the segments), S_j = sum_h exp(u_{j,h} - log Zhat_h) for the
//     rank's blocks as order-preserving uint32 keys (empty blocks key 0), and the rank's
//     candidates: its own best under (S desc, index asc).
//  2. Rank 0 takes the global Top-K_b from the C candidate lists, read over distributed shared
//     memory; the global Top-K_b under this strict order always lies inside the union of the
//     local ones, so the result is exact. For K_b <= 32, and for K_b <= 128 when a rank holds
//     at most 1024 blocks, the lists are each rank's best 32 LS as 64-bit codes (key, then
//     index; LS = 1, 2 or 4 entries per lane), built with warp bitonic networks, merged within
//     the CTA by counting (lists of 32: each entry's rank among the warps' lists) or by warp
//     bitonic merges, and at rank 0 by a tree of warp bitonic merges; otherwise radix selection. Meanwhile the other ranks merge the compensation partials of
//     the kv-head's segments, a slice of channels each.
//  3. Rank c attends the c-th contiguous slice of rank 0's ordered selection (balanced whatever
//     the blocks' positions; rank 0 writes each rank's slots into its shared memory and releases
//     them through st.async bytes counted on the rank's mbarrier): their K and V rows read
//     straight into registers (up to the cache capacity; rows past the block's token count are
//     masked) with the blocks' mean values, exact logits, an online softmax per warp and head,
//     P.V, and removal of the blocks' compensation terms (taken against a reference at least
//     every processed block's mean logit, so nothing overflows; a block's compensation mass
//     never exceeds its exact mass, so the removal cancels at most what it adds).
//  4. Every rank pushes its partial of each output slice into the rank that merges the slice
//     (st.async into the receiver's shared memory, counted on its mbarrier); each merging rank
//     combines its slice from local memory with the compensation partial (with selection, the
//     slice whose compensation sum it merged).
// Flags run steps 1-2 only (score/select call) or steps 3-4 only on a given selection (sparse
// decode call). Launched with programmatic dependent launch: the prologue overlaps the previous
// kernel's tail.
#include <cooperative_groups.h>

#include <mutex>

#include "attend.cuh"
#include "common.cuh"
#include "topk_lists.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace compkv {
namespace {

constexpr int kMaxCluster = 16;
constexpr int kWarpTopK = 128;  // K_b up to this: warp bitonic Top-K (lists of 32 LS); above: radix

// Entries per lane of the warp Top-K lists for K_b (lists of 32, 64 or 128 codes).
__host__ __device__ inline int list_slots(int Kb) { return Kb <= 32 ? 1 : (Kb <= 64 ? 2 : 4); }

__host__ __device__ inline size_t a16(size_t x) { return (x + 15) & ~static_cast<size_t>(15); }

// Shared-memory layout, identical on host and device.
struct FLay {
  int chunk, ccap, gcap, slots;
  size_t keys, ck, ci, gk, gi, hist, bc, sh, misc, zm, zs, fm, fl, cslice, selm;
  size_t q, wacc, wml, red, acc, ml, sc, fac, mbar, total;
  __host__ __device__ void build(int chunk_, int Kb, int C, int slots_, int G, int D) {
    chunk = chunk_;
    slots = slots_;
    ccap = Kb < chunk ? Kb : chunk;
    gcap = ccap * C;
    size_t o = 0;
    // radix histograms, or the warp Top-K's lists: [kWarps] warp lists, [kMaxCluster] pushed
    // rank lists and 2 x [kWarps] merge levels, of 32 * list_slots(K_b) codes each
    const size_t lists = sizeof(uint64_t) * (3 * kWarps + kMaxCluster) * 32 * list_slots(Kb);
    hist = o;   o = a16(o + (Kb <= kWarpTopK && lists > sizeof(uint32_t) * 2592 ? lists : sizeof(uint32_t) * 2592));
    keys = o;   o = a16(o + sizeof(uint32_t) * chunk);
    ck = o;     o = a16(o + sizeof(uint32_t) * (ccap + 1));
    ci = o;     o = a16(o + sizeof(int) * (ccap + 1));
    gk = o;     o = a16(o + sizeof(uint32_t) * (gcap + 1));
    gi = o;     o = a16(o + sizeof(int) * (gcap + 1));
    bc = o;     o = a16(o + sizeof(uint32_t) * 4);
    sh = o;     o = a16(o + sizeof(int) * 2 * kWarps);
    misc = o;   o = a16(o + sizeof(int) * 96);
    zm = o;     o = a16(o + sizeof(float) * slots * G);
    zs = o;     o = a16(o + sizeof(float) * slots * G);
    fm = o;     o = a16(o + sizeof(float) * slots * G);
    fl = o;     o = a16(o + sizeof(float) * slots * G);
    cslice = o; o = a16(o + sizeof(float) * G * D);
    selm = o;   o = a16(o + sizeof(int) * (Kb + 1));
    q = o;      o = a16(o + sizeof(float) * G * D);
    wacc = o;   o = a16(o + sizeof(float) * kWarps * G * D);      // the warps' partial sums
    wml = o;    o = a16(o + sizeof(float) * (3 * kWarps * G + 2 * G));  // (M, L), factors, rank's
    red = o;    o = a16(o + sizeof(float) * 256);                    // compensation merge scratch
    acc = o;    o = a16(o + sizeof(float) * 2 * G * D);          // received partials [C][slice]
    ml = o;     o = a16(o + sizeof(float) * kMaxCluster * 2 * G);  // received (m, l) [C][G][2]
    sc = o;     o = a16(o + sizeof(float) * 8);
    fac = o;    o = a16(o + sizeof(float) * G * 34);
    mbar = o;   o = a16(o + 8 * 3);
    total = o;
  }
};

struct FParams {
  FLay L;
  int mode, do_select, do_attend;
  int Nb, Kb, T, chunk, bpc, slots, nctas_stream, tiles_per_pair, total_tiles;
  float scale;
  const void* q;
  const void* K;
  const void* V;
  const void* mean_v;  // [pairs][Nb][D] of the summary type
  const float* u;
  const float* xrec;
  const float* zpart;
  const float* comp_seg;
  float* comp;        // merged compensation partial [pairs][G][D+2] (written by select-only,
                      // read by attend-only)
  int32_t* sel_idx;   // [pairs][Kb]: written by select, read by attend-only
  float* scores;
  float* out;
  int32_t* status;
};

// One lane's part of a K or V row: VEP consecutive elements as one vector load (read-only path).
template <int BYTES> struct RawOf;
template <> struct RawOf<4> { using type = uint32_t; };
template <> struct RawOf<8> { using type = uint2; };
template <> struct RawOf<16> { using type = uint4; };

template <typename T, int VEP>
struct RowPart {
  using Raw = typename RawOf<VEP * static_cast<int>(sizeof(T))>::type;
  static __device__ __forceinline__ Raw load(const T* row, int lane) {
    return __ldg(reinterpret_cast<const Raw*>(row) + lane);
  }
  static __device__ __forceinline__ Raw zero() {
    Raw z;
    uint32_t* u = reinterpret_cast<uint32_t*>(&z);
#pragma unroll
    for (int i = 0; i < static_cast<int>(sizeof(Raw)) / 4; ++i) u[i] = 0u;
    return z;
  }
  static __device__ __forceinline__ void unpack(const Raw& w, float (&f)[VEP]) {
    const uint32_t* u = reinterpret_cast<const uint32_t*>(&w);
    if constexpr (sizeof(T) == 2) {
#pragma unroll
      for (int i = 0; i < VEP / 2; ++i) {
        f[2 * i] = __uint_as_float(u[i] << 16);
        f[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
      }
    } else {
#pragma unroll
      for (int i = 0; i < VEP; ++i) f[i] = __uint_as_float(u[i]);
    }
  }
};

// The G log scores of one block (G consecutive floats, aligned to G floats) as vector loads.
template <int G>
__device__ __forceinline__ void load_scores(const float* src, float (&d)[G]) {
  if constexpr (G % 4 == 0) {
#pragma unroll
    for (int i = 0; i < G / 4; ++i) {
      const float4 t = reinterpret_cast<const float4*>(src)[i];
      d[4 * i] = t.x;
      d[4 * i + 1] = t.y;
      d[4 * i + 2] = t.z;
      d[4 * i + 3] = t.w;
    }
  } else if constexpr (G == 2) {
    const float2 t = *reinterpret_cast<const float2*>(src);
    d[0] = t.x;
    d[1] = t.y;
  } else {
#pragma unroll
    for (int i = 0; i < G; ++i) d[i] = src[i];
  }
}

__device__ __forceinline__ int stream_cta_of_tile(long long f, int nctas, int F) {
  return static_cast<int>(((f + 1) * nctas - 1) / F);
}


// S: summary storage type (float or __half); LS: entries per lane of the warp Top-K lists.
template <typename T, int D, int G, typename S, int LS>
__global__ void __launch_bounds__(kThreads) decode_fused_kernel(const __grid_constant__ FParams p) {
  constexpr int XS = xrec_stride(G);
  extern __shared__ __align__(128) unsigned char sm[];
  const FLay& L = p.L;
  cg::cluster_group cluster = cg::this_cluster();
  const int C = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  const int pr = blockIdx.x / C;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool compensate = p.mode != COMPKV_MODE_MASS;

  uint32_t* hist = reinterpret_cast<uint32_t*>(sm + L.hist);
  uint32_t* keys = reinterpret_cast<uint32_t*>(sm + L.keys);
  uint32_t* ck = reinterpret_cast<uint32_t*>(sm + L.ck);
  int* ci = reinterpret_cast<int*>(sm + L.ci);
  uint32_t* gk = reinterpret_cast<uint32_t*>(sm + L.gk);
  int* gi = reinterpret_cast<int*>(sm + L.gi);
  uint32_t* bc = reinterpret_cast<uint32_t*>(sm + L.bc);
  int* shs = reinterpret_cast<int*>(sm + L.sh);
  int* misc = reinterpret_cast<int*>(sm + L.misc);  // [0] candidates [1] gathered [6] selected [24..] gather offsets
  float* logz = reinterpret_cast<float*>(misc + 64);  // [8]
  float* cM = logz + 8;                               // [8] compensation max per head
  float* cl = logz + 16;                              // [8] compensation sum per head
  float* zm_s = reinterpret_cast<float*>(sm + L.zm);
  float* zs_s = reinterpret_cast<float*>(sm + L.zs);
  float* fm_s = reinterpret_cast<float*>(sm + L.fm);
  float* fl_s = reinterpret_cast<float*>(sm + L.fl);
  float* cslice = reinterpret_cast<float*>(sm + L.cslice);
  int* selm = reinterpret_cast<int*>(sm + L.selm);
  float* q_s = reinterpret_cast<float*>(sm + L.q);
  float* red = reinterpret_cast<float*>(sm + L.red);
  float* acc_s = reinterpret_cast<float*>(sm + L.acc);
  float* ml_s = reinterpret_cast<float*>(sm + L.ml);
  float* sc_s = reinterpret_cast<float*>(sm + L.sc);
  float* fac_s = reinterpret_cast<float*>(sm + L.fac);
  uint64_t* mbar = reinterpret_cast<uint64_t*>(sm + L.mbar);

  // Exchanges between the ranks are pushes: a rank writes into the receiver's shared memory with
  // st.async, which completes bytes on the receiver's mbarrier, and the receiver waits (bounded)
  // on its own mbarrier for exactly the bytes it expects:
  //   mbar[0]  rank 0: the C candidate lists (warp Top-K path)
  //   mbar[1]  this rank's selection slots, from rank 0 (warp Top-K path)
  //   mbar[2]  merging ranks: the C partials of their output slice and (M, L) of its heads
  constexpr int E = G * D;
  const bool warp_topk = p.do_select && p.Kb > 0 && p.Kb <= 32 * LS;
  constexpr int LW = 32 * LS;  // entries of a warp Top-K list
  const int first_owner = (p.do_select && C > 1) ? 1 : 0;
  const int n_owners = C - first_owner;
  const int per_o = ((E + n_owners - 1) / n_owners + 3) & ~3;  // a multiple of 4: 16-byte pushes
  const int wr = rank - first_owner;                    // this rank's output slice, if >= 0
  const int oe0 = wr >= 0 ? min(E, wr * per_o) : E, oe1 = wr >= 0 ? min(E, oe0 + per_o) : E;
  const int per_slot = (p.Kb + C - 1) / C;
  const int my_slots = max(0, min(per_slot, p.Kb - rank * per_slot));
  if (tid == 0) {
    mbar_init(&mbar[0], 1);
    mbar_init(&mbar[1], 1);
    mbar_init(&mbar[2], 1);
    mbar_init_fence();
    if (warp_topk && rank == 0) mbar_arrive_expect_tx(&mbar[0], static_cast<uint32_t>(C * LW * 8));
    if (warp_topk && p.do_attend && my_slots > 0) mbar_arrive_expect_tx(&mbar[1], static_cast<uint32_t>(my_slots * 4));
    if (p.do_attend && oe0 < oe1) {
      const int nh = (oe1 - 1) / D - oe0 / D + 1;
      mbar_arrive_expect_tx(&mbar[2], static_cast<uint32_t>(C * ((oe1 - oe0) * 4 + nh * 8)));
    }
  }
  if (p.do_attend) {
    const T* qp = static_cast<const T*>(p.q) + static_cast<size_t>(pr) * G * D;
    for (int i = tid; i < G * D; i += kThreads) q_s[i] = to_float(qp[i]);
  }
  __syncthreads();
  cluster_arrive_relaxed();  // matched by cluster_wait() before this CTA first writes a peer

  pdl_wait();  // the previous kernel's outputs are visible from here on
  pdl_launch_dependents();  // every CTA of this grid is resident: the next grid may stage in

  const int Kb = p.Kb;
  const int j0 = rank * p.chunk;
  const int nloc = max(0, min(p.chunk, p.Nb - j0));
  int nsel = 0;

  if (p.do_select) {
    const long long f_first = static_cast<long long>(pr) * p.tiles_per_pair;
    const int c_first = stream_cta_of_tile(f_first, p.nctas_stream, p.total_tiles);
    const int nseg = stream_cta_of_tile(f_first + p.tiles_per_pair - 1, p.nctas_stream, p.total_tiles) - c_first + 1;
    const float* zp = p.zpart + static_cast<size_t>(pr) * p.slots * G * 2;
    const float* cs = p.comp_seg + static_cast<size_t>(pr) * p.slots * G * (D + 2);
    const float* up = p.u + (static_cast<size_t>(pr) * p.Nb + j0) * G;
    // ---- 1a. segment partials (one round trip); per-block log scores stay in flight meanwhile
    for (int t = tid; t < nseg * G; t += kThreads) {
      zm_s[t] = zp[2 * t];
      zs_s[t] = zp[2 * t + 1];
      if (compensate) {
        fm_s[t] = cs[static_cast<size_t>(t) * (D + 2)];
        fl_s[t] = cs[static_cast<size_t>(t) * (D + 2) + 1];
      }
    }
    // warp w keys the local blocks [w span, w span + span), 32 at a time (lane-contiguous)
    const int span = ((nloc + kWarps * 32 - 1) / (kWarps * 32)) * 32;
    const int jb = warp * span;
    constexpr int UPT = 4;  // log-score rows prefetched per thread before log Zhat is known
    float ur[UPT][G];
#pragma unroll
    for (int k = 0; k < UPT; ++k) {
      const int j = jb + k * 32 + lane;
#pragma unroll
      for (int h = 0; h < G; ++h) ur[k][h] = 0.f;
      if (k * 32 < span && j < nloc) load_scores<G>(up + static_cast<size_t>(j) * G, ur[k]);
    }
    __syncthreads();
    // ---- 1b. log Zhat per head; compensation max, factors and sum per head
    if (warp < G) {  // the largest segment maximum, then the segment sums rescaled to it
      const int h = warp;
      float m = -CUDART_INF_F;
      for (int t = lane; t < nseg; t += 32) m = fmaxf(m, zm_s[t * G + h]);
      m = warp_max(m);
      float s = 0.f;
      for (int t = lane; t < nseg; t += 32) {
        const float mt = zm_s[t * G + h];
        if (mt != -CUDART_INF_F) s = fmaf(zs_s[t * G + h], __expf(mt - m), s);
      }
      s = warp_sum(s);
      if (lane == 0) logz[h] = (m == -CUDART_INF_F) ? -CUDART_INF_F : m + logf(s);
    }
    __syncthreads();
    // ---- 1c/1d. keys of this rank's blocks and its candidates
    float lz[G];
#pragma unroll
    for (int h = 0; h < G; ++h) lz[h] = logz[h];
    // S_j of chunk k of this warp, as a key (empty blocks: 0); also written to `scores`
    auto key_of = [&](int k, int j) -> uint32_t {
      if (j >= nloc) return 0u;
      float S = 0.f;
      if (k < UPT) {
#pragma unroll
        for (int kk = 0; kk < UPT; ++kk)
          if (kk == k) {
#pragma unroll
            for (int h = 0; h < G; ++h) S += __expf(ur[kk][h] - lz[h]);
          }
      } else {
        float uj[G];
        load_scores<G>(up + static_cast<size_t>(j) * G, uj);
#pragma unroll
        for (int h = 0; h < G; ++h) S += __expf(uj[h] - lz[h]);
      }
      const bool empty = S != S;
      if (p.scores) p.scores[static_cast<size_t>(pr) * p.Nb + j0 + j] = empty ? 0.f : S;
      return empty ? 0u : score_key(S);
    };
    if (tid == 0) misc[0] = 0;
    uint64_t* h64 = reinterpret_cast<uint64_t*>(hist);
    uint64_t best[LS];  // warp 0 ends with this rank's best-LW list (warp Top-K path)
#pragma unroll
    for (int e = 0; e < LS; ++e) best[e] = 0ull;
    if (warp_topk) {
      // this rank's best LW (descending codes): a superset of its share
      if constexpr (LS == 1) {
        // chunks go in pairs: two independent sorts, then one merge
        for (int k = 0; k * 32 < span; k += 2) {
          const int ja = jb + k * 32 + lane, jc = ja + 32;
          const uint32_t ka = key_of(k, ja);
          const uint32_t kc = ((k + 1) * 32 < span) ? key_of(k + 1, jc) : 0u;
          const uint64_t sa = warp_sort_desc(ja < nloc ? topk_code(ka, j0 + ja) : 0ull);
          const uint64_t sc = warp_sort_desc(((k + 1) * 32 < span && jc < nloc) ? topk_code(kc, j0 + jc) : 0ull);
          const uint64_t m2 = warp_merge_top32(sa, sc);
          best[0] = (k == 0) ? m2 : warp_merge_top32(best[0], m2);
        }
        // the rank's list: each of the 8 warps' 256 entries finds its rank among them (the
        // entries above it in all 8 lists, its own list giving its position; the searches are
        // independent, with no branch between them) and the best 32 land in place
        uint64_t* rl = h64 + kWarps * LW + kMaxCluster * LW;  // rank 0's merge scratch, free now
        h64[warp * 32 + lane] = best[0];
        if (warp == 0) rl[lane] = 0ull;
        __syncthreads();
        {
          const uint64_t x = best[0];
          int rk = 0;
#pragma unroll
          for (int w2 = 0; w2 < kWarps; ++w2) rk += count_greater<32>(h64 + w2 * 32, x);
          if (x != 0ull && rk < 32) rl[rk] = x;
        }
        __syncthreads();
        best[0] = rl[lane];
      } else {
        // chunks of 32 go LS at a time: one list sort, then a merge into the running list
        for (int c0 = 0; c0 * 32 < span; c0 += LS) {
          uint64_t v[LS];
#pragma unroll
          for (int e = 0; e < LS; ++e) {
            const int c = c0 + e, j = jb + c * 32 + lane;
            v[e] = 0ull;
            if (c * 32 < span) {
              const uint32_t key = key_of(c, j);
              if (j < nloc) v[e] = topk_code(key, j0 + j);
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
        list_pairs_merge<LS>(best, h64);  // warp 0: the rank's list
      }
      // warp 1 when every warp holds the rank's list (lists of 32), so that warp 0 pushes it at once
      if (p.do_attend && warp == ((LS == 1) ? 1 : 0)) {
        // speculative: this rank's likeliest picks start moving from HBM to L2 while the global
        // cut runs (about 2 K_b / C of them: the global Top-K_b holds K_b / C per rank on average)
        const int m = min(32, max(1, (2 * Kb + C - 1) / C));
        const uint64_t code = best[0];
        if (lane < m && code != 0ull) {
          const int j = topk_index(code);
          const size_t off = (static_cast<size_t>(pr) * p.T + static_cast<size_t>(j) * kBlockTokens) * D;
          const size_t bytes = static_cast<size_t>(min(kBlockTokens, p.T - j * kBlockTokens)) * D * sizeof(T);
          prefetch_l2_range(static_cast<const T*>(p.K) + off, bytes);
          prefetch_l2_range(static_cast<const T*>(p.V) + off, bytes);
        }
      }
    } else {
      for (int k = 0; k * 32 < span; ++k) {
        const int j = jb + k * 32 + lane;
        const uint32_t key = key_of(k, j);
        if (j < nloc) keys[j] = key;
      }
      __syncthreads();
      if (Kb > 0) {
        int ncand;
        if (nloc <= Kb) {
          for (int j = tid; j < nloc; j += kThreads) {
            ck[j] = keys[j];
            ci[j] = j0 + j;
          }
          ncand = nloc;
        } else {
          auto kat = [&](int i) { return keys[i]; };
          const RadixCut cut = cta_topk_cut(kat, nloc, Kb, hist, bc, shs);
          ncand = cta_select_ordered_w(kat, nloc, cut, shs, [&](int i, int pos) {
            ck[pos] = keys[i];
            ci[pos] = j0 + i;
          });
        }
        if (tid == 0) misc[0] = ncand;
      }
    }
    cluster_wait();  // every rank has started: peers' shared memory may be written
    if (warp_topk && warp == 0) {  // push this rank's list into rank 0
#pragma unroll
      for (int e = 0; e < LS; ++e)
        st_async_b64(cluster_smem_addr(h64 + kWarps * LW + rank * LW + e * 32 + lane, 0), best[e],
                     cluster_smem_addr(&mbar[0], 0));
    }
    if (!warp_topk) cluster.sync();  // #1 (radix path): every rank's candidates are visible

    // ---- 2. rank 0: global Top-K_b from the ranks' candidates; other ranks: compensation merge
    if (rank == 0 && warp_topk) {
      // merge the C ranks' best-LW lists pairwise (the first level straight from the ranks'
      // shared memory), then order the first K_b by block index
      mbar_wait_cluster(&mbar[0], 0, p.status);  // the C lists have arrived
      const uint64_t* rl = h64 + kWarps * LW;    // [C][LW] pushed
      uint64_t* g0 = h64 + kWarps * LW + kMaxCluster * LW;
      uint64_t* g1 = g0 + kWarps * LW;
      // list o of `from` and list o + 1, merged into list w of `to` (one warp)
      auto merge_pair = [&](const uint64_t* from, int o, uint64_t* to, int w) {
        uint64_t a[LS], b[LS];
#pragma unroll
        for (int e = 0; e < LS; ++e) {
          a[e] = from[o * LW + e * 32 + lane];
          b[e] = from[(o + 1) * LW + e * 32 + lane];
        }
        list_merge_top<LS>(a, b);
#pragma unroll
        for (int e = 0; e < LS; ++e) to[w * LW + e * 32 + lane] = a[e];
      };
      int nl = 1;
      if (C == 1) {
        if (warp == 0) {
#pragma unroll
          for (int e = 0; e < LS; ++e) g0[e * 32 + lane] = rl[e * 32 + lane];
        }
      } else {
        if (warp < C / 2) merge_pair(rl, 2 * warp, g0, warp);
        nl = C / 2;
      }
      __syncthreads();
      uint64_t* src = g0;
      uint64_t* dst = g1;
      while (nl > 1) {
        if (warp < nl / 2) merge_pair(src, 2 * warp, dst, warp);
        __syncthreads();
        uint64_t* t = src;
        src = dst;
        dst = t;
        nl /= 2;
      }
      if (warp == 0) {
        if constexpr (LS == 1) {
          // block order: each selected block counts the selected blocks below it; slot i goes
          // to rank i / per_slot, which starts as soon as its bytes land (no cluster barrier)
          int* sel_i = reinterpret_cast<int*>(dst);  // the other merge buffer, free now
          const int mine = lane < Kb ? topk_index(src[lane]) : 0x7fffffff;
          sel_i[lane] = mine;
          __syncwarp();
          int pos = 0;
          for (int j2 = 0; j2 < Kb; ++j2) pos += sel_i[j2] < mine ? 1 : 0;
          if (lane < Kb) {
            if (p.sel_idx) p.sel_idx[static_cast<size_t>(pr) * Kb + pos] = mine;
            if (p.do_attend) {
              const int r = pos / per_slot;
              st_async_b32(cluster_smem_addr(&selm[pos - r * per_slot], r), static_cast<uint32_t>(mine),
                           cluster_smem_addr(&mbar[1], r));
            }
          }
        } else {
          int v[LS];
#pragma unroll
          for (int e = 0; e < LS; ++e) {
            const int i = e * 32 + lane;
            v[e] = i < Kb ? topk_index(src[i]) : 0x7fffffff;
          }
          list_sort_asc<LS>(v);
#pragma unroll
          for (int e = 0; e < LS; ++e) {
            const int i = e * 32 + lane;  // the i-th selected block in block order
            if (i < Kb) {
              if (p.sel_idx) p.sel_idx[static_cast<size_t>(pr) * Kb + i] = v[e];
              if (p.do_attend) {  // slot i goes to rank i / per_slot, which starts when its bytes land
                const int r = i / per_slot;
                st_async_b32(cluster_smem_addr(&selm[i - r * per_slot], r), static_cast<uint32_t>(v[e]),
                             cluster_smem_addr(&mbar[1], r));
              }
            }
          }
        }
        if (lane == 0) misc[6] = Kb;
      }
    } else if (rank == 0 && Kb > 0) {
      if (tid < C) misc[24 + tid] = *cluster.map_shared_rank(&misc[0], tid);
      __syncthreads();
      if (tid == 0) {
        int off = 0;
        for (int c = 0; c < C; ++c) {
          const int n = misc[24 + c];
          misc[24 + c] = off;
          off += n;
        }
        misc[24 + C] = off;
        misc[1] = off;
      }
      __syncthreads();
      const int M = misc[1];
      for (int i = tid; i < M; i += kThreads) {
        int c = 0;
        while (c + 1 < C && misc[24 + c + 1] <= i) ++c;
        const int k = i - misc[24 + c];
        gk[i] = *cluster.map_shared_rank(&ck[k], c);
        gi[i] = *cluster.map_shared_rank(&ci[k], c);
      }
      __syncthreads();
      auto kat = [&](int i) { return gk[i]; };
      RadixCut cut{0u, 0u, M, true};  // fewer candidates than K_b: keep them all
      if (M > Kb) cut = cta_topk_cut(kat, M, Kb, hist, bc, shs);
      int32_t* sel = p.sel_idx ? p.sel_idx + static_cast<size_t>(pr) * Kb : nullptr;
      const int nout = cta_select_ordered_w(kat, M, cut, shs, [&](int i, int pos) {
        selm[pos] = gi[i];
        if (sel) sel[pos] = gi[i];
      });
      if (tid == 0) misc[6] = nout;
    }
    if (compensate && (C == 1 || rank != 0)) {
      // compensation reference, segment factors and sum per head (off the selection's path)
      if (warp < G) {
        const int h = warp;
        float M = -CUDART_INF_F;
        for (int t = lane; t < nseg; t += 32) M = fmaxf(M, fm_s[t * G + h]);
        M = warp_max(M);
        float l = 0.f;
        for (int t = lane; t < nseg; t += 32) {
          const float mt = fm_s[t * G + h];
          const float f = (mt == -CUDART_INF_F) ? 0.f : __expf(mt - M);
          fm_s[t * G + h] = f;
          l = fmaf(f, fl_s[t * G + h], l);
        }
        l = warp_sum(l);
        if (lane == 0) {
          cM[h] = M;
          cl[h] = l;
        }
      }
      __syncthreads();
      // merge a slice of the compensation partials' channels: lanes along channels (coalesced),
      // 4 segment groups summed in a fixed order
      const int E = G * D, W = (C == 1) ? 1 : C - 1, wr = (C == 1) ? 0 : rank - 1;
      const int per = ((E + W - 1) / W + 3) & ~3;  // the output slices' partition
      const int e0 = wr * per, e1 = min(E, e0 + per);
      float* mrg = red;  // scratch (the attention has not started)
      const int ei = tid % 64, sg = tid / 64;
      for (int base = e0; base < e1; base += 64) {
        const int e = base + ei;
        float a = 0.f;
        if (e < e1) {
          const int h = e / D, c = e % D;
#pragma unroll 8
          for (int t = sg; t < nseg; t += 4)
            a = fmaf(fm_s[t * G + h], cs[(static_cast<size_t>(t) * G + h) * (D + 2) + 2 + c], a);
        }
        mrg[sg * 64 + ei] = a;
        __syncthreads();
        if (tid < 64 && base + tid < e1) {
          const int e2 = base + tid;
          const float v = ((mrg[tid] + mrg[64 + tid]) + mrg[128 + tid]) + mrg[192 + tid];
          cslice[e2] = v;
          if (!p.do_attend) p.comp[(static_cast<size_t>(pr) * G + e2 / D) * (D + 2) + 2 + (e2 % D)] = v;
        }
        __syncthreads();
      }
    }
    if (compensate && !p.do_attend && rank == (C == 1 ? 0 : 1) && tid < G) {
      float* o = p.comp + (static_cast<size_t>(pr) * G + tid) * (D + 2);
      o[0] = cM[tid];
      o[1] = cl[tid];
    }
    if (!warp_topk) cluster.sync();  // #2 (radix path): the cut is visible

    // ---- 3a. this rank's share of the selection: a contiguous slice of rank 0's ordered list
    if (p.do_attend && warp_topk) {  // rank 0 pushes this rank's slots
      nsel = (my_slots == 0 || __syncthreads_and(mbar_wait_cluster(&mbar[1], 0, p.status))) ? my_slots : 0;
    } else if (p.do_attend && Kb > 0) {
      const int total = *cluster.map_shared_rank(&misc[6], 0);
      const int per = (total + C - 1) / C;
      const int s0 = min(total, rank * per), s1 = min(total, s0 + per);
      if (rank != 0) {
        const int* sel0 = cluster.map_shared_rank(selm, 0);
        for (int i = tid; i < s1 - s0; i += kThreads) selm[i] = sel0[s0 + i];
      }
      nsel = s1 - s0;
      __syncthreads();
    }
  }
  if (!p.do_select && p.do_attend) {  // attend a given selection: rank c takes a slice of slots
    const int s0 = min(Kb, rank * p.bpc), s1 = min(Kb, s0 + p.bpc);
    for (int i = tid; i < s1 - s0; i += kThreads) selm[i] = p.sel_idx[static_cast<size_t>(pr) * Kb + s0 + i];
    nsel = s1 - s0;
    __syncthreads();
  }
  if (!p.do_attend) {  // select only: no CTA leaves while a peer's push into it may be in flight
    cluster.sync();
    return;
  }

  // ---- 3b. exact attention over this rank's selected blocks. Work unit: a group of 4 rows of
  // one block; warp w takes groups w, w + 8, ... Each lane holds VEP = D / 32 channels of every
  // row, read straight into registers (one vector load per row; no shared-memory staging, no
  // CTA barrier), with an online softmax per warp and head. The group of a block's first rows
  // also removes the block's compensation term, taken against a reference raised to at least
  // its mean logit, so no weight exceeds 1.
  constexpr int VEP = D / 32;
  constexpr int GR = 4;                      // rows per group
  constexpr int GPB = kBlockTokens / GR;     // groups per block
  constexpr int NV = GR * G;                 // (row, head) logits of a group
  constexpr int LPV = 32 / NV;               // lanes per (row, head) after the reduce
  static_assert(NV <= 32 && VEP >= 2, "unsupported head layout");
  using RP = RowPart<T, VEP>;
  const T* Kbase = static_cast<const T*>(p.K) + static_cast<size_t>(pr) * p.T * D;
  const T* Vbase = static_cast<const T*>(p.V) + static_cast<size_t>(pr) * p.T * D;
  const S* NUbase = static_cast<const S*>(p.mean_v) + static_cast<size_t>(pr) * p.Nb * D;
  const float* XRbase = p.xrec + static_cast<size_t>(pr) * p.Nb * XS;
  float qv[G][VEP];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < VEP; ++e) qv[h][e] = q_s[h * D + lane * VEP + e];
  float acc[G][VEP], mw[G], lw[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    mw[h] = -CUDART_INF_F;
    lw[h] = 0.f;
#pragma unroll
    for (int e = 0; e < VEP; ++e) acc[h][e] = 0.f;
  }
  const int my_v = lane / LPV, my_r = my_v / G, my_h = my_v % G;
  const int ngroups = nsel * GPB;
#pragma unroll 1
  for (int g = warp; g < ngroups; g += kWarps) {
    const int s2 = g / GPB, t0 = (g % GPB) * GR;
    int j = selm[s2];
    if (j < 0 || j >= p.Nb) j = -1;
    const bool first = (g % GPB) == 0;  // this group removes the block's compensation term
    // loads: the rows up to the cache capacity, the record, and the mean value (first group)
    typename RP::Raw kr[GR], vr[GR];
    const int cap = (j >= 0) ? min(kBlockTokens, p.T - j * kBlockTokens) : 0;
#pragma unroll
    for (int r = 0; r < GR; ++r) {
      const bool in = t0 + r < cap;
      const size_t row = (static_cast<size_t>(j) * kBlockTokens + t0 + r) * D;
      kr[r] = in ? RP::load(Kbase + row, lane) : RP::zero();
      vr[r] = in ? RP::load(Vbase + row, lane) : RP::zero();
    }
    const float* rec = XRbase + static_cast<size_t>(j >= 0 ? j : 0) * XS;
    const int n = (j >= 0) ? max(0, min(__float_as_int(__ldg(rec + G)), cap)) : 0;
    float xh = -CUDART_INF_F;
    float nu[VEP];
#pragma unroll
    for (int e = 0; e < VEP; ++e) nu[e] = 0.f;
    if (compensate && first && j >= 0) {
      xh = __ldg(rec + my_h);
      const S* nrow = NUbase + static_cast<size_t>(j) * D + lane * VEP;
#pragma unroll
      for (int e = 0; e < VEP; ++e) nu[e] = sload(nrow + e);
    }
    // logits: partial dots over this lane's channels, one transpose-reduce for the group
    float v[NV];
    float vf[GR][VEP];
#pragma unroll
    for (int r = 0; r < GR; ++r) {
      float kf[VEP];
      RP::unpack(kr[r], kf);
      RP::unpack(vr[r], vf[r]);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float sdot = 0.f;
#pragma unroll
        for (int e = 0; e < VEP; ++e) sdot = fmaf(qv[h][e], kf[e], sdot);
        v[r * G + h] = sdot;
      }
    }
    TransposeReduce<NV, 16>::run(v, lane);  // lane holds (row my_r, head my_h)
    const bool live = t0 + my_r < n;
    const float lg = live ? p.scale * v[0] : -CUDART_INF_F;
    // zero the V parts of rows past the token count (their weight is 0, but 0 * NaN is NaN)
#pragma unroll
    for (int r = 0; r < GR; ++r)
      if (t0 + r >= n) {
#pragma unroll
        for (int e = 0; e < VEP; ++e) vf[r][e] = 0.f;
      }
    // group max per head (over the rows), raised to the removed block's record if any
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
    float mme = mn[0];
#pragma unroll
    for (int h = 1; h < G; ++h) mme = (my_h == h) ? mn[h] : mme;
    const float pe = (lg == -CUDART_INF_F) ? 0.f : __expf(lg - mme);
    float ps = pe;
#pragma unroll
    for (int o = LPV * G; o < 32; o <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
    const float pw = (xh == -CUDART_INF_F) ? 0.f : __expf(xh - mme);
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float psum = __shfl_sync(0xffffffffu, ps, h * LPV);
      const float pwh = __shfl_sync(0xffffffffu, pw, h * LPV);
      lw[h] = lw[h] * sc[h] + psum - pwh;
      mw[h] = mn[h];
#pragma unroll
      for (int e = 0; e < VEP; ++e) acc[h][e] = fmaf(-pwh, nu[e], acc[h][e] * sc[h]);
#pragma unroll
      for (int r = 0; r < GR; ++r) {
        const float prh = __shfl_sync(0xffffffffu, pe, (r * G + h) * LPV);
#pragma unroll
        for (int e = 0; e < VEP; ++e) acc[h][e] = fmaf(prh, vf[r][e], acc[h][e]);
      }
    }
  }

  // ---- the warps' partials -> this rank's partial (M_h, L_h, A_h) in shared memory
  float* wacc = reinterpret_cast<float*>(sm + L.wacc);  // [kWarps][G][D]
  float* wml = reinterpret_cast<float*>(sm + L.wml);    // [kWarps][G][2], then factors [kWarps][G]
#pragma unroll
  for (int h = 0; h < G; ++h) {
#pragma unroll
    for (int e = 0; e < VEP; ++e) wacc[(warp * G + h) * D + lane * VEP + e] = acc[h][e];
  }
  if (lane == 0) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      wml[(warp * G + h) * 2] = mw[h];
      wml[(warp * G + h) * 2 + 1] = lw[h];
    }
  }
  __syncthreads();
  float* wf = wml + kWarps * G * 2;  // [kWarps][G] factors
  float* rM = wf + kWarps * G;       // [G] this rank's reference per head
  float* rL = rM + G;                // [G]
  if (warp < G) {  // warp h: head h's factors over the 8 warps (lanes 0..7, butterflies of 8)
    const int h = warp;
    const float mwv = lane < kWarps ? wml[(lane * G + h) * 2] : -CUDART_INF_F;
    float M = mwv;
#pragma unroll
    for (int o = kWarps / 2; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const float f = (mwv == -CUDART_INF_F) ? 0.f : __expf(mwv - M);
    float Lsum = lane < kWarps ? f * wml[(lane * G + h) * 2 + 1] : 0.f;
#pragma unroll
    for (int o = kWarps / 2; o > 0; o >>= 1) Lsum += __shfl_xor_sync(0xffffffffu, Lsum, o);
    if (lane < kWarps) wf[lane * G + h] = f;
    if (lane == 0) {
      rM[h] = M;
      rL[h] = Lsum;
    }
  }
  __syncthreads();
  // ---- this rank's partial, pushed to the ranks that merge the outputs. Output channels
  // [0, E) are cut into slices, one per merging rank: with selection ranks 1..C-1 (each holds
  // the compensation sum of its slice), without it ranks 0..C-1 (C = 1: rank 0 alone). Every
  // rank writes its partial of a slice into the merging rank's receive buffers.
  float* racc = acc_s;  // [C][per_o] received partial sums
  float* rml = ml_s;    // [C][G][2] received (M, L)
  if (!p.do_select) cluster_wait();  // every rank has started: peers may be written
  if (warp < G) {  // (M, L) of head `warp` to every merging rank whose slice touches the head
    const int h = warp;
    const int o_lo = first_owner + (h * D) / per_o, o_hi = first_owner + (h * D + D - 1) / per_o;
    const int o = o_lo + lane;
    if (o <= o_hi) {
      const uint64_t ml = (static_cast<uint64_t>(__float_as_uint(rL[h])) << 32) | __float_as_uint(rM[h]);
      st_async_b64(cluster_smem_addr(rml + (rank * G + h) * 2, o), ml, cluster_smem_addr(&mbar[2], o));
    }
  }
  for (int i = 4 * tid; i < E; i += 4 * kThreads) {  // 4 channels of one head per thread
    const int h = i / D;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float f = wf[w * G + h];
      const float4 x = *reinterpret_cast<const float4*>(wacc + w * E + i);
      a.x = fmaf(f, x.x, a.x);
      a.y = fmaf(f, x.y, a.y);
      a.z = fmaf(f, x.z, a.z);
      a.w = fmaf(f, x.w, a.w);
    }
    const int ow = i / per_o;
    st_async_v4(cluster_smem_addr(racc + rank * per_o + (i - ow * per_o), first_owner + ow), a,
                cluster_smem_addr(&mbar[2], first_owner + ow));
  }
  cluster_arrive();  // this rank's pushes are issued (matched by the wait before exit)

  // ---- 4. outputs of this rank's slice, from its receive buffers (local reads only)
  bool have = false;  // uniform over the CTA (a wait that gave up in any thread skips the merge)
  if (wr >= 0 && oe0 < oe1) have = __syncthreads_and(mbar_wait_cluster(&mbar[2], 0, p.status)) != 0;
  if (have) {
    const int e0 = oe0, e1 = oe1;
    const float* cpg = p.comp + static_cast<size_t>(pr) * G * (D + 2);
    if (e0 < e1) {
      const int hlo = e0 / D, nh = (e1 - 1) / D - hlo + 1;
      if (warp < nh) {  // warp w: head hlo + w's factors over the C ranks and the compensation
        const int h = hlo + warp;
        float cmh = -CUDART_INF_F, clh = 0.f;
        if (compensate) {
          cmh = p.do_select ? cM[h] : cpg[h * (D + 2)];
          clh = p.do_select ? cl[h] : cpg[h * (D + 2) + 1];
        }
        const float ms = lane < C ? rml[(lane * G + h) * 2] : -CUDART_INF_F;
        const float ls = lane < C ? rml[(lane * G + h) * 2 + 1] : 0.f;
        const float M = fmaxf(warp_max(ms), cmh);
        const float f = (ms == -CUDART_INF_F) ? 0.f : __expf(ms - M);
        const float fc = (cmh == -CUDART_INF_F) ? 0.f : __expf(cmh - M);
        const float den = fmaf(fc, clh, warp_sum(f * ls));
        if (lane < C) fac_s[warp * 17 + lane] = f;
        if (lane == 0) {
          fac_s[warp * 17 + 16] = fc;
          sc_s[warp] = den > 0.f ? 1.f / den : 0.f;
        }
      }
      __syncthreads();
      float* o = p.out + static_cast<size_t>(pr) * E;
      for (int i = e0 + tid; i < e1; i += kThreads) {
        const int hs = i / D - hlo, c = i % D;
        float a = 0.f;
        if (compensate) a = fac_s[hs * 17 + 16] * (p.do_select ? cslice[i] : cpg[(hs + hlo) * (D + 2) + 2 + c]);
        for (int s2 = 0; s2 < C; ++s2) a = fmaf(fac_s[hs * 17 + s2], racc[s2 * per_o + (i - e0)], a);
        o[i] = a * sc_s[hs];
      }
    }
  }
  cluster_wait();  // no CTA leaves while a peer's push into it may be in flight
}

template <typename T, int D, typename S, int LS>
const void* kptr_g(int G) {
  switch (G) {
    case 1: return reinterpret_cast<const void*>(&decode_fused_kernel<T, D, 1, S, LS>);
    case 2: return reinterpret_cast<const void*>(&decode_fused_kernel<T, D, 2, S, LS>);
    case 4: return reinterpret_cast<const void*>(&decode_fused_kernel<T, D, 4, S, LS>);
    case 8: return reinterpret_cast<const void*>(&decode_fused_kernel<T, D, 8, S, LS>);
  }
  return nullptr;
}

template <typename S, int LS>
const void* pick_se(bool bf16, int D, int G) {
  if (bf16) return D == 128 ? kptr_g<uint16_t, 128, S, LS>(G) : (D == 64 ? kptr_g<uint16_t, 64, S, LS>(G) : nullptr);
  return D == 128 ? kptr_g<float, 128, S, LS>(G) : (D == 64 ? kptr_g<float, 64, S, LS>(G) : nullptr);
}

template <typename S>
const void* pick_s(bool bf16, int D, int G, int ls) {
  switch (ls) {
    case 2: return pick_se<S, 2>(bf16, D, G);
    case 4: return pick_se<S, 4>(bf16, D, G);
    default: return pick_se<S, 1>(bf16, D, G);
  }
}

// The kernel for `ls` entries per lane of the Top-K lists (1 also serves the radix path).
const void* pick(bool bf16, int D, int G, bool fp16, int ls) {
  return fp16 ? pick_s<__half>(bf16, D, G, ls) : pick_s<float>(bf16, D, G, ls);
}

// Preferred cluster size: the largest power of two <= 16 that keeps the grid within two CTAs
// per SM and at least 64 blocks per rank.
int preferred_cluster(int pairs, int Nb, int sms) {
  int C0 = 1;
  while (C0 < kMaxCluster && pairs * (2 * C0) <= 2 * sms && (Nb + 2 * C0 - 1) / (2 * C0) >= 64) C0 *= 2;
  return C0;
}

// Lists above 32 entries pay a sort of every 32 of a rank's blocks per list entry slot; with
// more than this many blocks per rank the radix cut is cheaper (measured at 4096 blocks).
constexpr int kListMaxChunk = 1024;

// Launch plan of one problem shape: the cluster size and the shared-memory layout.
struct Plan {
  const void* kern = nullptr;
  int dev = -1, pairs = 0, Nb = 0, Kb = 0, slots = 0;
  int C = 0, chunk = 0;
  FLay L;
};
Plan g_plans[32];
int g_nplans = 0, g_next = 0;
std::mutex g_mu;

cudaLaunchConfig_t make_cfg(int pairs, int C, size_t smem, cudaStream_t st, cudaLaunchAttribute* attr, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pairs * C, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cfg;
}

// Cluster size: the largest power of two <= 16 that keeps the grid within two CTAs per SM and
// at least 64 blocks per rank, then the largest one the device can co-schedule.
cudaError_t make_plan(const void* kern, const FusedArgs& a, Plan* out) {
  int dev = 0, sms = 0, optin = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  const int C0 = preferred_cluster(a.pairs, a.Nb, sms);
  for (int C = C0; C >= 1; C /= 2) {
    const int chunk = (a.Nb + C - 1) / C;
    FLay L;
    L.build(chunk, a.Kb, C, a.slots, a.G, a.D);
    if (L.total > static_cast<size_t>(optin)) continue;
    // the opt-in maximum, so that plans of different sizes share the kernel's attribute
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    cudaLaunchAttribute attr[2];
    cudaLaunchConfig_t cfg = make_cfg(a.pairs, C, L.total, nullptr, attr, false);
    int ncl = 0;
    if (cudaOccupancyMaxActiveClusters(&ncl, kern, &cfg) != cudaSuccess) {
      cudaGetLastError();
      ncl = 0;
    }
    if (ncl >= 1) {
      out->C = C;
      out->chunk = chunk;
      out->L = L;
      return cudaSuccess;
    }
  }
  return cudaErrorInvalidConfiguration;
}

}  // namespace

cudaError_t launch_decode_fused(const FusedArgs& a, cudaStream_t st) {
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int chunk0 = (a.Nb + preferred_cluster(a.pairs, a.Nb, sms) - 1) / preferred_cluster(a.pairs, a.Nb, sms);
  const int ls = (a.Kb <= 32) ? 1 : ((a.Kb <= kWarpTopK && chunk0 <= kListMaxChunk) ? list_slots(a.Kb) : 1);
  const void* kern = pick(a.bf16, a.D, a.G, a.fp16_summ, ls);
  if (!kern) return cudaErrorInvalidValue;
  Plan plan;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    int found = -1;
    for (int i = 0; i < g_nplans; ++i) {
      const Plan& q = g_plans[i];
      if (q.kern == kern && q.dev == dev && q.pairs == a.pairs && q.Nb == a.Nb && q.Kb == a.Kb && q.slots == a.slots)
        found = i;
    }
    if (found >= 0) {
      plan = g_plans[found];
    } else {
      cudaError_t e = make_plan(kern, a, &plan);
      if (e != cudaSuccess) return e;
      plan.kern = kern;
      plan.dev = dev;
      plan.pairs = a.pairs;
      plan.Nb = a.Nb;
      plan.Kb = a.Kb;
      plan.slots = a.slots;
      const int slot = g_nplans < 32 ? g_nplans++ : (g_next++ % 32);
      g_plans[slot] = plan;
    }
  }
  FParams p;
  p.L = plan.L;
  p.mode = a.mode;
  p.do_select = a.do_select ? 1 : 0;
  p.do_attend = a.do_attend ? 1 : 0;
  p.Nb = a.Nb;
  p.Kb = a.Kb;
  p.T = a.T;
  p.chunk = plan.chunk;
  p.bpc = (a.Kb + plan.C - 1) / plan.C;
  p.slots = a.slots;
  p.nctas_stream = a.nctas_stream;
  p.tiles_per_pair = (a.Nb + kStreamTile - 1) / kStreamTile;
  p.total_tiles = a.pairs * p.tiles_per_pair;
  p.scale = a.scale;
  p.q = a.q;
  p.K = a.K;
  p.V = a.V;
  p.mean_v = a.mean_v;
  p.u = a.u;
  p.xrec = a.xrec;
  p.zpart = a.zpart;
  p.comp_seg = a.comp_seg;
  p.comp = a.comp;
  p.sel_idx = a.sel_idx;
  p.scores = a.scores;
  p.out = a.out;
  p.status = a.status;
  cudaLaunchAttribute attr[2];
  cudaLaunchConfig_t cfg = make_cfg(a.pairs, plan.C, plan.L.total, st, attr, a.pdl);
  void* args[] = {&p};
  return cudaLaunchKernelExC(&cfg, kern, args);
}

}  // namespace compkv
