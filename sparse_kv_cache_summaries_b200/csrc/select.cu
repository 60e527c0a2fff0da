// a1 (second half) + a2. Normalised group score and Top-K selection per (sequence, kv-head), and
// the merge of the Mean-compensation partial sums (CompKV review, Summary: blocks are selected
// up to a token budget by the compensation-aware score; Key claims: Top-K).
//
// Input: the per-block log scores u_{j,h} and the per-segment partials written by the streaming
// kernel. For each kv-head: log Zhat_h = logsumexp over segments, S_j = sum_h exp(u_{j,h} -
// log Zhat_h), and the K_b largest S_j (ties to the lower index) are written in ascending order.
//
// One thread-block cluster of C CTAs per (sequence, kv-head). Rank c keys the blocks of its
// chunk (order-preserving uint32 of S_j; empty blocks get key 0) and keeps its local Top-K_b by
// radix select; rank 0 then gathers the C candidate lists over distributed shared memory (they
// arrive in ascending block order) and selects the global Top-K_b from them. Under the strict
// order (S desc, index asc) the global Top-K_b always lies inside the union of the local ones,
// so the selection is exact. While rank 0 selects, the compensation partials of the kv-head's
// segments are merged, a slice of channels per rank, into one partial per (sequence, kv-head).
#include <cooperative_groups.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace compkv {
namespace {

constexpr int kMaxCluster = 16;

__host__ __device__ inline size_t a16(size_t x) { return (x + 15) & ~static_cast<size_t>(15); }

struct SelLay {
  int chunk, cand_cap, gcap, slots, G;
  size_t keys, cand_key, cand_idx, gkey, gidx, hist, bc, scan, misc, zm, zs, fac, cl, mrg, total;
  __host__ __device__ void build(int chunk_, int Kb, int C, int slots_, int G_) {
    chunk = chunk_;
    slots = slots_;
    G = G_;
    cand_cap = Kb < chunk ? Kb : chunk;
    gcap = cand_cap * C;
    size_t o = 0;
    keys = o;     o = a16(o + sizeof(uint32_t) * chunk);
    cand_key = o; o = a16(o + sizeof(uint32_t) * (cand_cap + 1));
    cand_idx = o; o = a16(o + sizeof(int) * (cand_cap + 1));
    gkey = o;     o = a16(o + sizeof(uint32_t) * (gcap + 1));
    gidx = o;     o = a16(o + sizeof(int) * (gcap + 1));
    hist = o;     o = a16(o + sizeof(uint32_t) * 512);
    bc = o;       o = a16(o + sizeof(uint32_t) * 4);
    scan = o;     o = a16(o + sizeof(int) * (kWarps + 1));
    misc = o;     o = a16(o + sizeof(int) * 64);
    zm = o;       o = a16(o + sizeof(float) * slots * G);
    zs = o;       o = a16(o + sizeof(float) * slots * G);
    fac = o;      o = a16(o + sizeof(float) * slots * G);
    cl = o;       o = a16(o + sizeof(float) * slots * G);
    mrg = o;      o = a16(o + sizeof(float) * kThreads);
    total = o;
  }
};

struct SelParams {
  SelLay L;
  int mode, Nb, Kb, chunk, slots, nctas_stream, tiles_per_pair, total_tiles;
  const float* u;
  const float* zpart;
  const float* comp_seg;
  float* comp;
  int32_t* sel_idx;
  float* scores;
};

// First and last streaming CTA whose tile range touches pair p (see score_stream.cu).
__device__ __forceinline__ int stream_cta_of_tile(long long f, int nctas, int F) {
  return static_cast<int>(((f + 1) * nctas - 1) / F);
}

template <int G, int D>
__global__ void __launch_bounds__(kThreads) select_kernel(const __grid_constant__ SelParams p) {
  extern __shared__ __align__(128) unsigned char sm[];
  const SelLay& L = p.L;
  cg::cluster_group cluster = cg::this_cluster();
  const int C = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  const int pr = blockIdx.x / C;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool compensate = p.mode != COMPKV_MODE_MASS;
  uint32_t* keys = reinterpret_cast<uint32_t*>(sm + L.keys);
  uint32_t* cand_key = reinterpret_cast<uint32_t*>(sm + L.cand_key);
  int* cand_idx = reinterpret_cast<int*>(sm + L.cand_idx);
  uint32_t* gkey = reinterpret_cast<uint32_t*>(sm + L.gkey);
  int* gidx = reinterpret_cast<int*>(sm + L.gidx);
  uint32_t* hist = reinterpret_cast<uint32_t*>(sm + L.hist);
  uint32_t* bc = reinterpret_cast<uint32_t*>(sm + L.bc);
  int* scan = reinterpret_cast<int*>(sm + L.scan);
  int* misc = reinterpret_cast<int*>(sm + L.misc);
  float* logz = reinterpret_cast<float*>(misc + 32);
  float* zm_s = reinterpret_cast<float*>(sm + L.zm);
  float* zs_s = reinterpret_cast<float*>(sm + L.zs);
  float* fac_s = reinterpret_cast<float*>(sm + L.fac);

  const int j0 = rank * p.chunk;
  const int nloc = max(0, min(p.chunk, p.Nb - j0));
  const long long f_first = static_cast<long long>(pr) * p.tiles_per_pair;
  const int c_first = stream_cta_of_tile(f_first, p.nctas_stream, p.total_tiles);
  const int nseg = stream_cta_of_tile(f_first + p.tiles_per_pair - 1, p.nctas_stream, p.total_tiles) - c_first + 1;

  pdl_wait();  // the streaming kernel's outputs are visible from here on
  pdl_launch_dependents();

  // ---- log Zhat per head from the segment partials, and the compensation maxima and sums
  float* cl_s = reinterpret_cast<float*>(sm + L.cl);
  const float* zp = p.zpart + static_cast<size_t>(pr) * p.slots * G * 2;
  const float* cs = p.comp_seg + static_cast<size_t>(pr) * p.slots * G * (D + 2);
  for (int t = tid; t < nseg * G; t += kThreads) {
    zm_s[t] = zp[2 * t];
    zs_s[t] = zp[2 * t + 1];
    if (compensate) {
      fac_s[t] = cs[static_cast<size_t>(t) * (D + 2)];
      cl_s[t] = cs[static_cast<size_t>(t) * (D + 2) + 1];
    }
  }
  __syncthreads();
  if (warp < G) {
    const int h = warp;
    float m = -CUDART_INF_F, s = 0.f;
    for (int t = lane; t < nseg; t += 32) lse_merge(m, s, zm_s[t * G + h], zs_s[t * G + h]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
      const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
      lse_merge(m, s, m2, s2);
    }
    if (lane == 0) logz[h] = (m == -CUDART_INF_F) ? -CUDART_INF_F : m + logf(s);
    if (compensate) {  // common max of the compensation partials, their factors and the sum l
      float M = -CUDART_INF_F;
      for (int t = lane; t < nseg; t += 32) M = fmaxf(M, fac_s[t * G + h]);
      M = warp_max(M);
      float l = 0.f;
      for (int t = lane; t < nseg; t += 32) {
        const float mt = fac_s[t * G + h];
        const float f = (mt == -CUDART_INF_F) ? 0.f : __expf(mt - M);
        fac_s[t * G + h] = f;
        l = fmaf(f, cl_s[t * G + h], l);
      }
      l = warp_sum(l);
      if (rank == 0 && lane == 0) {
        float* out = p.comp + (static_cast<size_t>(pr) * G + h) * (D + 2);
        out[0] = M;
        out[1] = l;
      }
    }
  }
  __syncthreads();

  // ---- keys of this rank's blocks
  const float* up = p.u + (static_cast<size_t>(pr) * p.Nb + j0) * G;
  for (int j = tid; j < nloc; j += kThreads) {
    float S = 0.f;
    if constexpr (G == 4) {
      const float4 v = reinterpret_cast<const float4*>(up)[j];
      S = __expf(v.x - logz[0]) + __expf(v.y - logz[1]) + __expf(v.z - logz[2]) + __expf(v.w - logz[3]);
    } else {
#pragma unroll
      for (int h = 0; h < G; ++h) S += __expf(up[j * G + h] - logz[h]);
    }
    const bool empty = S != S;
    keys[j] = empty ? 0u : score_key(S);
    if (p.scores) p.scores[static_cast<size_t>(pr) * p.Nb + j0 + j] = empty ? 0.f : S;
  }
  __syncthreads();

  // ---- local Top-K_b candidates, in ascending block order
  const int Kb = p.Kb;
  if (tid == 0) misc[0] = 0;
  if (Kb > 0) {
    int ncand;
    if (nloc <= Kb) {
      for (int j = tid; j < nloc; j += kThreads) {
        cand_key[j] = keys[j];
        cand_idx[j] = j0 + j;
      }
      ncand = nloc;
    } else {
      auto kat = [&](int i) { return keys[i]; };
      const RadixCut cut = cta_radix_cut(kat, nloc, Kb, hist, bc);
      ncand = cta_select_ordered(kat, nloc, cut, scan, [&](int i, int pos) {
        cand_key[pos] = keys[i];
        cand_idx[pos] = j0 + i;
      });
    }
    if (tid == 0) misc[0] = ncand;
  }

  cluster.sync();  // #1: every rank's candidates are visible

  if (rank == 0 && Kb > 0) {
    if (tid < C) misc[8 + tid] = *cluster.map_shared_rank(&misc[0], tid);
    __syncthreads();
    if (tid == 0) {
      int off = 0;
      for (int c = 0; c < C; ++c) {
        const int n = misc[8 + c];
        misc[8 + c] = off;
        off += n;
      }
      misc[1] = off;
    }
    __syncthreads();
    const int M = misc[1];
    for (int i = tid; i < M; i += kThreads) {
      int c = 0;
      while (c + 1 < C && misc[8 + c + 1] <= i) ++c;
      const int k = i - misc[8 + c];
      gkey[i] = *cluster.map_shared_rank(&cand_key[k], c);
      gidx[i] = *cluster.map_shared_rank(&cand_idx[k], c);
    }
  }
  if (rank == 0 && Kb > 0) {
    const int M = misc[1];
    int32_t* sel = p.sel_idx + static_cast<size_t>(pr) * Kb;
    if (M <= Kb) {
      for (int i = tid; i < M; i += kThreads) sel[i] = gidx[i];
    } else {
      auto kat = [&](int i) { return gkey[i]; };
      const RadixCut cut = cta_radix_cut(kat, M, Kb, hist, bc);
      cta_select_ordered(kat, M, cut, scan, [&](int i, int pos) { sel[pos] = gidx[i]; });
    }
  }
  if (compensate && (C == 1 || rank != 0)) {
    // merge a slice of the compensation partials' channels: lanes along channels (coalesced),
    // 4 segment groups per slice summed in a fixed order
    float* mrg = reinterpret_cast<float*>(sm + L.mrg);
    const int E = G * D, W = (C == 1) ? 1 : C - 1, wr = (C == 1) ? 0 : rank - 1;
    const int per = (E + W - 1) / W;
    const int e0 = wr * per, e1 = min(E, e0 + per);
    const int ei = tid % 64, sg = tid / 64;
    for (int base = e0; base < e1; base += 64) {
      const int e = base + ei;
      float a = 0.f;
      if (e < e1) {
        const int h = e / D, c = e % D;
#pragma unroll 8
        for (int t = sg; t < nseg; t += 4)
          a = fmaf(fac_s[t * G + h], cs[(static_cast<size_t>(t) * G + h) * (D + 2) + 2 + c], a);
      }
      mrg[sg * 64 + ei] = a;
      __syncthreads();
      if (tid < 64 && base + tid < e1) {
        const int e2 = base + tid;
        p.comp[(static_cast<size_t>(pr) * G + e2 / D) * (D + 2) + 2 + (e2 % D)] =
            ((mrg[tid] + mrg[64 + tid]) + mrg[128 + tid]) + mrg[192 + tid];
      }
      __syncthreads();
    }
  }
  cluster.sync();  // #2: no rank reads another rank's shared memory after this
}

template <int G, int D>
const void* kptr() {
  return reinterpret_cast<const void*>(&select_kernel<G, D>);
}

const void* pick(int D, int G) {
  if (D == 128) {
    switch (G) {
      case 1: return kptr<1, 128>();
      case 2: return kptr<2, 128>();
      case 4: return kptr<4, 128>();
      case 8: return kptr<8, 128>();
    }
  } else {
    switch (G) {
      case 1: return kptr<1, 64>();
      case 2: return kptr<2, 64>();
      case 4: return kptr<4, 64>();
      case 8: return kptr<8, 64>();
    }
  }
  return nullptr;
}

struct Plan {
  const void* kern = nullptr;
  int dev = -1, pairs = 0, Nb = 0, Kb = 0, slots = 0;
  int C = 0, chunk = 0;
  SelLay L;
};
Plan g_plans[32];
int g_nplans = 0, g_next = 0;
std::mutex g_mu;

cudaError_t make_plan(const void* kern, int pairs, int Nb, int Kb, int slots, int G, Plan* out) {
  int dev = 0, sms = 0, optin = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  int C0 = 1;
  while (C0 < kMaxCluster && pairs * (2 * C0) <= 2 * sms && (Nb + 2 * C0 - 1) / (2 * C0) >= 64) C0 *= 2;
  for (int pass = 0; pass < 2; ++pass) {
    for (int C = (pass == 0 ? C0 : C0 / 2); C >= 1 && C <= kMaxCluster; C = (pass == 0 ? C * 2 : C / 2)) {
      const int chunk = (Nb + C - 1) / C;
      SelLay L;
      L.build(chunk, Kb, C, slots, G);
      if (L.total > static_cast<size_t>(optin)) continue;
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(L.total));
      if (e != cudaSuccess) return e;
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e != cudaSuccess) return e;
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(pairs * C, 1, 1);
      cfg.blockDim = dim3(kThreads, 1, 1);
      cfg.dynamicSmemBytes = L.total;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = C;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
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
      if (pass == 0) break;
    }
  }
  return cudaErrorInvalidConfiguration;
}

}  // namespace

cudaError_t launch_select(const SelectArgs& a, cudaStream_t st) {
  const void* kern = pick(a.D, a.G);
  if (!kern) return cudaErrorInvalidValue;
  int dev = 0;
  cudaGetDevice(&dev);
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
      cudaError_t e = make_plan(kern, a.pairs, a.Nb, a.Kb, a.slots, a.G, &plan);
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
  SelParams p;
  p.L = plan.L;
  p.mode = a.mode;
  p.Nb = a.Nb;
  p.Kb = a.Kb;
  p.chunk = plan.chunk;
  p.slots = a.slots;
  p.nctas_stream = a.nctas_stream;
  p.tiles_per_pair = (a.Nb + kStreamTile - 1) / kStreamTile;
  p.total_tiles = a.pairs * p.tiles_per_pair;
  p.u = a.u;
  p.zpart = a.zpart;
  p.comp_seg = a.comp_seg;
  p.comp = a.comp;
  p.sel_idx = a.sel_idx;
  p.scores = a.scores;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.pairs * plan.C, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = plan.L.total;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = plan.C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  void* args[] = {&p};
  return cudaLaunchKernelExC(&cfg, kern, args);
}

}  // namespace compkv
