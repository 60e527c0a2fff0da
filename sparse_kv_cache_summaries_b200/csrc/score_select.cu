// a1 + a2. Compensation-aware block score and Top-K selection (CompKV review, Summary: the
// residual of an omitted block is governed by its attention mass and within-block logit
// variance, Section 3 Eq. 4-7; blocks are scored from compact summaries with a second-order mass
// estimate), plus the Mean-compensation sum over all blocks that the sparse attention consumes.
//
// Design (B200):
//  * One thread-block cluster of C CTAs (C <= 16) per (sequence, kv-head); CTA `rank` owns the
//    contiguous block range [rank*chunk, rank*chunk + nloc). The per-head normaliser Zhat needs
//    every block of the kv-head before any block can be ranked, so the CTAs exchange per-head
//    log-sum-exp partials over distributed shared memory (DSMEM) after one cluster barrier.
//  * The summaries of a tile of 32 blocks (mean key, mean value: bulk copies; grouped variance
//    and count: 4-byte cp.async) land in a 4-stage shared-memory ring tracked by mbarriers, so
//    the two HBM streams (mean keys, mean values) stay in flight while earlier tiles are scored.
//  * Per tile: (1) every warp dots its blocks' mean keys with the G query heads of the kv-head
//    (D/8 lanes per block, 8 channels per lane, transpose-reduce over the lane group); (2) warp h
//    turns head h's 32 dots into lbar, V, the log second-order mass and the log score, updates the
//    Zhat partial and the Mean-compensation running max / sum; (3) all threads add the tile's
//    weighted mean values into per-head accumulators (all G heads per thread, so each mean value
//    is read from shared memory once).
//  * Top-K: each CTA takes its local Top-K_b under (score desc, index asc) by radix select; rank 0
//    gathers the C candidate lists over DSMEM (they arrive in ascending block order) and selects
//    the global Top-K_b from them. The global Top-K_b under a strict order is always inside the
//    union of the local ones, so the result is exact.
//  * Mean-compensation partials of the C CTAs are merged over DSMEM by the non-zero ranks while
//    rank 0 runs the final selection; one merged partial per kv-head goes to the workspace.
#include <cfloat>
#include <mutex>

#include "attend.cuh"
#include "common.cuh"
#include "internal.h"

namespace compkv {
namespace {

constexpr int kTile = 32;    // blocks per pipeline stage (== warp size: warp h owns head h)
constexpr int kMaxCluster = 16;

__host__ __device__ inline size_t al16(size_t x) { return (x + 15) & ~static_cast<size_t>(15); }

// Shared-memory layout, computed identically on host and device.
struct Layout {
  int stages, D, G, r, chunk_cap, cand_cap, gcap;
  size_t mbar, stage0, stage_bytes, off_mu, off_nu, off_var, off_cnt;
  size_t u, dots, ws, sc, zpart, logz, headml, qs, qn, comp, fac, cand_key, cand_idx, gkey, gidx,
      hist, bc, scan, misc, total;

  __host__ __device__ void build(int stages_, int D_, int G_, int r_, int chunk, int Kb, int C) {
    stages = stages_;
    D = D_;
    G = G_;
    r = r_;
    chunk_cap = (chunk + 3) & ~3;
    cand_cap = (Kb < chunk ? Kb : chunk);
    cand_cap = (cand_cap + 3) & ~3;
    gcap = cand_cap * C;
    size_t o = 0;
    mbar = o;
    o = al16(o + 8 * stages);
    off_mu = 0;
    off_nu = al16(off_mu + sizeof(float) * kTile * D);
    off_var = al16(off_nu + sizeof(float) * kTile * D);
    off_cnt = al16(off_var + sizeof(float) * kTile * r);
    stage_bytes = al16(off_cnt + sizeof(int) * kTile);
    stage0 = o;
    o = al16(o + stage_bytes * stages);
    u = o;       o = al16(o + sizeof(float) * G * chunk_cap);
    dots = o;    o = al16(o + sizeof(float) * G * kTile);
    ws = o;      o = al16(o + sizeof(float) * G * kTile);
    sc = o;      o = al16(o + sizeof(float) * 8);
    zpart = o;   o = al16(o + sizeof(float) * 2 * 8);
    logz = o;    o = al16(o + sizeof(float) * 8);
    headml = o;  o = al16(o + sizeof(float) * 2 * 8);
    qs = o;      o = al16(o + sizeof(float) * G * D);
    qn = o;      o = al16(o + sizeof(float) * G * r);
    comp = o;    o = al16(o + sizeof(float) * G * D);
    fac = o;     o = al16(o + sizeof(float) * G * kMaxCluster);
    cand_key = o; o = al16(o + sizeof(uint32_t) * cand_cap);
    cand_idx = o; o = al16(o + sizeof(int) * cand_cap);
    gkey = o;    o = al16(o + sizeof(uint32_t) * gcap);
    gidx = o;    o = al16(o + sizeof(int) * gcap);
    hist = o;    o = al16(o + sizeof(uint32_t) * 256);
    bc = o;      o = al16(o + sizeof(uint32_t) * 4);
    scan = o;    o = al16(o + sizeof(int) * (kWarps + 1));
    misc = o;    o = al16(o + sizeof(int) * (kMaxCluster + 4));
    total = o;
  }
};

struct Params {
  Layout L;
  int mode, Hkv, Nb, Kb, chunk;
  float scale;
  const void* q;
  const float* mean_k;
  const float* var_g;
  const float* mean_v;
  const int32_t* count;
  int32_t* sel_idx;
  float* scores;
  float* comp;
  int32_t* status;
};

template <typename TQ, int D, int G>
__global__ void __launch_bounds__(kThreads, 1) score_select_kernel(const __grid_constant__ Params p) {
  extern __shared__ __align__(128) unsigned char sm[];
  const Layout& L = p.L;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int C = static_cast<int>(cluster_size());
  const int rank = static_cast<int>(cluster_rank());
  const int bk = blockIdx.x / C;                 // b * Hkv + g
  const int j0 = rank * p.chunk;
  const int nloc = max(0, min(p.chunk, p.Nb - j0));
  const int ntiles = (nloc + kTile - 1) / kTile;
  const bool compensate = p.mode != COMPKV_MODE_MASS;
  const int r = L.r;

  uint64_t* mbar = reinterpret_cast<uint64_t*>(sm + L.mbar);
  float* u_s = reinterpret_cast<float*>(sm + L.u);
  float* dot_s = reinterpret_cast<float*>(sm + L.dots);   // [G][kTile]
  float* ws_s = reinterpret_cast<float*>(sm + L.ws);      // [kTile][G]
  float* sc_s = reinterpret_cast<float*>(sm + L.sc);
  float* zpart_s = reinterpret_cast<float*>(sm + L.zpart);
  float* logz_s = reinterpret_cast<float*>(sm + L.logz);
  float* headml_s = reinterpret_cast<float*>(sm + L.headml);
  float* q_s = reinterpret_cast<float*>(sm + L.qs);
  float* qn_s = reinterpret_cast<float*>(sm + L.qn);
  float* comp_s = reinterpret_cast<float*>(sm + L.comp);
  float* fac_s = reinterpret_cast<float*>(sm + L.fac);
  uint32_t* cand_key = reinterpret_cast<uint32_t*>(sm + L.cand_key);
  int* cand_idx = reinterpret_cast<int*>(sm + L.cand_idx);
  uint32_t* gkey = reinterpret_cast<uint32_t*>(sm + L.gkey);
  int* gidx = reinterpret_cast<int*>(sm + L.gidx);
  uint32_t* hist = reinterpret_cast<uint32_t*>(sm + L.hist);
  uint32_t* bc = reinterpret_cast<uint32_t*>(sm + L.bc);
  int* scan = reinterpret_cast<int*>(sm + L.scan);
  int* misc = reinterpret_cast<int*>(sm + L.misc);

  const float* mk_base = p.mean_k + static_cast<size_t>(bk) * p.Nb * D;
  const float* mv_base = p.mean_v + static_cast<size_t>(bk) * p.Nb * D;
  const float* vg_base = p.var_g + static_cast<size_t>(bk) * p.Nb * r;
  const int32_t* cn_base = p.count + static_cast<size_t>(bk) * p.Nb;
  const uint64_t policy = l2_evict_first_policy();

  // Issue the loads of local tile `t` into its stage. All threads take part (cp.async of the
  // grouped variances and counts, then one noinc arrival each); thread 0 adds the bulk copies.
  auto issue = [&](int t) {
    const int st = t % L.stages;
    unsigned char* sb = sm + L.stage0 + L.stage_bytes * st;
    const int jt0 = j0 + t * kTile;
    const int tn = min(kTile, nloc - t * kTile);
    float* var_d = reinterpret_cast<float*>(sb + L.off_var);
    int* cnt_d = reinterpret_cast<int*>(sb + L.off_cnt);
    for (int i = tid; i < tn * r; i += kThreads) cp_async4(var_d + i, vg_base + static_cast<size_t>(jt0) * r + i);
    for (int i = tid; i < tn; i += kThreads) cp_async4(cnt_d + i, cn_base + jt0 + i);
    if (tid == 0) {
      const uint32_t bytes = static_cast<uint32_t>(tn) * D * sizeof(float);
      mbar_arrive_expect_tx(&mbar[st], compensate ? 2 * bytes : bytes);
      bulk_g2s_stream(sb + L.off_mu, mk_base + static_cast<size_t>(jt0) * D, bytes, &mbar[st], policy);
      if (compensate)
        bulk_g2s_stream(sb + L.off_nu, mv_base + static_cast<size_t>(jt0) * D, bytes, &mbar[st], policy);
    }
    cp_async_arrive(&mbar[st]);
  };

  if (tid == 0) {
    for (int s = 0; s < L.stages; ++s) mbar_init(&mbar[s], kThreads + 1);
    mbar_init_fence();
  }
  // query heads of this kv-head -> fp32 smem; s^2 |q_{h,C_g}|^2 per group
  for (int i = tid; i < G * D; i += kThreads) {
    const TQ* qp = static_cast<const TQ*>(p.q) + static_cast<size_t>(bk) * G * D;
    q_s[i] = to_float(qp[i]);
  }
  __syncthreads();
  for (int t = 0; t < min(ntiles, L.stages - 1); ++t) issue(t);
  pdl_launch_dependents();
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

  // phase-1 lane geometry: LPB lanes per block, 8 channels per lane (two float4)
  constexpr int LPB = D / 8;
  constexpr int BPP = 32 / LPB;
  constexpr int LPH = LPB / G;  // lanes per head after the transpose-reduce
  const int li = lane % LPB, bsub = lane / LPB;
  float qreg[G][8];
#pragma unroll
  for (int h = 0; h < G; ++h) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      qreg[h][e] = q_s[h * D + li * 4 + e];
      qreg[h][4 + e] = q_s[h * D + D / 2 + li * 4 + e];
    }
  }
  // phase-3 geometry: 4 channels per thread, NJS block subsets
  constexpr int NC4 = D / 4;
  constexpr int NJS = kThreads / NC4;
  const int c4 = tid % NC4, js = tid / NC4;
  float acc[G][4];
#pragma unroll
  for (int h = 0; h < G; ++h) acc[h][0] = acc[h][1] = acc[h][2] = acc[h][3] = 0.f;
  // per-head running state, held by warp h (all lanes equal for m/l; per-lane for Zhat)
  float m_r = -CUDART_INF_F, l_r = 0.f, zmax_r = -CUDART_INF_F, zsum_r = 0.f;
  bool ok = true;
  int issued = min(ntiles, L.stages - 1), waited = ntiles;

#pragma unroll 1
  for (int t = 0; t < ntiles; ++t) {
    const int st = t % L.stages;
    unsigned char* sb = sm + L.stage0 + L.stage_bytes * st;
    const float* mu_t = reinterpret_cast<const float*>(sb + L.off_mu);
    const float* nu_t = reinterpret_cast<const float*>(sb + L.off_nu);
    const float* var_t = reinterpret_cast<const float*>(sb + L.off_var);
    const int* cnt_t = reinterpret_cast<const int*>(sb + L.off_cnt);
    const int tn = min(kTile, nloc - t * kTile);
    const bool got = mbar_wait(&mbar[st], (t / L.stages) & 1, p.status);

    // (1) dots q_h . mu_j
#pragma unroll
    for (int pass = 0; pass < kTile / (kWarps * BPP); ++pass) {
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
      if ((li % LPH) == 0 && jt < tn) dot_s[(li / LPH) * kTile + jt] = v[0];
    }
    ok = __syncthreads_and(got) != 0;
    if (!ok) {                      // give up on the data (uniform over the CTA); drain below
      waited = t;
      break;
    }
    if (t + L.stages - 1 < ntiles) {
      issue(t + L.stages - 1);
      ++issued;
    }

    // (2) per-head scalars, warp h, lane = block in tile
    if (warp < G) {
      const int h = warp, jt = lane;
      float x = -CUDART_INF_F, lm = -CUDART_INF_F;
      if (jt < tn) {
        const int n = cnt_t[jt];
        const float lbar = p.scale * dot_s[h * kTile + jt];
        float vh = 0.f;
        for (int g = 0; g < r; ++g) vh = fmaf(qn_s[h * r + g], var_t[jt * r + g], vh);
        float uu;
        if (n > 0) {
          x = lbar + logf(static_cast<float>(n));
          lm = x + log1pf(0.5f * vh);
          uu = (p.mode == COMPKV_MODE_COMPKV) ? lm + logf(0.5f * vh) : lm;
        } else {
          uu = __int_as_float(0x7fffffff);  // NaN marks an empty block
        }
        u_s[h * L.chunk_cap + t * kTile + jt] = uu;
      }
      if (lm != -CUDART_INF_F) {
        const float nm = fmaxf(zmax_r, lm);
        zsum_r = (zmax_r == -CUDART_INF_F ? 0.f : zsum_r * expf(zmax_r - nm)) + expf(lm - nm);
        zmax_r = nm;
      }
      if (compensate) {
        const float m_new = fmaxf(m_r, warp_max(x));
        const float w = (x == -CUDART_INF_F) ? 0.f : __expf(x - m_new);
        const float sc = (m_r == -CUDART_INF_F) ? 0.f : __expf(m_r - m_new);
        ws_s[jt * G + h] = w;
        l_r = l_r * sc + warp_sum(w);
        m_r = m_new;
        if (lane == 0) sc_s[h] = sc;
      }
    }
    __syncthreads();

    // (3) Mean-compensation accumulators: acc_h += w_{h,j} nu_j, 4 channels x G heads per thread
    if (compensate) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float sc = sc_s[h];
        acc[h][0] *= sc; acc[h][1] *= sc; acc[h][2] *= sc; acc[h][3] *= sc;
      }
      for (int jt = js; jt < tn; jt += NJS) {
        const float4 nv = reinterpret_cast<const float4*>(nu_t + jt * D)[c4];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float w = ws_s[jt * G + h];
          acc[h][0] = fmaf(w, nv.x, acc[h][0]);
          acc[h][1] = fmaf(w, nv.y, acc[h][1]);
          acc[h][2] = fmaf(w, nv.z, acc[h][2]);
          acc[h][3] = fmaf(w, nv.w, acc[h][3]);
        }
      }
    }
  }
  if (!ok) {  // a wait gave up: wait (bounded) for the copies still in flight before reuse
    for (int t = waited; t < issued; ++t) mbar_wait(&mbar[t % L.stages], (t / L.stages) & 1, nullptr);
  }
  __syncthreads();  // every stage is consumed: the ring is free for scratch below

  // ---------------------------------------------------------------- per-CTA partials
  if (warp < G) {
    float zm = zmax_r, zs = zsum_r;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float m2 = __shfl_xor_sync(0xffffffffu, zm, o);
      const float s2 = __shfl_xor_sync(0xffffffffu, zs, o);
      lse_merge(zm, zs, m2, s2);
    }
    if (lane == 0) {
      zpart_s[2 * warp] = zm;
      zpart_s[2 * warp + 1] = zs;
      headml_s[2 * warp] = m_r;
      headml_s[2 * warp + 1] = l_r;
    }
  }
  if (compensate) {
    float* red = reinterpret_cast<float*>(sm + L.stage0);  // [NJS][G][D]
#pragma unroll
    for (int h = 0; h < G; ++h)
      reinterpret_cast<float4*>(red + (js * G + h) * D)[c4] =
          make_float4(acc[h][0], acc[h][1], acc[h][2], acc[h][3]);
    __syncthreads();
    for (int i = tid; i < G * D; i += kThreads) {
      float s = 0.f;
      for (int k = 0; k < NJS; ++k) s += red[k * G * D + i];
      comp_s[i] = s;
    }
  }
  cluster_sync();  // #1: Zhat partials and compensation partials of every rank are visible

  if (tid < G) {
    float zm = -CUDART_INF_F, zs = 0.f;
    for (int c = 0; c < C; ++c) {
      const float m2 = ld_dsmem_f32(dsmem_addr(&zpart_s[2 * tid], c));
      const float s2 = ld_dsmem_f32(dsmem_addr(&zpart_s[2 * tid + 1], c));
      lse_merge(zm, zs, m2, s2);
    }
    logz_s[tid] = (zm == -CUDART_INF_F) ? -CUDART_INF_F : zm + logf(zs);
  }
  __syncthreads();

  // ---------------------------------------------------------------- keys and local Top-K
  uint32_t* key_s = reinterpret_cast<uint32_t*>(u_s);   // keys overwrite head-0 scores in place
  for (int j = tid; j < nloc; j += kThreads) {
    float S = 0.f;
#pragma unroll
    for (int h = 0; h < G; ++h) S += expf(u_s[h * L.chunk_cap + j] - logz_s[h]);
    const bool empty = S != S;
    key_s[j] = empty ? 0u : score_key(S);
    if (p.scores) p.scores[static_cast<size_t>(bk) * p.Nb + j0 + j] = empty ? 0.f : S;
  }
  __syncthreads();
  const int Kb = p.Kb;
  int ncand = 0;
  if (Kb > 0) {
    if (nloc <= Kb) {
      for (int j = tid; j < nloc; j += kThreads) {
        cand_key[j] = key_s[j];
        cand_idx[j] = j0 + j;
      }
      ncand = nloc;
    } else {
      uint32_t tau;
      int ngt;
      auto kat = [&](int i) { return key_s[i]; };
      cta_radix_select(kat, nloc, Kb, hist, bc, tau, ngt);
      ncand = cta_select_ordered(kat, nloc, Kb, tau, ngt, scan, [&](int i, int pos) {
        cand_key[pos] = key_s[i];
        cand_idx[pos] = j0 + i;
      });
    }
  }
  if (tid == 0) misc[0] = ncand;
  cluster_sync();  // #2: candidates of every rank are visible

  if (rank == 0 && Kb > 0) {
    if (tid == 0) {
      int off = 0;
      for (int c = 0; c < C; ++c) {
        misc[4 + c] = off;
        off += static_cast<int>(ld_dsmem_u32(dsmem_addr(&misc[0], c)));
      }
      misc[1] = off;
    }
    __syncthreads();
    const int M = misc[1];
    for (int c = 0; c < C; ++c) {
      const int off = misc[4 + c];
      const int nc = (c + 1 < C ? misc[4 + c + 1] : M) - off;
      for (int i = tid; i < nc; i += kThreads) {
        gkey[off + i] = ld_dsmem_u32(dsmem_addr(&cand_key[i], c));
        gidx[off + i] = static_cast<int>(ld_dsmem_u32(dsmem_addr(&cand_idx[i], c)));
      }
    }
  }
  if (compensate && (C == 1 || rank != 0)) {
    const int workers = (C == 1) ? 1 : C - 1;
    const int wrank = (C == 1) ? 0 : rank - 1;
    if (tid < G * C) {
      const int h = tid / C, c = tid % C;
      fac_s[h * kMaxCluster + c] = ld_dsmem_f32(dsmem_addr(&headml_s[2 * h], c));
    }
    __syncthreads();
    float* out = p.comp + static_cast<size_t>(bk) * G * (D + 2);
    for (int e = wrank * kThreads + tid; e < G * D; e += workers * kThreads) {
      const int h = e / D, c = e % D;
      float M = -CUDART_INF_F;
      for (int k = 0; k < C; ++k) M = fmaxf(M, fac_s[h * kMaxCluster + k]);
      float a = 0.f, l = 0.f;
      for (int k = 0; k < C; ++k) {
        const float mk = fac_s[h * kMaxCluster + k];
        if (mk == -CUDART_INF_F) continue;
        const float f = __expf(mk - M);
        a = fmaf(f, ld_dsmem_f32(dsmem_addr(&comp_s[h * D + c], k)), a);
        if (c == 0) l = fmaf(f, ld_dsmem_f32(dsmem_addr(&headml_s[2 * h + 1], k)), l);
      }
      out[h * (D + 2) + 2 + c] = a;
      if (c == 0) {
        out[h * (D + 2)] = M;
        out[h * (D + 2) + 1] = l;
      }
    }
  }
  cluster_sync();  // #3: no rank reads another rank's shared memory after this point

  if (rank == 0 && Kb > 0) {
    const int M = misc[1];
    int32_t* sel = p.sel_idx + static_cast<size_t>(bk) * Kb;
    if (M <= Kb) {
      for (int i = tid; i < M; i += kThreads) sel[i] = gidx[i];
    } else {
      uint32_t tau;
      int ngt;
      auto kat = [&](int i) { return gkey[i]; };
      cta_radix_select(kat, M, Kb, hist, bc, tau, ngt);
      cta_select_ordered(kat, M, Kb, tau, ngt, scan, [&](int i, int pos) { sel[pos] = gidx[i]; });
    }
  }
}

template <typename TQ, int D, int G>
const void* kernel_ptr() {
  return reinterpret_cast<const void*>(&score_select_kernel<TQ, D, G>);
}

const void* pick_kernel(bool bf16, int D, int G) {
  if (bf16) {
    if (D == 128) {
      switch (G) {
        case 1: return kernel_ptr<uint16_t, 128, 1>();
        case 2: return kernel_ptr<uint16_t, 128, 2>();
        case 4: return kernel_ptr<uint16_t, 128, 4>();
        case 8: return kernel_ptr<uint16_t, 128, 8>();
      }
    } else {
      switch (G) {
        case 1: return kernel_ptr<uint16_t, 64, 1>();
        case 2: return kernel_ptr<uint16_t, 64, 2>();
        case 4: return kernel_ptr<uint16_t, 64, 4>();
        case 8: return kernel_ptr<uint16_t, 64, 8>();
      }
    }
  } else {
    if (D == 128) {
      switch (G) {
        case 1: return kernel_ptr<float, 128, 1>();
        case 2: return kernel_ptr<float, 128, 2>();
        case 4: return kernel_ptr<float, 128, 4>();
        case 8: return kernel_ptr<float, 128, 8>();
      }
    } else {
      switch (G) {
        case 1: return kernel_ptr<float, 64, 1>();
        case 2: return kernel_ptr<float, 64, 2>();
        case 4: return kernel_ptr<float, 64, 4>();
        case 8: return kernel_ptr<float, 64, 8>();
      }
    }
  }
  return nullptr;
}

struct Plan {
  int C = 0, stages = 0, chunk = 0;
  Layout L;
};

// Largest power-of-two cluster (<= 16) that keeps about one CTA per SM over all kv-heads and at
// least two tiles per CTA, then the deepest pipeline (4..2 stages) whose shared memory fits; a
// cluster the device cannot co-schedule at that size steps down (or up, when the per-CTA block
// range does not fit in shared memory).
cudaError_t make_plan(const void* kern, int B, int Hkv, int G, int D, int r, int Nb, int Kb, Plan* out) {
  int dev = 0, sms = 0, optin = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  const int pairs = B * Hkv;
  int C0 = 1;
  while (C0 < kMaxCluster && pairs * (2 * C0) <= sms + sms / 8 && (Nb + 2 * C0 - 1) / (2 * C0) >= 2 * kTile)
    C0 *= 2;
  for (int pass = 0; pass < 2; ++pass) {
    // pass 0: C0 and larger (shared-memory fit), pass 1: smaller than C0
    for (int C = (pass == 0 ? C0 : C0 / 2); C >= 1 && C <= kMaxCluster; C = (pass == 0 ? C * 2 : C / 2)) {
      const int chunk = (Nb + C - 1) / C;
      for (int stages = 4; stages >= 2; --stages) {
        Layout L;
        L.build(stages, D, G, r, chunk, Kb, C);
        if (L.total > static_cast<size_t>(optin)) continue;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(L.total));
        if (e != cudaSuccess) return e;
        if (C > 8) {
          e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
          if (e != cudaSuccess) return e;
        }
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
        int nclusters = 0;
        e = cudaOccupancyMaxActiveClusters(&nclusters, kern, &cfg);
        if (e != cudaSuccess) {
          cudaGetLastError();
          nclusters = 0;
        }
        if (nclusters >= 1) {
          out->C = C;
          out->stages = stages;
          out->chunk = chunk;
          out->L = L;
          return cudaSuccess;
        }
        break;  // fewer stages will not make the cluster schedulable; try another size
      }
    }
  }
  return cudaErrorInvalidConfiguration;
}

struct PlanKey {
  const void* kern;
  int dev, B, Hkv, r, Nb, Kb;
  bool operator==(const PlanKey& o) const {
    return kern == o.kern && dev == o.dev && B == o.B && Hkv == o.Hkv && r == o.r && Nb == o.Nb && Kb == o.Kb;
  }
};

constexpr int kPlanCache = 32;
PlanKey g_keys[kPlanCache];
Plan g_plans[kPlanCache];
int g_nplans = 0, g_next = 0;
std::mutex g_plan_mu;

cudaError_t get_plan(const void* kern, const ScoreSelectArgs& a, Plan* out) {
  int dev = 0;
  cudaGetDevice(&dev);
  const PlanKey key{kern, dev, a.B, a.Hkv, a.r, a.Nb, a.Kb};
  std::lock_guard<std::mutex> lock(g_plan_mu);
  for (int i = 0; i < g_nplans; ++i)
    if (g_keys[i] == key) {
      *out = g_plans[i];
      return cudaSuccess;
    }
  Plan p;
  cudaError_t e = make_plan(kern, a.B, a.Hkv, a.G, a.D, a.r, a.Nb, a.Kb, &p);
  if (e != cudaSuccess) return e;
  const int slot = g_nplans < kPlanCache ? g_nplans++ : (g_next++ % kPlanCache);
  g_keys[slot] = key;
  g_plans[slot] = p;
  *out = p;
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_score_select(const ScoreSelectArgs& a, cudaStream_t st) {
  const void* kern = pick_kernel(a.bf16, a.D, a.G);
  if (kern == nullptr) return cudaErrorInvalidValue;
  Plan plan;
  cudaError_t e = get_plan(kern, a, &plan);
  if (e != cudaSuccess) return e;
  Params p;
  p.L = plan.L;
  p.mode = a.mode;
  p.Hkv = a.Hkv;
  p.Nb = a.Nb;
  p.Kb = a.Kb;
  p.chunk = plan.chunk;
  p.scale = a.scale;
  p.q = a.q;
  p.mean_k = a.mean_k;
  p.var_g = a.var_g;
  p.mean_v = a.mean_v;
  p.count = a.count;
  p.sel_idx = a.sel_idx;
  p.scores = a.scores;
  p.comp = a.comp;
  p.status = a.status;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.B * a.Hkv * plan.C, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = plan.L.total;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = plan.C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  void* args[] = {&p};
  return cudaLaunchKernelExC(&cfg, kern, args);
}

int score_select_cluster(int B, int Hkv, int G, int D, int r, int Nb, int Kb, bool bf16, size_t* smem_bytes) {
  const void* kern = pick_kernel(bf16, D, G);
  if (!kern) return -1;
  ScoreSelectArgs a = {};
  a.B = B;
  a.Hkv = Hkv;
  a.G = G;
  a.D = D;
  a.r = r;
  a.Nb = Nb;
  a.Kb = Kb;
  Plan plan;
  if (get_plan(kern, a, &plan) != cudaSuccess) return -1;
  if (smem_bytes) *smem_bytes = plan.L.total;
  return plan.C;
}

}  // namespace compkv
