// a3. Exact attention over the selected blocks plus Mean compensation of every omitted block, in
// one softmax (CompKV abstract: exact attention over a selected subset with compensation of the
// omitted tail; review, Summary: "omitted blocks contribute their block-mean logit").
//
// The score kernel already accumulated, per query head, the compensation term of EVERY block
// (logit lbar_j + log n_j, value nu_j) while it streamed the summaries. This kernel therefore
// only touches the K_b selected blocks: it adds their exact token terms and removes their
// compensation terms. Both are taken relative to the running max of the exact logits, which is
// at least the block-mean logit of every processed block, so no term overflows; and because a
// block's compensation mass never exceeds its exact mass (Jensen), the removal cancels at most
// the magnitude it adds, keeping the rounding error relative to the final denominator.
//
// One cluster of NS CTAs per (sequence, kv-head); CTA `rank` takes selection slots
// [rank*bpc, rank*bpc + bpc), in rounds of up to kRound blocks whose K and V rows are bulk-copied
// into shared memory (n_j rows each, so a partial last block never reads past the cache). Split
// partials (m, l, acc) are merged by rank 0 over DSMEM together with the compensation partial.
// Launched with programmatic dependent launch after the score kernel: the q prologue runs before
// griddepcontrol.wait, everything that reads the selection after it.
#include <cooperative_groups.h>

#include "attend.cuh"
#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace compkv {
namespace {

constexpr int kRound = 8;   // blocks per shared-memory round
constexpr int kRows = kRound * kBlockTokens;

struct SParams {
  int mode, Hkv, T, Nb, Kb, bpc;
  float scale;
  const void* q;
  const void* K;
  const void* V;
  const float* mean_v;
  const int32_t* sel_idx;
  const float* comp;
  const float* xrec;
  float* out;
  int32_t* status;
};

template <typename T, int D, int G>
struct SLayout {
  static constexpr size_t kv_bytes = sizeof(T) * kRows * D;
  static constexpr size_t off_k = 0;
  static constexpr size_t off_v = off_k + kv_bytes;
  static constexpr size_t off_nu = off_v + kv_bytes;                     // [kRound][D] fp32
  static constexpr size_t off_lg = off_nu + sizeof(float) * kRound * D;  // [G][kRows]
  static constexpr size_t off_p = off_lg + sizeof(float) * G * kRows;    // [kRows][G]
  static constexpr size_t off_q = off_p + sizeof(float) * G * kRows;     // [G][D]
  static constexpr size_t off_red = off_q + sizeof(float) * G * D;       // [kSub][G][D]
  static constexpr size_t off_acc = off_red + sizeof(float) * PV<T, D, G>::kSub * G * D;  // [G][D]
  static constexpr size_t off_cp = off_acc + sizeof(float) * G * D;      // [G][D+2] compensation
  static constexpr size_t off_ml = off_cp + sizeof(float) * G * (D + 2); // [G][2]
  static constexpr size_t off_blk = off_ml + sizeof(float) * 2 * 8;      // j, n
  static constexpr size_t off_xr = off_blk + sizeof(int) * 2 * kRound;   // [kRound][G] x
  static constexpr size_t off_pw = off_xr + sizeof(float) * G * kRound;  // [G][kRound]
  static constexpr size_t off_sc = off_pw + sizeof(float) * G * kRound;  // [G]
  static constexpr size_t off_fac = off_sc + sizeof(float) * 8;          // [G][17] x 2
  static constexpr size_t off_mbar = (off_fac + sizeof(float) * G * 34 + 15) & ~size_t(15);
  static constexpr size_t total = off_mbar + 16;
};

template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreads) sparse_decode_kernel(const __grid_constant__ SParams p) {
  using LY = SLayout<T, D, G>;
  using RG = RowGeom<T, D>;
  using PVt = PV<T, D, G>;
  constexpr int EPV = RG::kEpv, VEC = PVt::kVec;
  constexpr int XS = xrec_stride(G);
  extern __shared__ __align__(128) unsigned char sm[];
  T* kbuf = reinterpret_cast<T*>(sm + LY::off_k);
  T* vbuf = reinterpret_cast<T*>(sm + LY::off_v);
  float* nu_s = reinterpret_cast<float*>(sm + LY::off_nu);
  float* lg = reinterpret_cast<float*>(sm + LY::off_lg);
  float* pT = reinterpret_cast<float*>(sm + LY::off_p);
  float* q_s = reinterpret_cast<float*>(sm + LY::off_q);
  float* red = reinterpret_cast<float*>(sm + LY::off_red);
  float* acc_s = reinterpret_cast<float*>(sm + LY::off_acc);
  float* cp_s = reinterpret_cast<float*>(sm + LY::off_cp);
  float* ml_s = reinterpret_cast<float*>(sm + LY::off_ml);
  int* blk_j = reinterpret_cast<int*>(sm + LY::off_blk);
  int* blk_n = blk_j + kRound;
  float* xr_s = reinterpret_cast<float*>(sm + LY::off_xr);
  float* pw_s = reinterpret_cast<float*>(sm + LY::off_pw);
  float* sc_s = reinterpret_cast<float*>(sm + LY::off_sc);
  float* fac_s = reinterpret_cast<float*>(sm + LY::off_fac);
  uint64_t* mbar = reinterpret_cast<uint64_t*>(sm + LY::off_mbar);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  cg::cluster_group cluster = cg::this_cluster();
  const int NS = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  const int bk = blockIdx.x / NS;
  const bool compensate = p.mode != COMPKV_MODE_MASS;

  // ---- prologue: inputs written before the select kernel started
  if (tid == 0) {
    mbar_init(mbar, 1);
    mbar_init_fence();
  }
  {
    const T* qp = static_cast<const T*>(p.q) + static_cast<size_t>(bk) * G * D;
    for (int i = tid; i < G * D; i += kThreads) q_s[i] = to_float(qp[i]);
  }
  __syncthreads();
  const int li = lane % RG::kLpr;
  float qr[G][EPV];
  load_q_regs<T, D, G>(q_s, li, qr);
  const int cv = tid % PVt::kCols, sub = tid / PVt::kCols;
  float acc[G][VEC];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < VEC; ++e) acc[h][e] = 0.f;
  float m_run = -CUDART_INF_F, l_run = 0.f;  // warp h's running state for head h

  pdl_wait();  // selection, records and compensation partial are visible from here on

  if (rank == 0 && compensate) {  // prefetch the compensation partial for the merge
    const float* cp = p.comp + static_cast<size_t>(bk) * G * (D + 2);
    for (int i = tid; i < G * (D + 2); i += kThreads) cp_s[i] = cp[i];
  }
  const T* Kbase = static_cast<const T*>(p.K) + static_cast<size_t>(bk) * p.T * D;
  const T* Vbase = static_cast<const T*>(p.V) + static_cast<size_t>(bk) * p.T * D;
  const float* NUbase = p.mean_v + static_cast<size_t>(bk) * p.Nb * D;
  const float* XRbase = p.xrec + static_cast<size_t>(bk) * p.Nb * XS;
  const int s0 = rank * p.bpc;
  const int s1 = min(p.Kb, s0 + p.bpc);
  uint32_t phase = 0;
#pragma unroll 1
  for (int rs0 = s0; rs0 < s1; rs0 += kRound) {
    const int nr = min(kRound, s1 - rs0);
    if (tid < kRound) {
      int j = -1;
      if (tid < nr) {
        j = p.sel_idx[static_cast<size_t>(bk) * p.Kb + rs0 + tid];
        if (j < 0 || j >= p.Nb) j = -1;
      }
      blk_j[tid] = j;
    }
    __syncthreads();
    // K and V rows up to the cache capacity (the block's token count arrives with its record)
    if (tid == 0) {
      uint32_t bytes = 0;
      for (int s = 0; s < nr; ++s) {
        const int j = blk_j[s];
        if (j < 0) continue;
        const int rows = min(kBlockTokens, p.T - j * kBlockTokens);
        bytes += 2u * rows * D * sizeof(T) + (compensate ? D * sizeof(float) : 0u);
      }
      mbar_arrive_expect_tx(mbar, bytes);
      for (int s = 0; s < nr; ++s) {
        const int j = blk_j[s];
        if (j < 0) continue;
        const int rows = min(kBlockTokens, p.T - j * kBlockTokens);
        const size_t off = static_cast<size_t>(j) * kBlockTokens * D;
        bulk_g2s(kbuf + s * kBlockTokens * D, Kbase + off, rows * D * sizeof(T), mbar);
        bulk_g2s(vbuf + s * kBlockTokens * D, Vbase + off, rows * D * sizeof(T), mbar);
        if (compensate) bulk_g2s(nu_s + s * D, NUbase + static_cast<size_t>(j) * D, D * sizeof(float), mbar);
      }
    }
    // records: x_h and the token count of each selected block
    if (tid < nr * (G + 1)) {
      const int s = tid / (G + 1), e = tid % (G + 1);
      const int j = blk_j[s];
      const float v = (j >= 0) ? XRbase[static_cast<size_t>(j) * XS + e] : 0.f;
      if (e < G) xr_s[s * G + e] = (j >= 0) ? v : -CUDART_INF_F;
      else blk_n[s] = (j >= 0) ? max(0, min(__float_as_int(v), min(kBlockTokens, p.T - j * kBlockTokens))) : 0;
    }
    if (tid >= nr && tid < kRound) blk_n[tid] = 0;
    const bool got = mbar_wait(mbar, phase, p.status);
    __syncthreads();  // records visible
    // V rows past a block's token count: zero them (their weight is 0, but 0 * NaN is not)
    for (int s = 0; s < nr; ++s) {
      const int n = blk_n[s];
      if (n < kBlockTokens) {
        T* vrow = vbuf + (static_cast<size_t>(s) * kBlockTokens + n) * D;
        for (int e = tid; e < (kBlockTokens - n) * D; e += kThreads) vrow[e] = T(0);
      }
    }
    fence_proxy_async();  // the next round's copies may land on these rows
    if (__syncthreads_and(got) == 0) {  // uniform: drain (bounded) and stop
      mbar_wait(mbar, phase, nullptr);
      break;
    }
    phase ^= 1;

    // logits of all rows of the round (rows past n_j are -inf)
    const int R = nr * kBlockTokens;
    const int Rpad = (R + kWarps * RG::kRpl - 1) / (kWarps * RG::kRpl) * (kWarps * RG::kRpl);
    tile_logits<T, D, G>(kbuf, Rpad, qr, p.scale, lg, kRows, [&](int row) {
      return row < R && (row % kBlockTokens) < blk_n[row / kBlockTokens];
    });
    __syncthreads();
    // softmax update, warp h for head h; compensation terms of the selected blocks removed
    if (warp < G) {
      const int h = warp;
      float mx = -CUDART_INF_F;
      for (int row = lane; row < R; row += 32) mx = fmaxf(mx, lg[h * kRows + row]);
      mx = warp_max(mx);
      const float m_new = fmaxf(m_run, mx);
      float ls = 0.f;
      for (int row = lane; row < R; row += 32) {
        const float x = lg[h * kRows + row];
        const float w = (x == -CUDART_INF_F) ? 0.f : __expf(x - m_new);
        pT[row * G + h] = w;
        ls += w;
      }
      ls = warp_sum(ls);
      float pw = 0.f;
      if (compensate && lane < nr) {
        const float xj = xr_s[lane * G + h];
        pw = (xj == -CUDART_INF_F) ? 0.f : __expf(xj - m_new);
      }
      if (lane < kRound) pw_s[h * kRound + lane] = pw;
      const float pws = warp_sum(pw);
      const float sc = (m_run == -CUDART_INF_F) ? 0.f : __expf(m_run - m_new);
      l_run = l_run * sc + ls - pws;
      m_run = m_new;
      if (lane == 0) sc_s[h] = sc;
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float sc = sc_s[h];
#pragma unroll
      for (int e = 0; e < VEC; ++e) acc[h][e] *= sc;
    }
    PVt::accumulate(vbuf, pT, R, sub, cv, acc);
    if (compensate && sub == 0) {
      for (int s = 0; s < nr; ++s) {
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          const float nv = nu_s[s * D + cv * VEC + e];
#pragma unroll
          for (int h = 0; h < G; ++h) acc[h][e] = fmaf(-pw_s[h * kRound + s], nv, acc[h][e]);
        }
      }
    }
    __syncthreads();  // buffers are reused by the next round
  }

  // ---- split partial -> shared memory
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < VEC; ++e) red[(sub * G + h) * D + cv * VEC + e] = acc[h][e];
  if (warp < G && lane == 0) {
    ml_s[2 * warp] = m_run;
    ml_s[2 * warp + 1] = l_run;
  }
  __syncthreads();
  for (int i = tid; i < G * D; i += kThreads) {
    float s = 0.f;
    for (int k = 0; k < PVt::kSub; ++k) s += red[k * G * D + i];
    acc_s[i] = s;
  }
  cluster.sync();  // #1: every split's partial is visible

  if (rank == 0) {
    // per head: common max over the splits and the compensation partial, factors, 1/denominator
    if (tid < G * NS) {
      const int h = tid / NS, s = tid % NS;
      const float* rml = cluster.map_shared_rank(ml_s, s);
      fac_s[h * 17 + s] = rml[2 * h];
      fac_s[G * 17 + h * 17 + s] = rml[2 * h + 1];
    }
    __syncthreads();
    if (tid < G) {
      const int h = tid;
      const float cm = compensate ? cp_s[h * (D + 2)] : -CUDART_INF_F;
      float M = cm;
      for (int s = 0; s < NS; ++s) M = fmaxf(M, fac_s[h * 17 + s]);
      float den = 0.f;
      if (cm != -CUDART_INF_F) {
        const float f = __expf(cm - M);
        fac_s[h * 17 + 16] = f;
        den = f * cp_s[h * (D + 2) + 1];
      } else {
        fac_s[h * 17 + 16] = 0.f;
      }
      for (int s = 0; s < NS; ++s) {
        const float ms = fac_s[h * 17 + s];
        const float f = (ms == -CUDART_INF_F) ? 0.f : __expf(ms - M);
        fac_s[h * 17 + s] = f;
        den = fmaf(f, fac_s[G * 17 + h * 17 + s], den);
      }
      sc_s[h] = den > 0.f ? 1.f / den : 0.f;
    }
    __syncthreads();
    float* o = p.out + static_cast<size_t>(bk) * G * D;
    for (int i = tid; i < G * D; i += kThreads) {
      const int h = i / D, c = i % D;
      float part[16];
#pragma unroll
      for (int s = 0; s < 16; ++s) part[s] = (s < NS) ? cluster.map_shared_rank(acc_s, s)[i] : 0.f;
      float a = compensate ? fac_s[h * 17 + 16] * cp_s[h * (D + 2) + 2 + c] : 0.f;
#pragma unroll
      for (int s = 0; s < 16; ++s) a = fmaf(fac_s[h * 17 + s], part[s], a);
      o[i] = a * sc_s[h];
    }
  }
  cluster.sync();  // #2: rank 0 is done reading the other ranks' shared memory
}

template <typename T, int D, int G>
cudaError_t launch_t(const SparseArgs& a, cudaStream_t st, int bpc, int ns) {
  auto kern = sparse_decode_kernel<T, D, G>;
  const size_t smem = SLayout<T, D, G>::total;
  static bool attrs_set = false;  // set once, so a launch inside stream capture only launches
  if (!attrs_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    attrs_set = true;
  }
  SParams p;
  p.mode = a.mode;
  p.Hkv = a.Hkv;
  p.T = a.T;
  p.Nb = a.Nb;
  p.Kb = a.Kb;
  p.bpc = bpc;
  p.scale = a.scale;
  p.q = a.q;
  p.K = a.K;
  p.V = a.V;
  p.mean_v = a.mean_v;
  p.sel_idx = a.sel_idx;
  p.comp = a.comp;
  p.xrec = a.xrec;
  p.out = a.out;
  p.status = a.status;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.B * a.Hkv * ns, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = ns;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

template <typename T, int D>
cudaError_t dispatch_g(const SparseArgs& a, cudaStream_t st, int bpc, int ns) {
  switch (a.G) {
    case 1: return launch_t<T, D, 1>(a, st, bpc, ns);
    case 2: return launch_t<T, D, 2>(a, st, bpc, ns);
    case 4: return launch_t<T, D, 4>(a, st, bpc, ns);
    case 8: return launch_t<T, D, 8>(a, st, bpc, ns);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

void sparse_split(int B, int Hkv, int Kb, int* blocks_per_cta, int* nsplit) {
  (void)B;
  (void)Hkv;
  const int ns = Kb <= 0 ? 1 : (Kb < 16 ? Kb : 16);
  const int bpc = Kb <= 0 ? 0 : (Kb + ns - 1) / ns;
  *blocks_per_cta = bpc;
  *nsplit = ns;
}

cudaError_t launch_sparse_decode(const SparseArgs& a, cudaStream_t st) {
  int bpc, ns;
  sparse_split(a.B, a.Hkv, a.Kb, &bpc, &ns);
  if (a.bf16) {
    return a.D == 128 ? dispatch_g<uint16_t, 128>(a, st, bpc, ns) : dispatch_g<uint16_t, 64>(a, st, bpc, ns);
  }
  return a.D == 128 ? dispatch_g<float, 128>(a, st, bpc, ns) : dispatch_g<float, 64>(a, st, bpc, ns);
}

}  // namespace compkv
