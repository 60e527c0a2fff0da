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
//
// bf16 caches run on the tensor cores instead (full_decode_mma_kernel): the same split-K plan,
// producer warp, ring and merge, with the tiles brought in by TMA tensor copies in the 128-byte
// swizzled layout, and each consumer warp taking whole tiles through mma.sync (bf16 operands,
// fp32 accumulation), transposed so that the tokens fill the 16-row side and the G query heads
// (padded to 8) the 8-column side:
//   S^T[t, h] = sum_d K[t, d] q[h, d]        (A = K rows via ldmatrix, B = q in registers)
//   O^T[d, h] += sum_t V[t, d] P[t, h]      (A = V^T via ldmatrix.trans, B = P^T)
// P^T's B fragments come from S^T's accumulators by an 8x8 register transpose (movmatrix), with
// P rounded to bf16 and the softmax sums taken over the same rounded weights. Every lane holds
// two heads' columns, so the rescaling of the accumulators needs no shuffle; the row sums stay
// per lane until the end.
#include <cuda.h>

#include <mutex>

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

// The 8 consumer warps' partials -> this split's partial (max, sum, acc) in the workspace; the
// last CTA of the kv-head (atomic ticket) merges the splits into the output and resets the ticket.
template <int D, int G>
__device__ __forceinline__ void merge_partials(float* part_ws, uint32_t* counters, float* out, int bk, int split,
                                               int nsplit, const float* wacc, const float* wml, float* fac,
                                               int* flag) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // ---- the 8 warps' partials -> this split's partial in the workspace
  float* mine = part_ws + (static_cast<size_t>(bk) * nsplit + split) * G * (D + 2);
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
  if (tid == 0) flag[0] = (atomicAdd(&counters[bk], 1u) == static_cast<uint32_t>(nsplit - 1));
  __syncthreads();
  if (!flag[0]) return;

  // ---- last CTA of this kv-head: merge the splits
  __threadfence();
  const float* parts = part_ws + static_cast<size_t>(bk) * nsplit * G * (D + 2);
  float* ml_s = sml;
  if (tid < G) {
    float M = -CUDART_INF_F;
    for (int s = 0; s < nsplit; ++s) M = fmaxf(M, __ldcg(parts + (static_cast<size_t>(s) * G + tid) * (D + 2)));
    float den = 0.f;
    for (int s = 0; s < nsplit; ++s) {
      const float* ps = parts + (static_cast<size_t>(s) * G + tid) * (D + 2);
      const float ms = __ldcg(ps);
      if (ms != -CUDART_INF_F) den = fmaf(__expf(ms - M), __ldcg(ps + 1), den);
    }
    ml_s[2 * tid] = M;
    ml_s[2 * tid + 1] = den > 0.f ? 1.f / den : 0.f;
  }
  __syncthreads();
  float* o = out + static_cast<size_t>(bk) * G * D;
  for (int i = tid; i < G * D; i += kFThreads) {
    const int h = i / D, c = i % D;
    const float M = ml_s[2 * h];
    float a = 0.f;
    for (int s = 0; s < nsplit; ++s) {
      const float* ps = parts + (static_cast<size_t>(s) * G + h) * (D + 2);
      const float ms = __ldcg(ps);
      if (ms != -CUDART_INF_F) a = fmaf(__expf(ms - M), __ldcg(ps + 2 + c), a);
    }
    o[i] = a * ml_s[2 * h + 1];
  }
  if (tid == 0) counters[bk] = 0u;
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

  merge_partials<D, G>(p.part, p.counters, p.out, bk, split, p.nsplit, wacc, wml, fac, flag);
}

// ------------------------------------------------------------------ tensor-core variant (bf16)

constexpr int kBoxCols = 64;  // bf16 columns per TMA box: 128 bytes, the swizzle span

struct MParams {
  CUtensorMap tmK;  // [B * Hkv * T rows][D] bf16, boxes of 32 rows x 64 columns, 128-byte swizzle
  CUtensorMap tmV;
  int Hkv, T, nsplit, stages;
  float scale;
  const void* q;
  const int32_t* ctx_lens;
  float* out;
  float* part;
  uint32_t* counters;
  int32_t* status;
};

template <int D, int G>
struct MLayout {
  static constexpr int kBoxes = D / kBoxCols;
  static constexpr size_t box_bytes = kTT * kBoxCols * 2;               // 4 KB
  static constexpr size_t stage_bytes = 2 * kBoxes * box_bytes;         // K boxes, then V boxes
  static constexpr size_t off_q = 0;                                    // [G][D] fp32
  static constexpr size_t off_wml = off_q + sizeof(float) * G * D;      // [kCons][G][2]
  static constexpr size_t off_fac = off_wml + sizeof(float) * kCons * G * 2;
  static constexpr size_t off_flag = off_fac + sizeof(float) * (kCons * G + 2 * G);
  static constexpr size_t off_bar = (off_flag + 16 + 15) & ~size_t(15);
  static constexpr size_t off_ring = off_bar + 8 * 2 * kMaxStages;      // aligned up to 1024 at run time
  static size_t total(int stages) { return off_ring + 1024 + stage_bytes * stages; }
  // the warps' partial sums [kCons][G][D] go into the ring once every tile is consumed
  static_assert(sizeof(float) * kCons * G * D <= 2 * stage_bytes, "partials must fit the ring");
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
// D += A (16 x 16, row-major) B (16 x 8, column-major), bf16 operands, fp32 accumulators.
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
               "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
               : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
               : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t a) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
  return d;
}
// Two fp32 values as a bf16 pair (round to nearest even); `lo` takes the lower half.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// One 2-D TMA tensor load (box at column x, row y) into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar,
                                            uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

// Byte offset of the 16-byte chunk j (columns 8j .. 8j + 7 of a box) of row n in a box written
// with the 128-byte swizzle: the chunk index is XORed with the row's index mod 8.
__device__ __forceinline__ uint32_t swz(int n, int j) {
  return static_cast<uint32_t>(n * 128 + ((j ^ (n & 7)) << 4));
}

template <int D, int G>
__global__ void __launch_bounds__(kFThreads, 2) full_decode_mma_kernel(const __grid_constant__ MParams p) {
  using LY = MLayout<D, G>;
  constexpr int NB = LY::kBoxes;
  constexpr int MT = D / 16;  // 16-channel tiles of O^T
  static_assert(G <= 8, "at most 8 query heads per kv-head");
  extern __shared__ __align__(128) unsigned char sm[];
  float* q_s = reinterpret_cast<float*>(sm + LY::off_q);
  float* wml = reinterpret_cast<float*>(sm + LY::off_wml);
  float* fac = reinterpret_cast<float*>(sm + LY::off_fac);
  int* flag = reinterpret_cast<int*>(sm + LY::off_flag);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + LY::off_bar);
  uint64_t* empty = full + kMaxStages;
  const uint32_t ring_off = static_cast<uint32_t>(LY::off_ring) +
                            ((1024u - ((smem_addr(sm) + static_cast<uint32_t>(LY::off_ring)) & 1023u)) & 1023u);
  unsigned char* ring = sm + ring_off;  // 1024-byte aligned, as the swizzled boxes need
  float* wacc = reinterpret_cast<float*>(ring);  // [kCons][G][D], after the last tile

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int NS = p.stages;
  const int bk = blockIdx.x / p.nsplit, split = blockIdx.x % p.nsplit;
  const int b = bk / p.Hkv;
  int Tb = p.ctx_lens ? p.ctx_lens[b] : p.T;
  Tb = max(0, min(Tb, p.T));
  const int per = ((Tb + p.nsplit - 1) / p.nsplit + kTT - 1) / kTT * kTT;
  const int t0 = min(Tb, split * per), t1 = min(Tb, t0 + per);
  const int ntiles = (t1 - t0 + kTT - 1) / kTT;
  const int row0 = bk * p.T + t0;  // first cache row of the range

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    flag[1] = 0;
    mbar_init_fence();
  }
  {
    const uint16_t* qp = static_cast<const uint16_t*>(p.q) + static_cast<size_t>(bk) * G * D;
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
        unsigned char* sb = ring + LY::stage_bytes * st;
        mbar_arrive_expect_tx(&full[st], static_cast<uint32_t>(LY::stage_bytes));
#pragma unroll
        for (int bx = 0; bx < NB; ++bx) {
          tma_load_2d(sb + bx * LY::box_bytes, &p.tmK, bx * kBoxCols, row0 + i * kTT, &full[st], policy);
          tma_load_2d(sb + (NB + bx) * LY::box_bytes, &p.tmV, bx * kBoxCols, row0 + i * kTT, &full[st], policy);
        }
      }
      ++issued;
    }
    if (*reinterpret_cast<volatile int*>(&flag[1]) != 0) {  // gave up: drain the copies in flight
      for (int i = max(0, issued - NS); i < issued; ++i)
        mbar_wait(&full[i % NS], static_cast<uint32_t>((i / NS) & 1), nullptr);
    }
  } else {  // ---- consumers: warp w < NS takes the tiles of stage w (i = w mod NS), whole, so
            // that it waits on that stage's phases in order (a parity wait cannot tell a phase
            // from the one two ahead); warps w >= NS hold empty partials
    const int gq = lane >> 2, cq = lane & 3;  // fragment row (group) and column pair
    // q as the B operand of S^T: k = channel, n = head (heads >= G are zero)
    uint32_t qb[D / 16][2];
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      const int h = gq, d0 = ks * 16 + 2 * cq;
      const bool real = h < G;
      qb[ks][0] = real ? pack_bf16(q_s[h * D + d0], q_s[h * D + d0 + 1]) : 0u;
      qb[ks][1] = real ? pack_bf16(q_s[h * D + d0 + 8], q_s[h * D + d0 + 9]) : 0u;
    }
    float o[MT][4];  // O^T accumulators: rows = channels, columns = heads 2 cq, 2 cq + 1
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
    float m0 = -CUDART_INF_F, m1 = -CUDART_INF_F, l0 = 0.f, l1 = 0.f;  // heads 2 cq, 2 cq + 1
    // ldmatrix lane roles: matrix mi = lane / 8, row rr = lane % 8
    const int mi = lane >> 3, rr = lane & 7;
    bool ok = true;
#pragma unroll 1
    for (int i = warp; i < ntiles && warp < NS; i += NS) {
      const int st = warp;
      ok = __all_sync(0xffffffffu, ok && mbar_wait(&full[st], static_cast<uint32_t>((i / NS) & 1), p.status));
      const int rows = ok ? min(kTT, t1 - t0 - i * kTT) : 0;
      unsigned char* kb = ring + LY::stage_bytes * st;
      unsigned char* vb = kb + NB * LY::box_bytes;
      if (rows < kTT) {  // rows past the range: zero V (their weight is 0, but 0 * NaN is NaN)
        for (int c = lane; c < (kTT - rows) * (D / 8); c += 32) {
          const int n = rows + c / (D / 8), ch = c % (D / 8);
          *reinterpret_cast<uint4*>(vb + (ch / 8) * LY::box_bytes + swz(n, ch % 8)) = make_uint4(0u, 0u, 0u, 0u);
        }
        __syncwarp();
      }
      // S^T: two 16-token tiles
      float s[2][4];
#pragma unroll
      for (int tt = 0; tt < 2; ++tt) {
        s[tt][0] = s[tt][1] = s[tt][2] = s[tt][3] = 0.f;
        const int n = tt * 16 + (mi & 1) * 8 + rr;  // token row this lane addresses
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const int ch = ks * 2 + (mi >> 1);        // 16-byte chunk of the row (8 channels)
          uint32_t a[4];
          ldsm_x4(smem_addr(kb + (ch / 8) * LY::box_bytes + swz(n, ch % 8)), a);
          mma_bf16(s[tt], a, qb[ks][0], qb[ks][1]);
        }
      }
      // scale, mask, the tile's maxima of this lane's two heads
      float tm0 = -CUDART_INF_F, tm1 = -CUDART_INF_F;
#pragma unroll
      for (int tt = 0; tt < 2; ++tt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int t = tt * 16 + gq + (e >> 1) * 8;
          const float v = t < rows ? p.scale * s[tt][e] : -CUDART_INF_F;
          s[tt][e] = v;
          if (e & 1) tm1 = fmaxf(tm1, v); else tm0 = fmaxf(tm0, v);
        }
#pragma unroll
      for (int o2 = 4; o2 < 32; o2 <<= 1) {
        tm0 = fmaxf(tm0, __shfl_xor_sync(0xffffffffu, tm0, o2));
        tm1 = fmaxf(tm1, __shfl_xor_sync(0xffffffffu, tm1, o2));
      }
      const float n0 = fmaxf(m0, tm0), n1 = fmaxf(m1, tm1);
      const float c0 = exp_diff(m0, n0), c1 = exp_diff(m1, n1);
      m0 = n0;
      m1 = n1;
      // P (bf16) and this lane's share of the sums, over the rounded weights
      uint32_t pk[2][2];
      float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
      for (int tt = 0; tt < 2; ++tt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const float pa = exp_diff(s[tt][2 * hh], n0), pb = exp_diff(s[tt][2 * hh + 1], n1);
          const uint32_t w = pack_bf16(pa, pb);
          ps0 += bf16_lo(w);
          ps1 += bf16_hi(w);
          pk[tt][hh] = movmatrix_t(w);  // -> B fragment: k = token, n = head
        }
      l0 = fmaf(l0, c0, ps0);
      l1 = fmaf(l1, c1, ps1);
      // O^T += V^T P^T
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        o[mt][0] *= c0;
        o[mt][1] *= c1;
        o[mt][2] *= c0;
        o[mt][3] *= c1;
#pragma unroll
        for (int tt = 0; tt < 2; ++tt) {
          const int n = tt * 16 + (mi >> 1) * 8 + rr;  // token row
          const int ch = mt * 2 + (mi & 1);            // chunk: channels mt * 16 + 8 (mi & 1)
          uint32_t a[4];
          ldsm_x4_t(smem_addr(vb + (ch / 8) * LY::box_bytes + swz(n, ch % 8)), a);
          mma_bf16(o[mt], a, pk[tt][0], pk[tt][1]);
        }
      }
      __syncwarp();
      if (lane == 0) {
        if (rows < kTT) fence_proxy_async();  // the zeroed rows before the next tensor copy
        mbar_arrive(&empty[st]);
      }
    }
    // this warp's partial: the sums over the lanes of each head column, then (M, L, A); the
    // sums go into the ring once no warp reads a tile any more
#pragma unroll
    for (int o2 = 4; o2 < 32; o2 <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, o2);
      l1 += __shfl_xor_sync(0xffffffffu, l1, o2);
    }
    named_bar_sync(1, kCons * 32);  // the consumer warps only: every tile consumed
    const int h0 = 2 * cq, h1 = 2 * cq + 1;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int h = (e & 1) ? h1 : h0, d = mt * 16 + gq + (e >> 1) * 8;
        if (h < G) wacc[(warp * G + h) * D + d] = o[mt][e];
      }
    if (gq == 0) {
      if (h0 < G) {
        wml[(warp * G + h0) * 2] = m0;
        wml[(warp * G + h0) * 2 + 1] = l0;
      }
      if (h1 < G) {
        wml[(warp * G + h1) * 2] = m1;
        wml[(warp * G + h1) * 2 + 1] = l1;
      }
    }
  }
  __syncthreads();
  merge_partials<D, G>(p.part, p.counters, p.out, bk, split, p.nsplit, wacc, wml, fac, flag);
}

// Stages that keep two CTAs per SM (the tile ring is the bulk of the shared memory), an even
// number: tile i goes to stage i % NS and warp group i % 2, so each stage always serves the same
// group, which then waits on its phases in order (a parity wait cannot tell a phase from the one
// two ahead).
template <typename T, int D, int G>
int stages_for() {
  using LY = FLayout<T, D, G>;
  int s = kMaxStages;
  while (s > 2 && LY::total(s) > (113u << 10)) --s;
  return s & ~1;
}

// cuTensorMapEncodeTiled, looked up once through the runtime (no link against the driver library).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// A bf16 cache [rows][D] as a 2-D tensor: boxes of 32 rows x 64 columns, 128-byte swizzle, rows
// past the end read as zeros. False if the base address or the driver does not allow it.
bool make_cache_map(CUtensorMap* m, const void* base, uint64_t rows, int D) {
  const EncodeTiledFn fn = encode_tiled();
  if (fn == nullptr || (reinterpret_cast<uintptr_t>(base) & 15u) != 0) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBoxCols), static_cast<cuuint32_t>(kTT)};
  const cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int G>
int mma_stages() {
  using LY = MLayout<D, G>;
  int s = kMaxStages;
  while (s > 2 && LY::total(s) > (113u << 10)) --s;
  return s;
}

// The tensor-core kernel for a bf16 cache; cudaErrorNotSupported when no tensor map can be made
// (the caller then runs the fp32-arithmetic kernel).
template <int D, int G>
cudaError_t launch_mma(const FullArgs& a, cudaStream_t st) {
  MParams p;
  const uint64_t rows = static_cast<uint64_t>(a.B) * a.Hkv * a.T;
  if (!make_cache_map(&p.tmK, a.K, rows, D) || !make_cache_map(&p.tmV, a.V, rows, D)) return cudaErrorNotSupported;
  auto kern = full_decode_mma_kernel<D, G>;
  const int stages = mma_stages<D, G>();
  const size_t smem = MLayout<D, G>::total(stages);
  static bool attrs_set = false;  // set once, so a launch inside stream capture only launches
  if (!attrs_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    attrs_set = true;
  }
  p.Hkv = a.Hkv;
  p.T = a.T;
  p.nsplit = a.nsplit;
  p.stages = stages;
  p.scale = a.scale;
  p.q = a.q;
  p.ctx_lens = a.ctx_lens;
  p.out = a.out;
  p.part = a.part;
  p.counters = a.counters;
  p.status = a.status;
  full_decode_mma_kernel<D, G><<<a.B * a.Hkv * a.nsplit, kFThreads, smem, st>>>(p);
  return cudaGetLastError();
}

template <typename T, int D, int G>
cudaError_t launch_t(const FullArgs& a, cudaStream_t st) {
  if constexpr (sizeof(T) == 2) {
    const cudaError_t e = launch_mma<D, G>(a, st);
    if (e != cudaErrorNotSupported) return e;
  }
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
