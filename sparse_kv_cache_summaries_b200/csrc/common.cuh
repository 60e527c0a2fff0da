// Device helpers shared by the CompKV kernels (sm_100a): mbarrier + bulk-copy pipelines,
// thread-block-cluster barriers and distributed shared memory, programmatic dependent launch,
// bf16 unpacking, warp/CTA reductions and an order-preserving float key.
#pragma once

#include <cuda_fp16.h>
#include <cstdint>
#include <cuda_runtime.h>
#include <math_constants.h>

#include "compkv.h"

namespace compkv {

constexpr int kBlockTokens = 16;      // tokens per KV block
constexpr int kThreads = 256;         // threads per CTA for every kernel here
constexpr int kWarps = kThreads / 32;

// ------------------------------------------------------------------------------ addresses

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------------------------------ mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

// Makes barrier initialisation visible to the async proxy (bulk copies) and the cluster.
__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for phase `parity` of a barrier, giving up after a bounded number of attempts (each
// attempt suspends the thread for a hardware-chosen interval). On giving up it records
// COMPKV_DEVERR_WAIT_TIMEOUT in *status and returns false; callers then skip the work that
// needed the data but keep every barrier of the CTA / cluster.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int32_t* status) {
  for (uint32_t it = 0; it < (1u << 22); ++it) {
    if (mbar_try_wait(bar, parity)) return true;
  }
  if (status != nullptr) atomicOr(status, COMPKV_DEVERR_WAIT_TIMEOUT);
  return false;
}

// Orders this thread's earlier generic-proxy shared-memory writes before later async-proxy
// (bulk copy) accesses of the same bytes.
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------------------ async copies

// Bulk (non-tensor) copy global -> this CTA's shared memory, completing on `bar` with a
// transaction count of `bytes`. dst, src and bytes must be multiples of 16 bytes. No multicast.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// Same, with an L2 evict-first hint for data that is read once per step.
__device__ __forceinline__ void bulk_g2s_stream(void* dst, const void* src, uint32_t bytes,
                                                uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Hint: bring the bytes [begin, begin + bytes) of global memory into L2 (no shared memory, no
// completion to wait for). The range is shrunk inward to 16-byte boundaries, so nothing outside
// it is touched. No multicast.
__device__ __forceinline__ void prefetch_l2_range(const void* begin, size_t bytes) {
  uintptr_t a = reinterpret_cast<uintptr_t>(begin);
  uintptr_t e = a + bytes;
  a = (a + 15) & ~static_cast<uintptr_t>(15);
  e &= ~static_cast<uintptr_t>(15);
  while (a < e) {
    const uint32_t n = static_cast<uint32_t>((e - a) < (1u << 20) ? (e - a) : (1u << 20));
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a), "r"(n) : "memory");
    a += n;
  }
}

// 4-byte asynchronous copy (any 4-byte aligned address); tracked by cp_async_arrive.
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_addr(dst)), "l"(src)
               : "memory");
}

// Arrives on `bar` once all of this thread's earlier cp.async copies have landed. The barrier's
// expected count must include this arrival (noinc).
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

// ------------------------------------------------------------------------------ clusters

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ uint32_t cluster_size() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}

// Full cluster barrier with release/acquire semantics for shared and global memory.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
               "barrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}

// Address of the same shared variable in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t dsmem_addr(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr(p)), "r"(rank));
  return r;
}

__device__ __forceinline__ float ld_dsmem_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ uint32_t ld_dsmem_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

// ------------------------------------------------------------------------------ PDL

// Blocks until the preceding grid on the stream has completed and its writes are visible.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Lets the next grid on the stream (launched with programmatic serialisation) start its prologue.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------------------------------ numerics

// Unpacks 8 bf16 (one 16-byte word) or 4 fp32 into floats.
__device__ __forceinline__ void unpack8_bf16(const uint4& w, float (&f)[8]) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(u[i] << 16);
    f[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
  }
}

// Summary storage of the mean key and mean value: fp32, or fp16 rounded to nearest even.
__device__ __forceinline__ float sload(const float* p) { return *p; }
__device__ __forceinline__ float sload(const __half* p) { return __half2float(*p); }
__device__ __forceinline__ void sstore(float* p, float x) { *p = x; }
__device__ __forceinline__ void sstore(__half* p, float x) { *p = __float2half_rn(x); }

__device__ __forceinline__ float to_float(float x) { return x; }
__device__ __forceinline__ float to_float(uint16_t x) {
  return __uint_as_float(static_cast<uint32_t>(x) << 16);
}

// Order-preserving map of a non-negative float to uint32 (larger float -> larger key); keys of
// real scores are >= 0x80000000, so key 0 ranks below every real score.
__device__ __forceinline__ uint32_t score_key(float s) {
  const uint32_t b = __float_as_uint(s);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// exp(a - b) that treats (-inf) - (-inf) as an empty term (0) instead of NaN.
__device__ __forceinline__ float exp_diff(float a, float b) {
  return (a == -CUDART_INF_F) ? 0.f : __expf(a - b);
}

// Online log-sum-exp pair (max, sum of exp(x - max)); merges another pair.
__device__ __forceinline__ void lse_merge(float& m, float& s, float m2, float s2) {
  if (m2 == -CUDART_INF_F) return;
  if (m == -CUDART_INF_F) {
    m = m2;
    s = s2;
    return;
  }
  const float mn = fmaxf(m, m2);
  s = s * __expf(m - mn) + s2 * __expf(m2 - mn);
  m = mn;
}

// ------------------------------------------------------------------------------ CTA helpers

// Exclusive prefix sum of one int per thread over the CTA; also returns the total.
// `sh` needs kWarps + 1 ints. Contains __syncthreads.
__device__ __forceinline__ int cta_exclusive_scan(int v, int* sh, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) sh[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = (lane < kWarps) ? sh[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += t;
    }
    if (lane < kWarps) sh[lane] = wi - w;
    if (lane == kWarps - 1) sh[kWarps] = wi;
  }
  __syncthreads();
  const int res = sh[warp] + incl - v;
  total = sh[kWarps];
  __syncthreads();
  return res;
}

// Top-K threshold by most-significant-digit radix select over 32-bit keys (8-bit digits).
// Finds the bucket (prefix under mask) that holds the K-th largest key (1 <= K <= n) and the
// number `quota` of keys in that bucket that belong to the top K; keys in higher buckets all
// belong. Stops early once the whole bucket is selected. `hist` holds 2 x 256 uints, `bc` 4
// uints. All threads call it and get the result; two CTA barriers per digit.
struct RadixCut {
  uint32_t prefix, mask;
  int quota;
  bool whole;  // every key of the bucket is kept (no tie ranking needed)
};

template <typename KeyAt>
__device__ RadixCut cta_radix_cut(KeyAt key_at, int n, int K, uint32_t* hist, uint32_t* bc) {
  uint32_t prefix = 0, mask = 0;
  uint32_t k = static_cast<uint32_t>(K);
  for (int i = threadIdx.x; i < 512; i += kThreads) hist[i] = 0;
  __syncthreads();
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    uint32_t* H = hist + (pass & 1) * 256;
    uint32_t* Hn = hist + ((pass + 1) & 1) * 256;
    // warp-aggregated counting: one atomic per distinct digit per warp (float keys crowd into a
    // few top-digit buckets, where plain per-key atomics serialise)
    const int n32 = (n + 31) & ~31;
    for (int i = threadIdx.x; i < n32; i += kThreads) {
      const uint32_t key = i < n ? key_at(i) : 0u;
      const bool m = i < n && (key & mask) == prefix;
      const uint32_t bin = (key >> shift) & 255u;
      const uint32_t grp = __match_any_sync(0xffffffffu, m ? bin : 256u + (threadIdx.x & 31));
      if (m && (__ffs(grp) - 1) == static_cast<int>(threadIdx.x & 31)) atomicAdd(&H[bin], __popc(grp));
    }
    for (int i = threadIdx.x; i < 256; i += kThreads) Hn[i] = 0;
    __syncthreads();
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      uint32_t c[8], tot = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        c[e] = H[255 - 8 * lane - e];
        tot += c[e];
      }
      uint32_t incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      const uint32_t excl = incl - tot;
      if (excl < k && k <= incl) {
        uint32_t run = excl;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if (run + c[e] >= k) {
            bc[0] = static_cast<uint32_t>(255 - 8 * lane - e);
            bc[1] = k - run;
            bc[2] = c[e];
            break;
          }
          run += c[e];
        }
      }
    }
    __syncthreads();
    const uint32_t bin = bc[0], cnt = bc[2];
    k = bc[1];
    prefix |= bin << shift;
    mask |= 255u << shift;
    if (cnt == k) break;  // every key of the bucket is in the top K
  }
  return RadixCut{prefix, mask, static_cast<int>(k)};
}

// Same contract as cta_radix_cut, tuned for non-negative float score keys: the first digit is
// the top 11 bits (sign, exponent and two mantissa bits), which spreads scores over hundreds of
// buckets, so the bucket holding the K-th largest key usually is selected whole after one pass.
// Later digits take 8, 8 and 5 bits. Each pass: one barrier after counting, one inside the
// block-wide scan of the bucket counts (in descending bucket order), one to publish the bucket.
// `hist` holds 2592 uints (2048 + 256 + 256 + 32 buckets), `bc` 4 uints.
namespace detail {
// One digit pass of cta_topk_cut over NB = 2^BITS buckets at bit SHIFT (see there).
template <int SHIFT, int BITS, typename KeyAt>
__device__ __forceinline__ bool topk_pass(KeyAt key_at, int n, uint32_t* H, uint32_t* bc, int* sh,
                                          uint32_t& prefix, uint32_t& mask, uint32_t& k) {
  constexpr int NB = 1 << BITS;
  constexpr uint32_t DM = NB - 1;
  constexpr int PER = (NB + kThreads - 1) / kThreads;  // buckets per thread: 8 or 1
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < n; i += kThreads) {
    const uint32_t key = key_at(i);
    if ((key & mask) == prefix) atomicAdd(&H[(key >> SHIFT) & DM], 1u);
  }
  __syncthreads();
  // descending scan: thread t owns buckets NB-1-t*PER ... NB-(t+1)*PER (first = highest)
  uint32_t c[PER];
  const int top = NB - 1 - static_cast<int>(threadIdx.x) * PER;
  if constexpr (PER == 8) {
    const uint4 lo = reinterpret_cast<const uint4*>(H + top - 7)[0];
    const uint4 hi = reinterpret_cast<const uint4*>(H + top - 7)[1];
    c[0] = hi.w; c[1] = hi.z; c[2] = hi.y; c[3] = hi.x; c[4] = lo.w; c[5] = lo.z; c[6] = lo.y; c[7] = lo.x;
  } else {
    c[0] = top >= 0 ? H[top] : 0u;
  }
  uint32_t cnt = 0;
#pragma unroll
  for (int e = 0; e < PER; ++e) cnt += c[e];
  uint32_t incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) sh[warp] = static_cast<int>(incl);
  __syncthreads();
  uint32_t base = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) base += (w < warp) ? static_cast<uint32_t>(sh[w]) : 0u;
  const uint32_t excl = base + incl - cnt;
  if (cnt > 0 && excl < k && k <= excl + cnt) {
    uint32_t run = excl;
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      if (run < k && run + c[e] >= k) {
        bc[0] = static_cast<uint32_t>(top - e);
        bc[1] = k - run;
        bc[2] = c[e];
      }
      run += c[e];
    }
  }
  __syncthreads();
  const uint32_t bin = bc[0], bcnt = bc[2];
  k = bc[1];
  prefix |= bin << SHIFT;
  mask |= DM << SHIFT;
  return bcnt == k;  // the whole bucket is in the top K
}
}  // namespace detail

// Same contract as cta_radix_cut, tuned for non-negative float score keys: the first digit is
// the top 11 bits (sign, exponent and two mantissa bits), which spreads scores over hundreds of
// buckets, so the bucket holding the K-th largest key usually is selected whole after one or two
// passes. Later digits take 8, 8 and 5 bits. `hist` holds 2592 uints (2048 + 256 + 256 + 32
// buckets, 16-byte aligned), `bc` 4 uints, `sh` kWarps ints. Two CTA barriers per pass.
template <typename KeyAt>
__device__ RadixCut cta_topk_cut(KeyAt key_at, int n, int K, uint32_t* hist, uint32_t* bc, int* sh) {
  for (int i = threadIdx.x; i < 2592 / 4; i += kThreads) reinterpret_cast<uint4*>(hist)[i] = make_uint4(0, 0, 0, 0);
  __syncthreads();
  uint32_t prefix = 0, mask = 0, k = static_cast<uint32_t>(K);
  if (detail::topk_pass<21, 11>(key_at, n, hist, bc, sh, prefix, mask, k))
    return RadixCut{prefix, mask, static_cast<int>(k), true};
  if (detail::topk_pass<13, 8>(key_at, n, hist + 2048, bc, sh, prefix, mask, k))
    return RadixCut{prefix, mask, static_cast<int>(k), true};
  if (detail::topk_pass<5, 8>(key_at, n, hist + 2304, bc, sh, prefix, mask, k))
    return RadixCut{prefix, mask, static_cast<int>(k), true};
  const bool whole = detail::topk_pass<0, 5>(key_at, n, hist + 2560, bc, sh, prefix, mask, k);
  return RadixCut{prefix, mask, static_cast<int>(k), whole};
}

// Warp-wise version of cta_select_ordered: warp w scans a contiguous run of items with its lanes
// on consecutive items (no shared-memory bank conflicts), ballots give positions inside the warp
// and one CTA barrier gives each warp's offset. `sh` needs 2 * kWarps ints.
template <typename KeyAt, typename Emit>
__device__ int cta_select_ordered_w(KeyAt key_at, int n, const RadixCut& cut, int* sh, Emit emit) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int span = ((n + kWarps * 32 - 1) / (kWarps * 32)) * 32;
  const int i0 = warp * span, i1 = min(n, i0 + span);
  const uint32_t lt = (1u << lane) - 1u;
  int gt_w = 0, eq_w = 0;
  for (int b = i0; b < i1; b += 32) {
    const int i = b + lane;
    const uint32_t km = i < i1 ? (key_at(i) & cut.mask) : 0u;
    const bool valid = i < i1;
    gt_w += __popc(__ballot_sync(0xffffffffu, valid && km > cut.prefix));
    eq_w += __popc(__ballot_sync(0xffffffffu, valid && km == cut.prefix));
  }
  if (lane == 0) {
    sh[warp] = gt_w;
    sh[kWarps + warp] = eq_w;
  }
  __syncthreads();
  int eq_before = 0, total = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const int e = sh[kWarps + w];
    const int kept_w = sh[w] + (cut.whole ? e : max(0, min(e, cut.quota - eq_before)));
    if (w < warp) total += kept_w;
    eq_before += (w < warp) ? e : 0;
  }
  // total is now this warp's output offset
  int pos = total, er = eq_before;
  for (int b = i0; b < i1; b += 32) {
    const int i = b + lane;
    const bool valid = i < i1;
    const uint32_t km = valid ? (key_at(i) & cut.mask) : 0u;
    const bool gt = valid && km > cut.prefix, eq = valid && km == cut.prefix;
    const uint32_t beq = __ballot_sync(0xffffffffu, eq);
    const int my_er = er + __popc(beq & lt);
    const bool keep = gt || (eq && (cut.whole || my_er < cut.quota));
    const uint32_t bk = __ballot_sync(0xffffffffu, keep);
    if (keep) emit(i, pos + __popc(bk & lt));
    pos += __popc(bk);
    er += __popc(beq);
  }
  int kept_total = 0, eqb = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const int e = sh[kWarps + w];
    kept_total += sh[w] + (cut.whole ? e : max(0, min(e, cut.quota - eqb)));
    eqb += e;
  }
  __syncthreads();
  return kept_total;
}

// Keeps item i if (key & mask) > prefix, or it equals prefix and fewer than `quota` such items
// precede it; visits kept items in index order with their output position: emit(i, pos).
// `sh` needs kWarps + 1 ints. Contains CTA barriers. Returns the number kept.
template <typename KeyAt, typename Emit>
__device__ int cta_select_ordered(KeyAt key_at, int n, const RadixCut& cut, int* sh, Emit emit) {
  const int per = (n + kThreads - 1) / kThreads;
  const int i0 = min(n, static_cast<int>(threadIdx.x) * per), i1 = min(n, i0 + per);
  if (cut.whole) {  // no ties to rank: keep every key at or above the bucket, one scan
    int kept = 0;
    for (int i = i0; i < i1; ++i) kept += ((key_at(i) & cut.mask) >= cut.prefix);
    int kept_total;
    int pos = cta_exclusive_scan(kept, sh, kept_total);
    for (int i = i0; i < i1; ++i)
      if ((key_at(i) & cut.mask) >= cut.prefix) emit(i, pos++);
    return kept_total;
  }
  int eq = 0, gt = 0;
  for (int i = i0; i < i1; ++i) {
    const uint32_t km = key_at(i) & cut.mask;
    eq += (km == cut.prefix);
    gt += (km > cut.prefix);
  }
  int eq_total;
  const int eq_before = cta_exclusive_scan(eq, sh, eq_total);
  const int kept_eq = max(0, min(eq, cut.quota - eq_before));
  int kept_total;
  int pos = cta_exclusive_scan(gt + kept_eq, sh, kept_total);
  int er = eq_before;
  for (int i = i0; i < i1; ++i) {
    const uint32_t km = key_at(i) & cut.mask;
    bool keep = km > cut.prefix;
    if (km == cut.prefix) {
      keep = er < cut.quota;
      ++er;
    }
    if (keep) emit(i, pos++);
  }
  return kept_total;
}


// Address of `p` (this CTA's shared memory) in the shared memory of cluster rank `rank`, as a
// shared::cluster address.
__device__ __forceinline__ uint32_t cluster_smem_addr(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr(p)), "r"(rank));
  return r;
}

// Arrives on an mbarrier of another CTA of the cluster; release at cluster scope, so this
// thread's earlier writes (to that CTA's shared memory too) are visible to its waiters.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// Bounded wait, with acquire at cluster scope (for arrivals made by other CTAs of the cluster).
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, int32_t* status) {
  for (uint32_t it = 0; it < (1u << 22); ++it) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    if (ok) return true;
  }
  if (status != nullptr) atomicOr(status, COMPKV_DEVERR_WAIT_TIMEOUT);
  return false;
}

// Asynchronous store into another CTA's shared memory (shared::cluster addresses from
// cluster_smem_addr), completing `bytes` of transactions on that CTA's mbarrier: the receiver
// waits on its own mbarrier for the bytes it expects; no cluster barrier and no release fence.
__device__ __forceinline__ void st_async_b32(uint32_t dst, uint32_t v, uint32_t bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];"
               ::"r"(dst), "r"(v), "r"(bar) : "memory");
}
__device__ __forceinline__ void st_async_b64(uint32_t dst, uint64_t v, uint32_t bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b64 [%0], %1, [%2];"
               ::"r"(dst), "l"(v), "r"(bar) : "memory");
}

// 16 bytes (four 32-bit words) into a peer's shared memory; `dst` 16-byte aligned.
__device__ __forceinline__ void st_async_v4(uint32_t dst, float4 v, uint32_t bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];"
               ::"r"(dst), "r"(__float_as_uint(v.x)), "r"(__float_as_uint(v.y)), "r"(__float_as_uint(v.z)),
                 "r"(__float_as_uint(v.w)), "r"(bar) : "memory");
}

// Split cluster barrier (all threads of every CTA of the cluster). An early relaxed arrive and a
// later wait cost almost nothing; after the wait every CTA of the cluster has started, so its
// shared memory may be written remotely.
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }

// ------------------------------------------------------------------ warp-level Top-32

// Selection order as one 64-bit code: higher is better. Score key descending, then block index
// ascending (ties go to the lower index); every real block's code is nonzero, so 0 pads a list.
__device__ __forceinline__ uint64_t topk_code(uint32_t key, int idx) {
  return (static_cast<uint64_t>(key) << 32) | static_cast<uint32_t>(~static_cast<uint32_t>(idx));
}
__device__ __forceinline__ int topk_index(uint64_t code) {
  return static_cast<int>(~static_cast<uint32_t>(code));
}

// Entries of a descending list of T codes (T a power of two, 0 pads the tail) above x > 0:
// a binary search of log2(T) + 1 reads.
// Each step is a predicated select (no branch: lanes of a warp search different lists in step).
__device__ __forceinline__ int add_if_greater(int pos, uint64_t v, uint64_t x, int s) {
  int r;
  asm("{\n\t.reg .pred p;\n\tsetp.gt.u64 p, %1, %2;\n\tselp.s32 %0, %3, 0, p;\n\t}"
      : "=r"(r) : "l"(v), "l"(x), "r"(s));
  return pos + r;
}
template <int T>
__device__ __forceinline__ int count_greater(const uint64_t* list, uint64_t x) {
  int pos = 0;
#pragma unroll
  for (int s = T >> 1; s > 0; s >>= 1) pos = add_if_greater(pos, list[pos + s - 1], x, s);
  return add_if_greater(pos, list[pos], x, 1);
}

__device__ __forceinline__ uint64_t shfl_xor_u64(uint64_t v, int o) {
  const uint32_t lo = __shfl_xor_sync(0xffffffffu, static_cast<uint32_t>(v), o);
  const uint32_t hi = __shfl_xor_sync(0xffffffffu, static_cast<uint32_t>(v >> 32), o);
  return (static_cast<uint64_t>(hi) << 32) | lo;
}
__device__ __forceinline__ uint64_t shfl_u64(uint64_t v, int src) {
  const uint32_t lo = __shfl_sync(0xffffffffu, static_cast<uint32_t>(v), src);
  const uint32_t hi = __shfl_sync(0xffffffffu, static_cast<uint32_t>(v >> 32), src);
  return (static_cast<uint64_t>(hi) << 32) | lo;
}

// Bitonic sort of one value per lane, descending over the lanes (15 compare-exchange steps).
__device__ __forceinline__ uint64_t warp_sort_desc(uint64_t v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      const uint64_t o = shfl_xor_u64(v, j);
      const bool keep_max = ((lane & k) == 0) == ((lane & j) == 0);
      v = keep_max ? (v > o ? v : o) : (v < o ? v : o);
    }
  }
  return v;
}

// The 32 largest of two descending lists (one entry per lane), descending: the elementwise max
// of a and reversed b is bitonic and holds them; a half-cleaner cascade sorts it.
__device__ __forceinline__ uint64_t warp_merge_top32(uint64_t a, uint64_t b) {
  const int lane = threadIdx.x & 31;
  const uint64_t br = shfl_u64(b, 31 - lane);
  uint64_t v = a > br ? a : br;
#pragma unroll
  for (int j = 16; j > 0; j >>= 1) {
    const uint64_t o = shfl_xor_u64(v, j);
    const bool lower = (lane & j) == 0;
    v = lower ? (v > o ? v : o) : (v < o ? v : o);
  }
  return v;
}

// Ascending bitonic sort of one int per lane.
__device__ __forceinline__ int warp_sort_asc(int v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      const int o = __shfl_xor_sync(0xffffffffu, v, j);
      const bool keep_min = ((lane & k) == 0) == ((lane & j) == 0);
      v = keep_min ? min(v, o) : max(v, o);
    }
  }
  return v;
}

// Named CTA barriers over `n` threads (a multiple of 32): a producer arrives, a consumer waits.
__device__ __forceinline__ void named_bar_arrive(int id, int n) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void named_bar_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

}  // namespace compkv
