// Warp-wide sorted lists of L = 32 E entries for the select-and-attend kernel's Top-K when
// K_b is above 32 (E = 2 or 4): entry i is slot i / 32 of lane i % 32, so compare-exchange
// strides of 32 and more stay inside a lane (slot s against slot s ^ (stride / 32)) and smaller
// strides are shuffles within one slot. The networks are the bitonic sorting network and the
// merge of two sorted lists through the elementwise max of one with the other reversed followed
// by a half-cleaner cascade (Batcher's bitonic merge), written out for this layout.
#pragma once

#include "common.cuh"

namespace compkv {

// (a, b) <- (max, min) if a_max, else (min, max).
__device__ __forceinline__ void cmpx_u64(uint64_t& a, uint64_t& b, bool a_max) {
  const uint64_t hi = a > b ? a : b, lo = a > b ? b : a;
  a = a_max ? hi : lo;
  b = a_max ? lo : hi;
}

// Sorts the warp's L entries into descending order.
template <int E>
__device__ __forceinline__ void list_sort_desc(uint64_t (&v)[E]) {
  const int lane = threadIdx.x & 31;
  constexpr int L = 32 * E;
#pragma unroll
  for (int k = 2; k <= L; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      if (j >= 32) {
#pragma unroll
        for (int s = 0; s < E; ++s) {
          const int t = s ^ (j >> 5);
          if (t > s) cmpx_u64(v[s], v[t], ((s * 32 + lane) & k) == 0);  // the lower entry keeps the max
        }
      } else {
#pragma unroll
        for (int s = 0; s < E; ++s) {
          const int i = s * 32 + lane;
          const uint64_t o = shfl_xor_u64(v[s], j);
          const bool keep_max = ((i & k) == 0) == ((i & j) == 0);
          v[s] = keep_max ? (v[s] > o ? v[s] : o) : (v[s] < o ? v[s] : o);
        }
      }
    }
  }
}

// a <- the L largest of the descending lists a and b, descending.
template <int E>
__device__ __forceinline__ void list_merge_top(uint64_t (&a)[E], const uint64_t (&b)[E]) {
  const int lane = threadIdx.x & 31;
  constexpr int L = 32 * E;
#pragma unroll
  for (int s = 0; s < E; ++s) {  // entry i of reversed b is b[L - 1 - i]
    const uint64_t br = shfl_u64(b[E - 1 - s], 31 - lane);
    a[s] = a[s] > br ? a[s] : br;
  }
#pragma unroll
  for (int j = L >> 1; j > 0; j >>= 1) {
    if (j >= 32) {
#pragma unroll
      for (int s = 0; s < E; ++s) {
        const int t = s ^ (j >> 5);
        if (t > s) cmpx_u64(a[s], a[t], true);
      }
    } else {
#pragma unroll
      for (int s = 0; s < E; ++s) {
        const uint64_t o = shfl_xor_u64(a[s], j);
        a[s] = ((lane & j) == 0) ? (a[s] > o ? a[s] : o) : (a[s] < o ? a[s] : o);
      }
    }
  }
}

// Sorts the warp's L ints into ascending order.
template <int E>
__device__ __forceinline__ void list_sort_asc(int (&v)[E]) {
  const int lane = threadIdx.x & 31;
  constexpr int L = 32 * E;
#pragma unroll
  for (int k = 2; k <= L; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      if (j >= 32) {
#pragma unroll
        for (int s = 0; s < E; ++s) {
          const int t = s ^ (j >> 5);
          if (t > s) {
            const bool lo_min = ((s * 32 + lane) & k) == 0;  // the lower entry keeps the min
            const int mn = min(v[s], v[t]), mx = max(v[s], v[t]);
            v[s] = lo_min ? mn : mx;
            v[t] = lo_min ? mx : mn;
          }
        }
      } else {
#pragma unroll
        for (int s = 0; s < E; ++s) {
          const int i = s * 32 + lane;
          const int o = __shfl_xor_sync(0xffffffffu, v[s], j);
          const bool keep_min = ((i & k) == 0) == ((i & j) == 0);
          v[s] = keep_min ? min(v[s], o) : max(v[s], o);
        }
      }
    }
  }
}

// The 8 warps' descending lists merged pairwise in 3 levels through `lists` ([kWarps][L]) and
// named barriers (ids 1..7) shared by the two warps of a pair; warp 0 ends with the CTA's
// best L. No CTA-wide barrier.
template <int E>
__device__ __forceinline__ void list_pairs_merge(uint64_t (&best)[E], uint64_t* lists) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int L = 32 * E;
  int id = 1;
#pragma unroll
  for (int s = 1; s < kWarps; s <<= 1) {
    if ((warp & (2 * s - 1)) == s) {  // producer at this level, done afterwards
#pragma unroll
      for (int e = 0; e < E; ++e) lists[warp * L + e * 32 + lane] = best[e];
      named_bar_arrive(id + (warp - s) / (2 * s), 64);
    } else if ((warp & (2 * s - 1)) == 0) {
      named_bar_sync(id + warp / (2 * s), 64);
      uint64_t b[E];
#pragma unroll
      for (int e = 0; e < E; ++e) b[e] = lists[(warp + s) * L + e * 32 + lane];
      list_merge_top<E>(best, b);
    }
    id += kWarps / (2 * s);
  }
}

}  // namespace compkv
