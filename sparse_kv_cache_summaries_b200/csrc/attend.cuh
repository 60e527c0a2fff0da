// Per-tile attention pieces shared by the sparse (selected blocks) and dense decode kernels:
// logits of shared-memory K rows against the G query heads of a kv-head, and P.V accumulation.
#pragma once

#include "common.cuh"

namespace compkv {

// Row geometry for 16-byte vector loads of a [rows][D] tile of element type T.
template <typename T, int D>
struct RowGeom {
  static constexpr int kEpv = 16 / static_cast<int>(sizeof(T));  // elements per vector
  static constexpr int kLpr = D / kEpv;                          // lanes per row
  static constexpr int kRpl = 32 / kLpr;                         // rows per warp per pass
  static_assert(kLpr >= 8 && kLpr <= 32, "unsupported head_dim / dtype");
};

// Transpose-reduce: NV partial values per lane, summed over the L lanes of an aligned lane
// group (xor offsets < L). At each of the first log2(NV) levels a lane keeps half of its values
// and receives the partner's half of the other ones, so the shuffle count is NV - 1 +
// log2(L / NV) instead of NV log2(L). Afterwards lane li of the group holds the total of value
// index li / (L / NV) in v[0].
template <int NV, int O>
struct TransposeReduce {
  static __device__ __forceinline__ void run(float* v, int li) {
    if constexpr (O > 0) {
      if constexpr (NV > 1) {
        constexpr int H = NV / 2;
        const bool upper = (li & O) != 0;
#pragma unroll
        for (int i = 0; i < H; ++i) {
          const float send = upper ? v[i] : v[i + H];
          const float keep = upper ? v[i + H] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, O);
        }
        TransposeReduce<H, O / 2>::run(v, li);
      } else {
        v[0] += __shfl_xor_sync(0xffffffffu, v[0], O);
        TransposeReduce<1, O / 2>::run(v, li);
      }
    }
  }
};

template <typename T, int EPV>
__device__ __forceinline__ void vec_to_floats(const uint4& w, float (&f)[EPV]) {
  if constexpr (sizeof(T) == 2) {
    unpack8_bf16(w, f);
  } else {
    f[0] = __uint_as_float(w.x);
    f[1] = __uint_as_float(w.y);
    f[2] = __uint_as_float(w.z);
    f[3] = __uint_as_float(w.w);
  }
}

// q registers of one lane: the kEpv channels at li * kEpv, for the G heads (fp32 from smem).
template <typename T, int D, int G>
__device__ __forceinline__ void load_q_regs(const float* q_s, int li,
                                            float (&qr)[G][RowGeom<T, D>::kEpv]) {
  constexpr int EPV = RowGeom<T, D>::kEpv;
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < EPV; ++e) qr[h][e] = q_s[h * D + li * EPV + e];
}

// Scaled logits s * q_h . k_row for rows [0, R) of a shared-memory tile (row stride D). R must be
// a multiple of kWarps * kRpl. Writes lg[h * ld + row], -inf where valid(row) is false.
template <typename T, int D, int G, typename Valid>
__device__ __forceinline__ void tile_logits(const T* rows, int R, const float (&qr)[G][RowGeom<T, D>::kEpv],
                                            float scale, float* lg, int ld, Valid valid) {
  using RG = RowGeom<T, D>;
  constexpr int EPV = RG::kEpv, LPR = RG::kLpr, RPL = RG::kRpl, LPH = LPR / G;
  static_assert(G <= LPR, "more heads than lanes per row");
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int li = lane % LPR, rs = lane / LPR;
  for (int base = warp * RPL; base < R; base += kWarps * RPL) {
    const int row = base + rs;
    const uint4 w = reinterpret_cast<const uint4*>(rows + static_cast<size_t>(row) * D)[li];
    float f[EPV];
    vec_to_floats<T, EPV>(w, f);
    float v[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float s = 0.f;
#pragma unroll
      for (int e = 0; e < EPV; ++e) s = fmaf(qr[h][e], f[e], s);
      v[h] = s;
    }
    TransposeReduce<G, LPR / 2>::run(v, li);
    if ((li % LPH) == 0) lg[(li / LPH) * ld + row] = valid(row) ? scale * v[0] : -CUDART_INF_F;
  }
}

// P.V over rows [r0, r1) for one thread: VEC channels (4 bytes of T) at cv * VEC, G heads.
// pT is [row][G] (weights), rows are [row][D] elements of T.
template <typename T, int D, int G>
struct PV {
  static constexpr int kVec = 4 / static_cast<int>(sizeof(T));  // channels per 4-byte word
  static constexpr int kCols = D / kVec;                         // threads per row
  static constexpr int kSub = kThreads / kCols;                  // row subsets
  __device__ __forceinline__ static void accumulate(const T* rows, const float* pT, int R, int sub,
                                                    int cv, float (&acc)[G][kVec]) {
    for (int row = sub; row < R; row += kSub) {
      float v[kVec];
      if constexpr (sizeof(T) == 2) {
        const uint32_t w = reinterpret_cast<const uint32_t*>(rows + static_cast<size_t>(row) * D)[cv];
        v[0] = __uint_as_float(w << 16);
        v[1] = __uint_as_float(w & 0xffff0000u);
      } else {
        v[0] = reinterpret_cast<const float*>(rows + static_cast<size_t>(row) * D)[cv];
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float p = pT[row * G + h];
#pragma unroll
        for (int e = 0; e < kVec; ++e) acc[h][e] = fmaf(p, v[e], acc[h][e]);
      }
    }
  }
};

}  // namespace compkv
