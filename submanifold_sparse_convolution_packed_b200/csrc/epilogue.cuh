// Conv output epilogue shared by the conv kernels and the norm kernels:
// activation, residual, and the per-(batch item, channel group) sums that a
// following GroupNorm normalises with (the layers around the decoders'
// convs: Pixal3D MLX README "Status", LATO.2 MLX port README "Status").
#pragma once

#include <cstdint>

#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace smc {

enum Act : int { kActNone = 0, kActRelu = 1, kActSilu = 2 };

// Options of a fused conv epilogue, y = act(conv + bias) + residual, and of
// the group statistics kernel (coords, stats, stripes, batch, groups).
struct Epilogue {
  const void* residual = nullptr;  // [n, cout] in the output type, or null (may equal out)
  const int32_t* coords = nullptr; // [n, 4] rows (b, z, y, x): b indexes the statistics
  double* stats = nullptr;         // [stripes, batch, groups, 3] += (sum, sum of squares, count)
  int stripes = 1;                 // copies of the statistics; block b adds into copy b % stripes
  int batch = 0;
  int groups = 1;                  // channels per group
  int act = kActNone;
};

// Statistics copy of this block: blocks add into one of `stripes` copies so
// that concurrent atomics on one (item, group) are spread over that many
// addresses; the copies are folded afterwards (k_stats_fold).
__device__ __forceinline__ double* stats_copy(const Epilogue& ep) {
  return ep.stats + static_cast<int64_t>(blockIdx.x % ep.stripes) * ep.batch * ep.groups * 3;
}

__device__ __forceinline__ float apply_act(float y, int act) {
  if (act == kActRelu) return fmaxf(y, 0.f);
  // y * sigmoid(y) with the fast exponential and a rounded reciprocal: within
  // a few fp32 ulp of y / (1 + exp(-y)), far below the output's rounding
  if (act == kActSilu) return y * __frcp_rn(1.f + __expf(-y));
  return y;
}

__device__ __forceinline__ float half_bits_to_float(uint16_t h, bool bf16) {
  return bf16 ? __bfloat162float(__ushort_as_bfloat16(h)) : __half2float(__ushort_as_half(h));
}

__device__ __forceinline__ uint16_t float_to_half_bits(float x, bool bf16) {
  return bf16 ? __bfloat16_as_ushort(__float2bfloat16_rn(x)) : __half_as_ushort(__float2half_rn(x));
}

// K values per lane (K a power of two, at most 32).  After this, lane l
// holds in w[0] the sum over all lanes of their w[l mod K]: first plain
// butterfly additions across lane distances >= K, then five minus log2(K)
// exchange steps in which each lane keeps one half of its values and
// receives the partner's half of the other.
template <int K>
__device__ __forceinline__ void transpose_reduce(double (&w)[K]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int s = 16; s >= K; s >>= 1) {
#pragma unroll
    for (int i = 0; i < K; ++i) w[i] += __shfl_xor_sync(0xffffffffu, w[i], s);
  }
#pragma unroll
  for (int s = K / 2; s >= 1; s >>= 1) {
    const bool up = (lane & s) != 0;
#pragma unroll
    for (int i = 0; i < s; ++i) {
      const double send = up ? w[i] : w[i + s];
      const double keep = up ? w[i + s] : w[i];
      w[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
    }
  }
}

// Whole-warp case with groups of G (dividing 32) channels aligned to the run:
// per lane the run's G-channel sums and sums of squares, then one transposing
// reduction; lane l adds value l.
// Lanes with `mine` false contribute zeros.
template <int G>
__device__ __forceinline__ void warp_group_stats_aligned(const float (&v)[32], bool mine, int c0, int ncols, int b,
                                                         int groups, double* sink, int rows) {
  constexpr int NG = 32 / G;
  const int lane = threadIdx.x & 31;
  double* row = sink + static_cast<int64_t>(b) * groups * 3;
  const int g0 = c0 / G;
  const int live = ncols / G;  // groups of this run with values
  if (NG <= 16) {
    // per lane: the run's NG group sums, then their NG sums of squares
    double w[2 * NG];
#pragma unroll
    for (int k = 0; k < NG; ++k) {
      double s1 = 0.0, s2 = 0.0;
#pragma unroll
      for (int j = 0; j < G; ++j) {
        const float x = mine ? v[k * G + j] : 0.f;
        s1 += x;
        s2 += static_cast<double>(x) * x;
      }
      w[k] = s1;
      w[NG + k] = s2;
    }
    transpose_reduce<2 * NG>(w);
    if (lane < 2 * NG && (lane % NG) < live) atomicAdd(row + (g0 + lane % NG) * 3 + lane / NG, w[0]);
    if (lane < live) atomicAdd(row + (g0 + lane) * 3 + 2, static_cast<double>(rows) * G);
  } else {  // G == 1: 32 groups, the sums and then the squares reduced in turn
    double w[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) w[k] = mine ? v[k] : 0.f;
    transpose_reduce<32>(w);
    if (lane < live) atomicAdd(row + (g0 + lane) * 3 + 0, w[0]);
#pragma unroll
    for (int k = 0; k < 32; ++k) w[k] = mine ? static_cast<double>(v[k]) * v[k] : 0.0;
    transpose_reduce<32>(w);
    if (lane < live) {
      atomicAdd(row + (g0 + lane) * 3 + 1, w[0]);
      atomicAdd(row + (g0 + lane) * 3 + 2, static_cast<double>(rows));
    }
  }
}

// Group statistics of the output channels c0 .. c0+ncols-1 (ncols <= 32) of
// this lane's row: v[j] is the stored value of channel c0 + j (0 past ncols);
// `valid` is false for lanes without a row (or with a batch index outside the
// stats).  Groups are runs of gch channels; G = gch when gch divides 32 (the
// run then holds whole groups: one transposing reduction per batch item
// present in the warp), else G = 0 (per group, a warp sum when all 32 lanes
// hold rows of one item, otherwise every lane adds its own row).  `sink` is
// the [batch, groups, 3] array the sums are added to.  Warp-collective:
// every lane of the warp calls it.
template <int G>
__device__ __forceinline__ void warp_group_stats(const float (&v)[32], int c0, int ncols, bool valid, int b,
                                                 int gch, int groups, double* sink) {
  const int lane = threadIdx.x & 31;
  if constexpr (G > 0) {
    // lanes of other items and lanes without rows contribute zeros
    uint32_t todo = __ballot_sync(0xffffffffu, valid);
    while (todo) {
      const int bb = __shfl_sync(0xffffffffu, b, __ffs(todo) - 1);
      const bool mine = valid && b == bb;
      const uint32_t rows = __ballot_sync(0xffffffffu, mine);
      warp_group_stats_aligned<G>(v, mine, c0, ncols, bb, groups, sink, __popc(rows));
      todo &= ~rows;
    }
  } else {
    const int b0 = __shfl_sync(0xffffffffu, b, 0);
    const bool whole = __all_sync(0xffffffffu, valid && b == b0);
    const int g_first = c0 / gch, g_last = (c0 + ncols - 1) / gch;
    for (int g = g_first; g <= g_last; ++g) {
      const int lo = (g * gch > c0 ? g * gch : c0) - c0;
      const int hi = ((g + 1) * gch < c0 + ncols ? (g + 1) * gch : c0 + ncols) - c0;
      double d1 = 0.0, d2 = 0.0;  // fp64 from the first term: E[y^2] - E[y]^2 needs it
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (j >= lo && j < hi) {
          d1 += v[j];
          d2 += static_cast<double>(v[j]) * v[j];
        }
      if (whole) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          d1 += __shfl_xor_sync(0xffffffffu, d1, o);
          d2 += __shfl_xor_sync(0xffffffffu, d2, o);
        }
      }
      if (whole ? lane == 0 : valid) {
        double* st = sink + (static_cast<int64_t>(b) * groups + g) * 3;
        atomicAdd(st + 0, d1);
        atomicAdd(st + 1, d2);
        atomicAdd(st + 2, static_cast<double>(whole ? 32 : 1) * (hi - lo));
      }
    }
  }
}

}  // namespace smc
