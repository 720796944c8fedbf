// The layers around the decoders' convs (Pixal3D MLX README "Status": norms,
// activations, ResBlock; LATO.2 MLX port README "Status": SparseGroupNorm32).
// The population of a (batch item, channel group) is every active row of the
// item times the group's channels.
//   k_rows_pass    behind a conv: y = act(x) + residual in row order, and the
//                  (sum, sum of squares, count) of the stored values per
//                  (item, group) into striped fp64 copies of a
//                  [batch, groups, 3] array, folded by k_stats_fold; with no
//                  y, the statistics of x alone.
//   k_group_norm   y = act(gamma * (x - mean) * rsqrt(var + eps) + beta), with
//                  mean and (biased) variance from such statistics.
// The tensor-core conv stores its tile rows in schedule order; doing the
// activation and residual here, in row order, measured faster than in the
// conv's epilogue, where they lengthen every tile's hold on its SM slot.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <type_traits>

#include "common.cuh"
#include "epilogue.cuh"
#include "kernels.h"

namespace smc {

namespace {

constexpr int kNormThreads = 256;
constexpr int kMaxBatchGroups = 1024;  // batch * groups held in shared memory


template <typename T> __device__ __forceinline__ float ld_f(const T* p, int64_t i);
template <> __device__ __forceinline__ float ld_f<float>(const float* p, int64_t i) { return p[i]; }
template <> __device__ __forceinline__ float ld_f<__nv_bfloat16>(const __nv_bfloat16* p, int64_t i) {
  return __bfloat162float(p[i]);
}
template <> __device__ __forceinline__ float ld_f<__half>(const __half* p, int64_t i) { return __half2float(p[i]); }

template <typename T> __device__ __forceinline__ T st_f(float x);
template <> __device__ __forceinline__ float st_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 st_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }
template <> __device__ __forceinline__ __half st_f<__half>(float x) { return __float2half_rn(x); }

// The row pass behind a conv: one thread per row, a warp per 32 consecutive
// rows (grid-stride over warps).  Per 32-channel run of the row: x and the
// residual are loaded (16-byte vectors when the rows allow), y = act(x) +
// residual is rounded to T and stored (when y is given; y may be x, and the
// residual may be x too: every element is read before it is written, by the
// same thread), and the group statistics of the stored values are reduced by
// warp_group_stats into this warp's own shared-memory sums (the block's, when
// the batch x group table is too large for one per warp).  The block's sums
// reach its striped global copy once.  Rows outside the statistics' batch
// range are transformed but not counted.
template <typename T, bool kStats, int G>
__global__ void __launch_bounds__(kNormThreads) k_rows_pass(const T* x, T* y, const T* residual, int act, int64_t n,
                                                            int c, const int32_t* __restrict__ coords, Epilogue ep,
                                                            int vec, int per_warp) {
  extern __shared__ double s_acc[];
  constexpr bool do_stats = kStats;
  const int entries = do_stats ? ep.batch * ep.groups * 3 : 0;
  const int warp = threadIdx.x >> 5;
  const int sinks = per_warp ? kNormThreads / 32 : 1;
  for (int i = threadIdx.x; i < sinks * entries; i += kNormThreads) s_acc[i] = 0.0;
  __syncthreads();
  double* sink = s_acc + (per_warp ? warp * entries : 0);
  const int gch = do_stats ? c / ep.groups : 1;
  constexpr int kPer = 16 / sizeof(T);
  const int64_t rows_all = (n + 31) / 32 * 32;  // every lane of a warp runs every round
  for (int64_t row = blockIdx.x * static_cast<int64_t>(kNormThreads) + threadIdx.x; row < rows_all;
       row += static_cast<int64_t>(gridDim.x) * kNormThreads) {
    const bool live = row < n;
    int b = -1;
    if (do_stats && live) {
      b = coords[4 * row];
      if (b < 0 || b >= ep.batch) b = -1;
    }
    for (int c0 = 0; c0 < c; c0 += 32) {
      const int ncols = c - c0 < 32 ? c - c0 : 32;
      const bool whole = live && vec && ncols == 32;
      const int64_t at = row * c + c0;
      float v[32];
      if (whole) {
#pragma unroll
        for (int q = 0; q < 32 / kPer; ++q) {
          const uint4 u = *reinterpret_cast<const uint4*>(x + at + q * kPer);
          const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
          for (int j = 0; j < kPer; ++j) v[q * kPer + j] = ld_f<T>(e, j);
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = (live && j < ncols) ? ld_f<T>(x + at, j) : 0.f;
      }
      if (y) {
        // y = act(x) + residual, 16 bytes at a time; v keeps the stored values
        if (whole) {
#pragma unroll
          for (int q = 0; q < 32 / kPer; ++q) {
            uint4 rv = make_uint4(0, 0, 0, 0);
            if (residual) rv = *reinterpret_cast<const uint4*>(residual + at + q * kPer);
            const T* re = reinterpret_cast<const T*>(&rv);
            uint4 o;
            T* oe = reinterpret_cast<T*>(&o);
#pragma unroll
            for (int j = 0; j < kPer; ++j) {
              oe[j] = st_f<T>(apply_act(v[q * kPer + j], act) + (residual ? ld_f<T>(re, j) : 0.f));
              v[q * kPer + j] = ld_f<T>(oe, j);
            }
            *reinterpret_cast<uint4*>(y + at + q * kPer) = o;
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            if (live && j < ncols) {
              const T t = st_f<T>(apply_act(v[j], act) + (residual ? ld_f<T>(residual + at, j) : 0.f));
              y[at + j] = t;
              v[j] = ld_f<T>(&t, 0);
            }
          }
        }
      }
      if constexpr (kStats) warp_group_stats<G>(v, c0, ncols, b >= 0, b < 0 ? 0 : b, gch, ep.groups, sink);
    }
  }
  if constexpr (!kStats) return;
  __syncthreads();
  double* gst = stats_copy(ep);
  for (int i = threadIdx.x; i < entries; i += kNormThreads) {
    double t = 0.0;
    for (int w = 0; w < sinks; ++w) t += s_acc[w * entries + i];
    if (t != 0.0) atomicAdd(gst + i, t);
  }
}

// The same pass over the flat [n, c] array, coalesced: a thread takes units
// of kU elements (16 bytes, or one element) at a fixed stride of whole rows
// (the grid's thread count is a multiple of the units per row), so its
// units are always the same channels ch0 .. ch0+kU-1 of successive rows.
// With statistics it keeps fp64 per-channel sums of the stored values in
// registers and adds them into the (item, group) sums of its warp's shared
// array only when its rows' batch item changes, and at the end.
// kG: channels per group when every group of the unit is whole and
// lies in it or holds it (a power of two; kG >= kU: the unit lies in one
// group), else 0 (sums per channel, added to their groups at a flush).
// Accumulator slots of a k_rows_flat thread with statistics (see kSlots).
constexpr int flat_slots(int u, int g) { return g == 0 ? u : u / (g < u ? g : u); }

// With statistics and at most four accumulator slots the kernel is held to
// 64 registers (four blocks per SM): measured faster than 74 registers at
// three blocks.  With more slots (one channel per group) that would spill.
template <typename T, bool kStats, int kU, int kG>
__global__ void __launch_bounds__(kNormThreads, kStats && flat_slots(kU, kG) <= 4 ? 4 : 1) k_rows_flat(const T* x, T* y, const T* residual, int act, int64_t n,
                                                            int c, const int32_t* __restrict__ coords, Epilogue ep) {
  extern __shared__ double s_acc[];
  constexpr int kWarps = kNormThreads / 32;
  const int entries = kStats ? ep.batch * ep.groups * 3 : 0;
  if constexpr (kStats) {
    for (int i = threadIdx.x; i < kWarps * entries; i += kNormThreads) s_acc[i] = 0.0;
    __syncthreads();
  }
  double* sink = s_acc + (threadIdx.x >> 5) * entries;
  const int units = c / kU;  // per row
  const int64_t total = n * units;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kNormThreads;
  const int64_t t0 = blockIdx.x * static_cast<int64_t>(kNormThreads) + threadIdx.x;
  const int ch0 = static_cast<int>(t0 % units) * kU;
  const int gch = kStats ? c / ep.groups : 1;
  using Vec = typename std::conditional<kU == 1, T, uint4>::type;
  // accumulator slots: one per group of the unit, or one per channel
  constexpr int kPerSlot = kG == 0 ? 1 : (kG < kU ? kG : kU);  // channels of the unit per slot
  constexpr int kSlots = kU / kPerSlot;
  double s1[kSlots], s2[kSlots];
#pragma unroll
  for (int k = 0; k < kSlots; ++k) s1[k] = s2[k] = 0.0;
  int64_t cnt = 0;
  int cur = -1;
  auto flush = [&]() {
    if (cur >= 0 && cnt > 0) {
#pragma unroll
      for (int k = 0; k < kSlots; ++k) {
        double* st = sink + (static_cast<int64_t>(cur) * ep.groups + (ch0 + k * kPerSlot) / gch) * 3;
        atomicAdd(st + 0, s1[k]);
        atomicAdd(st + 1, s2[k]);
        atomicAdd(st + 2, static_cast<double>(cnt) * kPerSlot);
      }
    }
#pragma unroll
    for (int k = 0; k < kSlots; ++k) s1[k] = s2[k] = 0.0;
    cnt = 0;
  };
  // kFlatUnroll units per thread and round, all loaded before any is
  // processed (they are distinct addresses, so this holds in place too);
  // two per round measured slower than one, with and without statistics
  constexpr int kFlatUnroll = 1;
  for (int64_t t = t0; t < total; t += kFlatUnroll * stride) {
    Vec u[kFlatUnroll], rv[kFlatUnroll];
#pragma unroll
    for (int k = 0; k < kFlatUnroll; ++k) {
      const int64_t tk = t + k * stride;
      if (tk < total) {
        u[k] = reinterpret_cast<const Vec*>(x)[tk];
        if (y && residual) rv[k] = reinterpret_cast<const Vec*>(residual)[tk];
      }
    }
#pragma unroll
    for (int k = 0; k < kFlatUnroll; ++k) {
      const int64_t tk = t + k * stride;
      if (tk >= total) break;
      const int64_t row = tk / units;
      const T* e = reinterpret_cast<const T*>(&u[k]);
      float v[kU];
#pragma unroll
      for (int j = 0; j < kU; ++j) v[j] = ld_f<T>(e, j);
      if (y) {
        const T* re = reinterpret_cast<const T*>(&rv[k]);
        Vec o;
        T* oe = reinterpret_cast<T*>(&o);
#pragma unroll
        for (int j = 0; j < kU; ++j) {
          oe[j] = st_f<T>(apply_act(v[j], act) + (residual ? ld_f<T>(re, j) : 0.f));
          v[j] = ld_f<T>(oe, j);  // the statistics are those of the stored values
        }
        reinterpret_cast<Vec*>(y)[tk] = o;
      }
      if constexpr (kStats) {
        int b = coords[4 * row];
        if (b < 0 || b >= ep.batch) b = -1;
        if (b != cur) {
          flush();
          cur = b;
        }
        if (b >= 0) {
#pragma unroll
          for (int k = 0; k < kSlots; ++k) {
            double a1 = 0.0, a2 = 0.0;  // fp64 from the first term: E[y^2] - E[y]^2 needs it
#pragma unroll
            for (int j = 0; j < kPerSlot; ++j) {
              a1 += v[k * kPerSlot + j];
              a2 += static_cast<double>(v[k * kPerSlot + j]) * v[k * kPerSlot + j];
            }
            s1[k] += a1;
            s2[k] += a2;
          }
          ++cnt;
        }
      }
    }
  }
  if constexpr (kStats) {
    flush();
    __syncthreads();
    double* gst = stats_copy(ep);
    for (int i = threadIdx.x; i < entries; i += kNormThreads) {
      double t = 0.0;
      for (int w = 0; w < kWarps; ++w) t += s_acc[w * entries + i];
      if (t != 0.0) atomicAdd(gst + i, t);
    }
  }
}

// stats[i] += sum over the copies of copies[s][i].
__global__ void k_stats_fold(const double* __restrict__ copies, int stripes, int64_t len, double* __restrict__ stats) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < len;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    double t = 0.0;
#pragma unroll 8
    for (int s = 0; s < stripes; ++s) t += copies[s * len + i];
    stats[i] += t;
  }
}

template <typename T>
__global__ void __launch_bounds__(kNormThreads) k_group_norm(const T* __restrict__ x, int64_t n, int c,
                                                             const int32_t* __restrict__ coords, int batch, int groups,
                                                             const double* __restrict__ stats,
                                                             const T* __restrict__ gamma, const T* __restrict__ beta,
                                                             float eps, int act, T* __restrict__ out) {
  __shared__ float s_mean[kMaxBatchGroups];
  __shared__ float s_rstd[kMaxBatchGroups];
  const int bg = batch * groups;
  for (int i = threadIdx.x; i < bg; i += kNormThreads) {
    const double cnt = stats[3 * i + 2] > 0.0 ? stats[3 * i + 2] : 1.0;
    const double mean = stats[3 * i + 0] / cnt;
    double var = stats[3 * i + 1] / cnt - mean * mean;
    if (var < 0.0) var = 0.0;
    s_mean[i] = static_cast<float>(mean);
    s_rstd[i] = static_cast<float>(1.0 / sqrt(var + static_cast<double>(eps)));
  }
  __syncthreads();
  const int gch = c / groups;
  const int64_t total = n * c;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(kNormThreads) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * kNormThreads) {
    const int64_t row = i / c;
    const int ch = static_cast<int>(i - row * c);
    int b = coords[4 * row];
    if (b < 0 || b >= batch) b = 0;  // rows outside the statistics: normalised with item 0's
    const int k = b * groups + ch / gch;
    float y = (ld_f<T>(x, i) - s_mean[k]) * s_rstd[k];
    if (gamma) y *= ld_f<T>(gamma, ch);
    if (beta) y += ld_f<T>(beta, ch);
    out[i] = st_f<T>(apply_act(y, act));
  }
}

unsigned grid_for(int64_t total) {
  const int64_t blocks = (total + kNormThreads - 1) / kNormThreads;
  return static_cast<unsigned>(blocks < 148 * 16 ? (blocks > 0 ? blocks : 1) : 148 * 16);
}

}  // namespace

static int64_t gcd64(int64_t a, int64_t b) {
  while (b) {
    const int64_t t = a % b;
    a = b;
    b = t;
  }
  return a;
}

cudaError_t launch_rows_pass(const void* x, void* y, const void* residual, int act, int64_t n, int c,
                             const int32_t* coords, const Epilogue& ep, int dtype, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  const int entries = ep.stats ? ep.batch * ep.groups * 3 : 0;
  if (entries > kMaxBatchGroups * 3) return cudaErrorInvalidValue;
  constexpr int kWarps = kNormThreads / 32;
  const int es = dtype == kF32 ? 4 : 2;
  const bool aligned = (reinterpret_cast<uintptr_t>(x) & 15u) == 0 && (reinterpret_cast<uintptr_t>(y) & 15u) == 0 &&
                       (reinterpret_cast<uintptr_t>(residual) & 15u) == 0;
  const int vec = (static_cast<int64_t>(c) * es) % 16 == 0 && aligned;
  // Flat coalesced pass: the thread count must be a multiple of the units
  // per row, within the grid cap, and (with statistics) every warp's sums
  // must fit the default 48 KB of dynamic shared memory.
  const int64_t units = vec ? static_cast<int64_t>(c) * es / 16 : c;
  const int64_t step = units / gcd64(units, kNormThreads);  // blocks per whole number of rows
  const int64_t want = (n * units + kNormThreads - 1) / kNormThreads;
  const int64_t cap = 148 * 8;
  int64_t blocks = (want < cap ? want : cap + step - 1) / step * step;
  if (blocks < step) blocks = step;
  const size_t flat_smem = static_cast<size_t>(entries) * kWarps * sizeof(double);
  // For statistics alone on rows under 256 bytes (64-channel bf16/fp16) the
  // per-row kernel measured faster (decoder stage 3: 113 vs 123 us; a thread
  // keeps its whole row in flight); with the transform too, this one (721 vs
  // 772 us for the conv and the pass).
  const bool flat = step <= cap && flat_smem <= 48 * 1024 &&
                    (!ep.stats || y != nullptr || static_cast<int64_t>(c) * es >= 256);
  if (flat) {
    const unsigned g = static_cast<unsigned>(blocks);
    auto run = [&](auto tag, auto per) {
      using T = decltype(tag);
      constexpr int kU = decltype(per)::value;
      const T* xt = static_cast<const T*>(x);
      T* yt = static_cast<T*>(y);
      const T* rt = static_cast<const T*>(residual);
      const int gch = ep.stats ? c / ep.groups : 0;
      if (!ep.stats) {
        k_rows_flat<T, false, kU, 0><<<g, kNormThreads, 0, s>>>(xt, yt, rt, act, n, c, coords, ep);
      } else if (kU == 1 || (gch >= kU && gch % kU == 0)) {  // the unit lies in one group
        k_rows_flat<T, true, kU, kU><<<g, kNormThreads, flat_smem, s>>>(xt, yt, rt, act, n, c, coords, ep);
      } else if (gch == 1) {
        k_rows_flat<T, true, kU, 1><<<g, kNormThreads, flat_smem, s>>>(xt, yt, rt, act, n, c, coords, ep);
      } else if (gch == 2) {
        k_rows_flat<T, true, kU, 2><<<g, kNormThreads, flat_smem, s>>>(xt, yt, rt, act, n, c, coords, ep);
      } else if (gch == 4 && kU >= 4) {
        k_rows_flat<T, true, kU, 4><<<g, kNormThreads, flat_smem, s>>>(xt, yt, rt, act, n, c, coords, ep);
      } else {
        k_rows_flat<T, true, kU, 0><<<g, kNormThreads, flat_smem, s>>>(xt, yt, rt, act, n, c, coords, ep);
      }
    };
    switch (dtype) {
      case kF32:
        if (vec) run(float{}, std::integral_constant<int, 4>());
        else run(float{}, std::integral_constant<int, 1>());
        break;
      case kBF16:
        if (vec) run(__nv_bfloat16{}, std::integral_constant<int, 8>());
        else run(__nv_bfloat16{}, std::integral_constant<int, 1>());
        break;
      case kF16:
        if (vec) run(__half{}, std::integral_constant<int, 8>());
        else run(__half{}, std::integral_constant<int, 1>());
        break;
      default:
        return cudaErrorInvalidValue;
    }
    count_launches(1);
    return cudaGetLastError();
  }
  // otherwise one thread per row
  const int per_warp = entries * kWarps * 8 <= 48 * 1024 ? 1 : 0;
  const size_t smem = static_cast<size_t>(entries) * (per_warp ? kWarps : 1) * sizeof(double);
  const int64_t rblocks = (n + kNormThreads - 1) / kNormThreads;
  const unsigned g = static_cast<unsigned>(rblocks < cap ? rblocks : cap);
  auto run = [&](auto tag) {
    using T = decltype(tag);
    const T* xt = static_cast<const T*>(x);
    T* yt = static_cast<T*>(y);
    const T* rt = static_cast<const T*>(residual);
    const int gch = ep.stats ? c / ep.groups : 0;
    if (!ep.stats)
      k_rows_pass<T, false, 0><<<g, kNormThreads, 0, s>>>(xt, yt, rt, act, n, c, coords, ep, vec, 0);
    else if (gch == 1)
      k_rows_pass<T, true, 1><<<g, kNormThreads, smem, s>>>(xt, yt, rt, act, n, c, coords, ep, vec, per_warp);
    else if (gch == 2)
      k_rows_pass<T, true, 2><<<g, kNormThreads, smem, s>>>(xt, yt, rt, act, n, c, coords, ep, vec, per_warp);
    else if (gch == 4)
      k_rows_pass<T, true, 4><<<g, kNormThreads, smem, s>>>(xt, yt, rt, act, n, c, coords, ep, vec, per_warp);
    else if (gch == 8)
      k_rows_pass<T, true, 8><<<g, kNormThreads, smem, s>>>(xt, yt, rt, act, n, c, coords, ep, vec, per_warp);
    else if (gch == 16)
      k_rows_pass<T, true, 16><<<g, kNormThreads, smem, s>>>(xt, yt, rt, act, n, c, coords, ep, vec, per_warp);
    else
      k_rows_pass<T, true, 0><<<g, kNormThreads, smem, s>>>(xt, yt, rt, act, n, c, coords, ep, vec, per_warp);
  };
  switch (dtype) {
    case kF32: run(float{}); break;
    case kBF16: run(__nv_bfloat16{}); break;
    case kF16: run(__half{}); break;
    default: return cudaErrorInvalidValue;
  }
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_group_stats(const void* x, int64_t n, int c, const int32_t* coords, const Epilogue& ep, int dtype,
                               cudaStream_t s) {
  return launch_rows_pass(x, nullptr, nullptr, kActNone, n, c, coords, ep, dtype, s);
}

cudaError_t launch_stats_fold(const double* copies, int stripes, int64_t len, double* stats, cudaStream_t s) {
  k_stats_fold<<<static_cast<unsigned>((len + 255) / 256), 256, 0, s>>>(copies, stripes, len, stats);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_group_norm(const void* x, int64_t n, int c, const int32_t* coords, int batch, int groups,
                              const double* stats, const void* gamma, const void* beta, float eps, int act,
                              void* out, int dtype, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  if (batch * groups > kMaxBatchGroups) return cudaErrorInvalidValue;
  const unsigned g = grid_for(n * c);
  switch (dtype) {
    case kF32:
      k_group_norm<float><<<g, kNormThreads, 0, s>>>(static_cast<const float*>(x), n, c, coords, batch, groups, stats,
                                                     static_cast<const float*>(gamma),
                                                     static_cast<const float*>(beta), eps, act,
                                                     static_cast<float*>(out));
      break;
    case kBF16:
      k_group_norm<__nv_bfloat16><<<g, kNormThreads, 0, s>>>(
          static_cast<const __nv_bfloat16*>(x), n, c, coords, batch, groups, stats,
          static_cast<const __nv_bfloat16*>(gamma), static_cast<const __nv_bfloat16*>(beta), eps, act,
          static_cast<__nv_bfloat16*>(out));
      break;
    case kF16:
      k_group_norm<__half><<<g, kNormThreads, 0, s>>>(static_cast<const __half*>(x), n, c, coords, batch, groups,
                                                      stats, static_cast<const __half*>(gamma),
                                                      static_cast<const __half*>(beta), eps, act,
                                                      static_cast<__half*>(out));
      break;
    default:
      return cudaErrorInvalidValue;
  }
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace smc
