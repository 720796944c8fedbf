// GroupNorm over a sparse tensor, for the layers around the decoders' convs
// (Pixal3D MLX README "Status": norms, activations, ResBlock; LATO.2 MLX port
// README "Status": SparseGroupNorm32).  The population of a (batch item,
// channel group) is every active row of the item times the group's channels.
//   k_group_stats  adds (sum, sum of squares, count) of x per (item, group)
//                  into striped fp64 copies of a [batch, groups, 3] array
//                  (warp sums first), folded by k_stats_fold.
//   k_group_norm   y = act(gamma * (x - mean) * rsqrt(var + eps) + beta), with
//                  mean and (biased) variance from such statistics.
// A conv can produce the statistics of its own output in its epilogue
// (Epilogue::stats), so a conv -> GroupNorm pair reads the tensor once.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

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

// One thread per row (grid-stride over warps of 32 rows); each 32-channel run
// of the row is loaded and handed to warp_group_stats (the same reduction as
// the conv epilogue's), which adds into the block's shared-memory sums; the
// block's sums reach its global statistics copy (Epilogue striping) once.
template <typename T>
__global__ void __launch_bounds__(kNormThreads) k_group_stats(const T* __restrict__ x, int64_t n, int c,
                                                              const int32_t* __restrict__ coords, Epilogue ep) {
  __shared__ double s_acc[kMaxBatchGroups * 3];
  const int entries = ep.batch * ep.groups * 3;
  for (int i = threadIdx.x; i < entries; i += kNormThreads) s_acc[i] = 0.0;
  __syncthreads();
  const int gch = c / ep.groups;
  const int64_t rows_all = (n + 31) / 32 * 32;  // every lane of a warp runs every round
  for (int64_t row = blockIdx.x * static_cast<int64_t>(kNormThreads) + threadIdx.x; row < rows_all;
       row += static_cast<int64_t>(gridDim.x) * kNormThreads) {
    int b = -1;
    if (row < n) {
      b = coords[4 * row];
      if (b < 0 || b >= ep.batch) b = -1;
    }
    for (int c0 = 0; c0 < c; c0 += 32) {
      const int ncols = c - c0 < 32 ? c - c0 : 32;
      float v[32];
      const T* src = x + row * c + c0;
      if (b >= 0 && ncols == 32 && (c * sizeof(T)) % 16 == 0) {
        // 16-byte vector loads of the run
        constexpr int kPer = 16 / sizeof(T);
#pragma unroll
        for (int q = 0; q < 32 / kPer; ++q) {
          const uint4 u = *reinterpret_cast<const uint4*>(src + q * kPer);
          const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
          for (int j = 0; j < kPer; ++j) v[q * kPer + j] = ld_f<T>(e, j);
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = (b >= 0 && j < ncols) ? ld_f<T>(src, j) : 0.f;
      }
      warp_group_stats(v, c0, ncols, b >= 0, b < 0 ? 0 : b, gch, ep.groups, s_acc);
    }
  }
  __syncthreads();
  double* gst = stats_copy(ep);
  for (int i = threadIdx.x; i < entries; i += kNormThreads)
    if (s_acc[i] != 0.0) atomicAdd(gst + i, s_acc[i]);
}

// stats[i] += sum over the copies of copies[s][i].
__global__ void k_stats_fold(const double* __restrict__ copies, int stripes, int64_t len, double* __restrict__ stats) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < len;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    double t = 0.0;
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

cudaError_t launch_group_stats(const void* x, int64_t n, int c, const int32_t* coords, const Epilogue& ep, int dtype,
                               cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  const int64_t blocks = (n + kNormThreads - 1) / kNormThreads;
  const unsigned g = static_cast<unsigned>(blocks < 148 * 8 ? blocks : 148 * 8);
  switch (dtype) {
    case kF32:
      k_group_stats<float><<<g, kNormThreads, 0, s>>>(static_cast<const float*>(x), n, c, coords, ep);
      break;
    case kBF16:
      k_group_stats<__nv_bfloat16><<<g, kNormThreads, 0, s>>>(static_cast<const __nv_bfloat16*>(x), n, c, coords, ep);
      break;
    case kF16:
      k_group_stats<__half><<<g, kNormThreads, 0, s>>>(static_cast<const __half*>(x), n, c, coords, ep);
      break;
    default:
      return cudaErrorInvalidValue;
  }
  count_launches(1);
  return cudaGetLastError();
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
