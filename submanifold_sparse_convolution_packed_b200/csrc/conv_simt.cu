// FMA implicit gather-GEMM for submanifold convolution (any dtype, any shape).
//
// out[v] = bias + sum_d feats[nbr(v, d)] @ W[:, d, :]^T  (LATO.2 MLX port
// README, "The scope, once measured"; weights in KRSC layout [O,kz,ky,kx,I]).
// Each block owns 64 output rows x 64 output channels; for every tap that has
// at least one neighbour among its rows it gathers the neighbour rows (zero
// rows for missing ones) and the tap's weight slice through shared memory in
// K chunks of 16 and accumulates with fp32 fused multiply-adds, in tap order
// then channel order.  fp32 inputs therefore run in exact fp32 FMA (no TF32);
// bf16/fp16 inputs are widened to fp32.  This kernel is the path for fp32 and
// for shapes the tensor-core kernel does not take.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "epilogue.cuh"
#include "kernels.h"

namespace smc {

template <typename T> __device__ __forceinline__ float to_f(T x);
template <> __device__ __forceinline__ float to_f<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }
template <> __device__ __forceinline__ float to_f<__half>(__half x) { return __half2float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }
template <> __device__ __forceinline__ __half from_f<__half>(float x) { return __float2half_rn(x); }

constexpr int kBM = 64, kBN = 64, kBK = 16, kSimtThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kSimtThreads) k_conv_simt(
    const T* __restrict__ feats, const T* __restrict__ weight, const T* __restrict__ bias,
    T* __restrict__ out, const int32_t* __restrict__ nbr, int64_t n, int cin, int cout, int taps,
    int orientation, const Epilogue ep) {
  __shared__ float As[kBK][kBM + 4];
  __shared__ float Ws[kBK][kBN + 4];
  __shared__ int32_t s_idx[kBM];
  __shared__ int s_any;
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * kBM;
  const int col0 = blockIdx.y * kBN;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  for (int d = 0; d < taps; ++d) {
    if (tid == 0) s_any = 0;
    __syncthreads();
    if (tid < kBM) {
      const int64_t v = row0 + tid;
      int32_t u = -1;
      if (v < n) u = taps == 1 ? static_cast<int32_t>(v) : nbr[v * kTaps + (orientation > 0 ? d : kTaps - 1 - d)];
      s_idx[tid] = u;
      if (u >= 0) s_any = 1;
    }
    __syncthreads();
    if (!s_any) continue;
    for (int k0 = 0; k0 < cin; k0 += kBK) {
      for (int e = tid; e < kBM * kBK; e += kSimtThreads) {
        const int m = e / kBK, k = e % kBK;
        const int32_t u = s_idx[m];
        As[k][m] = (u >= 0 && k0 + k < cin) ? to_f<T>(feats[static_cast<int64_t>(u) * cin + k0 + k]) : 0.f;
      }
      for (int e = tid; e < kBN * kBK; e += kSimtThreads) {
        const int c = e / kBK, k = e % kBK;
        const int o = col0 + c;
        Ws[k][c] = (o < cout && k0 + k < cin)
                       ? to_f<T>(weight[(static_cast<int64_t>(o) * taps + d) * cin + k0 + k])
                       : 0.f;
      }
      __syncthreads();
#pragma unroll
      for (int k = 0; k < kBK; ++k) {
        float a[4], b[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = As[k][ty * 4 + i];
#pragma unroll
        for (int j = 0; j < 4; ++j) b[j] = Ws[k][tx * 4 + j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
      }
      __syncthreads();
    }
  }
  // epilogue: y = act(acc + bias) + residual, rounded
  const T* res = static_cast<const T*>(ep.residual);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t m = row0 + ty * 4 + i;
    if (m >= n) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int o = col0 + tx * 4 + j;
      if (o >= cout) break;
      float y = apply_act(acc[i][j] + (bias ? to_f<T>(bias[o]) : 0.f), ep.act);
      if (res) y += to_f<T>(res[m * cout + o]);
      out[m * cout + o] = from_f<T>(y);
    }
  }
}

cudaError_t launch_conv_simt(const ConvArgs& a, cudaStream_t s) {
  if (a.n == 0) return cudaSuccess;
  dim3 grid(static_cast<unsigned>((a.n + kBM - 1) / kBM), static_cast<unsigned>((a.cout + kBN - 1) / kBN));
  switch (a.dtype) {
    case kF32:
      k_conv_simt<float><<<grid, kSimtThreads, 0, s>>>(
          static_cast<const float*>(a.feats), static_cast<const float*>(a.weight),
          static_cast<const float*>(a.bias), static_cast<float*>(a.out), a.nbr, a.n, a.cin, a.cout,
          a.taps, a.orientation, a.ep);
      break;
    case kBF16:
      k_conv_simt<__nv_bfloat16><<<grid, kSimtThreads, 0, s>>>(
          static_cast<const __nv_bfloat16*>(a.feats), static_cast<const __nv_bfloat16*>(a.weight),
          static_cast<const __nv_bfloat16*>(a.bias), static_cast<__nv_bfloat16*>(a.out), a.nbr, a.n,
          a.cin, a.cout, a.taps, a.orientation, a.ep);
      break;
    case kF16:
      k_conv_simt<__half><<<grid, kSimtThreads, 0, s>>>(
          static_cast<const __half*>(a.feats), static_cast<const __half*>(a.weight),
          static_cast<const __half*>(a.bias), static_cast<__half*>(a.out), a.nbr, a.n, a.cin, a.cout,
          a.taps, a.orientation, a.ep);
      break;
    default:
      return cudaErrorInvalidValue;
  }
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace smc
