// Downsample by 2 (pooling into parent voxels) and the feature gather of the
// masked upsample by 2 (shared sparse-core commit log: downsample modes 'max'
// and 'mean', upsample a masked expansion whose child index runs with the z
// axis fastest; Pixal3D MLX README "Status").
//
// Downsample, one launch each:
//   k_down_insert  one thread per row: validate it, form its parent's key,
//                  find or claim the parent's slot in the lookup structure
//                  (a dense grid over the parent box, or an open-addressing
//                  hash), atomicMin the row into the slot's first row and
//                  atomicOr the row's child bit into the slot's mask.
//   k_down_flags   1 where a row is its parent's first row.
//   scan           exclusive scan of the flags (k_scan_lookback): parents
//                  are numbered in order of first appearance; M comes out.
//   k_down_emit    one thread per row: its parent's number; the first row
//                  also writes the parent's coordinates and mask; every row
//                  enters itself as child j of its parent.
//   k_down_pool    one thread per (parent, 16-byte vector of channels): max
//                  or mean over the children present, j ascending, in fp32.
// Upsample: the children's coordinates come from the subdivision kernels of
// map_build.cu in mask order; k_expand_rows copies each parent's row to its
// children.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace smc {

namespace {

constexpr int kThreads = 256;
#ifndef SMC_POOL_BLOCKS_PER_SM
#define SMC_POOL_BLOCKS_PER_SM 3
#endif
constexpr int kPoolBlocksPerSm = SMC_POOL_BLOCKS_PER_SM;  // 85 registers a thread: no spills
constexpr uint32_t kNoSlot = 0xFFFFFFFFu;
constexpr unsigned long long kFree = ~0ull;
constexpr uint64_t kFibHash = 0x9E3779B97F4A7C15ull;

__device__ __forceinline__ bool in_box(int4 c, int32_t batch, int32_t Z, int32_t Y, int32_t X) {
  return c.x >= 0 && c.x < batch && c.y >= 0 && c.y < Z && c.z >= 0 && c.z < Y && c.w >= 0 && c.w < X;
}

// Child index inside the parent: z offset + 2 * y offset + 4 * x offset.
__device__ __forceinline__ uint32_t child_index(int4 c) {
  return static_cast<uint32_t>((c.y & 1) | ((c.z & 1) << 1) | ((c.w & 1) << 2));
}

unsigned grid_of(int64_t work) {
  const int64_t blocks = (work + kThreads - 1) / kThreads;
  return static_cast<unsigned>(blocks < 148 * 8 ? (blocks > 0 ? blocks : 1) : 148 * 8);
}

template <bool kDense>
__global__ void __launch_bounds__(kThreads) k_down_insert(DownArgs a) {
  const int64_t Zc = (a.Z + 1) >> 1, Yc = (a.Y + 1) >> 1, Xc = (a.X + 1) >> 1;
  const uint64_t mask = (1ull << a.lg) - 1;
  const int4* coords = reinterpret_cast<const int4*>(a.coords);
  for (int64_t v = blockIdx.x * static_cast<int64_t>(kThreads) + threadIdx.x; v < a.n;
       v += static_cast<int64_t>(gridDim.x) * kThreads) {
    const int4 c = coords[v];
    uint32_t slot = kNoSlot;
    if (!in_box(c, a.batch, a.Z, a.Y, a.X)) {
      atomicOr(a.err, kErrRange);
    } else {
      const uint64_t key = ((static_cast<uint64_t>(c.x) * Zc + (c.y >> 1)) * Yc + (c.z >> 1)) * Xc + (c.w >> 1);
      if (kDense) {
        slot = static_cast<uint32_t>(key);
      } else {
        uint64_t s = (key * kFibHash) >> (64 - a.lg);
        for (uint64_t probe = 0; probe <= mask; ++probe) {
          const unsigned long long prev = atomicCAS(&a.keys[s], kFree, key);
          if (prev == kFree || prev == key) {
            slot = static_cast<uint32_t>(s);
            break;
          }
          s = (s + 1) & mask;
        }
        if (slot == kNoSlot) atomicOr(a.err, kErrCapacity);
      }
      if (slot != kNoSlot) {
        atomicMin(&a.first[slot], static_cast<int32_t>(v));
        const uint32_t bit = 1u << child_index(c);
        if (atomicOr(&a.bits[slot], bit) & bit) atomicOr(a.err, kErrDuplicate);
      }
    }
    a.slot_of_row[v] = slot;
  }
}

__global__ void __launch_bounds__(kThreads) k_down_flags(DownArgs a) {
  for (int64_t v = blockIdx.x * static_cast<int64_t>(kThreads) + threadIdx.x; v < a.n;
       v += static_cast<int64_t>(gridDim.x) * kThreads) {
    const uint32_t slot = a.slot_of_row[v];
    a.flags[v] = slot != kNoSlot && a.first[slot] == static_cast<int32_t>(v);
  }
}

// Byte k of the result is bit k of b (k < 4).
__device__ __forceinline__ uint32_t spread4(uint32_t b) {
  return (b & 1u) | ((b >> 1) & 1u) << 8 | ((b >> 2) & 1u) << 16 | ((b >> 3) & 1u) << 24;
}

__global__ void __launch_bounds__(kThreads) k_down_emit(DownArgs a) {
  const int4* coords = reinterpret_cast<const int4*>(a.coords);
  for (int64_t v = blockIdx.x * static_cast<int64_t>(kThreads) + threadIdx.x; v < a.n;
       v += static_cast<int64_t>(gridDim.x) * kThreads) {
    const uint32_t slot = a.slot_of_row[v];
    int64_t p = -1;
    if (slot != kNoSlot) {
      const int32_t f = a.first[slot];
      p = a.pos[f];
      if (p < 0 || p >= a.n) p = -1;  // only when the scan gave up on a wait (error bit set)
      if (p >= 0) {
        const int4 c = coords[v];
        a.child_rows[8 * p + child_index(c)] = static_cast<int32_t>(v);
        if (f == static_cast<int32_t>(v)) {
          reinterpret_cast<int4*>(a.parent_coords)[p] = make_int4(c.x, c.y >> 1, c.z >> 1, c.w >> 1);
          const uint32_t b = a.bits[slot];
          a.pbits[p] = static_cast<uint8_t>(b);
          reinterpret_cast<uint2*>(a.mask)[p] = make_uint2(spread4(b & 15u), spread4(b >> 4));
        }
      }
    }
    if (a.parent) a.parent[v] = static_cast<int32_t>(p);
  }
}

template <typename T> struct Lanes;
template <> struct Lanes<float> {
  static __device__ __forceinline__ float get(const float* p, int i) { return p[i]; }
  static __device__ __forceinline__ void put(float* p, int i, float x) { p[i] = x; }
};
template <> struct Lanes<__nv_bfloat16> {
  static __device__ __forceinline__ float get(const __nv_bfloat16* p, int i) { return __bfloat162float(p[i]); }
  static __device__ __forceinline__ void put(__nv_bfloat16* p, int i, float x) { p[i] = __float2bfloat16_rn(x); }
};
template <> struct Lanes<__half> {
  static __device__ __forceinline__ float get(const __half* p, int i) { return __half2float(p[i]); }
  static __device__ __forceinline__ void put(__half* p, int i, float x) { p[i] = __float2half_rn(x); }
};

// kV channels per thread: 16 / sizeof(T) (one 16-byte load per child) or 1.
// The grid-stride loop is software-pipelined: the next item's child list
// (rows and mask) is loaded before this item's features, so that its latency
// overlaps theirs.
template <typename T, int kV>
__global__ void __launch_bounds__(kThreads, kPoolBlocksPerSm) k_down_pool(const T* __restrict__ feats, int c,
                                                                          const int32_t* __restrict__ child_rows,
                                                                          const uint8_t* __restrict__ pbits,
                                                                          const int64_t* __restrict__ count,
                                                                          int64_t n, int mode, T* __restrict__ out) {
  using Vec = typename std::conditional<kV == 1, T, uint4>::type;
  const int64_t m = *count < n ? *count : n;
  const int nv = c / kV;
  const int64_t total = m * nv;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
  int64_t t = blockIdx.x * static_cast<int64_t>(kThreads) + threadIdx.x;
  int4 r0 = make_int4(0, 0, 0, 0), r1 = r0;
  uint32_t b = 0;
  if (t < total) {
    const int64_t p = t / nv;
    b = pbits[p];
    r0 = reinterpret_cast<const int4*>(child_rows)[2 * p];
    r1 = reinterpret_cast<const int4*>(child_rows)[2 * p + 1];
  }
  for (; t < total; t += stride) {
    const int64_t p = t / nv;
    const int q = static_cast<int>(t - p * nv);
    const uint32_t bc = b;
    const int32_t row[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
    const int64_t tn = t + stride;
    if (tn < total) {
      const int64_t pn = tn / nv;
      b = pbits[pn];
      r0 = reinterpret_cast<const int4*>(child_rows)[2 * pn];
      r1 = reinterpret_cast<const int4*>(child_rows)[2 * pn + 1];
    }
    Vec u[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (((bc >> j) & 1u) && static_cast<uint64_t>(row[j]) < static_cast<uint64_t>(n))  // rows are valid unless
        u[j] = __ldg(reinterpret_cast<const Vec*>(feats + static_cast<int64_t>(row[j]) * c) + q);  // the call fails
    float acc[kV];
#pragma unroll
    for (int e = 0; e < kV; ++e) acc[e] = 0.f;
    bool any = false;  // a parent has at least one child
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (((bc >> j) & 1u) && static_cast<uint64_t>(row[j]) < static_cast<uint64_t>(n)) {
        const T* x = reinterpret_cast<const T*>(&u[j]);
#pragma unroll
        for (int e = 0; e < kV; ++e) {
          const float y = Lanes<T>::get(x, e);
          acc[e] = mode == 0 ? (any ? fmaxf(acc[e], y) : y) : acc[e] + y;
        }
        any = true;
      }
    }
    if (mode == 1) {
      const float cnt = static_cast<float>(__popc(bc));
#pragma unroll
      for (int e = 0; e < kV; ++e) acc[e] = acc[e] / cnt;
    }
    Vec w;
    T* y = reinterpret_cast<T*>(&w);
#pragma unroll
    for (int e = 0; e < kV; ++e) Lanes<T>::put(y, e, acc[e]);
    reinterpret_cast<Vec*>(out + p * c)[q] = w;
  }
}

// Parent p's row copied to its children, rows first[p] .. first[p] + cnt - 1
// of the output (children are listed parent by parent): one thread per
// (parent, unit of U), one load and up to eight stores; each store
// instruction of a warp writes whole runs of child rows.
template <typename U>
__global__ void __launch_bounds__(kThreads) k_expand_rows(const U* __restrict__ rows, int64_t units,
                                                          const int64_t* __restrict__ first,
                                                          const uint8_t* __restrict__ bits, int64_t n, int64_t cap,
                                                          U* __restrict__ out) {
  const int64_t total = n * units;
  for (int64_t t = blockIdx.x * static_cast<int64_t>(kThreads) + threadIdx.x; t < total;
       t += static_cast<int64_t>(gridDim.x) * kThreads) {
    const int64_t p = t / units;
    const int64_t q = t - p * units;
    const int64_t r0 = first[p];
    const int cnt = __popc(static_cast<uint32_t>(bits[p]));
    if (cnt == 0 || r0 < 0 || r0 + cnt > cap) continue;  // out of range only if the scan failed
    const U x = __ldg(rows + t);
    U* dst = out + r0 * units + q;
    for (int i = 0; i < cnt; ++i) dst[i * units] = x;
  }
}

// Grid of a grid-stride kernel: as many blocks as fit on the device at once
// (blocks per SM from the occupancy calculator, times the SM count), capped
// by the work.
template <typename K>
unsigned resident_grid(K kernel, int64_t work) {
  static int per_sm = 0, sms = 0;
  if (per_sm == 0) {
    int dev = 0, b = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kernel, kThreads, 0);
    sms = n > 0 ? n : 148;
    per_sm = b > 0 ? b : 1;
  }
  const int64_t blocks = (work + kThreads - 1) / kThreads;
  const int64_t cap = static_cast<int64_t>(per_sm) * sms;
  return static_cast<unsigned>(blocks < cap ? (blocks > 0 ? blocks : 1) : cap);
}

template <typename T>
void pool_launch(const DownArgs& a, cudaStream_t s, bool vec) {
  constexpr int kV = 16 / sizeof(T);
  const T* f = static_cast<const T*>(a.feats);
  T* o = static_cast<T*>(a.out);
  if (vec)
    k_down_pool<T, kV><<<resident_grid(k_down_pool<T, kV>, a.n * (a.c / kV)), kThreads, 0, s>>>(
        f, a.c, a.child_rows, a.pbits, a.info + kTaps, a.n, a.mode, o);
  else
    k_down_pool<T, 1><<<resident_grid(k_down_pool<T, 1>, a.n * a.c), kThreads, 0, s>>>(
        f, a.c, a.child_rows, a.pbits, a.info + kTaps, a.n, a.mode, o);
}

}  // namespace

cudaError_t launch_downsample(const DownArgs& a, cudaStream_t s) {
  if (a.n == 0) return cudaSuccess;
  const unsigned g = grid_of(a.n);
  if (a.keys)
    k_down_insert<false><<<g, kThreads, 0, s>>>(a);
  else
    k_down_insert<true><<<g, kThreads, 0, s>>>(a);
  k_down_flags<<<g, kThreads, 0, s>>>(a);
  count_launches(2);
  cudaError_t e = launch_scan_counts(a.flags, a.n, a.pos, a.scan_status, a.scan_ticket, a.err, a.info, a.n, s);
  if (e != cudaSuccess) return e;
  k_down_emit<<<g, kThreads, 0, s>>>(a);
  count_launches(1);
  if (a.feats) {
    const int es = a.dtype == kF32 ? 4 : 2;
    const bool vec = (a.c * es) % 16 == 0 && (reinterpret_cast<uintptr_t>(a.feats) & 15u) == 0 &&
                     (reinterpret_cast<uintptr_t>(a.out) & 15u) == 0;
    switch (a.dtype) {
      case kF32: pool_launch<float>(a, s, vec); break;
      case kBF16: pool_launch<__nv_bfloat16>(a, s, vec); break;
      case kF16: pool_launch<__half>(a, s, vec); break;
      default: return cudaErrorInvalidValue;
    }
    count_launches(1);
  }
  return cudaGetLastError();
}

cudaError_t launch_expand_rows(const void* rows, int64_t row_bytes, const int64_t* first, const uint8_t* bits,
                               int64_t n, void* out, int elem_bytes, cudaStream_t s) {
  if (n == 0 || row_bytes == 0) return cudaSuccess;
  const bool vec = row_bytes % 16 == 0 && (reinterpret_cast<uintptr_t>(rows) & 15u) == 0 &&
                   (reinterpret_cast<uintptr_t>(out) & 15u) == 0;
  const int64_t cap = 8 * n;
  if (vec) {
    const int64_t units = row_bytes / 16;
    k_expand_rows<uint4><<<resident_grid(k_expand_rows<uint4>, n * units), kThreads, 0, s>>>(
        static_cast<const uint4*>(rows), units, first, bits, n, cap, static_cast<uint4*>(out));
  } else if (elem_bytes == 4) {
    const int64_t units = row_bytes / 4;
    k_expand_rows<uint32_t><<<resident_grid(k_expand_rows<uint32_t>, n * units), kThreads, 0, s>>>(
        static_cast<const uint32_t*>(rows), units, first, bits, n, cap, static_cast<uint32_t*>(out));
  } else {
    const int64_t units = row_bytes / 2;
    k_expand_rows<uint16_t><<<resident_grid(k_expand_rows<uint16_t>, n * units), kThreads, 0, s>>>(
        static_cast<const uint16_t*>(rows), units, first, bits, n, cap, static_cast<uint16_t*>(out));
  }
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace smc
