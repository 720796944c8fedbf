// Per-offset gather-GEMM-scatter convolution (bf16 / fp16, tcgen05).
//
// The comparator the pages measure their fused kernel against: for every
// kernel offset d, gather the input rows of that offset's pair list, multiply
// them by the offset's weight slice and scatter-add the products into the
// output (LATO.2 MLX port README, "The scope, once measured": the fused
// kernel against the per-offset loop).  Here all 27 offsets run in one launch:
// CTA (list l, tile t) takes pairs 128t .. 128t+127 of list l, gathers
// feats[in_idx] with TMA tile::gather4, runs tcgen05 MMAs with W[:, d, :]
// (d = l, or 26 - l for orientation -1: list l holds nbr[v][l]) into TMEM and
// adds the 128 x BN block into an fp32 accumulator at rows out_idx with
// vector red.add.  A second kernel adds the bias and rounds to the output
// type.  The fp32 accumulation order across offsets is not fixed (atomics),
// so results agree with the fused kernel to rounding, not bit for bit.
//
// Warp roles: warp 0 weight slices (3-D TMA), warp 1 TMEM + MMA issue, warps
// 2-5 the gather and then the epilogue for 32 rows each.  Every wait is
// bounded; on timeout the error word gets a bit and the CTA winds down.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "epilogue.cuh"
#include "kernels.h"

namespace smc {

namespace {

constexpr int kOffThreads = 192;
constexpr int kOffMaxStages = 4;

struct OffParams {
  const int32_t* in_idx;
  const int32_t* out_idx;
  const int64_t* offsets;  // [28] starts of the 27 pair lists, then the total
  float* acc;              // [n, cout] fp32, zeroed
  uint32_t* err;
  int cin, cout, bn, nsplit, stages, kb_elems, orientation, is_bf16;
  uint32_t tmem_cols;
  uint64_t wait_ns;  // bound of every mbarrier wait
};

__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

__global__ void __launch_bounds__(kOffThreads, 3) k_conv_offsets(const __grid_constant__ CUtensorMap fmap,
                                                                 const __grid_constant__ CUtensorMap wmap,
                                                                 const OffParams p) {
  // The (list, tile) of this CTA: tiles are numbered list by list.  The grid
  // is sized for the largest possible total; CTAs past the end leave at once.
  const int64_t unit = blockIdx.x / p.nsplit;
  const int n0 = static_cast<int>(blockIdx.x % p.nsplit) * p.bn;
  int list = -1;
  int64_t first = 0, rows = 0;
  {
    int64_t u = unit;
    for (int l = 0; l < kTaps; ++l) {
      const int64_t o0 = __ldg(p.offsets + l), o1 = __ldg(p.offsets + l + 1);
      const int64_t tiles = (o1 - o0 + kTileRows - 1) / kTileRows;
      if (u < tiles) {
        list = l;
        first = o0 + u * kTileRows;
        rows = o1 - first < kTileRows ? o1 - first : kTileRows;
        break;
      }
      u -= tiles;
    }
  }
  if (list < 0) return;
  const int d = p.orientation > 0 ? list : kTaps - 1 - list;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw);
  const uint32_t row_bytes = static_cast<uint32_t>(p.kb_elems) * 2;
  const uint32_t a_bytes = kTileRows * row_bytes;
  const uint32_t b_bytes = static_cast<uint32_t>(p.bn) * row_bytes;
  const uint32_t a_off = 0, b_off = p.stages * a_bytes, bar_off = b_off + p.stages * b_bytes;
  const uint32_t bar_full = sbase + bar_off;
  const uint32_t bar_empty = bar_full + kOffMaxStages * 8;
  const uint32_t bar_acc = bar_empty + kOffMaxStages * 8;
  volatile uint32_t* s_misc = reinterpret_cast<volatile uint32_t*>(smem + bar_off + (2 * kOffMaxStages + 2) * 8);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int kblocks = (p.cin + p.kb_elems - 1) / p.kb_elems;
  const int last_ksteps = (p.cin - (kblocks - 1) * p.kb_elems + 15) / 16;

  if (tid == 0) {
    prefetch_tmap(&fmap);
    prefetch_tmap(&wmap);
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(bar_full + 8 * s, 5);  // weight loader + 4 gather warps
      mbar_init(bar_empty + 8 * s, 1);
    }
    mbar_init(bar_acc, 1);
    s_misc[1] = 0;
    fence_mbarrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(const_cast<uint32_t*>(&s_misc[0])), p.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = s_misc[0];

  if (warp == 0) {
    // ---------------------------------------------------------- weight slice
    if (lane == 0) {
      for (int kb = 0; kb < kblocks; ++kb) {
        const uint32_t stage = kb % p.stages, phase = (kb / p.stages) & 1u;
        if (!mbar_wait_bounded(bar_empty + 8 * stage, phase ^ 1u, p.err, p.wait_ns) || s_misc[1]) {
          s_misc[1] = 1;
          break;
        }
        const uint32_t full = bar_full + 8 * stage;
        mbar_arrive_expect_tx(full, b_bytes);
        tma_load_3d(sbase + b_off + stage * b_bytes, &wmap, full, kb * p.kb_elems, d, n0);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_f16(static_cast<uint32_t>(p.is_bf16), static_cast<uint32_t>(p.bn));
      for (int kb = 0; kb < kblocks; ++kb) {
        const uint32_t stage = kb % p.stages, phase = (kb / p.stages) & 1u;
        if (!mbar_wait_bounded(bar_full + 8 * stage, phase, p.err, p.wait_ns) || s_misc[1]) {
          s_misc[1] = 1;
          break;
        }
        tc_fence_after();
        const uint64_t adesc = kmajor_desc(sbase + a_off + stage * a_bytes, row_bytes);
        const uint64_t bdesc = kmajor_desc(sbase + b_off + stage * b_bytes, row_bytes);
        const int ksteps = kb == kblocks - 1 ? last_ksteps : p.kb_elems / 16;
        for (int k = 0; k < ksteps; ++k)
          umma_f16(tmem_base, adesc + 2 * k, bdesc + 2 * k, idesc, (kb > 0 || k > 0) ? 1u : 0u);
        umma_commit(bar_empty + 8 * stage);
      }
      umma_commit(bar_acc);
    }
  } else {
    // ---------------------------------------------------------- gather
    const int q = warp & 3;
    const int r = q * 32 + lane;  // tile row = pair first + r
    const int32_t in = r < rows ? __ldg(p.in_idx + first + r) : -1;
    const int32_t out = r < rows ? __ldg(p.out_idx + first + r) : -1;
    const int src = (lane & 7) * 4;
    const int32_t r0 = __shfl_sync(0xffffffffu, in, src + 0);
    const int32_t r1 = __shfl_sync(0xffffffffu, in, src + 1);
    const int32_t r2 = __shfl_sync(0xffffffffu, in, src + 2);
    const int32_t r3 = __shfl_sync(0xffffffffu, in, src + 3);
    for (int kb = 0; kb < kblocks; ++kb) {
      const uint32_t stage = kb % p.stages, phase = (kb / p.stages) & 1u;
      int w_ok = 1;
      if (lane == 0)
        w_ok = mbar_wait_bounded(bar_empty + 8 * stage, phase ^ 1u, p.err, p.wait_ns) && !s_misc[1];
      w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
      if (!w_ok) {
        if (lane == 0) s_misc[1] = 1;
        break;
      }
      const uint32_t full = bar_full + 8 * stage;
      if (lane == 0) mbar_arrive_expect_tx(full, 32u * row_bytes);
      __syncwarp();
      if (lane < 8)
        tma_gather4(sbase + a_off + stage * a_bytes + (q * 32 + 4 * lane) * row_bytes, &fmap, full,
                    kb * p.kb_elems, r0, r1, r2, r3);
    }
    // ---------------------------------------------------------- scatter-add
    const bool ready = mbar_wait_bounded(bar_acc, 0, p.err, p.wait_ns) && !s_misc[1];
    tc_fence_after();
    if (ready) {
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
      for (int c0 = 0; c0 < p.bn; c0 += 32) {
        float v[32];
        tmem_ld_32cols(t_row + c0, v);
        if (out < 0) continue;
        float* dst = p.acc + static_cast<int64_t>(out) * p.cout + n0 + c0;
#pragma unroll
        for (int j = 0; j < 32; j += 4)
          if (c0 + j < p.bn && n0 + c0 + j < p.cout) red_add_v4(dst + j, v[j], v[j + 1], v[j + 2], v[j + 3]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, p.tmem_cols);
  }
}

// out = round(act(acc + bias) + residual), four values per thread.
__global__ void k_offsets_finalize(const float4* __restrict__ acc, const uint16_t* __restrict__ bias,
                                   uint16_t* __restrict__ out, int64_t n4, int cout, int is_bf16, const Epilogue ep) {
  const bool bf = is_bf16 != 0;
  const uint16_t* res = static_cast<const uint16_t*>(ep.residual);
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4 a = acc[i];
    float x[4] = {a.x, a.y, a.z, a.w};
    const int c = static_cast<int>((i * 4) % cout);
    uint16_t h[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (bias) x[e] += half_bits_to_float(__ldg(bias + c + e), bf);
      x[e] = apply_act(x[e], ep.act);
      if (res) x[e] += half_bits_to_float(res[i * 4 + e], bf);
      h[e] = float_to_half_bits(x[e], bf);
    }
    reinterpret_cast<uint2*>(out)[i] =
        make_uint2(static_cast<uint32_t>(h[0]) | (static_cast<uint32_t>(h[1]) << 16),
                   static_cast<uint32_t>(h[2]) | (static_cast<uint32_t>(h[3]) << 16));
  }
}

uint32_t pow2_at_least(uint32_t x) {
  uint32_t v = 32;
  while (v < x) v <<= 1;
  return v;
}

}  // namespace

cudaError_t launch_conv_offsets(const ConvArgs& a, float* acc, cudaStream_t s) {
  if (a.n == 0) return cudaSuccess;
  EncodeTiledFn enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  const CUtensorMapDataType dt = a.dtype == kBF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  OffParams p;
  p.nsplit = (a.cout + 255) / 256;
  p.bn = ((a.cout + p.nsplit - 1) / p.nsplit + 15) / 16 * 16;
  p.tmem_cols = pow2_at_least(static_cast<uint32_t>(p.bn));
  p.kb_elems = 64;
  const int kblocks = (a.cin + p.kb_elems - 1) / p.kb_elems;
  const uint32_t stage_bytes = static_cast<uint32_t>(kTileRows + p.bn) * p.kb_elems * 2;
  const int ctas_per_sm = p.tmem_cols <= 128 ? 3 : 2;
  const uint32_t budget = 228u * 1024u / ctas_per_sm - 2048u;
  int stages = static_cast<int>(budget / stage_bytes);
  if (stages > kOffMaxStages) stages = kOffMaxStages;
  if (stages > kblocks) stages = kblocks;
  if (stages < 1) stages = 1;
  p.stages = stages;
  const uint32_t smem = stages * stage_bytes + (2 * kOffMaxStages + 2) * 8 + 16 + 1024;

  CUtensorMap fmap, wmap;
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(a.cin), static_cast<cuuint64_t>(a.n)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.cin) * 2};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(p.kb_elems), 1u};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&fmap, dt, 2, const_cast<void*>(a.feats), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(a.cin), static_cast<cuuint64_t>(kTaps),
                                static_cast<cuuint64_t>(a.cout)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(a.cin) * 2, static_cast<cuuint64_t>(a.cin) * kTaps * 2};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(p.kb_elems), 1, static_cast<cuuint32_t>(p.bn)};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (enc(&wmap, dt, 3, const_cast<void*>(a.weight), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  p.in_idx = a.in_idx;
  p.out_idx = a.out_idx;
  p.offsets = a.pair_offsets;
  p.acc = acc;
  p.err = a.err;
  // A conv's waits are bounded too, but never below 100 ms: a CTA that
  // gave up a wait early would leave with its TMA loads still in flight.
  p.wait_ns = scan_wait_limit_ns() > 100000000ull ? scan_wait_limit_ns() : 100000000ull;
  p.cin = a.cin;
  p.cout = a.cout;
  p.orientation = a.orientation;
  p.is_bf16 = a.dtype == kBF16 ? 1 : 0;

  cudaError_t e = cudaMemsetAsync(acc, 0, static_cast<size_t>(a.n) * a.cout * sizeof(float), s);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(k_conv_offsets, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  // at most ceil(count_l / 128) <= ceil(n / 128) tiles per list
  const int64_t units = static_cast<int64_t>(kTaps) * ((a.n + kTileRows - 1) / kTileRows) * p.nsplit;
  k_conv_offsets<<<static_cast<unsigned>(units), kOffThreads, smem, s>>>(fmap, wmap, p);
  const int64_t n4 = a.n * a.cout / 4;
  k_offsets_finalize<<<static_cast<unsigned>((n4 + 255) / 256 < 148 * 16 ? (n4 + 255) / 256 : 148 * 16), 256, 0,
                       s>>>(reinterpret_cast<const float4*>(acc), static_cast<const uint16_t*>(a.bias),
                            static_cast<uint16_t*>(a.out), n4, a.cout, p.is_bf16, a.ep);
  count_launches(2);
  return cudaGetLastError();
}

}  // namespace smc
