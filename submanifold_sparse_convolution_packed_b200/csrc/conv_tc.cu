// tcgen05 implicit gather-GEMM for submanifold convolution (bf16 / fp16).
//
// out[v] = bias + sum_d feats[nbr(v, d)] @ W[:, d, :]^T, W in KRSC layout
// [O, kz, ky, kx, I] (LATO.2 MLX port README, summary and "The scope, once
// measured"; orientation per its "Correctness" section).  Seen as a GEMM it
// is M = active voxels, N = Cout, K = 27 * Cin, where the A rows of tap d are
// the gathered neighbour rows and B is the weight tensor itself read as
// [Cout, 27*Cin] (K-major, no re-layout).
//
// One CTA computes one 128-row x BN-column output tile, accumulating all taps
// in TMEM (fp32):
//   * the tile's rows are 128 consecutive entries of the map's tile schedule
//     (rows grouped by neighbour pattern), and the CTA issues only the taps
//     at least one of its rows has;
//   * warp 0 (one lane) streams (tap, 64-channel block) stages: the 128
//     gathered A rows by TMA tile::gather4 (missing neighbours are row -1,
//     which TMA reads as zeros) and the weight slice by a 3-D TMA tile load,
//     both into 128-byte-swizzled shared memory, completion on an mbarrier;
//   * warp 1 (one lane) issues tcgen05.mma (M=128, N=BN, K=16) and commits
//     each stage back to its producer barrier;
//   * warps 2-5 drain TMEM with tcgen05.ld, add the bias in fp32, round to
//     the storage type and store 16-byte vectors to the output rows.
// Every mbarrier wait is bounded; on timeout the error word gets a bit and the
// CTA winds down without touching further memory.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.h"

namespace smc {

constexpr int kTileM = 128;
constexpr int kKBlock = 64;                       // channels per stage (128 bytes of bf16)
constexpr uint32_t kABytes = kTileM * kKBlock * 2;  // 16 KB
constexpr int kTcThreads = 192;
constexpr int kMaxStages = 8;

struct TcSmemLayout {
  uint32_t a_off, b_off, idx_off, rows_off, bar_off, misc_off, total;
};

__host__ __device__ inline TcSmemLayout tc_layout(int stages, int bn) {
  TcSmemLayout L;
  const uint32_t b_bytes = static_cast<uint32_t>(bn) * kKBlock * 2;
  L.a_off = 0;
  L.b_off = L.a_off + stages * kABytes;
  L.idx_off = L.b_off + stages * b_bytes;
  L.rows_off = L.idx_off + kTaps * kTileM * 4;
  L.bar_off = L.rows_off + kTileM * 4;
  L.misc_off = L.bar_off + (2 * kMaxStages + 1) * 8;
  L.total = L.misc_off + 64;
  return L;
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__global__ void __launch_bounds__(kTcThreads, 1) k_conv_tc(
    const __grid_constant__ CUtensorMap fmap, const __grid_constant__ CUtensorMap wmap,
    const int32_t* __restrict__ nbr, const int32_t* __restrict__ perm, int64_t n, int cin,
    int cout, int taps, int orientation, int bn, int stages, uint32_t tmem_cols, int is_bf16,
    const uint16_t* __restrict__ bias, uint16_t* __restrict__ out, uint32_t* err) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte swizzle atoms
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw);
  const TcSmemLayout L = tc_layout(stages, bn);
  int32_t* s_idx = reinterpret_cast<int32_t*>(smem + L.idx_off);   // [27][128]
  int32_t* s_rows = reinterpret_cast<int32_t*>(smem + L.rows_off);  // [128]
  const uint32_t bar_full = sbase + L.bar_off;                      // [stages]
  const uint32_t bar_empty = bar_full + kMaxStages * 8;             // [stages]
  const uint32_t bar_accum = bar_empty + kMaxStages * 8;
  uint32_t* s_misc = reinterpret_cast<uint32_t*>(smem + L.misc_off);  // [0]=tmem base, [1..4]=warp masks

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t tile = blockIdx.x;
  const int n0 = blockIdx.y * bn;
  const uint32_t b_bytes = static_cast<uint32_t>(bn) * kKBlock * 2;

  if (tid == 0) {
    prefetch_tmap(&fmap);
    prefetch_tmap(&wmap);
    for (int s = 0; s < stages; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 1);
    }
    mbar_init(bar_accum, 1);
    fence_mbarrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&s_misc[0]), tmem_cols);
    tmem_relinquish();
  }
  // Gather indices of the tile: s_idx[d][r] = row of the tap-d neighbour of
  // tile row r (orientation applied), -1 when absent.
  if (tid < kTileM) {
    const int64_t g = tile * kTileM + tid;
    const int32_t v = g < n ? (perm ? perm[g] : static_cast<int32_t>(g)) : -1;
    s_rows[tid] = v;
    uint32_t m = 0;
    if (taps == kTaps) {
      const int32_t* row = nbr + static_cast<int64_t>(v < 0 ? 0 : v) * kTaps;
      int32_t u[kTaps];
#pragma unroll
      for (int d = 0; d < kTaps; ++d) u[d] = v >= 0 ? __ldg(row + (orientation > 0 ? d : kTaps - 1 - d)) : -1;
#pragma unroll
      for (int d = 0; d < kTaps; ++d) {
        s_idx[d * kTileM + tid] = u[d];
        m |= static_cast<uint32_t>(u[d] >= 0) << d;
      }
    } else {
      s_idx[tid] = v;
      m = v >= 0 ? 1u : 0u;
    }
    m = __reduce_or_sync(0xffffffffu, m);
    if (lane == 0) s_misc[1 + warp] = m;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = s_misc[0];
  const uint32_t tap_mask = s_misc[1] | s_misc[2] | s_misc[3] | s_misc[4];
  const int kblocks = (cin + kKBlock - 1) / kKBlock;
  const int last_ksteps = (cin - (kblocks - 1) * kKBlock + 15) / 16;
  const uint32_t idesc = idesc_f16(static_cast<uint32_t>(is_bf16), static_cast<uint32_t>(bn));

  if (warp == 0) {
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (uint32_t m = tap_mask; m && ok; m &= m - 1) {
        const int d = __ffs(m) - 1;
        const int32_t* idx = s_idx + d * kTileM;
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const uint32_t stage = it % stages, phase = (it / stages) & 1u;
          if (!mbar_wait_bounded(bar_empty + 8 * stage, phase ^ 1u, err)) { ok = false; break; }
          const uint32_t full = bar_full + 8 * stage;
          mbar_arrive_expect_tx(full, kABytes + b_bytes);
          const uint32_t a_dst = sbase + L.a_off + stage * kABytes;
          const int x = kb * kKBlock;
#pragma unroll 8
          for (int j = 0; j < kTileM / 4; ++j) {
            const int4 r = *reinterpret_cast<const int4*>(idx + 4 * j);
            tma_gather4(a_dst + j * 4 * 128, &fmap, full, x, r.x, r.y, r.z, r.w);
          }
          tma_load_3d(sbase + L.b_off + stage * b_bytes, &wmap, full, x, taps == kTaps ? d : 0, n0);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (uint32_t m = tap_mask; m && ok; m &= m - 1) {
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const uint32_t stage = it % stages, phase = (it / stages) & 1u;
          if (!mbar_wait_bounded(bar_full + 8 * stage, phase, err)) { ok = false; break; }
          tc_fence_after();
          const uint64_t adesc = sw128_kmajor_desc(sbase + L.a_off + stage * kABytes);
          const uint64_t bdesc = sw128_kmajor_desc(sbase + L.b_off + stage * b_bytes);
          const int ksteps = kb == kblocks - 1 ? last_ksteps : kKBlock / 16;
          for (int k = 0; k < ksteps; ++k)
            umma_f16(tmem_base, adesc + 2 * k, bdesc + 2 * k, idesc, (it > 0 || k > 0) ? 1u : 0u);
          umma_commit(bar_empty + 8 * stage);
        }
      }
      umma_commit(bar_accum);
    }
  } else {
    // epilogue: warps 2..5 own TMEM lane quarters (warp % 4)
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const bool ready = mbar_wait_bounded(bar_accum, 0, err);
    tc_fence_after();
    const int32_t v = s_rows[r];
    if (ready && tap_mask != 0) {
      for (int c0 = 0; c0 < bn; c0 += 32) {
        float acc[32];
        tmem_ld_32cols(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + c0, acc);
        if (v >= 0) {
#pragma unroll
          for (int j = 0; j < 32; j += 8) {
            const int col = n0 + c0 + j;
            if (col < cout && c0 + j < bn) {
              uint32_t packed[4];
#pragma unroll
              for (int e = 0; e < 8; e += 2) {
                float x0 = acc[j + e], x1 = acc[j + e + 1];
                if (bias) {
                  const uint16_t b0 = __ldg(bias + col + e), b1 = __ldg(bias + col + e + 1);
                  if (is_bf16) {
                    x0 += __bfloat162float(__ushort_as_bfloat16(b0));
                    x1 += __bfloat162float(__ushort_as_bfloat16(b1));
                  } else {
                    x0 += __half2float(__ushort_as_half(b0));
                    x1 += __half2float(__ushort_as_half(b1));
                  }
                }
                uint16_t h0, h1;
                if (is_bf16) {
                  h0 = __bfloat16_as_ushort(__float2bfloat16_rn(x0));
                  h1 = __bfloat16_as_ushort(__float2bfloat16_rn(x1));
                } else {
                  h0 = __half_as_ushort(__float2half_rn(x0));
                  h1 = __half_as_ushort(__float2half_rn(x1));
                }
                packed[e / 2] = static_cast<uint32_t>(h0) | (static_cast<uint32_t>(h1) << 16);
              }
              *reinterpret_cast<uint4*>(out + static_cast<int64_t>(v) * cout + col) =
                  make_uint4(packed[0], packed[1], packed[2], packed[3]);
            }
          }
        }
      }
    } else if (v >= 0 && ready) {
      // no tap at all (cannot happen for a live row, whose centre tap exists): bias only
      for (int col = n0; col < n0 + bn && col < cout; ++col) {
        float x = 0.f;
        if (bias) x = is_bf16 ? __bfloat162float(__ushort_as_bfloat16(bias[col]))
                              : __half2float(__ushort_as_half(bias[col]));
        out[static_cast<int64_t>(v) * cout + col] =
            is_bf16 ? __bfloat16_as_ushort(__float2bfloat16_rn(x)) : __half_as_ushort(__float2half_rn(x));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, tmem_cols);
  }
}

// ------------------------------------------------------------------ host
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool conv_tc_supported(const ConvArgs& a) {
  return (a.dtype == kBF16 || a.dtype == kF16) && a.cin >= 64 && a.cin % 16 == 0 && a.cout >= 16 &&
         a.cout % 16 == 0 && aligned16(a.feats) && aligned16(a.weight) && aligned16(a.out) &&
         a.n < (1ll << 31) && (a.taps == 1 || a.taps == kTaps) && encode_fn() != nullptr;
}

static int next_pow2(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

cudaError_t launch_conv_tc(const ConvArgs& a, cudaStream_t s) {
  if (a.n == 0) return cudaSuccess;
  EncodeTiledFn enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  const CUtensorMapDataType dt = a.dtype == kBF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  // Output channel split: at most 256 columns (one MMA N) per CTA.
  const int nsplit = (a.cout + 255) / 256;
  int bn = (a.cout + nsplit - 1) / nsplit;
  bn = (bn + 15) / 16 * 16;
  const uint32_t tmem_cols = static_cast<uint32_t>(next_pow2(bn < 32 ? 32 : bn));

  CUtensorMap fmap, wmap;
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(a.cin), static_cast<cuuint64_t>(a.n)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.cin) * 2};
    const cuuint32_t box[2] = {kKBlock, 1};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&fmap, dt, 2, const_cast<void*>(a.feats), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(a.cin), static_cast<cuuint64_t>(a.taps),
                                static_cast<cuuint64_t>(a.cout)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(a.cin) * 2,
                                   static_cast<cuuint64_t>(a.cin) * a.taps * 2};
    const cuuint32_t box[3] = {kKBlock, 1, static_cast<cuuint32_t>(bn)};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (enc(&wmap, dt, 3, const_cast<void*>(a.weight), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  // Stages: fill about half an SM's shared memory when two CTAs can share
  // the SM's TMEM, otherwise most of it.
  const uint32_t stage_bytes = kABytes + static_cast<uint32_t>(bn) * kKBlock * 2;
  const uint32_t fixed = tc_layout(0, bn).total + 1024;
  const uint32_t budget = tmem_cols <= 256 ? 115 * 1024 - 1024 : 227 * 1024;
  int stages = static_cast<int>((budget - fixed) / stage_bytes);
  if (stages > kMaxStages) stages = kMaxStages;
  if (stages < 2) stages = 2;
  const uint32_t smem = tc_layout(stages, bn).total + 1024;
  cudaError_t e = cudaFuncSetAttribute(k_conv_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t ntiles = (a.n + kTileM - 1) / kTileM;
  dim3 grid(static_cast<unsigned>(ntiles), static_cast<unsigned>(nsplit));
  k_conv_tc<<<grid, kTcThreads, smem, s>>>(fmap, wmap, a.nbr, a.taps == kTaps ? a.perm : nullptr, a.n, a.cin,
                                           a.cout, a.taps, a.orientation, bn, stages, tmem_cols,
                                           a.dtype == kBF16 ? 1 : 0, static_cast<const uint16_t*>(a.bias),
                                           static_cast<uint16_t*>(a.out), a.err);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace smc
