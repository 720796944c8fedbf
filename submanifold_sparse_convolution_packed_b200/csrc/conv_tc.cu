// tcgen05 implicit gather-GEMM for submanifold convolution (bf16 / fp16).
//
// out[v] = bias + sum_d feats[nbr(v, d)] @ W[:, d, :]^T, W in KRSC layout
// [O, kz, ky, kx, I] (LATO.2 MLX port README, summary and "The scope, once
// measured"; orientation per its "Correctness" section).  As a GEMM it is
// M = active voxels, N = Cout, K = 27 * Cin: the A rows of tap d are the
// gathered neighbour rows and B is the weight tensor itself read as a K-major
// [Cout, 27*Cin] matrix (no re-layout).
//
// One CTA computes one work unit: a 128-row tile of the map's tile schedule
// times one block of BN <= 256 output channels.  Only the taps present in the
// tile (precomputed tile mask) are issued; all of them accumulate in one TMEM
// buffer.  Several small CTAs share an SM (up to four when BN <= 128): on
// B200 the rate at which one CTA can pull scattered rows from L2 is capped,
// while the SM as a whole sustains several times more, and co-resident CTAs
// also hide each other's index loads and epilogues.  Warp roles:
//   warp 0     weight slices by 3-D TMA tile loads (and the A tile for k=1);
//   warp 1     TMEM allocation and tcgen05.mma issue (M=128, N=BN, K=16);
//   warps 2-5  first the A gather: each warp owns 32 tile rows, keeps their
//              27 neighbour rows in registers and lets 8 lanes issue TMA
//              tile::gather4 row loads (missing neighbours are row -1, which
//              TMA reads as zeros); then the epilogue for the same rows:
//              tcgen05.ld, bias in fp32, rounding, 16-byte stores.
//              (Or warps 2-9, 16 rows each, 4 issuing lanes: see kGW; or
//              two tiles per CTA, warps 2-9 with 32 rows each: see kMT.)
// Pipeline stages are (tap, channel block) pairs of KB = 32 or 64 channels in
// swizzled shared memory (64-byte or 128-byte swizzle).  Every wait is
// bounded; on timeout the error word gets a bit and the CTA winds down.
#include <atomic>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "epilogue.cuh"
#include "kernels.h"

namespace smc {

constexpr int kTcThreads = 192;  // weight loader, MMA issuer and 4 gather / epilogue warps
constexpr int kMaxStages = 8;

struct TcSmemLayout {
  uint32_t a_off, b_off, bar_off, misc_off, bias_off, total;
};

__host__ __device__ inline TcSmemLayout tc_layout(int stages, int bn, int kb_elems, int mt = 1) {
  TcSmemLayout L;
  const uint32_t a_bytes = static_cast<uint32_t>(mt * kTileRows) * kb_elems * 2;
  const uint32_t b_bytes = static_cast<uint32_t>(bn) * kb_elems * 2;
  L.a_off = 0;
  L.b_off = L.a_off + stages * a_bytes;
  L.bar_off = L.b_off + stages * b_bytes;
  L.misc_off = L.bar_off + (2 * kMaxStages + 2) * 8;
  L.bias_off = L.misc_off + 32;  // the unit's BN bias values (bf16/fp16 bits), 16-byte aligned
  L.total = L.bias_off + 512;
  return L;
}

struct TcParams {
  const int32_t* nbr;
  const int32_t* perm;
  const uint32_t* tile_mask;
  const uint16_t* bias;
  uint16_t* out;
  uint32_t* err;
  int64_t n;
  int64_t ntiles;
  int cin, cout, taps, orientation, bn, nsplit, stages, is_bf16, kb_elems;
  int bias_vec;  // bias present and 16-byte aligned: read 8 values per load
  int stage_out;  // plain epilogue staged through the (then free) stage buffers
  uint32_t tmem_cols;
  uint64_t wait_ns;  // bound of every mbarrier wait
  Epilogue ep;  // activation and residual
};

// kPair: the CTA is one of a cluster pair sharing M = 256 MMAs (rows of two
// consecutive schedule tiles, the union of their tap masks); it loads its own
// 128 gathered rows and half of the weight block's N columns, and every load
// and arrival counts on the even CTA's full barriers.
// kEpi: 0 = bias only; 1 = activation and residual, used only when
// set_conv_epilogue(1) asks for them here: by default a row pass behind the
// conv applies them (k_rows_pass), which measured faster, since everything in
// this epilogue lengthens the tile's hold on its SM slot and the residual rows
// are read in schedule order.  Separate instances keep the plain conv free of
// the extra epilogue code, which measured 5-19% slower even when unused.
// kGW: gather warps (4 or 8).  With 8, warps w and w + 4 share a TMEM lane
// quarter: each gathers 16 of its 32 rows (4 issuing lanes) and, in the
// epilogue, writes half of its columns.  Selected by measurement for the
// plain conv at three CTAs per SM.
// kMT = 2 (with kGW = 8, plain epilogue, k = 3): the CTA owns two consecutive
// schedule tiles and every weight stage feeds two M = 128 MMAs, one per tile,
// into two TMEM accumulators (the union of the two tiles' tap masks is
// issued); warps 2-5 gather and drain the first tile, warps 6-9 the second.
// It halves the weight bytes per output row, at two CTAs per SM.
template <bool kPair, int kEpi, int kGW, int kMT = 1>
__global__ void __launch_bounds__(64 + 32 * kGW, kMT == 2 ? 2 : (kGW == 8 ? 3 : 4))
    k_conv_tc(const __grid_constant__ CUtensorMap fmap,
                                                        const __grid_constant__ CUtensorMap wmap,
                                                        const TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;  // swizzle atoms need aligned bases
  uint8_t* smem = smem_raw + (sbase - raw);
  const int bn_cta = kPair ? p.bn / 2 : p.bn;  // weight rows (output channels) this CTA loads
  const TcSmemLayout L = tc_layout(p.stages, bn_cta, p.kb_elems, kMT);
  const uint32_t bar_full = sbase + L.bar_off;
  const uint32_t bar_empty = bar_full + kMaxStages * 8;
  const uint32_t bar_acc = bar_empty + kMaxStages * 8;
  volatile uint32_t* s_misc = reinterpret_cast<volatile uint32_t*>(smem + L.misc_off);  // [0] tmem, [1] abort

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool k3 = p.taps == kTaps;
  const uint32_t rank = kPair ? cluster_ctarank() : 0u;
  const uint32_t row_bytes = static_cast<uint32_t>(p.kb_elems) * 2;
  const uint32_t a_bytes = kMT * kTileRows * row_bytes;
  const uint32_t b_bytes = static_cast<uint32_t>(bn_cta) * row_bytes;
  const int kblocks = (p.cin + p.kb_elems - 1) / p.kb_elems;
  const int last_ksteps = (p.cin - (kblocks - 1) * p.kb_elems + 15) / 16;
  // One-CTA launches take the schedule's tiles last to first: the schedule
  // sorts rows by ascending corner/edge key, so the tiles with the most taps
  // come last, and launching them first leaves the lighter tiles to fill the
  // final partial wave.
  const int64_t unit = kPair ? blockIdx.x / 2 : gridDim.x - 1 - blockIdx.x;
  const int64_t tile0 = (unit / p.nsplit) * (kPair ? 2 : kMT);  // first tile of the unit
  const int64_t tile = tile0 + rank;
  const int n0 = static_cast<int>(unit % p.nsplit) * p.bn;
  uint32_t mask = 1u;
  if (k3) {
    mask = __ldg(p.tile_mask + tile0);
    if ((kPair || kMT == 2) && tile0 + 1 < p.ntiles) mask |= __ldg(p.tile_mask + tile0 + 1);
    if (p.orientation < 0) mask = mirror27(mask);
  }

  // The gather / epilogue warps (2 ..) own epilogue tile row r (TMEM lane)
  // and its output row v, and gather tile row rg: for k = 3 its 27 neighbour
  // rows, loaded here so that the loads overlap the barrier set-up and the
  // TMEM allocation below.  With 4 gather warps r == rg.
  constexpr int kRPW = kMT * kTileRows / kGW;  // tile rows gathered per warp
  const int q = warp & 3;                // TMEM lane quarter
  // kGW = 8: half of the quarter (rows gathered, columns written); with
  // kMT = 2 the warp's tile instead (all of its 32 rows, all columns)
  const int h = kGW == 8 ? ((warp - 2) >> 2) : 0;
  const int r = q * 32 + lane;
  const int rg = kMT == 2 ? r : q * 32 + h * kRPW + (lane % kRPW);
  const int64_t row0 = (kMT == 2 ? tile0 + h : tile) * kTileRows;  // first schedule entry of the warp's tile
  int32_t v = -1;
  int32_t nb[kTaps];
  // The unit's bias values go to shared memory once, so that the epilogue
  // reads them from there: read from global memory chunk by chunk, their
  // latency was most of the epilogue's time.
  uint16_t* s_bias = reinterpret_cast<uint16_t*>(smem + L.bias_off);
  if (warp >= 2 && p.bias) {
    const int t = tid - 64;
    const int nb_cols = p.cout - n0 < p.bn ? p.cout - n0 : p.bn;
    if (p.bias_vec) {
      if (8 * t < nb_cols) reinterpret_cast<uint4*>(s_bias)[t] = __ldg(reinterpret_cast<const uint4*>(p.bias + n0) + t);
    } else {
      for (int c = t; c < nb_cols; c += 32 * kGW) s_bias[c] = __ldg(p.bias + n0 + c);
    }
  }
  if (warp >= 2) {
    const int64_t g = row0 + r;
    v = g < p.n ? (k3 ? __ldg(p.perm + g) : static_cast<int32_t>(g)) : -1;
    if (v >= p.n) v = -1;  // a schedule left incomplete by a failed build is skipped, never followed
    int32_t vg = v;
    if (kGW != 4 && kMT == 1) {
      const int64_t gg = row0 + rg;
      vg = gg < p.n ? (k3 ? __ldg(p.perm + gg) : static_cast<int32_t>(gg)) : -1;
      if (vg >= p.n) vg = -1;
    }
    if (k3) {
      const int32_t* row = p.nbr + static_cast<int64_t>(vg < 0 ? 0 : vg) * kTaps;
#pragma unroll
      for (int d = 0; d < kTaps; ++d) nb[d] = vg >= 0 ? __ldg(row + (p.orientation > 0 ? d : kTaps - 1 - d)) : -1;
    }
  }

  if (tid == 0) {
    prefetch_tmap(&fmap);
    prefetch_tmap(&wmap);
    for (int s = 0; s < p.stages; ++s) {
      // weight loader (+ the gather warps), of both CTAs for a pair
      mbar_init(bar_full + 8 * s, (k3 ? 1 + kGW : 1) * (kPair ? 2 : 1));
      mbar_init(bar_empty + 8 * s, 1);
    }
    mbar_init(bar_acc, 1);
    s_misc[1] = 0;
    fence_mbarrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    if (kPair) {
      tmem_alloc_pair(smem_u32(const_cast<uint32_t*>(&s_misc[0])), p.tmem_cols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(const_cast<uint32_t*>(&s_misc[0])), p.tmem_cols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (kPair) cluster_sync();  // both CTAs' barriers exist before any remote arrival
  tc_fence_after();
  const uint32_t tmem_base = s_misc[0];
  // full barriers that loads and arrivals count on: the even CTA's for a pair
  const uint32_t full_tgt = kPair ? mapa_shared(bar_full, 0) : bar_full;

  if (warp == 0) {
    // ---------------------------------------------------------- weight loader
    // The whole warp runs the loop (warp-uniform values); lane 0 waits, the
    // warp agrees on the outcome, and one elected lane issues the loads.
    {
      uint32_t it = 0;
      bool ok = true;
      for (uint32_t m = mask; m && ok; m &= m - 1) {
        const int d = __ffs(m) - 1;
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const uint32_t stage = it % p.stages, phase = (it / p.stages) & 1u;
          int w_ok = 1;
          if (lane == 0)
            w_ok = mbar_wait_bounded(bar_empty + 8 * stage, phase ^ 1u, p.err, p.wait_ns) && !s_misc[1];
          if (!__shfl_sync(0xffffffffu, w_ok, 0)) {
            if (lane == 0) s_misc[1] = 1;
            ok = false;
            break;
          }
          const uint32_t full = full_tgt + 8 * stage;
          const uint32_t a_dst = sbase + L.a_off + stage * a_bytes, b_dst = sbase + L.b_off + stage * b_bytes;
          const int32_t a_row = static_cast<int32_t>(tile * kTileRows);
          const int32_t b_row = n0 + static_cast<int32_t>(rank) * bn_cta;
          if (elect_one()) {
            if (kPair) {
              mbar_arrive_expect_tx_cluster(full, b_bytes + (k3 ? 0u : a_bytes));
              if (!k3) tma_load_2d_pair(a_dst, &fmap, full, kb * p.kb_elems, a_row);
              tma_load_3d_pair(b_dst, &wmap, full, kb * p.kb_elems, k3 ? d : 0, b_row);
            } else {
              mbar_arrive_expect_tx(full, b_bytes + (k3 ? 0u : a_bytes));
              if (!k3) tma_load_2d(a_dst, &fmap, full, kb * p.kb_elems, a_row);
              tma_load_3d(b_dst, &wmap, full, kb * p.kb_elems, k3 ? d : 0, b_row);
            }
          }
          __syncwarp();
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    // The whole warp runs the loop with warp-uniform values and one elected
    // lane issues each MMA and commit: measured on B200, a lone thread in a
    // lane-divergent branch issues MMAs about half as fast.  (For a pair only
    // the even CTA issues; the odd one only holds TMEM.)
    if (rank == 0) {
      const uint32_t idesc =
          idesc_f16(static_cast<uint32_t>(p.is_bf16), static_cast<uint32_t>(p.bn), kPair ? 256u : 128u);
      uint32_t it = 0;
      bool ok = true;
      for (uint32_t m = mask; m && ok; m &= m - 1) {
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const uint32_t stage = it % p.stages, phase = (it / p.stages) & 1u;
          const bool w_ok = mbar_wait_bounded(bar_full + 8 * stage, phase, p.err, p.wait_ns);
          if (!__all_sync(0xffffffffu, w_ok && !s_misc[1])) {
            if (lane == 0) s_misc[1] = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t bdesc = kmajor_desc(sbase + L.b_off + stage * b_bytes, row_bytes);
          const int ksteps = kb == kblocks - 1 ? last_ksteps : p.kb_elems / 16;
#pragma unroll
          for (int t = 0; t < kMT; ++t) {
            // tile t's rows and accumulator (columns t * BN ..)
            const uint64_t adesc =
                kmajor_desc(sbase + L.a_off + stage * a_bytes + t * kTileRows * row_bytes, row_bytes);
            const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(t * p.bn);
            for (int k = 0; k < ksteps; ++k) {
              if (kPair)
                umma_f16_pair_elect(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, (it > 0 || k > 0) ? 1u : 0u);
              else
                umma_f16_elect(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, (it > 0 || k > 0) ? 1u : 0u);
            }
          }
          if (kPair) umma_commit_pair_elect(bar_empty + 8 * stage, 3);
          else umma_commit_elect(bar_empty + 8 * stage);
        }
      }
      if (kPair) umma_commit_pair_elect(bar_acc, 3);
      else umma_commit_elect(bar_acc);
    }
  } else {
    // Gather / epilogue warps: this thread's tile row v and its neighbour rows nb.
    if constexpr (kEpi >= 1) {
      // the epilogue reads this row's residual: bring it into L2 now, while
      // the tile's taps are gathered and multiplied
      if (p.ep.residual && v >= 0) {
        const char* rrow = static_cast<const char*>(p.ep.residual) + (static_cast<int64_t>(v) * p.cout + n0) * 2;
        const int bytes = (p.cout - n0 < p.bn ? p.cout - n0 : p.bn) * 2;
        for (int off = 0; off < bytes; off += 128) asm volatile("prefetch.global.L2 [%0];" ::"l"(rrow + off));
      }
    }
    // ---------------------------------------------------------- A gather (k=3)
    if (k3) {
      uint32_t it = 0;
      bool ok = true;
#pragma unroll
      for (int d = 0; d < kTaps; ++d) {
        if (!((mask >> d) & 1u) || !ok) continue;
        // lane j < kRPW / 4 gathers rows 4j .. 4j + 3 of the warp's kRPW rows
        const int src = (lane % (kRPW / 4)) * 4;
        const int32_t r0 = __shfl_sync(0xffffffffu, nb[d], src + 0);
        const int32_t r1 = __shfl_sync(0xffffffffu, nb[d], src + 1);
        const int32_t r2 = __shfl_sync(0xffffffffu, nb[d], src + 2);
        const int32_t r3 = __shfl_sync(0xffffffffu, nb[d], src + 3);
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const uint32_t stage = it % p.stages, phase = (it / p.stages) & 1u;
          int w_ok = 1;
          if (lane == 0)
            w_ok = mbar_wait_bounded(bar_empty + 8 * stage, phase ^ 1u, p.err, p.wait_ns) && !s_misc[1];
          w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
          if (!w_ok) {
            if (lane == 0) s_misc[1] = 1;
            ok = false;
            break;
          }
          const uint32_t full = full_tgt + 8 * stage;
          if (lane == 0) {
            if (kPair) mbar_arrive_expect_tx_cluster(full, kRPW * row_bytes);
            else mbar_arrive_expect_tx(full, kRPW * row_bytes);
          }
          __syncwarp();
          if (lane < kRPW / 4) {
            const int arow = kMT == 2 ? h * kTileRows + q * 32 + 4 * lane : q * 32 + h * kRPW + 4 * lane;
            const uint32_t dst = sbase + L.a_off + stage * a_bytes + arow * row_bytes;
            if (kPair) tma_gather4_pair(dst, &fmap, full, kb * p.kb_elems, r0, r1, r2, r3);
            else tma_gather4(dst, &fmap, full, kb * p.kb_elems, r0, r1, r2, r3);
          }
        }
      }
    }
    // ---------------------------------------------------------- epilogue
    // y = act(acc + bias) + residual, rounded and stored as 16-byte vectors.
    constexpr bool extra = kEpi >= 1;  // activation and residual
    const uint16_t* res = static_cast<const uint16_t*>(p.ep.residual);
    // Residual of 32 output columns from c0 (4 x 16 bytes; zeros past the
    // row's columns).  The first chunk's is loaded before the accumulator is
    // ready (while the last MMAs run) and each later chunk's one chunk ahead;
    // a thread reads and writes only its own row, and loads a column before
    // storing it, so this holds for a residual that is the output buffer.
    auto load_res = [&](int c0, uint4 (&rq)[4]) {
      int nc = p.bn - c0 < 32 ? p.bn - c0 : 32;
      if (p.cout - (n0 + c0) < nc) nc = p.cout - (n0 + c0);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        rq[j] = make_uint4(0, 0, 0, 0);
        if (extra && res && v >= 0 && 8 * j < nc)
          rq[j] = *reinterpret_cast<const uint4*>(res + static_cast<int64_t>(v) * p.cout + n0 + c0 + 8 * j);
      }
    };
    uint4 rcur[4], rnext[4];
    if constexpr (extra) load_res(0, rcur);
    const bool ready = mbar_wait_bounded(bar_acc, 0, p.err, p.wait_ns) && !s_misc[1];
    tc_fence_after();
    if (!extra && ready && p.stage_out) {
      // Plain epilogue through shared memory: the accumulator is complete, so
      // every MMA has consumed its operands and the stage buffers are free.
      // Each warp converts its 32 rows (bias in fp32, rounding) into its own
      // padded row block, then writes whole output rows with coalesced
      // 16-byte stores (a row's bytes are contiguous in `out`), instead of 32
      // scattered rows per store instruction.
      const bool bf = p.is_bf16 != 0;
      const int bw = kMT == 2 ? p.bn : p.bn / (kGW / 4);  // columns this warp writes
      const int c_lo = kMT == 2 ? 0 : h * bw;
      const uint32_t pitch = static_cast<uint32_t>(bw) * 2u + 16u;
      uint8_t* blk = smem + L.a_off + static_cast<uint32_t>(warp - 2) * 32u * pitch;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(c_lo) +
                             (kMT == 2 ? static_cast<uint32_t>(h * p.bn) : 0u);
      int ncols_all = p.cout - n0 - c_lo < bw ? p.cout - n0 - c_lo : bw;
      for (int c0 = 0; c0 < ncols_all; c0 += 32) {
        float acc[32];
        tmem_ld_32cols(t_row + c0, acc);
#pragma unroll
        for (int j = 0; j < 32; j += 8) {
          if (c0 + j >= ncols_all) break;
          float bv[8];
          if (p.bias) {
            const uint4 bq = *reinterpret_cast<const uint4*>(s_bias + c_lo + c0 + j);
            const uint32_t bwd[4] = {bq.x, bq.y, bq.z, bq.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              bv[2 * e] = half_bits_to_float(static_cast<uint16_t>(bwd[e] & 0xFFFFu), bf);
              bv[2 * e + 1] = half_bits_to_float(static_cast<uint16_t>(bwd[e] >> 16), bf);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) bv[e] = 0.f;
          }
          uint32_t packed[4];
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            const uint16_t h0 = float_to_half_bits(acc[j + e] + bv[e], bf);
            const uint16_t h1 = float_to_half_bits(acc[j + e + 1] + bv[e + 1], bf);
            packed[e / 2] = static_cast<uint32_t>(h0) | (static_cast<uint32_t>(h1) << 16);
          }
          *reinterpret_cast<uint4*>(blk + lane * pitch + (c0 + j) * 2) =
              make_uint4(packed[0], packed[1], packed[2], packed[3]);
        }
      }
      __syncwarp();
      // copy out: `cpr` 16-byte chunks per row, 32 / cpr rows per pass
      const int cpr = ncols_all / 8;
      const int rpp = 32 / cpr > 0 ? 32 / cpr : 1;
      for (int r0 = 0; r0 < 32; r0 += rpp) {
        const int rr = r0 + lane / cpr, ch = lane % cpr;
        const int32_t vr = __shfl_sync(0xffffffffu, v, rr < 32 ? rr : 31);
        if (lane < rpp * cpr && rr < 32 && vr >= 0) {
          const uint4 x = *reinterpret_cast<const uint4*>(blk + rr * pitch + ch * 16);
          *reinterpret_cast<uint4*>(p.out + static_cast<int64_t>(vr) * p.cout + n0 + c_lo + ch * 8) = x;
        }
      }
    } else if (ready) {
      const bool bf = p.is_bf16 != 0;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             (kMT == 2 ? static_cast<uint32_t>(h * p.bn) : 0u);
      for (int c0 = 0; c0 < p.bn; c0 += 32) {
        if constexpr (extra) {
          if (c0 + 32 < p.bn) load_res(c0 + 32, rnext);
        }
        float acc[32];
        tmem_ld_32cols(t_row + c0, acc);
        int ncols = p.bn - c0 < 32 ? p.bn - c0 : 32;
        if (p.cout - (n0 + c0) < ncols) ncols = p.cout - (n0 + c0);
        if (v >= 0) {
#pragma unroll
          for (int j = 0; j < 32; j += 8) {
            if (j >= ncols) break;
            const int col = n0 + c0 + j;
            const int64_t at = static_cast<int64_t>(v) * p.cout + col;
            uint32_t rw[4] = {0u, 0u, 0u, 0u};
            if constexpr (extra) {
              rw[0] = rcur[j / 8].x;
              rw[1] = rcur[j / 8].y;
              rw[2] = rcur[j / 8].z;
              rw[3] = rcur[j / 8].w;
            }
            // the 8 bias values of these columns, from shared memory
            float bv[8];
            if (p.bias) {
              const uint4 bq = *reinterpret_cast<const uint4*>(s_bias + c0 + j);
              const uint32_t bw[4] = {bq.x, bq.y, bq.z, bq.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                bv[2 * e] = half_bits_to_float(static_cast<uint16_t>(bw[e] & 0xFFFFu), bf);
                bv[2 * e + 1] = half_bits_to_float(static_cast<uint16_t>(bw[e] >> 16), bf);
              }
            } else {
#pragma unroll
              for (int e = 0; e < 8; ++e) bv[e] = 0.f;
            }
            uint32_t packed[4];
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
              float x0 = acc[j + e] + bv[e], x1 = acc[j + e + 1] + bv[e + 1];
              if constexpr (extra) {
                x0 = apply_act(x0, p.ep.act);
                x1 = apply_act(x1, p.ep.act);
              }
              if (extra && res) {
                x0 += half_bits_to_float(static_cast<uint16_t>(rw[e / 2] & 0xFFFFu), bf);
                x1 += half_bits_to_float(static_cast<uint16_t>(rw[e / 2] >> 16), bf);
              }
              const uint16_t h0 = float_to_half_bits(x0, bf), h1 = float_to_half_bits(x1, bf);
              packed[e / 2] = static_cast<uint32_t>(h0) | (static_cast<uint32_t>(h1) << 16);
            }
            *reinterpret_cast<uint4*>(p.out + at) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
          }
        }
        if constexpr (extra) {
#pragma unroll
          for (int j = 0; j < 4; ++j) rcur[j] = rnext[j];
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (kPair) cluster_sync();  // every MMA of the pair is done and both CTAs have read their TMEM
  if (warp == 1) {
    tc_fence_after();
    if (kPair) tmem_dealloc_pair(tmem_base, p.tmem_cols);
    else tmem_dealloc(tmem_base, p.tmem_cols);
  }
}

// ------------------------------------------------------------------ host
EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

static bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

// SMs of the current device (queried once per device).
static int sm_count() {
  static std::atomic<int> cache[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 148;
  int v = cache[dev].load();
  if (v == 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) {
      cudaGetLastError();
      v = 148;
    }
    cache[dev].store(v);
  }
  return v;
}

bool conv_tc_supported(const ConvArgs& a) {
  return (a.dtype == kBF16 || a.dtype == kF16) && a.cin >= 64 && a.cin % 16 == 0 && a.cout >= 16 &&
         a.cout % 16 == 0 && aligned16(a.feats) && aligned16(a.weight) && aligned16(a.out) &&
         aligned16(a.ep.residual) &&
         a.n < (1ll << 31) && (a.taps == 1 || (a.taps == kTaps && a.perm && a.tile_mask)) &&
         encode_fn() != nullptr;
}

static uint32_t next_pow2(uint32_t x) {
  uint32_t v = 1;
  while (v < x) v <<= 1;
  return v;
}

// Launch shape of one conv: channel split, channel block, CTA pairing and stage count.
struct TcShape {
  int nsplit, bn, kb_elems, stages, ctas_per_sm, mt;
  bool pair;
  uint32_t tmem_cols, smem;
};

static std::atomic<int> g_conv_variant{0};
static std::atomic<int> g_gather_warps{0};  // 0 = by shape; 4 = always four gather warps

static TcShape choose_shape(int cin, int cout, int64_t ntiles, int mt) {
  TcShape t;
  t.mt = mt;
  // At most 256 output channels (one MMA N) per CTA or CTA pair.
  t.nsplit = (cout + 255) / 256;
  t.bn = ((cout + t.nsplit - 1) / t.nsplit + 15) / 16 * 16;
  t.tmem_cols = next_pow2(t.bn < 32 ? 32u : static_cast<uint32_t>(mt * t.bn));
  // CTA pairs halve the weight bytes each CTA pulls through its TMA path, but
  // a cluster launch of a kernel that uses tcgen05 is limited to one cluster
  // per TPC (74 on B200, from the occupancy API and ncu), i.e. one CTA per
  // SM, and this kernel's row-gather rate grows with the CTAs per SM.  The
  // pairs measured 1.5-1.7x slower on every workload, so one CTA per tile is
  // the default and pairs are kept as a selectable, tested alternative.
  (void)ntiles;
  t.pair = g_conv_variant.load() == 2;
  const int bn_cta = t.pair ? t.bn / 2 : t.bn;
  // 64-channel blocks (128-byte rows): one row request per gathered row and
  // K block.  Measured faster than 32-channel blocks with more CTAs per SM
  // (shells 128^3/128ch: 122 us vs 180 us), so the SM holds three CTAs of two
  // or more stages each when BN <= 128.
  // More CTAs per SM pull gathered rows faster than deeper pipelines: at
  // BN = 128, 3 CTAs x 2 stages beat 2 x 3 and 1 x 6 (shells 128^3/128ch:
  // 111 / 135 / 221 us); at BN <= 64, 4 x 2 beat 3 x 3 (256^3 varlen, 64ch:
  // 776 vs 817 us) and 5 x 3 with 32-channel blocks (944 us).  (Pairs use the
  // same per-CTA budget: sized for one CTA per SM, with eight stages, they
  // measured slower still.)
  t.ctas_per_sm = t.tmem_cols <= 64 ? 4 : (t.tmem_cols <= 128 ? 3 : 2);
  if (mt == 2) t.ctas_per_sm = 2;  // TMEM: two accumulators of up to 128 columns
  t.kb_elems = 64;
  (void)cin;
  const uint32_t per_sm = 228u * 1024u;
  const uint32_t budget = per_sm / t.ctas_per_sm - 1024u;  // 1 KB per CTA is reserved by the system
  const uint32_t stage_bytes = static_cast<uint32_t>(mt * kTileRows + bn_cta) * t.kb_elems * 2;
  const uint32_t fixed = tc_layout(0, bn_cta, t.kb_elems, mt).total + 1024u;
  int stages = budget > fixed ? static_cast<int>((budget - fixed) / stage_bytes) : 0;
  if (stages > kMaxStages) stages = kMaxStages;
  if (stages < 2) stages = 2;
  t.stages = stages;
  t.smem = tc_layout(stages, bn_cta, t.kb_elems, mt).total + 1024u;
  return t;
}

void set_conv_variant(int v) { g_conv_variant.store(v); }

static std::atomic<int> g_conv_epilogue{0};
void set_conv_epilogue(int where) { g_conv_epilogue.store(where); }
int conv_epilogue() { return g_conv_epilogue.load(); }
int conv_variant() { return g_conv_variant.load(); }

cudaError_t launch_conv_tc(const ConvArgs& a, cudaStream_t s) {
  if (a.n == 0) return cudaSuccess;
  EncodeTiledFn enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  const CUtensorMapDataType dt = a.dtype == kBF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const int64_t ntiles = (a.n + kTileRows - 1) / kTileRows;
  const int epi = a.ep.act != kActNone || a.ep.residual ? 1 : 0;
  const int variant = g_conv_variant.load();
  // Two tiles per CTA (the plain k = 3 conv, 64 or 128 output channels):
  // the default for 64 output channels, and for 128 when the map has at
  // least eight waves of two-tile units at two CTAs per SM.  Measured on
  // B200 (conv alone, L2 flushed, one tile per CTA -> two): 512^3 decoder
  // stage, 64 ch, 0.500 -> 0.447 ms; four-item 256^3 set, 64 ch fp16, 0.683
  // -> 0.628 ms.  At 128 channels the weight bytes halve too, but a small
  // map's tiles fill fewer waves of the two CTA slots per SM: 6-shell 128^3,
  // 0.098 -> 0.123 ms; on the full 128^3 grid (16384 tiles) even at full
  // clock (1.92 ms) and 10% faster inside pipelined steps under the power
  // cap (2.16 -> 1.94 ms at 1.6 GHz).  Four stages at one CTA per SM were
  // slower everywhere (6-shell 0.125 ms, decoder stage 0.879 ms).
  const bool big = ntiles >= 8ll * 2 * 2 * sm_count();
  const bool two = (variant == 4 || (variant == 0 && (a.cout == 64 || (a.cout == 128 && big)))) && epi == 0 &&
                   a.taps == kTaps && a.cout <= 128 && a.cout % 64 == 0;
  const TcShape t = choose_shape(a.cin, a.cout, ntiles, two ? 2 : 1);
  const CUtensorMapSwizzle sw = t.kb_elems == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;

  CUtensorMap fmap, wmap;
  {
    // feats [n, cin]: gather4 boxes of one row (k=3) or tiles of 128 rows (k=1)
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(a.cin), static_cast<cuuint64_t>(a.n)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.cin) * 2};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(t.kb_elems),
                               a.taps == kTaps ? 1u : static_cast<cuuint32_t>(kTileRows)};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&fmap, dt, 2, const_cast<void*>(a.feats), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    // weight [cout, taps, cin]; a CTA of a pair loads half of the block's rows
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(a.cin), static_cast<cuuint64_t>(a.taps),
                                static_cast<cuuint64_t>(a.cout)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(a.cin) * 2,
                                   static_cast<cuuint64_t>(a.cin) * a.taps * 2};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(t.kb_elems), 1,
                               static_cast<cuuint32_t>(t.pair ? t.bn / 2 : t.bn)};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (enc(&wmap, dt, 3, const_cast<void*>(a.weight), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  TcParams p;
  p.nbr = a.nbr;
  p.perm = a.perm;
  p.tile_mask = a.tile_mask;
  p.bias = static_cast<const uint16_t*>(a.bias);
  p.bias_vec = a.bias && aligned16(a.bias) ? 1 : 0;
  // The staged epilogue needs gather warps x 32 rows x (the warp's row bytes
  // + 16) of the stage buffers (A and B regions, contiguous).  Eight gather
  // warps serve the plain k = 3 conv at three CTAs per SM when it fits.
  auto staged_fits = [&](int gw) {
    const uint32_t bw = t.mt == 2 ? static_cast<uint32_t>(t.bn) : static_cast<uint32_t>(t.bn) / (gw / 4);
    const uint32_t need = static_cast<uint32_t>(gw) * 32u * (bw * 2u + 16u);
    const uint32_t have =
        static_cast<uint32_t>(t.stages) * (static_cast<uint32_t>(t.mt * kTileRows + t.bn) * t.kb_elems * 2u);
    return need <= have;
  };
  const bool gw8 = !t.pair && epi == 0 && a.taps == kTaps && t.ctas_per_sm == 3 && t.bn % 64 == 0 &&
                   staged_fits(8) && g_gather_warps.load() != 4;
  if (two && !staged_fits(8)) return cudaErrorInvalidConfiguration;  // does not happen for BN <= 128
  p.stage_out = !t.pair && staged_fits(gw8 || two ? 8 : 4) ? 1 : 0;
  p.out = static_cast<uint16_t*>(a.out);
  p.err = a.err;
  // A conv's waits are bounded too, but never below 100 ms: a CTA that
  // gave up a wait early would leave with its TMA loads still in flight.
  p.wait_ns = scan_wait_limit_ns() > 100000000ull ? scan_wait_limit_ns() : 100000000ull;
  p.n = a.n;
  p.ntiles = ntiles;
  p.cin = a.cin;
  p.cout = a.cout;
  p.taps = a.taps;
  p.orientation = a.orientation;
  p.bn = t.bn;
  p.nsplit = t.nsplit;
  p.stages = t.stages;
  p.is_bf16 = a.dtype == kBF16 ? 1 : 0;
  p.kb_elems = t.kb_elems;
  p.tmem_cols = t.tmem_cols;
  p.ep = a.ep;
  cudaError_t e;
  if (t.pair) {
    auto kern = epi == 1 ? k_conv_tc<true, 1, 4> : k_conv_tc<true, 0, 4>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(t.smem));
    if (e != cudaSuccess) return e;
    const int64_t ctas = 2 * ((ntiles + 1) / 2) * t.nsplit;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(ctas), 1, 1);
    cfg.blockDim = dim3(kTcThreads, 1, 1);
    cfg.dynamicSmemBytes = t.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, fmap, wmap, p);
  } else {
    auto kern = two   ? k_conv_tc<false, 0, 8, 2>
                : gw8 ? k_conv_tc<false, 0, 8>
                      : (epi == 1 ? k_conv_tc<false, 1, 4> : k_conv_tc<false, 0, 4>);
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(t.smem));
    if (e != cudaSuccess) return e;
    const int64_t units = (two ? (ntiles + 1) / 2 : ntiles) * t.nsplit;
    const int threads = gw8 || two ? 64 + 32 * 8 : kTcThreads;
    kern<<<static_cast<unsigned>(units), threads, t.smem, s>>>(fmap, wmap, p);
    e = cudaGetLastError();
  }
  count_launches(1);
  return e;
}

}  // namespace smc
