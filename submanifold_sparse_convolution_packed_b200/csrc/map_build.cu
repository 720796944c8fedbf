// Neighbour-map construction for submanifold convolution (sm_100a).
//
// The pages build a "sorted-key indice map" with 27 vectorised lookups per
// voxel, cached per coordinate set (LATO.2 MLX port README, summary).  Here
// the lookup structure is an open-addressing hash table in device memory:
//   k_insert      one thread per voxel: validate (b,z,y,x), form the 64-bit
//                 linear site key, insert (key,row) with atomicCAS and linear
//                 probing; duplicates and a full table set error bits.
//   k_neighbours  one thread per voxel: 27 lookups -> int32 [n,27] map row
//                 (staged in shared memory, written coalesced), the row's
//                 schedule key, per-block hit counts and the histogram of the
//                 first radix digit of the schedule keys.
//   scan          single-pass exclusive scan (decoupled look-back) of the
//                 block counts in (offset, block) order.
//   k_pairs       stable compaction of every map column into the per-offset
//                 pair lists (ascending output row).
//   radix sort    stable 2x10-bit LSD sort of rows by the schedule key: the
//                 order in which the tensor-core conv forms 128-row tiles.
//                 Each pass is one look-back scan of its histogram plus one
//                 scatter; the first scatter also counts the second digit,
//                 the second one ORs the tile tap masks.
#include <atomic>
#include <cstdint>
#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace smc {

constexpr uint64_t kEmpty = ~0ull;
constexpr int kMapBlock = 256;       // rows per neighbour / pair block
constexpr int kRadixBits = 10;
constexpr int kRadixBins = 1 << kRadixBits;
constexpr int kRadixThreads = 256;
constexpr int kRadixRounds = 8;
constexpr int kRadixChunk = kRadixThreads * kRadixRounds;  // rows per radix block
static_assert(kRadixChunk % kMapBlock == 0, "a radix chunk is a whole number of map blocks");

// Radix histograms are laid out segment by segment: [segment][digit][chunk of
// the segment], cps chunks per segment.  Scanning that layout in order sorts
// every segment of cps * kRadixChunk consecutive rows on its own and keeps the
// segments in input order (cps = all chunks: one stable sort of the map).
__host__ __device__ __forceinline__ int64_t hist_index(uint32_t digit, int64_t chunk, int cps, int bins) {
  return ((chunk / cps) * bins + digit) * cps + chunk % cps;
}
constexpr uint64_t kFib = 0x9E3779B97F4A7C15ull;

__device__ __forceinline__ uint64_t slot_of(uint64_t key, int lg) { return (key * kFib) >> (64 - lg); }

__device__ __forceinline__ bool site_ok(int4 c, int32_t batch, int32_t Z, int32_t Y, int32_t X) {
  return c.x >= 0 && c.x < batch && c.y >= 0 && c.y < Z && c.z >= 0 && c.z < Y && c.w >= 0 &&
         c.w < X;
}

__device__ __forceinline__ uint64_t site_key(int4 c, int32_t Z, int32_t Y, int32_t X) {
  return ((static_cast<uint64_t>(c.x) * Z + c.y) * Y + c.z) * X + c.w;
}

// Lookup structures (MapKind): packed hash slots, one word (key << 32) | row,
// for keys < 2^32 - 1; wide hash slots, two words, key then row; or a dense
// index grid, one int32 row per site of the batch x Z x Y x X box, either
// cleared to -1 at every build (kMapDense) or left as it is and read only
// where a cleared occupancy bitmap, one bit per site, has the site's bit set
// (kMapDenseOcc: a 32x smaller clear for boxes much larger than L2).
template <int kKind>
__global__ void __launch_bounds__(256) k_insert(const int4* __restrict__ coords, int64_t n, int32_t batch,
                                                int32_t Z, int32_t Y, int32_t X,
                                                unsigned long long* table, int lg, uint32_t* occ,
                                                uint32_t* err, uint32_t* __restrict__ zero, int64_t nzero) {
  const uint64_t mask = (1ull << lg) - 1;
  // words later kernels accumulate into (the tile tap masks)
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < nzero;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    zero[i] = 0u;
  for (int64_t v = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; v < n;
       v += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int4 c = coords[v];
    if (!site_ok(c, batch, Z, Y, X)) {
      atomicOr(err, kErrRange);
      continue;
    }
    const uint64_t key = site_key(c, Z, Y, X);
    if (kKind == kMapDense) {
      const int prev = atomicCAS(reinterpret_cast<int*>(table) + key, -1, static_cast<int>(v));
      if (prev != -1) atomicOr(err, kErrDuplicate);
      continue;
    }
    if (kKind == kMapDenseOcc) {
      // the first row to set the site's bit owns the grid entry; the entry is
      // read only after this kernel, so no later reader sees it unwritten
      const uint32_t bit = 1u << (key & 31u);
      if (atomicOr(occ + (key >> 5), bit) & bit) atomicOr(err, kErrDuplicate);
      else reinterpret_cast<int32_t*>(table)[key] = static_cast<int32_t>(v);
      continue;
    }
    uint64_t s = slot_of(key, lg);
    bool placed = false;
    for (uint64_t probe = 0; probe <= mask; ++probe) {
      if (kKind == kMapPacked) {
        const unsigned long long want = (key << 32) | static_cast<uint32_t>(v);
        const unsigned long long prev = atomicCAS(&table[s], kEmpty, want);
        if (prev == kEmpty) { placed = true; break; }
        if ((prev >> 32) == key) { atomicOr(err, kErrDuplicate); placed = true; break; }
      } else {
        const unsigned long long prev = atomicCAS(&table[2 * s], kEmpty, key);
        if (prev == kEmpty) { table[2 * s + 1] = static_cast<uint64_t>(v); placed = true; break; }
        if (prev == key) { atomicOr(err, kErrDuplicate); placed = true; break; }
      }
      s = (s + 1) & mask;
    }
    if (!placed) atomicOr(err, kErrCapacity);
  }
}

// Linear probing from slot s; at most one pass over the table.
template <int kKind>
__device__ __noinline__ int32_t lookup_from(const unsigned long long* __restrict__ table, uint64_t mask,
                                            uint64_t s, uint64_t key) {
  for (uint64_t probe = 0; probe <= mask; ++probe) {
    if (kKind == kMapPacked) {
      const uint64_t e = __ldg(&table[s]);
      if (e == kEmpty) return -1;
      if ((e >> 32) == key) return static_cast<int32_t>(e & 0xFFFFFFFFull);
    } else {
      const uint64_t k = __ldg(&table[2 * s]);
      if (k == kEmpty) return -1;
      if (k == key) return static_cast<int32_t>(__ldg(&table[2 * s + 1]));
    }
    s = (s + 1) & mask;
  }
  return -1;
}

// Schedule key of a row, from its 27-bit hit mask.  Bits 19..0 hold the 8
// corner offsets then the 12 edge offsets, most significant first: rows whose
// rarer neighbours agree sort next to each other, so a 128-row tile shares
// most of its absent taps.  Bits 26..20 carry the other 7 hit bits (the 6
// faces and the centre), so the key holds the whole mask; the sort reads
// bits 19..0 only.
__device__ __forceinline__ uint32_t group_key(uint32_t m) {
  constexpr int kOrder[27] = {0, 2, 6, 8, 18, 20, 24, 26, 1, 3, 5, 7, 9, 11,
                              15, 17, 19, 21, 23, 25, 4, 10, 12, 13, 14, 16, 22};
  uint32_t k = 0;
#pragma unroll
  for (int i = 0; i < 20; ++i) k |= ((m >> kOrder[i]) & 1u) << (19 - i);
#pragma unroll
  for (int i = 20; i < 27; ++i) k |= ((m >> kOrder[i]) & 1u) << i;
  return k;
}

// The hit mask back from a schedule key.
__device__ __forceinline__ uint32_t key_hits(uint32_t k) {
  constexpr int kOrder[27] = {0, 2, 6, 8, 18, 20, 24, 26, 1, 3, 5, 7, 9, 11,
                              15, 17, 19, 21, 23, 25, 4, 10, 12, 13, 14, 16, 22};
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < 20; ++i) m |= ((k >> (19 - i)) & 1u) << kOrder[i];
#pragma unroll
  for (int i = 20; i < 27; ++i) m |= ((k >> i) & 1u) << kOrder[i];
  return m;
}

// Maps of at most kOnePassRows rows get a one-pass tile schedule: a stable
// sort on the high 8 bits of the key (the 8 corner offsets), 256 bins.  For
// them the schedule's launches are latency-bound: a second pass costs more
// (a look-back scan and a scatter, about 20 us on B200) than the conv gains
// from the finer grouping (tap efficiency 0.855 with 10 bits and 0.882 with
// all 20 on the 6-shell 128^3 workload), and 256 bins instead of 1024 cut
// the scatter's per-block work (its digit table and offsets) by four for a
// tap efficiency of 0.846.
constexpr int64_t kOnePassRows = 131072;
constexpr int kOnePassBits = 8;
constexpr int kOnePassBins = 1 << kOnePassBits;
__host__ __device__ __forceinline__ bool schedule_one_pass(int64_t n) { return n <= kOnePassRows; }
// Radix bins of a map's first (or only) schedule pass.
__host__ __device__ __forceinline__ int schedule_bins(int64_t n) {
  return schedule_one_pass(n) ? kOnePassBins : kRadixBins;
}

// Schedule segments are whole radix chunks (see set_schedule_segment_rows).
static_assert(kScheduleSegmentDefault % kRadixChunk == 0, "segments are whole radix chunks");

// The end of a 256-row block of a map-building kernel, once each thread's row
// is in s_nbr and its hit mask and schedule key are known: the first radix
// digit's histogram (one atomic per distinct digit of a warp), the per-offset
// hit counts of the block, and the block's map rows stored in 16-byte vectors.
__device__ __forceinline__ void emit_map_block(const int32_t* s_nbr, int32_t (*s_cnt)[kTaps], uint32_t hits,
                                               uint32_t gk, int64_t base, int64_t n, int32_t* __restrict__ nbr,
                                               int32_t* __restrict__ block_counts, int nblocks,
                                               int32_t* __restrict__ hist1, int radix_cps) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t v = base + tid;
  if (hist1) {
    // the digit of the schedule's first pass: the low 10 bits, or the high
    // 10 for a map sorted in one pass
    const bool one = schedule_one_pass(n);
    const int shift = one ? 2 * kRadixBits - kOnePassBits : 0;
    const int bins = one ? kOnePassBins : kRadixBins;
    const uint32_t digit = v < n ? ((gk >> shift) & static_cast<uint32_t>(bins - 1)) : 0xFFFFFFFFu;
    const uint32_t peers = __match_any_sync(0xffffffffu, digit);
    if (v < n && (__ffs(peers) - 1) == lane)
      atomicAdd(&hist1[hist_index(digit, base / kRadixChunk, radix_cps, bins)], __popc(peers));
  }
#pragma unroll
  for (int d = 0; d < kTaps; ++d) {
    const uint32_t b = __ballot_sync(0xffffffffu, (hits >> d) & 1u);
    if (lane == 0) s_cnt[warp][d] = __popc(b);
  }
  __syncthreads();
  const int64_t rows = n - base < kMapBlock ? n - base : kMapBlock;
  const int total = static_cast<int>(rows) * kTaps;
  int32_t* dst = nbr + base * kTaps;  // base*27*4 bytes is a multiple of 16
  const int vec = total >> 2;
  for (int i = tid; i < vec; i += kMapBlock)
    reinterpret_cast<int4*>(dst)[i] = reinterpret_cast<const int4*>(s_nbr)[i];
  for (int i = (vec << 2) + tid; i < total; i += kMapBlock) dst[i] = s_nbr[i];
  if (tid < kTaps) {
    int32_t c = 0;
#pragma unroll
    for (int w = 0; w < kMapBlock / 32; ++w) c += s_cnt[w][tid];
    block_counts[static_cast<int64_t>(tid) * nblocks + blockIdx.x] = c;
  }
}

// The 27 neighbour rows of the valid site c (key `key`) from the dense index
// grid: the 9 (dz, dy) lines, three consecutive x sites each.  Returns the
// 27-bit hit mask.
__device__ __forceinline__ uint32_t dense_row_lookups(const int32_t* __restrict__ g, int4 c, uint64_t key,
                                                      int32_t Z, int32_t Y, int32_t X, int32_t* out) {
  const int64_t sz = static_cast<int64_t>(Y) * X;
  uint32_t hits = 0;
#pragma unroll
  for (int l = 0; l < 9; ++l) {
    const int dz = l / 3 - 1, dy = l % 3 - 1;
    const bool line = c.y + dz >= 0 && c.y + dz < Z && c.z + dy >= 0 && c.z + dy < Y;
    const int64_t at = static_cast<int64_t>(key) + dz * sz + static_cast<int64_t>(dy) * X;
    const int32_t r0 = line && c.w > 0 ? __ldg(g + at - 1) : -1;
    const int32_t r1 = line ? __ldg(g + at) : -1;
    const int32_t r2 = line && c.w + 1 < X ? __ldg(g + at + 1) : -1;
    out[3 * l + 0] = r0;
    out[3 * l + 1] = r1;
    out[3 * l + 2] = r2;
    hits |= (static_cast<uint32_t>(r0 >= 0) | static_cast<uint32_t>(r1 >= 0) << 1 |
             static_cast<uint32_t>(r2 >= 0) << 2) << (3 * l);
  }
  return hits;
}

// The same 27 lookups over a grid that was not cleared: each line's three
// sites are first looked up in the occupancy bitmap (one or two words), and
// only sites whose bit is set read the grid.
__device__ __forceinline__ uint32_t dense_occ_row_lookups(const int32_t* __restrict__ g,
                                                          const uint32_t* __restrict__ occ, int4 c, uint64_t key,
                                                          int32_t Z, int32_t Y, int32_t X, int32_t* out) {
  const int64_t sz = static_cast<int64_t>(Y) * X;
  uint32_t hits = 0;
#pragma unroll
  for (int l = 0; l < 9; ++l) {
    const int dz = l / 3 - 1, dy = l % 3 - 1;
    const bool line = c.y + dz >= 0 && c.y + dz < Z && c.z + dy >= 0 && c.z + dy < Y;
    const int64_t at = static_cast<int64_t>(key) + dz * sz + static_cast<int64_t>(dy) * X;
    uint32_t b3 = 0;  // bit j: site at - 1 + j is occupied
    if (line) {
      const int64_t lo = c.w > 0 ? at - 1 : at;       // first site of the run inside the box
      const int64_t hi = c.w + 1 < X ? at + 1 : at;   // last one
      const uint32_t wl = __ldg(occ + (lo >> 5));
      const uint32_t wh = (hi >> 5) != (lo >> 5) ? __ldg(occ + (hi >> 5)) : wl;
#pragma unroll
      for (int j = 0; j < 3; ++j) {
        const int64_t k = at - 1 + j;
        if (k < lo || k > hi) continue;
        const uint32_t w = (k >> 5) == (lo >> 5) ? wl : wh;
        b3 |= ((w >> (k & 31)) & 1u) << j;
      }
    }
    const int32_t r0 = (b3 & 1u) ? __ldg(g + at - 1) : -1;
    const int32_t r1 = (b3 & 2u) ? __ldg(g + at) : -1;
    const int32_t r2 = (b3 & 4u) ? __ldg(g + at + 1) : -1;
    out[3 * l + 0] = r0;
    out[3 * l + 1] = r1;
    out[3 * l + 2] = r2;
    hits |= b3 << (3 * l);
  }
  return hits;
}

template <int kKind>
__global__ void __launch_bounds__(kMapBlock) k_neighbours(
    const int4* __restrict__ coords, int64_t n, int32_t batch, int32_t Z, int32_t Y, int32_t X,
    const unsigned long long* __restrict__ table, int lg, const uint32_t* __restrict__ occ,
    int32_t* __restrict__ nbr, uint32_t* __restrict__ gkey, int32_t* __restrict__ block_counts, int nblocks,
    int32_t* __restrict__ hist1, int radix_cps) {
  __shared__ int32_t s_nbr[kMapBlock * kTaps];
  __shared__ int32_t s_cnt[kMapBlock / 32][kTaps];
  const uint64_t mask = (1ull << lg) - 1;
  const int tid = threadIdx.x;
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kMapBlock;
  const int64_t v = base + tid;
  uint32_t hits = 0, gk = 0;
  const int4 c = v < n ? coords[v] : make_int4(-1, 0, 0, 0);
  if (v < n && !site_ok(c, batch, Z, Y, X)) {
    // a row outside the box (the build reports SMC_E_RANGE) has no
    // neighbours, so every map entry stays -1 or a valid row
#pragma unroll
    for (int d = 0; d < kTaps; ++d) s_nbr[tid * kTaps + d] = -1;
    gk = group_key(0u);
    gkey[v] = gk;
  } else if (v < n) {
    const uint64_t key = site_key(c, Z, Y, X);
    const int64_t sz = static_cast<int64_t>(Y) * X;
    if (kKind == kMapDense) {
      hits = dense_row_lookups(reinterpret_cast<const int32_t*>(table), c, key, Z, Y, X, s_nbr + tid * kTaps);
    } else if (kKind == kMapDenseOcc) {
      hits = dense_occ_row_lookups(reinterpret_cast<const int32_t*>(table), occ, c, key, Z, Y, X,
                                   s_nbr + tid * kTaps);
    } else if (kKind == kMapWide) {
      // two-word slots: plain linear probing per lookup
#pragma unroll 1
      for (int d = 0; d < kTaps; ++d) {
        const int dz = d / 9 - 1, dy = (d / 3) % 3 - 1, dx = d % 3 - 1;
        int32_t r = -1;
        if (c.y + dz >= 0 && c.y + dz < Z && c.z + dy >= 0 && c.z + dy < Y && c.w + dx >= 0 && c.w + dx < X) {
          const uint64_t nk = key + static_cast<uint64_t>(dz * sz + static_cast<int64_t>(dy) * X + dx);
          r = lookup_from<kMapWide>(table, mask, slot_of(nk, lg), nk);
        }
        s_nbr[tid * kTaps + d] = r;
        hits |= static_cast<uint32_t>(r >= 0) << d;
      }
    } else {
    // Per kernel plane (dz) the 9 lookups run in lockstep: each round loads,
    // for every still-unresolved lookup, the aligned 2-slot group (16 bytes)
    // holding its next probe position and scans it in probing order.  With
    // the table at <= 1/4 load almost every lookup resolves in the first round.
#pragma unroll
    for (int pz = 0; pz < 3; ++pz) {
      const uint64_t pkey = key + static_cast<uint64_t>((pz - 1) * sz);  // key of the (dz, 0, 0) neighbour
      auto nkey = [&](int j) -> uint64_t {
        return pkey + static_cast<uint64_t>(static_cast<int64_t>(j / 3 - 1) * X + (j % 3 - 1));
      };
      uint64_t pos[9];
      int32_t res[9];
      uint32_t pend = 0, odd = 0;
#pragma unroll
      for (int j = 0; j < 9; ++j) {
        const int dz = pz - 1, dy = j / 3 - 1, dx = j % 3 - 1;
        const bool in = c.y + dz >= 0 && c.y + dz < Z && c.z + dy >= 0 && c.z + dy < Y && c.w + dx >= 0 &&
                        c.w + dx < X;
        const uint64_t h = slot_of(nkey(j), lg);
        pos[j] = h & ~static_cast<uint64_t>(1);
        odd |= static_cast<uint32_t>(h & 1u) << j;  // probing starts at the group's second slot
        res[j] = -1;
        pend |= static_cast<uint32_t>(in) << j;
      }
      for (uint64_t round = 0; pend != 0 && round <= (mask >> 1); ++round) {
        ulonglong2 g[9];
#pragma unroll
        for (int j = 0; j < 9; ++j)
          if ((pend >> j) & 1u) g[j] = __ldg(reinterpret_cast<const ulonglong2*>(table + pos[j]));
#pragma unroll
        for (int j = 0; j < 9; ++j) {
          if (!((pend >> j) & 1u)) continue;
          bool done = false;
          if (!((odd >> j) & 1u)) {
            if (g[j].x == kEmpty) {
              done = true;
            } else if ((g[j].x >> 32) == nkey(j)) {
              res[j] = static_cast<int32_t>(g[j].x & 0xFFFFFFFFull);
              done = true;
            }
          }
          if (!done) {
            if (g[j].y == kEmpty) {
              done = true;
            } else if ((g[j].y >> 32) == nkey(j)) {
              res[j] = static_cast<int32_t>(g[j].y & 0xFFFFFFFFull);
              done = true;
            }
          }
          if (done) pend &= ~(1u << j);
          else pos[j] = (pos[j] + 2) & mask;
        }
        odd = 0;
      }
#pragma unroll
      for (int j = 0; j < 9; ++j) {
        s_nbr[tid * kTaps + 9 * pz + j] = res[j];
        hits |= static_cast<uint32_t>(res[j] >= 0) << (9 * pz + j);
      }
    }
    }
    gk = group_key(hits);
    gkey[v] = gk;
  }
  emit_map_block(s_nbr, s_cnt, hits, gk, base, n, nbr, block_counts, nblocks, hist1, radix_cps);
}

// ------------------------------------------------------------ subdivision
// The children of parent row v are the sites (b, 2z+a, 2y+c, 2x+e), kept
// where keep[8v + k] is nonzero (all when keep is null) and numbered in
// (parent row, k) order, where k is the octant o = 4a + 2c + e (C order,
// subdivide) or, for order 1, the upsample mask's index j = a + 2c + 4e.
__device__ __forceinline__ int octant_of(int k, int order) {
  return order ? ((k & 1) << 2) | (k & 2) | ((k >> 2) & 1) : k;
}

__global__ void k_subdiv_count(const uint8_t* __restrict__ keep, int64_t n, uint8_t* __restrict__ bits,
                               int32_t* __restrict__ cnt) {
  for (int64_t v = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; v < n;
       v += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    uint32_t b = 0xFFu;
    if (keep) {
      b = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) b |= static_cast<uint32_t>(keep[8 * v + k] != 0) << k;
    }
    bits[v] = static_cast<uint8_t>(b);
    cnt[v] = __popc(b);
  }
}

// One block of kEmitBlock parents: their children form one contiguous run of
// the output, staged in shared memory and stored coalesced.
constexpr int kEmitBlock = 256;

__global__ void __launch_bounds__(kEmitBlock) k_subdiv_emit(const int4* __restrict__ coords, int64_t n, int order,
                                                            const uint8_t* __restrict__ bits,
                                                            const int64_t* __restrict__ first,
                                                            int4* __restrict__ child_coords,
                                                            int32_t* __restrict__ child_src,
                                                            int32_t* __restrict__ remap) {
  __shared__ int4 s_coords[8 * kEmitBlock];
  __shared__ int32_t s_src[8 * kEmitBlock];
  __shared__ int s_total;
  const int tid = threadIdx.x;
  const int64_t v0 = static_cast<int64_t>(blockIdx.x) * kEmitBlock;
  const int64_t v = v0 + tid;
  const int64_t base = first[v0];
  if (tid == 0) s_total = 0;
  __syncthreads();
  if (v < n) {
    const int4 c = coords[v];
    const uint32_t b = bits[v];
    const int64_t local = first[v] - base;
    // always in range, unless the scan gave up on a wait (error bit set)
    const bool ok = local >= 0 && local + __popc(b) <= 8 * kEmitBlock;
    int r = static_cast<int>(ok ? local : 0);
    int32_t rm[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int o = octant_of(k, order);
      rm[o] = -1;
      if (ok && ((b >> k) & 1u)) {
        s_coords[r] = make_int4(c.x, 2 * c.y + (o >> 2), 2 * c.z + ((o >> 1) & 1), 2 * c.w + (o & 1));
        s_src[r] = static_cast<int32_t>(8 * v + o);
        rm[o] = static_cast<int32_t>(base + r);
        ++r;
      }
    }
    reinterpret_cast<int4*>(remap)[2 * v] = make_int4(rm[0], rm[1], rm[2], rm[3]);
    reinterpret_cast<int4*>(remap)[2 * v + 1] = make_int4(rm[4], rm[5], rm[6], rm[7]);
    if (ok) atomicMax(&s_total, r);
  }
  __syncthreads();
  const int total = s_total;
  const int64_t cap = 8 * n;
  for (int i = tid; i < total; i += kEmitBlock) {
    if (base + i < cap) {
      child_coords[base + i] = s_coords[i];
      child_src[base + i] = s_src[i];
    }
  }
}

// Map rows of the children, read off the parent map with no lookup
// structure: child 2p+o and offset D reach the site 2p+o+D, whose parent is
// p's neighbour at offset floor((o+D)/2) and whose octant is (o+D) mod 2;
// that child's row is remap[8*parent + octant] (-1 if it was not kept).
__global__ void __launch_bounds__(kMapBlock) k_subdiv_neighbours(
    const int32_t* __restrict__ parent_nbr, const int32_t* __restrict__ child_src,
    const int32_t* __restrict__ remap, int64_t m, int32_t* __restrict__ nbr, uint32_t* __restrict__ gkey,
    int32_t* __restrict__ block_counts, int nblocks, int32_t* __restrict__ hist1, int radix_cps) {
  __shared__ int32_t s_nbr[kMapBlock * kTaps];
  __shared__ int32_t s_cnt[kMapBlock / 32][kTaps];
  const int tid = threadIdx.x;
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kMapBlock;
  const int64_t v = base + tid;
  uint32_t hits = 0, gk = 0;
  if (v < m) {
    const int32_t src = child_src[v];
    const int64_t p = src >> 3;
    const int oz = (src >> 2) & 1, oy = (src >> 1) & 1, ox = src & 1;
    const int32_t* prow = parent_nbr + p * kTaps;
#pragma unroll
    for (int d = 0; d < kTaps; ++d) {
      const int tz = oz + d / 9 - 1, ty = oy + (d / 3) % 3 - 1, tx = ox + d % 3 - 1;  // in -1 .. 2
      const int pd = 9 * ((tz >> 1) + 1) + 3 * ((ty >> 1) + 1) + ((tx >> 1) + 1);
      const int32_t q = __ldg(prow + pd);
      const int32_t r = q < 0 ? -1 : __ldg(remap + 8 * static_cast<int64_t>(q) + 4 * (tz & 1) + 2 * (ty & 1) + (tx & 1));
      s_nbr[tid * kTaps + d] = r;
      hits |= static_cast<uint32_t>(r >= 0) << d;
    }
    gk = group_key(hits);
    gkey[v] = gk;
  }
  emit_map_block(s_nbr, s_cnt, hits, gk, base, m, nbr, block_counts, nblocks, hist1, radix_cps);
}

// The block's share of every pair list, from its rows of the map staged in
// s_nbr: pairs of offset d go to block_offsets[d][block] onwards, in row order.
__device__ __forceinline__ void emit_pairs_block(const int32_t* s_nbr, int64_t n, int64_t base,
                                                 const int64_t* __restrict__ block_offsets, int nblocks,
                                                 int32_t* __restrict__ in_idx, int32_t* __restrict__ out_idx) {
  __shared__ int32_t s_pre[kMapBlock / 32][kTaps];
  __shared__ int64_t s_off[kTaps];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t rows = n - base < kMapBlock ? n - base : kMapBlock;
  if (tid < kTaps) s_off[tid] = block_offsets[static_cast<int64_t>(tid) * nblocks + blockIdx.x];
  __syncthreads();
  const int64_t v = base + tid;
  const bool live = tid < rows;
#pragma unroll
  for (int d = 0; d < kTaps; ++d) {
    const bool hit = live && s_nbr[tid * kTaps + d] >= 0;
    const uint32_t b = __ballot_sync(0xffffffffu, hit);
    if (lane == 0) s_pre[warp][d] = __popc(b);
  }
  __syncthreads();
  if (tid < kTaps) {
    int32_t run = 0;
#pragma unroll
    for (int w = 0; w < kMapBlock / 32; ++w) {
      const int32_t t = s_pre[w][tid];
      s_pre[w][tid] = run;
      run += t;
    }
  }
  __syncthreads();
  const uint32_t lt = (1u << lane) - 1u;
#pragma unroll 1
  for (int d = 0; d < kTaps; ++d) {
    const int32_t u = live ? s_nbr[tid * kTaps + d] : -1;
    const uint32_t b = __ballot_sync(0xffffffffu, u >= 0);
    if (u >= 0) {
      const int64_t pos = s_off[d] + s_pre[warp][d] + __popc(b & lt);
      if (pos < kTaps * n) {  // always, unless the scan gave up on a wait (error bit set)
        in_idx[pos] = u;
        out_idx[pos] = static_cast<int32_t>(v);
      }
    }
  }
}

// Pair lists from the map the neighbour kernel wrote (read back, 108 bytes a row).
__global__ void __launch_bounds__(kMapBlock) k_pairs(const int32_t* __restrict__ nbr, int64_t n,
                                                     const int64_t* __restrict__ block_offsets,
                                                     int nblocks, int32_t* __restrict__ in_idx,
                                                     int32_t* __restrict__ out_idx) {
  __shared__ int32_t s_nbr[kMapBlock * kTaps];
  const int tid = threadIdx.x;
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kMapBlock;
  const int64_t rows = n - base < kMapBlock ? n - base : kMapBlock;
  const int total = static_cast<int>(rows) * kTaps;
  const int32_t* src = nbr + base * kTaps;
  const int vec = total >> 2;
  for (int i = tid; i < vec; i += kMapBlock)
    reinterpret_cast<int4*>(s_nbr)[i] = reinterpret_cast<const int4*>(src)[i];
  for (int i = (vec << 2) + tid; i < total; i += kMapBlock) s_nbr[i] = src[i];
  emit_pairs_block(s_nbr, n, base, block_offsets, nblocks, in_idx, out_idx);
}

// Pair lists with the dense index grid: each row's 27 lookups are made again
// from its coordinates (16 bytes a row and lines of the grid, which
// neighbouring rows share) instead of reading its map row back (108 bytes).
// Rows outside the box have no neighbours, as in the map.
__global__ void __launch_bounds__(kMapBlock) k_pairs_dense(const int4* __restrict__ coords, int64_t n,
                                                           int32_t batch, int32_t Z, int32_t Y, int32_t X,
                                                           const int32_t* __restrict__ grid,
                                                           const int64_t* __restrict__ block_offsets, int nblocks,
                                                           int32_t* __restrict__ in_idx,
                                                           int32_t* __restrict__ out_idx) {
  __shared__ int32_t s_nbr[kMapBlock * kTaps];
  const int tid = threadIdx.x;
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kMapBlock;
  const int64_t v = base + tid;
  if (v < n) {
    const int4 c = coords[v];
    if (site_ok(c, batch, Z, Y, X)) {
      dense_row_lookups(grid, c, site_key(c, Z, Y, X), Z, Y, X, s_nbr + tid * kTaps);
    } else {
#pragma unroll
      for (int d = 0; d < kTaps; ++d) s_nbr[tid * kTaps + d] = -1;
    }
  }
  emit_pairs_block(s_nbr, n, base, block_offsets, nblocks, in_idx, out_idx);
}

// ------------------------------------------------------------------ scan
constexpr int kScanThreads = 512;
constexpr int kScanItems = 8;
constexpr int kScanSeg = kScanThreads * kScanItems;
constexpr unsigned long long kFlagAggregate = 1ull << 62;
constexpr unsigned long long kFlagPrefix = 2ull << 62;
constexpr unsigned long long kValueMask = (1ull << 62) - 1;

__device__ __forceinline__ unsigned long long ld_relaxed_gpu(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_relaxed_gpu(unsigned long long* p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ int64_t block_exclusive_scan(int64_t x, int64_t* s_warp, int64_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int64_t incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int64_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    int64_t w = lane < nw ? s_warp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < nw) s_warp[lane] = w;
  }
  __syncthreads();
  const int64_t before = warp > 0 ? s_warp[warp - 1] : 0;
  if (total) *total = s_warp[(blockDim.x >> 5) - 1];
  __syncthreads();
  return before + incl - x;
}

// Single-pass exclusive scan of int32 counts into int64 offsets (decoupled
// look-back).  A block takes the next segment in start order (a ticket),
// publishes the segment's total, then sums the totals of earlier segments,
// reading a window of blockDim predecessors per step and stopping at the
// nearest one that has published its inclusive prefix; last it publishes its
// own inclusive prefix.  Statuses are one word each: flag (aggregate /
// prefix) in bits 63..62, value below, so no fence orders them.  A block waits
// only on segments with smaller tickets, which are resident and running, so
// every wait ends; it is still bounded (wait_ns, 2 s unless a test sets it),
// after which the error word gets kErrTimeout and the offsets are not to be
// trusted.  The segment whose ticket is `hold` (a test hook; -1 = none)
// publishes nothing, so the waits of the segments after it run out.
//
// When `info` is given, the offsets at positions d * stride (d < 27) -- the
// starts of the per-offset pair lists -- and the grand total go to info[0..27].
__global__ void __launch_bounds__(kScanThreads) k_scan_lookback(const int32_t* __restrict__ in, int64_t L,
                                                                int64_t* __restrict__ out,
                                                                unsigned long long* status, uint32_t* ticket,
                                                                uint32_t* err, int64_t* __restrict__ info,
                                                                int64_t stride, uint64_t wait_ns, int64_t hold) {
  __shared__ int64_t s_warp[32];
  __shared__ int64_t s_t;
  __shared__ int s_first;
  __shared__ int s_abort;
  const int tid = threadIdx.x;
  if (tid == 0) {
    s_t = atomicAdd(ticket, 1u);
    s_first = kScanThreads;
    s_abort = 0;
  }
  __syncthreads();
  const int64_t t = s_t;
  const int64_t nseg = (L + kScanSeg - 1) / kScanSeg;
  const int64_t b0 = t * kScanSeg + static_cast<int64_t>(tid) * kScanItems;
  int32_t v[kScanItems];
  int64_t sum = 0;
#pragma unroll
  for (int i = 0; i < kScanItems; ++i) {
    v[i] = b0 + i < L ? in[b0 + i] : 0;
    sum += v[i];
  }
  int64_t tot;
  const int64_t mine = block_exclusive_scan(sum, s_warp, &tot);
  if (tid == 0 && t != hold)
    st_relaxed_gpu(&status[t], (t == 0 ? kFlagPrefix : kFlagAggregate) | static_cast<unsigned long long>(tot));
  int64_t excl = 0;
  if (t > 0) {
    int64_t top = t - 1;  // nearest predecessor not summed yet
    const uint64_t t_start = globaltimer_ns();
    for (;;) {
      const int64_t j = top - tid;
      const unsigned long long w = j >= 0 ? ld_relaxed_gpu(&status[j]) : kFlagPrefix;
      const unsigned long long flag = w & ~kValueMask;
      if (flag == kFlagPrefix) atomicMin(&s_first, tid);
      __syncthreads();
      const int first = s_first;  // window index of the nearest inclusive prefix, or kScanThreads
      if (!__syncthreads_and(tid > first || flag != 0)) {
        // a predecessor up to that prefix has not published yet: read again
        if (tid == 0) {
          s_first = kScanThreads;
          if (globaltimer_ns() - t_start > wait_ns) {
            atomicOr(err, kErrTimeout);
            s_abort = 1;
          }
        }
        __syncthreads();
        if (s_abort) break;
        continue;
      }
      int64_t part;
      block_exclusive_scan(tid <= first ? static_cast<int64_t>(w & kValueMask) : 0, s_warp, &part);
      excl += part;
      if (first < kScanThreads) break;
      top -= kScanThreads;
    }
    if (tid == 0 && t != hold) st_relaxed_gpu(&status[t], kFlagPrefix | static_cast<unsigned long long>(excl + tot));
  }
  int64_t run = excl + mine;
#pragma unroll
  for (int i = 0; i < kScanItems; ++i) {
    const int64_t j = b0 + i;
    if (j < L) {
      out[j] = run;
      if (info && j % stride == 0 && j / stride < kTaps) info[j / stride] = run;
    }
    run += v[i];
  }
  if (info && t == nseg - 1 && tid == 0) info[kTaps] = excl + tot;
}

// ------------------------------------------------------------ radix sort
// Stable scatter of one radix pass over a histogram already scanned into
// `offsets` (laid out by hist_index, cps chunks per segment).  Warp w of a block ranks elements
// 256w .. 256w + 255 of the block's chunk in 8 rounds of 32, keeping a
// warp-private count per digit in shared memory (no block barrier between
// rounds); the 8 warps' counts are then scanned per digit on top of the
// block's base offset.  An element's position is base[digit] + (its digit in
// earlier warps) + (in earlier rounds of its warp) + (in earlier lanes of its
// round), so the input order is kept.
// First pass (kLast false): writes keys and row indices and counts the next
// digit per destination chunk into hist_next.  Last pass: writes the row
// order and ORs each row's hit mask into the mask of its 128-row tile.
template <bool kLast, int kBins>
__global__ void __launch_bounds__(kRadixThreads) k_radix_scatter(
    const uint32_t* __restrict__ keys_in, const int32_t* __restrict__ vals_in, int64_t n, int shift,
    const int64_t* __restrict__ offsets, int cps, uint32_t* __restrict__ keys_out,
    int32_t* __restrict__ vals_out, int32_t* __restrict__ hist_next, uint32_t* __restrict__ tile_mask,
    uint32_t* err) {
  constexpr int kWarps = kRadixThreads / 32;
  __shared__ int32_t s_cnt[kWarps][kBins];  // counts, then positions (< n < 2^31)
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < kWarps * kBins; i += kRadixThreads) (&s_cnt[0][0])[i] = 0;
  const int64_t w0 = static_cast<int64_t>(blockIdx.x) * kRadixChunk + warp * (kRadixRounds * 32);
  const uint32_t lt = (1u << lane) - 1u;
  uint32_t keys[kRadixRounds];
  int32_t vals[kRadixRounds], rank[kRadixRounds];
#pragma unroll
  for (int round = 0; round < kRadixRounds; ++round) {
    const int64_t j = w0 + round * 32 + lane;
    keys[round] = j < n ? keys_in[j] : 0u;
    vals[round] = j < n ? (vals_in ? vals_in[j] : static_cast<int32_t>(j)) : 0;
  }
  __syncthreads();
  int32_t* my = s_cnt[warp];
#pragma unroll
  for (int round = 0; round < kRadixRounds; ++round) {
    const bool valid = w0 + round * 32 + lane < n;
    const uint32_t digit = (keys[round] >> shift) & (kBins - 1);
    const uint32_t peers = __match_any_sync(0xffffffffu, valid ? digit : 0xFFFFFFFFu);
    const int32_t before = valid ? my[digit] : 0;
    rank[round] = before + __popc(peers & lt);
    __syncwarp();
    if (valid && (__ffs(peers) - 1) == lane) my[digit] = before + __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  for (int d = tid; d < kBins; d += kRadixThreads) {
    int64_t run = offsets[hist_index(static_cast<uint32_t>(d), blockIdx.x, cps, kBins)];
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const int32_t c = s_cnt[w][d];
      s_cnt[w][d] = static_cast<int32_t>(run);
      run += c;
    }
  }
  __syncthreads();
#pragma unroll
  for (int round = 0; round < kRadixRounds; ++round) {
    const bool valid = w0 + round * 32 + lane < n;
    const uint32_t key = keys[round];
    const uint32_t digit = (key >> shift) & (kBins - 1);
    long long pos = -1;
    if (valid) {
      pos = static_cast<long long>(my[digit]) + rank[round];
      if (pos < 0 || pos >= n) {  // only after a scan gave up on a wait
        atomicOr(err, kErrTimeout);
        pos = -1;
      }
    }
    if (pos >= 0) {
      if (!kLast) keys_out[pos] = key;
      vals_out[pos] = vals[round];
    }
    if (!kLast) {
      // next digit, counted per destination chunk: one atomic per distinct (digit, chunk) of the warp
      const uint32_t tag = pos >= 0 ? ((((key >> (shift + kRadixBits)) & (kRadixBins - 1)) << 21) |
                                       static_cast<uint32_t>(pos / kRadixChunk))
                                    : 0xFFFFFFFFu;
      const uint32_t grp = __match_any_sync(0xffffffffu, tag);
      if (tag != 0xFFFFFFFFu && (__ffs(grp) - 1) == lane)
        atomicAdd(&hist_next[hist_index(tag >> 21, tag & ((1u << 21) - 1), cps, kRadixBins)], __popc(grp));
    } else {
      // tile tap masks: a warp whose rows all land in one tile (dense data)
      // ORs them first; otherwise every row ORs its own mask in
      const uint32_t tile = pos >= 0 ? static_cast<uint32_t>(pos / kTileRows) : 0xFFFFFFFFu;
      const uint32_t hm = pos >= 0 ? key_hits(key) : 0u;
      const uint32_t t0 = __reduce_min_sync(0xffffffffu, tile);
      if (__all_sync(0xffffffffu, tile == t0 || tile == 0xFFFFFFFFu)) {
        const uint32_t r = __reduce_or_sync(0xffffffffu, hm);
        if (lane == 0 && t0 != 0xFFFFFFFFu) atomicOr(&tile_mask[t0], r);
      } else if (pos >= 0) {
        atomicOr(&tile_mask[tile], hm);
      }
    }
  }
}

// ------------------------------------------------------------ launchers
static cudaError_t scan_i32(const int32_t* in, int64_t L, int64_t* out, unsigned long long* status,
                            uint32_t* ticket, uint32_t* err, int64_t* info, int64_t stride, cudaStream_t s) {
  const int64_t nseg = (L + kScanSeg - 1) / kScanSeg;
  if (nseg == 0) return cudaSuccess;
  k_scan_lookback<<<static_cast<unsigned>(nseg), kScanThreads, 0, s>>>(in, L, out, status, ticket, err, info,
                                                                       stride, scan_wait_limit_ns(),
                                                                       scan_hold_ticket());
  count_launches(1);
  return cudaGetLastError();
}

int64_t scan_status_len(int64_t L) { return (L + kScanSeg - 1) / kScanSeg; }
int map_nblocks(int64_t n) { return static_cast<int>((n + kMapBlock - 1) / kMapBlock); }
int radix_nblocks(int64_t n) { return static_cast<int>((n + kRadixChunk - 1) / kRadixChunk); }

// Schedule segment length in rows (0 = one segment, the default).  Segments
// keep the rows of each wave of conv tiles within a window of consecutive
// input rows, so a map whose input order is spatially coherent (C order,
// subdivision order) gathers from a feature working set that stays in L2.
// Measured on B200 with 131072-row segments: the conv's DRAM reads on the
// 512^3 decoder stage (64 channels, 1.26M voxels) fell from 897 to 304 MB
// with its time unchanged (0.49 ms: the gathers' L2 -> SM rate, not DRAM,
// bounds it), while the split key groups cost tap efficiency (0.950 -> 0.891
// on the four-item 256^3 set, a 3% longer conv).  So it is off by default.
static std::atomic<int64_t> g_segment_rows{kScheduleSegmentDefault};
void set_schedule_segment_rows(int64_t rows) { g_segment_rows.store(rows); }
int64_t schedule_segment_rows() { return g_segment_rows.load(); }
int radix_seg_chunks(int64_t n) {
  const int nblk = radix_nblocks(n);
  const int64_t rows = g_segment_rows.load();
  if (rows <= 0 || nblk == 0) return nblk > 0 ? nblk : 1;
  const int64_t cps = rows / kRadixChunk;
  return cps >= nblk ? nblk : static_cast<int>(cps);
}
int64_t radix_hist_len(int64_t n, int cps) {
  const int64_t nblk = radix_nblocks(n);
  const int64_t nseg = (nblk + cps - 1) / cps;
  return nseg * cps * schedule_bins(n);
}

cudaError_t launch_map_lookups(const MapBuildArgs& a, cudaStream_t s) {
  const int64_t n = a.n;
  if (n == 0) return cudaSuccess;
  const int nb = map_nblocks(n);
  const int grid_ins = static_cast<int>((n + 255) / 256);
  auto run = [&](auto kind) {
    constexpr int K = decltype(kind)::value;
    k_insert<K><<<grid_ins, 256, 0, s>>>(reinterpret_cast<const int4*>(a.coords), n, a.batch, a.Z, a.Y, a.X,
                                         a.table, a.lg, a.occ, a.err, a.zero, a.nzero);
    k_neighbours<K><<<nb, kMapBlock, 0, s>>>(reinterpret_cast<const int4*>(a.coords), n, a.batch, a.Z, a.Y, a.X,
                                             a.table, a.lg, a.occ, a.nbr, a.gkey, a.block_counts, nb, a.hist1,
                                             a.radix_cps);
  };
  if (a.kind == kMapDense) run(std::integral_constant<int, kMapDense>());
  else if (a.kind == kMapDenseOcc) run(std::integral_constant<int, kMapDenseOcc>());
  else if (a.kind == kMapWide) run(std::integral_constant<int, kMapWide>());
  else run(std::integral_constant<int, kMapPacked>());
  count_launches(2);
  return cudaGetLastError();
}

cudaError_t launch_pair_lists(const MapBuildArgs& a, cudaStream_t s) {
  const int64_t n = a.n;
  if (n == 0) return cudaSuccess;
  const int nb = map_nblocks(n);
  const int64_t L = static_cast<int64_t>(kTaps) * nb;
  cudaError_t e = scan_i32(a.block_counts, L, a.block_offsets, a.scan_status, a.scan_ticket, a.err, a.info, nb, s);
  if (e != cudaSuccess) return e;
  // With a dense grid small enough to stay in L2 the pair kernel makes the
  // lookups again instead of reading the map back (measured on B200: 18%
  // faster on the 128^3 full grid); a larger grid is read from DRAM and the
  // map read-back is faster (256^3 and 512^3 boxes).
  const bool l2_grid = static_cast<double>(a.batch) * a.Z * a.Y * a.X * 4.0 <= 32.0 * (1 << 20);
  if (a.kind == kMapDense && a.table && l2_grid)
    k_pairs_dense<<<nb, kMapBlock, 0, s>>>(reinterpret_cast<const int4*>(a.coords), n, a.batch, a.Z, a.Y, a.X,
                                           reinterpret_cast<const int32_t*>(a.table), a.block_offsets, nb,
                                           a.in_idx, a.out_idx);
  else
    k_pairs<<<nb, kMapBlock, 0, s>>>(a.nbr, n, a.block_offsets, nb, a.in_idx, a.out_idx);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_scan_counts(const int32_t* in, int64_t L, int64_t* out, unsigned long long* status,
                               uint32_t* ticket, uint32_t* err, int64_t* info, int64_t stride, cudaStream_t s) {
  return scan_i32(in, L, out, status, ticket, err, info, stride, s);
}

cudaError_t launch_subdiv_count(const uint8_t* keep, int64_t n, int order, uint8_t* bits, int32_t* cnt,
                                cudaStream_t s) {
  (void)order;  // the mask's bit k is child k in either numbering
  if (n == 0) return cudaSuccess;
  const int64_t blocks = (n + 255) / 256;
  k_subdiv_count<<<static_cast<unsigned>(blocks < 148 * 8 ? blocks : 148 * 8), 256, 0, s>>>(keep, n, bits, cnt);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_subdiv_emit(const int32_t* coords, int64_t n, int order, const uint8_t* bits,
                               const int64_t* first, int32_t* child_coords, int32_t* child_src, int32_t* remap,
                               cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  k_subdiv_emit<<<static_cast<unsigned>((n + kEmitBlock - 1) / kEmitBlock), kEmitBlock, 0, s>>>(
      reinterpret_cast<const int4*>(coords), n, order, bits, first, reinterpret_cast<int4*>(child_coords), child_src,
      remap);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_subdiv_lookups(const MapBuildArgs& a, const int32_t* parent_nbr, const int32_t* child_src,
                                  const int32_t* remap, cudaStream_t s) {
  const int64_t n = a.n;
  if (n == 0) return cudaSuccess;
  const int nb = map_nblocks(n);
  k_subdiv_neighbours<<<nb, kMapBlock, 0, s>>>(parent_nbr, child_src, remap, n, a.nbr, a.gkey, a.block_counts, nb,
                                               a.hist1, a.radix_cps);
  count_launches(1);
  return cudaGetLastError();
}

// Hash insert and the 27-lookup neighbour kernel alone (one-word slots), for
// the entry point that writes the map into caller memory with fixed scratch.
cudaError_t launch_neighbour_map_only(const int32_t* coords, int64_t n, int32_t batch, int32_t Z, int32_t Y,
                                      int32_t X, unsigned long long* table, int lg, uint32_t* err, int32_t* nbr,
                                      uint32_t* gkey, int32_t* block_counts, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  const int nb = map_nblocks(n);
  const int grid_ins = static_cast<int>((n + 255) / 256);
  k_insert<kMapPacked><<<grid_ins, 256, 0, s>>>(reinterpret_cast<const int4*>(coords), n, batch, Z, Y, X, table,
                                                lg, nullptr, err, nullptr, 0);
  k_neighbours<kMapPacked><<<nb, kMapBlock, 0, s>>>(reinterpret_cast<const int4*>(coords), n, batch, Z, Y, X, table, lg,
                                               nullptr, nbr, gkey, block_counts, nb, nullptr, 0);
  count_launches(2);
  return cudaGetLastError();
}

cudaError_t launch_schedule(const ScheduleArgs& a, cudaStream_t s) {
  const int64_t n = a.n;
  if (n == 0) return cudaSuccess;
  const int nblk = radix_nblocks(n);
  const int cps = a.radix_cps;
  const int64_t L = radix_hist_len(n, cps);
  if (schedule_one_pass(n)) {
    // small maps: one stable pass on the high 8 bits (the 8 corner offsets);
    // the histogram of that digit comes from the neighbour kernel
    cudaError_t e = scan_i32(a.hist1, L, a.hoff, a.status1, a.tickets, a.err, nullptr, 1, s);
    if (e != cudaSuccess) return e;
    k_radix_scatter<true, kOnePassBins><<<nblk, kRadixThreads, 0, s>>>(
        a.gkey, nullptr, n, 2 * kRadixBits - kOnePassBits, a.hoff, cps, nullptr, a.perm, nullptr, a.tile_mask, a.err);
    count_launches(1);
    return cudaGetLastError();
  }
  // pass 1: low 10 bits, rows in input order (histogram from the neighbour kernel)
  cudaError_t e = scan_i32(a.hist1, L, a.hoff, a.status1, a.tickets, a.err, nullptr, 1, s);
  if (e != cudaSuccess) return e;
  k_radix_scatter<false, kRadixBins><<<nblk, kRadixThreads, 0, s>>>(a.gkey, nullptr, n, 0, a.hoff, cps, a.key_tmp,
                                                        a.val_tmp, a.hist2, nullptr, a.err);
  count_launches(1);
  // pass 2: high 10 bits
  e = scan_i32(a.hist2, L, a.hoff, a.status2, a.tickets + 1, a.err, nullptr, 1, s);
  if (e != cudaSuccess) return e;
  k_radix_scatter<true, kRadixBins><<<nblk, kRadixThreads, 0, s>>>(a.key_tmp, a.val_tmp, n, kRadixBits, a.hoff, cps,
                                                       nullptr, a.perm, nullptr, a.tile_mask, a.err);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace smc
