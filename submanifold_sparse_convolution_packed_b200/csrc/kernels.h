// Internal launch interface between the host library (api.cu) and the kernels.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "epilogue.cuh"

namespace smc {

// Lookup structure of a map build (see map_build.cu).
// kMapDenseOcc: the dense grid is not cleared; an occupancy bitmap (one bit
// per site, cleared) says which of its entries this build wrote.
enum MapKind : int { kMapPacked = 0, kMapWide = 1, kMapDense = 2, kMapDenseOcc = 3 };

struct MapBuildArgs {
  const int32_t* coords;  // [n, 4] (b, z, y, x)
  int64_t n;
  int32_t batch, Z, Y, X;
  int kind;                    // MapKind
  unsigned long long* table;   // hash: 2^lg slots pre-filled with ~0; dense: int32 grid pre-filled with -1
                               // (kMapDenseOcc: int32 grid, not cleared)
  uint32_t* occ;               // kMapDenseOcc: occupancy bitmap, one bit per site, zeroed
  int lg;
  uint32_t* err;               // error bits (zeroed)
  uint32_t* zero;              // [nzero] words k_insert clears (the tile tap masks)
  int64_t nzero;
  int32_t* nbr;                // [n, 27]
  uint32_t* gkey;              // [n] schedule key of every row (carries the 27-bit hit mask)
  int32_t* block_counts;       // [27, nblocks]
  int64_t* block_offsets;      // [27, nblocks]
  unsigned long long* scan_status;  // [scan_status_len(27 * nblocks)], zeroed
  uint32_t* scan_ticket;       // zeroed
  int32_t* hist1;              // [radix_hist_len], zeroed: first schedule digit per chunk
  int radix_cps;               // radix chunks per schedule segment (radix_seg_chunks)
  int64_t* info;               // [28]: offsets of the per-offset pair lists
  int32_t* in_idx;             // [27 n] capacity
  int32_t* out_idx;            // [27 n] capacity
};

struct ScheduleArgs {
  const uint32_t* gkey;   // [n]
  int64_t n;
  int radix_cps;          // radix chunks per schedule segment (radix_seg_chunks)
  int32_t* hist1;         // [radix_hist_len] filled by the neighbour kernel
  int32_t* hist2;         // [radix_hist_len] zeroed
  int64_t* hoff;          // [radix_hist_len]
  unsigned long long* status1;  // [scan_status_len(radix_hist_len)] each, zeroed
  unsigned long long* status2;
  uint32_t* tickets;      // [2], zeroed
  uint32_t* key_tmp;      // [n]
  int32_t* val_tmp;       // [n]
  int32_t* perm;          // [n] result: tile order
  uint32_t* tile_mask;    // [ceil(n/128)] result, zeroed: OR of the hit masks of each tile's rows
  uint32_t* err;          // error bits
};

constexpr int kTileRows = 128;  // output rows per tensor-core tile

// Running count of kernels this library has launched (measurement hook).
void count_launches(int k);

int map_nblocks(int64_t n);
int radix_nblocks(int64_t n);
// The tile schedule sorts rows within segments of consecutive input rows
// (0 = the whole map is one segment).  radix_seg_chunks: 2048-row radix
// chunks per segment for a map of n rows (the segment length in force now);
// radix_hist_len: histogram length for that many chunks per segment.
constexpr int64_t kScheduleSegmentDefault = 0;
void set_schedule_segment_rows(int64_t rows);
int64_t schedule_segment_rows();
int radix_seg_chunks(int64_t n);
int64_t radix_hist_len(int64_t n, int cps);
int64_t scan_status_len(int64_t L);
// Bound of every device-side wait -- the look-back scans' waits on their
// predecessors and the convs' mbarrier waits -- (2 s unless a test sets it),
// and the test hook that holds one scan segment back (-1 = none).
uint64_t scan_wait_limit_ns();
int64_t scan_hold_ticket();

// Hash insert + neighbour lookups (map, schedule keys, block counts, first
// radix histogram), then, on any stream ordered after them, the pair lists.
cudaError_t launch_map_lookups(const MapBuildArgs& a, cudaStream_t s);
cudaError_t launch_pair_lists(const MapBuildArgs& a, cudaStream_t s);
cudaError_t launch_neighbour_map_only(const int32_t* coords, int64_t n, int32_t batch, int32_t Z, int32_t Y,
                                      int32_t X, unsigned long long* table, int lg, uint32_t* err, int32_t* nbr,
                                      uint32_t* gkey, int32_t* block_counts, cudaStream_t s);
cudaError_t launch_schedule(const ScheduleArgs& a, cudaStream_t s);
// Single-pass exclusive scan of int32 counts (k_scan_lookback); status and
// ticket zeroed, status of scan_status_len(L) words.
cudaError_t launch_scan_counts(const int32_t* in, int64_t L, int64_t* out, unsigned long long* status,
                               uint32_t* ticket, uint32_t* err, int64_t* info, int64_t stride, cudaStream_t s);
// Subdivision: children per parent (bit mask and count), the children's
// coordinates with their (parent, octant) and the parent-slot -> child-row
// remap, then the children's map rows from the parent map.
// `order` numbers the children and lists them: 0 = C-order octant
// o = 4a + 2c + e (subdivide), 1 = the upsample mask's index
// j = a + 2c + 4e (z offset fastest).  child_src always holds 8 * parent + o.
cudaError_t launch_subdiv_count(const uint8_t* keep, int64_t n, int order, uint8_t* bits, int32_t* cnt,
                                cudaStream_t s);
cudaError_t launch_subdiv_emit(const int32_t* coords, int64_t n, int order, const uint8_t* bits,
                               const int64_t* first, int32_t* child_coords, int32_t* child_src, int32_t* remap,
                               cudaStream_t s);
cudaError_t launch_subdiv_lookups(const MapBuildArgs& a, const int32_t* parent_nbr, const int32_t* child_src,
                                  const int32_t* remap, cudaStream_t s);

// Downsample by 2 (resample.cu): parents numbered in order of first
// appearance, their coordinates, subdivision mask, each row's parent, and the
// pooled features.
struct DownArgs {
  const int32_t* coords;  // [n, 4] (b, z, y, x)
  int64_t n;
  int32_t batch, Z, Y, X;
  unsigned long long* keys;  // hash: 2^lg parent keys pre-filled with ~0; null: dense parent grid
  int lg;
  int32_t* first;          // per slot, pre-filled with 0x7F7F7F7F: smallest row of the parent
  uint32_t* bits;          // per slot, zeroed: children present (bit j)
  uint32_t* slot_of_row;   // [n]
  int32_t* flags;          // [n]
  int64_t* pos;            // [n]
  unsigned long long* scan_status;  // [scan_status_len(n)], zeroed
  uint32_t* scan_ticket;   // zeroed
  uint32_t* err;           // error bits, zeroed
  int64_t* info;           // [28]: info[27] receives the parent count M
  int32_t* child_rows;     // [8 n]: row of child j of parent p at 8 p + j (where present)
  uint8_t* pbits;          // [n]: children present per parent
  int32_t* parent_coords;  // [n, 4] capacity
  uint8_t* mask;           // [n, 8] capacity, 8-byte aligned
  int32_t* parent;         // [n] or null
  const void* feats;       // [n, c] or null (no pooling)
  void* out;               // [n, c] capacity
  int c, dtype, mode;      // mode 0 max, 1 mean
};
cudaError_t launch_downsample(const DownArgs& a, cudaStream_t s);
// Row p of `rows` (row_bytes bytes of elem_bytes-byte elements) copied to
// output rows first[p] .. first[p] + popc(bits[p]) - 1, for p < n.
cudaError_t launch_expand_rows(const void* rows, int64_t row_bytes, const int64_t* first, const uint8_t* bits,
                               int64_t n, void* out, int elem_bytes, cudaStream_t s);

// GroupNorm over a sparse tensor (norm.cu): statistics of x per (batch item,
// channel group) added into stats [batch, groups, 3], and the normalisation
// y = act(gamma * (x - mean) / sqrt(var + eps) + beta) from such statistics.
cudaError_t launch_group_stats(const void* x, int64_t n, int c, const int32_t* coords, const Epilogue& ep, int dtype,
                               cudaStream_t s);
// y = act(x) + residual (residual may be null; y may be x, and so may the
// residual), in row order, with the statistics of y when ep.stats is set.
cudaError_t launch_rows_pass(const void* x, void* y, const void* residual, int act, int64_t n, int c,
                             const int32_t* coords, const Epilogue& ep, int dtype, cudaStream_t s);
// Where the tensor-core conv applies activation and residual: 0 = a row pass
// behind it (default), 1 = its own epilogue.
void set_conv_epilogue(int where);
int conv_epilogue();
// stats[i] += sum over s < stripes of copies[s * len + i]
cudaError_t launch_stats_fold(const double* copies, int stripes, int64_t len, double* stats, cudaStream_t s);
cudaError_t launch_group_norm(const void* x, int64_t n, int c, const int32_t* coords, int batch, int groups,
                              const double* stats, const void* gamma, const void* beta, float eps, int act,
                              void* out, int dtype, cudaStream_t s);

// dtype codes as in smc.h
enum DType : int { kF32 = 0, kBF16 = 1, kF16 = 2 };

struct ConvArgs {
  const void* feats;    // [n, cin]
  const void* weight;   // [cout, taps, cin]
  const void* bias;     // [cout] or null
  void* out;            // [n, cout]
  const int32_t* nbr;   // [n, 27] (taps == 27)
  const int32_t* perm;  // [n] tile order (tensor-core kernel, taps == 27) or null
  const uint32_t* tile_mask;  // [ceil(n/128)] taps present in each tile (taps == 27)
  const int32_t* in_idx;      // pair lists (per-offset kernel)
  const int32_t* out_idx;
  const int64_t* pair_offsets;  // [28] device copy of the list offsets
  int64_t n;
  int cin, cout, taps, orientation, dtype;
  uint32_t* err;
  Epilogue ep;                // activation, residual, group statistics
};

// cuTensorMapEncodeTiled, fetched from the driver through the runtime.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);
EncodeTiledFn encode_fn();

// FMA kernel: every dtype, every shape.
cudaError_t launch_conv_simt(const ConvArgs& a, cudaStream_t s);
// tcgen05 kernel: bf16/fp16, cin % 16 == 0 and cin >= 64, cout % 16 == 0, 16-byte aligned
// (feats, weight, out and residual).
bool conv_tc_supported(const ConvArgs& a);
cudaError_t launch_conv_tc(const ConvArgs& a, cudaStream_t s);
// Conv kernel variant: 0 = default, 1 = one CTA per tile, 2 = CTA pairs,
// 3 = per-offset gather-GEMM-scatter.
void set_conv_variant(int v);
int conv_variant();
// Per-offset gather-GEMM-scatter over the map's pair lists (bf16/fp16 on the
// tensor-core shapes, k = 3); acc is [n, cout] fp32 scratch.
cudaError_t launch_conv_offsets(const ConvArgs& a, float* acc, cudaStream_t s);


}  // namespace smc
