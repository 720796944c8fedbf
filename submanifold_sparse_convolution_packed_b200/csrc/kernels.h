// Internal launch interface between the host library (api.cu) and the kernels.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace smc {

struct MapBuildArgs {
  const int32_t* coords;  // [n, 4] (b, z, y, x)
  int64_t n;
  int32_t batch, Z, Y, X;
  bool wide;                   // two-word hash slots (keys >= 2^32 - 1)
  unsigned long long* table;   // 2^lg slots, pre-filled with ~0
  int lg;
  uint32_t* err;               // error bits
  int32_t* nbr;                // [n, 27]
  uint32_t* gkey;              // [n] grouping key of the tile schedule
  uint32_t* hmask;             // [n] 27-bit neighbour hit mask of every row
  int32_t* block_counts;       // [27, nblocks]
  int64_t* block_offsets;      // [27, nblocks]
  int64_t* scan_partials;      // scan_partials_len(27 * nblocks)
  int64_t* info;               // [28]: offsets of the per-offset pair lists
  int32_t* in_idx;             // [27 n] capacity
  int32_t* out_idx;            // [27 n] capacity
};

struct ScheduleArgs {
  const uint32_t* gkey;   // [n]
  int64_t n;
  int32_t* hist;          // [bins, nblk]
  int64_t* hoff;          // [bins, nblk]
  int64_t* scan_partials; // scan_partials_len(bins * nblk)
  uint32_t* key_tmp;      // [n]
  int32_t* val_tmp;       // [n]
  int32_t* perm;          // [n] result: tile order
  const uint32_t* hmask;  // [n] hit masks
  uint32_t* tile_mask;    // [ceil(n/128)] result: OR of the hit masks of each tile's rows
};

constexpr int kTileRows = 128;  // output rows per tensor-core tile

// Running count of kernels this library has launched (measurement hook).
void count_launches(int k);

int map_nblocks(int64_t n);
int radix_nblocks(int64_t n);
int radix_bins();
int64_t scan_partials_len(int64_t L);

cudaError_t launch_map_build(const MapBuildArgs& a, cudaStream_t s);
cudaError_t launch_neighbour_map_only(const int32_t* coords, int64_t n, int32_t batch, int32_t Z, int32_t Y,
                                      int32_t X, unsigned long long* table, int lg, uint32_t* err, int32_t* nbr,
                                      uint32_t* gkey, uint32_t* hmask, int32_t* block_counts, cudaStream_t s);
cudaError_t launch_schedule(const ScheduleArgs& a, cudaStream_t s);

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
  int64_t n;
  int cin, cout, taps, orientation, dtype;
  uint32_t* err;
};

// cuTensorMapEncodeTiled, fetched from the driver through the runtime.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);
EncodeTiledFn encode_fn();

// FMA kernel: every dtype, every shape.
cudaError_t launch_conv_simt(const ConvArgs& a, cudaStream_t s);
// tcgen05 kernel: bf16/fp16, cin % 16 == 0 and cin >= 64, cout % 16 == 0, 16-byte aligned.
bool conv_tc_supported(const ConvArgs& a);
cudaError_t launch_conv_tc(const ConvArgs& a, cudaStream_t s);


}  // namespace smc
