/*
 * smc.h -- C ABI of the B200 submanifold sparse convolution library (libsmc.so).
 *
 * The operation (LATO.2 MLX port README, summary and "The scope, once
 * measured"; Pixal3D working notes, "Measured facts"): a submanifold 3x3x3
 * convolution, stride 1, no padding (spconv's SubMConv3d).  Outputs exist only
 * at the input's active voxels:
 *
 *     out[v] = bias + sum_{d=0}^{26} feats[nbr(v, d)] @ W[:, d, :]^T
 *
 * where nbr(v, d) is the active voxel at coordinate c_v + s*delta_d (missing
 * or out-of-grid neighbours contribute nothing), delta_d = (kz-1, ky-1, kx-1)
 * with d = 9*kz + 3*ky + kx, and W is in spconv's KRSC layout
 * [Cout, kz, ky, kx, Cin] (LATO.2 README summary; Pixal3D commit log,
 * converter paragraph).  The neighbour lookup is an "indice map" built once
 * per coordinate set and reused by every conv on it, the way spconv's
 * indice_key caches it (LATO.2 README summary).  s is the kernel orientation:
 * +1 gathers feats[c+d] (cross-correlation), -1 gathers feats[c-d]; the
 * README's "Correctness" section flags this choice as silent when wrong, so
 * both are offered.  k = 1 is the centre tap alone, a per-voxel linear layer
 * (LATO.2 README, "Status").
 *
 * Conventions for every entry point
 *  - Pointers marked "device" are CUDA device pointers on the current device;
 *    "host" pointers are ordinary host memory.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *  - Return value: SMC_OK (0) or a negative SMC_E_* code.  Nothing traps,
 *    aborts or hangs: device-side problems are recorded in an error word and
 *    surface as a return code.  A CUDA error from an earlier asynchronous
 *    launch surfaces at the next call as SMC_E_CUDA.
 *  - The caller owns every buffer it passes in; the library owns the map.
 */
#ifndef SMC_H_
#define SMC_H_

#include <stdint.h>

#if defined(__GNUC__)
#define SMC_API __attribute__((visibility("default")))
#else
#define SMC_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Opaque neighbour-map handle: library-owned, immutable after build. */
typedef struct smc_map smc_map;

/* Storage type of feats, weight, bias and out in smc_conv. */
typedef enum { SMC_F32 = 0, SMC_BF16 = 1, SMC_F16 = 2 } smc_dtype;

/* Activations of the conv epilogue (smc_conv_ex) and of smc_group_norm. */
typedef enum { SMC_ACT_NONE = 0, SMC_ACT_RELU = 1, SMC_ACT_SILU = 2 } smc_act;

/* Pooling of smc_downsample: elementwise max, or mean over the children present. */
typedef enum { SMC_POOL_MAX = 0, SMC_POOL_MEAN = 1 } smc_pool;

enum {
  SMC_OK = 0,
  SMC_E_ARG = -1,       /* null pointer, negative size, bad ksize/orientation/dtype value */
  SMC_E_RANGE = -2,     /* a coordinate outside [0,batch) x [0,Z) x [0,Y) x [0,X) */
  SMC_E_DUPLICATE = -3, /* the same (b,z,y,x) appears twice */
  SMC_E_DTYPE = -4,     /* unsupported dtype for this call */
  SMC_E_SHAPE = -5,     /* channel count or N does not match the map / limits */
  SMC_E_ALIAS = -6,     /* out overlaps feats, weight or bias */
  SMC_E_CAPACITY = -7,  /* hash table full after a bounded probe sequence */
  SMC_E_OOM = -8,       /* device allocation failed */
  SMC_E_CUDA = -9,      /* a CUDA runtime error (launch, copy, earlier async fault) */
  SMC_E_TIMEOUT = -10,  /* a bounded device-side wait ran out; results are invalid */
  SMC_E_ALIGN = -11     /* a device pointer lacks the alignment stated below */
};

/*
 * smc_build_map -- build the neighbour map of one coordinate set: the pages'
 * indice map, 27 lookups per voxel, built once per coordinate set and cached
 * the way spconv's indice_key caches it (LATO.2 MLX port README, summary;
 * the map table of its "The scope, once measured").
 *
 * coords : device, int32 [n, 4], rows (b, z, y, x), contiguous, 16-byte aligned.
 *          Row order is arbitrary; row v of the map corresponds to row v here.
 * n      : number of active voxels (n >= 0; n == 0 gives an empty map).
 * batch  : number of batch items; every b must lie in [0, batch).
 * grid   : host, int32 [3] = (Z, Y, X); every coordinate must lie inside.
 *          batch * Z * Y * X must be below 2^62.
 * stream : work is enqueued on it; the call synchronises it once, at the end,
 *          to read the per-offset counts and the error word.
 * out    : receives the handle; left NULL on failure.
 *
 * Builds, on the device: 64-bit site keys, a lookup structure of the sites
 * (a dense int32 index grid over the batch x Z x Y x X box when the box has
 * at most 2^28 sites and at most 256 sites per voxel, with an occupancy
 * bitmap instead of a clear above 2^23 sites or 16 sites per voxel, else an
 * open-addressing hash
 * table; smc_set_map_lookup forces any of them), the int32
 * [n, 27] neighbour map (-1 = absent), the per-offset pair lists (stable
 * compaction of each map column, ascending output row), and the tile
 * schedule used by the tensor-core conv.  coords may be freed
 * once the call returns.  Device memory comes from a per-device
 * stream-ordered pool owned by the library that keeps freed memory for
 * later builds.  Errors: SMC_E_ARG, SMC_E_ALIGN, SMC_E_RANGE,
 * SMC_E_DUPLICATE, SMC_E_CAPACITY, SMC_E_OOM, SMC_E_CUDA, and SMC_E_TIMEOUT
 * if a bounded wait of the single-pass scans ran out (not expected: a scan
 * block waits only on blocks that started before it).
 */
SMC_API int smc_build_map(const int32_t* coords, int64_t n, int32_t batch, const int32_t grid[3],
                  void* stream, smc_map** out);

/*
 * smc_build_map_async -- the same build with no synchronisation: the work is
 * enqueued and the handle returns at once.  Work enqueued on `stream` after
 * the call is ordered after the neighbour map and the tile schedule.  The
 * pair lists are built on a library-owned stream, concurrently with the tile
 * schedule, and are complete once smc_map_wait, smc_map_info or smc_map_pairs
 * has returned.  Argument errors
 * are returned immediately; errors found on the device (SMC_E_RANGE,
 * SMC_E_DUPLICATE, SMC_E_CAPACITY, SMC_E_TIMEOUT) are returned by smc_map_wait and by every
 * later smc_map_* query, and smc_conv refuses a map known to have failed.
 * A conv enqueued before the outcome is known reads a map whose entries are
 * always -1 or valid rows, so it stays memory-safe.  coords must stay valid
 * until the build has run on `stream`.
 */
SMC_API int smc_build_map_async(const int32_t* coords, int64_t n, int32_t batch, const int32_t grid[3],
                        void* stream, smc_map** out);

/* Block until the map's build has finished; return its outcome. */
SMC_API int smc_map_wait(const smc_map* map);

/*
 * smc_subdivide -- the map of a parent map's children, built from the parent
 * map without any lookup structure (the decoders' x2 upsampling step: every
 * voxel splits into its 8 children in C order; LATO.2 MLX port README, "The
 * scope, once measured" table, and the shared sparse-core commit log).
 *
 * parent        : a built map; the call waits for its build and returns its
 *                 error if it failed.
 * parent_coords : device int32 [n, 4], the coordinates the parent was built
 *                 from (same rows), 16-byte aligned.
 * keep          : device uint8 [n * 8] or NULL (keep all): keep[8v + o] != 0
 *                 keeps child o = 4a + 2c + e of parent v, the site
 *                 (b, 2z + a, 2y + c, 2x + e).
 * child_coords  : device int32 [8n, 4] capacity, 16-byte aligned; receives
 *                 the m kept children in (parent row, octant) order.
 * m             : host, receives m.
 * child         : receives the children's map on the grid (2Z, 2Y, 2X), the
 *                 same batch; as a smc_build_map_async result (pair lists on
 *                 the side stream, errors at smc_map_wait).
 * One host synchronisation of `stream` (to read m).  A child's neighbour at
 * offset D is the kept child, in octant (o + D) mod 2, of the parent's
 * neighbour at offset floor((o + D) / 2).  Errors: SMC_E_ARG, SMC_E_ALIGN,
 * SMC_E_OOM, SMC_E_CUDA, SMC_E_TIMEOUT, or the parent's build error.
 */
SMC_API int smc_subdivide(const smc_map* parent, const int32_t* parent_coords, const uint8_t* keep,
                  int32_t* child_coords, int64_t* m, void* stream, smc_map** child);

/*
 * smc_downsample -- pooling by 2 into parent voxels (SparseDownsample(2);
 * shared sparse-core commit log: modes 'max' and 'mean', which differ between
 * the models; Pixal3D MLX README "Status").
 *
 * Row i at (b, z, y, x) pools into the parent (b, z/2, y/2, x/2) (integer
 * halves; odd extents give a partial last window).  Parents are numbered in
 * order of first appearance among the rows (the row order, not a sort).
 *
 * coords        : device int32 [n, 4], 16-byte aligned, inside
 *                 [0, batch) x [0, grid[0]) x [0, grid[1]) x [0, grid[2]).
 * grid          : host int32[3] (Z, Y, X) of the input.
 * feats         : device [n, c] row-major, dtype `dtype`, or NULL (structure
 *                 only; parent_feats must then be NULL too).
 * mode          : SMC_POOL_MAX or SMC_POOL_MEAN (sum in fp32 over the children
 *                 in index order, divided by their count, rounded to nearest
 *                 even in the output type).
 * parent_coords : device int32 [n, 4] capacity, 16-byte aligned; receives the
 *                 m parents' (b, z, y, x) on the grid ((Z+1)/2, (Y+1)/2, (X+1)/2).
 * parent_feats  : device [n, c] capacity, dtype `dtype`; must not overlap feats.
 * mask          : device uint8 [n, 8] capacity, 8-byte aligned; receives the
 *                 subdivision mask: mask[8p + j] = 1 if parent p has the child
 *                 at index j = dz + 2 dy + 4 dx (z offset fastest), else 0.
 *                 It is what smc_upsample takes to restore the children.
 * parent        : device int32 [n] or NULL; receives each row's parent number.
 * m             : host, receives the number of parents m (1 <= m <= n).
 * Synchronises `stream` once, at the end, to read m and the error word; all
 * outputs are complete on return.  Errors: SMC_E_ARG (also n >= 2^30),
 * SMC_E_ALIGN, SMC_E_DTYPE, SMC_E_SHAPE (c < 1 or above 2^24), SMC_E_ALIAS,
 * SMC_E_RANGE, SMC_E_DUPLICATE, SMC_E_OOM, SMC_E_CUDA, SMC_E_TIMEOUT; after an
 * error the outputs are undefined (but every access stayed in bounds).
 */
SMC_API int smc_downsample(const int32_t* coords, int64_t n, int32_t batch, const int32_t grid[3],
                   const void* feats, int64_t c, int32_t dtype, int32_t mode, int32_t* parent_coords,
                   void* parent_feats, uint8_t* mask, int32_t* parent, int64_t* m, void* stream);

/*
 * smc_upsample -- masked expansion by 2 (SparseUpsample(2); shared sparse-core
 * commit log: a voxel emits 0 to 8 children chosen by a 0/1 subdivision mask
 * whose child index runs with the z offset fastest, the reverse of
 * smc_subdivide's C order; Pixal3D MLX README, remaining ops).
 *
 * coords      : device int32 [n, 4], 16-byte aligned (the coarse voxels).
 * mask        : device uint8 [n * 8], or NULL (every child): mask[8p + j] != 0
 *               emits child j of parent p, the site
 *               (b, 2z + j % 2, 2y + (j / 2) % 2, 2x + j / 4).
 * feats       : device [n, c], dtype `dtype`, or NULL (coordinates only).
 * map         : NULL, or the map built from `coords` (same n): then `child`
 *               receives the children's map on the grid (2Z, 2Y, 2X), read off
 *               this map without a lookup structure, as smc_subdivide does.
 * child_coords: device int32 [8n, 4] capacity, 16-byte aligned; receives the
 *               m children parent by parent, j ascending.
 * child_feats : device [8n, c] capacity, dtype `dtype` (with feats); child r
 *               receives its parent's row (nearest upsampling).  Must not
 *               overlap feats.
 * m           : host, receives m.
 * child       : receives the child map (when map is given; may be NULL
 *               otherwise), as a smc_build_map_async result.
 * One host synchronisation of `stream` (to read m).  Without a map the
 * children's coordinates are computed in int32 and not range-checked.
 * Errors: SMC_E_ARG, SMC_E_ALIGN, SMC_E_DTYPE, SMC_E_SHAPE, SMC_E_ALIAS,
 * SMC_E_OOM, SMC_E_CUDA, SMC_E_TIMEOUT, or the map's build error.
 */
SMC_API int smc_upsample(const int32_t* coords, int64_t n, const uint8_t* mask, const void* feats, int64_t c,
                 int32_t dtype, const smc_map* map, int32_t* child_coords, void* child_feats, int64_t* m,
                 void* stream, smc_map** child);

/* Make `stream` wait (on the device, without blocking the host) until the
 * whole build has finished, pair lists included: work enqueued on `stream`
 * afterwards may read every part of the map. */
SMC_API int smc_map_stream_wait(const smc_map* map, void* stream);

/*
 * smc_conv -- one submanifold convolution over a built map:
 * out[v] = bias + sum_d feats[nbr(v, d)] @ W[:, d, :]^T with KRSC weights
 * (LATO.2 MLX port README, summary and "The scope, once measured"; the
 * orientation choice per its "Correctness" section).
 *
 * feats  : device, [n, cin] row-major, dtype `dtype`.
 * weight : device, KRSC [cout, k, k, k, cin] row-major, dtype `dtype`.
 * bias   : device, [cout], dtype `dtype`, or NULL for no bias.
 * out    : device, [n, cout] row-major, dtype `dtype`; fully overwritten.
 *          Must not overlap feats, weight or bias.
 * ksize  : 3 (27 taps through the map) or 1 (centre tap only; the map is used
 *          only for n).
 * orientation : +1 gathers feats[c+d], -1 gathers feats[c-d]; ignored for k=1.
 * dtype  : SMC_F32 (exact fp32 FMA accumulation, no TF32), SMC_BF16 or
 *          SMC_F16 (fp32 accumulation, bias added in fp32, output rounded to
 *          nearest even).
 *
 * Asynchronous on `stream`; no synchronisation.  When `stream` is not the
 * stream the map was built on, the conv first waits (on the device) for the
 * build to finish.  bf16/fp16 with cin a
 * multiple of 16 and at least 64, cout a multiple of 16 and 16-byte aligned
 * buffers run on the tcgen05 tensor-core kernel; every other shape runs on
 * the FMA kernel.  A bounded device-side wait that runs out is reported by
 * smc_status as SMC_E_TIMEOUT.
 * Errors: SMC_E_ARG, SMC_E_SHAPE (cin, cout < 1), SMC_E_ALIAS, SMC_E_DTYPE,
 * SMC_E_CUDA.
 */
SMC_API int smc_conv(const smc_map* map, const void* feats, int64_t cin, const void* weight,
             const void* bias, void* out, int64_t cout, int32_t ksize, int32_t orientation,
             int32_t dtype, void* stream);

/*
 * smc_conv_ex -- smc_conv with the epilogue of the layers around the
 * decoders' convs (norms, activations and ResBlocks: Pixal3D MLX README
 * "Status"; SparseGroupNorm32 and activations: LATO.2 MLX port README
 * "Status"):
 *
 *   out = round(act(bias + conv(feats)) + residual)
 *
 * On the tensor-core kernel the activation, the residual and the statistics
 * are applied by one row pass enqueued right behind the conv, which sees the
 * conv's stored (rounded) output (smc_set_conv_epilogue selects the conv's
 * own epilogue instead; a residual that is `out` itself always uses it); the
 * FMA kernel applies them in its epilogue and the per-offset variant in its
 * final pass.
 *
 * residual : device [n, cout] in the output type, or NULL; it may be `out`
 *            itself (y = conv + out) but must not otherwise overlap it.
 * act      : SMC_ACT_NONE, SMC_ACT_RELU (max(y, 0)) or SMC_ACT_SILU
 *            (y / (1 + exp(-y)), in fp32 with the fast exponential),
 *            applied before the residual.
 * stats    : device fp64 [batch, groups, 3] or NULL: for every batch item b
 *            and channel group g (cout / groups channels each), the sum, the
 *            sum of squares and the number of the stored output values of
 *            the item's rows are ADDED (the caller zeroes it) -- what a
 *            following smc_group_norm normalises with.  Computed in the
 *            row pass, or by the smc_group_stats pass over `out` enqueued
 *            right behind the conv.
 * coords   : device int32 [n, 4], the map's coordinates (the batch index of
 *            each row); needed with stats.
 * groups   : >= 1 and dividing cout; used with stats.
 * Other arguments and errors as smc_conv.  smc_conv(...) is
 * smc_conv_ex(..., residual NULL, act NONE, coords NULL, stats NULL, 1, ...).
 */
SMC_API int smc_conv_ex(const smc_map* map, const void* feats, int64_t cin, const void* weight,
                const void* bias, const void* residual, void* out, int64_t cout, int32_t ksize,
                int32_t orientation, int32_t dtype, int32_t act, const int32_t* coords, double* stats,
                int32_t groups, void* stream);

/*
 * smc_group_stats -- add to stats (device fp64 [batch, groups, 3], zeroed by
 * the caller) the sum, sum of squares and count of x (device [n, c], dtype)
 * over each batch item's rows and each group of c / groups channels; the
 * batch index of row v is coords[4v] (rows outside [0, batch) are skipped).
 * batch * groups <= 1024.  Asynchronous on `stream`.
 * Errors: SMC_E_ARG, SMC_E_DTYPE, SMC_E_SHAPE, SMC_E_CUDA.
 */
SMC_API int smc_group_stats(const void* x, int64_t n, int64_t c, const int32_t* coords, int32_t batch,
                    int32_t groups, double* stats, int32_t dtype, void* stream);

/*
 * smc_group_norm -- GroupNorm over a sparse tensor and an activation:
 *   out = round(act(gamma * (x - mean) / sqrt(var + eps) + beta))
 * with mean and biased variance of the row's (batch item, channel group) from
 * stats (as filled by smc_group_stats or smc_conv_ex).  gamma, beta: device
 * [c] in dtype, or NULL (1 and 0).  out may equal x.  batch * groups <= 1024.
 * Asynchronous on `stream`.  Errors: SMC_E_ARG, SMC_E_DTYPE, SMC_E_SHAPE,
 * SMC_E_CUDA.
 */
SMC_API int smc_group_norm(const void* x, int64_t n, int64_t c, const int32_t* coords, int32_t batch,
                   int32_t groups, const double* stats, const void* gamma, const void* beta, float eps,
                   int32_t act, void* out, int32_t dtype, void* stream);

/* n and the per-offset pair counts counts[27] (host) of a map: the hit
 * counts of the indice map's 27 offsets (LATO.2 MLX port README, "Correctness":
 * indice-map hit rates). */
SMC_API int smc_map_info(const smc_map* map, int64_t* n, int64_t counts[27]);

/* Device pointer to the int32 [n, 27] neighbour map (-1 = absent): the
 * indice map of the LATO.2 MLX port README summary. */
SMC_API int smc_map_nbr(const smc_map* map, const int32_t** nbr);

/*
 * Per-offset pair lists, the operands of the per-offset gather-GEMM-scatter
 * the pages compare their fused kernel with (shared sparse-core commit log,
 * the 13.8 ms / 5.9x test commit): device pointers in_idx[P], out_idx[P] (int32) and
 * host offsets[28] (int64, offsets[0] = 0, offsets[27] = P).  Pairs of offset
 * d occupy [offsets[d], offsets[d+1]) in ascending out_idx:
 * (in_idx, out_idx) = (nbr[v][d], v) for every v with nbr[v][d] >= 0.
 */
SMC_API int smc_map_pairs(const smc_map* map, const int32_t** in_idx, const int32_t** out_idx,
                  int64_t offsets[28]);

/*
 * Tile schedule of the tensor-core conv (this library's own; the pages give
 * none): device pointer to perm[n] (int32), the order in which output rows
 * are grouped into tiles of 128 (a permutation of 0..n-1: rows are stably
 * sorted by which of the 8 corner and 12 edge offsets they hit, or, for maps
 * of at most 131072 rows, by the 8 corners alone, so
 * that each tile skips the offsets none of its rows has).
 */
SMC_API int smc_map_schedule(const smc_map* map, const int32_t** perm);

/*
 * Schedule segment (this library's own): the sort of smc_map_schedule runs
 * within each segment of `rows` consecutive input rows, segments kept in
 * input order, so that the tiles in flight at once gather from a window of
 * nearby rows.  rows = 0 (the default): the whole map is one segment;
 * rows > 0: a multiple of 2048; -1 restores the default.  Segments cut the
 * conv's DRAM reads on maps whose features exceed L2 when the input rows are
 * in a spatially coherent order, at some cost in skipped offsets.  Applies
 * to maps built after the call.  SMC_E_ARG otherwise.
 */
SMC_API int smc_set_schedule_segment(int64_t rows);

/* Release a map (its memory returns to the library's pool, ordered on the
 * build stream).  Work on other streams that reads the map must have
 * completed. */
SMC_API int smc_free_map(smc_map* map);

/* Synchronise `stream`, then return and clear the device-side error word
 * (SMC_E_TIMEOUT if a bounded wait in a conv kernel ran out), or SMC_OK. */
SMC_API int smc_status(void* stream);

/* Static description of an error code. */
SMC_API const char* smc_strerror(int code);

/*
 * Test and measurement hooks.
 * smc_set_hash_capacity: force the hash table to `slots` entries (rounded up
 *   to a power of two, minimum 16) for later builds; 0 restores automatic
 *   sizing (2^ceil(log2(4n)), or 2^ceil(log2(2n)) for keys of 32 bits or
 *   more).  Used to exercise SMC_E_CAPACITY.
 * smc_set_profiling: when on, smc_build_map records CUDA events on its stream
 *   around its kernels; smc_map_timing then returns, in milliseconds,
 *   ms[0] = the clears of the lookup structure and scratch, the insert and the
 *   neighbour lookups, ms[1] = tile schedule, and
 *   ms[2] = pair lists (built on a library-owned side stream, concurrently
 *   with the tile schedule; measured from the end of the lookups).
 * smc_kernel_launches: number of CUDA kernels this library has launched in
 *   the process so far (memsets and copies excluded).
 * smc_set_map_lookup: lookup structure of later builds: 0 = by size
 *   (default: a dense int32 index grid over the batch x Z x Y x X box when it
 *   has at most 2^28 sites and at most 256 sites per voxel -- cleared at
 *   every build when it has at most 2^23 sites and fewer than 16 per voxel,
 *   else left uncleared behind a cleared occupancy bitmap of one bit per
 *   site -- else a hash table), 1 = hash table, 2 = cleared dense grid and
 *   3 = dense grid with occupancy bitmap, each whenever the box has at most
 *   2^28 sites.  Maps are identical either way.  A forced hash capacity
 *   (smc_set_hash_capacity) always selects the hash table.  SMC_E_ARG for
 *   any other value.
 * smc_set_conv_variant: tensor-core conv kernel for later convs (bf16/fp16
 *   shapes the tensor cores take; others always use the FMA kernel): 0 =
 *   default (4 for a k = 3 conv with no fused activation or residual and 64
 *   output channels, or 128 on a map of at least 2 x 2 x 8 x SMs tiles of
 *   128 rows; else 1), 1 = fused 27-tap gather-GEMM, one CTA
 *   per 128-row tile, 2 = the same with CTA pairs (a cluster of two CTAs
 *   sharing M = 256 tcgen05 MMAs, each loading half of the weight block;
 *   slower on B200, where such clusters run one per TPC), 3 = per-offset
 *   gather-GEMM-scatter over the pair lists with fp32 atomic accumulation
 *   (k = 3 only; waits for the whole build; results equal to rounding),
 *   4 = fused, one CTA per two consecutive tiles, each weight stage feeding
 *   both tiles' MMAs (k = 3 with 64 or 128 output channels and no fused
 *   activation or residual; otherwise as 1).  1, 2 and 4 give identical
 *   bits.  Used to test and measure the variants.  SMC_E_ARG for any other
 *   value.
 */
/*
 * smc_neighbour_map_noalloc -- the int32 [n, 27] neighbour map of smc_build_map
 * (same values: nbr[v][d] = row of the site at c_v + delta_d, -1 if absent),
 * written into caller memory without allocating any device memory.  The pages
 * have no counterpart; this serves callers that may not allocate device memory
 * while they run: applications that reserve a fixed device-memory budget up
 * front and forbid allocation in their steady-state loop (an allocation can
 * stall, synchronise the device or fail part-way through), and plug-ins inside
 * a host framework that owns the device allocator.
 *
 * coords : device, int32 [n, 4] (b, z, y, x), 16-byte aligned.
 * nbr    : device, int32 [n, 27], 16-byte aligned; fully overwritten.
 * n      : at most 262144 (SMC_E_SHAPE above that).
 * batch, grid : as for smc_build_map; batch * Z * Y * X must be below
 *          2^32 - 1 (SMC_E_ARG otherwise).
 * stream : work is enqueued on it and the call synchronises it once, to read
 *          the error word (SMC_E_RANGE, SMC_E_DUPLICATE as for smc_build_map).
 *
 * Scratch: one file-scope device array of about 9.5 MB, which every GPU that
 * loads the library holds until the process exits; no cudaMalloc or other
 * allocating call is made.  The first call on a device looks up the array's
 * device address (cudaGetSymbolAddress) with that device current and caches
 * it with the device's current context; make that first call before any
 * stream capture.  After cudaDeviceReset (a new context) the next call looks
 * the address up again, so it too should come before any capture.  Every
 * call shares the array and clears what it reads; calls whose work overlaps on the GPU
 * (different streams or host threads) race on it and must be serialised by
 * the caller.  No pair lists or tile schedule are produced.
 */
SMC_API int smc_neighbour_map_noalloc(const int32_t* coords, int64_t n, int32_t batch, const int32_t grid[3],
                              int32_t* nbr, void* stream);

SMC_API int smc_set_hash_capacity(int64_t slots);
SMC_API int smc_set_profiling(int32_t on);
SMC_API int smc_map_timing(const smc_map* map, float ms[3]);
SMC_API int smc_kernel_launches(int64_t* count);
SMC_API int smc_set_conv_variant(int32_t variant);

/*
 * Stream of the convs (this library's own): 1 (default) runs each conv's
 * kernels on one of two library-owned streams of the greatest priority,
 * forked from the caller's stream by an event and joined back to it by
 * another, so the caller's stream orders the conv exactly as if it ran there;
 * the conv's CTAs are then dispatched before those of other work queued beside
 * it (e.g. a map build on another stream).  0 runs them on the caller's
 * stream.  SMC_E_ARG for any other value.
 */
SMC_API int smc_set_conv_priority(int32_t on);
/* smc_set_conv_epilogue: where smc_conv_ex applies the activation and the
 *   residual for the tensor-core conv: 0 = a row pass behind the conv, in
 *   row order, with the GroupNorm statistics in the same pass (default;
 *   measured faster; a residual that is the output buffer itself always
 *   goes through the epilogue), 1 = in the conv's own epilogue.  Results
 *   agree to rounding: the row pass sees the conv's stored (rounded) output,
 *   as a separate activation layer would.  Used to test and measure the
 *   two.  SMC_E_ARG for any other value. */
SMC_API int smc_set_conv_epilogue(int32_t where);
SMC_API int smc_set_map_lookup(int32_t mode);

/*
 * Failure-path test hooks (host side: no GPU fault is involved).
 * smc_set_alloc_fail_after: k >= 1 makes the k-th device allocation the
 *   library asks its pool for, counted from this call, report failure once;
 *   the entry point that asked returns SMC_E_OOM, leaves its handle output
 *   NULL and releases whatever it had allocated.  0 disarms the hook.
 *   SMC_E_ARG for k < 0.
 * smc_set_wait_limit_ns: bound, in nanoseconds, of every device-side wait:
 *   the single-pass scans' waits on earlier segments (every build,
 *   subdivision, upsample and downsample runs such scans) and the convs'
 *   pipeline waits (never below 100 ms for those, so that no CTA gives up
 *   with loads in flight); 0 restores the default 2 s.  SMC_E_ARG for ns < 0.
 * smc_set_scan_hold: in every later scan, the segment with this ticket
 *   (0-based, in start order) publishes nothing, so the waits of the
 *   segments after it run out and the call reports SMC_E_TIMEOUT; every
 *   access stays in bounds and the device stays usable.  -1 (default) turns
 *   it off; SMC_E_ARG below -1.  Meant for use with a short wait limit.
 */
SMC_API int smc_set_alloc_fail_after(int64_t k);
SMC_API int smc_set_wait_limit_ns(int64_t ns);
SMC_API int smc_set_scan_hold(int64_t ticket);

#ifdef __cplusplus
}
#endif

#endif /* SMC_H_ */
