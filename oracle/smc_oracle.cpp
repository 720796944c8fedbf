// CPU oracle for submanifold sparse convolution (SubMConv3d, stride 1).
//
// TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously-correct
// definition that the CUDA library is checked against.  Only the tests, the
// smoke check and the benchmark's CPU-baseline leg may load it; the product
// path never does.  It shares no code, header, table or constant with the
// CUDA library: coordinates are keyed by the (b, z, y, x) tuple itself in an
// ordered std::map (no key packing, no hashing), and every sum runs in fp64.
//
// What it computes (LATO.2 MLX port README, "The scope, once measured" and
// "Correctness"; Pixal3D working notes, "Measured facts"):
//   * The layer is a submanifold 3x3x3 convolution: outputs exist only at the
//     input's active sites, and each output sums, over the k^3 kernel offsets,
//     the feature row of the active neighbour at that offset times the weight
//     slice of that offset.  Inactive or out-of-grid neighbours contribute 0.
//   * Weights use the spconv KRSC layout [Cout, kz, ky, kx, Cin] (LATO.2 README,
//     summary; Pixal3D commit log, converter paragraph).
//   * Orientation: +1 gathers feats[c + d] (cross-correlation, the port's
//     implemented convention), -1 gathers feats[c - d] (LATO.2 README,
//     "Correctness": the kernel-orientation caveat).
//   * k = 1 is the centre tap alone, i.e. a per-voxel linear layer (LATO.2
//     README, "Status").
// Readings where the pages are silent (coordinate column order (b,z,y,x),
// offset enumeration in C order of (kz,ky,kx), duplicates and out-of-grid
// coordinates being errors, bias added once per output row) are the plainest
// ones and are listed in the design notes.
//
// Build: g++ -O2 -fopenmp -shared -fPIC smc_oracle.cpp -o libsmc_oracle.so

#include <array>
#include <cstdint>
#include <map>
#include <vector>

namespace {

using Site = std::array<int32_t, 4>;        // (b, z, y, x)
using SiteIndex = std::map<Site, int64_t>;  // site -> input row

constexpr int kOk = 0;
constexpr int kErrArg = -1;
constexpr int kErrRange = -2;
constexpr int kErrDuplicate = -3;

// Build the site -> row dictionary; reject out-of-grid and repeated sites.
int index_sites(const int32_t* coords, int64_t n, const int32_t* grid, SiteIndex& index) {
  for (int64_t r = 0; r < n; ++r) {
    const int32_t* c = coords + 4 * r;
    if (c[0] < 0) return kErrRange;
    for (int a = 0; a < 3; ++a)
      if (c[1 + a] < 0 || c[1 + a] >= grid[a]) return kErrRange;
    Site s = {c[0], c[1], c[2], c[3]};
    if (!index.emplace(s, r).second) return kErrDuplicate;
  }
  return kOk;
}

// The kernel offset of tap d (C order over kz, ky, kx), relative to the centre.
void tap_offset(int d, int k, int32_t delta[3]) {
  const int h = (k - 1) / 2;
  const int kz = d / (k * k), ky = (d / k) % k, kx = d % k;
  delta[0] = kz - h;
  delta[1] = ky - h;
  delta[2] = kx - h;
}

// Row of the active site at c + sign * delta, or -1.
int64_t neighbour(const SiteIndex& index, const int32_t* c, const int32_t delta[3], int sign) {
  Site s = {c[0], c[1] + sign * delta[0], c[2] + sign * delta[1], c[3] + sign * delta[2]};
  auto it = index.find(s);
  return it == index.end() ? -1 : it->second;
}

}  // namespace

extern "C" {

// Neighbour map: nbr[v * k^3 + d] = row of the site at c_v + offset(d), or -1.
int oracle_neighbour_map(const int32_t* coords, int64_t n, const int32_t* grid, int32_t k,
                         int32_t* nbr) {
  if (n < 0 || (k != 1 && k != 3) || (n > 0 && (!coords || !nbr)) || !grid) return kErrArg;
  SiteIndex index;
  int rc = index_sites(coords, n, grid, index);
  if (rc != kOk) return rc;
  const int taps = k * k * k;
  for (int64_t v = 0; v < n; ++v) {
    for (int d = 0; d < taps; ++d) {
      int32_t delta[3];
      tap_offset(d, k, delta);
      nbr[v * taps + d] = static_cast<int32_t>(neighbour(index, coords + 4 * v, delta, +1));
    }
  }
  return kOk;
}

// Per-offset pair lists, each in ascending output row:
//   pairs_d = [(nbr[v][d], v) for v = 0..n-1 if nbr[v][d] >= 0]
// concatenated in d order.  counts[d] = |pairs_d|.  in_idx / out_idx must
// hold sum(counts) entries; pass NULL to only count.
int oracle_pair_lists(const int32_t* nbr, int64_t n, int32_t taps, int64_t* counts,
                      int32_t* in_idx, int32_t* out_idx) {
  if (n < 0 || taps <= 0 || !counts || (n > 0 && !nbr)) return kErrArg;
  int64_t pos = 0;
  for (int d = 0; d < taps; ++d) {
    counts[d] = 0;
    for (int64_t v = 0; v < n; ++v) {
      const int32_t u = nbr[v * taps + d];
      if (u < 0) continue;
      if (in_idx) in_idx[pos] = u;
      if (out_idx) out_idx[pos] = static_cast<int32_t>(v);
      ++pos;
      ++counts[d];
    }
  }
  return kOk;
}

// Submanifold convolution for the output rows listed in `rows` (all rows when
// rows == NULL, then nrows must equal n):
//   out[j][o] = bias[o] + sum_d sum_i feats[u][i] * weight[o][d][i],
//   u = row of the active site at c_v + orientation * offset(d), v = rows[j];
// terms with no active site there are dropped.  All arithmetic is fp64, the
// sum runs over d then i.
int oracle_conv(const int32_t* coords, int64_t n, const int32_t* grid, const double* feats,
                int64_t cin, const double* weight, const double* bias, int64_t cout, int32_t k,
                int32_t orientation, const int64_t* rows, int64_t nrows, double* out,
                int32_t threads) {
  if (n < 0 || cin <= 0 || cout <= 0 || (k != 1 && k != 3) ||
      (orientation != 1 && orientation != -1) || !grid || nrows < 0)
    return kErrArg;
  if (!rows && nrows != n) return kErrArg;
  if (n > 0 && (!coords || !feats || !weight || !out)) return kErrArg;
  SiteIndex index;
  int rc = index_sites(coords, n, grid, index);
  if (rc != kOk) return rc;
  if (rows)
    for (int64_t j = 0; j < nrows; ++j)
      if (rows[j] < 0 || rows[j] >= n) return kErrArg;
  const int taps = k * k * k;
#pragma omp parallel for schedule(dynamic, 64) num_threads(threads > 0 ? threads : 1)
  for (int64_t j = 0; j < nrows; ++j) {
    const int64_t v = rows ? rows[j] : j;
    std::vector<double> acc(cout, 0.0);
    for (int d = 0; d < taps; ++d) {
      int32_t delta[3];
      tap_offset(d, k, delta);
      const int64_t u = neighbour(index, coords + 4 * v, delta, orientation);
      if (u < 0) continue;
      const double* f = feats + u * cin;
      for (int64_t o = 0; o < cout; ++o) {
        const double* w = weight + (o * taps + d) * cin;
        double s = acc[o];
        for (int64_t i = 0; i < cin; ++i) s += f[i] * w[i];
        acc[o] = s;
      }
    }
    for (int64_t o = 0; o < cout; ++o) out[j * cout + o] = acc[o] + (bias ? bias[o] : 0.0);
  }
  return kOk;
}

}  // extern "C"
