// smc_neighbour_map_noalloc: the int32 [n, 27] neighbour map written into
// caller memory without any device allocation.
//
// Some callers cannot allocate device memory while they run: applications
// that reserve a fixed device-memory budget up front and forbid allocation in
// their steady-state loop (an allocation can stall, synchronise the device or
// fail part-way through a frame), and plug-ins hosted by a framework that
// owns the device allocator and does not hand out cudaMalloc.  This entry
// point serves them.  Its scratch (hash table, error word and the per-row
// outputs the lookup kernel also writes) lives in one file-scope __device__
// array of fixed size, which every GPU that loads the library keeps until the
// process exits.
//
// The array's name is a host-side stand-in in host code, not a device
// address; the first call on each device looks the address up with
// cudaGetSymbolAddress while that device is current and caches it together
// with the device's current context.  A call that finds another context
// current (after cudaDeviceReset, or a re-created primary context) looks the
// address up again, so a cached address never outlives its context.  All
// calls share the one array and it keeps the last call's contents, so the
// table and the error word are cleared on every call, and calls whose work
// overlaps on the GPU (different streams, or several host threads) race with
// each other.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "smc.h"
#include "common.cuh"
#include "kernels.h"

namespace {

constexpr int64_t kNoAllocMaxN = 1 << 18;  // voxels per call
constexpr int kNoAllocMaxLg = 20;          // 2^20 hash slots: load <= 1/4 at the maximum n
constexpr int kNoAllocMaxBlocks = static_cast<int>(kNoAllocMaxN / 256);

struct NoAllocScratch {
  unsigned long long table[1ull << kNoAllocMaxLg];
  uint32_t gkey[kNoAllocMaxN];
  int32_t block_counts[smc::kTaps * kNoAllocMaxBlocks];
  uint32_t err;
};

// About 9.5 MB per device.
static __device__ __align__(256) NoAllocScratch g_noalloc_scratch;

constexpr int kMaxDevices = 64;
NoAllocScratch* g_scratch_addr[kMaxDevices] = {};
void* g_scratch_ctx[kMaxDevices] = {};  // the context the cached address belongs to
std::mutex g_scratch_mu;

// The driver's cuCtxGetCurrent, reached through the runtime (the library
// links only the CUDA runtime).
using CtxGetCurrentFn = int (*)(void**);
CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
    cudaGetLastError();
  });
  return fn;
}

// Device address of the scratch array on `dev` (the current device): looked
// up once per device and context, and again whenever the current context is
// not the one the cached address was found in.
NoAllocScratch* scratch_on(int dev) {
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  CtxGetCurrentFn get_ctx = ctx_get_current();
  if (!get_ctx) return nullptr;
  void* ctx = nullptr;  // null before the runtime has made the device's context current
  if (get_ctx(&ctx) != 0) return nullptr;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!ctx || !g_scratch_addr[dev] || g_scratch_ctx[dev] != ctx) {
    g_scratch_addr[dev] = nullptr;
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) {
      cudaGetLastError();
      return nullptr;
    }
    if (get_ctx(&ctx) != 0 || !ctx) return nullptr;  // current now: the lookup needed it
    g_scratch_addr[dev] = static_cast<NoAllocScratch*>(ptr);
    g_scratch_ctx[dev] = ctx;
  }
  return g_scratch_addr[dev];
}

}  // namespace

extern "C" int smc_neighbour_map_noalloc(const int32_t* coords, int64_t n, int32_t batch, const int32_t grid[3],
                                         int32_t* nbr, void* stream) {
  if (!grid || n < 0 || batch < 1 || (n > 0 && (!coords || !nbr))) return SMC_E_ARG;
  if (grid[0] < 1 || grid[1] < 1 || grid[2] < 1) return SMC_E_ARG;
  if (n > kNoAllocMaxN) return SMC_E_SHAPE;
  const double sites = static_cast<double>(batch) * grid[0] * grid[1] * grid[2];
  if (sites > 4294967294.0) return SMC_E_ARG;  // keys must fit the one-word hash slots
  if (n == 0) return SMC_OK;
  if ((reinterpret_cast<uintptr_t>(coords) & 15u) || (reinterpret_cast<uintptr_t>(nbr) & 15u)) return SMC_E_ALIGN;
  if (cudaGetLastError() != cudaSuccess) return SMC_E_CUDA;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SMC_E_CUDA;
  NoAllocScratch* sc = scratch_on(dev);
  if (!sc) return SMC_E_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int lg = 4;
  while ((1ll << lg) < 4 * n) ++lg;
  const size_t cap = size_t(1) << lg;
  cudaError_t e = cudaMemsetAsync(sc->table, 0xFF, cap * sizeof(unsigned long long), s);
  if (e == cudaSuccess) e = cudaMemsetAsync(&sc->err, 0, sizeof(uint32_t), s);
  if (e == cudaSuccess)
    e = smc::launch_neighbour_map_only(coords, n, batch, grid[0], grid[1], grid[2], sc->table, lg, &sc->err, nbr,
                                       sc->gkey, sc->block_counts, s);
  uint32_t err = 0;
  if (e == cudaSuccess) e = cudaMemcpyAsync(&err, &sc->err, sizeof(uint32_t), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return SMC_E_CUDA;
  }
  if (err & smc::kErrRange) return SMC_E_RANGE;
  if (err & smc::kErrDuplicate) return SMC_E_DUPLICATE;
  if (err & smc::kErrCapacity) return SMC_E_CAPACITY;
  return SMC_OK;
}
