// Host side of libsmc: the C ABI declared in include/smc.h.
//
// Owns the neighbour-map handle (device buffers allocated stream-ordered on
// the build stream), validates every argument before anything is launched,
// picks the conv kernel, and turns device error bits into SMC_E_* codes.
#include <cuda_runtime.h>

#include <atomic>
#include <cstddef>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "smc.h"
#include "common.cuh"
#include "kernels.h"

// Status block a build copies back to the host: error bits and pair offsets.
struct HostSlot {
  uint32_t err;
  uint32_t pad;
  int64_t info[28];
};

struct smc_map {
  int device;
  cudaStream_t stream;
  int64_t n;
  int32_t batch;
  int32_t grid[3];
  int32_t* nbr;
  int32_t* in_idx;
  int32_t* out_idx;
  int32_t* perm;
  uint32_t* tile_mask;
  int64_t* pair_offsets;  // device copy of the 28 pair-list offsets
  void* keep;           // one allocation holding nbr, pairs, schedule and tile masks
  mutable void* tmp;    // the build's scratch, released at the first wait on the map
  cudaEvent_t done;     // recorded after the status block is copied back
  cudaEvent_t prof[4];  // optional timing events
  HostSlot* slot;       // pinned status block
  // filled in when the build is first waited on
  mutable std::mutex mu;
  mutable bool resolved;
  mutable int status;
  mutable int64_t counts[27];
  mutable int64_t offsets[28];
  mutable float ms[3];
};

namespace {

std::atomic<int64_t> g_capacity_override{0};
// Test hooks of the failure paths (smc_set_alloc_fail_after, smc_set_wait_limit_ns, smc_set_scan_hold).
std::atomic<int64_t> g_alloc_fail_after{0};
std::atomic<int64_t> g_wait_limit_ns{static_cast<int64_t>(smc::kWaitLimitNs)};
std::atomic<int64_t> g_scan_hold{-1};
std::atomic<long long> g_launches{0};
std::atomic<int32_t> g_profiling{0};
std::atomic<int32_t> g_map_lookup{0};

// Largest box (batch * Z * Y * X sites) that gets a dense index grid: 1 GB of
// int32, cleared at every build.
constexpr double kDenseMaxSites = 268435456.0;
// Boxes above this many sites (a 32 MB grid) take the occupancy-bitmap grid,
// and so do sparser ones (see build_async).
constexpr double kOccMinSites = 8388608.0;

constexpr int kMaxDevices = 64;

// Per-device error word of the conv kernels (bounded-wait timeouts).
uint32_t* g_status[kMaxDevices] = {};
// Per-device stream-ordered memory pool that keeps its memory between builds
// (the default pool returns memory to the driver at every synchronisation,
// which made each build re-map its buffers).
cudaMemPool_t g_pool[kMaxDevices] = {};
std::mutex g_dev_mu;

uint32_t* device_status(int dev) {
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (!g_status[dev]) {
    void* p = nullptr;
    if (cudaMalloc(&p, 256) != cudaSuccess) return nullptr;
    if (cudaMemset(p, 0, 256) != cudaSuccess) return nullptr;
    g_status[dev] = static_cast<uint32_t*>(p);
  }
  return g_status[dev];
}

cudaMemPool_t device_pool(int dev) {
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (!g_pool[dev]) {
    cudaMemPoolProps props;
    std::memset(&props, 0, sizeof(props));
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t pool = nullptr;
    if (cudaMemPoolCreate(&pool, &props) != cudaSuccess) return nullptr;
    uint64_t keep_all = ~0ull;
    cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep_all);
    g_pool[dev] = pool;
  }
  return g_pool[dev];
}

// Per-device side stream: the pair lists are built there, concurrently with
// the tile schedule on the build stream (the conv needs the schedule, not the
// pair lists).
cudaStream_t g_side[kMaxDevices] = {};

cudaStream_t side_stream(int dev) {
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (!g_side[dev] && cudaStreamCreateWithFlags(&g_side[dev], cudaStreamNonBlocking) != cudaSuccess) {
    cudaGetLastError();
    g_side[dev] = nullptr;
  }
  return g_side[dev];
}

// Per-device streams of the greatest priority that the convs run on, forked
// from and joined back to the caller's stream (smc_set_conv_priority): a
// conv's CTAs are then dispatched before those of map builds and other work
// queued beside it, e.g. the next step's build on another stream.  Two, used
// in turn, so that consecutive convs of different callers can overlap.
constexpr int kPrioStreams = 2;
cudaStream_t g_prio[kMaxDevices][kPrioStreams] = {};
std::atomic<uint32_t> g_prio_next[kMaxDevices] = {};
std::atomic<int32_t> g_conv_priority{1};

cudaStream_t prio_stream(int dev) {
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  const uint32_t k = g_prio_next[dev].fetch_add(1, std::memory_order_relaxed) % kPrioStreams;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (!g_prio[dev][k]) {
    int lo = 0, hi = 0;
    if (cudaDeviceGetStreamPriorityRange(&lo, &hi) != cudaSuccess ||
        cudaStreamCreateWithPriority(&g_prio[dev][k], cudaStreamNonBlocking, hi) != cudaSuccess) {
      cudaGetLastError();
      g_prio[dev][k] = nullptr;
    }
  }
  return g_prio[dev][k];
}

// Per-device pool of timing-free events (fork/join points and the maps'
// completion events), reused instead of created per build.
std::mutex g_ev_mu;
std::vector<cudaEvent_t> g_events[kMaxDevices];

std::vector<cudaEvent_t> g_timing_events[kMaxDevices];  // the same, with timing (profiling)

cudaEvent_t take_event(int dev, bool timing = false) {
  {
    std::lock_guard<std::mutex> lk(g_ev_mu);
    std::vector<cudaEvent_t>& pool = timing ? g_timing_events[dev] : g_events[dev];
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreateWithFlags(&e, timing ? cudaEventDefault : cudaEventDisableTiming) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return e;
}

// An event may go back once every wait on it has been enqueued (a wait binds
// to the record made before it) or, for a completion or timing event, once
// it is done.
void give_event(int dev, cudaEvent_t e, bool timing = false) {
  if (!e) return;
  std::lock_guard<std::mutex> lk(g_ev_mu);
  (timing ? g_timing_events[dev] : g_events[dev]).push_back(e);
}

// Pinned host status blocks, handed out from chunks of 256.
std::mutex g_slot_mu;
std::vector<HostSlot*> g_free_slots;

HostSlot* take_slot() {
  std::lock_guard<std::mutex> lk(g_slot_mu);
  if (g_free_slots.empty()) {
    void* p = nullptr;
    if (cudaMallocHost(&p, 256 * sizeof(HostSlot)) != cudaSuccess) return nullptr;
    HostSlot* s = static_cast<HostSlot*>(p);
    for (int i = 0; i < 256; ++i) g_free_slots.push_back(s + i);
  }
  HostSlot* s = g_free_slots.back();
  g_free_slots.pop_back();
  return s;
}

void give_slot(HostSlot* s) {
  if (!s) return;
  std::lock_guard<std::mutex> lk(g_slot_mu);
  g_free_slots.push_back(s);
}

// Every device allocation of the library goes through here: stream-ordered,
// from the library's pool.  When smc_set_alloc_fail_after(k) is armed, the
// k-th allocation from then on reports failure instead (once), which is how
// the SMC_E_OOM paths are exercised without exhausting a GPU.
cudaError_t pool_alloc(void** p, size_t bytes, cudaMemPool_t pool, cudaStream_t s) {
  *p = nullptr;
  if (!pool) return cudaErrorMemoryAllocation;
  int64_t k = g_alloc_fail_after.load();
  while (k > 0) {
    if (g_alloc_fail_after.compare_exchange_weak(k, k - 1)) {
      if (k == 1) return cudaErrorMemoryAllocation;
      break;
    }
  }
  return cudaMallocFromPoolAsync(p, bytes, pool, s);
}

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Bump allocator over one device allocation.
struct Carve {
  size_t off = 0;
  template <typename T>
  size_t take(size_t count) {
    const size_t o = align_up(off, 256);
    off = o + count * sizeof(T);
    return o;
  }
};

int pending_cuda_error() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SMC_OK : SMC_E_CUDA;
}

bool ranges_overlap(const void* a, size_t na, const void* b, size_t nb) {
  if (!a || !b || na == 0 || nb == 0) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + nb && b0 < a0 + na;
}

// The build's scratch goes back to the pool on the build stream once the
// build is known complete (its completion event has been waited on).  Freed
// there, the next build on that stream reuses it; released on the side
// stream, where its last user runs, it was never reused and the pool grew
// by the scratch size at every build.
void release_scratch(const smc_map* m) {
  if (!m->tmp) return;
  int cur = 0;
  cudaGetDevice(&cur);
  if (cur != m->device) cudaSetDevice(m->device);
  cudaFreeAsync(m->tmp, m->stream);
  m->tmp = nullptr;
  if (cur != m->device) cudaSetDevice(cur);
  cudaGetLastError();
}

void release_map(smc_map* m) {
  if (!m) return;
  int cur = 0;
  cudaGetDevice(&cur);
  if (cur != m->device) cudaSetDevice(m->device);
  if (m->done) cudaEventSynchronize(m->done);  // the status copy must land before the slot is reused
  release_scratch(m);
  if (m->keep) cudaFreeAsync(m->keep, m->stream);
  give_event(m->device, m->done);
  for (auto& e : m->prof) give_event(m->device, e, true);
  give_slot(m->slot);
  if (cur != m->device) cudaSetDevice(cur);
  cudaGetLastError();
  delete m;
}

// Wait for a build to finish and record its outcome (once).
int resolve(const smc_map* m) {
  std::lock_guard<std::mutex> lk(m->mu);
  if (m->resolved) return m->status;
  int rc = SMC_OK;
  if (m->done && cudaEventSynchronize(m->done) != cudaSuccess) {
    cudaGetLastError();
    rc = SMC_E_CUDA;
  } else if (m->slot) {
    release_scratch(m);
    const uint32_t err = m->slot->err;
    if (err & smc::kErrRange) rc = SMC_E_RANGE;
    else if (err & smc::kErrDuplicate) rc = SMC_E_DUPLICATE;
    else if (err & smc::kErrCapacity) rc = SMC_E_CAPACITY;
    else if (err & smc::kErrTimeout) rc = SMC_E_TIMEOUT;
    for (int d = 0; d < 28; ++d) m->offsets[d] = m->slot->info[d];
    for (int d = 0; d < 27; ++d) m->counts[d] = m->slot->info[d + 1] - m->slot->info[d];
  }
  if (rc == SMC_OK && m->prof[0]) {
    cudaEventElapsedTime(&m->ms[0], m->prof[0], m->prof[1]);
    cudaEventElapsedTime(&m->ms[1], m->prof[1], m->prof[2]);
    cudaEventElapsedTime(&m->ms[2], m->prof[1], m->prof[3]);
  }
  m->status = rc;
  m->resolved = true;
  return rc;
}

// Children of a parent map whose rows are read off the parent map
// (smc_subdivide): replaces the lookup structure and the lookup kernels.
struct SubdivSource {
  const int32_t* parent_nbr;
  const int32_t* child_src;  // [n] 8 * parent row + octant
  const int32_t* remap;      // [8 * parent n] child row or -1
};

// Enqueue a whole map build on `s`; no synchronisation.
int build_async(const int32_t* coords, int64_t n, int32_t batch, const int32_t grid[3], cudaStream_t s,
                smc_map** out, const SubdivSource* sub = nullptr) {
  if (!out) return SMC_E_ARG;
  *out = nullptr;
  if (!grid || n < 0 || batch < 1 || (n > 0 && !coords && !sub)) return SMC_E_ARG;
  if (grid[0] < 1 || grid[1] < 1 || grid[2] < 1) return SMC_E_ARG;
  if (n >= (1ll << 31) - 1) return SMC_E_ARG;  // rows are int32
  if (n > 0 && !sub && (reinterpret_cast<uintptr_t>(coords) & 15u)) return SMC_E_ALIGN;
  const double sites = static_cast<double>(batch) * grid[0] * grid[1] * grid[2];
  if (sites >= 4.6e18) return SMC_E_ARG;
  if (pending_cuda_error() != SMC_OK) return SMC_E_CUDA;

  smc_map* m = new (std::nothrow) smc_map();
  if (!m) return SMC_E_OOM;
  cudaGetDevice(&m->device);
  m->stream = s;
  m->n = n;
  m->batch = batch;
  for (int i = 0; i < 3; ++i) m->grid[i] = grid[i];
  if (n == 0) {
    m->resolved = true;
    *out = m;
    return SMC_OK;
  }
  cudaMemPool_t pool = device_pool(m->device);
  m->slot = take_slot();
  cudaStream_t side = side_stream(m->device);
  m->done = take_event(m->device);
  cudaEvent_t ev_fork = take_event(m->device), ev_sched = take_event(m->device);
  if (!pool || !m->slot || !side || !m->done || !ev_fork || !ev_sched) {
    give_event(m->device, ev_fork);
    give_event(m->device, ev_sched);
    release_map(m);
    return SMC_E_OOM;
  }

  // ---- sizes
  // Lookup structure.  A dense index grid turns each row's 27 lookups into 9
  // runs of three consecutive sites, which neighbouring rows share; it is
  // used when the box is at most 256 sites per voxel (clearing it then costs
  // less than hash probing) and at most 2^28 sites.  Otherwise a hash table.
  const int64_t forced = g_capacity_override.load();
  const int lookup = g_map_lookup.load();
  const bool dense = !sub && forced == 0 && sites <= kDenseMaxSites &&
                     (lookup == 2 || lookup == 3 || (lookup == 0 && sites <= 256.0 * static_cast<double>(n)));
  // A grid larger than L2, or one with 16 or more sites per voxel, is not
  // cleared: an occupancy bitmap, 1/32 of its size, is cleared instead (with
  // the build's other scratch, in one memset) and guards every read of it.
  // Measured on B200: 512^3 decoder stage, clears and lookups 0.163 -> 0.106
  // ms; 6-shell 128^3 (22 sites per voxel) 0.026 -> 0.024 ms; the full 128^3
  // grid, where every lookup hits, 0.088 -> 0.159 ms.
  const bool occ = dense && (lookup == 3 || (lookup == 0 && (sites > kOccMinSites ||
                                                              sites >= 16.0 * static_cast<double>(n))));
  const bool wide = !dense && sites > 4294967294.0;  // packed slots need keys < 2^32 - 1
  int lg = 4;
  // Packed slots: load <= 1/4, so lookups (which read 2-slot groups) resolve
  // in one round almost always (measured: 256^3 shells+planes map 0.59 ms at
  // 1/4 vs 0.83 ms at 1/2).  Two-word slots: load <= 1/2.
  const int64_t want = forced > 0 ? forced : (wide ? 2 : 4) * n;
  while ((1ll << lg) < want) ++lg;
  const int64_t cap = 1ll << lg;
  const int nb = smc::map_nblocks(n);
  const int64_t Lmap = 27ll * nb;
  const int radix_cps = smc::radix_seg_chunks(n);
  const int64_t Lrad = smc::radix_hist_len(n, radix_cps);
  const int64_t pair_cap = 27ll * n;

  Carve keep;
  const size_t o_nbr = keep.take<int32_t>(27ull * n);
  const size_t o_in = keep.take<int32_t>(pair_cap);
  const size_t o_out = keep.take<int32_t>(pair_cap);
  const size_t o_perm = keep.take<int32_t>(n);
  const size_t o_tmask = keep.take<uint32_t>((n + smc::kTileRows - 1) / smc::kTileRows);
  const size_t o_poff = keep.take<int64_t>(28);
  Carve tmp;
  const size_t table_bytes = sub     ? 16
                             : dense ? static_cast<size_t>(sites) * sizeof(int32_t)
                                     : (wide ? 2 : 1) * static_cast<size_t>(cap) * sizeof(unsigned long long);
  const size_t o_table = tmp.take<uint8_t>(table_bytes);
  const size_t o_gkey = tmp.take<uint32_t>(n);
  const size_t o_bc = tmp.take<int32_t>(Lmap);
  const size_t o_bo = tmp.take<int64_t>(Lmap);
  const size_t o_hoff = tmp.take<int64_t>(Lrad);
  const size_t o_ktmp = tmp.take<uint32_t>(n);
  const size_t o_vtmp = tmp.take<int32_t>(n);
  // zeroed by one memset: the device image of the status block (error word,
  // pair offsets), scan tickets and statuses, histograms
  const size_t o_err = tmp.take<HostSlot>(1);
  const size_t o_tick = tmp.take<uint32_t>(3);
  const size_t o_st0 = tmp.take<unsigned long long>(smc::scan_status_len(Lmap));
  const size_t o_st1 = tmp.take<unsigned long long>(smc::scan_status_len(Lrad));
  const size_t o_st2 = tmp.take<unsigned long long>(smc::scan_status_len(Lrad));
  const size_t o_h1 = tmp.take<int32_t>(Lrad);
  const size_t o_h2 = tmp.take<int32_t>(Lrad);
  const size_t o_occ = tmp.take<uint32_t>(occ ? (static_cast<size_t>(sites) + 31) / 32 : 0);
  const size_t zero_bytes = tmp.off - o_err;

  void* tp = nullptr;
  if (pool_alloc(&m->keep, keep.off, pool, s) != cudaSuccess) {
    cudaGetLastError();
    m->keep = nullptr;
    give_event(m->device, ev_fork);
    give_event(m->device, ev_sched);
    release_map(m);
    return SMC_E_OOM;
  }
  if (pool_alloc(&tp, tmp.off, pool, s) != cudaSuccess) {
    cudaGetLastError();
    give_event(m->device, ev_fork);
    give_event(m->device, ev_sched);
    release_map(m);
    return SMC_E_OOM;
  }
  char* K = static_cast<char*>(m->keep);
  char* T = static_cast<char*>(tp);
  m->nbr = reinterpret_cast<int32_t*>(K + o_nbr);
  m->in_idx = reinterpret_cast<int32_t*>(K + o_in);
  m->out_idx = reinterpret_cast<int32_t*>(K + o_out);
  m->perm = reinterpret_cast<int32_t*>(K + o_perm);
  m->tile_mask = reinterpret_cast<uint32_t*>(K + o_tmask);
  m->pair_offsets = reinterpret_cast<int64_t*>(K + o_poff);

  if (g_profiling.load() != 0)
    for (auto& e : m->prof) e = take_event(m->device, true);

  uint32_t* err = reinterpret_cast<uint32_t*>(T + o_err + offsetof(HostSlot, err));
  uint32_t* tickets = reinterpret_cast<uint32_t*>(T + o_tick);
  smc::MapBuildArgs a;
  a.coords = coords;
  a.n = n;
  a.batch = batch;
  a.Z = grid[0];
  a.Y = grid[1];
  a.X = grid[2];
  a.kind = occ ? smc::kMapDenseOcc : dense ? smc::kMapDense : (wide ? smc::kMapWide : smc::kMapPacked);
  a.occ = occ ? reinterpret_cast<uint32_t*>(T + o_occ) : nullptr;
  a.table = reinterpret_cast<unsigned long long*>(T + o_table);
  a.lg = lg;
  a.err = err;
  a.zero = m->tile_mask;
  a.nzero = (n + smc::kTileRows - 1) / smc::kTileRows;
  a.nbr = m->nbr;
  a.gkey = reinterpret_cast<uint32_t*>(T + o_gkey);
  a.block_counts = reinterpret_cast<int32_t*>(T + o_bc);
  a.block_offsets = reinterpret_cast<int64_t*>(T + o_bo);
  a.scan_status = reinterpret_cast<unsigned long long*>(T + o_st0);
  a.scan_ticket = tickets;
  a.hist1 = reinterpret_cast<int32_t*>(T + o_h1);
  a.radix_cps = radix_cps;
  a.info = reinterpret_cast<int64_t*>(T + o_err + offsetof(HostSlot, info));
  a.in_idx = m->in_idx;
  a.out_idx = m->out_idx;
  smc::ScheduleArgs b;
  b.gkey = a.gkey;
  b.n = n;
  b.hist1 = a.hist1;
  b.radix_cps = radix_cps;
  b.hist2 = reinterpret_cast<int32_t*>(T + o_h2);
  b.hoff = reinterpret_cast<int64_t*>(T + o_hoff);
  b.status1 = reinterpret_cast<unsigned long long*>(T + o_st1);
  b.status2 = reinterpret_cast<unsigned long long*>(T + o_st2);
  b.tickets = tickets + 1;
  b.key_tmp = reinterpret_cast<uint32_t*>(T + o_ktmp);
  b.val_tmp = reinterpret_cast<int32_t*>(T + o_vtmp);
  b.perm = m->perm;
  b.tile_mask = m->tile_mask;
  b.err = err;

  // Build stream s: clear, insert + lookups, then the tile schedule.  Side
  // stream: the pair lists (forked after the lookups), then -- once the
  // schedule is done too -- the status copy, the completion event and the
  // release of the scratch.  A conv enqueued on s behind the build waits for
  // the schedule only, and overlaps the pair lists.
  cudaError_t ce = m->prof[0] ? cudaEventRecord(m->prof[0], s) : cudaSuccess;  // the clears count as lookups
  if (ce == cudaSuccess && !occ) ce = cudaMemsetAsync(T + o_table, 0xFF, table_bytes, s);
  if (ce == cudaSuccess) ce = cudaMemsetAsync(T + o_err, 0, zero_bytes, s);
  if (ce == cudaSuccess && sub) {
    ce = cudaMemsetAsync(m->tile_mask, 0, a.nzero * sizeof(uint32_t), s);  // k_insert clears them otherwise
    if (ce == cudaSuccess) ce = smc::launch_subdiv_lookups(a, sub->parent_nbr, sub->child_src, sub->remap, s);
  } else if (ce == cudaSuccess) {
    ce = smc::launch_map_lookups(a, s);
  }
  if (ce == cudaSuccess && m->prof[1]) ce = cudaEventRecord(m->prof[1], s);
  if (ce == cudaSuccess) ce = cudaEventRecord(ev_fork, s);
  if (ce == cudaSuccess) ce = cudaStreamWaitEvent(side, ev_fork, 0);
  if (ce == cudaSuccess) ce = smc::launch_pair_lists(a, side);
  if (ce == cudaSuccess)
    ce = cudaMemcpyAsync(m->pair_offsets, a.info, 28 * sizeof(int64_t), cudaMemcpyDeviceToDevice, side);
  if (ce == cudaSuccess && m->prof[3]) ce = cudaEventRecord(m->prof[3], side);
  if (ce == cudaSuccess) ce = smc::launch_schedule(b, s);
  if (ce == cudaSuccess && m->prof[2]) ce = cudaEventRecord(m->prof[2], s);
  if (ce == cudaSuccess) ce = cudaEventRecord(ev_sched, s);
  if (ce == cudaSuccess) ce = cudaStreamWaitEvent(side, ev_sched, 0);
  // the only device->host traffic: error bits and pair offsets, into pinned memory
  if (ce == cudaSuccess) ce = cudaMemcpyAsync(m->slot, T + o_err, sizeof(HostSlot), cudaMemcpyDeviceToHost, side);
  if (ce == cudaSuccess) ce = cudaEventRecord(m->done, side);
  m->tmp = tp;  // released after the first wait on the map (release_scratch)
  give_event(m->device, ev_fork);  // their waits are enqueued
  give_event(m->device, ev_sched);
  if (ce != cudaSuccess) {
    cudaGetLastError();
    cudaStreamSynchronize(s);
    cudaStreamSynchronize(side);
    cudaGetLastError();
    m->tmp = tp;
    release_map(m);
    return SMC_E_CUDA;
  }
  *out = m;
  return SMC_OK;
}

// GroupNorm statistics are accumulated into kStatStripes copies (each block
// adds into copy blockIdx % kStatStripes, spreading concurrent fp64 atomics
// on one (item, group) over that many addresses) and folded into the
// caller's array at the end: one pool allocation, memset and fold per call.
constexpr int kStatStripes = 64;

int stats_begin(int dev, cudaStream_t s, int batch, int groups, double** copies) {
  *copies = nullptr;
  const size_t bytes = static_cast<size_t>(kStatStripes) * batch * groups * 3 * sizeof(double);
  cudaMemPool_t pool = device_pool(dev);
  void* p = nullptr;
  if (pool_alloc(&p, bytes, pool, s) != cudaSuccess) {
    cudaGetLastError();
    return SMC_E_OOM;
  }
  if (cudaMemsetAsync(p, 0, bytes, s) != cudaSuccess) {
    cudaGetLastError();
    cudaFreeAsync(p, s);
    return SMC_E_CUDA;
  }
  *copies = static_cast<double*>(p);
  return SMC_OK;
}

int stats_end(double* copies, int batch, int groups, double* stats, cudaStream_t s, bool ok) {
  cudaError_t e = cudaSuccess;
  if (ok) e = smc::launch_stats_fold(copies, kStatStripes, static_cast<int64_t>(batch) * groups * 3, stats, s);
  cudaFreeAsync(copies, s);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return SMC_E_CUDA;
  }
  return SMC_OK;
}

}  // namespace

namespace smc {
void count_launches(int k) { g_launches.fetch_add(k, std::memory_order_relaxed); }
uint64_t scan_wait_limit_ns() { return static_cast<uint64_t>(g_wait_limit_ns.load()); }
int64_t scan_hold_ticket() { return g_scan_hold.load(); }
}  // namespace smc

extern "C" {

const char* smc_strerror(int code) {
  switch (code) {
    case SMC_OK: return "ok";
    case SMC_E_ARG: return "invalid argument";
    case SMC_E_RANGE: return "coordinate outside the grid or batch range";
    case SMC_E_DUPLICATE: return "duplicate coordinate";
    case SMC_E_DTYPE: return "unsupported dtype";
    case SMC_E_SHAPE: return "shape mismatch";
    case SMC_E_ALIAS: return "output overlaps an input";
    case SMC_E_CAPACITY: return "hash table capacity exhausted";
    case SMC_E_OOM: return "device allocation failed";
    case SMC_E_CUDA: return "CUDA error";
    case SMC_E_TIMEOUT: return "device-side wait timed out";
    case SMC_E_ALIGN: return "misaligned device pointer";
    default: return "unknown error";
  }
}

int smc_set_hash_capacity(int64_t slots) {
  if (slots < 0) return SMC_E_ARG;
  g_capacity_override.store(slots);
  return SMC_OK;
}

int smc_set_alloc_fail_after(int64_t k) {
  if (k < 0) return SMC_E_ARG;
  g_alloc_fail_after.store(k);
  return SMC_OK;
}

int smc_set_wait_limit_ns(int64_t ns) {
  if (ns < 0) return SMC_E_ARG;
  g_wait_limit_ns.store(ns == 0 ? static_cast<int64_t>(smc::kWaitLimitNs) : ns);
  return SMC_OK;
}

int smc_set_scan_hold(int64_t ticket) {
  if (ticket < -1) return SMC_E_ARG;
  g_scan_hold.store(ticket);
  return SMC_OK;
}

int smc_set_schedule_segment(int64_t rows) {
  if (rows == -1) rows = smc::kScheduleSegmentDefault;
  if (rows < 0 || rows % 2048 != 0) return SMC_E_ARG;
  smc::set_schedule_segment_rows(rows);
  return SMC_OK;
}

int smc_set_map_lookup(int32_t mode) {
  if (mode < 0 || mode > 3) return SMC_E_ARG;
  g_map_lookup.store(mode);
  return SMC_OK;
}

int smc_set_conv_priority(int32_t on) {
  if (on != 0 && on != 1) return SMC_E_ARG;
  g_conv_priority.store(on);
  return SMC_OK;
}

int smc_set_conv_epilogue(int32_t where) {
  if (where != 0 && where != 1) return SMC_E_ARG;
  smc::set_conv_epilogue(where);
  return SMC_OK;
}

int smc_set_conv_variant(int32_t variant) {
  if (variant < 0 || variant > 4) return SMC_E_ARG;
  smc::set_conv_variant(variant);
  return SMC_OK;
}

int smc_set_profiling(int32_t on) {
  g_profiling.store(on ? 1 : 0);
  return SMC_OK;
}

int smc_build_map_async(const int32_t* coords, int64_t n, int32_t batch, const int32_t grid[3], void* stream,
                        smc_map** out) {
  return build_async(coords, n, batch, grid, static_cast<cudaStream_t>(stream), out);
}

int smc_map_wait(const smc_map* map) {
  if (!map) return SMC_E_ARG;
  return resolve(map);
}

// Children of n parent rows (smc_subdivide, smc_upsample): per-parent child
// bits and counts, their scan, one host read of the total m, the children's
// coordinates in (parent, k) order (`order` as in launch_subdiv_emit), then
// the rows of `feats` copied to the children (when feats is given) and the
// children's map read off the parent map (when parent is given).
static int spawn_children(const smc_map* parent, const int32_t* coords, int64_t n, const uint8_t* keep, int order,
                   const void* feats, int64_t row_bytes, int elem_bytes, void* child_feats, int32_t* child_coords,
                   int64_t* m_out, cudaStream_t s, smc_map** child) {
  int32_t grid2[3] = {1, 1, 1};
  if (parent) {
    for (int i = 0; i < 3; ++i) {
      if (parent->grid[i] > (1 << 30) - 1) return SMC_E_ARG;
      grid2[i] = 2 * parent->grid[i];
    }
    const int rc = resolve(parent);  // the parent map must be complete (and sound)
    if (rc != SMC_OK) return rc;
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev != parent->device) return SMC_E_ARG;
  }
  if (n == 0) return parent ? build_async(nullptr, 0, parent->batch, grid2, s, child) : SMC_OK;
  if (pending_cuda_error() != SMC_OK) return SMC_E_CUDA;
  int dev = 0;
  cudaGetDevice(&dev);
  cudaMemPool_t pool = device_pool(dev);
  HostSlot* slot = take_slot();
  if (!pool || !slot) {
    give_slot(slot);
    return SMC_E_OOM;
  }
  // scratch: error word + ticket, scan statuses, list info, per-parent bits,
  // counts and first child, the parent-slot -> child-row remap, child sources
  Carve c;
  const size_t o_hdr = c.take<HostSlot>(1);
  const size_t o_tick = c.take<uint32_t>(1);
  const size_t o_st = c.take<unsigned long long>(smc::scan_status_len(n));
  const size_t zero_bytes = c.off - o_hdr;
  const size_t o_bits = c.take<uint8_t>(n);
  const size_t o_cnt = c.take<int32_t>(n);
  const size_t o_first = c.take<int64_t>(n);
  const size_t o_remap = c.take<int32_t>(8 * n);
  const size_t o_src = c.take<int32_t>(8 * n);
  void* sp = nullptr;
  if (pool_alloc(&sp, c.off, pool, s) != cudaSuccess) {
    cudaGetLastError();
    give_slot(slot);
    return SMC_E_OOM;
  }
  char* S = static_cast<char*>(sp);
  uint32_t* err = reinterpret_cast<uint32_t*>(S + o_hdr + offsetof(HostSlot, err));
  int64_t* info = reinterpret_cast<int64_t*>(S + o_hdr + offsetof(HostSlot, info));
  uint8_t* bits = reinterpret_cast<uint8_t*>(S + o_bits);
  int32_t* cnt = reinterpret_cast<int32_t*>(S + o_cnt);
  int64_t* first = reinterpret_cast<int64_t*>(S + o_first);
  int32_t* remap = reinterpret_cast<int32_t*>(S + o_remap);
  int32_t* src = reinterpret_cast<int32_t*>(S + o_src);
  // children per parent, then their first row; the total comes back to size the child map
  cudaError_t ce = cudaMemsetAsync(S + o_hdr, 0, zero_bytes, s);
  if (ce == cudaSuccess) ce = smc::launch_subdiv_count(keep, n, order, bits, cnt, s);
  if (ce == cudaSuccess)
    ce = smc::launch_scan_counts(cnt, n, first, reinterpret_cast<unsigned long long*>(S + o_st),
                                 reinterpret_cast<uint32_t*>(S + o_tick), err, info, n, s);
  if (ce == cudaSuccess) ce = cudaMemcpyAsync(slot, S + o_hdr, sizeof(HostSlot), cudaMemcpyDeviceToHost, s);
  if (ce == cudaSuccess) ce = cudaStreamSynchronize(s);
  const uint32_t scan_err = slot->err;
  const int64_t m = slot->info[27];
  give_slot(slot);
  int out = SMC_OK;
  if (ce != cudaSuccess) {
    cudaGetLastError();
    out = SMC_E_CUDA;
  } else if (scan_err & smc::kErrTimeout) {
    out = SMC_E_TIMEOUT;
  } else if (m < 0 || m > 8 * n) {
    out = SMC_E_CUDA;
  }
  if (out == SMC_OK) {
    ce = smc::launch_subdiv_emit(coords, n, order, bits, first, child_coords, src, remap, s);
    if (ce == cudaSuccess && feats)
      ce = smc::launch_expand_rows(feats, row_bytes, first, bits, n, child_feats, elem_bytes, s);
    if (ce != cudaSuccess) {
      cudaGetLastError();
      out = SMC_E_CUDA;
    }
  }
  if (out == SMC_OK && parent) {
    const SubdivSource sub{parent->nbr, src, remap};
    out = build_async(child_coords, m, parent->batch, grid2, s, child, &sub);
  }
  cudaFreeAsync(sp, s);  // after the child lookups, which read remap and src, in stream order
  cudaGetLastError();
  if (out == SMC_OK) *m_out = m;
  return out;
}

int smc_subdivide(const smc_map* parent, const int32_t* parent_coords, const uint8_t* keep, int32_t* child_coords,
                  int64_t* m_out, void* stream, smc_map** child) {
  if (!child || !m_out) return SMC_E_ARG;
  *child = nullptr;
  *m_out = 0;
  if (!parent) return SMC_E_ARG;
  const int64_t n = parent->n;
  if (n > 0 && (!parent_coords || !child_coords)) return SMC_E_ARG;
  if (n > 0 && ((reinterpret_cast<uintptr_t>(parent_coords) & 15u) || (reinterpret_cast<uintptr_t>(child_coords) & 15u)))
    return SMC_E_ALIGN;
  if (8 * n >= (1ll << 31) - 1) return SMC_E_ARG;  // child rows and parent slots are int32
  return spawn_children(parent, parent_coords, n, keep, 0, nullptr, 0, 0, nullptr, child_coords, m_out,
                        static_cast<cudaStream_t>(stream), child);
}

int smc_upsample(const int32_t* coords, int64_t n, const uint8_t* mask, const void* feats, int64_t c, int32_t dtype,
                 const smc_map* map, int32_t* child_coords, void* child_feats, int64_t* m_out, void* stream,
                 smc_map** child) {
  if (!m_out) return SMC_E_ARG;
  *m_out = 0;
  if (child) *child = nullptr;
  if (map && !child) return SMC_E_ARG;
  if (n < 0 || (map && map->n != n)) return SMC_E_ARG;
  if (8 * n >= (1ll << 31) - 1) return SMC_E_ARG;  // child rows and parent slots are int32
  int es = 0;
  if (feats) {
    if (dtype != SMC_F32 && dtype != SMC_BF16 && dtype != SMC_F16) return SMC_E_DTYPE;
    es = dtype == SMC_F32 ? 4 : 2;
    if (c < 1 || c > (1 << 24)) return SMC_E_SHAPE;
    if (n > 0 && !child_feats) return SMC_E_ARG;
    if ((reinterpret_cast<uintptr_t>(feats) | reinterpret_cast<uintptr_t>(child_feats)) & (es - 1)) return SMC_E_ALIGN;
    if (n > 0 && ranges_overlap(feats, static_cast<size_t>(n) * c * es, child_feats, 8ull * n * c * es))
      return SMC_E_ALIAS;
  }
  if (n > 0 && (!coords || !child_coords)) return SMC_E_ARG;
  if (n > 0 && ((reinterpret_cast<uintptr_t>(coords) & 15u) || (reinterpret_cast<uintptr_t>(child_coords) & 15u)))
    return SMC_E_ALIGN;
  return spawn_children(map, coords, n, mask, 1, feats, feats ? c * es : 0, es, child_feats, child_coords, m_out,
                        static_cast<cudaStream_t>(stream), child);
}

int smc_downsample(const int32_t* coords, int64_t n, int32_t batch, const int32_t grid[3], const void* feats,
                   int64_t c, int32_t dtype, int32_t mode, int32_t* parent_coords, void* parent_feats,
                   uint8_t* mask, int32_t* parent, int64_t* m_out, void* stream) {
  if (!m_out) return SMC_E_ARG;
  *m_out = 0;
  if (!grid || n < 0 || batch < 1 || grid[0] < 1 || grid[1] < 1 || grid[2] < 1) return SMC_E_ARG;
  if (mode != SMC_POOL_MAX && mode != SMC_POOL_MEAN) return SMC_E_ARG;
  if (n >= (1ll << 30)) return SMC_E_ARG;  // rows are int32, hash slots below 2^31
  if (n == 0) return SMC_OK;
  if ((feats == nullptr) != (parent_feats == nullptr)) return SMC_E_ARG;
  int es = 0;
  if (feats) {
    if (dtype != SMC_F32 && dtype != SMC_BF16 && dtype != SMC_F16) return SMC_E_DTYPE;
    es = dtype == SMC_F32 ? 4 : 2;
    if (c < 1 || c > (1 << 24)) return SMC_E_SHAPE;
    if ((reinterpret_cast<uintptr_t>(feats) | reinterpret_cast<uintptr_t>(parent_feats)) & (es - 1))
      return SMC_E_ALIGN;
    if (n > 0 && ranges_overlap(feats, static_cast<size_t>(n) * c * es, parent_feats, static_cast<size_t>(n) * c * es))
      return SMC_E_ALIAS;
  }
  if (!coords || !parent_coords || !mask) return SMC_E_ARG;
  if ((reinterpret_cast<uintptr_t>(coords) & 15u) || (reinterpret_cast<uintptr_t>(parent_coords) & 15u) ||
      (reinterpret_cast<uintptr_t>(mask) & 7u) || (reinterpret_cast<uintptr_t>(parent) & 3u))
    return SMC_E_ALIGN;
  const double psites = static_cast<double>(batch) * ((grid[0] + 1) / 2) * ((grid[1] + 1) / 2) * ((grid[2] + 1) / 2);
  if (psites >= 4.6e18) return SMC_E_ARG;
  if (pending_cuda_error() != SMC_OK) return SMC_E_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int dev = 0;
  cudaGetDevice(&dev);
  cudaMemPool_t pool = device_pool(dev);
  HostSlot* slot = take_slot();
  if (!pool || !slot) {
    give_slot(slot);
    return SMC_E_OOM;
  }
  // Parent lookup: a dense grid over the parent box (8 bytes a site) when it
  // holds at most 32 sites per row and 2^28 sites, else a hash at load <= 1/2.
  const int lookup = g_map_lookup.load();
  const bool dense = psites <= kDenseMaxSites && (lookup == 2 || (lookup == 0 && psites <= 32.0 * n));
  int lg = 4;
  while ((1ll << lg) < 2 * n) ++lg;
  const size_t slots = dense ? static_cast<size_t>(psites) : (size_t(1) << lg);
  Carve cv;
  const size_t o_hdr = cv.take<HostSlot>(1);
  const size_t o_tick = cv.take<uint32_t>(1);
  const size_t o_st = cv.take<unsigned long long>(smc::scan_status_len(n));
  const size_t o_bits = cv.take<uint32_t>(slots);
  const size_t zero_bytes = cv.off - o_hdr;
  const size_t o_first = cv.take<int32_t>(slots);
  const size_t o_keys = dense ? 0 : cv.take<unsigned long long>(slots);
  const size_t o_sor = cv.take<uint32_t>(n);
  const size_t o_flags = cv.take<int32_t>(n);
  const size_t o_pos = cv.take<int64_t>(n);
  const size_t o_rows = cv.take<int32_t>(8 * n);
  const size_t o_pbits = cv.take<uint8_t>(n);
  void* sp = nullptr;
  if (pool_alloc(&sp, cv.off, pool, s) != cudaSuccess) {
    cudaGetLastError();
    give_slot(slot);
    return SMC_E_OOM;
  }
  char* S = static_cast<char*>(sp);
  smc::DownArgs a{};
  a.coords = coords;
  a.n = n;
  a.batch = batch;
  a.Z = grid[0];
  a.Y = grid[1];
  a.X = grid[2];
  a.keys = dense ? nullptr : reinterpret_cast<unsigned long long*>(S + o_keys);
  a.lg = lg;
  a.first = reinterpret_cast<int32_t*>(S + o_first);
  a.bits = reinterpret_cast<uint32_t*>(S + o_bits);
  a.slot_of_row = reinterpret_cast<uint32_t*>(S + o_sor);
  a.flags = reinterpret_cast<int32_t*>(S + o_flags);
  a.pos = reinterpret_cast<int64_t*>(S + o_pos);
  a.scan_status = reinterpret_cast<unsigned long long*>(S + o_st);
  a.scan_ticket = reinterpret_cast<uint32_t*>(S + o_tick);
  a.err = reinterpret_cast<uint32_t*>(S + o_hdr + offsetof(HostSlot, err));
  a.info = reinterpret_cast<int64_t*>(S + o_hdr + offsetof(HostSlot, info));
  a.child_rows = reinterpret_cast<int32_t*>(S + o_rows);
  a.pbits = reinterpret_cast<uint8_t*>(S + o_pbits);
  a.parent_coords = parent_coords;
  a.mask = mask;
  a.parent = parent;
  a.feats = feats;
  a.out = parent_feats;
  a.c = static_cast<int>(c);
  a.dtype = dtype;
  a.mode = mode;
  cudaError_t ce = cudaMemsetAsync(S + o_hdr, 0, zero_bytes, s);
  if (ce == cudaSuccess) ce = cudaMemsetAsync(a.first, 0x7F, slots * sizeof(int32_t), s);
  if (ce == cudaSuccess && !dense) ce = cudaMemsetAsync(a.keys, 0xFF, slots * sizeof(unsigned long long), s);
  if (ce == cudaSuccess) ce = smc::launch_downsample(a, s);
  if (ce == cudaSuccess) ce = cudaMemcpyAsync(slot, S + o_hdr, sizeof(HostSlot), cudaMemcpyDeviceToHost, s);
  if (ce == cudaSuccess) ce = cudaStreamSynchronize(s);
  const uint32_t e = slot->err;
  const int64_t m = slot->info[27];
  give_slot(slot);
  cudaFreeAsync(sp, s);
  if (ce != cudaSuccess) {
    cudaGetLastError();
    return SMC_E_CUDA;
  }
  if (e & smc::kErrRange) return SMC_E_RANGE;
  if (e & smc::kErrDuplicate) return SMC_E_DUPLICATE;
  if (e & smc::kErrCapacity) return SMC_E_CAPACITY;
  if (e & smc::kErrTimeout) return SMC_E_TIMEOUT;
  if (m < 1 || m > n) return SMC_E_CUDA;
  *m_out = m;
  return SMC_OK;
}

int smc_group_stats(const void* x, int64_t n, int64_t c, const int32_t* coords, int32_t batch, int32_t groups,
                    double* stats, int32_t dtype, void* stream) {
  if (n < 0 || c < 1 || batch < 1 || groups < 1 || c % groups != 0) return SMC_E_ARG;
  if (dtype != SMC_F32 && dtype != SMC_BF16 && dtype != SMC_F16) return SMC_E_DTYPE;
  if (n == 0) return SMC_OK;
  if (!x || !coords || !stats) return SMC_E_ARG;
  if (static_cast<int64_t>(batch) * groups > 1024 || c > (1 << 24)) return SMC_E_SHAPE;
  if (pending_cuda_error() != SMC_OK) return SMC_E_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int dev = 0;
  cudaGetDevice(&dev);
  smc::Epilogue ep;
  ep.batch = batch;
  ep.groups = groups;
  ep.stripes = kStatStripes;
  const int rc = stats_begin(dev, s, batch, groups, &ep.stats);
  if (rc != SMC_OK) return rc;
  const cudaError_t e = smc::launch_group_stats(x, n, static_cast<int>(c), coords, ep, dtype, s);
  if (e != cudaSuccess) cudaGetLastError();
  const int rc2 = stats_end(ep.stats, batch, groups, stats, s, e == cudaSuccess);
  if (e != cudaSuccess) return SMC_E_CUDA;
  return rc2;
}

int smc_group_norm(const void* x, int64_t n, int64_t c, const int32_t* coords, int32_t batch, int32_t groups,
                   const double* stats, const void* gamma, const void* beta, float eps, int32_t act, void* out,
                   int32_t dtype, void* stream) {
  if (n < 0 || c < 1 || batch < 1 || groups < 1 || c % groups != 0 || !(eps >= 0.f)) return SMC_E_ARG;
  if (act != SMC_ACT_NONE && act != SMC_ACT_RELU && act != SMC_ACT_SILU) return SMC_E_ARG;
  if (dtype != SMC_F32 && dtype != SMC_BF16 && dtype != SMC_F16) return SMC_E_DTYPE;
  if (n == 0) return SMC_OK;
  if (!x || !coords || !stats || !out) return SMC_E_ARG;
  if (static_cast<int64_t>(batch) * groups > 1024 || c > (1 << 24)) return SMC_E_SHAPE;
  if (pending_cuda_error() != SMC_OK) return SMC_E_CUDA;
  if (smc::launch_group_norm(x, n, static_cast<int>(c), coords, batch, groups, stats, gamma, beta, eps, act, out,
                             dtype, static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return SMC_E_CUDA;
  }
  return SMC_OK;
}

int smc_map_stream_wait(const smc_map* map, void* stream) {
  if (!map) return SMC_E_ARG;
  if (!map->done) return SMC_OK;  // empty map: nothing was enqueued
  if (cudaStreamWaitEvent(static_cast<cudaStream_t>(stream), map->done, 0) != cudaSuccess) {
    cudaGetLastError();
    return SMC_E_CUDA;
  }
  return SMC_OK;
}

int smc_build_map(const int32_t* coords, int64_t n, int32_t batch, const int32_t grid[3], void* stream,
                  smc_map** out) {
  if (!out) return SMC_E_ARG;
  *out = nullptr;
  smc_map* m = nullptr;
  int rc = build_async(coords, n, batch, grid, static_cast<cudaStream_t>(stream), &m);
  if (rc != SMC_OK) return rc;
  rc = resolve(m);
  if (rc != SMC_OK) {
    release_map(m);
    return rc;
  }
  *out = m;
  return SMC_OK;
}

int smc_conv(const smc_map* map, const void* feats, int64_t cin, const void* weight, const void* bias,
             void* out, int64_t cout, int32_t ksize, int32_t orientation, int32_t dtype, void* stream) {
  return smc_conv_ex(map, feats, cin, weight, bias, nullptr, out, cout, ksize, orientation, dtype, SMC_ACT_NONE,
                     nullptr, nullptr, 1, stream);
}

int smc_conv_ex(const smc_map* map, const void* feats, int64_t cin, const void* weight, const void* bias,
                const void* residual, void* out, int64_t cout, int32_t ksize, int32_t orientation, int32_t dtype,
                int32_t act, const int32_t* coords, double* stats, int32_t groups, void* stream) {
  if (!map) return SMC_E_ARG;
  if (act != SMC_ACT_NONE && act != SMC_ACT_RELU && act != SMC_ACT_SILU) return SMC_E_ARG;
  if (stats && (!coords || groups < 1 || cout % groups != 0)) return SMC_E_ARG;
  if (ksize != 1 && ksize != 3) return SMC_E_ARG;
  if (orientation != 1 && orientation != -1) return SMC_E_ARG;
  if (dtype != SMC_F32 && dtype != SMC_BF16 && dtype != SMC_F16) return SMC_E_DTYPE;
  if (cin < 1 || cout < 1 || cin > (1 << 24) || cout > (1 << 24)) return SMC_E_SHAPE;
  const int64_t n = map->n;
  if (n == 0) return SMC_OK;
  if (!feats || !weight || !out) return SMC_E_ARG;
  {
    std::lock_guard<std::mutex> lk(map->mu);
    if (map->resolved && map->status != SMC_OK) return map->status;
  }
  const size_t esz = dtype == SMC_F32 ? 4 : 2;
  const int taps = ksize == 3 ? 27 : 1;
  // the residual may be the output itself (y = conv + out), not a part of it
  if (residual && residual != out && ranges_overlap(out, n * cout * esz, residual, n * cout * esz))
    return SMC_E_ALIAS;
  if (ranges_overlap(out, n * cout * esz, feats, n * cin * esz) ||
      ranges_overlap(out, n * cout * esz, weight, static_cast<size_t>(cout) * taps * cin * esz) ||
      ranges_overlap(out, n * cout * esz, bias, static_cast<size_t>(cout) * esz))
    return SMC_E_ALIAS;
  if (pending_cuda_error() != SMC_OK) return SMC_E_CUDA;
  int dev = 0;
  cudaGetDevice(&dev);
  uint32_t* st = device_status(dev);
  if (!st) return SMC_E_OOM;
  smc::ConvArgs a;
  a.feats = feats;
  a.weight = weight;
  a.bias = bias;
  a.out = out;
  a.nbr = map->nbr;
  a.perm = map->perm;
  a.tile_mask = map->tile_mask;
  a.n = n;
  a.cin = static_cast<int>(cin);
  a.cout = static_cast<int>(cout);
  a.taps = taps;
  a.orientation = orientation;
  a.dtype = dtype;
  a.err = st;
  a.ep.residual = residual;
  a.ep.act = act;
  if (stats && static_cast<int64_t>(map->batch) * groups > 1024) return SMC_E_SHAPE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dev != map->device) return SMC_E_ARG;
  a.in_idx = map->in_idx;
  a.out_idx = map->out_idx;
  a.pair_offsets = map->pair_offsets;
  const bool tc = smc::conv_tc_supported(a);
  const bool per_offset = tc && taps == 27 && smc::conv_variant() == 3;
  // The per-offset kernel reads the pair lists, which are built on the side
  // stream: it waits for the whole build even on the build stream.
  if ((s != map->stream || per_offset) && map->done && cudaStreamWaitEvent(s, map->done, 0) != cudaSuccess) {
    cudaGetLastError();
    return SMC_E_CUDA;
  }
  // The tensor-core kernel leaves activation and residual to a row pass
  // behind it (unless set to do them itself, or unless the residual is the
  // output buffer, which the conv overwrites: then its epilogue reads each
  // row's residual before storing the row); so do the statistics.
  const bool pass = tc && !per_offset && smc::conv_epilogue() == 0 && (act != SMC_ACT_NONE || residual) &&
                    residual != out;
  if (pass) {
    a.ep.residual = nullptr;
    a.ep.act = SMC_ACT_NONE;
  }
  // The conv runs on one of the library's streams of the greatest priority,
  // forked from the caller's stream and joined back to it (unless
  // smc_set_conv_priority(0)), so that its CTAs are dispatched before those
  // of work queued beside it.  Measured on B200 with steps pipelined over two
  // streams (the next step's map build beside this conv): 6-shell 128^3,
  // 0.117-0.123 -> 0.112-0.113 ms per step; the large maps even; one step
  // alone about 2 us longer (the fork and the join).
  cudaStream_t run = s;
  if (g_conv_priority.load() != 0) {
    cudaStream_t hp = prio_stream(dev);
    cudaEvent_t fork = hp ? take_event(dev) : nullptr;
    if (fork && cudaEventRecord(fork, s) == cudaSuccess && cudaStreamWaitEvent(hp, fork, 0) == cudaSuccess)
      run = hp;
    else
      cudaGetLastError();
    give_event(dev, fork);  // its wait is enqueued
  }
  auto launch = [&](cudaStream_t ls) -> int {
    cudaError_t e;
    if (per_offset) {
      void* acc = nullptr;
      cudaMemPool_t pool = device_pool(dev);
      if (pool_alloc(&acc, static_cast<size_t>(n) * cout * sizeof(float), pool, ls) != cudaSuccess) {
        cudaGetLastError();
        return SMC_E_OOM;
      }
      e = smc::launch_conv_offsets(a, static_cast<float*>(acc), ls);
      cudaFreeAsync(acc, ls);
    } else {
      e = tc ? smc::launch_conv_tc(a, ls) : smc::launch_conv_simt(a, ls);
    }
    if (e != cudaSuccess) {
      cudaGetLastError();
      return SMC_E_CUDA;
    }
    // Group statistics of the stored output: in the row pass, or a statistics
    // pass right behind the conv on the same stream (both measured faster than
    // folding them into the conv's epilogue, see conv_tc.cu).
    if (pass) {
      smc::Epilogue ep;
      ep.batch = map->batch;
      ep.groups = stats ? groups : 1;
      ep.stripes = kStatStripes;
      if (stats) {
        const int rc = stats_begin(dev, ls, map->batch, groups, &ep.stats);
        if (rc != SMC_OK) return rc;
      }
      e = smc::launch_rows_pass(out, out, residual, act, n, static_cast<int>(cout), coords, ep, dtype, ls);
      if (e != cudaSuccess) cudaGetLastError();
      const int rc2 = stats ? stats_end(ep.stats, map->batch, groups, stats, ls, e == cudaSuccess) : SMC_OK;
      if (e != cudaSuccess) return SMC_E_CUDA;
      return rc2;
    }
    if (stats) return smc_group_stats(out, n, cout, coords, map->batch, groups, stats, dtype, ls);
    return SMC_OK;
  };
  int rc = launch(run);
  if (run != s) {
    cudaEvent_t join = take_event(dev);
    if (!join || cudaEventRecord(join, run) != cudaSuccess || cudaStreamWaitEvent(s, join, 0) != cudaSuccess) {
      cudaGetLastError();
      cudaStreamSynchronize(run);  // no join event: the caller's stream must not run ahead of the conv
      if (rc == SMC_OK) rc = SMC_E_CUDA;
    }
    give_event(dev, join);
  }
  return rc;
}

int smc_map_info(const smc_map* map, int64_t* n, int64_t counts[27]) {
  if (!map) return SMC_E_ARG;
  const int rc = resolve(map);
  if (rc != SMC_OK) return rc;
  if (n) *n = map->n;
  if (counts)
    for (int d = 0; d < 27; ++d) counts[d] = map->counts[d];
  return SMC_OK;
}

int smc_map_nbr(const smc_map* map, const int32_t** nbr) {
  if (!map || !nbr) return SMC_E_ARG;
  *nbr = map->nbr;
  return SMC_OK;
}

int smc_map_pairs(const smc_map* map, const int32_t** in_idx, const int32_t** out_idx, int64_t offsets[28]) {
  if (!map) return SMC_E_ARG;
  const int rc = resolve(map);
  if (rc != SMC_OK) return rc;
  if (in_idx) *in_idx = map->in_idx;
  if (out_idx) *out_idx = map->out_idx;
  if (offsets)
    for (int d = 0; d < 28; ++d) offsets[d] = map->offsets[d];
  return SMC_OK;
}

int smc_map_schedule(const smc_map* map, const int32_t** perm) {
  if (!map || !perm) return SMC_E_ARG;
  *perm = map->perm;
  return SMC_OK;
}

int smc_kernel_launches(int64_t* count) {
  if (!count) return SMC_E_ARG;
  *count = g_launches.load();
  return SMC_OK;
}

int smc_map_timing(const smc_map* map, float ms[3]) {
  if (!map || !ms) return SMC_E_ARG;
  const int rc = resolve(map);
  if (rc != SMC_OK) return rc;
  ms[0] = map->ms[0];
  ms[1] = map->ms[1];
  ms[2] = map->ms[2];
  return SMC_OK;
}

int smc_free_map(smc_map* map) {
  if (!map) return SMC_OK;
  release_map(map);
  return SMC_OK;
}

int smc_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return SMC_E_CUDA;
  }
  int dev = 0;
  cudaGetDevice(&dev);
  uint32_t* st = device_status(dev);
  if (!st) return SMC_E_OOM;
  uint32_t h = 0;
  if (cudaMemcpy(&h, st, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return SMC_E_CUDA;
  if (h) cudaMemset(st, 0, sizeof(uint32_t));
  return (h & smc::kErrTimeout) ? SMC_E_TIMEOUT : SMC_OK;
}

}  // extern "C"
