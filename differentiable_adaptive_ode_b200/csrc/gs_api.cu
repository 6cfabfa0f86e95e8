// gs_api.cu -- the C ABI declared in include/gradsolve_b200.h: argument checks, record lifecycle,
// kernel launches.  Every entry point returns a status; nothing here aborts.
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <initializer_list>
#include <atomic>
#include <map>
#include <mutex>
#include <new>
#include <string>
#include <unordered_map>

#include "gradsolve_b200.h"
#include "gs_kernels.cuh"
#include "gs_mlp.cuh"

// NVTX range over one entry point (header-only NVTX v3): profilers show each library call as a
// named range around its kernels.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};

namespace {

thread_local std::string g_err;

gs_status fail(gs_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
gs_status fail(gs_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return s;
}

#define GS_CUDA(call)                                                                    \
  do {                                                                                   \
    cudaError_t e_ = (call);                                                             \
    if (e_ != cudaSuccess)                                                               \
      return fail(GS_ERR_CUDA, "%s failed: %s (%s:%d)", #call, cudaGetErrorString(e_),   \
                  __FILE__, __LINE__);                                                   \
  } while (0)

struct FieldInfo {
  int d, m;
  bool tsit5, ros;
};

bool field_info(int field, FieldInfo* fi) {
  switch (field) {
    case GS_LOTKA_VOLTERRA: *fi = {2, 4, true, false}; return true;
    case GS_LORENZ63: *fi = {3, 3, true, false}; return true;
    case GS_MLP_4_32_32_4: *fi = {4, 1348, true, false}; return true;
    case GS_ROBERTSON: *fi = {3, 3, false, true}; return true;
    case GS_NFW_MN: *fi = {6, 5, true, false}; return true;
    case GS_LINEAR: *fi = {3, 9, true, true}; return true;
    case GS_LOG_HALO: *fi = {6, 2, true, false}; return true;
    case GS_HIRES: *fi = {8, 12, false, true}; return true;
    default: return false;
  }
}

gs_status check_system(const gs_system* sys) {
  if (!sys) return fail(GS_ERR_INVALID_ARG, "gs_system pointer is NULL");
  FieldInfo fi;
  if (!field_info(sys->field, &fi)) return fail(GS_ERR_INVALID_ARG, "unknown field %d", sys->field);
  if (sys->dtype != GS_F64 && sys->dtype != GS_F32)
    return fail(GS_ERR_INVALID_ARG, "unknown dtype %d", sys->dtype);
  if (sys->method != GS_TSIT5 && sys->method != GS_ROS34PW2 && sys->method != GS_VERN7 &&
      sys->method != GS_ROSENBROCK23)
    return fail(GS_ERR_INVALID_ARG, "unknown method %d", sys->method);
  if (sys->d != fi.d || sys->m != fi.m)
    return fail(GS_ERR_INVALID_ARG, "field %d has d=%d m=%d, got d=%d m=%d", sys->field, fi.d,
                fi.m, sys->d, sys->m);
  if (((sys->method == GS_TSIT5 || sys->method == GS_VERN7) && !fi.tsit5) ||
      ((sys->method == GS_ROS34PW2 || sys->method == GS_ROSENBROCK23) && !fi.ros) ||
      (sys->method == GS_VERN7 && sys->field == GS_MLP_4_32_32_4))
    return fail(GS_ERR_UNSUPPORTED, "field %d is not built for method %d", sys->field, sys->method);
  if (sys->theta_shared != 0 && sys->theta_shared != 1)
    return fail(GS_ERR_INVALID_ARG, "theta_shared must be 0 or 1");
  if (sys->field == GS_MLP_4_32_32_4 && !sys->theta_shared)
    return fail(GS_ERR_UNSUPPORTED, "the MLP field takes one weight vector shared by the ensemble");
  return GS_OK;
}

// Per-device library state, created on first use and kept until exit: the SM count, a ring of
// work-queue counters (each call takes its own slot, zeroes it on its stream and hands it to its
// kernel, so calls on different streams never share a counter), cached occupancy figures, and
// the cache of record storage: blocks released by records (destroyed, or regrown) are kept here
// for the next records instead of going back to the driver, so that a new record costs no
// allocation and destroying one no cudaFree (about 6 ms for 12 GB), until gs_memory_trim hands
// them back.  New storage comes from cudaMalloc (about 2 ms for 12 GB; a stream-ordered memory
// pool took 83 ms to grow by the same amount the first time, measured on B200).
struct DeviceCtx {
  std::once_flag once;
  cudaError_t init_err = cudaSuccess;
  int sms = 148;
  int* ring = nullptr;
  std::atomic<unsigned> next{0};
  std::mutex occ_mu;
  std::unordered_map<const void*, int> occ;
  std::mutex mem_mu;
  std::multimap<size_t, void*> cached;      // released blocks by size
  std::unordered_map<void*, size_t> sizes;  // every block handed out or cached, by address
  size_t cached_bytes = 0;
  size_t total_mem = 0;                     // device memory, read once
};
constexpr int MAX_DEVICES = 64;
constexpr unsigned RING = 4096;
DeviceCtx g_dev[MAX_DEVICES];

DeviceCtx* device_ctx(cudaError_t* err) {
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= MAX_DEVICES) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  DeviceCtx& c = g_dev[dev];
  std::call_once(c.once, [&]() {
    c.init_err = cudaDeviceGetAttribute(&c.sms, cudaDevAttrMultiProcessorCount, dev);
    if (c.init_err == cudaSuccess) c.init_err = cudaMalloc(&c.ring, RING * sizeof(int));
    size_t free_b = 0;
    if (c.init_err == cudaSuccess && cudaMemGetInfo(&free_b, &c.total_mem) != cudaSuccess) {
      cudaGetLastError();
      c.total_mem = 0;
    }
  });
  *err = c.init_err;
  return c.init_err == cudaSuccess ? &c : nullptr;
}

// Hands cached blocks back to the driver until at most `keep` bytes stay cached (largest first).
cudaError_t release_cached(DeviceCtx* c, size_t keep) {
  std::lock_guard<std::mutex> lk(c->mem_mu);
  cudaError_t e = cudaSuccess;
  while (c->cached_bytes > keep && !c->cached.empty()) {
    auto it = std::prev(c->cached.end());
    const cudaError_t f = cudaFree(it->second);
    if (f != cudaSuccess) e = f;
    c->cached_bytes -= it->first;
    c->sizes.erase(it->second);
    c->cached.erase(it);
  }
  return e;
}

// Device storage of a record, usable by any stream: the smallest cached block that holds `bytes`
// without wasting more than half of itself, else new storage from cudaMalloc (after handing the
// cache back to the driver if the device is out of memory).
template <class T>
cudaError_t dalloc(T** p, size_t bytes, cudaStream_t) {
  cudaError_t e;
  DeviceCtx* c = device_ctx(&e);
  if (!c) return e;
  bytes = std::max<size_t>(bytes, 256);
  {
    std::lock_guard<std::mutex> lk(c->mem_mu);
    auto it = c->cached.lower_bound(bytes);
    if (it != c->cached.end() && it->first <= 2 * bytes) {
      *p = static_cast<T*>(it->second);
      c->cached_bytes -= it->first;
      c->cached.erase(it);
      return cudaSuccess;
    }
  }
  void* q = nullptr;
  e = cudaMalloc(&q, bytes);
  if (e == cudaErrorMemoryAllocation) {
    cudaGetLastError();  // clear the error before trying again
    release_cached(c, 0);
    e = cudaMalloc(&q, bytes);
  }
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(c->mem_mu);
  c->sizes[q] = bytes;
  *p = static_cast<T*>(q);
  return cudaSuccess;
}

// A zeroed work counter for one launch on stream s.
cudaError_t take_counter(cudaStream_t s, int** out) {
  cudaError_t e;
  DeviceCtx* c = device_ctx(&e);
  if (!c) return e;
  int* p = c->ring + (c->next.fetch_add(1) % RING);
  *out = p;
  return cudaMemsetAsync(p, 0, sizeof(int), s);
}

constexpr int BLOCK = 128;

template <class K>
int persistent_grid(K kernel, size_t smem, long long N) {
  cudaError_t e;
  DeviceCtx* c = device_ctx(&e);
  const int sms = c ? c->sms : 148;
  int nb = 0;
  const void* key = reinterpret_cast<const void*>(kernel);
  if (c) {
    std::lock_guard<std::mutex> lk(c->occ_mu);
    auto it = c->occ.find(key);
    if (it != c->occ.end()) nb = it->second;
  }
  if (nb == 0) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kernel, BLOCK, smem) != cudaSuccess ||
        nb < 1)
      nb = 1;
    if (c) {
      std::lock_guard<std::mutex> lk(c->occ_mu);
      c->occ[key] = nb;
    }
  }
  const long long g = (long long)sms * nb;
  const long long need = (N + BLOCK - 1) / BLOCK;
  return (int)std::max(1LL, std::min(g, need));
}

}  // namespace

// ------------------------------------------------------------------------------------------------
// Record object.
// ------------------------------------------------------------------------------------------------
struct gs_record {
  gs_system sys{};
  int64_t N = 0;
  int device = 0;
  int C = 0, E = 0;
  size_t rsz = 0;
  double t0 = 0, t1 = 0;
  // step pool
  void* pool = nullptr;
  int64_t pool_chunks = 0;
  int* chunk_traj = nullptr;
  int* chunk_seq = nullptr;
  int* chunk_table = nullptr;
  int64_t chunk_arrays_cap = 0;
  // per trajectory
  int64_t n_cap = 0;
  int* nsteps = nullptr;
  int* status = nullptr;
  long long* offsets = nullptr;
  long long* choff = nullptr;
  long long* tiles = nullptr;  // scan scratch (tile totals) + grand totals
  int* counters = nullptr;     // [0] queue [1] chunk count [2] parked [3] max S [4] max status
  int host[16] = {};           // read-back of counters, then offsets[N] at host+8
  // trajectories parked by a record pass (the pool ran out, or their first slice was done): their
  // ids, their states, and their order for the next pass
  int* park_list = nullptr;
  int* park_key = nullptr;       // estimated remaining steps of each parked trajectory
  int* park_order = nullptr;     // the parked trajectories by decreasing estimate
  void* park_r = nullptr;
  int* park_i = nullptr;
  long long* park_att = nullptr;
  int64_t park_n = 0;
  size_t park_r_bytes = 0;
  // visiting order of the replay kernels (longest records first) and its counting-sort scratch
  int* perm = nullptr;
  int64_t perm_cap = 0;
  int64_t perm_n = 0;   // ensemble size the current perm was built for (0: none)
  int* bins = nullptr;          // [nb] counts, then [nb] cursors
  long long* binoff = nullptr;  // [nb + 1]
  long long* btiles = nullptr;
  int64_t bins_cap = 0;
  // scratch of the replay calls (grown on demand; calls on one record are stream-ordered)
  void* red_scratch = nullptr;   // per-trajectory theta-bar [N][m] for a shared theta
  void* red_partials = nullptr;  // block partials of the reduction
  size_t red_bytes = 0, part_bytes = 0;
  void* y1_scratch = nullptr;    // y_S of gs_replay_forward when the caller passes no y1
  size_t y1_bytes = 0;
  // the theta the stored states y_n were computed at ([N][m], or [m] when shared); counters[8]
  // is the flag the device comparison with a caller's theta raises
  void* theta_kept = nullptr;
  size_t theta_kept_bytes = 0;
  bool theta_known = false;      // false after an import: the first use replays the states
  // device time of the solve kernel of the last record pass
  cudaEvent_t ev0 = nullptr, ev1 = nullptr;
  double solve_ms = 0;
  // summary
  int64_t nchunks = 0, total_steps = 0;
  int max_steps = 0;
};

namespace {

// Returns record storage to the device's cache.  The device is synchronised first (as cudaFree
// would): no queued work may still use a block that the next record could take.
void free_ptr(void* p, cudaStream_t) {
  if (!p) return;
  cudaError_t e;
  DeviceCtx* c = device_ctx(&e);
  if (!c) return;
  cudaDeviceSynchronize();
  std::lock_guard<std::mutex> lk(c->mem_mu);
  auto it = c->sizes.find(p);
  if (it == c->sizes.end()) {  // not a block of this device's cache
    cudaFree(p);
    return;
  }
  c->cached.emplace(it->second, p);
  c->cached_bytes += it->second;
}

gs_status ensure_traj_arrays(gs_record* r, int64_t N, cudaStream_t s) {
  if (r->n_cap >= N && r->counters) return GS_OK;
  free_ptr(r->nsteps, s); free_ptr(r->status, s); free_ptr(r->offsets, s); free_ptr(r->choff, s);
  free_ptr(r->tiles, s);
  r->nsteps = r->status = nullptr;
  r->offsets = r->choff = r->tiles = nullptr;
  const int64_t n = std::max<int64_t>(N, 1);
  const int64_t ntiles = (n + gs::SCAN_BLOCK - 1) / gs::SCAN_BLOCK;
  GS_CUDA(dalloc(&r->nsteps, n * sizeof(int), s));
  GS_CUDA(dalloc(&r->status, n * sizeof(int), s));
  GS_CUDA(dalloc(&r->offsets, (n + 1) * sizeof(long long), s));
  GS_CUDA(dalloc(&r->choff, (n + 1) * sizeof(long long), s));
  GS_CUDA(dalloc(&r->tiles, 2 * (ntiles + 2) * sizeof(long long), s));  // two scans side by side
  if (!r->counters) GS_CUDA(dalloc(&r->counters, 16 * sizeof(int), s));
  r->n_cap = n;
  return GS_OK;
}

gs_status ensure_park(gs_record* r, int64_t N, cudaStream_t s) {
  const int64_t n = std::max<int64_t>(N, 1);
  const size_t rb = (size_t)n * (2 + 2 * r->sys.d) * r->rsz;
  if (r->park_n >= n && r->park_r_bytes >= rb) return GS_OK;
  free_ptr(r->park_list, s); free_ptr(r->park_r, s);
  free_ptr(r->park_i, s); free_ptr(r->park_att, s); free_ptr(r->park_key, s);
  free_ptr(r->park_order, s);
  r->park_list = nullptr;
  r->park_key = r->park_order = nullptr;
  r->park_r = nullptr;
  r->park_i = nullptr;
  r->park_att = nullptr;
  r->park_n = 0;
  r->park_r_bytes = 0;
  GS_CUDA(dalloc(&r->park_list, n * sizeof(int), s));
  GS_CUDA(dalloc(&r->park_r, rb, s));
  GS_CUDA(dalloc(&r->park_i, n * 4 * sizeof(int), s));
  GS_CUDA(dalloc(&r->park_att, n * sizeof(long long), s));
  GS_CUDA(dalloc(&r->park_key, n * sizeof(int), s));
  GS_CUDA(dalloc(&r->park_order, n * sizeof(int), s));
  r->park_n = n;
  r->park_r_bytes = rb;
  return GS_OK;
}

// Enlarges the pool to `chunks`, keeping the first `keep` chunks (entries and labels).
gs_status grow_pool(gs_record* r, int64_t chunks, int64_t keep, cudaStream_t s) {
  if (chunks > 0x7fffffffLL)
    return fail(GS_ERR_CAPACITY, "record needs %lld chunks, more than 2^31-1", (long long)chunks);
  const size_t cb = (size_t)r->C * r->E * r->rsz;
  void* pool = nullptr;
  int *traj = nullptr, *seq = nullptr, *table = nullptr;
  auto undo = [&]() {
    free_ptr(pool, s); free_ptr(traj, s); free_ptr(seq, s); free_ptr(table, s);
  };
  if (dalloc(&pool, (size_t)chunks * cb, s) != cudaSuccess ||
      dalloc(&traj, chunks * sizeof(int), s) != cudaSuccess ||
      dalloc(&seq, chunks * sizeof(int), s) != cudaSuccess ||
      dalloc(&table, chunks * sizeof(int), s) != cudaSuccess) {
    undo();
    return fail(GS_ERR_CUDA, "cannot grow the record pool to %lld chunks", (long long)chunks);
  }
  if (keep > 0 &&
      (cudaMemcpyAsync(pool, r->pool, (size_t)keep * cb, cudaMemcpyDeviceToDevice, s) != cudaSuccess ||
       cudaMemcpyAsync(traj, r->chunk_traj, keep * sizeof(int), cudaMemcpyDeviceToDevice, s) !=
           cudaSuccess ||
       cudaMemcpyAsync(seq, r->chunk_seq, keep * sizeof(int), cudaMemcpyDeviceToDevice, s) !=
           cudaSuccess)) {
    undo();
    return fail(GS_ERR_CUDA, "record pool copy failed");
  }
  free_ptr(r->pool, s); free_ptr(r->chunk_traj, s); free_ptr(r->chunk_seq, s);
  free_ptr(r->chunk_table, s);
  r->pool = pool;
  r->chunk_traj = traj;
  r->chunk_seq = seq;
  r->chunk_table = table;
  r->pool_chunks = r->chunk_arrays_cap = chunks;
  return GS_OK;
}

gs_status ensure_pool(gs_record* r, int64_t chunks, cudaStream_t s) {
  if (chunks > 0x7fffffffLL)
    return fail(GS_ERR_CAPACITY, "record needs %lld chunks, more than 2^31-1", (long long)chunks);
  if (r->pool_chunks >= chunks && r->chunk_arrays_cap >= chunks) return GS_OK;
  free_ptr(r->pool, s); free_ptr(r->chunk_traj, s); free_ptr(r->chunk_seq, s);
  free_ptr(r->chunk_table, s);
  r->pool = nullptr;
  r->chunk_traj = r->chunk_seq = r->chunk_table = nullptr;
  r->pool_chunks = r->chunk_arrays_cap = 0;
  const int64_t c = std::max<int64_t>(chunks, 1);
  GS_CUDA(dalloc(&r->pool, (size_t)c * r->C * r->E * r->rsz, s));
  GS_CUDA(dalloc(&r->chunk_traj, c * sizeof(int), s));
  GS_CUDA(dalloc(&r->chunk_seq, c * sizeof(int), s));
  GS_CUDA(dalloc(&r->chunk_table, c * sizeof(int), s));
  r->pool_chunks = r->chunk_arrays_cap = c;
  return GS_OK;
}

// exclusive scan of nsteps (MODE 0) or chunk counts (MODE 1) into out[0..N]
// Allocated sizes of a record's pool and chunk table (bounds of the checked build).
gs::RecBounds bounds_of(const gs_record* r) {
  return gs::RecBounds{(long long)r->chunk_arrays_cap, (long long)r->pool_chunks};
}

// The summary of a record pass: step offsets, chunk offsets, the largest step count and status
// (into counters[3] and counters[4], zeroed by the caller) in three kernels.
gs_status summarise_pass(gs_record* r, const int* status, int N, int C, cudaStream_t st) {
  const int ntiles = (N + gs::SCAN_BLOCK - 1) / gs::SCAN_BLOCK;
  gs::k_summary_tiles<<<ntiles, gs::SCAN_BLOCK, 0, st>>>(r->nsteps, status, N, C, r->offsets,
                                                         r->choff, r->tiles, r->counters + 3);
  gs::k_summary_totals<<<1, gs::SCAN_BLOCK, 0, st>>>(r->tiles, ntiles);
  gs::k_summary_add<<<(N + 255) / 256, 256, 0, st>>>(r->offsets, r->choff, N, r->tiles, ntiles);
  GS_CUDA(cudaGetLastError());
  return GS_OK;
}

template <int MODE>
gs_status scan_counts(const int* S, int N, int C, long long* out, long long* tiles,
                      cudaStream_t st) {
  const int ntiles = (N + gs::SCAN_BLOCK - 1) / gs::SCAN_BLOCK;
  gs::k_scan_tiles<MODE><<<ntiles, gs::SCAN_BLOCK, 0, st>>>(S, N, C, out, tiles);
  gs::k_scan_totals<<<1, gs::SCAN_BLOCK, 0, st>>>(tiles, ntiles, tiles + ntiles);
  gs::k_scan_add<<<(N + 255) / 256, 256, 0, st>>>(out, N, tiles, tiles + ntiles);
  GS_CUDA(cudaGetLastError());
  return GS_OK;
}

// out[j] = the j-th of the n entries of keys (values in [0, kmax]) in decreasing order: the
// entry's index, or ids[index] when ids is given.  Counting sort in the record's bin scratch.
gs_status counting_sort_desc(gs_record* r, const int* keys, int64_t n, int kmax, const int* ids,
                             int* out, cudaStream_t s) {
  if (n <= 0) return GS_OK;
  const int64_t nb = (int64_t)kmax + 1;
  if (r->bins_cap < nb) {
    free_ptr(r->bins, s); free_ptr(r->binoff, s); free_ptr(r->btiles, s);
    r->bins = nullptr; r->binoff = r->btiles = nullptr;
    r->bins_cap = 0;
    GS_CUDA(dalloc(&r->bins, 2 * nb * sizeof(int), s));
    GS_CUDA(dalloc(&r->binoff, (nb + 1) * sizeof(long long), s));
    GS_CUDA(dalloc(&r->btiles, (nb / gs::SCAN_BLOCK + 3) * sizeof(long long), s));
    r->bins_cap = nb;
  }
  GS_CUDA(cudaMemsetAsync(r->bins, 0, 2 * nb * sizeof(int), s));
  // up to 4,097 bins a block keeps its own histogram in shared memory (32 KB for the scatter)
  const bool small = nb <= 4097;
  const int threads = small ? 1024 : 256;
  const int grid = (int)((n + threads - 1) / threads);
  if (small)
    gs::k_bin_count_smem<<<grid, threads, nb * sizeof(int), s>>>(keys, (int)n, kmax, r->bins);
  else
    gs::k_bin_count<<<grid, threads, 0, s>>>(keys, (int)n, kmax, r->bins);
  if (small) {
    gs::k_scan_one_block<<<1, gs::SCAN_BLOCK, 0, s>>>(r->bins, (int)nb, r->binoff);
    GS_CUDA(cudaGetLastError());
  } else {
    gs_status st = scan_counts<0>(r->bins, (int)nb, 1, r->binoff, r->btiles, s);
    if (st != GS_OK) return st;
  }
  if (small)
    gs::k_bin_scatter_smem<<<grid, threads, 2 * nb * sizeof(int), s>>>(keys, (int)n, kmax,
                                                                      r->binoff, r->bins + nb,
                                                                      out, ids);
  else
    gs::k_bin_scatter<<<grid, threads, 0, s>>>(keys, (int)n, kmax, r->binoff, r->bins + nb, out,
                                               ids);
  GS_CUDA(cudaGetLastError());
  return GS_OK;
}

// perm = trajectories by decreasing S (needs r->nsteps, r->max_steps).
gs_status build_perm(gs_record* r, cudaStream_t s) {
  const int64_t N = r->N;
  if (N <= 0) return GS_OK;
  if (r->perm_cap < N) {
    free_ptr(r->perm, s);
    r->perm = nullptr;
    r->perm_cap = 0;
    GS_CUDA(dalloc(&r->perm, N * sizeof(int), s));
    r->perm_cap = N;
  }
  gs_status st = counting_sort_desc(r, r->nsteps, N, r->max_steps, nullptr, r->perm, s);
  if (st != GS_OK) return st;
  r->perm_n = N;
  return GS_OK;
}

// ------------------------------------------------------------------------------------------------
// Typed launchers.
// ------------------------------------------------------------------------------------------------
struct SolveCall {
  int64_t N;
  const void* theta;
  int theta_shared;
  const void* y0;
  double t0, t1, rtol, atol;
  long long max_attempts;
  void* y1;
  int* nsteps;
  int* nrejected;
  int* status;
  int* queue;
  gs_record* rec;  // non-null: record pass
  cudaStream_t stream;
  const void* sens0 = nullptr;  // forward sensitivities (Tsit5 forward solve only)
  void* sens1 = nullptr;
  const int* order = nullptr;   // visiting order of the trajectories (null: index order)
  int64_t nqueue = -1;          // queue positions to visit (-1: N)
  int resume = 0;               // record pass resuming the trajectories listed in `order`
  int slice = 0;                // record pass: attempts per trajectory before it is parked (0: all)
};

template <class F, class R, int METHOD>
gs_status launch_solve(const SolveCall& c) {
  gs::SolveParams<R> p{};
  p.N = (int)c.N;
  p.theta = static_cast<const R*>(c.theta);
  p.theta_stride = c.theta_shared ? 0 : F::M;
  p.y0 = static_cast<const R*>(c.y0);
  p.t0 = R(c.t0); p.t1 = R(c.t1); p.rtol = R(c.rtol); p.atol = R(c.atol);
  p.max_attempts = c.max_attempts;
  p.y1 = static_cast<R*>(c.y1);
  p.nsteps = c.nsteps;
  p.nrejected = c.nrejected;
  p.status = c.status;
  p.queue = c.queue;
  p.order = c.order;
  p.nqueue = (int)(c.nqueue < 0 ? c.N : c.nqueue);
  if (c.rec) {
    p.pool = static_cast<R*>(c.rec->pool);
    p.chunk_traj = c.rec->chunk_traj;
    p.chunk_seq = c.rec->chunk_seq;
    p.pool_chunks = (int)c.rec->pool_chunks;
    p.chunk_count = c.rec->counters + 1;
    p.park_count = c.rec->counters + 2;
    p.park_list = c.rec->park_list;
    p.park_r = static_cast<R*>(c.rec->park_r);
    p.park_i = c.rec->park_i;
    p.park_att = c.rec->park_att;
    p.resume = c.resume;
    p.slice = c.slice;
  }
  if constexpr (std::is_same_v<F, gs::FMlpWarp>) {
    if (c.rec) {
      auto kern = gs::k_solve_mlp<R, true>;
      kern<<<persistent_grid(kern, 0, (long long)p.nqueue * 32), BLOCK, 0, c.stream>>>(p);
    } else {
      auto kern = gs::k_solve_mlp<R, false>;
      kern<<<persistent_grid(kern, 0, c.N * 32), BLOCK, 0, c.stream>>>(p);
    }
    GS_CUDA(cudaGetLastError());
    return GS_OK;
  } else {
    if (c.rec) {
      const size_t smem = gs::solve_smem_bytes<F, R, true>();
      auto kern = gs::k_solve<F, R, METHOD, true>;
      GS_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
      const int grid = persistent_grid(kern, smem, p.nqueue);
      kern<<<grid, BLOCK, smem, c.stream>>>(p);
    } else if (c.sens1) {
      if constexpr (METHOD == gs::M_TSIT5) {
        p.sens0 = static_cast<const R*>(c.sens0);
        p.sens1 = static_cast<R*>(c.sens1);
        auto kern = gs::k_solve<F, R, METHOD, false, true>;
        const size_t smem = gs::solve_smem_bytes<F, R, false, true>();
        GS_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
        const int grid = persistent_grid(kern, smem, c.N);
        kern<<<grid, BLOCK, smem, c.stream>>>(p);
      } else {
        return fail(GS_ERR_UNSUPPORTED, "forward sensitivities are built for Tsit5 only");
      }
    } else {
      auto kern = gs::k_solve<F, R, METHOD, false>;
      const size_t smem = gs::solve_smem_bytes<F, R, false>();
      GS_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
      const int grid = persistent_grid(kern, smem, c.N);
      kern<<<grid, BLOCK, smem, c.stream>>>(p);
    }
    GS_CUDA(cudaGetLastError());
    return GS_OK;
  }
}

// Dynamic shared memory of the adjoint kernel: the per-lane stage tape of fields with TAPE > 0
// (6 stages for Tsit5, 9 for Verner 7, x TAPE reals x 128 lanes).
template <class F, class R, int METHOD>
constexpr size_t adjoint_smem() {
  if constexpr (std::is_same_v<F, gs::FMlpWarp>) return 0;
  else return (size_t)(METHOD == gs::M_VERN7 ? 9 : 6) * gs::TapeOf<F>::value * BLOCK * sizeof(R);
}

struct AdjCall {
  const gs_record* rec;
  const void* theta;
  const void* dL_dy1;
  void* dL_dy0;
  void* dL_dtheta_traj;  // [N][M] (may be scratch)
  int* queue;
  cudaStream_t stream;
};

template <class F, class R, int METHOD>
gs_status launch_adjoint(const AdjCall& c) {
  if constexpr (std::is_same_v<F, gs::FMlpWarp>) {
    return fail(GS_ERR_UNSUPPORTED, "the MLP field has its own adjoint launcher");
  } else {
  gs::AdjointParams<R> p{};
  const gs_record* r = c.rec;
  p.N = (int)r->N;
  p.theta = static_cast<const R*>(c.theta);
  p.theta_stride = r->sys.theta_shared ? 0 : F::M;
  p.dL_dy1 = static_cast<const R*>(c.dL_dy1);
  p.dL_dy0 = static_cast<R*>(c.dL_dy0);
  p.dL_dtheta = static_cast<R*>(c.dL_dtheta_traj);
  p.nsteps = r->nsteps;
  p.choff = r->choff;
  p.chunk_table = r->chunk_table;
  p.pool = static_cast<const R*>(r->pool);
  p.queue = c.queue;
  p.perm = r->perm;
  p.bounds = bounds_of(r);
  auto kern = gs::k_adjoint<F, R, METHOD>;
  const size_t smem = adjoint_smem<F, R, METHOD>();
  if (smem > 48 * 1024)
    GS_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  const int grid = persistent_grid(kern, smem, r->N);
  kern<<<grid, BLOCK, smem, c.stream>>>(p);
  GS_CUDA(cudaGetLastError());
  return GS_OK;
  }
}

template <class F, class R>
void layout_of(int* C, int* E) {
  *C = gs::RecLayout<F, R>::C;
  *E = gs::RecLayout<F, R>::E;
}

// Dispatch over (field, method, dtype) for the combinations that are built.
template <class Fn>
gs_status dispatch(const gs_system& s, Fn&& fn) {
  const bool f64 = s.dtype == GS_F64;
  using namespace gs;
  if (s.method == GS_TSIT5) {
    switch (s.field) {
      case GS_LOTKA_VOLTERRA:
        return f64 ? fn.template operator()<FLotkaVolterra, double, M_TSIT5>()
                   : fn.template operator()<FLotkaVolterra, float, M_TSIT5>();
      case GS_LORENZ63:
        return f64 ? fn.template operator()<FLorenz63, double, M_TSIT5>()
                   : fn.template operator()<FLorenz63, float, M_TSIT5>();
      case GS_NFW_MN:
        return f64 ? fn.template operator()<FNfwMiyamotoNagai, double, M_TSIT5>()
                   : fn.template operator()<FNfwMiyamotoNagai, float, M_TSIT5>();
      case GS_LINEAR:
        return f64 ? fn.template operator()<FLinear3, double, M_TSIT5>()
                   : fn.template operator()<FLinear3, float, M_TSIT5>();
      case GS_LOG_HALO:
        return f64 ? fn.template operator()<FLogHalo, double, M_TSIT5>()
                   : fn.template operator()<FLogHalo, float, M_TSIT5>();
      case GS_MLP_4_32_32_4:
        return f64 ? fn.template operator()<FMlpWarp, double, M_TSIT5>()
                   : fn.template operator()<FMlpWarp, float, M_TSIT5>();
      default: break;
    }
  } else if (s.method == GS_VERN7) {
    switch (s.field) {
      case GS_LOTKA_VOLTERRA:
        return f64 ? fn.template operator()<FLotkaVolterra, double, M_VERN7>()
                   : fn.template operator()<FLotkaVolterra, float, M_VERN7>();
      case GS_LORENZ63:
        return f64 ? fn.template operator()<FLorenz63, double, M_VERN7>()
                   : fn.template operator()<FLorenz63, float, M_VERN7>();
      case GS_NFW_MN:
        return f64 ? fn.template operator()<FNfwMiyamotoNagai, double, M_VERN7>()
                   : fn.template operator()<FNfwMiyamotoNagai, float, M_VERN7>();
      case GS_LINEAR:
        return f64 ? fn.template operator()<FLinear3, double, M_VERN7>()
                   : fn.template operator()<FLinear3, float, M_VERN7>();
      case GS_LOG_HALO:
        return f64 ? fn.template operator()<FLogHalo, double, M_VERN7>()
                   : fn.template operator()<FLogHalo, float, M_VERN7>();
      default: break;
    }
  } else if (s.method == GS_ROSENBROCK23) {
    switch (s.field) {
      case GS_ROBERTSON:
        return f64 ? fn.template operator()<FRobertson, double, M_RB23>()
                   : fn.template operator()<FRobertson, float, M_RB23>();
      case GS_HIRES:
        return f64 ? fn.template operator()<FHires, double, M_RB23>()
                   : fn.template operator()<FHires, float, M_RB23>();
      case GS_LINEAR:
        return f64 ? fn.template operator()<FLinear3, double, M_RB23>()
                   : fn.template operator()<FLinear3, float, M_RB23>();
      default: break;
    }
  } else {
    switch (s.field) {
      case GS_ROBERTSON:
        return f64 ? fn.template operator()<FRobertson, double, M_ROS>()
                   : fn.template operator()<FRobertson, float, M_ROS>();
      case GS_HIRES:
        return f64 ? fn.template operator()<FHires, double, M_ROS>()
                   : fn.template operator()<FHires, float, M_ROS>();
      case GS_LINEAR:
        return f64 ? fn.template operator()<FLinear3, double, M_ROS>()
                   : fn.template operator()<FLinear3, float, M_ROS>();
      default: break;
    }
  }
  return fail(GS_ERR_UNSUPPORTED, "field %d / method %d is not built", s.field, s.method);
}

gs_status check_common(const gs_system* sys, int64_t N, const void* theta, const void* y0,
                       double t0, double t1, double rtol, double atol, const void* y1) {
  gs_status st = check_system(sys);
  if (st != GS_OK) return st;
  if (N < 0 || N > 0x7fffffffLL) return fail(GS_ERR_INVALID_ARG, "N=%lld out of range", (long long)N);
  if (N > 0 && (!theta || !y0 || !y1))
    return fail(GS_ERR_INVALID_ARG, "theta, y0 and y1 must be non-NULL");
  if (!(rtol > 0) || !(atol > 0)) return fail(GS_ERR_INVALID_ARG, "rtol and atol must be > 0");
  if (!std::isfinite(t0) || !std::isfinite(t1))
    return fail(GS_ERR_INVALID_ARG, "t0 and t1 must be finite");
  return GS_OK;
}

// The caller's arrays must be readable by this device's kernels: plain (unregistered) host memory,
// or another device's memory, would make a kernel fault instead of returning an error.  Only a
// positive identification rejects a pointer (device, managed and page-locked host memory pass;
// when the runtime cannot tell, the pointer passes too).
struct NamedPtr { const void* p; const char* name; };
gs_status check_device(std::initializer_list<NamedPtr> ptrs) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return GS_OK;
  }
  for (const NamedPtr& a : ptrs) {
    if (!a.p) continue;
    cudaPointerAttributes at{};
    if (cudaPointerGetAttributes(&at, a.p) != cudaSuccess) {
      cudaGetLastError();
      continue;
    }
    if (at.type == cudaMemoryTypeUnregistered)
      return fail(GS_ERR_INVALID_ARG, "%s is host memory: a device pointer is required", a.name);
    if (at.type == cudaMemoryTypeDevice && at.device != dev)
      return fail(GS_ERR_INVALID_ARG, "%s is memory of device %d, the current device is %d",
                  a.name, at.device, dev);
  }
  return GS_OK;
}

long long attempts_of(const gs_options* opt) {
  return (opt && opt->max_attempts > 0) ? (long long)opt->max_attempts : 100000LL;
}

}  // namespace

// ------------------------------------------------------------------------------------------------
// The theta of the stored states.  Beside the states y_n, a record keeps a copy of the theta they
// were computed at (set by the record pass and by gs_replay_forward).  Every call that reads the
// stored states at a caller's theta first compares the two bit for bit on the device; when they
// differ, the mesh is replayed forward at the caller's theta from the stored y_0, rewriting the
// stored states (t_n and h_n are kept).  The result of such a call is therefore always that of
// the replay Psi(theta; sg[h]) over the recorded mesh ("gradsolve: fast exact gradients for ODE
// ensembles on GPUs", §3: the mesh is data; §4.8: one mesh serves the gradients of a whole fit).
// An equal theta costs one read of both copies and a replay launch that exits at once.
// ------------------------------------------------------------------------------------------------
namespace {

size_t theta_bytes(const gs_record* r) {
  return (size_t)(r->sys.theta_shared ? 1 : std::max<int64_t>(r->N, 1)) * r->sys.m * r->rsz;
}

gs_status ensure_theta_kept(gs_record* r, cudaStream_t s) {
  const size_t need = theta_bytes(r);
  if (r->theta_kept_bytes >= need) return GS_OK;
  free_ptr(r->theta_kept, s);
  r->theta_kept = nullptr;
  r->theta_kept_bytes = 0;
  GS_CUDA(dalloc(&r->theta_kept, need, s));
  r->theta_kept_bytes = need;
  return GS_OK;
}

// The stored states are now those of `theta`.
gs_status keep_theta(gs_record* r, const void* theta, cudaStream_t s) {
  GS_CUDA(cudaMemcpyAsync(r->theta_kept, theta, theta_bytes(r), cudaMemcpyDeviceToDevice, s));
  r->theta_known = true;
  return GS_OK;
}

// Makes the stored states those of `theta`.  `queue`: a work counter for the replay kernel, zeroed
// on stream s.  With `fixed_grid` (the entry point that allocates nothing) the grid comes from the
// occupancy query and `sms` alone, without the per-device context.
gs_status refresh_states(gs_record* r, const void* theta, int* queue, bool fixed_grid, int sms,
                         cudaStream_t s) {
  if (r->N == 0 || r->total_steps == 0) return GS_OK;  // no stored state
  if (!r->theta_kept) return fail(GS_ERR_INVALID_ARG, "record holds no parameter copy");
  int* stale = r->counters + 8;
  GS_CUDA(cudaMemsetAsync(stale, r->theta_known ? 0 : 1, sizeof(int), s));
  const long long count = (long long)(theta_bytes(r) / r->rsz);
  const int cgrid = (int)std::max(1LL, std::min<long long>((count + 255) / 256, 8LL * sms));
  if (r->rsz == 8)
    gs::k_theta_check<double><<<cgrid, 256, 0, s>>>(static_cast<const double*>(theta),
                                                   static_cast<double*>(r->theta_kept), count, stale);
  else
    gs::k_theta_check<float><<<cgrid, 256, 0, s>>>(static_cast<const float*>(theta),
                                                  static_cast<float*>(r->theta_kept), count, stale);
  GS_CUDA(cudaGetLastError());
  r->theta_known = true;
  return dispatch(r->sys, [&]<class F, class R, int METHOD>() {
    gs::ReplayParams<R> p{};
    p.N = (int)r->N;
    p.theta = static_cast<const R*>(theta);
    p.theta_stride = r->sys.theta_shared ? 0 : r->sys.m;
    p.y0 = nullptr;  // from the stored y_0
    p.y1 = nullptr;
    p.nsteps = r->nsteps;
    p.choff = r->choff;
    p.chunk_table = r->chunk_table;
    p.pool = static_cast<R*>(r->pool);
    p.queue = queue;
    p.perm = r->perm;
    p.bounds = bounds_of(r);
    p.gate = stale;
    auto launch = [&](auto kern, long long units) -> gs_status {
      int grid = 1;
      if (fixed_grid) {
        int nb = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, BLOCK, 0) != cudaSuccess ||
            nb < 1)
          nb = 1;
        grid = (int)std::max(1LL, std::min((long long)sms * nb, (units + BLOCK - 1) / BLOCK));
      } else {
        grid = persistent_grid(kern, 0, units);
      }
      kern<<<grid, BLOCK, 0, s>>>(p);
      GS_CUDA(cudaGetLastError());
      return GS_OK;
    };
    if constexpr (std::is_same_v<F, gs::FMlpWarp>) return launch(gs::k_replay_forward_mlp<R>, r->N * 32);
    else return launch(gs::k_replay_forward<F, R, METHOD>, r->N);
  });
}

int device_sms() {
  cudaError_t e;
  DeviceCtx* c = device_ctx(&e);
  return c ? c->sms : 148;
}

// The estimate of what the parked trajectories of a record pass still need (gs::k_park_estimate),
// for the first P entries of the park list, or for as many as the device counter `count` holds
// (at most P) when it is non-null.
void launch_park_estimate(gs_record* r, int P, const int* count, int d, double t0, double t1,
                          int C, unsigned long long* est, int kmax, cudaStream_t s) {
  const int eb = (std::max(P, 1) + 255) / 256;
  if (r->rsz == 8)
    gs::k_park_estimate<double><<<eb, 256, 0, s>>>(r->park_list, P, count,
                                                  static_cast<const double*>(r->park_r), r->park_i,
                                                  d, t0, t1, C, est, r->park_key, kmax);
  else
    gs::k_park_estimate<float><<<eb, 256, 0, s>>>(r->park_list, P, count,
                                                 static_cast<const float*>(r->park_r), r->park_i, d,
                                                 (float)t0, (float)t1, C, est, r->park_key, kmax);
}

}  // namespace

// Replay adjoint of the MLP field: one warp per trajectory, per-warp weight-cotangent partials,
// then a fixed-order sum over warps.
static gs_status replay_grad_mlp(const gs_record* rec, const void* theta, const void* dL_dy1,
                          void* dL_dtheta, void* dL_dy0, cudaStream_t s) {
  gs_record* r = const_cast<gs_record*>(rec);
  auto run = [&](auto zero) -> gs_status {
    using R = decltype(zero);
    auto kern = gs::k_adjoint_mlp<R>;
    const int grid = persistent_grid(kern, 0, rec->N * 32);
    const int nwarps = grid * (BLOCK / 32);
    R* partials = nullptr;
    if (dL_dtheta) {
      const size_t need = (size_t)nwarps * gs::MLP_M * sizeof(R);
      if (r->part_bytes < need) {
        free_ptr(r->red_partials, s);
        r->red_partials = nullptr;
        r->part_bytes = 0;
        GS_CUDA(dalloc(&r->red_partials, need, s));
        r->part_bytes = need;
      }
      partials = static_cast<R*>(r->red_partials);
    }
    gs::MlpAdjParams<R> p{};
    p.N = (int)rec->N;
    p.theta = static_cast<const R*>(theta);
    p.dL_dy1 = static_cast<const R*>(dL_dy1);
    p.dL_dy0 = static_cast<R*>(dL_dy0);
    p.partials = partials;
    p.nsteps = rec->nsteps;
    p.choff = rec->choff;
    p.chunk_table = rec->chunk_table;
    p.pool = static_cast<const R*>(rec->pool);
    p.perm = rec->perm;
    p.bounds = bounds_of(rec);
    kern<<<grid, BLOCK, 0, s>>>(p);
    if (partials)
      gs::k_reduce_partials<R><<<(gs::MLP_M + 255) / 256, 256, 0, s>>>(partials, nwarps, gs::MLP_M,
                                                                    static_cast<R*>(dL_dtheta));
    GS_CUDA(cudaGetLastError());
    return GS_OK;
  };
  return rec->sys.dtype == GS_F64 ? run(0.0) : run(0.0f);
}

extern "C" {

const char* gs_last_error(void) { return g_err.c_str(); }

const char* gs_version(void) { return "gradsolve_b200 0.1 (sm_100a)"; }

gs_status gs_solve_forward(const gs_system* sys, const gs_options* opt, int64_t N,
                           const void* theta, const void* y0, double t0, double t1, double rtol,
                           double atol, void* y1, int32_t* nsteps, int32_t* nrejected,
                           int32_t* status, void* stream) {
  NvtxRange nvtx_range("gs_solve_forward");
  gs_status st = check_common(sys, N, theta, y0, t0, t1, rtol, atol, y1);
  if (st != GS_OK) return st;
  if (N == 0) return GS_OK;
  st = check_device({{theta, "theta"}, {y0, "y0"}, {y1, "y1"}, {nsteps, "nsteps"},
                     {nrejected, "nrejected"}, {status, "status"},
                     {opt ? opt->start_order : nullptr, "start_order"}});
  if (st != GS_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* queue = nullptr;
  GS_CUDA(take_counter(s, &queue));
  SolveCall c{N, theta, sys->theta_shared, y0, t0, t1, rtol, atol, attempts_of(opt), y1,
              nsteps, nrejected, status, queue, nullptr, s};
  c.order = opt ? opt->start_order : nullptr;
  return dispatch(*sys, [&]<class F, class R, int METHOD>() { return launch_solve<F, R, METHOD>(c); });
}

gs_status gs_solve_forward_sens(const gs_system* sys, const gs_options* opt, int64_t N,
                                const void* theta, const void* y0, const void* S0, double t0,
                                double t1, double rtol, double atol, void* y1, void* S1,
                                int32_t* nsteps, int32_t* nrejected, int32_t* status,
                                void* stream) {
  NvtxRange nvtx_range("gs_solve_forward_sens");
  gs_status st = check_common(sys, N, theta, y0, t0, t1, rtol, atol, y1);
  if (st != GS_OK) return st;
  if (sys->method != GS_TSIT5 || sys->field == GS_MLP_4_32_32_4)
    return fail(GS_ERR_UNSUPPORTED,
                "forward sensitivities are built for the Tsit5 fields other than the MLP");
  if (N > 0 && !S1) return fail(GS_ERR_INVALID_ARG, "S1 must be non-NULL");
  if (N == 0) return GS_OK;
  st = check_device({{theta, "theta"}, {y0, "y0"}, {S0, "S0"}, {y1, "y1"}, {S1, "S1"},
                     {nsteps, "nsteps"}, {nrejected, "nrejected"}, {status, "status"},
                     {opt ? opt->start_order : nullptr, "start_order"}});
  if (st != GS_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* queue = nullptr;
  GS_CUDA(take_counter(s, &queue));
  SolveCall c{N, theta, sys->theta_shared, y0, t0, t1, rtol, atol, attempts_of(opt), y1,
              nsteps, nrejected, status, queue, nullptr, s, S0, S1};
  c.order = opt ? opt->start_order : nullptr;
  return dispatch(*sys, [&]<class F, class R, int METHOD>() { return launch_solve<F, R, METHOD>(c); });
}

gs_status gs_solve_record(const gs_system* sys, const gs_options* opt, int64_t N,
                          const void* theta, const void* y0, double t0, double t1, double rtol,
                          double atol, gs_record** rec, void* y1, int32_t* status, void* stream) {
  NvtxRange nvtx_range("gs_solve_record");
  gs_status st = check_common(sys, N, theta, y0, t0, t1, rtol, atol, y1);
  if (st != GS_OK) return st;
  if (!rec) return fail(GS_ERR_INVALID_ARG, "rec must be non-NULL");
  if (N > 0) {
    st = check_device({{theta, "theta"}, {y0, "y0"}, {y1, "y1"}, {status, "status"},
                       {opt ? opt->start_order : nullptr, "start_order"}});
    if (st != GS_OK) return st;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  gs_record* r = *rec;
  bool fresh = false;
  if (!r) {
    r = new (std::nothrow) gs_record();
    if (!r) return fail(GS_ERR_CAPACITY, "out of host memory");
    fresh = true;
  }
  auto bail = [&](gs_status e) {
    if (fresh) gs_record_destroy(r);
    return e;
  };
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return bail(fail(GS_ERR_CUDA, "cudaGetDevice failed"));
  if (!fresh && r->device != dev)
    return bail(fail(GS_ERR_INVALID_ARG, "record belongs to device %d, current is %d", r->device, dev));
  r->device = dev;
  // layout of this system
  int C = 0, E = 0;
  st = dispatch(*sys, [&]<class F, class R, int METHOD>() {
    layout_of<F, R>(&C, &E);
    return GS_OK;
  });
  if (st != GS_OK) return bail(st);
  const size_t rsz = sys->dtype == GS_F64 ? 8 : 4;
  if (!fresh && (r->C != C || r->E != E || r->rsz != rsz)) {
    // a different layout: drop the old pool
    free_ptr(r->pool, s); free_ptr(r->chunk_traj, s); free_ptr(r->chunk_seq, s);
    free_ptr(r->chunk_table, s);
    r->pool = nullptr; r->chunk_traj = r->chunk_seq = r->chunk_table = nullptr;
    r->pool_chunks = r->chunk_arrays_cap = 0;
  }
  const bool order_ok = !fresh && r->perm && r->perm_n == N;
  r->sys = *sys;
  r->N = N;
  r->C = C;
  r->E = E;
  r->rsz = rsz;
  r->t0 = t0;
  r->t1 = t1;
  if ((st = ensure_traj_arrays(r, N, s)) != GS_OK) return bail(st);
  // A record that is made again for an ensemble of the same size starts its trajectories in the
  // previous solve's longest-first order: long trajectories begin early instead of forming the
  // tail of the launch.  Scheduling only -- every trajectory's result is independent of it.
  const int* order0 = (opt && opt->start_order) ? opt->start_order : (order_ok ? r->perm : nullptr);
  // With no order at hand (a first solve of this ensemble), every trajectory first takes a short
  // slice of SLICE attempts; the rest of the record then resumes them by decreasing estimate of
  // their remaining steps (from the progress of the slice), and the pool is sized from the same
  // estimate.  The one-warp-per-trajectory neural field, and small ensembles, start in index order.
  constexpr int SLICE = 16;
  const bool slice_mode = !order0 && N >= 4096 && sys->field != GS_MLP_4_32_32_4;
  const int64_t warps = std::min<int64_t>((std::max<int64_t>(N, 1) + 31) / 32, 1 << 16);
  int64_t want_chunks = r->pool_chunks;
  if (want_chunks == 0) {
    if (opt && opt->record_capacity_steps > 0)
      want_chunks = (opt->record_capacity_steps + C - 1) / C + std::max<int64_t>(N, 1);
    else if (slice_mode)  // the slice: at most SLICE + C - 1 accepted steps, one chunk to spare
      want_chunks = N * ((SLICE + 2 * C - 2) / C + 1) + (int64_t)gs::CHUNK_BATCH * warps + 1024;
    else
      want_chunks = (std::max<int64_t>(N, 1) * 64 + C - 1) / C + std::max<int64_t>(N, 1);
  }
  if ((st = ensure_pool(r, want_chunks, s)) != GS_OK) return bail(st);
  if (N == 0) {
    r->nchunks = r->total_steps = 0;
    r->max_steps = 0;
    return GS_OK;
  }
  int32_t* status_out = status ? status : r->status;
  if (!r->ev0 && (cudaEventCreate(&r->ev0) != cudaSuccess || cudaEventCreate(&r->ev1) != cudaSuccess))
    return bail(fail(GS_ERR_CUDA, "cudaEventCreate failed"));
  r->solve_ms = 0;
  if ((st = ensure_park(r, N, s)) != GS_OK) return bail(st);
  if (cudaMemsetAsync(r->counters, 0, 16 * sizeof(int), s) != cudaSuccess)
    return bail(fail(GS_ERR_CUDA, "cudaMemsetAsync failed"));
  // Pass 0 takes every trajectory (in slice mode for SLICE attempts each).  Trajectories that are
  // parked -- their slice spent, or the pool found full -- resume in the next pass from their
  // parked states, by decreasing estimate of their remaining steps, after the pool has grown
  // (its contents kept) by the estimate of what they still need.
  int64_t nq = N;
  int64_t pass_start = 0;  // chunks handed out before this pass
  constexpr int KMAX = 4096;  // remaining-step keys beyond this count as the longest
  for (int pass = 0;; ++pass) {
    const bool sliced = slice_mode && pass == 0;
    SolveCall c{N, theta, sys->theta_shared, y0, t0, t1, rtol, atol, attempts_of(opt), y1,
                r->nsteps, nullptr, status_out, r->counters, r, s};
    c.order = pass == 0 ? order0 : r->park_order;
    c.nqueue = nq;
    c.resume = pass > 0;
    c.slice = sliced ? SLICE : 0;
    cudaEventRecord(r->ev0, s);
    st = dispatch(*sys, [&]<class F, class R, int METHOD>() { return launch_solve<F, R, METHOD>(c); });
    if (st != GS_OK) return bail(st);
    cudaEventRecord(r->ev1, s);
    // summary over the ensemble (complete once no trajectory is parked): statuses, the longest
    // record, the worst status, the step and chunk offsets
    if (status_out != r->status &&
        cudaMemcpyAsync(r->status, status_out, N * sizeof(int), cudaMemcpyDeviceToDevice, s) !=
            cudaSuccess)
      return bail(fail(GS_ERR_CUDA, "status copy failed"));
    if ((st = summarise_pass(r, status_out, (int)N, C, s)) != GS_OK) return bail(st);
    // a slice parks (nearly) every trajectory: the estimate of what they still need is queued
    // right behind the pass, with the parked count read on the device, and comes back with the
    // summary in one synchronisation
    unsigned long long* est = reinterpret_cast<unsigned long long*>(r->counters + 10);
    if (sliced) {
      if (cudaMemsetAsync(est, 0, 2 * sizeof(unsigned long long), s) != cudaSuccess)
        return bail(fail(GS_ERR_CUDA, "cudaMemsetAsync failed"));
      launch_park_estimate(r, (int)nq, r->counters + 2, sys->d, t0, t1, C, est, KMAX, s);
    }
    if (cudaMemcpyAsync(r->host, r->counters, 14 * sizeof(int), cudaMemcpyDeviceToHost, s) !=
            cudaSuccess ||
        cudaMemcpyAsync(r->host + 8, r->offsets + N, sizeof(long long), cudaMemcpyDeviceToHost, s) !=
            cudaSuccess)
      return bail(fail(GS_ERR_CUDA, "readback failed"));
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess)
      return bail(fail(GS_ERR_CUDA, "record solve failed: %s", cudaGetErrorString(e)));
    float pass_ms = 0;
    if (cudaEventElapsedTime(&pass_ms, r->ev0, r->ev1) == cudaSuccess) r->solve_ms += pass_ms;
    const int64_t used = std::min<int64_t>(r->host[1], r->pool_chunks);
    const int parked = r->host[2];
    if (parked == 0) {
      r->nchunks = used;  // reserved, some possibly unused
      r->max_steps = r->host[3];
      long long tot;
      std::memcpy(&tot, r->host + 8, sizeof(tot));
      r->total_steps = tot;
      break;
    }
    if (pass >= 64) return bail(fail(GS_ERR_CAPACITY, "record pool still full after %d passes", pass));
    // what the parked trajectories still need (from their progress; for those parked before
    // their first step twice the mean use of the trajectories that did start in this pass), and
    // their order for the next pass: largest estimate first
    unsigned long long hest[2] = {0, 0};
    if (sliced) {
      std::memcpy(hest, r->host + 10, sizeof(hest));
    } else {
      if (cudaMemsetAsync(est, 0, 2 * sizeof(unsigned long long), s) != cudaSuccess)
        return bail(fail(GS_ERR_CUDA, "cudaMemsetAsync failed"));
      launch_park_estimate(r, parked, nullptr, sys->d, t0, t1, C, est, KMAX, s);
      if (cudaMemcpyAsync(hest, est, sizeof(hest), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
          cudaStreamSynchronize(s) != cudaSuccess)
        return bail(fail(GS_ERR_CUDA, "park estimate failed"));
    }
    // the next pass's order (queued; only that pass reads it)
    if ((st = counting_sort_desc(r, r->park_key, parked, KMAX, r->park_list, r->park_order, s)) !=
        GS_OK)
      return bail(st);
    const int64_t unstarted = (int64_t)hest[1];
    const int64_t started = std::max<int64_t>(1, nq - unstarted);
    const int64_t per_new = 2 * std::max<int64_t>(used - pass_start, 1) / started + 2;
    int64_t extra = std::max<int64_t>((int64_t)hest[0] + unstarted * per_new, 2 * (int64_t)parked);
    // after a pool found full the pool at most triples per pass, so that a wild estimate costs a
    // pass, not the device's memory
    if (!sliced) extra = std::min<int64_t>(extra, std::max<int64_t>(2 * used + 1024, 2 * (int64_t)parked));
    // and never beyond 80 % of the device memory that is free (the cache's blocks count as
    // free).  Asking the driver costs 0.1-0.8 ms, so it is asked only when the pool would take
    // an eighth of the device or more, or when growing without asking failed.
    const int64_t chunk_b = (int64_t)C * E * (int64_t)rsz + 3 * (int64_t)sizeof(int);
    auto cap_by_free = [&](int64_t x) {
      size_t free_b = 0, total_b = 0;
      if (cudaMemGetInfo(&free_b, &total_b) != cudaSuccess) {
        cudaGetLastError();
        return x;
      }
      cudaError_t ce;
      DeviceCtx* dc = device_ctx(&ce);
      if (dc) {
        std::lock_guard<std::mutex> lk(dc->mem_mu);
        free_b += dc->cached_bytes;
      }
      return std::min<int64_t>(x, std::max<int64_t>((int64_t)(free_b * 0.8) / chunk_b,
                                                    2 * (int64_t)parked));
    };
    cudaError_t ce;
    const DeviceCtx* dc = device_ctx(&ce);
    const size_t total_mem = dc ? dc->total_mem : 0;
    const bool asked = total_mem == 0 || (double)(used + extra) * chunk_b >= 0.125 * total_mem;
    if (asked) extra = cap_by_free(extra);
    int64_t want = used + extra + (int64_t)gs::CHUNK_BATCH * warps + 1024;
    if (want > r->pool_chunks) {
      st = grow_pool(r, want, used, s);
      if (st != GS_OK && !asked) {
        cudaGetLastError();
        extra = cap_by_free(extra);
        want = used + extra + (int64_t)gs::CHUNK_BATCH * warps + 1024;
        st = want > r->pool_chunks ? grow_pool(r, want, used, s) : GS_OK;
      }
      if (st != GS_OK) return bail(st);
    }
    // the next pass: the parked trajectories, a fresh queue, park count and summary, and chunks
    // handed out after the kept ones
    if (cudaMemsetAsync(r->counters, 0, 5 * sizeof(int), s) != cudaSuccess)
      return bail(fail(GS_ERR_CUDA, "counter reset failed"));
    gs::k_set_int<<<1, 1, 0, s>>>(r->counters + 1, (int)used);
    if (cudaGetLastError() != cudaSuccess) return bail(fail(GS_ERR_CUDA, "counter reset failed"));
    pass_start = used;
    nq = parked;
  }
  // chunk table (the chunk offsets came with the last pass's summary)
  if (r->nchunks > 0)
    gs::k_chunk_table<<<(int)((r->nchunks + 255) / 256), 256, 0, s>>>(
        r->chunk_traj, r->chunk_seq, (int)r->nchunks, r->choff, r->chunk_table, bounds_of(r));
  if (cudaGetLastError() != cudaSuccess) return bail(fail(GS_ERR_CUDA, "chunk table launch failed"));
  if ((st = build_perm(r, s)) != GS_OK) return bail(st);
  if ((st = ensure_theta_kept(r, s)) != GS_OK || (st = keep_theta(r, theta, s)) != GS_OK)
    return bail(st);
  *rec = r;
  if (r->host[4] != 0) {
    fail(GS_ERR_TRAJ_FAILED, "some trajectories did not reach t1 (max status %d)", r->host[4]);
    return GS_ERR_TRAJ_FAILED;
  }
  return GS_OK;
}

gs_status gs_replay_grad(const gs_record* rec, const void* theta, const void* dL_dy1,
                         void* dL_dtheta, void* dL_dy0, void* stream) {
  NvtxRange nvtx_range("gs_replay_grad");
  if (!rec) return fail(GS_ERR_INVALID_ARG, "record is NULL");
  if (rec->N == 0) return GS_OK;
  if (!theta || !dL_dy1) return fail(GS_ERR_INVALID_ARG, "theta and dL_dy1 must be non-NULL");
  if (!dL_dtheta && !dL_dy0) return fail(GS_ERR_INVALID_ARG, "no output requested");
  gs_status st = check_device({{theta, "theta"}, {dL_dy1, "dL_dy1"}, {dL_dtheta, "dL_dtheta"},
                               {dL_dy0, "dL_dy0"}});
  if (st != GS_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int M = rec->sys.m;
  const int64_t N = rec->N;
  gs_record* r = const_cast<gs_record*>(rec);
  int* rq = nullptr;
  GS_CUDA(take_counter(s, &rq));
  if ((st = refresh_states(r, theta, rq, false, device_sms(), s)) != GS_OK) return st;
  if (rec->sys.field == GS_MLP_4_32_32_4) return replay_grad_mlp(rec, theta, dL_dy1, dL_dtheta, dL_dy0, s);
  const bool shared = rec->sys.theta_shared && dL_dtheta;
  const int per_block = 4096;
  const int nred = (int)((N + per_block - 1) / per_block);
  if (shared) {
    const size_t need = (size_t)N * M * rec->rsz, needp = (size_t)nred * M * rec->rsz;
    if (r->red_bytes < need) {
      free_ptr(r->red_scratch, s);
      r->red_scratch = nullptr;
      r->red_bytes = 0;
      GS_CUDA(dalloc(&r->red_scratch, need, s));
      r->red_bytes = need;
    }
    if (r->part_bytes < needp) {
      free_ptr(r->red_partials, s);
      r->red_partials = nullptr;
      r->part_bytes = 0;
      GS_CUDA(dalloc(&r->red_partials, needp, s));
      r->part_bytes = needp;
    }
  }
  void* scratch = r->red_scratch;
  void* partials = r->red_partials;
  int* queue = nullptr;
  GS_CUDA(take_counter(s, &queue));
  AdjCall c{rec, theta, dL_dy1, dL_dy0, shared ? scratch : dL_dtheta, queue, s};
  return dispatch(rec->sys, [&]<class F, class R, int METHOD>() {
    gs_status rs = launch_adjoint<F, R, METHOD>(c);
    if (rs != GS_OK || !shared) return rs;
    gs::k_reduce_theta<R><<<nred, gs::RED_BLOCK, 0, s>>>(static_cast<const R*>(scratch), (int)N, M,
                                                        per_block, static_cast<R*>(partials));
    gs::k_reduce_partials<R><<<1, 256, 0, s>>>(static_cast<const R*>(partials), nred, M,
                                               static_cast<R*>(dL_dtheta));
    GS_CUDA(cudaGetLastError());
    return GS_OK;
  });
}

gs_status gs_replay_forward(gs_record* rec, const void* theta, const void* y0, void* y1,
                            void* stream) {
  NvtxRange nvtx_range("gs_replay_forward");
  if (!rec) return fail(GS_ERR_INVALID_ARG, "record is NULL");
  if (rec->N == 0) return GS_OK;
  if (!theta || !y0) return fail(GS_ERR_INVALID_ARG, "theta and y0 must be non-NULL");
  const gs_status dst = check_device({{theta, "theta"}, {y0, "y0"}, {y1, "y1"}});
  if (dst != GS_OK) return dst;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  void* y1buf = y1;
  if (!y1buf) {
    const size_t need = (size_t)rec->N * rec->sys.d * rec->rsz;
    if (rec->y1_bytes < need) {
      free_ptr(rec->y1_scratch, s);
      rec->y1_scratch = nullptr;
      rec->y1_bytes = 0;
      GS_CUDA(dalloc(&rec->y1_scratch, need, s));
      rec->y1_bytes = need;
    }
    y1buf = rec->y1_scratch;
  }
  int* queue = nullptr;
  GS_CUDA(take_counter(s, &queue));
  gs_status st = dispatch(rec->sys, [&]<class F, class R, int METHOD>() {
    gs::ReplayParams<R> p{};
    if constexpr (std::is_same_v<F, gs::FMlpWarp>) {
      p.N = (int)rec->N;
      p.theta = static_cast<const R*>(theta);
      p.y0 = static_cast<const R*>(y0);
      p.y1 = static_cast<R*>(y1buf);
      p.nsteps = rec->nsteps;
      p.choff = rec->choff;
      p.chunk_table = rec->chunk_table;
      p.pool = static_cast<R*>(rec->pool);
      p.queue = queue;
      p.perm = rec->perm;
      p.bounds = bounds_of(rec);
      auto kern = gs::k_replay_forward_mlp<R>;
      kern<<<persistent_grid(kern, 0, rec->N * 32), BLOCK, 0, s>>>(p);
      GS_CUDA(cudaGetLastError());
      return GS_OK;
    } else {
    p.N = (int)rec->N;
    p.theta = static_cast<const R*>(theta);
    p.theta_stride = rec->sys.theta_shared ? 0 : F::M;
    p.y0 = static_cast<const R*>(y0);
    p.y1 = static_cast<R*>(y1buf);
    p.nsteps = rec->nsteps;
    p.choff = rec->choff;
    p.chunk_table = rec->chunk_table;
    p.pool = static_cast<R*>(rec->pool);
    p.queue = queue;
    p.perm = rec->perm;
    p.bounds = bounds_of(rec);
    auto kern = gs::k_replay_forward<F, R, METHOD>;
    const int grid = persistent_grid(kern, 0, rec->N);
    kern<<<grid, BLOCK, 0, s>>>(p);
    GS_CUDA(cudaGetLastError());
    return GS_OK;
    }
  });
  if (st != GS_OK) return st;
  return keep_theta(rec, theta, s);  // the stored states are now those of theta
}

}  // extern "C"

namespace {

gs_status check_out_times(const gs_record* rec, int32_t J, const double* tau) {
  if (!rec) return fail(GS_ERR_INVALID_ARG, "record is NULL");
  if (J < 1 || J > GS_MAX_OUTPUT_TIMES)
    return fail(GS_ERR_INVALID_ARG, "J=%d outside [1, %d]", J, GS_MAX_OUTPUT_TIMES);
  if (!tau) return fail(GS_ERR_INVALID_ARG, "tau is NULL");
  for (int j = 0; j < J; ++j) {
    if (!std::isfinite(tau[j])) return fail(GS_ERR_INVALID_ARG, "tau[%d] is not finite", j);
    if (j > 0 && tau[j] < tau[j - 1])
      return fail(GS_ERR_INVALID_ARG, "tau must be ascending (tau[%d] < tau[%d])", j, j - 1);
  }
  return GS_OK;
}

// How many of the ascending times are before t1, compared in the record's precision as the kernels
// compare them.
int outputs_before_t1(const gs_record* rec, int32_t J, const double* tau) {
  const bool f32 = rec->rsz == sizeof(float);
  int jS = 0;
  while (jS < J && (f32 ? (float)tau[jS] < (float)rec->t1 : tau[jS] < rec->t1)) ++jS;
  return jS;
}

template <class R>
void fill_times(gs::OutTimes<R>& ot, const gs_record* rec, int32_t J, const double* tau) {
  ot.J = J;
  ot.t1 = R(rec->t1);
  for (int j = 0; j < J; ++j) ot.tau[j] = R(tau[j]);
}

template <class R>
void fill_replay_params(gs::ReplayParams<R>& p, const gs_record* rec, const void* theta, int M,
                        int* queue) {
  p.N = (int)rec->N;
  p.theta = static_cast<const R*>(theta);
  p.theta_stride = rec->sys.theta_shared ? 0 : M;
  p.nsteps = rec->nsteps;
  p.choff = rec->choff;
  p.chunk_table = rec->chunk_table;
  p.pool = static_cast<R*>(rec->pool);
  p.queue = queue;
  p.perm = rec->perm;
  p.bounds = bounds_of(rec);
}

// Gradient of a loss on the outputs at requested times, MLP field: one warp per trajectory
// (the extra pullbacks taken where the walk meets them), per-warp weight-cotangent partials, then a
// fixed-order sum over warps.
static gs_status replay_grad_outputs_mlp(const gs_record* rec, const void* theta, int32_t J,
                                         const double* tau, const void* dL_dyout,
                                         const void* dL_dy1, void* dL_dtheta, void* dL_dy0,
                                         cudaStream_t s) {
  gs_record* r = const_cast<gs_record*>(rec);
  auto run = [&](auto zero) -> gs_status {
    using R = decltype(zero);
    auto kern = gs::k_adjoint_outputs_mlp<R>;
    const int grid = persistent_grid(kern, 0, rec->N * 32);
    const int nwarps = grid * (BLOCK / 32);
    R* partials = nullptr;
    if (dL_dtheta) {
      const size_t need = (size_t)nwarps * gs::MLP_M * sizeof(R);
      if (r->part_bytes < need) {
        free_ptr(r->red_partials, s);
        r->red_partials = nullptr;
        r->part_bytes = 0;
        GS_CUDA(dalloc(&r->red_partials, need, s));
        r->part_bytes = need;
      }
      partials = static_cast<R*>(r->red_partials);
    }
    gs::MlpOutAdjParams<R> q{};
    gs::MlpAdjParams<R>& p = q.ap;
    p.N = (int)rec->N;
    p.theta = static_cast<const R*>(theta);
    p.dL_dy1 = static_cast<const R*>(dL_dy1);
    p.dL_dy0 = static_cast<R*>(dL_dy0);
    p.partials = partials;
    p.nsteps = rec->nsteps;
    p.choff = rec->choff;
    p.chunk_table = rec->chunk_table;
    p.pool = static_cast<const R*>(rec->pool);
    p.perm = rec->perm;
    p.bounds = bounds_of(rec);
    q.dL_dyout = static_cast<const R*>(dL_dyout);
    fill_times<R>(q.ot, rec, J, tau);
    q.jS = outputs_before_t1(rec, J, tau);
    kern<<<grid, BLOCK, 0, s>>>(q);
    if (partials)
      gs::k_reduce_partials<R><<<(gs::MLP_M + 255) / 256, 256, 0, s>>>(partials, nwarps, gs::MLP_M,
                                                                    static_cast<R*>(dL_dtheta));
    GS_CUDA(cudaGetLastError());
    return GS_OK;
  };
  return rec->sys.dtype == GS_F64 ? run(0.0) : run(0.0f);
}

}  // namespace

extern "C" {

gs_status gs_replay_outputs(const gs_record* rec, const void* theta, const void* y0, int32_t J,
                            const double* tau, void* y_out, void* stream) {
  NvtxRange nvtx_range("gs_replay_outputs");
  gs_status st = check_out_times(rec, J, tau);
  if (st != GS_OK) return st;
  if (rec->N == 0) return GS_OK;
  if (!theta || !y0 || !y_out)
    return fail(GS_ERR_INVALID_ARG, "theta, y0 and y_out must be non-NULL");
  st = check_device({{theta, "theta"}, {y0, "y0"}, {y_out, "y_out"}});
  if (st != GS_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* rq = nullptr;
  GS_CUDA(take_counter(s, &rq));
  st = refresh_states(const_cast<gs_record*>(rec), theta, rq, false, device_sms(), s);
  if (st != GS_OK) return st;
  return dispatch(rec->sys, [&]<class F, class R, int METHOD>() {
    gs::OutParams<R> q{};
    fill_replay_params<R>(q.rp, rec, theta, F::M, nullptr);
    q.rp.y0 = static_cast<const R*>(y0);
    q.y_out = static_cast<R*>(y_out);
    fill_times<R>(q.ot, rec, J, tau);
    q.jS = outputs_before_t1(rec, J, tau);
    if constexpr (std::is_same_v<F, gs::FMlpWarp>) {
      auto kern = gs::k_replay_outputs_mlp<R>;  // one warp per trajectory
      kern<<<persistent_grid(kern, 0, rec->N * 32), BLOCK, 0, s>>>(q);
    } else {
      gs::k_replay_outputs<F, R, METHOD><<<(unsigned)((rec->N + BLOCK - 1) / BLOCK), BLOCK, 0, s>>>(q);
    }
    GS_CUDA(cudaGetLastError());
    return GS_OK;
  });
}

gs_status gs_replay_grad_outputs(const gs_record* rec, const void* theta, int32_t J,
                                 const double* tau, const void* dL_dyout, const void* dL_dy1,
                                 void* dL_dtheta, void* dL_dy0, void* stream) {
  NvtxRange nvtx_range("gs_replay_grad_outputs");
  gs_status st = check_out_times(rec, J, tau);
  if (st != GS_OK) return st;
  if (rec->N == 0) return GS_OK;
  if (!theta || !dL_dyout) return fail(GS_ERR_INVALID_ARG, "theta and dL_dyout must be non-NULL");
  if (!dL_dtheta && !dL_dy0) return fail(GS_ERR_INVALID_ARG, "no output requested");
  st = check_device({{theta, "theta"}, {dL_dyout, "dL_dyout"}, {dL_dy1, "dL_dy1"},
                     {dL_dtheta, "dL_dtheta"}, {dL_dy0, "dL_dy0"}});
  if (st != GS_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int M = rec->sys.m;
  const int64_t N = rec->N;
  const bool shared = rec->sys.theta_shared && dL_dtheta;
  const int per_block = 4096;
  const int nred = (int)((N + per_block - 1) / per_block);
  gs_record* r = const_cast<gs_record*>(rec);
  int* rq = nullptr;
  GS_CUDA(take_counter(s, &rq));
  if ((st = refresh_states(r, theta, rq, false, device_sms(), s)) != GS_OK) return st;
  if (rec->sys.field == GS_MLP_4_32_32_4)
    return replay_grad_outputs_mlp(rec, theta, J, tau, dL_dyout, dL_dy1, dL_dtheta, dL_dy0, s);
  if (shared) {
    const size_t need = (size_t)N * M * rec->rsz, needp = (size_t)nred * M * rec->rsz;
    if (r->red_bytes < need) {
      free_ptr(r->red_scratch, s);
      r->red_scratch = nullptr;
      r->red_bytes = 0;
      GS_CUDA(dalloc(&r->red_scratch, need, s));
      r->red_bytes = need;
    }
    if (r->part_bytes < needp) {
      free_ptr(r->red_partials, s);
      r->red_partials = nullptr;
      r->part_bytes = 0;
      GS_CUDA(dalloc(&r->red_partials, needp, s));
      r->part_bytes = needp;
    }
  }
  const int jS = outputs_before_t1(rec, J, tau);
  int* queue = nullptr;
  GS_CUDA(take_counter(s, &queue));
  return dispatch(rec->sys, [&]<class F, class R, int METHOD>() {
    if constexpr (std::is_same_v<F, gs::FMlpWarp>) {
      return fail(GS_ERR_UNSUPPORTED, "the MLP field takes replay_grad_outputs_mlp");
    } else {
      gs::AdjOutParams<R> q{};
      gs::AdjointParams<R>& p = q.ap;
      p.N = (int)N;
      p.theta = static_cast<const R*>(theta);
      p.theta_stride = rec->sys.theta_shared ? 0 : F::M;
      p.dL_dy1 = static_cast<const R*>(dL_dy1);
      p.dL_dy0 = static_cast<R*>(dL_dy0);
      p.dL_dtheta = shared ? static_cast<R*>(r->red_scratch) : static_cast<R*>(dL_dtheta);
      p.nsteps = rec->nsteps;
      p.choff = rec->choff;
      p.chunk_table = rec->chunk_table;
      p.pool = static_cast<const R*>(rec->pool);
      p.queue = queue;
      p.perm = rec->perm;
      p.bounds = bounds_of(rec);
      q.dL_dyout = static_cast<const R*>(dL_dyout);
      fill_times<R>(q.ot, rec, J, tau);
      q.jS = jS;
      // the stage tape, then each lane's cotangent slot for the passes that take an output
      const size_t smem = adjoint_smem<F, R, METHOD>() + (size_t)F::D * BLOCK * sizeof(R);
      auto kern = gs::k_adjoint_outputs<F, R, METHOD>;
      if (smem > 48 * 1024)
        GS_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
      kern<<<persistent_grid(kern, smem, N), BLOCK, smem, s>>>(q);
      if (shared) {
        gs::k_reduce_theta<R><<<nred, gs::RED_BLOCK, 0, s>>>(static_cast<const R*>(r->red_scratch),
                                                            (int)N, M, per_block,
                                                            static_cast<R*>(r->red_partials));
        gs::k_reduce_partials<R><<<1, 256, 0, s>>>(static_cast<const R*>(r->red_partials), nred, M,
                                                   static_cast<R*>(dL_dtheta));
      }
      GS_CUDA(cudaGetLastError());
      return GS_OK;
    }
  });
}

gs_status gs_checked_violations(int64_t* count) {
#ifdef GS_CHECKED
  if (!count) return fail(GS_ERR_INVALID_ARG, "count must be non-NULL");
  unsigned long long v = 0, z = 0;
  GS_CUDA(cudaMemcpyFromSymbol(&v, gs::g_gs_violations, sizeof(v)));
  GS_CUDA(cudaMemcpyToSymbol(gs::g_gs_violations, &z, sizeof(z)));
  *count = (int64_t)v;
  return GS_OK;
#else
  (void)count;
  return fail(GS_ERR_UNSUPPORTED, "not a checked build (compile with -DGS_CHECKED)");
#endif
}

gs_status gs_record_info(const gs_record* rec, gs_record_info_t* out) {
  if (!rec || !out) return fail(GS_ERR_INVALID_ARG, "NULL argument");
  out->N = rec->N;
  out->total_steps = rec->total_steps;
  out->max_steps = rec->max_steps;
  out->chunk_steps = rec->C;
  out->entry_reals = rec->E;
  out->dtype = rec->sys.dtype;
  out->nchunks = rec->nchunks;
  out->pool_bytes = (int64_t)rec->pool_chunks * rec->C * rec->E * (int64_t)rec->rsz;
  out->nsteps = rec->nsteps;
  out->status = rec->status;
  out->offsets = reinterpret_cast<const int64_t*>(rec->offsets);
  out->chunk_offsets = reinterpret_cast<const int64_t*>(rec->choff);
  out->chunk_table = rec->chunk_table;
  out->pool = rec->pool;
  out->solve_ms = rec->solve_ms;
  out->order = rec->perm_n == rec->N ? rec->perm : nullptr;
  return GS_OK;
}

gs_status gs_record_export(const gs_record* rec, void* T, void* H, void* Y, int64_t* offsets,
                           void* stream) {
  NvtxRange nvtx_range("gs_record_export");
  if (!rec) return fail(GS_ERR_INVALID_ARG, "record is NULL");
  gs_status st = check_device({{T, "T"}, {H, "H"}, {Y, "Y"}, {offsets, "offsets"}});
  if (st != GS_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (offsets && rec->N >= 0)
    GS_CUDA(cudaMemcpyAsync(offsets, rec->offsets, (rec->N + 1) * sizeof(long long),
                            cudaMemcpyDeviceToDevice, s));
  if (rec->total_steps == 0) return GS_OK;
  const int nb = (int)((rec->total_steps + 255) / 256);
  if (rec->sys.dtype == GS_F64)
    gs::k_export<double><<<nb, 256, 0, s>>>(static_cast<const double*>(rec->pool), rec->chunk_table,
                                            rec->choff, rec->offsets, (int)rec->N, rec->sys.d,
                                            rec->C, rec->total_steps, static_cast<double*>(T),
                                            static_cast<double*>(H), static_cast<double*>(Y),
                                            bounds_of(rec));
  else
    gs::k_export<float><<<nb, 256, 0, s>>>(static_cast<const float*>(rec->pool), rec->chunk_table,
                                           rec->choff, rec->offsets, (int)rec->N, rec->sys.d,
                                           rec->C, rec->total_steps, static_cast<float*>(T),
                                           static_cast<float*>(H), static_cast<float*>(Y),
                                           bounds_of(rec));
  GS_CUDA(cudaGetLastError());
  return GS_OK;
}

gs_status gs_record_import(const gs_system* sys, int64_t N, const int32_t* nsteps, const void* T,
                           const void* H, const void* Y, gs_record** rec, void* stream) {
  NvtxRange nvtx_range("gs_record_import");
  gs_status st = check_system(sys);
  if (st != GS_OK) return st;
  if (!rec) return fail(GS_ERR_INVALID_ARG, "rec must be non-NULL");
  if (N < 0 || N > 0x7fffffffLL) return fail(GS_ERR_INVALID_ARG, "N out of range");
  if (N > 0 && (!nsteps || !H || !Y)) return fail(GS_ERR_INVALID_ARG, "nsteps, H, Y required");
  if (N > 0) {
    st = check_device({{nsteps, "nsteps"}, {T, "T"}, {H, "H"}, {Y, "Y"}});
    if (st != GS_OK) return st;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  gs_record* r = new (std::nothrow) gs_record();
  if (!r) return fail(GS_ERR_CAPACITY, "out of host memory");
  auto bail = [&](gs_status e) {
    gs_record_destroy(r);
    return e;
  };
  int C = 0, E = 0;
  st = dispatch(*sys, [&]<class F, class R, int METHOD>() {
    layout_of<F, R>(&C, &E);
    return GS_OK;
  });
  if (st != GS_OK) return bail(st);
  cudaGetDevice(&r->device);
  r->sys = *sys;
  r->N = N;
  r->C = C;
  r->E = E;
  r->rsz = sys->dtype == GS_F64 ? 8 : 4;
  if ((st = ensure_traj_arrays(r, N, s)) != GS_OK) return bail(st);
  if (N > 0) {
    if (cudaMemcpyAsync(r->nsteps, nsteps, N * sizeof(int), cudaMemcpyDeviceToDevice, s) !=
            cudaSuccess ||
        cudaMemsetAsync(r->status, 0, N * sizeof(int), s) != cudaSuccess ||
        cudaMemsetAsync(r->counters, 0, 16 * sizeof(int), s) != cudaSuccess)
      return bail(fail(GS_ERR_CUDA, "import copies failed"));
    if ((st = scan_counts<0>(r->nsteps, (int)N, C, r->offsets, r->tiles, s)) != GS_OK) return bail(st);
    gs::k_max_int<<<(int)((N + 255) / 256), 256, 0, s>>>(r->nsteps, (int)N, r->counters + 3);
    if ((st = scan_counts<1>(r->nsteps, (int)N, C, r->choff, r->tiles, s)) != GS_OK) return bail(st);
    long long tot[2] = {0, 0};
    if (cudaMemcpyAsync(&tot[0], r->offsets + N, sizeof(long long), cudaMemcpyDeviceToHost, s) !=
            cudaSuccess ||
        cudaMemcpyAsync(&tot[1], r->choff + N, sizeof(long long), cudaMemcpyDeviceToHost, s) !=
            cudaSuccess ||
        cudaMemcpyAsync(r->host, r->counters, 8 * sizeof(int), cudaMemcpyDeviceToHost, s) !=
            cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
      return bail(fail(GS_ERR_CUDA, "import readback failed"));
    r->total_steps = tot[0];
    r->nchunks = tot[1];
    r->max_steps = r->host[3];
    if ((st = ensure_pool(r, std::max<int64_t>(r->nchunks, 1), s)) != GS_OK) return bail(st);
    if (r->nchunks > 0) {
      gs::k_iota<<<(int)((r->nchunks + 255) / 256), 256, 0, s>>>(r->chunk_table, (int)r->nchunks);
      const int nb = (int)((r->total_steps + 255) / 256);
      if (sys->dtype == GS_F64)
        gs::k_import<double><<<nb, 256, 0, s>>>(static_cast<double*>(r->pool), r->choff, r->offsets,
                                                (int)N, sys->d, C, r->total_steps,
                                                static_cast<const double*>(T),
                                                static_cast<const double*>(H),
                                                static_cast<const double*>(Y), bounds_of(r));
      else
        gs::k_import<float><<<nb, 256, 0, s>>>(static_cast<float*>(r->pool), r->choff, r->offsets,
                                               (int)N, sys->d, C, r->total_steps,
                                               static_cast<const float*>(T),
                                               static_cast<const float*>(H),
                                               static_cast<const float*>(Y), bounds_of(r));
      if (cudaGetLastError() != cudaSuccess) return bail(fail(GS_ERR_CUDA, "import launch failed"));
    }
    if ((st = build_perm(r, s)) != GS_OK) return bail(st);
    if ((st = ensure_theta_kept(r, s)) != GS_OK) return bail(st);
  }
  r->theta_known = false;  // the states' theta is not known: the first use replays them
  *rec = r;
  return GS_OK;
}

void gs_record_destroy(gs_record* r) {
  if (!r) return;
  int prev = 0;
  cudaGetDevice(&prev);
  cudaSetDevice(r->device);
  cudaDeviceSynchronize();  // nothing queued may still use the storage handed back below
  cudaStream_t s = 0;
  free_ptr(r->pool, s); free_ptr(r->chunk_traj, s); free_ptr(r->chunk_seq, s);
  free_ptr(r->chunk_table, s);
  free_ptr(r->nsteps, s); free_ptr(r->status, s); free_ptr(r->offsets, s); free_ptr(r->choff, s);
  free_ptr(r->tiles, s); free_ptr(r->counters, s);
  free_ptr(r->red_scratch, s); free_ptr(r->red_partials, s); free_ptr(r->y1_scratch, s);
  free_ptr(r->theta_kept, s);
  free_ptr(r->perm, s); free_ptr(r->bins, s); free_ptr(r->binoff, s); free_ptr(r->btiles, s);
  free_ptr(r->park_list, s); free_ptr(r->park_r, s);
  free_ptr(r->park_i, s); free_ptr(r->park_att, s); free_ptr(r->park_key, s);
  free_ptr(r->park_order, s);
  if (r->ev0) cudaEventDestroy(r->ev0);
  if (r->ev1) cudaEventDestroy(r->ev1);
  cudaSetDevice(prev);
  delete r;
}

gs_status gs_memory_trim(int64_t keep_bytes) {
  cudaError_t e;
  DeviceCtx* c = device_ctx(&e);
  if (!c) return fail(GS_ERR_CUDA, "device context: %s", cudaGetErrorString(e));
  if (keep_bytes < 0) keep_bytes = 0;
  GS_CUDA(cudaDeviceSynchronize());
  GS_CUDA(release_cached(c, (size_t)keep_bytes));
  return GS_OK;
}

}  // extern "C"

// ------------------------------------------------------------------------------------------------
// gs_replay_grad_noalloc: the replay gradient with its scratch in a fixed device array, for
// callers that cannot allocate device memory when they ask for a gradient.
// Layout of the array: [0, 256) work counters (the adjoint's at byte 0, the forward replay's at
// byte 64); then theta-bar per trajectory [N][m]; then the block partials [nred][m] of the
// shared-theta sum.
// ------------------------------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_noalloc_scratch[GS_NOALLOC_SCRATCH_BYTES];

namespace {

struct NoallocDevice {
  std::once_flag once;
  cudaError_t err = cudaSuccess;
  unsigned char* ptr = nullptr;  // device address of g_noalloc_scratch on this device
  int sms = 0;
};
NoallocDevice g_noalloc[MAX_DEVICES];

// Once per device, with that device current: the device address of the array (host code may
// not use the array's name as an address) and the SM count.
gs_status noalloc_setup(NoallocDevice** out) {
  int dev = 0;
  GS_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= MAX_DEVICES) return fail(GS_ERR_CUDA, "device %d out of range", dev);
  NoallocDevice& d = g_noalloc[dev];
  std::call_once(d.once, [&]() {
    d.err = cudaGetSymbolAddress(reinterpret_cast<void**>(&d.ptr), g_noalloc_scratch);
    if (d.err == cudaSuccess) d.err = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
  });
  if (d.err != cudaSuccess)
    return fail(GS_ERR_CUDA, "no-alloc scratch set-up failed on device %d: %s", dev,
                cudaGetErrorString(d.err));
  *out = &d;
  return GS_OK;
}

template <class F, class R, int METHOD>
gs_status noalloc_adjoint(const gs_record* r, const void* theta, const void* dL_dy1,
                          void* dL_dtheta, void* dL_dy0, unsigned char* scratch, int sms,
                          cudaStream_t s) {
  if constexpr (std::is_same_v<F, gs::FMlpWarp>) {
    return fail(GS_ERR_UNSUPPORTED, "gs_replay_grad_noalloc does not take the MLP field");
  } else {
    const bool shared = r->sys.theta_shared && dL_dtheta;
    const int M = F::M;
    const int64_t N = r->N;
    const int per_block = 4096;
    const int nred = (int)((N + per_block - 1) / per_block);
    R* traj = reinterpret_cast<R*>(scratch + 256);
    R* partials = traj + (size_t)N * M;
    gs::AdjointParams<R> p{};
    p.N = (int)N;
    p.theta = static_cast<const R*>(theta);
    p.theta_stride = r->sys.theta_shared ? 0 : M;
    p.dL_dy1 = static_cast<const R*>(dL_dy1);
    p.dL_dy0 = static_cast<R*>(dL_dy0);
    p.dL_dtheta = shared ? traj : static_cast<R*>(dL_dtheta);
    p.nsteps = r->nsteps;
    p.choff = r->choff;
    p.chunk_table = r->chunk_table;
    p.pool = static_cast<const R*>(r->pool);
    p.queue = reinterpret_cast<int*>(scratch);
    p.perm = r->perm;
    p.bounds = bounds_of(r);
    auto kern = gs::k_adjoint<F, R, METHOD>;
    const size_t smem = adjoint_smem<F, R, METHOD>();
    if (smem > 48 * 1024)
      GS_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    int nb = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, BLOCK, smem) != cudaSuccess || nb < 1)
      nb = 1;
    const long long grid =
        std::max(1LL, std::min((long long)sms * nb, (long long)((N + BLOCK - 1) / BLOCK)));
    kern<<<(int)grid, BLOCK, smem, s>>>(p);
    if (shared) {
      gs::k_reduce_theta<R><<<nred, gs::RED_BLOCK, 0, s>>>(traj, (int)N, M, per_block, partials);
      gs::k_reduce_partials<R><<<1, 256, 0, s>>>(partials, nred, M, static_cast<R*>(dL_dtheta));
    }
    GS_CUDA(cudaGetLastError());
    return GS_OK;
  }
}

}  // namespace

extern "C" gs_status gs_replay_grad_noalloc(const gs_record* rec, const void* theta,
                                            const void* dL_dy1, void* dL_dtheta, void* dL_dy0,
                                            void* stream) {
  NvtxRange nvtx_range("gs_replay_grad_noalloc");
  if (!rec) return fail(GS_ERR_INVALID_ARG, "record is NULL");
  if (rec->N == 0) return GS_OK;
  if (!theta || !dL_dy1) return fail(GS_ERR_INVALID_ARG, "theta and dL_dy1 must be non-NULL");
  if (!dL_dtheta && !dL_dy0) return fail(GS_ERR_INVALID_ARG, "no output requested");
  if (rec->sys.field == GS_MLP_4_32_32_4)
    return fail(GS_ERR_UNSUPPORTED, "gs_replay_grad_noalloc does not take the MLP field");
  gs_status st = check_device({{theta, "theta"}, {dL_dy1, "dL_dy1"}, {dL_dtheta, "dL_dtheta"},
                               {dL_dy0, "dL_dy0"}});
  if (st != GS_OK) return st;
  const bool shared = rec->sys.theta_shared && dL_dtheta;
  const size_t nred = (size_t)((rec->N + 4095) / 4096);
  const size_t need = 256 + (shared ? ((size_t)rec->N + nred) * rec->sys.m * rec->rsz : 0);
  if (need > GS_NOALLOC_SCRATCH_BYTES)
    return fail(GS_ERR_CAPACITY,
                "gs_replay_grad_noalloc needs %zu bytes of scratch for N=%lld, m=%d; its fixed "
                "array holds %u bytes (use gs_replay_grad)",
                need, (long long)rec->N, rec->sys.m, GS_NOALLOC_SCRATCH_BYTES);
  NoallocDevice* d = nullptr;
  st = noalloc_setup(&d);
  if (st != GS_OK) return st;
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev != rec->device)
    return fail(GS_ERR_INVALID_ARG, "record belongs to device %d, current is %d", rec->device, dev);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  GS_CUDA(cudaMemsetAsync(d->ptr, 0, 128, s));  // both work counters start at zero
  st = refresh_states(const_cast<gs_record*>(rec), theta, reinterpret_cast<int*>(d->ptr + 64),
                      true, d->sms, s);
  if (st != GS_OK) return st;
  return dispatch(rec->sys, [&]<class F, class R, int METHOD>() {
    return noalloc_adjoint<F, R, METHOD>(rec, theta, dL_dy1, dL_dtheta, dL_dy0, d->ptr, d->sms, s);
  });
}
