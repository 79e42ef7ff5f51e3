// libmpzch: C ABI, table handle and launch orchestration for the Memory Layer
// table kernels (see include/mpzch.h for the contract of every entry point).
#include "mpzch.h"
#include "mpzch_internal.h"
#include "mpzch_kernels.cuh"
#include "mpzch_tier.cuh"

#include <cuda_runtime.h>

#include <atomic>
#include <cstdlib>
#include <utility>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

using namespace mpzch;

namespace {

std::atomic<int> g_fail_allocs{0};
std::atomic<int64_t> g_launches{0};

int dev_alloc(void** p, size_t bytes) {
  *p = nullptr;
  if (bytes == 0) return MPZCH_OK;
  if (g_fail_allocs.load() > 0) {
    g_fail_allocs.fetch_sub(1);
    return MPZCH_ENOMEM;
  }
  if (cudaMalloc(p, bytes) != cudaSuccess) {
    cudaGetLastError();
    *p = nullptr;
    return MPZCH_ENOMEM;
  }
  return MPZCH_OK;
}

void dev_free(void* p) {
  if (p) cudaFree(p);
}

// Pinned host memory mapped into the device address space, zero-filled: the
// kernels reach it over the host link with the same pointer arithmetic.
int host_mapped_alloc(void** dev_ptr, void** host_ptr, size_t bytes) {
  *dev_ptr = *host_ptr = nullptr;
  if (g_fail_allocs.load() > 0) {
    g_fail_allocs.fetch_sub(1);
    return MPZCH_ENOMEM;
  }
  if (cudaHostAlloc(host_ptr, bytes, cudaHostAllocMapped | cudaHostAllocPortable) != cudaSuccess) {
    cudaGetLastError();
    *host_ptr = nullptr;
    return MPZCH_ENOMEM;
  }
  std::memset(*host_ptr, 0, bytes);
  if (cudaHostGetDevicePointer(dev_ptr, *host_ptr, 0) != cudaSuccess) {
    cudaGetLastError();
    cudaFreeHost(*host_ptr);
    *host_ptr = nullptr;
    *dev_ptr = nullptr;
    return MPZCH_ECUDA;
  }
  return MPZCH_OK;
}

inline cudaStream_t S(void* s) { return reinterpret_cast<cudaStream_t>(s); }

int sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

// Grid for a grid-stride kernel: enough blocks for `work` threads, at most
// `per_sm` resident blocks on every SM.
unsigned grid_for(int64_t work_threads, int block, int per_sm = 8) {
  int64_t g = (work_threads + block - 1) / block;
  const int64_t cap = (int64_t)sm_count() * per_sm;
  if (g > cap) g = cap;
  if (g < 1) g = 1;
  return (unsigned)g;
}

// Blocks of `kern` (with `block` threads, `smem` dynamic bytes) resident on
// one SM, looked up once per kernel and device; at least 1.
int resident_blocks(const void* kern, int block, size_t smem) {
  struct Entry {
    const void* kern;
    int device, block;
    size_t smem;
    int blocks;
  };
  static std::mutex mu;
  static std::vector<Entry> done;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(mu);
  for (const Entry& e : done)
    if (e.kern == kern && e.device == dev && e.block == block && e.smem == smem) return e.blocks;
  int b = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kern, block, smem) != cudaSuccess) {
    cudaGetLastError();
    b = 1;
  }
  if (b < 1) b = 1;
  done.push_back({kern, dev, block, smem, b});
  return b;
}

int after_launch() {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return cudaGetLastError() == cudaSuccess ? MPZCH_OK : MPZCH_ECUDA;
}

// Raises a kernel's dynamic shared-memory limit to `bytes` on the current
// device, once per (kernel, device) and size: the attribute belongs to the
// kernel function on one device, so kernels sharing a signature (template
// instances) and devices are tracked separately.
int allow_dynamic_smem(const void* kern, size_t bytes) {
  struct Entry {
    const void* kern;
    int device;
    size_t bytes;
  };
  static std::mutex mu;
  static std::vector<Entry> done;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MPZCH_ECUDA;
  std::lock_guard<std::mutex> lock(mu);
  for (const Entry& e : done)
    if (e.kern == kern && e.device == dev && e.bytes >= bytes) return MPZCH_OK;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) !=
      cudaSuccess) {
    cudaGetLastError();
    return MPZCH_ECUDA;
  }
  done.push_back({kern, dev, bytes});
  return MPZCH_OK;
}

// Launches a kernel; with `pdl` it may start while the previous kernel of the
// stream drains (programmatic dependent launch: every kernel waits for its
// predecessors with griddepcontrol.wait before touching memory).
template <typename... KArgs, typename... Args>
int launch(void (*kern)(KArgs...), unsigned grid, unsigned block, cudaStream_t st, bool pdl,
           Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return MPZCH_ECUDA;
  }
  return MPZCH_OK;
}

template <typename... KArgs, typename... Args>
int launch_smem(void (*kern)(KArgs...), unsigned grid, unsigned block, size_t smem,
                cudaStream_t st, bool pdl, Args&&... args) {
  int rc = allow_dynamic_smem(reinterpret_cast<const void*>(kern), smem);
  if (rc) return rc;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return MPZCH_ECUDA;
  }
  return MPZCH_OK;
}

// Grid of a one-warp-per-row kernel over n rows: per_sm > 0 caps it at per_sm
// resident blocks per SM (grid-stride, long-lived blocks); per_sm == 0 gives
// one row per warp (short-lived blocks, so blocks of other streams find free
// slots while it runs).
unsigned row_grid(int64_t n, int per_sm) {
  if (per_sm > 0) return grid_for(n * 32, kBlock, per_sm);
  int64_t g = (n * 32 + kBlock - 1) / kBlock;
  if (g < 1) g = 1;
  if (g > 0x7FFFFFFF) g = 0x7FFFFFFF;
  return (unsigned)g;
}

uint64_t pow2_at_least(uint64_t x) {
  uint64_t p = 1;
  while (p < x) p <<= 1;
  return p;
}

Geo make_geo(int64_t C, int32_t P) {
  Geo g;
  g.C = C;
  g.pow2 = (C & (C - 1)) == 0;
  g.mask = g.pow2 ? (uint64_t)(C - 1) : 0;
  g.P = P;
  return g;
}

enum Phase { PH_LOOKUP = 0, PH_GATHER, PH_DEDUP, PH_INSERT, PH_WRITEBACK, PH_SELECT, PH_EXPORT };

}  // namespace

struct mpzch_table {
  int64_t C = 0;
  int32_t D = 0, P = 0;
  int device = 0;
  Geo geo{};
  // table state (row-indexed arrays)
  long long* keys = nullptr;
  long long* last = nullptr;
  float* M = nullptr;          // device-accessible address of the values
  void* M_host = nullptr;      // host allocation when the values live in host memory
  bool values_on_host = false;
  // insert scratch: three claim arrays of C slots (claim-round path)
  unsigned long long* claims[3] = {nullptr, nullptr, nullptr};
  // cluster placement path: tagged per-slot list heads (C slots) and the tag
  // of the last call (0 is never a call's tag; shead starts all zero)
  unsigned long long* shead = nullptr;
  int32_t* wentry = nullptr;  // write-list entry of each row's owner in the current step
  int emit_list = 1;          // cluster path: write list emitted at re-probe and placement
  uint32_t tag = 0;
  bool tag_wrapped = false;
  int cluster_insert = 1;
  // per-batch scratch, sized for `cap` ids
  int64_t cap = 0;
  uint64_t hmask = 0;
  unsigned long long* hkey = nullptr;
  uint32_t* hpos = nullptr;
  int32_t* hrow = nullptr;  // pre-insert row of each scratch-hash slot's id (train-step lookup)
  int32_t* slot_of = nullptr;
  int32_t* bcount = nullptr;
  long long* ukey = nullptr;
  // first positions and rows of the distinct ids, two sets used by alternate
  // Writebacks (on the cluster path they are the write list the row update reads)
  int32_t* upos[2] = {nullptr, nullptr};
  int32_t* urow[2] = {nullptr, nullptr};
  uint8_t* uhit[2] = {nullptr, nullptr};  // resident before the step, per distinct id
  uint8_t* whit[2] = {nullptr, nullptr};  // the same, aligned with the compacted write lists
  int32_t* snext = nullptr;  // next key of the same home slot (cluster path)
  long long* lkey[3] = {nullptr, nullptr, nullptr};  // insert round lists: keys
  int32_t* lidx[3] = {nullptr, nullptr, nullptr};    // and their distinct-id index
  // write lists (row, position of e), two buffers used by alternate Writebacks
  int32_t* wrow[2] = {nullptr, nullptr};
  int32_t* wpos[2] = {nullptr, nullptr};
  int32_t* wcnt = nullptr;  // device int32[4]: list lengths [0..1], entries taken [2..3]
  const void* prev_rows = nullptr;  // rows/hit buffers of the previous train step
  const void* prev_hit = nullptr;
  int wset = 0;             // buffer of the next Writeback
  // small device words
  StepCtr* ctr = nullptr;
  WbStats* stats = nullptr;  // used when the caller passes no stats buffer
  int32_t* status = nullptr;
  // select: per-tile ballot words and row counts
  uint32_t* sel_masks = nullptr;
  int32_t* sel_tcount = nullptr;
  int32_t* h_status = nullptr;  // pinned host word for mpzch_get_status
  int64_t last_step = -1;
  int wide_rounds = 3;  // grid-wide insert rounds before the single-block finisher
  int side_high_priority = 1;  // priority of the side stream (set before its first use)
  float eta = 1.0f;            // learning rate of the Writeback step
  int row_blocks_per_sm = 8;   // row kernels: 0 = one row per warp, else grid-stride cap
  int row_kernel = 0;          // 0 = rows through registers, 1 = bulk copies into shared memory
  int bulk_warps = 8;          // bulk row kernels: warps per block
  int bulk_blocks = 1;         // bulk row kernels: blocks per SM (persistent grid)
  int l2_hint_rows = 0;        // bulk row kernels: L2 policy of table-row accesses (L2Hint)
  // hot/cold tier (values in host memory): HBM cache of tier_rows rows, 0 = none
  int64_t tier_rows = 0;
  Tier tier{};
  // mpzch_train_step: the row map runs on a second (high-priority) stream
  cudaStream_t side = nullptr;
  cudaEvent_t ev_fork = nullptr, ev_lookup = nullptr, ev_map = nullptr;
  cudaEvent_t ev_update[2] = {nullptr, nullptr};  // row update that read write list b
  cudaEvent_t ev_user = nullptr;    // end of every other call so far (created with the table)
  cudaStream_t user_stream = nullptr;  // stream ev_user was last recorded on
  bool user_marked = false;
  cudaEvent_t ev_gather = nullptr;  // end of the last train step's gather
  // tracing
  bool trace = false;
  struct Rec {
    cudaEvent_t a, b;
    int phase;
  };
  std::vector<Rec> pending;
  std::vector<cudaEvent_t> pool;
  double ms[MPZCH_NPHASES] = {0};
  int64_t launches[MPZCH_NPHASES] = {0};
};

namespace {

void free_batch_scratch(mpzch_table* t) {
  dev_free(t->hkey);
  dev_free(t->hpos);
  dev_free(t->hrow);
  t->hrow = nullptr;
  dev_free(t->slot_of);
  dev_free(t->bcount);
  dev_free(t->ukey);
  for (auto& l : t->upos) dev_free(l), l = nullptr;
  for (auto& l : t->urow) dev_free(l), l = nullptr;
  for (auto& l : t->uhit) dev_free(l), l = nullptr;
  for (auto& l : t->whit) dev_free(l), l = nullptr;
  dev_free(t->snext);
  t->snext = nullptr;
  for (auto& l : t->lkey) dev_free(l), l = nullptr;
  for (auto& l : t->lidx) dev_free(l), l = nullptr;
  for (auto& l : t->wrow) dev_free(l), l = nullptr;
  for (auto& l : t->wpos) dev_free(l), l = nullptr;
  t->hkey = nullptr;
  t->hpos = nullptr;
  t->slot_of = t->bcount = nullptr;
  t->ukey = nullptr;
  t->cap = 0;
  t->hmask = 0;
}

void free_all(mpzch_table* t) {
  free_batch_scratch(t);
  dev_free(t->keys);
  dev_free(t->last);
  if (t->M_host)
    cudaFreeHost(t->M_host);
  else
    dev_free(t->M);
  for (auto& c : t->claims) dev_free(c), c = nullptr;
  dev_free(t->shead);
  dev_free(t->wentry);
  dev_free(t->tier.cache);
  dev_free(t->tier.owner);
  dev_free(t->tier.won);
  dev_free(t->tier.claim);
  dev_free(t->tier.stats);
  dev_free(t->ctr);
  dev_free(t->wcnt);
  dev_free(t->stats);
  dev_free(t->status);
  dev_free(t->sel_masks);
  dev_free(t->sel_tcount);
  if (t->h_status) cudaFreeHost(t->h_status);
  for (auto& r : t->pending) {
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
  }
  for (auto e : t->pool) cudaEventDestroy(e);
  if (t->ev_fork) cudaEventDestroy(t->ev_fork);
  if (t->ev_lookup) cudaEventDestroy(t->ev_lookup);
  if (t->ev_map) cudaEventDestroy(t->ev_map);
  for (auto& e : t->ev_update)
    if (e) cudaEventDestroy(e);
  if (t->ev_user) cudaEventDestroy(t->ev_user);
  if (t->ev_gather) cudaEventDestroy(t->ev_gather);
  if (t->side) cudaStreamDestroy(t->side);
}

int ensure_side_stream(mpzch_table* t) {
  if (t->side) return MPZCH_OK;
  int least = 0, greatest = 0;
  if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess ||
      cudaStreamCreateWithPriority(&t->side, cudaStreamNonBlocking,
                                   t->side_high_priority ? greatest : least) != cudaSuccess ||
      cudaEventCreateWithFlags(&t->ev_fork, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&t->ev_lookup, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&t->ev_map, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&t->ev_update[0], cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&t->ev_update[1], cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&t->ev_gather, cudaEventDisableTiming) != cudaSuccess) {
    cudaGetLastError();
    return MPZCH_ECUDA;
  }
  return MPZCH_OK;
}

// Grow the per-batch scratch to hold batches of n ids.
int ensure_batch(mpzch_table* t, int64_t n, cudaStream_t st) {
  if (n <= t->cap) return MPZCH_OK;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) return MPZCH_ECUDA;
  if (cs != cudaStreamCaptureStatusNone) return MPZCH_ECAPTURE;
  int64_t cap = n < 4096 ? 4096 : n;
  // The old scratch may still be in use by queued work.
  if (t->cap > 0 && cudaDeviceSynchronize() != cudaSuccess) return MPZCH_ECUDA;
  free_batch_scratch(t);
  const uint64_t H = pow2_at_least((uint64_t)cap * 2);
  const int64_t tiles = (cap + kTile - 1) / kTile + 1;
  int rc = MPZCH_OK;
  if (!rc) rc = dev_alloc((void**)&t->hkey, H * sizeof(unsigned long long));
  if (!rc) rc = dev_alloc((void**)&t->hpos, H * sizeof(uint32_t));
  if (!rc) rc = dev_alloc((void**)&t->hrow, H * sizeof(int32_t));
  if (!rc) rc = dev_alloc((void**)&t->slot_of, cap * sizeof(int32_t));
  if (!rc) rc = dev_alloc((void**)&t->bcount, tiles * sizeof(int32_t));
  if (!rc) rc = dev_alloc((void**)&t->ukey, cap * sizeof(long long));
  for (int i = 0; i < 2 && !rc; ++i) rc = dev_alloc((void**)&t->upos[i], cap * sizeof(int32_t));
  for (int i = 0; i < 2 && !rc; ++i) rc = dev_alloc((void**)&t->urow[i], cap * sizeof(int32_t));
  for (int i = 0; i < 2 && !rc; ++i) rc = dev_alloc((void**)&t->uhit[i], cap);
  for (int i = 0; i < 2 && !rc; ++i) rc = dev_alloc((void**)&t->whit[i], cap);
  if (!rc) rc = dev_alloc((void**)&t->snext, cap * sizeof(int32_t));
  for (int i = 0; i < 3 && !rc; ++i) rc = dev_alloc((void**)&t->lkey[i], cap * sizeof(long long));
  for (int i = 0; i < 3 && !rc; ++i) rc = dev_alloc((void**)&t->lidx[i], cap * sizeof(int32_t));
  for (int i = 0; i < 2 && !rc; ++i) rc = dev_alloc((void**)&t->wrow[i], cap * sizeof(int32_t));
  for (int i = 0; i < 2 && !rc; ++i) rc = dev_alloc((void**)&t->wpos[i], cap * sizeof(int32_t));
  if (rc) {
    free_batch_scratch(t);
    return rc;
  }
  // Scratch hash: empty key (-1) and empty position (all ones).  The fill is
  // waited for here: the helper streams of mpzch_train_step are not ordered
  // after `st` when the caller passes an inputs-ready event, so they must not
  // find the fill still queued (growth is rare and already synchronises).
  if (cudaMemsetAsync(t->hkey, 0xFF, H * sizeof(unsigned long long), st) != cudaSuccess ||
      cudaMemsetAsync(t->hpos, 0xFF, H * sizeof(uint32_t), st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess) {
    cudaGetLastError();
    free_batch_scratch(t);
    return MPZCH_ECUDA;
  }
  t->cap = cap;
  t->hmask = H - 1;
  return MPZCH_OK;
}

bool on_device(const mpzch_table* t) {
  int d = -1;
  return cudaGetDevice(&d) == cudaSuccess && d == t->device;
}

cudaEvent_t take_event(mpzch_table* t) {
  if (!t->pool.empty()) {
    cudaEvent_t e = t->pool.back();
    t->pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

// Brackets the launches of one phase with events when tracing is on.
struct PhaseScope {
  mpzch_table* t;
  int phase;
  cudaStream_t st;
  cudaEvent_t a = nullptr;
  int64_t start_launches;
  PhaseScope(mpzch_table* t_, int ph, cudaStream_t s) : t(t_), phase(ph), st(s) {
    start_launches = g_launches.load();
    if (t->trace) {
      a = take_event(t);
      cudaEventRecord(a, st);
    }
  }
  ~PhaseScope() {
    t->launches[phase] += g_launches.load() - start_launches;
    if (t->trace && a) {
      cudaEvent_t b = take_event(t);
      cudaEventRecord(b, st);
      t->pending.push_back({a, b, phase});
    }
  }
};

// The three dedup phases.
int run_dedup(mpzch_table* t, const int64_t* ids, int64_t n, long long* uniq, int32_t* pos,
              long long* dev_count, WbStats* stats, cudaStream_t st) {
  const long long* id = reinterpret_cast<const long long*>(ids);
  const unsigned tiles = (unsigned)((n + kTile - 1) / kTile);
  k_dedup_insert<<<tiles, kDedupThreads, 0, st>>>(id, n, t->hkey, t->hpos, t->hmask, t->slot_of, t->ctr,
                                           stats, t->status, nullptr, nullptr);
  if (after_launch()) return MPZCH_ECUDA;
  k_dedup_count<<<tiles, kBlock, 0, st>>>(t->slot_of, t->hpos, n, t->bcount);
  if (after_launch()) return MPZCH_ECUDA;
  k_dedup_compact<<<tiles, kBlock, 0, st>>>(id, n, t->slot_of, t->hkey, t->hpos, t->bcount, uniq,
                                            pos, dev_count, stats);
  return after_launch();
}

}  // namespace

namespace {

// Select in two launches (marks + counts, then offsets + scatter), the second
// with programmatic dependent launch.
int launch_select(mpzch_table* t, int64_t since, int32_t* rows_out, int64_t* dev_count,
                  cudaStream_t st) {
  const unsigned tiles = (unsigned)((t->C + kScanTile - 1) / kScanTile);
  int rc = launch(k_select_mark, tiles, kScanThreads, st, false, (const long long*)t->keys,
                  (const long long*)t->last, t->C, (long long)since, t->sel_masks,
                  t->sel_tcount);
  if (!rc)
    rc = launch(k_select_scatter, tiles, kScanThreads, st, true, (const uint32_t*)t->sel_masks,
                (const int32_t*)t->sel_tcount, t->C, rows_out,
                reinterpret_cast<long long*>(dev_count));
  return rc;
}

int enqueue_lookup(mpzch_table* t, const int64_t* ids, int64_t n, int32_t* rows, uint8_t* hit,
                   cudaStream_t st, bool pdl) {
  PhaseScope ps(t, PH_LOOKUP, st);
  int G = (int)pow2_at_least((uint64_t)t->P);
  if (G > 32) G = 32;
  return launch(k_lookup, grid_for(n * G, kBlock), kBlock, st, pdl,
                reinterpret_cast<const long long*>(ids), n, (const long long*)t->keys, t->geo, G,
                rows, hit, t->status);
}

int check_gather(mpzch_table* t, const int32_t* rows, const uint8_t* hit, int64_t n,
                 const float* ao_table, int64_t ao_nrows, int32_t ao_dim, const int32_t* ao_rows,
                 const float* out) {
  if (!t || n < 0 || n > 0x7FFFFFFFLL) return MPZCH_EINVAL;
  const bool has_ao = ao_table != nullptr;
  if (has_ao && (ao_dim <= 0 || ao_dim % 4 != 0 || ao_nrows <= 0 || !ao_rows)) return MPZCH_EINVAL;
  if (!has_ao && (ao_dim != 0 || ao_rows)) return MPZCH_EINVAL;
  if (n == 0) return MPZCH_OK;
  if (!rows || !hit || !out || !on_device(t)) return MPZCH_EINVAL;
  if ((reinterpret_cast<uintptr_t>(out) & 15) ||
      (has_ao && (reinterpret_cast<uintptr_t>(ao_table) & 15)))
    return MPZCH_EINVAL;
  return MPZCH_OK;
}

// Launch shape of a bulk row kernel with `stage_bytes` per stage: warps per
// block (halved until the block's shared memory fits kBulkSmemMax) and its
// shared memory; false when even one warp does not fit (the register kernel
// runs instead), or when the values live in host memory.
constexpr size_t kBulkSmemMax = 112 * 1024;

bool bulk_shape(const mpzch_table* t, size_t stage_bytes, int* warps, size_t* smem) {
  if (t->row_kernel != 1 || t->values_on_host) return false;
  for (int w = t->bulk_warps; w >= 1; w >>= 1) {
    const size_t b = bulk_smem_bytes(w, stage_bytes);
    if (b <= kBulkSmemMax) {
      *warps = w;
      *smem = b;
      return true;
    }
  }
  return false;
}

int enqueue_gather(mpzch_table* t, const int32_t* rows, const uint8_t* hit, int64_t n,
                   const float* ao_table, int64_t ao_nrows, int32_t ao_dim,
                   const int32_t* ao_rows, float* out, cudaStream_t st, bool pdl) {
  PhaseScope ps(t, PH_GATHER, st);
  const bool has_ao = ao_table != nullptr;
  if (t->tier_rows > 0) {
    const int W4 = t->D / 4 + (has_ao ? ao_dim / 4 : 0);
    const int vec = W4 > 32 * kTierGatherVecMax ? kTierGatherVecMax : (W4 + 31) / 32;
    auto go = [&](auto kern) {
      // one resident wave, grid-stride over the rows
      int per_sm = t->row_blocks_per_sm;
      if (per_sm > 0) {
        const int res = resident_blocks(reinterpret_cast<const void*>(kern), kBlock, 0);
        if (per_sm > res) per_sm = res;
      }
      return launch(kern, row_grid(n, per_sm), kBlock, st, pdl, rows, hit, n, t->tier,
                    reinterpret_cast<const float4*>(t->M), t->C, t->D / 4,
                    reinterpret_cast<const float4*>(ao_table), ao_nrows, has_ao ? ao_dim / 4 : 0,
                    ao_rows, reinterpret_cast<float4*>(out), t->status);
    };
    switch (vec) {
      case 1: return go(k_tier_gather<1>);
      case 2: return go(k_tier_gather<2>);
      case 3: return go(k_tier_gather<3>);
      case 4: return go(k_tier_gather<4>);
      case 5: return go(k_tier_gather<5>);
      case 6: return go(k_tier_gather<6>);
      case 7: return go(k_tier_gather<7>);
      default: return go(k_tier_gather<kTierGatherVecMax>);
    }
  }
  int warps = 0;
  size_t smem = 0;
  if (bulk_shape(t, (size_t)(t->D + (has_ao ? ao_dim : 0)) * 4, &warps, &smem)) {
    int64_t g = (int64_t)sm_count() * t->bulk_blocks;
    const int64_t need = (n + warps - 1) / warps;
    if (g > need) g = need;
    return launch_smem(k_gather_bulk, (unsigned)g, (unsigned)(warps * 32), smem, st, pdl, rows,
                       hit, n, reinterpret_cast<const float4*>(t->M), t->C, t->D / 4,
                       reinterpret_cast<const float4*>(ao_table), ao_nrows,
                       has_ao ? ao_dim / 4 : 0, ao_rows, reinterpret_cast<float4*>(out),
                       t->l2_hint_rows, t->status);
  }
  // at most one resident wave: the blocks a second, partial wave would add
  // only start as the first wave's finish, and the step waits for them
  int per_sm = t->row_blocks_per_sm;
  if (per_sm > 0) {
    const int res = resident_blocks(reinterpret_cast<const void*>(k_gather_fused), kBlock, 0);
    if (per_sm > res) per_sm = res;
  }
  return launch(k_gather_fused, row_grid(n, per_sm), kBlock, st, pdl, rows, hit, n,
                reinterpret_cast<const float4*>(t->M), t->C, t->D / 4,
                reinterpret_cast<const float4*>(ao_table), ao_nrows, has_ao ? ao_dim / 4 : 0,
                ao_rows, reinterpret_cast<float4*>(out), t->status);
}

int check_writeback(mpzch_table* t, const int64_t* ids, const float* e, int64_t n, int64_t step) {
  if (!t || n < 0 || n > 0x7FFFFFFFLL) return MPZCH_EINVAL;
  if (step <= t->last_step) return MPZCH_EINVAL;
  if (t->tier_rows > 0 && step >= (int64_t)1 << 31) return MPZCH_EINVAL;  // claim words hold 31 bits
  if (n > 0 && (!ids || !e)) return MPZCH_EINVAL;
  if (!on_device(t)) return MPZCH_EINVAL;
  if (reinterpret_cast<uintptr_t>(e) & 15) return MPZCH_EINVAL;
  return MPZCH_OK;
}

WbParams make_params(mpzch_table* t, const int64_t* ids, const float* e, int64_t n, int64_t step,
                     WbStats* stats) {
  WbParams p;
  p.ids = reinterpret_cast<const long long*>(ids);
  p.n = n;
  p.e = reinterpret_cast<const float4*>(e);
  p.D4 = t->D / 4;
  p.hkey = t->hkey;
  p.hpos = t->hpos;
  p.hrow = t->hrow;
  p.n_fill = 0;
  p.fill_rows = nullptr;
  p.fill_hit = nullptr;
  p.hmask = t->hmask;
  p.slot_of = t->slot_of;
  p.ukey = t->ukey;
  p.upos = t->upos[t->wset];
  p.urow = t->urow[t->wset];
  p.keys = t->keys;
  p.last = t->last;
  p.M = reinterpret_cast<float4*>(t->M);
  p.g = t->geo;
  p.step = (long long)step;
  for (int i = 0; i < 3; ++i) {
    p.lkey[i] = t->lkey[i];
    p.lidx[i] = t->lidx[i];
    p.claims[i] = t->claims[i];
  }
  p.ctr = t->ctr;
  p.stats = stats;
  p.status = t->status;
  p.wide_rounds = t->wide_rounds;
  p.cluster = t->cluster_insert;
  if (++t->tag == 0) {  // 2^32 calls: old entries could alias the new tag
    t->tag = 1;
    t->tag_wrapped = true;
  }
  p.tag = t->tag;
  p.shead = t->shead;
  p.snext = t->snext;
  p.wcount = t->wcnt + t->wset;
  p.wtake = t->wcnt + 2 + t->wset;
  p.emit = (t->cluster_insert && t->emit_list) ? 1 : 0;
  p.wentry = t->wentry;
  // emit: the distinct-id arrays are the list; otherwise k_write_list fills
  // the compacted buffers
  p.wrow = p.emit ? p.urow : t->wrow[t->wset];
  p.wpos = p.emit ? p.upos : t->wpos[t->wset];
  p.uhit = t->uhit[t->wset];
  p.whit = p.emit ? p.uhit : t->whit[t->wset];
  return p;
}

// Row map of one Writeback on stream `st`: dedup + re-probe + refresh, then
// the inserts (and, on the claim-round path or without emitted lists, the
// write list).  With p.n_fill > 0 (train step) the first n_fill positions'
// lookup results are filled from the re-probe, after `fill_after` (the
// previous gather, which may still read the same rows/hit buffers), and
// `fill_done` is recorded once they are written.
int enqueue_row_map(mpzch_table* t, const WbParams& p, cudaStream_t st, cudaEvent_t fill_after,
                    cudaEvent_t fill_done) {
  const int64_t n = p.n;
  int rc;
  if (t->tag_wrapped) {
    if (cudaMemsetAsync(t->shead, 0, t->C * sizeof(unsigned long long), st) != cudaSuccess)
      return MPZCH_ECUDA;
    t->tag_wrapped = false;
  }
  {
    PhaseScope ps(t, PH_DEDUP, st);
    rc = launch(k_dedup_insert, (unsigned)((n + kTile - 1) / kTile), kDedupThreads, st, false,
                p.ids, n, t->hkey, t->hpos, t->hmask, t->slot_of, t->ctr, p.stats, t->status,
                p.wcount, p.wtake);
    if (!rc) rc = launch(k_first_reprobe, grid_for(n, kBlock), kBlock, st, true, p);
    if (rc) return rc;
  }
  const bool wait = p.n_fill > 0 && fill_after;
  if (wait && cudaStreamWaitEvent(st, fill_after, 0) != cudaSuccess) return MPZCH_ECUDA;
  if (p.cluster) {
    // cluster placement (its first pass also fills the lookup); the
    // single-block finisher only acts when the windows may cover the whole
    // ring or a cluster exceeds the warp path
    PhaseScope ps(t, PH_INSERT, st);
    const bool recorded = p.n_fill > 0 && fill_done;
    rc = launch(k_place_clusters, grid_for(n, kBlock, 4), kBlock, st, !wait, p);
    if (!rc && recorded && cudaEventRecord(fill_done, st) != cudaSuccess) rc = MPZCH_ECUDA;
    // one warp per multi-key cluster, as many resident warps as the SMs hold
    const int multi_per_sm = resident_blocks(reinterpret_cast<const void*>(k_place_multi), kBlock, 0);
    if (!rc)
      rc = launch(k_place_multi, grid_for(n * 32, kBlock, multi_per_sm), kBlock, st, !recorded, p);
    if (!rc) rc = launch_smem(k_insert_finish, 1, 1024, kClusterSmem, st, true, p, 0);
    if (!rc && !p.emit) rc = launch(k_write_list, grid_for(n, kBlock, 4), kBlock, st, true, p);
    return rc;
  }
  {
    PhaseScope ps(t, PH_INSERT, st);
    if (p.n_fill > 0) {
      rc = launch(k_lookup_fill, grid_for(p.n_fill, kBlock), kBlock, st, !wait, p);
      if (!rc && fill_done && cudaEventRecord(fill_done, st) != cudaSuccess) rc = MPZCH_ECUDA;
    }
    const unsigned grid = grid_for(n, kBlock, 4);
    for (int r = 0; r < t->wide_rounds && !rc; ++r)
      rc = launch(k_insert_round, grid, kBlock, st, r > 0 || (!wait && p.n_fill == 0), p, r);
    if (!rc)
      rc = launch_smem(k_insert_finish, 1, 1024, kClusterSmem, st,
                       t->wide_rounds > 0 || p.n_fill == 0, p, t->wide_rounds);
    if (!rc) rc = launch(k_write_list, grid_for(n, kBlock, 4), kBlock, st, true, p);
  }
  return rc;
}

int enqueue_row_update(mpzch_table* t, const WbParams& p, cudaStream_t st, bool pdl) {
  {
    PhaseScope ps(t, PH_WRITEBACK, st);
    int warps = 0;
    size_t smem = 0;
    int rc;
    if (t->tier_rows > 0) {
      // claims, evictions, then the update (three passes over the write list)
      const unsigned g = row_grid(p.n, t->row_blocks_per_sm);
      float4* host = p.M;
      rc = launch(k_tier_claim, grid_for(p.n, kBlock), kBlock, st, pdl, (const int32_t*)p.wrow,
                  (const uint8_t*)p.whit, (const int32_t*)p.wcount, t->tier, (long long)p.step);
      if (!rc)
        rc = launch(k_tier_evict, g, kBlock, st, true, (const int32_t*)p.wrow,
                    (const int32_t*)p.wcount, t->tier, host, p.D4, (long long)p.step);
      if (!rc)
        rc = launch(k_tier_update, g, kBlock, st, true, (const int32_t*)p.wrow,
                    (const int32_t*)p.wpos, (const int32_t*)p.wcount, t->tier, host, p.e, p.D4,
                    t->eta, (long long)p.step);
    } else if (bulk_shape(t, (size_t)t->D * 8, &warps, &smem)) {
      int64_t g = (int64_t)sm_count() * t->bulk_blocks;
      const int64_t need = (p.n + 32 * warps - 1) / (32 * warps);
      if (g > need) g = need;
      rc = launch_smem(k_writeback_bulk, (unsigned)g, (unsigned)(warps * 32), smem, st, pdl,
                       (const int32_t*)p.wrow, (const int32_t*)p.wpos, (const int32_t*)p.wcount,
                       p.wtake, p.M, p.e, p.D4, t->eta, t->l2_hint_rows, t->status);
    } else {
      rc = launch(k_writeback, row_grid(p.n, t->row_blocks_per_sm), kBlock, st, pdl,
                  (const int32_t*)p.wrow, (const int32_t*)p.wpos, (const int32_t*)p.wcount, p.M,
                  p.e, p.D4, t->eta);
    }
    if (rc) return rc;
  }
  if (t->side && cudaEventRecord(t->ev_update[t->wset], st) != cudaSuccess) return MPZCH_ECUDA;
  t->wset ^= 1;
  return MPZCH_OK;
}

// Calls other than mpzch_train_step run on the caller's stream: they first
// wait for the side stream's work, and the next train step's helper streams
// wait for them (ev_user).
int join_side(mpzch_table* t, cudaStream_t st) {
  if (!t->side) return MPZCH_OK;
  return cudaStreamWaitEvent(st, t->ev_map, 0) == cudaSuccess ? MPZCH_OK : MPZCH_ECUDA;
}

// ev_user marks the end of every call made so far outside mpzch_train_step.
// A call on a stream other than the previous one first makes that stream wait
// for the old mark, so the new mark also covers the calls on the old stream.
int mark_user(mpzch_table* t, cudaStream_t st, int rc) {
  if (rc) return rc;
  if (t->user_marked && st != t->user_stream &&
      cudaStreamWaitEvent(st, t->ev_user, 0) != cudaSuccess)
    return MPZCH_ECUDA;
  if (cudaEventRecord(t->ev_user, st) != cudaSuccess) return MPZCH_ECUDA;
  t->user_marked = true;
  t->user_stream = st;
  return MPZCH_OK;
}

}  // namespace

// ---------------------------------------------------------------------------
// Scratch of mpzch_dedup_static: a fixed static device array, so that call
// never allocates.  Layout (256-byte aligned sections), for at most
// MPZCH_DEDUP_STATIC_MAX_IDS ids:
//   hash keys   8 B x kStaticHash   (all ones = empty)
//   hash pos    4 B x kStaticHash   (all ones = none)
//   slot_of     4 B x max ids
//   tile counts 4 B x (max ids / kTile + 1)
//   StepCtr     (cleared by k_dedup_insert)
// ---------------------------------------------------------------------------
namespace {
constexpr int64_t kStaticMaxIds = MPZCH_DEDUP_STATIC_MAX_IDS;
constexpr uint64_t kStaticHash = 2 * (uint64_t)kStaticMaxIds;  // a power of two
static_assert((kStaticHash & (kStaticHash - 1)) == 0, "static hash size must be a power of two");
constexpr size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }
constexpr size_t kOffHkey = 0;
constexpr size_t kOffHpos = align256(kOffHkey + 8 * kStaticHash);
constexpr size_t kOffSlot = align256(kOffHpos + 4 * kStaticHash);
constexpr size_t kOffBcnt = align256(kOffSlot + 4 * (size_t)kStaticMaxIds);
constexpr size_t kOffCtr = align256(kOffBcnt + 4 * (size_t)(kStaticMaxIds / kTile + 1));
constexpr size_t kStaticBytes = align256(kOffCtr + sizeof(StepCtr));
}  // namespace

static __device__ __align__(256) unsigned char g_dedup_scratch[kStaticBytes];

namespace {
std::mutex g_static_mu;
constexpr int kMaxDevices = 64;
void* g_static_addr[kMaxDevices] = {};

// Device address of g_dedup_scratch on the current device, looked up once per
// device.  (In host code the array's name is only a host-side stand-in.)
int static_scratch(unsigned char** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return MPZCH_ECUDA;
  }
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (!g_static_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dedup_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return MPZCH_ECUDA;
    }
    g_static_addr[dev] = p;
  }
  *out = static_cast<unsigned char*>(g_static_addr[dev]);
  return MPZCH_OK;
}
}  // namespace

extern "C" {

int mpzch_dedup_static(const int64_t* ids, int64_t n, int64_t* uniq, int32_t* pos,
                       int64_t* dev_count, int32_t* dev_status, void* stream) {
  if (n < 0 || !dev_count) return MPZCH_EINVAL;
  if (n > kStaticMaxIds) return MPZCH_ERANGE;
  if (n > 0 && (!ids || !uniq || !pos)) return MPZCH_EINVAL;
  unsigned char* base = nullptr;
  int rc = static_scratch(&base);
  if (rc) return rc;
  cudaStream_t st = S(stream);
  if (n == 0)
    return cudaMemsetAsync(dev_count, 0, sizeof(int64_t), st) == cudaSuccess ? MPZCH_OK
                                                                              : MPZCH_ECUDA;
  unsigned long long* hkey = reinterpret_cast<unsigned long long*>(base + kOffHkey);
  uint32_t* hpos = reinterpret_cast<uint32_t*>(base + kOffHpos);
  int32_t* slot_of = reinterpret_cast<int32_t*>(base + kOffSlot);
  int32_t* bcount = reinterpret_cast<int32_t*>(base + kOffBcnt);
  StepCtr* ctr = reinterpret_cast<StepCtr*>(base + kOffCtr);
  // Hash of 2^k >= 2n slots; clear only that part (the rest is not read).
  uint64_t H = pow2_at_least((uint64_t)n * 2);
  if (H < 1024) H = 1024;
  if (cudaMemsetAsync(hkey, 0xFF, H * sizeof(unsigned long long), st) != cudaSuccess ||
      cudaMemsetAsync(hpos, 0xFF, H * sizeof(uint32_t), st) != cudaSuccess)
    return MPZCH_ECUDA;
  const long long* id = reinterpret_cast<const long long*>(ids);
  const unsigned tiles = (unsigned)((n + kTile - 1) / kTile);
  k_dedup_insert<<<tiles, kDedupThreads, 0, st>>>(id, n, hkey, hpos, H - 1, slot_of, ctr, nullptr,
                                           dev_status, nullptr, nullptr);
  if (after_launch()) return MPZCH_ECUDA;
  k_dedup_count<<<tiles, kBlock, 0, st>>>(slot_of, hpos, n, bcount);
  if (after_launch()) return MPZCH_ECUDA;
  k_dedup_compact<<<tiles, kBlock, 0, st>>>(id, n, slot_of, hkey, hpos, bcount,
                                            reinterpret_cast<long long*>(uniq), pos,
                                            reinterpret_cast<long long*>(dev_count), nullptr);
  return after_launch();
}

int mpzch_create(int64_t capacity, int32_t dim, int32_t probes, void* stream, mpzch_table** out) {
  return mpzch_create_ex(capacity, dim, probes, 0u, stream, out);
}

int mpzch_create_ex(int64_t capacity, int32_t dim, int32_t probes, uint32_t flags, void* stream,
                    mpzch_table** out) {
  if (!out) return MPZCH_EINVAL;
  *out = nullptr;
  if (capacity < 1 || capacity > 0x7FFFFFFFLL || dim <= 0 || dim % 4 != 0 || probes < 1 ||
      (int64_t)probes > capacity || (flags & ~(uint32_t)MPZCH_VALUES_IN_HOST_MEMORY))
    return MPZCH_EINVAL;
  mpzch_table* t = new (std::nothrow) mpzch_table;
  if (!t) return MPZCH_ENOMEM;
  t->C = capacity;
  t->D = dim;
  t->P = probes;
  t->geo = make_geo(capacity, probes);
  t->values_on_host = (flags & MPZCH_VALUES_IN_HOST_MEMORY) != 0;
  cudaStream_t st = S(stream);
  int rc = MPZCH_OK;
  if (!rc) rc = dev_alloc((void**)&t->keys, capacity * sizeof(long long));
  if (!rc) rc = dev_alloc((void**)&t->last, capacity * sizeof(long long));
  if (!rc) {
    const size_t bytes = (size_t)capacity * dim * sizeof(float);
    if (t->values_on_host)
      rc = host_mapped_alloc((void**)&t->M, &t->M_host, bytes);
    else
      rc = dev_alloc((void**)&t->M, bytes);
  }
  for (int i = 0; i < 3 && !rc; ++i)
    rc = dev_alloc((void**)&t->claims[i], capacity * sizeof(unsigned long long));
  if (!rc) rc = dev_alloc((void**)&t->shead, capacity * sizeof(unsigned long long));
  if (!rc) rc = dev_alloc((void**)&t->wentry, capacity * sizeof(int32_t));
  if (!rc) rc = dev_alloc((void**)&t->ctr, sizeof(StepCtr));
  if (!rc) rc = dev_alloc((void**)&t->wcnt, 4 * sizeof(int32_t));
  if (!rc) rc = dev_alloc((void**)&t->stats, sizeof(WbStats));
  if (!rc) rc = dev_alloc((void**)&t->status, sizeof(int32_t));
  const int64_t sel_tiles = (capacity + kScanTile - 1) / kScanTile;
  if (!rc) rc = dev_alloc((void**)&t->sel_masks, sel_tiles * kScanWords * sizeof(uint32_t));
  if (!rc) rc = dev_alloc((void**)&t->sel_tcount, sel_tiles * sizeof(int32_t));
  if (!rc && cudaHostAlloc((void**)&t->h_status, sizeof(int32_t), cudaHostAllocDefault) != cudaSuccess) {
    t->h_status = nullptr;
    rc = MPZCH_ENOMEM;
  }
  if (!rc && cudaGetDevice(&t->device) != cudaSuccess) rc = MPZCH_ECUDA;
  if (!rc && cudaEventCreateWithFlags(&t->ev_user, cudaEventDisableTiming) != cudaSuccess)
    rc = MPZCH_ECUDA;
  if (!rc) {
    bool ok = cudaMemsetAsync(t->keys, 0xFF, capacity * sizeof(long long), st) == cudaSuccess &&
              cudaMemsetAsync(t->last, 0xFF, capacity * sizeof(long long), st) == cudaSuccess &&
              (t->values_on_host ||
               cudaMemsetAsync(t->M, 0, (size_t)capacity * dim * sizeof(float), st) ==
                   cudaSuccess) &&
              cudaMemsetAsync(t->ctr, 0, sizeof(StepCtr), st) == cudaSuccess &&
              cudaMemsetAsync(t->wcnt, 0, 4 * sizeof(int32_t), st) == cudaSuccess &&
              cudaMemsetAsync(t->shead, 0, capacity * sizeof(unsigned long long), st) ==
                  cudaSuccess &&
              cudaMemsetAsync(t->stats, 0, sizeof(WbStats), st) == cudaSuccess &&
              cudaMemsetAsync(t->status, 0, sizeof(int32_t), st) == cudaSuccess;
    for (int i = 0; i < 3 && ok; ++i)
      ok = cudaMemsetAsync(t->claims[i], 0xFF, capacity * sizeof(unsigned long long), st) ==
           cudaSuccess;
    // the table is complete when the call returns: later calls on other
    // streams (the helper streams of a pipelined train step) need no order
    // after `stream`
    if (ok) ok = cudaStreamSynchronize(st) == cudaSuccess;
    if (!ok) rc = MPZCH_ECUDA;
  }
  if (rc) {
    if (rc == MPZCH_ECUDA) cudaGetLastError();
    free_all(t);
    delete t;
    return rc;
  }
  *out = t;
  return MPZCH_OK;
}

int mpzch_destroy(mpzch_table* t) {
  if (!t) return MPZCH_OK;
  cudaDeviceSynchronize();
  free_all(t);
  delete t;
  return MPZCH_OK;
}

int mpzch_reserve(mpzch_table* t, int64_t max_batch, void* stream) {
  if (!t || max_batch < 0 || max_batch > 0x7FFFFFFFLL) return MPZCH_EINVAL;
  if (!on_device(t)) return MPZCH_EINVAL;
  return ensure_batch(t, max_batch, S(stream));
}

int mpzch_lookup(mpzch_table* t, const int64_t* ids, int64_t n, int32_t* rows, uint8_t* hit,
                 void* stream) {
  if (!t || n < 0 || n > 0x7FFFFFFFLL) return MPZCH_EINVAL;
  if (n == 0) return MPZCH_OK;
  if (!ids || !rows || !hit || !on_device(t)) return MPZCH_EINVAL;
  cudaStream_t st = S(stream);
  int rc = join_side(t, st);
  if (!rc) rc = enqueue_lookup(t, ids, n, rows, hit, st, false);
  return mark_user(t, st, rc);
}

int mpzch_gather_fused(mpzch_table* t, const int32_t* rows, const uint8_t* hit, int64_t n,
                       const float* ao_table, int64_t ao_nrows, int32_t ao_dim,
                       const int32_t* ao_rows, float* out, void* stream) {
  int rc = check_gather(t, rows, hit, n, ao_table, ao_nrows, ao_dim, ao_rows, out);
  if (rc || n == 0) return rc;
  cudaStream_t st = S(stream);
  rc = join_side(t, st);
  if (!rc)
    rc = enqueue_gather(t, rows, hit, n, ao_table, ao_nrows, ao_dim, ao_rows, out, st, false);
  return mark_user(t, st, rc);
}

int mpzch_dedup(mpzch_table* t, const int64_t* ids, int64_t n, int64_t* uniq, int32_t* pos,
                int64_t* dev_count, void* stream) {
  if (!t || n < 0 || n > 0x7FFFFFFFLL || !dev_count) return MPZCH_EINVAL;
  if (n > 0 && (!ids || !uniq || !pos)) return MPZCH_EINVAL;
  if (!on_device(t)) return MPZCH_EINVAL;
  cudaStream_t st = S(stream);
  if (n == 0)
    return mark_user(t, st, cudaMemsetAsync(dev_count, 0, sizeof(int64_t), st) == cudaSuccess
                                ? MPZCH_OK
                                : MPZCH_ECUDA);
  int rc = join_side(t, st);
  if (!rc) rc = ensure_batch(t, n, st);
  if (rc) return rc;
  {
    PhaseScope ps(t, PH_DEDUP, st);
    rc = run_dedup(t, ids, n, reinterpret_cast<long long*>(uniq), pos,
                   reinterpret_cast<long long*>(dev_count), nullptr, st);
  }
  return mark_user(t, st, rc);
}

int mpzch_writeback(mpzch_table* t, const int64_t* ids, const float* e, int64_t n, int64_t step,
                    mpzch_wb_stats* dev_stats, void* stream) {
  int rc = check_writeback(t, ids, e, n, step);
  if (rc) return rc;
  cudaStream_t st = S(stream);
  WbStats* stats = dev_stats ? reinterpret_cast<WbStats*>(dev_stats) : t->stats;
  rc = join_side(t, st);
  if (rc) return rc;
  if (n == 0) {
    if (cudaMemsetAsync(stats, 0, sizeof(WbStats), st) != cudaSuccess) return MPZCH_ECUDA;
    t->last_step = step;
    return mark_user(t, st, MPZCH_OK);
  }
  rc = ensure_batch(t, n, st);
  if (rc) return rc;
  const WbParams p = make_params(t, ids, e, n, step, stats);
  rc = enqueue_row_map(t, p, st, nullptr, nullptr);
  if (!rc) rc = enqueue_row_update(t, p, st, true);
  if (rc) return rc;
  t->last_step = step;
  return mark_user(t, st, MPZCH_OK);
}

int mpzch_train_step(mpzch_table* t, const int64_t* ids, int64_t n, int64_t n_labeled,
                     const float* e, int64_t step, const float* ao_table, int64_t ao_nrows,
                     int32_t ao_dim, const int32_t* ao_rows, int32_t* rows, uint8_t* hit,
                     float* out, mpzch_wb_stats* dev_stats, void* inputs_ready, void* stream) {
  if (!t || n_labeled < 0 || n_labeled > n) return MPZCH_EINVAL;
  int rc = check_writeback(t, ids, e, n, step);
  if (rc) return rc;
  if (n_labeled > 0) {
    if (!rows || !hit) return MPZCH_EINVAL;
    rc = check_gather(t, rows, hit, n_labeled, ao_table, ao_nrows, ao_dim, ao_rows, out);
    if (rc) return rc;
  }
  cudaStream_t st = S(stream);
  WbStats* stats = dev_stats ? reinterpret_cast<WbStats*>(dev_stats) : t->stats;
  rc = ensure_batch(t, n > 0 ? n : 1, st);
  if (!rc) rc = ensure_side_stream(t);
  if (rc) return rc;
  if (n == 0) {
    if (cudaStreamWaitEvent(st, t->ev_map, 0) != cudaSuccess ||
        cudaMemsetAsync(stats, 0, sizeof(WbStats), st) != cudaSuccess)
      return MPZCH_ECUDA;
    t->last_step = step;
    return mark_user(t, st, MPZCH_OK);
  }
  WbParams p = make_params(t, ids, e, n, step, stats);
  p.n_fill = n_labeled;
  p.fill_rows = rows;
  p.fill_hit = hit;
  // Two streams.  Side stream (high priority): the row map -- dedup, re-probe
  // (which also gives the labeled ids' lookup: the rows their ids held before
  // this step's inserts), placement with the lookup fill, write list.
  // Caller's stream: the gather once the fill is done, then the row update
  // once the row map is done.
  // Without inputs_ready the side stream starts after everything earlier on
  // the caller's stream.  With it (pipelined) the side stream waits only for
  // the inputs, the table's other calls and the row update that last read this
  // step's write-list buffers -- so the row map overlaps the previous step's
  // gather and row update -- and, when this step reuses the previous step's
  // rows/hit buffers, its fill waits for the previous gather, which reads them.
  // The row map touches nothing a gather reads except rows/hit: keys, steps,
  // scratch and the write list, never the values.
  cudaEvent_t fill_after = nullptr;
  if (inputs_ready) {
    cudaEvent_t in = reinterpret_cast<cudaEvent_t>(inputs_ready);
    if (cudaStreamWaitEvent(t->side, in, 0) != cudaSuccess ||
        cudaStreamWaitEvent(t->side, t->ev_user, 0) != cudaSuccess ||
        cudaStreamWaitEvent(t->side, t->ev_update[t->wset], 0) != cudaSuccess)
      return MPZCH_ECUDA;
    if (rows == t->prev_rows || hit == t->prev_hit) fill_after = t->ev_gather;
  } else if (cudaEventRecord(t->ev_fork, st) != cudaSuccess ||
             cudaStreamWaitEvent(t->side, t->ev_fork, 0) != cudaSuccess ||
             cudaStreamWaitEvent(t->side, t->ev_user, 0) != cudaSuccess) {
    return MPZCH_ECUDA;
  }
  rc = enqueue_row_map(t, p, t->side, fill_after, t->ev_lookup);
  if (rc) return rc;
  if (cudaEventRecord(t->ev_map, t->side) != cudaSuccess) return MPZCH_ECUDA;
  t->prev_rows = rows;
  t->prev_hit = hit;
  // Caller's stream: gather once the lookup fill is done, then the row update
  // once the row map is done (and after the gather has read the values).
  if (n_labeled > 0) {
    if (cudaStreamWaitEvent(st, t->ev_lookup, 0) != cudaSuccess) return MPZCH_ECUDA;
    rc = enqueue_gather(t, rows, hit, n_labeled, ao_table, ao_nrows, ao_dim, ao_rows, out, st,
                        false);
    if (rc) return rc;
  }
  if (cudaEventRecord(t->ev_gather, st) != cudaSuccess ||
      cudaStreamWaitEvent(st, t->ev_map, 0) != cudaSuccess)
    return MPZCH_ECUDA;
  rc = enqueue_row_update(t, p, st, false);
  if (rc) return rc;
  t->last_step = step;
  return MPZCH_OK;
}

int mpzch_select_written_since(mpzch_table* t, int64_t since_step, int32_t* rows_out,
                               int64_t* dev_count, void* stream) {
  if (!t || !rows_out || !dev_count || !on_device(t)) return MPZCH_EINVAL;
  cudaStream_t st = S(stream);
  int rc = join_side(t, st);
  if (rc) return rc;
  {
    PhaseScope ps(t, PH_SELECT, st);
    rc = launch_select(t, since_step, rows_out, dev_count, st);
  }
  return mark_user(t, st, rc);
}

namespace {
// Writes every row the hot/cold tier's HBM cache holds back to its host row.
int tier_flush(mpzch_table* t, cudaStream_t st) {
  if (t->tier_rows <= 0) return MPZCH_OK;
  return launch(k_tier_flush, row_grid(t->tier_rows, t->row_blocks_per_sm), kBlock, st, false,
                t->tier, t->tier_rows, reinterpret_cast<float4*>(t->M), t->D / 4);
}

// Row export: the interleaved register kernel for D = 128, 256, 512, 1024 (one
// resident wave, grid-stride), the generic kernel for every other dim.
int launch_export(mpzch_table* t, const int32_t* rows, int64_t n, const int64_t* dev_n, int8_t* q,
                  float* scale, int64_t* keys_out, int64_t* last_out, cudaStream_t st) {
  // a tiered table's export reads host rows: cached rows are written back first
  if (int rc = tier_flush(t, st)) return rc;
  const long long* dn = reinterpret_cast<const long long*>(dev_n);
  const float4* M = reinterpret_cast<const float4*>(t->M);
  long long* ko = reinterpret_cast<long long*>(keys_out);
  long long* lo = reinterpret_cast<long long*>(last_out);
  uint32_t* qw = reinterpret_cast<uint32_t*>(q);  // 4-byte aligned (checked by the callers)
  const long long* lst = static_cast<const long long*>(t->last);
  const long long* kk = static_cast<const long long*>(t->keys);
  // one resident wave of the register-heavy row exporter, grid-stride over rows
  auto go = [&](auto kern) {
    const int per_sm = resident_blocks(reinterpret_cast<const void*>(kern), kBlock, 0);
    return launch(kern, grid_for(n * 32, kBlock, per_sm), kBlock, st, false, rows, n, dn, M, kk,
                  t->C, qw, scale, ko, t->status, lst, lo);
  };
  switch (t->D) {
    case 128: return go(k_export_rows<1>);
    case 256: return go(k_export_rows<2>);
    case 512: return go(k_export_rows<4>);
    case 1024: return go(k_export_rows<8>);
    default: break;
  }
  k_export_int8<<<grid_for(n * 32, kBlock), kBlock, 0, st>>>(
      rows, n, dn, M, t->keys, t->C, t->D / 4, reinterpret_cast<char4*>(q), scale, ko, t->status,
      t->last, lo);
  return after_launch();
}
}  // namespace

int mpzch_export_int8(mpzch_table* t, const int32_t* rows, int64_t n, const int64_t* dev_n,
                      int8_t* q, float* scale, int64_t* keys_out, void* stream) {
  if (!t || n < 0 || n > 0x7FFFFFFFLL) return MPZCH_EINVAL;
  if (n == 0) return MPZCH_OK;
  if (!rows || !q || !scale || !keys_out || !on_device(t)) return MPZCH_EINVAL;
  if (reinterpret_cast<uintptr_t>(q) & 3) return MPZCH_EINVAL;
  cudaStream_t st = S(stream);
  int rc = join_side(t, st);
  if (rc) return rc;
  {
    PhaseScope ps(t, PH_EXPORT, st);
    rc = launch_export(t, rows, n, dev_n, q, scale, keys_out, nullptr, st);
  }
  return mark_user(t, st, rc);
}

int mpzch_serve_gather(const int64_t* snap_keys, int64_t capacity, int32_t probes,
                       const int8_t* snap_q, const float* snap_scale, int32_t dim,
                       const int64_t* ids, int64_t n, int32_t* rows, uint8_t* hit, float* out,
                       int32_t* dev_status, void* stream) {
  if (capacity < 1 || capacity > 0x7FFFFFFFLL || probes < 1 || (int64_t)probes > capacity ||
      dim <= 0 || dim % 4 != 0 || n < 0 || n > 0x7FFFFFFFLL)
    return MPZCH_EINVAL;
  if (n == 0) return MPZCH_OK;
  if (!snap_keys || !snap_q || !snap_scale || !ids || !rows || !hit || !out) return MPZCH_EINVAL;
  if ((reinterpret_cast<uintptr_t>(out) & 15) || (reinterpret_cast<uintptr_t>(snap_q) & 3))
    return MPZCH_EINVAL;
  cudaStream_t st = S(stream);
  // one resident wave, grid-stride over the ids
  const int per_sm = resident_blocks(reinterpret_cast<const void*>(k_serve_gather), kBlock, 0);
  k_serve_gather<<<grid_for(n * 32, kBlock, per_sm), kBlock, 0, st>>>(
      reinterpret_cast<const long long*>(snap_keys), make_geo(capacity, probes),
      reinterpret_cast<const char4*>(snap_q), snap_scale, dim / 4,
      reinterpret_cast<const long long*>(ids), n, rows, hit, reinterpret_cast<float4*>(out),
      dev_status);
  return after_launch();
}

int64_t mpzch_owner_partition_workspace(int64_t n, int32_t n_owners) {
  if (n < 0 || n > 0x7FFFFFFFLL || n_owners < 1 || n_owners > kMaxOwners) return -1;
  const int64_t nb = (n + kPartTile - 1) / kPartTile;
  return ((nb * n_owners * (int64_t)sizeof(int32_t)) + 255) / 256 * 256;
}

int mpzch_owner_partition(const int64_t* ids, const int32_t* src_pos, int64_t n,
                          const int64_t* dev_n, int32_t n_owners, const float* e, int32_t dim,
                          int64_t* ids_out, int32_t* pos_out, float* e_out, int64_t* dev_counts,
                          void* workspace, int64_t workspace_bytes, void* stream) {
  const int64_t need = mpzch_owner_partition_workspace(n, n_owners);
  if (need < 0 || !dev_counts) return MPZCH_EINVAL;
  if (e && (dim <= 0 || dim % 4 != 0 || !e_out || (reinterpret_cast<uintptr_t>(e) & 15) ||
            (reinterpret_cast<uintptr_t>(e_out) & 15)))
    return MPZCH_EINVAL;
  cudaStream_t st = S(stream);
  const int nb = (int)((n + kPartTile - 1) / kPartTile);
  if (n > 0 && (!ids || !ids_out || !pos_out || !workspace || workspace_bytes < need))
    return MPZCH_EINVAL;
  int32_t* blk = static_cast<int32_t*>(workspace);
  const long long* dn = reinterpret_cast<const long long*>(dev_n);
  long long* cnt = reinterpret_cast<long long*>(dev_counts);
  if (nb == 0) {  // empty batch: every owner gets nothing
    return cudaMemsetAsync(dev_counts, 0, sizeof(int64_t) * n_owners, st) == cudaSuccess
               ? MPZCH_OK
               : MPZCH_ECUDA;
  }
  const long long* k = reinterpret_cast<const long long*>(ids);
  int rc = launch(k_owner_count, nb, kPartTile, st, false, k, n, dn, (int)n_owners, blk);
  if (!rc) rc = launch(k_owner_offsets, 1, 1024, st, true, blk, nb, (int)n_owners, cnt);
  if (!rc)
    rc = launch(k_owner_scatter, nb, kPartTile, st, true, k, src_pos, n, dn, (int)n_owners,
                static_cast<const int32_t*>(blk), reinterpret_cast<long long*>(ids_out), pos_out);
  if (!rc && e) {
    const int per_sm = resident_blocks(reinterpret_cast<const void*>(k_owner_pack_rows), kBlock, 0);
    rc = launch(k_owner_pack_rows, grid_for(n * 32, kBlock, per_sm), kBlock, st, true,
                static_cast<const int32_t*>(pos_out), n, dn, reinterpret_cast<const float4*>(e),
                dim / 4, reinterpret_cast<float4*>(e_out));
  }
  return rc;
}

int mpzch_owner_combine(const int64_t* send_ids, const int32_t* pos, int64_t n, int32_t n_owners,
                        int64_t shard_capacity, const int32_t* recv_rows, const float* recv_feat,
                        int32_t dim, const float* ao_table, int64_t ao_nrows, int32_t ao_dim,
                        const int32_t* ao_rows, int32_t* rows, uint8_t* hit, float* out,
                        int32_t* dev_status, void* stream) {
  if (n < 0 || n > 0x7FFFFFFFLL || n_owners < 1 || n_owners > kMaxOwners || shard_capacity < 1 ||
      (int64_t)n_owners * shard_capacity > 0x7FFFFFFFLL || dim <= 0 || dim % 4 != 0)
    return MPZCH_EINVAL;
  if (ao_table && (ao_dim <= 0 || ao_dim % 4 != 0 || ao_nrows < 1 || !ao_rows)) return MPZCH_EINVAL;
  if (!ao_table && (ao_dim != 0 || ao_nrows != 0 || ao_rows)) return MPZCH_EINVAL;
  if (n == 0) return MPZCH_OK;
  if (!send_ids || !pos || !recv_rows || !recv_feat || !rows || !hit || !out) return MPZCH_EINVAL;
  if ((reinterpret_cast<uintptr_t>(out) & 15) || (reinterpret_cast<uintptr_t>(recv_feat) & 15) ||
      (reinterpret_cast<uintptr_t>(ao_table) & 15))
    return MPZCH_EINVAL;
  cudaStream_t st = S(stream);
  const int W4 = dim / 4 + (ao_table ? ao_dim / 4 : 0);
  const int vec = W4 > 32 * kCombineVecMax ? kCombineVecMax : (W4 + 31) / 32;
  auto go = [&](auto kern) {
    // one resident wave, grid-stride over the entries
    const int per_sm = resident_blocks(reinterpret_cast<const void*>(kern), kBlock, 0);
    return launch(kern, grid_for(n * 32, kBlock, per_sm), kBlock, st, false,
                  reinterpret_cast<const long long*>(send_ids), pos, n, (int)n_owners,
                  shard_capacity, recv_rows, reinterpret_cast<const float4*>(recv_feat), dim / 4,
                  reinterpret_cast<const float4*>(ao_table), ao_nrows, ao_table ? ao_dim / 4 : 0,
                  ao_rows, rows, hit, reinterpret_cast<float4*>(out), dev_status);
  };
  switch (vec) {
    case 1: return go(k_owner_combine<1>);
    case 2: return go(k_owner_combine<2>);
    case 3: return go(k_owner_combine<3>);
    case 4: return go(k_owner_combine<4>);
    case 5: return go(k_owner_combine<5>);
    case 6: return go(k_owner_combine<6>);
    case 7: return go(k_owner_combine<7>);
    default: return go(k_owner_combine<kCombineVecMax>);
  }
}

int mpzch_state_views(mpzch_table* t, int64_t** keys, int64_t** last, float** M) {
  if (!t) return MPZCH_EINVAL;
  if (keys) *keys = reinterpret_cast<int64_t*>(t->keys);
  if (last) *last = reinterpret_cast<int64_t*>(t->last);
  if (M) *M = t->M;
  return MPZCH_OK;
}

int mpzch_get_last_step(mpzch_table* t, int64_t* step) {
  if (!t || !step) return MPZCH_EINVAL;
  *step = t->last_step;
  return MPZCH_OK;
}

int mpzch_set_last_step(mpzch_table* t, int64_t step) {
  if (!t || step < -1) return MPZCH_EINVAL;
  t->last_step = step;
  return MPZCH_OK;
}

int mpzch_get_status(mpzch_table* t, int32_t* status, void* stream) {
  if (!t || !status || !on_device(t)) return MPZCH_EINVAL;
  cudaStream_t st = S(stream);
  if (join_side(t, st) != MPZCH_OK ||
      cudaMemcpyAsync(t->h_status, t->status, sizeof(int32_t), cudaMemcpyDeviceToHost, st) !=
          cudaSuccess ||
      cudaMemsetAsync(t->status, 0, sizeof(int32_t), st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return MPZCH_ECUDA;
  *status = *t->h_status;
  return MPZCH_OK;
}

int mpzch_trace_enable(mpzch_table* t, int32_t on) {
  if (!t) return MPZCH_EINVAL;
  t->trace = on != 0;
  return MPZCH_OK;
}

int mpzch_trace_read(mpzch_table* t, double* ms, int64_t* launches, int32_t nphases) {
  if (!t || nphases < 0) return MPZCH_EINVAL;
  for (auto& r : t->pending) {
    float x = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&x, r.a, r.b) != cudaSuccess)
      return MPZCH_ECUDA;
    t->ms[r.phase] += x;
    t->pool.push_back(r.a);
    t->pool.push_back(r.b);
  }
  t->pending.clear();
  for (int i = 0; i < nphases && i < MPZCH_NPHASES; ++i) {
    if (ms) ms[i] = t->ms[i];
    if (launches) launches[i] = t->launches[i];
  }
  for (int i = 0; i < MPZCH_NPHASES; ++i) {
    t->ms[i] = 0;
    t->launches[i] = 0;
  }
  return MPZCH_OK;
}

namespace {
// Replaces the tier by one of `rows` slots (0 = none), after writing every
// cached row back; the device is synchronised around the change.
int set_tier_rows(mpzch_table* t, int64_t rows) {
  if (rows < 0 || rows > t->C || (rows & (rows - 1)) != 0 || (rows > 0 && !t->values_on_host) ||
      !on_device(t))
    return MPZCH_EINVAL;
  if (t->tier_rows > 0) {
    if (tier_flush(t, nullptr) != MPZCH_OK || cudaDeviceSynchronize() != cudaSuccess)
      return MPZCH_ECUDA;
  } else if (cudaDeviceSynchronize() != cudaSuccess) {
    return MPZCH_ECUDA;
  }
  dev_free(t->tier.cache);
  dev_free(t->tier.owner);
  dev_free(t->tier.won);
  dev_free(t->tier.claim);
  dev_free(t->tier.stats);
  t->tier = Tier{};
  t->tier_rows = 0;
  if (rows == 0) return MPZCH_OK;
  Tier tr{};
  int rc = dev_alloc((void**)&tr.cache, (size_t)rows * t->D * sizeof(float));
  if (!rc) rc = dev_alloc((void**)&tr.owner, rows * sizeof(int32_t));
  if (!rc) rc = dev_alloc((void**)&tr.won, rows * sizeof(long long));
  if (!rc) rc = dev_alloc((void**)&tr.claim, rows * sizeof(unsigned long long));
  if (!rc) rc = dev_alloc((void**)&tr.stats, kTierStats * sizeof(unsigned long long));
  if (!rc && (cudaMemset(tr.owner, 0xFF, rows * sizeof(int32_t)) != cudaSuccess ||
              cudaMemset(tr.stats, 0, kTierStats * sizeof(unsigned long long)) != cudaSuccess ||
              cudaMemset(tr.won, 0xFF, rows * sizeof(long long)) != cudaSuccess ||
              cudaMemset(tr.claim, 0, rows * sizeof(unsigned long long)) != cudaSuccess ||
              cudaDeviceSynchronize() != cudaSuccess))
    rc = MPZCH_ECUDA;
  if (rc) {
    cudaGetLastError();
    dev_free(tr.cache);
    dev_free(tr.owner);
    dev_free(tr.won);
    dev_free(tr.claim);
    dev_free(tr.stats);
    return rc;
  }
  tr.mask = (uint32_t)(rows - 1);
  t->tier = tr;
  t->tier_rows = rows;
  return MPZCH_OK;
}
}  // namespace

int mpzch_tier_sync(mpzch_table* t, int32_t discard, void* stream) {
  if (!t || (discard != 0 && discard != 1) || !on_device(t)) return MPZCH_EINVAL;
  if (t->tier_rows <= 0) return MPZCH_OK;
  cudaStream_t st = S(stream);
  int rc = join_side(t, st);
  if (rc) return rc;
  if (discard) {
    rc = cudaMemsetAsync(t->tier.owner, 0xFF, t->tier_rows * sizeof(int32_t), st) == cudaSuccess
             ? MPZCH_OK
             : MPZCH_ECUDA;
  } else {
    rc = tier_flush(t, st);
  }
  return mark_user(t, st, rc);
}

int mpzch_tier_stats(mpzch_table* t, int64_t* counts, int32_t reset, void* stream) {
  if (!t || !counts || (reset != 0 && reset != 1) || !on_device(t)) return MPZCH_EINVAL;
  for (int i = 0; i < kTierStats; ++i) counts[i] = 0;
  if (t->tier_rows <= 0) return MPZCH_OK;
  cudaStream_t st = S(stream);
  int rc = join_side(t, st);
  if (rc) return rc;
  unsigned long long h[kTierStats];
  if (cudaMemcpyAsync(h, t->tier.stats, sizeof(h), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      (reset && cudaMemsetAsync(t->tier.stats, 0, sizeof(h), st) != cudaSuccess) ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return MPZCH_ECUDA;
  for (int i = 0; i < kTierStats; ++i) counts[i] = (int64_t)h[i];
  return mark_user(t, st, MPZCH_OK);
}

int mpzch_set_option(mpzch_table* t, int32_t option, int64_t value) {
  if (!t) return MPZCH_EINVAL;
  if (option == MPZCH_OPT_SIDE_PRIORITY) {
    if ((value != 0 && value != 1) || t->side) return MPZCH_EINVAL;
    t->side_high_priority = (int)value;
    return MPZCH_OK;
  }
  if (option == MPZCH_OPT_ROW_GRID) {
    if (value < 0 || value > 32) return MPZCH_EINVAL;
    t->row_blocks_per_sm = (int)value;
    return MPZCH_OK;
  }
  if (option == MPZCH_OPT_WIDE_ROUNDS) {
    if (value < 0 || value > 64) return MPZCH_EINVAL;
    t->wide_rounds = (int)value;
    return MPZCH_OK;
  }
  if (option == MPZCH_OPT_CLUSTER_INSERT) {
    if (value != 0 && value != 1) return MPZCH_EINVAL;
    t->cluster_insert = (int)value;
    return MPZCH_OK;
  }
  if (option == MPZCH_OPT_ROW_KERNEL) {
    if (value != 0 && value != 1) return MPZCH_EINVAL;
    t->row_kernel = (int)value;
    return MPZCH_OK;
  }
  if (option == MPZCH_OPT_BULK_WARPS) {
    if (value != 1 && value != 2 && value != 4 && value != 8 && value != 16) return MPZCH_EINVAL;
    t->bulk_warps = (int)value;
    return MPZCH_OK;
  }
  if (option == MPZCH_OPT_BULK_BLOCKS) {
    if (value < 1 || value > 8) return MPZCH_EINVAL;
    t->bulk_blocks = (int)value;
    return MPZCH_OK;
  }
  if (option == MPZCH_OPT_HBM_CACHE_ROWS) return set_tier_rows(t, value);
  if (option == MPZCH_OPT_WRITE_LIST) {
    if (value != 0 && value != 1) return MPZCH_EINVAL;
    t->emit_list = (int)value;
    return MPZCH_OK;
  }
  if (option == MPZCH_OPT_L2_HINT_ROWS) {
    if (value < 0 || value > 2) return MPZCH_EINVAL;
    t->l2_hint_rows = (int)value;
    return MPZCH_OK;
  }
  return MPZCH_EINVAL;
}

int mpzch_get_option(mpzch_table* t, int32_t option, int64_t* value) {
  if (!t || !value) return MPZCH_EINVAL;
  switch (option) {
    case MPZCH_OPT_WIDE_ROUNDS: *value = t->wide_rounds; break;
    case MPZCH_OPT_SIDE_PRIORITY: *value = t->side_high_priority; break;
    case MPZCH_OPT_ROW_GRID: *value = t->row_blocks_per_sm; break;
    case MPZCH_OPT_CLUSTER_INSERT: *value = t->cluster_insert; break;
    case MPZCH_OPT_ROW_KERNEL: *value = t->row_kernel; break;
    case MPZCH_OPT_BULK_WARPS: *value = t->bulk_warps; break;
    case MPZCH_OPT_BULK_BLOCKS: *value = t->bulk_blocks; break;
    case MPZCH_OPT_L2_HINT_ROWS: *value = t->l2_hint_rows; break;
    case MPZCH_OPT_WRITE_LIST: *value = t->emit_list; break;
    case MPZCH_OPT_HBM_CACHE_ROWS: *value = t->tier_rows; break;
    default: return MPZCH_EINVAL;
  }
  return MPZCH_OK;
}

int mpzch_set_learning_rate(mpzch_table* t, float eta) {
  if (!t || !(eta == eta) || eta > 3.0e38f || eta < -3.0e38f) return MPZCH_EINVAL;
  t->eta = eta;
  return MPZCH_OK;
}

int mpzch_debug_fail_allocs(int32_t count) {
  if (count < 0) return MPZCH_EINVAL;
  g_fail_allocs.store(count);
  return MPZCH_OK;
}

int64_t mpzch_launch_count(void) { return g_launches.load(); }

}  // extern "C"

// ---------------------------------------------------------------------------
// Internal entry points used by the streaming exporter (mpzch_res.cu).
// ---------------------------------------------------------------------------
namespace mpzch_internal {

int64_t table_capacity(const mpzch_table* t) { return t->C; }
int32_t table_dim(const mpzch_table* t) { return t->D; }
int table_device(const mpzch_table* t) { return t->device; }

int export_since(mpzch_table* t, int64_t since, int32_t* rows, int64_t* dev_count, int64_t max_rows,
                 int8_t* q, float* scale, int64_t* keys, int64_t* last, cudaStream_t st) {
  if (!t || !rows || !dev_count || !q || !scale || !keys || !last || max_rows < 1) return MPZCH_EINVAL;
  if (!on_device(t)) return MPZCH_EINVAL;
  int rc = join_side(t, st);
  if (rc) return rc;
  {
    PhaseScope ps(t, PH_SELECT, st);
    rc = launch_select(t, since, rows, dev_count, st);
  }
  if (!rc) {
    PhaseScope ps(t, PH_EXPORT, st);
    rc = launch_export(t, rows, max_rows, dev_count, q, scale, keys, last, st);
  }
  return mark_user(t, st, rc);
}

}  // namespace mpzch_internal
