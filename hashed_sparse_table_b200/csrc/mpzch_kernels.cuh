// Device code of libmpzch: the Memory Layer table kernels for sm_100a.
//
// All kernels are HBM/L2-bound hashing, scanning and row-copy work; nothing
// here is a dense contraction, so no tensor-core path is used.  Rows are moved
// as 16-byte vectors by whole warps (one 2 KiB row = 4 x 512 B coalesced
// requests at D = 512).  Every loop has a static bound; no kernel waits on a
// flag written by another block, and no kernel traps.
#pragma once
#include <cooperative_groups.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mpzch {

namespace cg = cooperative_groups;

constexpr unsigned long long kEmptyKey = 0xFFFFFFFFFFFFFFFFull;  // key -1
constexpr unsigned long long kNoClaim = 0xFFFFFFFFFFFFFFFFull;   // larger than any key
constexpr uint32_t kNoPos = 0xFFFFFFFFu;
constexpr int kBlock = 256;
constexpr int kTile = 1024;  // ids per block in the ordered compactions (4 per thread)

// Status bits (mirror of the MPZCH_STATUS_* values of the public header).
constexpr int kStBadKey = 1, kStBadRow = 2, kStBadAo = 4, kStInternal = 8;

struct Geo {
  int64_t C;
  uint64_t mask;  // C - 1 when C is a power of two
  int32_t pow2;
  int32_t P;
};

// Device counters of one Writeback (cleared at the start of each call).
struct StepCtr {
  int32_t cnt[4];    // insert-round list sizes; round r appends to cnt[(r + 1) % 4]
  int32_t n_unique;  // distinct ids of the batch
  int32_t n_multi;   // cluster path: heads of clusters with several keys (list lidx[1])
  int32_t n_serial;  // cluster path: clusters left to the single-block kernel (list lidx[2])
  int32_t pad;
};

// Per-Writeback counters; same layout as mpzch_wb_stats.
struct WbStats {
  long long n_ids, n_unique, n_hit_unique, n_inserted, n_evicted, n_dropped, n_rounds;
};

// SplitMix64 generator output for state x (Steele, Lea, Flood, OOPSLA 2014):
// add the golden gamma, two xor-shift-multiply rounds, a final xor-shift.
__device__ __forceinline__ uint64_t splitmix64(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ int64_t home_slot(int64_t k, const Geo& g) {
  const uint64_t h = splitmix64((uint64_t)k);
  return g.pow2 ? (int64_t)(h & g.mask) : (int64_t)(h % (uint64_t)g.C);
}

// Slot h + j of a window (h < C, j < P <= C, so one subtraction wraps it).
__device__ __forceinline__ int64_t wslot(int64_t h, int32_t j, const Geo& g) {
  int64_t s = h + j;
  return s >= g.C ? s - g.C : s;
}

__device__ __forceinline__ long long ld_cg(const long long* p) { return __ldcg(p); }
__device__ __forceinline__ unsigned long long ld_cg(const unsigned long long* p) {
  return __ldcg(p);
}

// 64-bit signed add through the unsigned atomic (two's complement).
__device__ __forceinline__ void atomic_add_ll(long long* p, long long v) {
  atomicAdd(reinterpret_cast<unsigned long long*>(p), (unsigned long long)v);
}

__device__ __forceinline__ void set_status(int32_t* st, int bits) {
  if (st) atomicOr(st, bits);
}

// Waits on other warps or on copies in flight give up after this long and set
// MPZCH_STATUS_TIMEOUT (far beyond any legitimate wait).
constexpr int kStTimeout = 16;
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Programmatic dependent launch.  pdl_enter waits until every earlier grid of
// the stream has completed and its memory is visible; every kernel calls it
// first, so nothing is read before the producer has finished.  pdl_trigger
// lets the next kernel of the stream launch; kernels of the row-map chain call
// it once their main work is done, so the next kernel's blocks are scheduled
// during this kernel's tail rather than parked on the SMs (holding warps and
// shared memory that the concurrently running row kernels need) for its whole
// run.  A kernel that never calls it triggers when its blocks exit.  Both are
// no-ops for a kernel launched without the programmatic-serialisation
// attribute.
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void pdl_enter() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Row of `k` by one thread scanning the whole window (first match in probe
// order; the identity map holds at most one).  -1 if absent.  Loads of 8
// slots are issued together.
__device__ __forceinline__ int64_t find_row_thread(const long long* __restrict__ keys, int64_t k,
                                                   int64_t h, const Geo& g) {
  int64_t found = -1;
  for (int32_t j0 = 0; j0 < g.P; j0 += 8) {
    long long v[8];
#pragma unroll
    for (int q = 0; q < 8; ++q)
      v[q] = (j0 + q < g.P) ? ld_cg(keys + wslot(h, j0 + q, g)) : -2;
#pragma unroll
    for (int q = 0; q < 8; ++q)
      if (found < 0 && v[q] == k) found = wslot(h, j0 + q, g);
  }
  return found;
}

// ---------------------------------------------------------------------------
// Lookup: G lanes cooperate on one id (G = next power of two >= P, at most 32),
// so the P keys of a window are fetched by one coalesced request.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kBlock) k_lookup(const long long* __restrict__ ids, int64_t n,
                                                   const long long* __restrict__ keys, Geo g,
                                                   int G, int32_t* __restrict__ rows,
                                                   uint8_t* __restrict__ hit, int32_t* status) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int sub = lane & (G - 1);
  const unsigned gmask = (G == 32) ? 0xFFFFFFFFu : (((1u << G) - 1u) << (lane & ~(G - 1)));
  const int64_t groups_per_grid = ((int64_t)gridDim.x * blockDim.x) / G;
  for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / G; i < n;
       i += groups_per_grid) {
    const long long k = ids[i];
    int32_t best = 0x7FFFFFFF;
    if (k >= 0) {
      const int64_t h = home_slot(k, g);
      for (int32_t j = sub; j < g.P; j += G)
        if (__ldg(keys + wslot(h, j, g)) == k && j < best) best = j;
    }
    for (int off = G >> 1; off > 0; off >>= 1) {
      const int32_t o = __shfl_xor_sync(gmask, best, off, G);
      best = o < best ? o : best;
    }
    if (sub == 0) {
      int32_t r = -1;
      if (k < 0)
        set_status(status, kStBadKey);
      else if (best != 0x7FFFFFFF)
        r = (int32_t)wslot(home_slot(k, g), best, g);
      rows[i] = r;
      hit[i] = r >= 0 ? 1 : 0;
    }
  }
}

// ---------------------------------------------------------------------------
// Fused gather: out[i] = [hit ? M[rows[i]] : +0] ++ ao[ao_rows[i]], one warp per
// output row, 16-byte vectors, all loads of a chunk issued before its stores.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kBlock) k_gather_fused(
    const int32_t* __restrict__ rows, const uint8_t* __restrict__ hit, int64_t n,
    const float4* __restrict__ M, int64_t C, int D4, const float4* __restrict__ ao,
    int64_t ao_n, int A4, const int32_t* __restrict__ ao_rows, float4* __restrict__ out,
    int32_t* status) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int64_t warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int W4 = D4 + A4;
  for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; i < n; i += warps) {
    int32_t r = rows[i];
    bool h = hit[i] != 0;
    if (h && (r < 0 || (int64_t)r >= C)) {
      if (lane == 0) set_status(status, kStBadRow);
      h = false;
    }
    int32_t a = 0;
    bool has_a = A4 > 0;
    if (has_a) {
      a = ao_rows[i];
      if (a < 0 || (int64_t)a >= ao_n) {
        if (lane == 0) set_status(status, kStBadAo);
        has_a = false;
      }
    }
    const float4* src = M + (int64_t)(h ? r : 0) * D4;
    const float4* asrc = ao + (int64_t)a * A4;
    float4* dst = out + i * (int64_t)W4;
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int base = 0; base < W4; base += 4 * 32) {
      float4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = base + u * 32 + lane;
        v[u] = z;
        if (c < D4) {
          if (h) v[u] = __ldcs(src + c);
        } else if (c < W4 && has_a) {
          v[u] = __ldcs(asrc + (c - D4));
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = base + u * 32 + lane;
        if (c < W4) __stcs(dst + c, v[u]);
      }
    }
  }
}

// Block-wide exclusive scan of one int per thread; returns the block total.
__device__ __forceinline__ int block_excl_scan(int v, int* smem /* >= 33 ints */, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x = v;
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xFFFFFFFFu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) smem[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nw ? smem[lane] : 0;
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xFFFFFFFFu, w, off);
      if (lane >= off) w += y;
    }
    if (lane < nw) smem[lane] = w;
    if (lane == nw - 1) smem[32] = w;
  }
  __syncthreads();
  const int before = (warp ? smem[warp - 1] : 0) + x - v;
  total = smem[32];
  __syncthreads();
  return before;
}

__device__ __forceinline__ long long block_sum_ll(long long v, long long* smem /* >= 32 */) {
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  if (lane == 0) smem[warp] = v;
  __syncthreads();
  long long t = 0;
  if (threadIdx.x == 0)
    for (int w = 0; w < nw; ++w) t += smem[w];
  __syncthreads();
  if (threadIdx.x == 0) smem[0] = t;
  __syncthreads();
  t = smem[0];
  __syncthreads();
  return t;
}

// ---------------------------------------------------------------------------
// Dedup, phase 1: every id goes into an open-addressing scratch hash holding
// (key, smallest position).  Each block first dedups its tile of kTile
// positions in shared memory, so a hot id costs one global CAS per tile
// instead of one per copy; then each distinct id of the tile is inserted once
// with its smallest tile position, and every position learns its global slot.
// Block 0 also clears the step counters used by the later phases.
// ---------------------------------------------------------------------------
constexpr int kTileHash = 2 * kTile;  // shared-memory slots per tile (load <= 1/2)
constexpr int kDedupThreads = kTile;  // one tile position per thread

__global__ void __launch_bounds__(kDedupThreads) k_dedup_insert(
    const long long* __restrict__ ids, int64_t n, unsigned long long* __restrict__ hkey,
    uint32_t* __restrict__ hpos, uint64_t hmask, int32_t* __restrict__ slot_of, StepCtr* ctr,
    WbStats* stats, int32_t* status, int32_t* wcount, int32_t* wtake) {
  pdl_enter();
  __shared__ unsigned long long s_key[kTileHash];
  __shared__ uint32_t s_pos[kTileHash];
  __shared__ int32_t s_gslot[kTileHash];
  __shared__ int16_t s_list[kTile];  // occupied shared slots (at most one per position)
  __shared__ int s_scan[33];
  if (blockIdx.x == 0 && threadIdx.x < sizeof(StepCtr) / 4)
    reinterpret_cast<int32_t*>(ctr)[threadIdx.x] = 0;
  if (stats && blockIdx.x == 0 && threadIdx.x < 7)
    reinterpret_cast<long long*>(stats)[threadIdx.x] = 0;
  if (wcount && blockIdx.x == 0 && threadIdx.x == 0) *wcount = 0;
  if (wtake && blockIdx.x == 0 && threadIdx.x == 0) *wtake = 0;
  for (int j = threadIdx.x; j < kTileHash; j += blockDim.x) {
    s_key[j] = kEmptyKey;
    s_pos[j] = kNoPos;
  }
  __syncthreads();
  // 1. tile-local dedup
  const int64_t i = (int64_t)blockIdx.x * kTile + threadIdx.x;
  int lslot = -1;
  if (i < n) {
    const long long k = ids[i];
    if (k < 0) {
      slot_of[i] = -1;
      set_status(status, kStBadKey);
    } else {
      int j = (int)(splitmix64((uint64_t)k ^ 0x5851F42D4C957F2Dull) & (kTileHash - 1));
      for (int probe = 0; probe < kTileHash; ++probe) {
        const unsigned long long cur = atomicCAS(&s_key[j], kEmptyKey, (unsigned long long)k);
        if (cur == kEmptyKey || cur == (unsigned long long)k) {
          atomicMin(&s_pos[j], (uint32_t)i);
          lslot = j;
          break;
        }
        j = (j + 1) & (kTileHash - 1);
      }
    }
  }
  __syncthreads();
  // 2. one global insert per distinct id of the tile (compacted: at most one
  //    per thread); a collision falls back to linear probing.
  {
    const int occ = (s_key[2 * threadIdx.x] != kEmptyKey) + (s_key[2 * threadIdx.x + 1] != kEmptyKey);
    int total = 0;
    int at = block_excl_scan(occ, s_scan, total);
    if (s_key[2 * threadIdx.x] != kEmptyKey) s_list[at++] = (int16_t)(2 * threadIdx.x);
    if (s_key[2 * threadIdx.x + 1] != kEmptyKey) s_list[at++] = (int16_t)(2 * threadIdx.x + 1);
    __syncthreads();
    if ((int)threadIdx.x < total) {
      const int jj = s_list[threadIdx.x];
      const unsigned long long kk = s_key[jj];
      int64_t sl = (int64_t)(splitmix64(kk ^ 0xD6E8FEB86659FD93ull) & hmask);
      unsigned long long cur = __ldcg(hkey + sl);
      if (cur == kEmptyKey) cur = atomicCAS(hkey + sl, kEmptyKey, kk);
      bool placed = cur == kEmptyKey || cur == kk;
      for (uint64_t probe = 1; probe <= hmask && !placed; ++probe) {
        sl = (sl + 1) & (int64_t)hmask;
        unsigned long long c = __ldcg(hkey + sl);
        if (c == kEmptyKey) c = atomicCAS(hkey + sl, kEmptyKey, kk);
        placed = c == kEmptyKey || c == kk;
      }
      if (!placed) set_status(status, kStInternal);  // scratch hash sized >= 2n: never expected
      atomicMin(hpos + sl, s_pos[jj]);
      s_gslot[jj] = (int32_t)sl;
    }
  }
  pdl_trigger();
  __syncthreads();
  // 3. every position learns the global slot of its id
  if (i < n && lslot >= 0) slot_of[i] = s_gslot[lslot];
}

// Sum of cnt[0 .. upto) by the whole block.
__device__ __forceinline__ long long block_prefix_of_counts(const int32_t* cnt, int64_t upto,
                                                            long long* smem) {
  long long acc = 0;
  for (int64_t b = threadIdx.x; b < upto; b += blockDim.x) acc += cnt[b];
  return block_sum_ll(acc, smem);
}

// Dedup, phase 2: per tile of kTile positions, count first occurrences.
__global__ void __launch_bounds__(kBlock) k_dedup_count(const int32_t* __restrict__ slot_of,
                                                        const uint32_t* __restrict__ hpos,
                                                        int64_t n, int32_t* __restrict__ bcount) {
  pdl_enter();
  __shared__ long long sm[33];
  const int64_t base = (int64_t)blockIdx.x * kTile + threadIdx.x * 4;
  int c = 0;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int64_t i = base + u;
    if (i < n) {
      const int32_t s = slot_of[i];
      c += (s >= 0 && __ldcg(hpos + s) == (uint32_t)i);
    }
  }
  const long long t = block_sum_ll(c, sm);
  if (threadIdx.x == 0) bcount[blockIdx.x] = (int32_t)t;
}

// Dedup, phase 3: ordered compaction of first occurrences into (uniq, pos),
// and reset of the scratch hash slots for the next call.  The last block
// writes the number of distinct ids.
__global__ void __launch_bounds__(kBlock) k_dedup_compact(
    const long long* __restrict__ ids, int64_t n, const int32_t* __restrict__ slot_of,
    unsigned long long* __restrict__ hkey, uint32_t* __restrict__ hpos,
    const int32_t* __restrict__ bcount, long long* __restrict__ ukey, int32_t* __restrict__ upos,
    long long* dev_count, WbStats* stats) {
  pdl_enter();
  __shared__ long long sm[33];
  __shared__ int smi[33];
  const long long offset = block_prefix_of_counts(bcount, blockIdx.x, sm);
  const int64_t base = (int64_t)blockIdx.x * kTile + threadIdx.x * 4;
  int flags = 0, c = 0, nvalid = 0;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int64_t i = base + u;
    if (i < n) {
      const int32_t s = slot_of[i];
      nvalid += s >= 0;
      if (s >= 0 && __ldcg(hpos + s) == (uint32_t)i) {
        flags |= 1 << u;
        ++c;
      }
    }
  }
  int total = 0;
  int rank = block_excl_scan(c, smi, total);
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    if (!(flags & (1 << u))) continue;
    const int64_t i = base + u;
    const int64_t uidx = offset + rank++;
    const int32_t s = slot_of[i];
    ukey[uidx] = ids[i];
    upos[uidx] = (int32_t)i;
    hkey[s] = kEmptyKey;  // only this thread owns slot s now
    hpos[s] = kNoPos;
  }
  if (stats) {
    const long long bv = block_sum_ll(nvalid, sm);
    if (threadIdx.x == 0 && bv) atomic_add_ll(&stats->n_ids, bv);
  }
  if (blockIdx.x == gridDim.x - 1 && threadIdx.x == 0) {
    const long long U = offset + total;
    if (dev_count) *dev_count = U;
    if (stats) stats->n_unique = U;
  }
}

// Slot index of list entry m among the lanes of this warp that append together;
// one atomic per warp instead of one per lane.
__device__ __forceinline__ int warp_append(int32_t* counter) {
  auto grp = cg::coalesced_threads();
  int base = 0;
  if (grp.thread_rank() == 0) base = atomicAdd(counter, (int)grp.size());
  return grp.shfl(base, 0) + (int)grp.thread_rank();
}

__device__ __forceinline__ void claim_window(unsigned long long* claims, long long k, const Geo& g) {
  const int64_t h = home_slot(k, g);
  for (int32_t j = 0; j < g.P; ++j) atomicMin(claims + wslot(h, j, g), (unsigned long long)k);
}

__device__ __forceinline__ void clear_window(unsigned long long* claims, long long k, const Geo& g) {
  const int64_t h = home_slot(k, g);
  for (int32_t j = 0; j < g.P; ++j) claims[wslot(h, j, g)] = kNoClaim;
}

// ---------------------------------------------------------------------------
// Insert of missing keys in conflict rounds.
//
// Sequential rule: missing keys are inserted one at a time in ascending key
// order, each into the row of its window with the smallest (last, row).  A key
// k may be placed as soon as no smaller missing key that is still unplaced has
// a window overlapping W(k): then the rows of W(k) already hold their final
// state with respect to every smaller key, and no larger key can touch them
// before k in the sequential order.  Each round every unplaced key writes
// atomicMin(claim[s], k) on its window; a key that finds its own value in all
// of its P claim slots is the smallest unplaced key over every overlapping
// window, so it commits.  Keys committing in the same round have disjoint
// windows (a shared slot would hold the smaller key), so they write the table
// independently.  The smallest unplaced key always commits, so rounds end.
//
// Round r checks claims[r % 3], makes round-(r+1) claims in claims[(r+1) % 3]
// and clears round-(r-1) claims in claims[(r-1) % 3], so one round never uses
// an array for two purposes.  The (key, distinct-id index) lists rotate the
// same way.
// ---------------------------------------------------------------------------
struct WbParams;
__device__ __forceinline__ void emit_placement(const WbParams& p, int64_t row,
                                               long long victim_last, int32_t uidx);

__device__ __forceinline__ bool try_commit(const WbParams& p, long long k, int32_t uidx,
                                           const unsigned long long* claims,
                                           long long* __restrict__ keys,
                                           long long* __restrict__ last, const Geo& g,
                                           long long step, int32_t* __restrict__ urow,
                                           long long& evicted) {
  const int64_t h = home_slot(k, g);
  int64_t best = -1;
  long long best_last = 0;
  for (int32_t j0 = 0; j0 < g.P; j0 += 8) {
    // claims and last-write steps of 8 window slots, all requests in flight together
    unsigned long long c[8];
    long long l[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const bool in = j0 + q < g.P;
      const int64_t s = wslot(h, in ? j0 + q : 0, g);
      c[q] = in ? ld_cg(claims + s) : (unsigned long long)k;
      l[q] = in ? ld_cg(last + s) : 0;
    }
    bool mine = true;
#pragma unroll
    for (int q = 0; q < 8; ++q) mine &= c[q] == (unsigned long long)k;
    if (!mine) return false;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      if (j0 + q >= g.P) continue;
      const int64_t s = wslot(h, j0 + q, g);
      if (best < 0 || l[q] < best_last || (l[q] == best_last && s < best)) {
        best = s;
        best_last = l[q];
      }
    }
  }
  // A row is empty exactly when its last-write step is -1 (key and step are
  // always set together), so a victim with a step is a live key.
  if (best_last != -1) ++evicted;
  emit_placement(p, best, best_last, uidx);
  keys[best] = k;
  last[best] = step;
  urow[uidx] = (int32_t)best;
  return true;
}

// Arguments of the Writeback kernels.
struct WbParams {
  const long long* ids;
  int64_t n;
  const float4* e;
  int D4;
  unsigned long long* hkey;
  uint32_t* hpos;
  uint64_t hmask;
  int32_t* slot_of;
  long long* ukey;
  int32_t* upos;
  int32_t* urow;
  long long* keys;
  long long* last;
  float4* M;
  Geo g;
  long long step;
  long long* lkey[3];
  int32_t* lidx[3];
  unsigned long long* claims[3];
  StepCtr* ctr;
  WbStats* stats;
  int32_t* status;
  int wide_rounds;  // grid-wide insert rounds of this Writeback (claim-round path)
  // cluster placement path: per-slot lists of this call's missing keys.
  // shead[s] = (tag << 32) | list-0 index of the last key linked at home slot
  // s, valid only when its upper half equals this call's tag (so entries of
  // earlier calls read as empty and nothing is ever cleared); snext[m] = the
  // next key of the same home slot, or -1.
  int cluster;
  uint32_t tag;
  unsigned long long* shead;
  int32_t* snext;
  // write list of this Writeback: (row, position of e) of every distinct id
  // that still owns its row; one of two buffers, alternating by call
  int32_t* wrow;
  int32_t* wpos;
  int32_t* wcount;
  // per distinct id: 1 when it was resident before the step (set by the
  // re-probe), and the same flag aligned with the write list (uhit itself on
  // the cluster path, a compacted copy written by k_write_list otherwise)
  uint8_t* uhit;
  uint8_t* whit;
  int32_t* wtake;  // entries of the list already taken by the bulk row update
  // emit = 1 (cluster path): the write list is the distinct-id arrays of this
  // call themselves -- entry u = (urow[u], upos[u]), wrow/wpos point at them
  // and *wcount is set to the number of distinct ids -- so nothing is
  // appended.  wentry[row] holds the distinct-id index of the row's owner in
  // this step (set by the re-probe for resident ids and by each placement); a
  // placement that evicts an id written earlier in this step marks that id's
  // urow as kDroppedRow, which the row update skips.  emit = 0: k_write_list
  // builds a compacted list in separate buffers after all placements.
  int emit;
  int32_t* wentry;
  // lookup of the first n_fill batch positions (the labeled ids of a train
  // step) taken from the re-probe: the re-probe stores, per scratch-hash slot,
  // the row its id held before this step's inserts (hrow), and the fill pass
  // gives every position its id's row (rows, hit); n_fill = 0: no fill
  int32_t* hrow;
  int64_t n_fill;
  int32_t* fill_rows;
  uint8_t* fill_hit;
};

// Lookup result of batch position i < n_fill: the row its id held before the
// step's inserts (-1: missing; negative ids have no scratch slot and were
// flagged by the dedup).  Reads only what the dedup and the re-probe wrote.
__device__ __forceinline__ void fill_lookup(const WbParams& p, int64_t i) {
  const int32_t s = p.slot_of[i];
  const int32_t r = s >= 0 ? __ldcg(p.hrow + s) : -1;
  p.fill_rows[i] = r;
  p.fill_hit[i] = r >= 0 ? 1 : 0;
}

// urow value of a distinct id that was placed and then evicted again later in
// the same step (it gets no write); -1 still means "not placed yet".
constexpr int32_t kDroppedRow = -2;

// Bookkeeping of a placement into `row` for distinct id uidx (emit mode): a
// previous owner written in this step (its last-write step is this step: a
// resident id refreshed by the re-probe, or an id placed earlier in the
// step) loses its write (n_dropped), and uidx becomes the row's owner.
__device__ __forceinline__ void emit_placement(const WbParams& p, int64_t row,
                                               long long victim_last, int32_t uidx) {
  if (!p.emit) return;
  if (victim_last == p.step) {
    p.urow[p.wentry[row]] = kDroppedRow;
    atomic_add_ll(&p.stats->n_dropped, 1LL);
  }
  p.wentry[row] = uidx;
}

// Two per-thread counts packed as 16-bit halves (each <= the block size).
__device__ __forceinline__ int pack2(int a, int b) { return a | (b << 16); }

// Block-aggregated append: every thread with want != 0 gets a distinct slot of
// the list whose length counter is `counter`; one global atomic per block.
// All threads of the block must call it.
__device__ __forceinline__ void block_append2(int wa, int wb, int32_t* ca, int32_t* cb, int& ia,
                                              int& ib, int* smi) {
  int total = 0;
  const int before = block_excl_scan(pack2(wa, wb), smi, total);
  __shared__ int s_base[2];
  if (threadIdx.x == 0) {
    const int ta = total & 0xFFFF, tb = total >> 16;
    s_base[0] = ta ? atomicAdd(ca, ta) : 0;
    s_base[1] = tb ? atomicAdd(cb, tb) : 0;
  }
  __syncthreads();
  ia = s_base[0] + (before & 0xFFFF);
  ib = s_base[1] + (before >> 16);
  __syncthreads();
}

// Writeback, dedup phase 2 + re-probe, one pass over the batch positions: a
// position whose id's scratch-hash entry holds that position is the id's
// first occurrence.  Its thread appends the distinct id (key, first position)
// to the distinct-id list (in block order; the Writeback result does not
// depend on that order), resets the hash slot for the next call, and probes
// the table: a resident id refreshes last[row] = step; a missing id enters
// insert round 0 (list 0) and claims its window in claims[0].
__global__ void __launch_bounds__(kBlock) k_first_reprobe(WbParams p) {
  pdl_enter();
  __shared__ long long sm[33];
  __shared__ int smi[33];
  const Geo g = p.g;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  long long hits = 0, nvalid = 0;
  for (int64_t base = (int64_t)blockIdx.x * blockDim.x; base < p.n; base += stride) {
    const int64_t i = base + threadIdx.x;
    bool first = false;
    long long k = 0;
    int64_t h = 0, r = -1;
    if (i < p.n) {
      const int32_t s = p.slot_of[i];
      if (s >= 0) {
        ++nvalid;
        if (__ldcg(p.hpos + s) == (uint32_t)i) {
          first = true;
          k = p.ids[i];
          p.hkey[s] = kEmptyKey;  // only this thread owns slot s now
          p.hpos[s] = kNoPos;
          h = home_slot(k, g);
          r = find_row_thread(p.keys, k, h, g);
          if (p.n_fill) p.hrow[s] = (int32_t)r;
        }
      }
    }
    int u = 0, m = 0;
    block_append2(first, first && r < 0, &p.ctr->n_unique, &p.ctr->cnt[0], u, m, smi);
    if (first) {
      p.ukey[u] = k;
      p.upos[u] = (int32_t)i;
      p.urow[u] = (int32_t)r;
      p.uhit[u] = r >= 0 ? 1 : 0;
      if (r >= 0) {
        p.last[r] = p.step;
        ++hits;
        if (p.emit) p.wentry[r] = u;
      } else {
        p.lkey[0][m] = k;
        p.lidx[0][m] = u;
        if (p.cluster) {
          const unsigned long long old =
              atomicExch(p.shead + h, ((unsigned long long)p.tag << 32) | (uint32_t)m);
          p.snext[m] = (uint32_t)(old >> 32) == p.tag ? (int32_t)(uint32_t)old : -1;
        } else {
          claim_window(p.claims[0], k, g);
        }
      }
    }
  }
  pdl_trigger();
  const long long bh = block_sum_ll(hits, sm);
  const long long bv = block_sum_ll(nvalid, sm);
  if (threadIdx.x == 0) {
    if (bh) atomic_add_ll(&p.stats->n_hit_unique, bh);
    if (bv) atomic_add_ll(&p.stats->n_ids, bv);
  }
}

// The lookup fill as a kernel of its own (claim-round insert path, where no
// placement pass follows the re-probe).
__global__ void __launch_bounds__(kBlock) k_lookup_fill(WbParams p) {
  pdl_enter();
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < p.n_fill; i += stride)
    fill_lookup(p, i);
}

// Grid-wide insert round r (see the insert comment above): clears the claims
// of round r-1, tries to commit every key of round r, and moves the others to
// round r+1 (block-aggregated append, claims in claims[(r+1) % 3]).
__global__ void __launch_bounds__(kBlock) k_insert_round(WbParams p, int r) {
  pdl_enter();
  __shared__ long long sm[33];
  __shared__ int smi[33];
  const Geo g = p.g;
  const int32_t nprev = r > 0 ? p.ctr->cnt[(r + 3) & 3] : 0;
  const int32_t ncur = p.ctr->cnt[r & 3];
  const int32_t nmax = nprev > ncur ? nprev : ncur;
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    // counter that round r+1 appends to; its last reader was round r-1
    p.ctr->cnt[(r + 2) & 3] = 0;
    if (r == 0) p.stats->n_inserted = ncur;
  }
  const int64_t first_i = (int64_t)blockIdx.x * blockDim.x;
  if (first_i >= nmax) return;  // whole block idle (block-uniform)
  const int rp = (r + 2) % 3, rc = r % 3, rn = (r + 1) % 3;
  long long evicted = 0;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t base = first_i; base < nmax; base += stride) {
    const int64_t i = base + threadIdx.x;
    if (i < nprev) clear_window(p.claims[rp], p.lkey[rp][i], g);
    bool defer = false;
    long long k = 0;
    int32_t u = 0;
    if (i < ncur) {
      k = p.lkey[rc][i];
      u = p.lidx[rc][i];
      defer = !try_commit(p, k, u, p.claims[rc], p.keys, p.last, g, p.step, p.urow, evicted);
    }
    int m = 0, unused = 0;
    block_append2(defer, 0, &p.ctr->cnt[(r + 1) & 3], &p.ctr->cnt[(r + 1) & 3], m, unused, smi);
    if (defer) {
      p.lkey[rn][m] = k;
      p.lidx[rn][m] = u;
      // the single-block finisher claims for itself if it needs claims
      if (r + 1 < p.wide_rounds) claim_window(p.claims[rn], k, g);
    }
  }
  pdl_trigger();
  const long long ev = block_sum_ll(evicted, sm);
  if (threadIdx.x == 0 && ev) atomic_add_ll(&p.stats->n_evicted, ev);
  if (blockIdx.x == 0 && threadIdx.x == 0 && ncur > 0) atomic_add_ll(&p.stats->n_rounds, 1LL);
}

// Remaining rounds in one block by the claim rule (block barriers only); lists,
// claims and counters rotate exactly as in k_insert_round.  Used when too many
// keys are left for the cluster path.
__device__ void finish_by_rounds(const WbParams& p, int r0, int32_t nprev, int32_t ncur,
                                 long long& evicted, long long& rounds) {
  __shared__ int32_t s_cnt[2];  // next-list counters, alternating by iteration parity
  const Geo g = p.g;
  const int32_t bound = ncur + 2;  // each round commits at least one key
  int r = r0;
  for (int32_t it = 0; it <= bound; ++it) {
    // s_cnt[it & 1] was last read right after the barrier that ended iteration
    // it - 2, before every thread passed the first barrier of iteration it - 1.
    int32_t* s_next = &s_cnt[it & 1];
    if (threadIdx.x == 0) *s_next = 0;
    __syncthreads();
    const int32_t nmax = nprev > ncur ? nprev : ncur;
    const int rp = (r + 2) % 3, rc = r % 3, rn = (r + 1) % 3;
    for (int32_t i = threadIdx.x; i < nmax; i += blockDim.x) {
      if (i < nprev) clear_window(p.claims[rp], __ldcg(p.lkey[rp] + i), g);
      if (i < ncur) {
        const long long k = __ldcg(p.lkey[rc] + i);
        const int32_t u = __ldcg(p.lidx[rc] + i);
        if (!try_commit(p, k, u, p.claims[rc], p.keys, p.last, g, p.step, p.urow, evicted)) {
          const int m = atomicAdd(s_next, 1);
          p.lkey[rn][m] = k;
          p.lidx[rn][m] = u;
          claim_window(p.claims[rn], k, g);
        }
      }
    }
    rounds += ncur > 0;
    __threadfence();
    __syncthreads();
    nprev = ncur;
    ncur = *s_next;
    ++r;
    if (nprev == 0 && ncur == 0) break;
    if (it == bound && threadIdx.x == 0) set_status(p.status, kStInternal);
  }
}

// Places one missing key by the sequential rule (victim = smallest (last, row)
// in its window).  The caller guarantees that no other thread touches the
// window meanwhile.
__device__ __forceinline__ void place_key(const WbParams& p, long long k, int32_t u,
                                          long long& evicted) {
  const Geo& g = p.g;
  const int64_t h = home_slot(k, g);
  int64_t best = -1;
  long long best_last = 0;
  for (int32_t j0 = 0; j0 < g.P; j0 += 8) {
    long long l[8];
#pragma unroll
    for (int q = 0; q < 8; ++q)
      l[q] = j0 + q < g.P ? ld_cg(p.last + wslot(h, j0 + q, g)) : 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      if (j0 + q >= g.P) continue;
      const int64_t s = wslot(h, j0 + q, g);
      if (best < 0 || l[q] < best_last || (l[q] == best_last && s < best)) {
        best = s;
        best_last = l[q];
      }
    }
  }
  if (best_last != -1) ++evicted;
  emit_placement(p, best, best_last, u);
  p.keys[best] = k;
  p.last[best] = p.step;
  p.urow[u] = (int32_t)best;
}

// One block that places what the grid-wide kernels left.  Claim-round path:
// the keys left after the grid-wide rounds.  Cluster placement path: the
// clusters listed by k_place_multi (beyond the warp path), one thread each,
// or -- when the windows may cover the whole ring -- every missing key, by the
// sort below.
//
// Sort path (at most kClusterMax keys): every key still unplaced only
// conflicts with unplaced keys whose windows overlap its own (keys placed in
// earlier rounds are smaller than every unplaced key overlapping them, so
// their effect already precedes in the sequential order).  The unplaced keys
// are sorted by home slot (bucket counting sort + insertion sort per bucket in
// shared memory); maximal runs whose consecutive home slots are less than P
// apart (cyclically) are clusters with pairwise disjoint window sets; one
// thread places a cluster's keys in ascending key order.  Claims left behind
// by the last grid-wide round are cleared by k_write_list (spread over the
// whole grid).  Larger leftovers fall back to claim rounds.
constexpr int kClusterMax = 4096;
constexpr int kClusterBuckets = 4096;
constexpr size_t kClusterSmem = (size_t)kClusterMax * (4 + 8 + 4) + (kClusterBuckets + 1) * 4;

constexpr int kClusterLocal = 32;  // cluster keys a serial thread sorts locally (else the slow walk)
constexpr int kSpanLocal = 96;     // slots of a cluster's windows a serial thread copies locally

// Scratch of one thread running place_cluster_serial (slot heads, keys and
// their distinct-id indices, the span's steps).
struct SerialScratch {
  unsigned long long heads[kClusterLocal];
  long long ck[kClusterLocal];
  long long sl[kSpanLocal];
  int32_t cu[kClusterLocal];
};
constexpr int kSerialThreads = 32;  // threads of k_insert_finish that place listed clusters
static_assert(sizeof(SerialScratch) * kSerialThreads <= kClusterSmem,
              "serial scratch must fit the finisher's dynamic shared memory");

__device__ void place_cluster_serial(const WbParams& p, int64_t h, int32_t N, SerialScratch& w,
                                     long long& evicted);

__global__ void __launch_bounds__(1024) k_insert_finish(WbParams p, int r0) {
  pdl_enter();
  extern __shared__ __align__(16) unsigned char dsm[];
  __shared__ long long sm[33];
  __shared__ int smi[33];
  const Geo g = p.g;
  const int32_t nprev = r0 > 0 ? p.ctr->cnt[(r0 + 3) & 3] : 0;
  const int32_t ncur = p.ctr->cnt[r0 & 3];
  // cluster placement path: when the windows may cover the whole ring the
  // grid-wide passes placed nothing and this block places every key; otherwise
  // it only places the clusters the warp path left (listed in lidx[2])
  if (p.cluster && (int64_t)ncur * g.P < g.C) {
    const int32_t S = p.ctr->n_serial;
    if (S == 0) return;  // block-uniform
    long long ev_serial = 0;
    // one warp, each thread with its scratch in the dynamic shared memory
    SerialScratch* scratch = reinterpret_cast<SerialScratch*>(dsm);
    if (threadIdx.x < kSerialThreads)
      for (int32_t i = threadIdx.x; i < S; i += kSerialThreads)
        place_cluster_serial(p, __ldcg(p.lidx[2] + i), ncur, scratch[threadIdx.x], ev_serial);
    const long long evs = block_sum_ll(ev_serial, sm);
    if (threadIdx.x == 0 && evs) atomic_add_ll(&p.stats->n_evicted, evs);
    return;
  }
  if (r0 == 0 && threadIdx.x == 0) p.stats->n_inserted = ncur;
  long long evicted = 0, rounds = 0;
  if (ncur > kClusterMax) {
    // claim rounds need this round's claims, which the last grid-wide round skipped
    for (int32_t i = threadIdx.x; i < ncur; i += blockDim.x)
      claim_window(p.claims[r0 % 3], __ldcg(p.lkey[r0 % 3] + i), g);
    __threadfence();
    __syncthreads();
    finish_by_rounds(p, r0, nprev, ncur, evicted, rounds);
  } else {
    long long* s_k = reinterpret_cast<long long*>(dsm);
    uint32_t* s_h = reinterpret_cast<uint32_t*>(dsm + 8 * kClusterMax);
    int32_t* s_u = reinterpret_cast<int32_t*>(dsm + 12 * kClusterMax);
    int32_t* s_off = reinterpret_cast<int32_t*>(dsm + 16 * kClusterMax);
    const int rc = r0 % 3;
    for (int b = threadIdx.x; b <= kClusterBuckets; b += blockDim.x) s_off[b] = 0;
    __syncthreads();
    // bucket of each key (buckets partition the slot range in order)
    constexpr int kPer = kClusterMax / 1024;
    long long kk[kPer];
    int32_t uu[kPer], bb[kPer], rk[kPer];
    uint32_t hh[kPer];
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      const int32_t i = threadIdx.x + q * 1024;
      bb[q] = -1;
      if (i < ncur) {
        kk[q] = __ldcg(p.lkey[rc] + i);
        uu[q] = __ldcg(p.lidx[rc] + i);
        hh[q] = (uint32_t)home_slot(kk[q], g);
        bb[q] = (int32_t)(((uint64_t)hh[q] * kClusterBuckets) / (uint64_t)g.C);
        rk[q] = atomicAdd(&s_off[bb[q]], 1);
      }
    }
    __syncthreads();
    {  // exclusive scan of the bucket counts (4 buckets per thread)
      constexpr int kBper = kClusterBuckets / 1024;
      int c[kBper], sum = 0;
#pragma unroll
      for (int q = 0; q < kBper; ++q) {
        c[q] = s_off[threadIdx.x * kBper + q];
        sum += c[q];
      }
      int total = 0;
      int run = block_excl_scan(sum, smi, total);
#pragma unroll
      for (int q = 0; q < kBper; ++q) {
        s_off[threadIdx.x * kBper + q] = run;
        run += c[q];
      }
      if (threadIdx.x == 0) s_off[kClusterBuckets] = total;
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      if (bb[q] < 0) continue;
      const int32_t at = s_off[bb[q]] + rk[q];
      s_k[at] = kk[q];
      s_h[at] = hh[q];
      s_u[at] = uu[q];
    }
    __syncthreads();
    // insertion sort of each bucket by home slot
    for (int b = threadIdx.x; b < kClusterBuckets; b += blockDim.x) {
      const int32_t lo = s_off[b], hi = s_off[b + 1];
      for (int32_t i = lo + 1; i < hi; ++i) {
        const uint32_t h = s_h[i];
        const long long k = s_k[i];
        const int32_t u = s_u[i];
        int32_t j = i - 1;
        while (j >= lo && s_h[j] > h) {
          s_h[j + 1] = s_h[j];
          s_k[j + 1] = s_k[j];
          s_u[j + 1] = s_u[j];
          --j;
        }
        s_h[j + 1] = h;
        s_k[j + 1] = k;
        s_u[j + 1] = u;
      }
    }
    __syncthreads();
    // clusters: a run ends where the next home slot is P or more further on
    const int32_t N = ncur;
    const bool wrap = N > 1 && ((int64_t)s_h[0] + g.C - (int64_t)s_h[N - 1]) < g.P;
    int any_inner_head = 0;
    for (int32_t i = 1 + threadIdx.x; i < N; i += blockDim.x)
      any_inner_head |= ((int64_t)s_h[i] - (int64_t)s_h[i - 1]) >= g.P;
    any_inner_head = __syncthreads_or(any_inner_head);
    for (int32_t i = threadIdx.x; i < N; i += blockDim.x) {
      bool head;
      if (i == 0)
        head = !wrap || !any_inner_head;
      else
        head = ((int64_t)s_h[i] - (int64_t)s_h[i - 1]) >= g.P;
      if (!head) continue;
      // members: i, i+1, ... up to (not including) the next head, cyclically
      int32_t m = 1;
      while (m < N) {
        const int32_t j = (i + m) % N;
        const bool jhead =
            j == 0 ? (!wrap || !any_inner_head) : ((int64_t)s_h[j] - (int64_t)s_h[j - 1]) >= g.P;
        if (jhead) break;
        ++m;
      }
      // place the members in ascending key order (placed members marked -1)
      for (int32_t done = 0; done < m; ++done) {
        int32_t arg = -1;
        long long kmin = 0;
        for (int32_t t = 0; t < m; ++t) {
          const int32_t j = (i + t) % N;
          const long long k = s_k[j];
          if (k >= 0 && (arg < 0 || k < kmin)) {
            arg = j;
            kmin = k;
          }
        }
        place_key(p, kmin, s_u[arg], evicted);
        s_k[arg] = -1;
      }
    }
    rounds = N > 0;
  }
  const long long ev = block_sum_ll(evicted, sm);
  if (threadIdx.x == 0) {
    if (ev) atomic_add_ll(&p.stats->n_evicted, ev);
    if (rounds) atomic_add_ll(&p.stats->n_rounds, rounds);
  }
}

// ---------------------------------------------------------------------------
// Cluster placement (default insert path), grid-wide and exact.
//
// Windows W(a) and W(b) overlap exactly when the home slots are less than P
// apart on the ring.  Cut the ring's occupied home slots wherever two
// consecutive ones are P or more apart: each run (cluster) touches a set of
// slots no other cluster touches, so placing each cluster's keys in ascending
// key order, clusters independently, gives the state of the sequential insert
// of all missing keys in ascending order.  The re-probe linked every missing
// key into the list of its home slot.  The key whose index heads its slot's
// list represents the slot; a representative with no occupied slot among the
// P-1 slots before its own heads its cluster.  Three places do the work:
//   k_place_clusters  one thread per missing key; a lone key (no other key
//                     within P-1 slots, none sharing its slot) is decided and
//                     placed from one batch of loads; heads of larger
//                     clusters are listed;
//   k_place_multi     one warp per listed cluster (place_cluster_warp);
//   k_insert_finish   clusters beyond the warp path's limits, one thread each
//                     (place_cluster_serial), and every key when the windows
//                     may cover the whole ring.
// A cut exists when the windows do not cover the whole ring, which is certain
// when N * P < C (N missing keys); otherwise the grid-wide passes place
// nothing.
// ---------------------------------------------------------------------------

__device__ __forceinline__ bool slot_used(unsigned long long v, uint32_t tag) {
  return (uint32_t)(v >> 32) == tag;
}

__device__ __forceinline__ int64_t ring_add(int64_t h, int64_t d, int64_t C) {
  int64_t s = h + d;  // |d| < C
  if (s < 0) s += C;
  if (s >= C) s -= C;
  return s;
}

// Adds (key, distinct-id index) to the first n entries of ck/cu, kept in
// ascending key order; false when kClusterLocal entries are already held.
__device__ __forceinline__ bool sorted_add(long long* ck, int32_t* cu, int& n, long long kk,
                                           int32_t uu) {
  if (n == kClusterLocal) return false;
  int j = n++;
  for (; j > 0 && ck[j - 1] > kk; --j) {
    ck[j] = ck[j - 1];
    cu[j] = cu[j - 1];
  }
  ck[j] = kk;
  cu[j] = uu;
  return true;
}

// Smallest unplaced key of the cluster [h, h + L] (urow < 0 until placed), by
// walking the slot lists; returns its list-0 index or -1.  Slow path for
// clusters too large to sort in registers (never on the benchmark workloads).
__device__ int32_t cluster_min_unplaced(const WbParams& p, int64_t h, int64_t L, int32_t N) {
  const Geo& g = p.g;
  int32_t arg = -1;
  long long kmin = 0;
  for (int64_t off = 0; off <= L; ++off) {
    const unsigned long long v = ld_cg(p.shead + ring_add(h, off, g.C));
    if (!slot_used(v, p.tag)) continue;
    for (int32_t x = (int32_t)(uint32_t)v, hops = 0; x >= 0 && hops <= N;
         x = __ldcg(p.snext + x), ++hops) {
      const long long k = __ldcg(p.lkey[0] + x);
      if (__ldcg(p.urow + __ldcg(p.lidx[0] + x)) == -1 && (arg < 0 || k < kmin)) {
        arg = x;
        kmin = k;
      }
    }
  }
  return arg;
}

// Serial placement of the cluster headed at slot h by one thread: walk 8 slot
// heads per batch, collect and sort the keys, copy the span's steps and decide
// every placement on the copy; clusters beyond the local limits place key by
// key in global memory.  Used where the warp path does not apply.
__device__ void place_cluster_serial(const WbParams& p, int64_t h, int32_t N, SerialScratch& w,
                                     long long& evicted) {
  const Geo& g = p.g;
  unsigned long long* heads = w.heads;
  int nh = 0;
  bool overflow = false;
  heads[nh++] = ld_cg(p.shead + h);
  int64_t L = 0;
  for (int64_t off = 1; off <= L + g.P - 1 && off < g.C;) {
    unsigned long long w[8];
#pragma unroll
    for (int q = 0; q < 8; ++q)
      w[q] = off + q < g.C ? ld_cg(p.shead + ring_add(h, off + q, g.C)) : 0;
    int q = 0;
    for (; q < 8; ++q) {
      const int64_t o = off + q;
      if (o > L + g.P - 1 || o >= g.C) break;
      if (slot_used(w[q], p.tag)) {
        L = o;
        if (nh < kClusterLocal)
          heads[nh++] = w[q];
        else
          overflow = true;
      }
    }
    off += q;
    if (q < 8) break;
  }
  long long* ck = w.ck;
  int32_t* cu = w.cu;
  int n = 0;
  for (int i = 0; i < nh && !overflow; ++i)
    for (int32_t x = (int32_t)(uint32_t)heads[i], hops = 0; x >= 0 && hops <= N && !overflow;
         x = __ldcg(p.snext + x), ++hops)
      overflow |= !sorted_add(ck, cu, n, __ldcg(p.lkey[0] + x), __ldcg(p.lidx[0] + x));
  const int64_t span = L + g.P;
  if (!overflow && span <= kSpanLocal) {
    long long* sl = w.sl;
    for (int64_t o0 = 0; o0 < span; o0 += 16) {
      long long v[16];
#pragma unroll
      for (int q = 0; q < 16; ++q)
        v[q] = o0 + q < span ? ld_cg(p.last + ring_add(h, o0 + q, g.C)) : 0;
#pragma unroll
      for (int q = 0; q < 16; ++q)
        if (o0 + q < span) sl[o0 + q] = v[q];
    }
    for (int j = 0; j < n; ++j) {
      const long long kk = ck[j];
      int64_t off = home_slot(kk, g) - h;
      if (off < 0) off += g.C;
      int64_t best = -1, best_o = 0;
      long long best_last = 0;
      for (int32_t q = 0; q < g.P; ++q) {
        const int64_t o = off + q;
        const int64_t s = ring_add(h, o, g.C);
        if (best < 0 || sl[o] < best_last || (sl[o] == best_last && s < best)) {
          best = s;
          best_o = o;
          best_last = sl[o];
        }
      }
      if (best_last != -1) ++evicted;
      emit_placement(p, best, best_last, cu[j]);
      sl[best_o] = p.step;
      p.keys[best] = kk;
      p.last[best] = p.step;
      p.urow[cu[j]] = (int32_t)best;
    }
    return;
  }
  if (!overflow) {
    for (int j = 0; j < n; ++j) place_key(p, ck[j], cu[j], evicted);
    return;
  }
  for (int32_t it = 0; it <= N; ++it) {
    const int32_t x = cluster_min_unplaced(p, h, L, N);
    if (x < 0) return;
    place_key(p, __ldcg(p.lkey[0] + x), __ldcg(p.lidx[0] + x), evicted);
  }
  set_status(p.status, kStInternal);  // more placements than keys: never expected
}

// Per-warp shared scratch of the warp path: the cluster's keys as collected
// and in ascending order.
constexpr int kWarpSpan = 64;  // slots (offsets 0..63 from the head) one warp loads at once
constexpr int kWarpKeys = 64;
struct WarpCluster {
  long long k[kWarpKeys];
  long long ks[kWarpKeys];
  int32_t u[kWarpKeys];
  int32_t us[kWarpKeys];
  int n;
};

// The whole warp places the cluster headed at slot h: lane l holds offsets l
// and l + 32 (slot head and last-write step, one batch of loads), the cluster
// end comes from the occupancy ballot, lanes fetch the slot lists' keys, a
// rank count orders them, and each placement is an argmin of (step, row) over
// lanes q < P of the window, exchanged by shuffles; lane 0 stores.  Returns
// false, having written nothing to the table, when the cluster is outside the
// path's limits (P > 32, span > 64 slots, more than 64 keys, C < 128).
__device__ bool place_cluster_warp(const WbParams& p, int64_t h, int32_t N, WarpCluster& sw,
                                   long long& evicted) {
  const Geo& g = p.g;
  const int lane = threadIdx.x & 31;
  if (g.P > 32 || g.C < 2 * kWarpSpan) return false;
  const int64_t s0 = ring_add(h, lane, g.C), s1 = ring_add(h, lane + 32, g.C);
  const unsigned long long v0 = ld_cg(p.shead + s0), v1 = ld_cg(p.shead + s1);
  long long l0 = ld_cg(p.last + s0), l1 = ld_cg(p.last + s1);
  const unsigned long long occ =
      (unsigned long long)__ballot_sync(0xFFFFFFFFu, slot_used(v0, p.tag)) |
      ((unsigned long long)__ballot_sync(0xFFFFFFFFu, slot_used(v1, p.tag)) << 32);
  int L = 0;  // offset of the cluster's last occupied slot
  while (L < 63) {
    const unsigned long long later = occ & ~((2ull << L) - 1ull);
    if (!later) break;
    const int o = __ffsll((long long)later) - 1;
    if (o > L + g.P - 1) break;
    L = o;
  }
  if (L + g.P > kWarpSpan) return false;
  __syncwarp();
  if (lane == 0) sw.n = 0;
  __syncwarp();
  bool too_many = false;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int o = lane + 32 * half;
    const unsigned long long v = half ? v1 : v0;
    if (o > L || !slot_used(v, p.tag)) continue;
    for (int32_t x = (int32_t)(uint32_t)v, hops = 0; x >= 0 && hops <= N;
         x = __ldcg(p.snext + x), ++hops) {
      const int at = atomicAdd(&sw.n, 1);
      if (at < kWarpKeys) {
        sw.k[at] = __ldcg(p.lkey[0] + x);
        sw.u[at] = __ldcg(p.lidx[0] + x);
      } else {
        too_many = true;
      }
    }
  }
  __syncwarp();
  if (__any_sync(0xFFFFFFFFu, too_many)) return false;
  const int n = sw.n;
  for (int j = lane; j < n; j += 32) {  // rank = number of smaller keys (keys are distinct)
    const long long kj = sw.k[j];
    int r = 0;
    for (int i = 0; i < n; ++i) r += sw.k[i] < kj;
    sw.ks[r] = kj;
    sw.us[r] = sw.u[j];
  }
  __syncwarp();
  int span_pow2 = 1;
  while (span_pow2 < g.P) span_pow2 <<= 1;
  for (int j = 0; j < n; ++j) {
    const long long k = sw.ks[j];
    int64_t off = home_slot(k, g) - h;
    if (off < 0) off += g.C;
    const int o = (int)off + lane;  // window offset of lane q = lane (< 64 for q < P)
    const long long a = __shfl_sync(0xFFFFFFFFu, l0, o & 31);
    const long long b = __shfl_sync(0xFFFFFFFFu, l1, o & 31);
    long long cl = o < 32 ? a : b;
    long long cs = ring_add(h, o, g.C);
    int co = o;
    if (lane >= g.P) {
      cl = 0x7FFFFFFFFFFFFFFFll;
      cs = 0x7FFFFFFFFFFFFFFFll;
    }
    // argmin over lanes 0..P-1 (lanes >= P hold +inf): the xor rounds below
    // the next power of two >= P reduce every aligned group of that width, so
    // lane 0 holds the window's minimum; it is then broadcast
    for (int d = span_pow2 >> 1; d > 0; d >>= 1) {
      const long long ol = __shfl_xor_sync(0xFFFFFFFFu, cl, d);
      const long long os = __shfl_xor_sync(0xFFFFFFFFu, cs, d);
      const int oo = __shfl_xor_sync(0xFFFFFFFFu, co, d);
      if (ol < cl || (ol == cl && os < cs)) {
        cl = ol;
        cs = os;
        co = oo;
      }
    }
    cl = __shfl_sync(0xFFFFFFFFu, cl, 0);
    cs = __shfl_sync(0xFFFFFFFFu, cs, 0);
    co = __shfl_sync(0xFFFFFFFFu, co, 0);
    if (co < 32) {
      if (lane == co) l0 = p.step;
    } else if (lane == co - 32) {
      l1 = p.step;
    }
    if (lane == 0) {
      if (cl != -1) ++evicted;
      emit_placement(p, cs, cl, sw.us[j]);
      p.keys[cs] = k;
      p.last[cs] = p.step;
      p.urow[sw.us[j]] = (int32_t)cs;
    }
  }
  return true;
}

// First look at missing key m by its own thread.  Places a lone key (no other
// key with a start slot within P-1 on either side, none sharing its own) from
// one batch of loads and returns 0; returns 0 for a key that is not its slot's
// representative or not the head of its cluster; returns 1, with its start
// slot in h_out, for the head of a cluster that needs more than that.
__device__ int place_lone(const WbParams& p, int32_t m, long long& evicted, int64_t& h_out) {
  const Geo& g = p.g;
  const long long k = __ldcg(p.lkey[0] + m);
  const int64_t h = home_slot(k, g);
  h_out = h;
  if (g.P > 8) {
    const unsigned long long vh = ld_cg(p.shead + h);
    if (!slot_used(vh, p.tag) || (int32_t)(uint32_t)vh != m) return 0;
    for (int64_t off = 1; off < g.P; ++off)
      if (slot_used(ld_cg(p.shead + ring_add(h, -off, g.C)), p.tag)) return 0;
    return 1;
  }
  // one batch: slot heads h-P+1 .. h+P-1, the key's list link, its window's steps
  unsigned long long v[15];
  long long l[8];
#pragma unroll
  for (int j = 0; j < 15; ++j)
    v[j] = j < 2 * g.P - 1 ? ld_cg(p.shead + ring_add(h, j - (g.P - 1), g.C)) : 0;
#pragma unroll
  for (int q = 0; q < 8; ++q) l[q] = q < g.P ? ld_cg(p.last + wslot(h, q, g)) : 0;
  const int32_t nx = __ldcg(p.snext + m);
  unsigned long long vh = 0;
  bool back = false, fwd = false;
#pragma unroll
  for (int j = 0; j < 15; ++j) {
    if (j >= 2 * g.P - 1) continue;
    const bool u = slot_used(v[j], p.tag);
    if (j < g.P - 1)
      back |= u;
    else if (j == g.P - 1)
      vh = v[j];
    else
      fwd |= u;
  }
  if (!slot_used(vh, p.tag) || (int32_t)(uint32_t)vh != m) return 0;  // not the representative
  if (back) return 0;  // not the head of its cluster
  if (fwd || nx >= 0) return 1;
  int64_t best = -1;
  long long best_last = 0;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    if (q >= g.P) continue;
    const int64_t s = wslot(h, q, g);
    if (best < 0 || l[q] < best_last || (l[q] == best_last && s < best)) {
      best = s;
      best_last = l[q];
    }
  }
  if (best_last != -1) ++evicted;
  const int32_t u = __ldcg(p.lidx[0] + m);
  emit_placement(p, best, best_last, u);
  p.keys[best] = k;
  p.last[best] = p.step;
  p.urow[u] = (int32_t)best;
  return 0;
}

// Pass 1 of the cluster path: one thread per missing key; lone keys are placed,
// heads of larger clusters are listed (start slot) for pass 2.
__global__ void __launch_bounds__(kBlock) k_place_clusters(WbParams p) {
  pdl_enter();
  __shared__ long long sm[33];
  const int32_t N = p.ctr->cnt[0];
  const bool ring_may_be_covered = (int64_t)N * p.g.P >= p.g.C;
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    p.stats->n_inserted = N;
    if (p.emit) {  // no k_write_list on this path: the list is the distinct-id arrays
      p.stats->n_unique = p.ctr->n_unique;
      *p.wcount = p.ctr->n_unique;
    }
    if (N > 0) atomic_add_ll(&p.stats->n_rounds, 1LL);
  }
  long long evicted = 0;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < p.n_fill; i += stride)
    fill_lookup(p, i);
  if (!ring_may_be_covered) {
    for (int64_t m = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; m < N; m += stride) {
      int64_t h = 0;
      if (place_lone(p, (int32_t)m, evicted, h)) p.lidx[1][warp_append(&p.ctr->n_multi)] = (int32_t)h;
    }
  }
  pdl_trigger();
  const long long ev = block_sum_ll(evicted, sm);
  if (threadIdx.x == 0 && ev) atomic_add_ll(&p.stats->n_evicted, ev);
}

// Pass 2: one warp per listed cluster head; clusters outside the warp path's
// limits are listed for the single-block kernel.
__global__ void __launch_bounds__(kBlock) k_place_multi(WbParams p) {
  pdl_enter();
  __shared__ long long sm[33];
  __shared__ WarpCluster s_warp[kBlock / 32];
  const int32_t N = p.ctr->cnt[0];
  const int32_t H = p.ctr->n_multi;
  const int lane = threadIdx.x & 31;
  WarpCluster& sw = s_warp[threadIdx.x >> 5];
  long long evicted = 0;
  const int64_t warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; w < H; w += warps) {
    const int64_t h = __ldcg(p.lidx[1] + w);
    if (!place_cluster_warp(p, h, N, sw, evicted) && lane == 0)
      p.lidx[2][atomicAdd(&p.ctr->n_serial, 1)] = (int32_t)h;
    __syncwarp();
  }
  pdl_trigger();
  const long long ev = block_sum_ll(evicted, sm);
  if (threadIdx.x == 0 && ev) atomic_add_ll(&p.stats->n_evicted, ev);
}

// ---------------------------------------------------------------------------
// End of the row map: the write list holds (row, position of e) for every
// distinct id that still owns its row after all inserts (a distinct id evicted
// again later in the same step gets no write, n_dropped).  Also clears the
// claims checked by the last grid-wide round (list 0's when there was none),
// still set at this point, and writes the remaining counters.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kBlock) k_write_list(WbParams p) {
  pdl_enter();
  __shared__ long long sm[33];
  __shared__ int smi[33];
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  if (!p.cluster) {
    // clearing a window that is already clear is harmless
    const int L = p.wide_rounds > 0 ? p.wide_rounds - 1 : 0;
    const int32_t nl = p.ctr->cnt[L & 3];
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nl; i += stride)
      clear_window(p.claims[L % 3], p.lkey[L % 3][i], p.g);
  }
  const int32_t U = p.ctr->n_unique;
  if (blockIdx.x == 0 && threadIdx.x == 0) p.stats->n_unique = U;
  long long dropped = 0;
  for (int64_t base = (int64_t)blockIdx.x * blockDim.x; base < U; base += stride) {
    const int64_t u = base + threadIdx.x;
    bool owned = false;
    int32_t r = -1;
    if (u < U) {
      r = p.urow[u];
      owned = r >= 0 && p.keys[r] == p.ukey[u];
      dropped += !owned;
    }
    int m = 0, unused = 0;
    block_append2(owned, 0, p.wcount, p.wcount, m, unused, smi);
    if (owned) {
      p.wrow[m] = r;
      p.wpos[m] = p.upos[u];
      p.whit[m] = p.uhit[u];
    }
  }
  pdl_trigger();
  const long long d = block_sum_ll(dropped, sm);
  if (threadIdx.x == 0 && d) atomic_add_ll(&p.stats->n_dropped, d);
}

// ---------------------------------------------------------------------------
// Writeback row update: M[r] <- fl(e_hat - fl(eta * fl(e_hat - e))) (eta = 1:
// the exact Writeback) for every entry of the write list; one warp per row, 16-byte vectors, loads of a chunk issued
// before its stores.  Reads only the write list, M and e.  Rows and targets
// are touched once per step, so they go through L2 as streaming (evict-first)
// accesses, which leaves the identity map, step and list arrays of the row
// map -- a few tens of MB -- resident in L2 while this kernel runs.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kBlock) k_writeback(const int32_t* __restrict__ wrow,
                                                      const int32_t* __restrict__ wpos,
                                                      const int32_t* wcount,
                                                      float4* __restrict__ M,
                                                      const float4* __restrict__ e, int D4,
                                                      float eta) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int32_t W = *wcount;
  const int64_t warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; w < W; w += warps) {
    const int32_t r = wrow[w];
    if (r < 0) continue;  // tombstone: the id lost its row later in the step
    float4* m = M + (int64_t)r * D4;
    const float4* ev = e + (int64_t)wpos[w] * D4;
    for (int base = 0; base < D4; base += 4 * 32) {
      float4 a[4], b[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int c = base + q * 32 + lane;
        if (c < D4) {
          a[q] = __ldcs(m + c);
          b[q] = __ldcs(ev + c);
        }
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int c = base + q * 32 + lane;
        if (c < D4) {
          // SGD step with gradient g = e_hat - e: M <- e_hat - fl(eta * g); every
          // operation rounded separately (eta = 1: e_hat - (e_hat - e) exactly,
          // since fl(1 * g) = g)
          float4 o;
          o.x = __fsub_rn(a[q].x, __fmul_rn(eta, __fsub_rn(a[q].x, b[q].x)));
          o.y = __fsub_rn(a[q].y, __fmul_rn(eta, __fsub_rn(a[q].y, b[q].y)));
          o.z = __fsub_rn(a[q].z, __fmul_rn(eta, __fsub_rn(a[q].z, b[q].z)));
          o.w = __fsub_rn(a[q].w, __fmul_rn(eta, __fsub_rn(a[q].w, b[q].w)));
          __stcs(m + c, o);
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Bulk-copy row kernels.  A warp keeps kBulkStages rows in flight: one lane
// issues 1-D bulk copies (cp.async.bulk, global -> shared, no multicast) of
// each row into the warp's own shared-memory stage, completed on that stage's
// mbarrier; the lanes read the stage as 16-byte vectors and store the result
// with coalesced 512 B requests.  The rows in flight live in shared memory, not
// in registers, so far fewer warps keep HBM busy than in the register path,
// which leaves warp slots to the latency-bound row-map kernels running
// alongside.  Every wait on an mbarrier has a time limit; past it the kernel
// sets MPZCH_STATUS_TIMEOUT, waits (again with a limit) for its copies still
// in flight and returns.
// ---------------------------------------------------------------------------
constexpr int kBulkStages = 3;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

// L2 eviction-priority policies for the cache-hinted accesses.
enum L2Hint { kL2EvictFirst = 0, kL2Normal = 1, kL2EvictLast = 2 };

__device__ __forceinline__ uint64_t l2_policy(int hint) {
  uint64_t pol;
  if (hint == kL2EvictFirst)
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  else if (hint == kL2EvictLast)
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  else
    asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// One arrival that also announces `bytes` of bulk-copy data for this phase.
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for phase `parity` of the mbarrier to complete, for at most
// kWaitLimitNs; false when the limit ran out.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (;;) {
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > kWaitLimitNs) return false;
  }
}

// 1-D bulk copy global -> this CTA's shared memory, completing `bytes` of
// transaction count on the mbarrier (16-byte aligned addresses, bytes % 16 == 0).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar), "l"(pol)
      : "memory");
}

__device__ __forceinline__ float4 lds4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr));
  return v;
}

__device__ __forceinline__ void stg4_hint(float4* p, float4 v, uint64_t pol) {
  asm volatile("st.global.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p), "f"(v.x),
               "f"(v.y), "f"(v.z), "f"(v.w), "l"(pol)
               : "memory");
}

// Shared memory of a bulk row kernel: per warp kBulkStages stages of
// `stage_bytes`, then one 8-byte mbarrier per (warp, stage).
__host__ __device__ constexpr size_t bulk_smem_bytes(int warps, size_t stage_bytes) {
  return (size_t)warps * kBulkStages * stage_bytes + (size_t)warps * kBulkStages * 8;
}

// Per-warp stream of work items taken in chunks of 32 from a shared counter
// (dynamic, so a warp that starts late takes less); lane l caches item
// base + l of the current chunk.  Warp-collective.
struct ChunkCursor {
  int32_t base, pos, end;
  bool done;
};

// Row update through shared memory (same result as k_writeback): for every
// write-list entry, M[r] <- fl(e_hat - fl(eta * fl(e_hat - e))).  Entries are
// taken from *wtake in chunks of 32 per warp.
__global__ void k_writeback_bulk(const int32_t* __restrict__ wrow, const int32_t* __restrict__ wpos,
                                 const int32_t* wcount, int32_t* wtake, float4* __restrict__ M,
                                 const float4* __restrict__ e, int D4, float eta, int hint_m,
                                 int32_t* status) {
  pdl_enter();
  extern __shared__ __align__(128) unsigned char bsm[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const uint32_t RB = (uint32_t)D4 * 16u;  // bytes of one row
  const size_t stage_bytes = 2 * (size_t)RB;
  const uint32_t stage0 = smem_addr(bsm + (size_t)warp * kBulkStages * stage_bytes);
  const uint32_t bar0 =
      smem_addr(bsm + (size_t)nwarps * kBulkStages * stage_bytes) + warp * kBulkStages * 8;
  if (lane == 0)
    for (int s = 0; s < kBulkStages; ++s) mbar_init(bar0 + 8 * s, 1);
  mbar_init_fence();
  __syncwarp();
  const uint64_t pol_e = l2_policy(kL2EvictFirst);
  const uint64_t pol_m = l2_policy(hint_m);
  const int32_t W = *wcount;
  ChunkCursor cur{0, 0, 0, false};
  int32_t c_row = 0, c_pos = 0;
  int32_t srow[kBulkStages];
  // warp-collective: next entry into stage s (srow[s] = -1 when none is left);
  // tombstones (row -1) are skipped, across chunk boundaries
  auto issue = [&](int s) {
    int32_t r = -1, q = 0;
    while (r < 0 && !cur.done) {
      if (cur.pos == cur.end) {
        int32_t b = 0;
        if (lane == 0) b = atomicAdd(wtake, 32);
        b = __shfl_sync(0xFFFFFFFFu, b, 0);
        if (b >= W) {
          cur.done = true;
        } else {
          cur.base = cur.pos = b;
          cur.end = b + 32 < W ? b + 32 : W;
          if (lane < cur.end - b) {
            c_row = wrow[b + lane];
            c_pos = wpos[b + lane];
          }
        }
        continue;
      }
      const int src = cur.pos - cur.base;
      r = __shfl_sync(0xFFFFFFFFu, c_row, src);
      q = __shfl_sync(0xFFFFFFFFu, c_pos, src);
      ++cur.pos;
    }
    if (r >= 0 && lane == 0) {
      const uint32_t st = stage0 + (uint32_t)(s * stage_bytes);
      mbar_expect_tx(bar0 + 8 * s, 2 * RB);
      bulk_load(st, M + (int64_t)r * D4, RB, bar0 + 8 * s, pol_m);
      bulk_load(st + RB, e + (int64_t)q * D4, RB, bar0 + 8 * s, pol_e);
    }
    srow[s] = r;
  };
#pragma unroll
  for (int s = 0; s < kBulkStages; ++s) issue(s);
  uint32_t pbits = 0;  // bit s: parity of the phase stage s's copies complete
  bool failed = false;
  while (!failed) {
    bool any = false;
#pragma unroll
    for (int s = 0; s < kBulkStages; ++s) {
      if (srow[s] < 0 || failed) continue;
      any = true;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(bar0 + 8 * s, (pbits >> s) & 1u))) {
        failed = true;
        continue;
      }
      pbits ^= 1u << s;
      const uint32_t st = stage0 + (uint32_t)(s * stage_bytes);
      float4* m = M + (int64_t)srow[s] * D4;
      for (int c = lane; c < D4; c += 32) {
        const float4 a = lds4(st + 16u * c);
        const float4 b = lds4(st + RB + 16u * c);
        float4 o;
        o.x = __fsub_rn(a.x, __fmul_rn(eta, __fsub_rn(a.x, b.x)));
        o.y = __fsub_rn(a.y, __fmul_rn(eta, __fsub_rn(a.y, b.y)));
        o.z = __fsub_rn(a.z, __fmul_rn(eta, __fsub_rn(a.z, b.z)));
        o.w = __fsub_rn(a.w, __fmul_rn(eta, __fsub_rn(a.w, b.w)));
        stg4_hint(m + c, o, pol_m);
      }
      __syncwarp();  // every lane has read the stage before it is refilled
      issue(s);
    }
    if (!any) break;
  }
  if (failed) {
    if (lane == 0) set_status(status, kStTimeout);
    // copies still in flight must land before the block's shared memory goes
    for (int s = 0; s < kBulkStages; ++s)
      if (srow[s] >= 0) mbar_wait(bar0 + 8 * s, (pbits >> s) & 1u);
  }
}

// Fused gather through shared memory (same result as k_gather_fused): per
// output row one bulk copy of the cached row (hits) and one of the always-on
// row, then the lanes write the row (zeros for a miss) with coalesced 16-byte
// stores.  Items i = warp, warp + warps, ... in chunks of 32 per warp.
__global__ void k_gather_bulk(const int32_t* __restrict__ rows, const uint8_t* __restrict__ hit,
                              int64_t n, const float4* __restrict__ M, int64_t C, int D4,
                              const float4* __restrict__ ao, int64_t ao_n, int A4,
                              const int32_t* __restrict__ ao_rows, float4* __restrict__ out,
                              int hint_m, int32_t* status) {
  pdl_enter();
  extern __shared__ __align__(128) unsigned char bsm[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const uint32_t RB = (uint32_t)D4 * 16u, AB = (uint32_t)A4 * 16u;
  const size_t stage_bytes = (size_t)RB + AB;
  const uint32_t stage0 = smem_addr(bsm + (size_t)warp * kBulkStages * stage_bytes);
  const uint32_t bar0 =
      smem_addr(bsm + (size_t)nwarps * kBulkStages * stage_bytes) + warp * kBulkStages * 8;
  if (lane == 0)
    for (int s = 0; s < kBulkStages; ++s) mbar_init(bar0 + 8 * s, 1);
  mbar_init_fence();
  __syncwarp();
  const uint64_t pol_m = l2_policy(hint_m);
  const uint64_t pol_a = l2_policy(kL2EvictFirst);
  const int64_t G = (int64_t)gridDim.x * nwarps;
  const int64_t g = (int64_t)blockIdx.x * nwarps + warp;
  const int W4 = D4 + A4;
  // this warp's items: g + k * G for k = 0, 1, ...; lane l caches item k0 + l
  int64_t k_next = 0;  // next item (as k) to issue
  int64_t k_base = -32;
  int32_t c_r = 0, c_a = 0;
  int c_flags = 0;  // bit 0 hit (in range), bit 1 always-on row in range
  int64_t sidx[kBulkStages];
  int sflags[kBulkStages];
  auto issue = [&](int s) {
    const int64_t i = g + k_next * G;
    if (i >= n) {
      sidx[s] = -1;
      return;
    }
    if (k_next >= k_base + 32) {
      k_base = k_next;
      const int64_t li = g + (k_base + lane) * G;
      c_flags = 0;
      if (li < n) {
        const int32_t r = rows[li];
        if (hit[li]) {
          if (r >= 0 && (int64_t)r < C)
            c_flags |= 1;
          else
            set_status(status, kStBadRow);
        }
        c_r = r;
        if (A4 > 0) {
          c_a = ao_rows[li];
          if (c_a >= 0 && (int64_t)c_a < ao_n)
            c_flags |= 2;
          else
            set_status(status, kStBadAo);
        }
      }
    }
    const int src = (int)(k_next - k_base);
    const int32_t r = __shfl_sync(0xFFFFFFFFu, c_r, src);
    const int32_t a = __shfl_sync(0xFFFFFFFFu, c_a, src);
    const int f = __shfl_sync(0xFFFFFFFFu, c_flags, src);
    ++k_next;
    if (lane == 0) {
      const uint32_t st = stage0 + (uint32_t)(s * stage_bytes);
      const uint32_t bytes = ((f & 1) ? RB : 0u) + ((f & 2) ? AB : 0u);
      mbar_expect_tx(bar0 + 8 * s, bytes);
      if (f & 1) bulk_load(st, M + (int64_t)r * D4, RB, bar0 + 8 * s, pol_m);
      if (f & 2) bulk_load(st + RB, ao + (int64_t)a * A4, AB, bar0 + 8 * s, pol_a);
    }
    sidx[s] = i;
    sflags[s] = f;
  };
#pragma unroll
  for (int s = 0; s < kBulkStages; ++s) issue(s);
  uint32_t pbits = 0;  // bit s: parity of the phase stage s's copies complete
  bool failed = false;
  while (!failed) {
    bool any = false;
#pragma unroll
    for (int s = 0; s < kBulkStages; ++s) {
      if (sidx[s] < 0 || failed) continue;
      any = true;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(bar0 + 8 * s, (pbits >> s) & 1u))) {
        failed = true;
        continue;
      }
      pbits ^= 1u << s;
      const uint32_t st = stage0 + (uint32_t)(s * stage_bytes);
      float4* dst = out + sidx[s] * (int64_t)W4;
      const int f = sflags[s];
      const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int c = lane; c < W4; c += 32) {
        float4 v = z;
        if (c < D4) {
          if (f & 1) v = lds4(st + 16u * c);
        } else if (f & 2) {
          v = lds4(st + 16u * c);
        }
        __stcs(dst + c, v);
      }
      __syncwarp();
      issue(s);
    }
    if (!any) break;
  }
  if (failed) {
    if (lane == 0) set_status(status, kStTimeout);
    for (int s = 0; s < kBulkStages; ++s)
      if (sidx[s] >= 0) mbar_wait(bar0 + 8 * s, (pbits >> s) & 1u);
  }
}

// ---------------------------------------------------------------------------
// Select rows written at or after `since`, ascending, in two launches over
// tiles of kScanTile rows.  Thread t of a block reads rows t + 256k (k < 8) of
// its tile, so every load instruction covers 256 contiguous bytes.
//   k_select_mark     per tile, the 64 ballot words of its (sub-tile, warp)
//                     groups and its row count (the only pass over the table);
//   k_select_scatter  per tile, the sum of the earlier tiles' counts (a block
//                     reduction over at most a few thousand ints, L2-resident),
//                     then every selected row written at that offset plus its
//                     rank inside the tile, from the ballot words.
// The second kernel is launched with programmatic dependent launch, so its
// blocks start while the first drains.  No block waits on another.
// ---------------------------------------------------------------------------
constexpr int kScanThreads = 256;
constexpr int kScanPer = 8;
constexpr int kScanTile = kScanThreads * kScanPer;
constexpr int kScanWords = kScanPer * (kScanThreads / 32);  // ballot words per tile

__global__ void __launch_bounds__(kScanThreads) k_select_mark(const long long* __restrict__ keys,
                                                              const long long* __restrict__ last,
                                                              int64_t C, long long since,
                                                              uint32_t* __restrict__ masks,
                                                              int32_t* __restrict__ tcount) {
  pdl_enter();
  __shared__ int s_cnt[kScanThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t base = (int64_t)blockIdx.x * kScanTile + threadIdx.x;
  long long kv[kScanPer], lv[kScanPer];
#pragma unroll
  for (int k = 0; k < kScanPer; ++k) {
    const int64_t r = base + k * kScanThreads;
    kv[k] = r < C ? __ldcs(keys + r) : -1;
    lv[k] = r < C ? __ldcs(last + r) : -1;
  }
  int c = 0;
#pragma unroll
  for (int k = 0; k < kScanPer; ++k) {
    const unsigned b = __ballot_sync(0xFFFFFFFFu, kv[k] != -1 && lv[k] >= since);
    if (lane == 0) masks[(int64_t)blockIdx.x * kScanWords + k * (kScanThreads / 32) + warp] = b;
    c += __popc(b);
  }
  pdl_trigger();
  if (lane == 0) s_cnt[warp] = c;
  __syncthreads();
  if (threadIdx.x == 0) {
    int t = 0;
    for (int w = 0; w < kScanThreads / 32; ++w) t += s_cnt[w];
    tcount[blockIdx.x] = t;
  }
}

__global__ void __launch_bounds__(kScanThreads) k_select_scatter(
    const uint32_t* __restrict__ masks, const int32_t* __restrict__ tcount, int64_t C,
    int32_t* __restrict__ rows_out, long long* dev_count) {
  pdl_enter();
  __shared__ long long sm[33];
  __shared__ int s_off[kScanWords + 1];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int tile = blockIdx.x;
  // offset of this tile: counts of tiles 0 .. tile-1
  long long acc = 0;
  for (int q = threadIdx.x; q < tile; q += kScanThreads) acc += tcount[q];
  const long long excl = block_sum_ll(acc, sm);
  if (warp == 0) {  // exclusive scan of the 64 group counts, in row order
    const uint32_t a = masks[(int64_t)tile * kScanWords + 2 * lane];
    const uint32_t b = masks[(int64_t)tile * kScanWords + 2 * lane + 1];
    const int ca = __popc(a), cb = __popc(b);
    int x = ca + cb;
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xFFFFFFFFu, x, off);
      if (lane >= off) x += y;
    }
    s_off[2 * lane] = x - ca - cb;
    s_off[2 * lane + 1] = x - cb;
    if (lane == 31) s_off[kScanWords] = x;
    static_assert(kScanWords == 64, "one warp scans two counts per lane");
  }
  __syncthreads();
  const int64_t base = (int64_t)tile * kScanTile + threadIdx.x;
  const unsigned lt = (1u << lane) - 1u;
#pragma unroll
  for (int k = 0; k < kScanPer; ++k) {
    const int g = k * (kScanThreads / 32) + warp;
    const uint32_t b = masks[(int64_t)tile * kScanWords + g];
    if (b >> lane & 1u) rows_out[excl + s_off[g] + __popc(b & lt)] = (int32_t)(base + k * kScanThreads);
  }
  if (tile == gridDim.x - 1 && threadIdx.x == 0) *dev_count = excl + s_off[kScanWords];
}

// ---------------------------------------------------------------------------
// int8 export: one warp per row.  a = max|x| (exact), scale = a/127 and x/scale
// as IEEE divisions, round-half-even, clamp to +-127.  With last_out, the row's
// last-write step is exported too (metadata of the streamed snapshot).
// ---------------------------------------------------------------------------
// q = rne(fl(x / s)), clamped to +-127.  Fast path: p = fl(x * fl(1/s)) differs
// from the exact quotient t = x/s by at most |t| 2^-23 + |t| 2^-24, and fl(t)
// from t by at most |t| 2^-24, so |p - fl(x/s)| < |t| 2^-22 <= 127.00001 * 2^-22
// < 3.1e-5.  When p is more than 1e-4 away from every half-integer, fl(x/s)
// rounds to the same integer as p; otherwise the IEEE division is taken.  (A
// reciprocal that is not finite, for a subnormal s, sends every element to
// the division.)
// Round-half-to-even of |v| < 2^22 without a conversion instruction: adding
// 1.5 * 2^23 leaves v's nearest integer (ties to even, IEEE rounding of the
// add) in the low mantissa bits, and subtracting it again gives that integer as
// a float.  Only full-rate FP32 / integer operations.
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23
constexpr int kRoundMagicBits = 0x4B400000;

__device__ __forceinline__ int rne_small(float v) {
  return __float_as_int(__fadd_rn(v, kRoundMagic)) - kRoundMagicBits;
}

// int8 code of x / s for the values of one lane.  The product p = x * fl(1/s)
// is within 3.1e-5 of x / s, so rne(p) = rne(x / s) whenever p lies at least
// 1e-4 from a half-integer; a lane with any value closer than that (or with no
// usable reciprocal) recomputes all of its values from the IEEE quotient.
// |x| <= a = 127 s, so every code lies in [-127, 127] (clamped all the same).
template <int kN>
__device__ __forceinline__ void quant_lane(const float (&x)[kN], float s, float rcp, bool fast,
                                           int (&t)[kN]) {
  bool amb = !fast;
#pragma unroll
  for (int e = 0; e < kN; ++e) {
    const float p = __fmul_rn(x[e], rcp);
    const float y = __fadd_rn(p, kRoundMagic);
    const float r = __fsub_rn(y, kRoundMagic);
    amb |= fabsf(__fsub_rn(p, r)) > 0.4999f;
    t[e] = __float_as_int(y) - kRoundMagicBits;
  }
  if (amb) {
#pragma unroll
    for (int e = 0; e < kN; ++e) t[e] = rne_small(__fdiv_rn(x[e], s));
  }
#pragma unroll
  for (int e = 0; e < kN; ++e) t[e] = max(-127, min(127, t[e]));
}

__device__ __forceinline__ uint32_t pack4(int a, int b, int c, int d) {
  return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

// Any dim (multiple of 4): two passes over the row (max, then quantise) with
// 4-byte stores.
__device__ __forceinline__ void export_row_generic(const float4* __restrict__ x, char4* qo, int D4,
                                                   float* sc, long long* ko, long long* lo,
                                                   long long key, long long lastv, int lane) {
  float a = 0.f;
  for (int c = lane; c < D4; c += 32) {
    const float4 v = x[c];
    a = fmaxf(a, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
  }
  for (int off = 16; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, off));
  const float s = a == 0.f ? 0.f : __fdiv_rn(a, 127.0f);
  const float rcp = a == 0.f ? 0.f : __frcp_rn(s);
  const bool fast = a != 0.f && isfinite(rcp);
  for (int c = lane; c < D4; c += 32) {
    const float4 f = x[c];
    const float v[4] = {f.x, f.y, f.z, f.w};
    int t[4] = {0, 0, 0, 0};
    if (a != 0.f) quant_lane<4>(v, s, rcp, fast, t);
    qo[c] = make_char4((signed char)t[0], (signed char)t[1], (signed char)t[2], (signed char)t[3]);
  }
  if (lane == 0) {
    *sc = s;
    *ko = key;
    if (lo) *lo = lastv;
  }
}

__global__ void __launch_bounds__(kBlock, 4) k_export_int8(
    const int32_t* __restrict__ rows, int64_t n, const long long* dev_n,
    const float4* __restrict__ M, const long long* __restrict__ keys, int64_t C, int D4,
    char4* __restrict__ q, float* __restrict__ scale, long long* __restrict__ keys_out,
    int32_t* status, const long long* __restrict__ last, long long* __restrict__ last_out) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  int64_t nn = n;
  if (dev_n) {
    const long long d = *dev_n;
    nn = d < nn ? d : nn;
  }
  const int64_t warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; i < nn; i += warps) {
    const int32_t r = rows[i];
    char4* qo = q + i * (int64_t)D4;
    long long* lo = last_out ? last_out + i : nullptr;
    if (r < 0 || (int64_t)r >= C) {
      if (lane == 0) {
        set_status(status, kStBadRow);
        scale[i] = 0.f;
        keys_out[i] = -1;
        if (lo) *lo = -1;
      }
      for (int c = lane; c < D4; c += 32) qo[c] = make_char4(0, 0, 0, 0);
      continue;
    }
    const float4* x = M + (int64_t)r * D4;
    const long long key = keys[r];
    const long long lastv = last_out ? last[r] : 0;
    export_row_generic(x, qo, D4, scale + i, keys_out + i, lo, key, lastv, lane);
  }
}

// Export of rows of D = 128 * kPer values, one warp per row, through
// registers: lane l holds the 16-byte vectors l + 32 j (j < kPer) of the row,
// so every load instruction of the warp reads 512 contiguous bytes, and writes
// their codes as the 4-byte words l + 32 j of the int8 row, so every store
// instruction writes 128 contiguous bytes.  The next row's values are loaded
// before the current row is reduced and quantised (two rows in flight per
// warp).  Same results as k_export_int8.
template <int kPer>
__global__ void __launch_bounds__(kBlock) k_export_rows(
    const int32_t* __restrict__ rows, int64_t n, const long long* dev_n,
    const float4* __restrict__ M, const long long* __restrict__ keys, int64_t C,
    uint32_t* __restrict__ q, float* __restrict__ scale, long long* __restrict__ keys_out,
    int32_t* status, const long long* __restrict__ last, long long* __restrict__ last_out) {
  pdl_enter();
  constexpr int D4 = 32 * kPer;
  const int lane = threadIdx.x & 31;
  int64_t nn = n;
  if (dev_n) {
    const long long d = *dev_n;
    nn = d < nn ? d : nn;
  }
  const int64_t warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  float4 cur[kPer];
  int32_t rc = -1;
  auto fetch = [&](int64_t k, float4 (&v)[kPer], int32_t& r) {
    r = -1;
    if (k < nn) {
      r = rows[k];
      if (r >= 0 && (int64_t)r < C) {
        const float4* x = M + (int64_t)r * D4 + lane;
#pragma unroll
        for (int j = 0; j < kPer; ++j) v[j] = __ldcs(x + 32 * j);
      }
    }
  };
  fetch(i, cur, rc);
  for (; i < nn; i += warps) {
    float4 nxt[kPer];
    int32_t rn;
    fetch(i + warps, nxt, rn);
    uint32_t* qo = q + i * (int64_t)D4;
    if (rc < 0 || (int64_t)rc >= C) {
      if (lane == 0) {
        set_status(status, kStBadRow);
        scale[i] = 0.f;
        keys_out[i] = -1;
        if (last_out) last_out[i] = -1;
      }
#pragma unroll
      for (int j = 0; j < kPer; ++j) qo[32 * j + lane] = 0u;
    } else {
      float x[4 * kPer];
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        x[4 * j] = cur[j].x;
        x[4 * j + 1] = cur[j].y;
        x[4 * j + 2] = cur[j].z;
        x[4 * j + 3] = cur[j].w;
      }
      float a = 0.f;
#pragma unroll
      for (int e = 0; e < 4 * kPer; ++e) a = fmaxf(a, fabsf(x[e]));
      for (int off = 16; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, off));
      const float sc = a == 0.f ? 0.f : __fdiv_rn(a, 127.0f);
      const float rcp = a == 0.f ? 0.f : __frcp_rn(sc);
      const bool fast = a != 0.f && isfinite(rcp);
      int c[4 * kPer];
#pragma unroll
      for (int e = 0; e < 4 * kPer; ++e) c[e] = 0;
      if (a != 0.f) quant_lane<4 * kPer>(x, sc, rcp, fast, c);
#pragma unroll
      for (int j = 0; j < kPer; ++j)
        __stcs(qo + 32 * j + lane, pack4(c[4 * j], c[4 * j + 1], c[4 * j + 2], c[4 * j + 3]));
      if (lane == 0) {
        scale[i] = sc;
        keys_out[i] = keys[rc];
        if (last_out) last_out[i] = last[rc];
      }
    }
#pragma unroll
    for (int j = 0; j < kPer; ++j) cur[j] = nxt[j];
    rc = rn;
  }
}

// ---------------------------------------------------------------------------
// Serving gather from an int8 snapshot: one warp per id; lanes j < P probe the
// window, the first matching probe offset wins; then out = hit ? q*scale : +0.
// Lane l stores the 16-byte vector l + 32*c, so every store request covers a
// contiguous 512 B of the output row.  A warp's ids are i, i + warps, ...,
// software-pipelined one id deep: while the current id's int8 row and scale
// load, the next id's window is probed and the id after it is loaded, so an
// id costs one dependent round trip to memory (three without the pipeline).
// ---------------------------------------------------------------------------
constexpr int kServeVec = 4;  // char4 codes per lane in the overlapped round (D <= 512)

// First probe load of key k (k < 0: none): lane j < min(P, 32) loads window
// slot j; returns that key (-1 when the lane loads nothing) and sets h.
__device__ __forceinline__ long long serve_probe_issue(const long long* __restrict__ snap_keys,
                                                       const Geo& g, long long k, int lane,
                                                       int64_t& h) {
  h = k >= 0 ? home_slot(k, g) : 0;
  return (k >= 0 && lane < g.P) ? __ldg(snap_keys + wslot(h, lane, g)) : -1;
}

// Row of key k from its first probe load w (and the window's slots 32.. when
// P > 32): the slot of the smallest matching offset, or -1.
__device__ __forceinline__ int64_t serve_probe_resolve(const long long* __restrict__ snap_keys,
                                                       const Geo& g, long long k, int lane,
                                                       int64_t h, long long w) {
  int32_t best = 0x7FFFFFFF;
  if (k >= 0) {
    if (lane < g.P && w == k) best = lane;
    for (int32_t j = lane + 32; j < g.P; j += 32)
      if (__ldg(snap_keys + wslot(h, j, g)) == k && j < best) best = j;
  }
  for (int off = 16; off > 0; off >>= 1) best = min(best, __shfl_xor_sync(0xFFFFFFFFu, best, off));
  return (k >= 0 && best != 0x7FFFFFFF) ? wslot(h, best, g) : -1;
}

__global__ void __launch_bounds__(kBlock) k_serve_gather(
    const long long* __restrict__ snap_keys, Geo g, const char4* __restrict__ q,
    const float* __restrict__ scale, int D4, const long long* __restrict__ ids, int64_t n,
    int32_t* __restrict__ rows, uint8_t* __restrict__ hit, float4* __restrict__ out,
    int32_t* status) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int64_t warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (i >= n) return;  // warp-uniform
  // prologue: the first id's row, the second id
  long long k = ids[i];
  long long kn = i + warps < n ? ids[i + warps] : -1;
  int64_t h = 0;
  const long long w0 = serve_probe_issue(snap_keys, g, k, lane, h);
  int64_t r = serve_probe_resolve(snap_keys, g, k, lane, h, w0);
  const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
  while (true) {
    const int64_t nx = i + warps;
    // issue: the next id's first probe load, the id after it, this id's row
    int64_t hn = 0;
    const long long wn = nx < n ? serve_probe_issue(snap_keys, g, kn, lane, hn) : -1;
    const long long kn2 = nx + warps < n ? ids[nx + warps] : -1;
    const char4* qr = q + (r >= 0 ? r : 0) * (int64_t)D4;
    const float sc = r >= 0 ? __ldg(scale + r) : 0.f;
    char4 v[kServeVec];
#pragma unroll
    for (int u = 0; u < kServeVec; ++u) {
      const int c = u * 32 + lane;
      v[u] = make_char4(0, 0, 0, 0);
      if (r >= 0 && c < D4) v[u] = __ldg(qr + c);
    }
    if (lane == 0) {
      if (k < 0) set_status(status, kStBadKey);
      rows[i] = (int32_t)r;
      hit[i] = r >= 0;
    }
    float4* o = out + i * (int64_t)D4;
#pragma unroll
    for (int u = 0; u < kServeVec; ++u) {
      const int c = u * 32 + lane;
      if (c < D4)
        __stcs(o + c, r >= 0 ? make_float4(__fmul_rn((float)v[u].x, sc), __fmul_rn((float)v[u].y, sc),
                                           __fmul_rn((float)v[u].z, sc), __fmul_rn((float)v[u].w, sc))
                             : z);
    }
    for (int c = kServeVec * 32 + lane; c < D4; c += 32) {  // rows wider than 512
      if (r >= 0) {
        const char4 x = __ldg(qr + c);
        __stcs(o + c, make_float4(__fmul_rn((float)x.x, sc), __fmul_rn((float)x.y, sc),
                                  __fmul_rn((float)x.z, sc), __fmul_rn((float)x.w, sc)));
      } else {
        __stcs(o + c, z);
      }
    }
    if (nx >= n) break;  // warp-uniform
    r = serve_probe_resolve(snap_keys, g, kn, lane, hn, wn);
    i = nx;
    k = kn;
    kn = kn2;
  }
}

// ---------------------------------------------------------------------------
// Hash-owner sharding (Memory Layer section 2: the table is sharded across
// devices and the distributed lookup keeps its all-to-all path; MTGR section
// 3.3: ids are exchanged all-to-all, with a dedup before and after).  Key k
// belongs to shard owner(k) = (splitmix64(k) >> 32) mod G.
//
// The partition is a stable counting sort by owner in three launches over
// tiles of kPartTile ids (one id per thread), and a fourth that packs e rows:
//   k_owner_count    per tile and owner, the number of ids (owner-major matrix);
//   k_owner_offsets  one block: exclusive scan of that matrix in owner-major
//                    order (= each tile's first output slot per owner) and the
//                    per-owner totals;
//   k_owner_scatter  each id's slot = its tile's offset for its owner + the ids
//                    of that owner in earlier warps of the tile + earlier lanes
//                    of its warp (__match_any_sync groups a warp by owner);
//   k_owner_pack_rows  with e rows: each slot's e row copied from its source
//                    position into the packed send buffer.
// Order within an owner is batch order, so the owner sees each rank's ids in
// the order the rank had them.
// ---------------------------------------------------------------------------
constexpr int kPartTile = 1024;
constexpr int kMaxOwners = 256;

__device__ __forceinline__ int owner_of(long long k, int G) {
  return (int)((splitmix64((uint64_t)k) >> 32) % (uint64_t)G);
}

__device__ __forceinline__ int64_t part_n(int64_t n, const long long* dev_n) {
  if (!dev_n) return n;
  const long long m = *dev_n;
  return m < 0 ? 0 : (m < n ? m : n);
}

// Per-warp owner counts of this thread's tile in wcnt[warp * G + o]; returns the
// thread's owner (G for an id past the end) and its rank among the earlier lanes
// of its warp with the same owner.
__device__ __forceinline__ int tile_owner_ranks(const long long* __restrict__ ids, int64_t i,
                                                int64_t n_eff, int G, uint16_t* wcnt,
                                                long long& key, int& rank) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int x = threadIdx.x; x < 32 * G; x += blockDim.x) wcnt[x] = 0;
  key = -1;
  int o = G;
  if (i < n_eff) {
    key = ids[i];
    o = owner_of(key, G);
  }
  const unsigned peers = __match_any_sync(0xFFFFFFFFu, o);
  rank = __popc(peers & ((1u << lane) - 1u));
  __syncthreads();
  if (o < G && rank == 0) wcnt[warp * G + o] = (uint16_t)__popc(peers);
  __syncthreads();
  return o;
}

__global__ void __launch_bounds__(kPartTile) k_owner_count(const long long* __restrict__ ids,
                                                          int64_t n, const long long* dev_n,
                                                          int G, int32_t* __restrict__ blk) {
  pdl_enter();
  __shared__ uint16_t wcnt[32 * kMaxOwners];
  const int64_t n_eff = part_n(n, dev_n);
  const int64_t i = (int64_t)blockIdx.x * kPartTile + threadIdx.x;
  long long key;
  int rank;
  tile_owner_ranks(ids, i, n_eff, G, wcnt, key, rank);
  for (int o = threadIdx.x; o < G; o += blockDim.x) {
    int c = 0;
    for (int w = 0; w < 32; ++w) c += wcnt[w * G + o];
    blk[(int64_t)o * gridDim.x + blockIdx.x] = c;
  }
}

// One block.  blk[o * nb + b] (counts) becomes the exclusive prefix in
// owner-major order; counts[o] = the owner's total.
__global__ void __launch_bounds__(1024) k_owner_offsets(int32_t* __restrict__ blk, int nb, int G,
                                                        long long* __restrict__ counts) {
  pdl_enter();
  __shared__ int sm[33];
  __shared__ int carry_s;
  const int64_t L = (int64_t)nb * G;
  if (threadIdx.x == 0) carry_s = 0;
  __syncthreads();
  for (int64_t base = 0; base < L; base += blockDim.x) {
    const int64_t x = base + threadIdx.x;
    const int v = x < L ? blk[x] : 0;
    int total;
    const int before = block_excl_scan(v, sm, total);
    const int carry = carry_s;
    if (x < L) blk[x] = carry + before;
    __syncthreads();
    if (threadIdx.x == 0) carry_s = carry + total;
    __syncthreads();
  }
  const int all = carry_s;
  for (int o = threadIdx.x; o < G; o += blockDim.x) {
    const int lo = blk[(int64_t)o * nb];
    const int hi = o + 1 < G ? blk[(int64_t)(o + 1) * nb] : all;
    counts[o] = hi - lo;
  }
}

__global__ void __launch_bounds__(kPartTile) k_owner_scatter(
    const long long* __restrict__ ids, const int32_t* __restrict__ src_pos, int64_t n,
    const long long* dev_n, int G, const int32_t* __restrict__ off,
    long long* __restrict__ ids_out, int32_t* __restrict__ pos_out) {
  pdl_enter();
  __shared__ uint16_t wcnt[32 * kMaxOwners];
  const int warp = threadIdx.x >> 5;
  const int64_t n_eff = part_n(n, dev_n);
  const int64_t i = (int64_t)blockIdx.x * kPartTile + threadIdx.x;
  long long key;
  int rank;
  const int o = tile_owner_ranks(ids, i, n_eff, G, wcnt, key, rank);
  // exclusive prefix over the warps of the tile, per owner, in place
  for (int q = threadIdx.x; q < G; q += blockDim.x) {
    int run = 0;
    for (int w = 0; w < 32; ++w) {
      const int c = wcnt[w * G + q];
      wcnt[w * G + q] = (uint16_t)run;
      run += c;
    }
  }
  __syncthreads();
  int64_t dst = -1;
  int32_t src = 0;
  if (o < G) {
    dst = (int64_t)off[(int64_t)o * gridDim.x + blockIdx.x] + wcnt[warp * G + o] + rank;
    src = src_pos ? src_pos[i] : (int32_t)i;
    ids_out[dst] = key;
    pos_out[dst] = src;
  }
}

// Packs the e rows of the partitioned ids into the send buffer, e_out[d] =
// e[pos_out[d]] for d < n_eff, one warp per row over a grid of every SM (the
// partition's tiles are too few to keep HBM busy: 96 tiles for 97k distinct
// ids); the next row's source position is loaded while the current row moves.
__global__ void __launch_bounds__(kBlock) k_owner_pack_rows(const int32_t* __restrict__ pos_out,
                                                            int64_t n, const long long* dev_n,
                                                            const float4* __restrict__ e,
                                                            int D4,
                                                            float4* __restrict__ e_out) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int64_t n_eff = part_n(n, dev_n);
  const int64_t warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  int64_t d = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  int32_t sp = d < n_eff ? pos_out[d] : 0;
  while (d < n_eff) {
    const float4* srow = e + (int64_t)sp * D4;
    float4* drow = e_out + d * D4;
    const int64_t nx = d + warps;
    for (int base = 0; base < D4; base += 4 * 32) {
      float4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = base + u * 32 + lane;
        if (c < D4) v[u] = __ldcs(srow + c);
      }
      if (base == 0 && nx < n_eff) sp = pos_out[nx];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = base + u * 32 + lane;
        if (c < D4) __stcs(drow + c, v[u]);
      }
    }
    d = nx;
  }
}

// Combine: the owners' answers come back in send order.  Id j of the send
// buffer came from batch position pos[j]; the answer is its owner's local row
// (-1 = miss) and D gathered values (+0 on a miss).  Writes, at pos[j], the
// global row owner * Cs + row (or -1), hit, and the fused feature row: the
// owner's D values, then the always-on row ao[ao_rows[pos[j]]].
constexpr int kCombineVecMax = 8;  // 16-byte vectors per lane and round (1024 floats per row)

// Indices of send-buffer entry j: its batch position, the owner's answer row
// and the position's always-on row.
__device__ __forceinline__ void combine_indices(const int32_t* __restrict__ pos,
                                                const int32_t* __restrict__ recv_rows,
                                                const int32_t* __restrict__ ao_rows, int A4,
                                                int64_t j, int32_t& p, int32_t& r, int32_t& a) {
  p = pos[j];
  r = recv_rows[j];
  a = A4 > 0 ? ao_rows[p] : 0;
}

// One warp per send-buffer entry, a resident wave grid-striding over them;
// the next entry's indices are loaded while the current row is in flight and
// all loads of a round (kVec vectors per lane: the answer and the always-on
// row together when they fit) are issued before its stores.
template <int kVec>
__global__ void __launch_bounds__(kBlock) k_owner_combine(
    const long long* __restrict__ send_ids, const int32_t* __restrict__ pos, int64_t n, int G,
    int64_t Cs, const int32_t* __restrict__ recv_rows, const float4* __restrict__ recv_feat,
    int D4, const float4* __restrict__ ao, int64_t ao_n, int A4,
    const int32_t* __restrict__ ao_rows, int32_t* __restrict__ rows, uint8_t* __restrict__ hit,
    float4* __restrict__ out, int32_t* status) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int64_t warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int W4 = D4 + A4;
  const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
  int64_t j = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  int32_t p = 0, r = -1, a = 0;
  if (j < n) combine_indices(pos, recv_rows, ao_rows, A4, j, p, r, a);
  while (j < n) {
    bool has_a = A4 > 0;
    if (has_a && (a < 0 || (int64_t)a >= ao_n)) {
      if (lane == 0) set_status(status, kStBadAo);
      has_a = false;
    }
    if (lane == 0) {
      const int o = owner_of(send_ids[j], G);
      rows[p] = r >= 0 ? (int32_t)((int64_t)o * Cs + r) : -1;
      hit[p] = r >= 0;
    }
    const float4* src = recv_feat + j * (int64_t)D4;
    const float4* asrc = ao + (int64_t)(has_a ? a : 0) * A4;
    float4* dst = out + (int64_t)p * W4;
    const int64_t nx = j + warps;
    for (int base = 0; base < W4; base += kVec * 32) {
      float4 v[kVec];
#pragma unroll
      for (int u = 0; u < kVec; ++u) {
        const int c = base + u * 32 + lane;
        v[u] = z;
        if (c < D4)
          v[u] = __ldcs(src + c);
        else if (c < W4 && has_a)
          v[u] = __ldg(asrc + (c - D4));
      }
      if (base == 0 && nx < n) combine_indices(pos, recv_rows, ao_rows, A4, nx, p, r, a);
#pragma unroll
      for (int u = 0; u < kVec; ++u) {
        const int c = base + u * 32 + lane;
        if (c < W4) __stcs(dst + c, v[u]);
      }
    }
    j = nx;
  }
}

}  // namespace mpzch
