// Device code of the hot/cold value tier: an HBM cache of table rows in front
// of values kept in (mapped) host memory.
//
// The Memory Layer page shards its 512-d vector table across GPU and CPU; a
// table whose values exceed HBM keeps them in host memory, and this cache
// keeps the rows the id stream touches most in HBM.  It is direct-mapped and
// write-back: table row r can only live in cache slot slot(r) = r mod H (H a
// power of two), owner[slot] names the row held there (-1 none), and a cached
// row's latest value is in the cache (the host copy may be older).  Which row
// holds a slot changes only inside a Writeback, in three passes over the
// write list:
//   k_tier_claim   every written row claims its slot with the 64-bit word
//                  (step, current owner?, ~row); the largest word wins, so a
//                  slot's current owner keeps it when it is written in this
//                  step, and otherwise the smallest written row takes it (the
//                  step in the high bits makes words of earlier steps lose).
//                  Admission: a row that was not resident before the step (a
//                  freshly inserted id, likelier to be cold) only claims an
//                  empty slot, so it does not push out a row kept from earlier
//                  steps;
//   k_tier_evict   the winner of each slot it does not own yet writes the old
//                  owner's cached value back to the host row and takes the
//                  slot (owner = row, won = step: its value is still on the host);
//   k_tier_update  the row update: e_hat from the cache when the row owned
//                  its slot before this step, else from the host; the result
//                  to the cache when the row owns its slot now, else to the host.
// The values every read sees are therefore exactly those of one plain table,
// whatever the placement.  Gathers and exports read a row from the cache when
// owner[slot] is that row, else from the host.  Counters (kTierStat*) record
// where each row update and gathered row was read and written, and the
// write-backs of evicted rows; each block sums its own in shared memory and
// adds them once.
#pragma once
#include "mpzch_kernels.cuh"

namespace mpzch {

struct Tier {
  float4* cache;         // [H][D4] cached rows
  int32_t* owner;        // [H] table row held in the slot, -1 none
  long long* won;        // [H] step in which the current owner took the slot
  unsigned long long* claim;  // [H] claim words (never cleared)
  unsigned long long* stats;  // [kTierStats] counters
  uint32_t mask;         // H - 1
};

// Counters: row updates whose e_hat came from the cache / the host, whose
// result went to the cache / the host; cached rows written back on eviction;
// gathered rows read from the cache / the host.
constexpr int kTierStatUpdReadCache = 0, kTierStatUpdReadHost = 1, kTierStatUpdWriteCache = 2,
              kTierStatUpdWriteHost = 3, kTierStatWriteBack = 4, kTierStatGatherCache = 5,
              kTierStatGatherHost = 6, kTierStats = 7;

// Block-level counter sums: lane 0 of a warp adds to shared memory; after the
// block's last row every thread passes tier_stats_flush, whose first threads
// add the sums to the global counters.
__device__ __forceinline__ void tier_stats_flush(unsigned* s, unsigned long long* g) {
  __syncthreads();
  if (threadIdx.x < kTierStats && s[threadIdx.x]) atomicAdd(g + threadIdx.x, (unsigned long long)s[threadIdx.x]);
}

__device__ __forceinline__ const float4* tier_row(const Tier& tr, const float4* host, int32_t r,
                                                  int D4) {
  const uint32_t s = (uint32_t)r & tr.mask;
  return __ldcg(tr.owner + s) == r ? tr.cache + (int64_t)s * D4 : host + (int64_t)r * D4;
}

__device__ __forceinline__ unsigned long long tier_claim_word(long long step, bool owner,
                                                              int32_t r) {
  return ((unsigned long long)step << 32) | ((unsigned long long)owner << 31) |
         (unsigned long long)(0x7FFFFFFFu - (uint32_t)r);
}

// Pass 1: claims (one thread per write-list entry; tombstones skipped).
__global__ void __launch_bounds__(kBlock) k_tier_claim(const int32_t* __restrict__ wrow,
                                                       const uint8_t* __restrict__ whit,
                                                       const int32_t* wcount, Tier tr,
                                                       long long step) {
  pdl_enter();
  const int32_t W = *wcount;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; w < W; w += stride) {
    const int32_t r = wrow[w];
    if (r < 0) continue;
    const uint32_t s = (uint32_t)r & tr.mask;
    const int32_t o = tr.owner[s];
    if (o != r && o >= 0 && !whit[w]) continue;  // admission: see the header
    atomicMax(tr.claim + s, tier_claim_word(step, o == r, r));
  }
  pdl_trigger();
}

// Pass 2: each slot's winner that is not its owner yet writes the old owner
// back to the host (one warp per entry, 16-byte vectors) and takes the slot.
__global__ void __launch_bounds__(kBlock) k_tier_evict(const int32_t* __restrict__ wrow,
                                                       const int32_t* wcount, Tier tr,
                                                       float4* __restrict__ host, int D4,
                                                       long long step) {
  pdl_enter();
  __shared__ unsigned s_st[kTierStats];
  if (threadIdx.x < kTierStats) s_st[threadIdx.x] = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int32_t W = *wcount;
  const int64_t warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; w < W; w += warps) {
    const int32_t r = wrow[w];
    if (r < 0) continue;
    const uint32_t s = (uint32_t)r & tr.mask;
    const int32_t o = tr.owner[s];
    if (o == r || __ldcg(tr.claim + s) != tier_claim_word(step, false, r)) continue;
    if (o >= 0) {
      const float4* src = tr.cache + (int64_t)s * D4;
      float4* dst = host + (int64_t)o * D4;
      for (int c = lane; c < D4; c += 32) dst[c] = __ldcg(src + c);
      if (lane == 0) atomicAdd(s_st + kTierStatWriteBack, 1u);
    }
    __syncwarp();
    if (lane == 0) {
      tr.owner[s] = r;
      tr.won[s] = step;
    }
  }
  pdl_trigger();
  tier_stats_flush(s_st, tr.stats);
}

// Pass 3: the row update M[r] <- fl(e_hat - fl(eta * fl(e_hat - e))), e_hat
// and the result in the cache or on the host as the header explains.
__global__ void __launch_bounds__(kBlock) k_tier_update(const int32_t* __restrict__ wrow,
                                                        const int32_t* __restrict__ wpos,
                                                        const int32_t* wcount, Tier tr,
                                                        float4* __restrict__ host,
                                                        const float4* __restrict__ e, int D4,
                                                        float eta, long long step) {
  pdl_enter();
  __shared__ unsigned s_st[kTierStats];
  if (threadIdx.x < kTierStats) s_st[threadIdx.x] = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int32_t W = *wcount;
  const int64_t warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; w < W; w += warps) {
    const int32_t r = wrow[w];
    if (r < 0) continue;
    const uint32_t s = (uint32_t)r & tr.mask;
    const bool owns = tr.owner[s] == r;
    const bool fresh = owns && tr.won[s] == step;  // took the slot in this step: value on the host
    const float4* src = (owns && !fresh) ? tr.cache + (int64_t)s * D4 : host + (int64_t)r * D4;
    float4* dst = owns ? tr.cache + (int64_t)s * D4 : host + (int64_t)r * D4;
    if (lane == 0) {
      atomicAdd(s_st + ((owns && !fresh) ? kTierStatUpdReadCache : kTierStatUpdReadHost), 1u);
      atomicAdd(s_st + (owns ? kTierStatUpdWriteCache : kTierStatUpdWriteHost), 1u);
    }
    const float4* ev = e + (int64_t)wpos[w] * D4;
    for (int base = 0; base < D4; base += 4 * 32) {
      float4 a[4], b[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int c = base + q * 32 + lane;
        if (c < D4) {
          a[q] = __ldcg(src + c);
          b[q] = __ldcs(ev + c);
        }
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int c = base + q * 32 + lane;
        if (c < D4) {
          float4 o;
          o.x = __fsub_rn(a[q].x, __fmul_rn(eta, __fsub_rn(a[q].x, b[q].x)));
          o.y = __fsub_rn(a[q].y, __fmul_rn(eta, __fsub_rn(a[q].y, b[q].y)));
          o.z = __fsub_rn(a[q].z, __fmul_rn(eta, __fsub_rn(a[q].z, b[q].z)));
          o.w = __fsub_rn(a[q].w, __fmul_rn(eta, __fsub_rn(a[q].w, b[q].w)));
          dst[c] = o;
        }
      }
    }
  }
  tier_stats_flush(s_st, tr.stats);
}

// Fused gather over the tier (same result as k_gather_fused on one table).
// A warp's rows are i, i + warps, ...; the next row's indices are loaded
// while the current row is in flight (host reads are long), and every load of
// a round (kVec vectors per lane: the table and always-on parts together when
// they fit) is issued before its stores.
constexpr int kTierGatherVecMax = 8;

template <int kVec>
__global__ void __launch_bounds__(kBlock) k_tier_gather(
    const int32_t* __restrict__ rows, const uint8_t* __restrict__ hit, int64_t n, Tier tr,
    const float4* __restrict__ host, int64_t C, int D4, const float4* __restrict__ ao,
    int64_t ao_n, int A4, const int32_t* __restrict__ ao_rows, float4* __restrict__ out,
    int32_t* status) {
  pdl_enter();
  __shared__ unsigned s_st[kTierStats];
  if (threadIdx.x < kTierStats) s_st[threadIdx.x] = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int W4 = D4 + A4;
  const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
  int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  int32_t r = 0, a = 0;
  uint8_t hb = 0;
  if (i < n) {
    r = rows[i];
    hb = hit[i];
    if (A4 > 0) a = ao_rows[i];
  }
  while (i < n) {
    bool h = hb != 0;
    if (h && (r < 0 || (int64_t)r >= C)) {
      if (lane == 0) set_status(status, kStBadRow);
      h = false;
    }
    bool has_a = A4 > 0;
    if (has_a && (a < 0 || (int64_t)a >= ao_n)) {
      if (lane == 0) set_status(status, kStBadAo);
      has_a = false;
    }
    const float4* src = h ? tier_row(tr, host, r, D4) : host;
    if (h && lane == 0)
      atomicAdd(s_st + (src == host + (int64_t)r * D4 ? kTierStatGatherHost : kTierStatGatherCache), 1u);
    const float4* asrc = ao + (int64_t)(has_a ? a : 0) * A4;
    float4* dst = out + i * (int64_t)W4;
    const int64_t nx = i + warps;
    for (int base = 0; base < W4; base += kVec * 32) {
      float4 v[kVec];
#pragma unroll
      for (int u = 0; u < kVec; ++u) {
        const int c = base + u * 32 + lane;
        v[u] = z;
        if (c < D4) {
          if (h) v[u] = __ldcg(src + c);
        } else if (c < W4 && has_a) {
          v[u] = __ldg(asrc + (c - D4));
        }
      }
      if (base == 0 && nx < n) {
        r = rows[nx];
        hb = hit[nx];
        if (A4 > 0) a = ao_rows[nx];
      }
#pragma unroll
      for (int u = 0; u < kVec; ++u) {
        const int c = base + u * 32 + lane;
        if (c < W4) __stcs(dst + c, v[u]);
      }
    }
    i = nx;
  }
  tier_stats_flush(s_st, tr.stats);
}

// Writes every cached row back to its host row (the cache stays valid).
__global__ void __launch_bounds__(kBlock) k_tier_flush(Tier tr, int64_t H, float4* __restrict__ host,
                                                       int D4) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int64_t warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t s = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; s < H; s += warps) {
    const int32_t o = tr.owner[s];
    if (o < 0) continue;
    const float4* src = tr.cache + s * D4;
    float4* dst = host + (int64_t)o * D4;
    for (int c = lane; c < D4; c += 32) dst[c] = __ldcg(src + c);
  }
}

}  // namespace mpzch
