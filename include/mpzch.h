/*
 * mpzch.h -- C ABI of libmpzch.so, the B200 (sm_100a) hot path of the Memory
 * Layer trainable in-model embedding cache.
 *
 * Source: "Memory Layer: Train the In-Model Cache for Recommendation Models"
 * (cited below as "Memory Layer"), section 2 (method) and section 5
 * (limitations: int8 row quantisation at serving time).  The table M maps an
 * item id to a dense D-dim item-tower vector.  A Multi-Probe Zero-Collision
 * Hashing (MPZCH) identity map sends raw ids to rows without collisions,
 * per-row metadata shares the row index, capacity is bounded and eviction is
 * LRU.  Training reads e_hat = M[i]; Writeback applies g = e_hat - e with an
 * exact SGD step of learning rate 1, i.e. M[i] <- e_hat - (e_hat - e), once
 * per row after in-batch dedup.  On a miss the cached branch is zeroed and the
 * always-on (author id) features remain.
 *
 * Fixed rules of this implementation (the page leaves them open):
 *   start slot   h(k) = splitmix64(k) mod C   (SplitMix64 generator output for state k)
 *   window       W(k) = { (h(k) + j) mod C : j = 0..P-1 }; lookups scan all P slots
 *   empty row    key -1, last-write step -1
 *   victim       the row of W(k) with the smallest (last-write step, row index)
 *   order        resident keys are refreshed first, then missing keys are
 *                inserted one at a time in ascending key order
 *   dedup        the first occurrence of an id in the batch supplies e
 *   export       a = max|x|, scale = a/127 (binary32), q = clamp(rne(x/scale), +-127)
 * Valid item ids are 0 <= k < 2^63.  Negative ids are skipped and raise
 * MPZCH_STATUS_BADKEY in the sticky device status.
 *
 * Conventions for every call:
 *  - Pointers named dev_* or documented as "device" are device pointers on the
 *    device that was current at mpzch_create; they are owned by the caller and
 *    must stay valid until the stream work completes.  The table's own storage
 *    (keys, last-write steps, values, scratch) is owned by the handle.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Every call is asynchronous on it unless stated otherwise.
 *  - The return value is MPZCH_OK or a negative MPZCH_E* code for errors the
 *    host can see (bad arguments, allocation, CUDA launch errors).  Errors the
 *    device sees (bad ids, rows out of range) set bits of a sticky device status
 *    word, read and cleared by mpzch_get_status.  No kernel traps or spins.
 *  - Calls must be issued with the table's device current.  A handle is not
 *    thread-safe: issue its calls from one host thread at a time.  Issue them
 *    on one stream.  (A call on a different stream than the previous call
 *    makes its stream wait for the earlier calls, so results stay correct,
 *    but the two streams are then serialised.)  mpzch_create and a growth of
 *    the per-batch scratch complete before they return.
 */
#ifndef MPZCH_H
#define MPZCH_H
#include <stdint.h>

#if defined(__GNUC__)
#define MPZCH_API __attribute__((visibility("default")))
#else
#define MPZCH_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define MPZCH_OK 0
#define MPZCH_EINVAL (-1)  /* bad argument (null pointer, size, step order, device) */
#define MPZCH_ENOMEM (-2)  /* device allocation failed */
#define MPZCH_ECUDA (-3)   /* a CUDA runtime call or launch failed */
#define MPZCH_ECAPTURE (-5) /* would allocate while the stream is being captured */
#define MPZCH_ERANGE (-6)  /* batch larger than a fixed maximum (mpzch_dedup_static) */
#define MPZCH_EBUSY (-7)   /* every staging slot of a streaming exporter is in use */
#define MPZCH_ETIMEDOUT (-8) /* a wait with a time limit ran out */

/* Sticky device status bits (mpzch_get_status). */
#define MPZCH_STATUS_BADKEY 1   /* a negative item id was given */
#define MPZCH_STATUS_BADROW 2   /* a row index outside [0, C) was given to gather/export */
#define MPZCH_STATUS_BADAO 4    /* an always-on row outside [0, ao_nrows) was given */
#define MPZCH_STATUS_INTERNAL 8 /* an internal bound was hit (never expected) */
#define MPZCH_STATUS_TIMEOUT 16 /* a bulk row copy did not complete within its time limit */

typedef struct mpzch_table mpzch_table;

/* Per-Writeback counters, written to device memory by mpzch_writeback. */
typedef struct {
  int64_t n_ids;        /* valid (non-negative) ids in the batch */
  int64_t n_unique;     /* distinct ids */
  int64_t n_hit_unique; /* distinct ids resident before the step */
  int64_t n_inserted;   /* distinct ids inserted (missing before the step) */
  int64_t n_evicted;    /* inserts that replaced a live key */
  int64_t n_dropped;    /* distinct ids evicted again later in the same step (no write) */
  int64_t n_rounds;     /* insert conflict rounds executed */
} mpzch_wb_stats;

/* Create a table with `capacity` rows (1 <= C <= 2^31-1) of `dim` fp32 values
 * (dim > 0, dim % 4 == 0 so rows are 16-byte vectors) and a `probes`-slot
 * window (1 <= P <= C).  Allocates keys[C] int64 = -1, last[C] int64 = -1,
 * M[C][dim] fp32 = +0 and insert scratch (3*C*8 bytes) on the current device,
 * initialised on `stream`.  Memory layout: keys, last and M are separate
 * row-indexed arrays (the metadata shares the row index with the vectors,
 * Memory Layer section 2).  Returns MPZCH_EINVAL for bad sizes or a null
 * `out`, MPZCH_ENOMEM if an allocation fails (nothing is leaked). */
MPZCH_API int mpzch_create(int64_t capacity, int32_t dim, int32_t probes, void* stream, mpzch_table** out);

/* As mpzch_create, with flags.  MPZCH_VALUES_IN_HOST_MEMORY: the value rows
 * M[C][dim] live in pinned host memory mapped into the device's address space
 * (zero-filled), the identity map, metadata and scratch stay in device memory;
 * every kernel reaches the values over the host link, so tables larger than
 * HBM fit (Memory Layer section 2: the 512-d vector table is sharded across
 * GPU and CPU), at host-link bandwidth.  Other flag bits: MPZCH_EINVAL. */
#define MPZCH_VALUES_IN_HOST_MEMORY 1u
MPZCH_API int mpzch_create_ex(int64_t capacity, int32_t dim, int32_t probes, uint32_t flags,
                              void* stream, mpzch_table** out);

/* Free all device memory of the table (synchronises the device). NULL is a no-op. */
MPZCH_API int mpzch_destroy(mpzch_table* t);

/* Pre-size the per-batch scratch for batches of up to `max_batch` ids so that
 * later calls never allocate (growth otherwise happens on demand inside
 * mpzch_writeback / mpzch_dedup, synchronises the device, and is refused with
 * MPZCH_ECAPTURE while `stream` is being captured). */
MPZCH_API int mpzch_reserve(mpzch_table* t, int64_t max_batch, void* stream);

/* MPZCH lookup (Memory Layer section 2: the identity map sends a raw id to its
 * row).  ids: device int64[n].  rows: device int32[n], the row holding the id
 * or -1.  hit: device uint8[n], 1 iff rows[i] >= 0.  Read-only on the table;
 * never refreshes LRU metadata.  n == 0 is a no-op. */
MPZCH_API int mpzch_lookup(mpzch_table* t, const int64_t* ids, int64_t n, int32_t* rows, uint8_t* hit,
                 void* stream);

/* Fused cached read with the always-on fallback (Memory Layer section 2: the
 * loss uses e_hat = M[i]; on a miss the cached branch is zeroed and the
 * always-on author embedding remains).  For i < n:
 *   out[i][0:dim]          = hit[i] ? M[rows[i]][:] : +0.0
 *   out[i][dim:dim+ao_dim] = ao_table[ao_rows[i]][:]
 * rows/hit: device, as produced by mpzch_lookup.  ao_table: device fp32
 * [ao_nrows][ao_dim] (ao_dim % 4 == 0), ao_rows: device int32[n]; pass
 * ao_table = NULL, ao_nrows = 0, ao_dim = 0, ao_rows = NULL for no concat.
 * out: device fp32 [n][dim + ao_dim], 16-byte aligned.  Out-of-range rows set
 * MPZCH_STATUS_BADROW / BADAO and produce zeros. */
MPZCH_API int mpzch_gather_fused(mpzch_table* t, const int32_t* rows, const uint8_t* hit, int64_t n,
                       const float* ao_table, int64_t ao_nrows, int32_t ao_dim,
                       const int32_t* ao_rows, float* out, void* stream);

/* In-batch dedup (Memory Layer section 2, Writeback paragraph: duplicate ids
 * of a batch are removed first so each row gets one exact write).  ids: device
 * int64[n].  uniq: device int64[n] and pos: device int32[n] receive the
 * distinct ids and the index of their first occurrence, in first-occurrence
 * order; dev_count: device int64, receives the number of distinct ids.
 * Negative ids are skipped (MPZCH_STATUS_BADKEY).  Uses the table's scratch. */
MPZCH_API int mpzch_dedup(mpzch_table* t, const int64_t* ids, int64_t n, int64_t* uniq, int32_t* pos,
                int64_t* dev_count, void* stream);

/* Dedup that allocates no device memory.  The pages have no counterpart to
 * this call; it is a variant of mpzch_dedup for callers that cannot call
 * cudaMalloc -- for example a plug-in running inside an inference server or
 * another framework that owns all device memory through its own pool (a raw
 * cudaMalloc there can fail once the pool has reserved the device, and it
 * bypasses the host's memory accounting), or a latency-critical path where a
 * cudaMalloc/cudaFree would synchronise the device.  Such a caller cannot
 * create a table handle either, so this call needs none.
 *
 * Output and argument meaning are those of mpzch_dedup: ids device int64[n];
 * uniq device int64[n] and pos device int32[n] receive the distinct ids and
 * the index of their first occurrence, in first-occurrence order; dev_count
 * (device int64) receives their number.  dev_status: nullable device int32,
 * OR-ed with MPZCH_STATUS_BADKEY when a negative id is skipped.
 *
 * Scratch: one fixed static device array of this library, about 7 MiB, which
 * every GPU that loads the library holds until the process exits.  n must be
 * at most MPZCH_DEDUP_STATIC_MAX_IDS; larger n returns MPZCH_ERANGE and
 * launches nothing.  The first call on a device looks up the array's device
 * address (cudaGetSymbolAddress) with that device current; make that first
 * call before any stream capture.  The address is kept for the life of the
 * process: after a cudaDeviceReset of that device (or any other teardown of
 * its primary context) do not call this function again in the same process.  Every call uses the same array and each
 * call clears the part of it that must start empty, so the contents left by
 * the previous call do not matter -- but calls that can overlap on the GPU
 * (different streams, or several host threads) race with each other and give
 * wrong results: order them on one stream. */
#define MPZCH_DEDUP_STATIC_MAX_IDS 262144
MPZCH_API int mpzch_dedup_static(const int64_t* ids, int64_t n, int64_t* uniq, int32_t* pos,
                                 int64_t* dev_count, int32_t* dev_status, void* stream);

/* One training step of the table (Memory Layer section 2, MPZCH and Writeback
 * paragraphs).  ids: device int64[n]; e: device fp32 [n][dim], the item-tower
 * targets, row i belonging to ids[i].  step must exceed every earlier step of
 * this table (host-checked; MPZCH_EINVAL otherwise).  In order:
 *   1. dedup (first occurrence supplies e);
 *   2. resident ids: last[row] = step;
 *   3. missing ids, ascending: victim = argmin over W(k) of (last, row);
 *      keys[victim] = k, last[victim] = step;
 *   4. every id still owning its row r: M[r] <- fl(e_hat - fl(e_hat - e)),
 *      e_hat = the row's content before this step.
 * dev_stats: nullable device mpzch_wb_stats, written before the call's work
 * completes on `stream`.  Call order within a step: lookup -> gather_fused ->
 * writeback (a gather issued after writeback sees the new values). */
MPZCH_API int mpzch_writeback(mpzch_table* t, const int64_t* ids, const float* e, int64_t n, int64_t step,
                    mpzch_wb_stats* dev_stats, void* stream);

/* One multi-table training step in one call (Memory Layer section 2,
 * Multi-Table paragraph: a labeled batch and an unlabeled candidate-pool batch
 * are merged, the item tower runs once, one Writeback covers both, and the
 * loss reads only the labeled part).  ids: device int64[n], the merged batch
 * with its n_labeled labeled ids first (0 <= n_labeled <= n); e: device fp32
 * [n][dim].  The call gives, bit for bit, the outputs of
 *   mpzch_lookup(ids, n_labeled, rows, hit);
 *   mpzch_gather_fused(rows, hit, n_labeled, ao_table, ao_nrows, ao_dim, ao_rows, out);
 *   mpzch_writeback(ids, e, n, step, dev_stats);
 * rows/hit/out/ao_* as in those calls (may be NULL when n_labeled == 0).
 *
 * Inside, the row map (dedup, refresh, inserts) runs on a second stream of
 * the table (MPZCH_OPT_SIDE_PRIORITY).  Its re-probe of the distinct ids also
 * gives the lookup: rows/hit of the labeled positions are the rows their ids
 * held before this step's inserts, filled in by the first placement pass.
 * The gather and the row update run on `stream`, the gather once the lookup
 * fill is done and the row update once the row map is done.  Later work on
 * `stream` is ordered after all of it (rows, hit, out, stats and the table are
 * complete there).
 *
 * inputs_ready: NULL, or a cudaEvent_t (as void*) recorded after ids, e and
 * ao_rows of this step were written.  With NULL the step starts after all
 * earlier work on `stream`.  With an event the step's row map starts as soon
 * as that event, the previous step's gather and the table's earlier calls
 * allow -- so it overlaps the previous step's row update (pipelined steps,
 * identical results).  Then the caller must also order before inputs_ready
 * every read of the previous step's rows, hit and stats buffers that are
 * reused for this step, and every write it made to the table's state itself
 * (a restore through mpzch_state_views). */
MPZCH_API int mpzch_train_step(mpzch_table* t, const int64_t* ids, int64_t n, int64_t n_labeled,
                               const float* e, int64_t step, const float* ao_table,
                               int64_t ao_nrows, int32_t ao_dim, const int32_t* ao_rows,
                               int32_t* rows, uint8_t* hit, float* out,
                               mpzch_wb_stats* dev_stats, void* inputs_ready, void* stream);

/* Rows written recently (Memory Layer section 2, RES paragraph: fresh rows are
 * streamed to the predictors): rows_out (device int32[C]) receives, in
 * ascending order, every row r with keys[r] != -1 and last[r] >= since_step;
 * dev_count (device int64) receives their number. */
MPZCH_API int mpzch_select_written_since(mpzch_table* t, int64_t since_step, int32_t* rows_out,
                               int64_t* dev_count, void* stream);

/* Per-row int8 export of the serving snapshot (Memory Layer section 2, RES:
 * rows are quantised before the push; section 5: serving uses int8 row
 * quantisation).  For i < min(n, *dev_n): with x = M[rows[i]],
 *   a = max|x|, scale[i] = a / 127 (binary32), q[i][d] = clamp(rne(x[d]/scale[i]), -127, 127),
 *   a == 0 gives scale 0 and q 0;  keys_out[i] = keys[rows[i]].
 * rows: device int32[n]; q: device int8[n][dim]; scale: device fp32[n];
 * keys_out: device int64[n]; dev_n: nullable device int64 count (e.g. the
 * dev_count of mpzch_select_written_since), NULL = n. */
MPZCH_API int mpzch_export_int8(mpzch_table* t, const int32_t* rows, int64_t n, const int64_t* dev_n,
                      int8_t* q, float* scale, int64_t* keys_out, void* stream);

/* Serving read from an int8 snapshot (Memory Layer section 2, RES: predictors
 * receive vectors + identity map; section 5: int8 rows).  The snapshot is a
 * table image: snap_keys device int64[capacity] (-1 = empty), snap_q device
 * int8[capacity][dim], snap_scale device fp32[capacity].  For each ids[i]
 * (device int64[n]): rows[i] = the snapshot row holding it or -1 (all `probes`
 * window slots scanned), hit[i] = rows[i] >= 0, and
 *   out[i][:] = hit ? fl((float)q * scale) : +0.0      (out: device fp32 [n][dim]).
 * dev_status: nullable device int32, OR-ed with MPZCH_STATUS_BADKEY for
 * negative ids.  Needs no table handle and allocates nothing. */
MPZCH_API int mpzch_serve_gather(const int64_t* snap_keys, int64_t capacity, int32_t probes,
                       const int8_t* snap_q, const float* snap_scale, int32_t dim,
                       const int64_t* ids, int64_t n, int32_t* rows, uint8_t* hit, float* out,
                       int32_t* dev_status, void* stream);

/* ---- Hash-owner sharding --------------------------------------------------
 * Memory Layer section 2 shards the table across devices and keeps the
 * distributed lookup's all-to-all path; MTGR (page "MTGR: Industrial-Scale
 * Generative Recommendation Framework in Meituan") section 3.3 exchanges ids
 * all-to-all between devices with a dedup before and after the exchange.
 * With G shards (one table per rank), key k belongs to shard
 *   owner(k) = (splitmix64(k) >> 32) mod G,
 * the upper half of the hash whose lower bits pick the home slot inside the
 * shard.  A rank partitions its ids (and e rows) by owner into one contiguous
 * segment per owner, exchanges the segments all-to-all (NCCL; the owner
 * receives ranks 0..G-1 in rank order), runs lookup/gather/Writeback on its
 * own table, and sends lookup answers back in the order received; the combine
 * step puts them at their batch positions.  Global row of shard s, local row
 * r: s * shard_capacity + r.  At most MPZCH_MAX_OWNERS shards. */
#define MPZCH_MAX_OWNERS 256

/* Bytes of device workspace mpzch_owner_partition needs for n ids and
 * n_owners owners (a multiple of 256), or -1 for bad sizes. */
MPZCH_API int64_t mpzch_owner_partition_workspace(int64_t n, int32_t n_owners);

/* Stable partition of ids by owner.  For i < n_eff (n_eff = n, or
 * min(n, *dev_n) when dev_n is given -- e.g. the dev_count of mpzch_dedup):
 * ids[i] goes to the segment of owner(ids[i]); segments are laid out in
 * ascending owner order and keep batch order inside, in ids_out (device
 * int64[n]).  pos_out[j] (device int32[n]) = src_pos ? src_pos[i] : i for the
 * id placed at j.  With e (device fp32 [..][dim], dim % 4 == 0, 16-byte
 * aligned) non-NULL, e_out row j (device fp32 [n][dim], 16-byte aligned) =
 * e row pos_out[j]: the packed send buffer of the ids' e rows.  dev_counts:
 * device int64[n_owners], the segment sizes (they sum to n_eff).  Slots past
 * n_eff are not written.  workspace: device memory of at least
 * mpzch_owner_partition_workspace(n, n_owners) bytes, owned by the caller,
 * not used after the call's work completes on `stream`.  Allocates nothing.
 * MPZCH_EINVAL for bad sizes, null pointers or misaligned rows. */
MPZCH_API int mpzch_owner_partition(const int64_t* ids, const int32_t* src_pos, int64_t n,
                                    const int64_t* dev_n, int32_t n_owners, const float* e,
                                    int32_t dim, int64_t* ids_out, int32_t* pos_out, float* e_out,
                                    int64_t* dev_counts, void* workspace,
                                    int64_t workspace_bytes, void* stream);

/* Combine the owners' lookup answers (they arrive in send order).  For j < n:
 * send_ids/pos are the ids_out/pos_out of the partition of the looked-up ids
 * (batch positions pos[j] < the caller's batch size), recv_rows (device
 * int32[n]) the owner's local row or -1, recv_feat (device fp32 [n][dim],
 * 16-byte aligned) the owner's gathered values (+0 on a miss).  Writes at
 * p = pos[j]:
 *   rows[p] = recv_rows[j] >= 0 ? owner(send_ids[j]) * shard_capacity + recv_rows[j] : -1,
 *   hit[p]  = recv_rows[j] >= 0,
 *   out[p][0:dim] = recv_feat[j],  out[p][dim:dim+ao_dim] = ao_table[ao_rows[p]]
 * -- bit for bit what mpzch_gather_fused gives on one table.  ao_* as in
 * mpzch_gather_fused (NULL/0 for no concat).  out: device fp32 [..][dim +
 * ao_dim], 16-byte aligned.  An always-on row outside [0, ao_nrows) gives
 * zeros and ORs MPZCH_STATUS_BADAO into dev_status (nullable device int32).
 * n_owners * shard_capacity must be below 2^31.  Needs no table handle. */
MPZCH_API int mpzch_owner_combine(const int64_t* send_ids, const int32_t* pos, int64_t n,
                                  int32_t n_owners, int64_t shard_capacity,
                                  const int32_t* recv_rows, const float* recv_feat, int32_t dim,
                                  const float* ao_table, int64_t ao_nrows, int32_t ao_dim,
                                  const int32_t* ao_rows, int32_t* rows, uint8_t* hit, float* out,
                                  int32_t* dev_status, void* stream);

/* ---- Streaming export of fresh rows to a host serving snapshot (RES) ----
 * Memory Layer section 2, RES paragraph: new vectors are copied to the host
 * asynchronously while they are in HBM; in the background they are deduped by
 * id, quantised and merged, and vectors + identity map + metadata are pushed
 * atomically every 15 s without blocking training.  Section 5: serving reads
 * int8 rows.  The host snapshot is a table image: keys[C] (-1 = empty), int8
 * q[C][dim], scale[C], last-write step last[C], at the table's row indices. */
typedef struct mpzch_res mpzch_res;

/* Exporter for table t (current device = the table's): `slots` device staging
 * slots of max_rows rows (max_rows <= 0: the capacity), a background host
 * thread, and a publish period in milliseconds.  Destroy it before the table. */
MPZCH_API int mpzch_res_create(mpzch_table* t, int64_t max_rows, int32_t slots, int32_t period_ms,
                               mpzch_res** out);

/* On `stream` (ordered like any table call): selects every row with a live key
 * written at or after since_step and exports it (int8 q, scale, key,
 * last-write step) into a free staging slot; the background thread copies it
 * to the host and merges it into the snapshot by row index (a row written
 * several times since the previous call is exported once, with its latest
 * value; a row reassigned to a new key carries the new key).  upto_step labels
 * the data (normally the last step written before the call).  Never waits on
 * the host: returns MPZCH_EBUSY if every slot is still being copied (a later
 * call with an earlier since_step covers the rows).  Rows beyond max_rows in
 * one call are not exported and are counted (mpzch_res_latency). */
MPZCH_API int mpzch_res_stream(mpzch_res* r, int64_t since_step, int64_t upto_step, void* stream);

/* Waits (at most timeout_ms) until every streamed slot is merged and a
 * snapshot containing them is published.  MPZCH_ETIMEDOUT otherwise. */
MPZCH_API int mpzch_res_flush(mpzch_res* r, int32_t timeout_ms);

/* Copies the latest published snapshot (host buffers of C entries each; any may
 * be NULL), its version (number of publishes) and the largest upto_step it
 * contains.  The copy is taken under the publish lock: one whole version. */
MPZCH_API int mpzch_res_read(mpzch_res* r, int64_t* keys, int8_t* q, float* scale, int64_t* last,
                             int64_t* version, int64_t* upto_step);

/* Propagation latency from mpzch_res_stream to the publish that contains its
 * rows: median, 99th percentile and maximum in ms over `samples` streamed
 * batches, and the number of rows dropped for exceeding max_rows. */
MPZCH_API int mpzch_res_latency(mpzch_res* r, double* p50_ms, double* p99_ms, double* max_ms,
                                int64_t* samples, int64_t* overflow_rows);

/* Stops the background thread after it has merged what is pending, frees all. */
MPZCH_API int mpzch_res_destroy(mpzch_res* r);

/* Device pointers to the table's state (for checkpoint/resume and tests):
 * keys int64[C], last int64[C], M fp32[C][dim].  Any argument may be NULL. */
MPZCH_API int mpzch_state_views(mpzch_table* t, int64_t** keys, int64_t** last, float** M);

/* Host-side last step (the step order check).  After restoring a saved state
 * through mpzch_state_views, set it to the saved table's last step. */
MPZCH_API int mpzch_get_last_step(mpzch_table* t, int64_t* step);
MPZCH_API int mpzch_set_last_step(mpzch_table* t, int64_t step);

/* Reads and clears the sticky device status word (MPZCH_STATUS_* bits).
 * Synchronises `stream`. */
MPZCH_API int mpzch_get_status(mpzch_table* t, int32_t* status, void* stream);

/* Per-phase timing with CUDA events recorded around each phase's launches on
 * the launching stream.  Phases (index): 0 lookup, 1 gather, 2 dedup (inside
 * mpzch_writeback: dedup, re-probe and refresh; also mpzch_dedup), 3 insert
 * (conflict rounds), 4 writeback (the row update kernel alone), 5 select,
 * 6 export.  mpzch_trace_read synchronises the events recorded since the last
 * read and returns, per phase, the summed device milliseconds and the number
 * of kernel launches. */
#define MPZCH_NPHASES 7
MPZCH_API int mpzch_trace_enable(mpzch_table* t, int32_t on);
MPZCH_API int mpzch_trace_read(mpzch_table* t, double* ms, int64_t* launches, int32_t nphases);

/* Options.  Results never depend on them.
 * MPZCH_OPT_CLUSTER_INSERT: how the missing ids of a Writeback are inserted.
 * 1 (default) = cluster placement: ids whose windows chain together (home
 * slots less than P apart) form a cluster, each cluster is placed by one
 * thread in ascending key order, clusters in parallel (when the windows may
 * cover the whole ring -- missing ids x P >= C -- one block places them all).
 * 0 = claim rounds: MPZCH_OPT_WIDE_ROUNDS grid-wide rounds in which every
 * unplaced id claims its window, then one block places the rest.
 * MPZCH_OPT_WIDE_ROUNDS: the number of those rounds (default 3, range
 * 0..64). */
#define MPZCH_OPT_WIDE_ROUNDS 1
#define MPZCH_OPT_CLUSTER_INSERT 4
/* MPZCH_OPT_SIDE_PRIORITY: 1 (default) = the side stream of mpzch_train_step
 * gets the device's highest stream priority, 0 = the lowest; only before the
 * first mpzch_train_step of the table (MPZCH_EINVAL afterwards). */
#define MPZCH_OPT_SIDE_PRIORITY 2
/* MPZCH_OPT_ROW_GRID: grid of the row kernels (fused gather, row update):
 * 0 = one row per warp, short-lived blocks; k > 0 = at most k blocks of 256
 * threads per SM, each striding over many rows (default 8; the fused gather
 * takes at most the blocks that fit on an SM at once). */
#define MPZCH_OPT_ROW_GRID 3
/* MPZCH_OPT_ROW_KERNEL: how the row kernels (fused gather, row update) move
 * rows.  0 (default) = through registers: every lane loads its 16-byte
 * vectors of a row, then stores them.  1 = through shared memory: one lane
 * per warp issues 1-D bulk copies (cp.async.bulk, completed on an mbarrier)
 * of the next rows into the warp's stages while the lanes finish the current
 * one; persistent grid of MPZCH_OPT_BULK_BLOCKS blocks per SM with
 * MPZCH_OPT_BULK_WARPS warps each (halved until the block's shared memory
 * fits 112 KiB; the register path runs for rows too large for one warp's
 * stages, and for values in host memory).  A row copy that has not completed
 * after one second sets MPZCH_STATUS_TIMEOUT and the kernel returns.
 * MPZCH_OPT_L2_HINT_ROWS: L2 eviction priority of the bulk kernels' table-row
 * loads and stores: 0 (default) evict-first, 1 normal, 2 evict-last. */
#define MPZCH_OPT_ROW_KERNEL 5
#define MPZCH_OPT_BULK_WARPS 6
#define MPZCH_OPT_BULK_BLOCKS 7
#define MPZCH_OPT_L2_HINT_ROWS 8
/* MPZCH_OPT_WRITE_LIST (cluster placement path): 1 (default) = the list of
 * rows the Writeback writes is built as ownership is decided -- the re-probe
 * adds every resident id, each placement the id it places, and a placement
 * that evicts an id written earlier in the same step cancels that id's entry;
 * 0 = one more kernel builds the list after all placements. */
#define MPZCH_OPT_WRITE_LIST 9
/* MPZCH_OPT_HBM_CACHE_ROWS (tables with MPZCH_VALUES_IN_HOST_MEMORY only):
 * keep an HBM cache of this many rows (a power of two <= capacity; 0 = none,
 * the default) in front of the host-memory values -- the hot/cold tier (Memory
 * Layer section 2: the 512-d table is sharded across GPU and CPU).  Row r can
 * live in cache slot r mod H; the cache is write-back.  In each Writeback a
 * written row keeps its slot; a slot whose owner was not written goes to the
 * smallest written row that was resident before the step (a freshly inserted
 * id only takes an empty slot), and the old owner's value is written back to
 * the host first; reads take a row from the cache when it holds it.  Every value read
 * or written is exactly that of a table without the cache.  Changing the size
 * writes every cached row back and synchronises the device.  Values read
 * through mpzch_state_views are the host rows: call mpzch_tier_sync first.
 * Steps of a tiered table must stay below 2^31. */
#define MPZCH_OPT_HBM_CACHE_ROWS 10
MPZCH_API int mpzch_set_option(mpzch_table* t, int32_t option, int64_t value);
/* Current value of an option (MPZCH_EINVAL for an unknown option). */
MPZCH_API int mpzch_get_option(mpzch_table* t, int32_t option, int64_t* value);

/* Hot/cold tier (MPZCH_OPT_HBM_CACHE_ROWS), on `stream`: discard = 0 writes
 * every cached row back to its host row (the cache stays valid; do this
 * before reading values through mpzch_state_views); discard = 1 empties the
 * cache without writing back (after the caller replaced the host values, e.g.
 * a restore).  A table without a cache: no-op.  The int8 export writes the
 * cache back by itself. */
MPZCH_API int mpzch_tier_sync(mpzch_table* t, int32_t discard, void* stream);

/* Hot/cold tier counters since the cache was created or last reset, read
 * after the work on `stream` (and the table's side stream) has completed
 * (the call synchronises `stream`).  counts: host int64[7] =
 *   [0] row updates whose e_hat was read from the cache, [1] from the host,
 *   [2] row updates whose result was written to the cache, [3] to the host,
 *   [4] cached rows written back to the host when another row took their slot,
 *   [5] gathered rows read from the cache, [6] from the host.
 * reset = 1 zeroes the counters after reading them.  A table without a cache
 * gives zeros. */
MPZCH_API int mpzch_tier_stats(mpzch_table* t, int64_t* counts, int32_t reset, void* stream);

/* Learning rate of the Writeback step for the following calls (Memory Layer
 * section 2, Writeback paragraph: the exact step is SGD at rate 1 on
 * g = e_hat - e; the alternative it is compared with, minimising
 * ||M[i] - sg(e_i)||^2, is the same SGD step at rate 2a for loss rate a; an
 * EMA cache c <- alpha c + (1 - alpha) v is the step at 1 - alpha).  Every
 * written row becomes M[r] <- fl(e_hat - fl(eta * fl(e_hat - e))); eta = 1
 * (the default) is the exact Writeback M[r] <- e_hat - (e_hat - e).  eta must
 * be finite (MPZCH_EINVAL otherwise).  Host-side only; affects later calls. */
MPZCH_API int mpzch_set_learning_rate(mpzch_table* t, float eta);

/* Test hook: the next `count` device allocations made by this library fail as
 * if the device were out of memory (no CUDA call is made for them). */
MPZCH_API int mpzch_debug_fail_allocs(int32_t count);

/* Number of kernel launches this library issued in the calling process. */
MPZCH_API int64_t mpzch_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* MPZCH_H */
