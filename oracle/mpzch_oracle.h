/*
 * CPU oracle for the Memory Layer hot path -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, single-threaded restatement of what the Memory Layer table
 * computes ("Memory Layer: Train the In-Model Cache for Recommendation
 * Models", section 2: the MPZCH identity map with bounded capacity and LRU
 * eviction, the cached read e_hat = M[i], the Writeback update
 * M[i] <- e_hat - (e_hat - e) once per row after in-batch dedup, the
 * always-on fallback that zeroes the cached branch on a miss; section 5:
 * int8 row quantisation of the serving snapshot).
 *
 * Only the tests, the smoke check and the benchmark's CPU-baseline leg load
 * this library.  It shares no source, header or helper with the CUDA library;
 * the product path never calls it.
 *
 * Every function returns 0 on success or a negative ORC_E* code.
 */
#ifndef MPZCH_ORACLE_H
#define MPZCH_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ORC_OK 0
#define ORC_EINVAL (-1)
#define ORC_ENOMEM (-2)
#define ORC_EBADKEY (-4)
#define ORC_EUNTRACKED (-5)

typedef struct orc_table orc_table;

typedef struct {
  int64_t n_ids, n_unique, n_hit_unique, n_inserted, n_evicted, n_dropped;
} orc_wb_stats;

/* SplitMix64 generator output for state x (Steele, Lea, Flood, OOPSLA 2014). */
uint64_t orc_splitmix64(uint64_t x);
/* Start slot h(k) = splitmix64(k) mod C. */
int64_t orc_home_slot(int64_t key, int64_t capacity);

/* Owning shard of a key among n_owners shards: (splitmix64(k) >> 32) mod n_owners. */
int32_t orc_owner(int64_t key, int32_t n_owners);
/* out[i] = orc_owner(ids[i], n_owners) for i < n. */
int orc_owners(const int64_t* ids, int64_t n, int32_t n_owners, int32_t* out);

/* track_all != 0: keep every value row (C*D floats of host memory).
 * track_all == 0: keep only rows later registered with orc_track_rows; the
 * identity map (keys, last-access) is always kept in full. */
int orc_create(int64_t capacity, int32_t dim, int32_t probes, int32_t track_all, orc_table** out);
void orc_destroy(orc_table* t);
int orc_track_rows(orc_table* t, const int32_t* rows, int64_t n);

int orc_lookup(const orc_table* t, const int64_t* ids, int64_t n, int32_t* rows, uint8_t* hit);
int orc_gather_fused(const orc_table* t, const int32_t* rows, const uint8_t* hit, int64_t n,
                     const float* ao, int64_t ao_nrows, int32_t ao_dim, const int32_t* ao_rows,
                     float* out);
/* First occurrence dedup: uniq/pos in first-occurrence order, *n_unique set. */
int orc_dedup(const int64_t* ids, int64_t n, int64_t* uniq, int64_t* pos, int64_t* n_unique);
int orc_writeback(orc_table* t, const int64_t* ids, const float* e, int64_t n, int64_t step,
                  orc_wb_stats* stats);
/* Learning rate eta of the Writeback step M <- e_hat - eta * (e_hat - e)
 * (default 1: the exact assignment). */
int orc_set_learning_rate(orc_table* t, float eta);
int orc_select_written_since(const orc_table* t, int64_t since, int32_t* rows_out, int64_t* count);
int orc_quantize_row(const float* x, int32_t dim, int8_t* q, float* scale);
int orc_export_int8(const orc_table* t, const int32_t* rows, int64_t n, int8_t* q, float* scale,
                    int64_t* keys);
int orc_serve_gather(const int64_t* snap_keys, int64_t capacity, int32_t probes,
                     const int8_t* snap_q, const float* snap_scale, int32_t dim,
                     const int64_t* ids, int64_t n, int32_t* rows, uint8_t* hit, float* out);

/* State access for comparisons (host pointers owned by the table). */
int orc_state(orc_table* t, int64_t** keys, int64_t** last, int64_t* last_step);
int orc_get_row(const orc_table* t, int32_t row, float* out);
/* Copies rows[0..n) of M into out[n][D] (every listed row must be kept). */
int orc_get_rows(const orc_table* t, const int32_t* rows, int64_t n, float* out);
int orc_set_row(orc_table* t, int32_t row, const float* in);
int orc_set_state(orc_table* t, const int64_t* keys, const int64_t* last, int64_t last_step);

#ifdef __cplusplus
}
#endif
#endif
