// CPU oracle for the Memory Layer hot path -- TEST INFRASTRUCTURE ONLY.
//
// Plain single-threaded C++; built with -O2 -ffp-contract=off and without
// fast-math, so every float operation below is one IEEE-754 binary32 operation
// rounded to nearest-even, in the order written.  Only the tests, the smoke
// check and the benchmark's CPU-baseline leg use it.  It shares no code with
// the CUDA library.
//
// Source of each rule ("Memory Layer: Train the In-Model Cache for
// Recommendation Models", abbreviated "Memory Layer" below):
//  * Memory Layer section 2, MPZCH paragraph: M is a sparse key->value table;
//    an identity tensor maps raw item ids collision-free to rows; runtime
//    metadata shares the row index with the vectors; capacity is bounded and
//    eviction is LRU.  The start slot is SplitMix64(key) mod C, the probe
//    window is the P slots h, h+1, ..., h+P-1 (mod C), the empty sentinel is
//    -1, the LRU key is the last step a row was written (ties: lowest row),
//    and missing keys are inserted in ascending key order -- these fixed
//    choices come with the workload definitions, not from the page.
//  * Memory Layer section 2, Writeback paragraph: gradient g = e_hat - e,
//    exact SGD with learning rate 1, M[i] <- e_hat - (e_hat - e); duplicate
//    ids of one batch are deduplicated first so each row gets one exact write.
//    The same paragraph compares it with minimising ||M[i] - sg(e_i)||^2,
//    whose SGD step with rate a is the same update with learning rate 2a;
//    orc_set_learning_rate covers that general step.
//  * Memory Layer section 2, always-on paragraph: on a miss the cached branch
//    is zeroed and the always-on (author id) embedding remains.
//  * Memory Layer section 2, RES paragraph and section 5: streamed rows are
//    deduplicated and quantised; serving uses int8 row quantisation.
#include "mpzch_oracle.h"

#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <new>
#include <unordered_map>
#include <vector>

struct orc_table {
  int64_t C;
  int32_t D;
  int32_t P;
  bool track_all;
  std::vector<int64_t> keys;  // identity map: row -> item key, -1 = empty
  std::vector<int64_t> last;  // metadata sharing the row index: last step written, -1 = never
  std::vector<float> M;       // value rows (track_all)
  std::unordered_map<int32_t, std::vector<float>> tracked;  // value rows (!track_all)
  int64_t last_step;
  float eta;  // learning rate of the SGD step (1: Writeback)
};

extern "C" uint64_t orc_splitmix64(uint64_t x) {
  // SplitMix64 (Steele, Lea, Flood 2014): advance the state by the golden
  // gamma, then two xor-shift-multiply rounds and a final xor-shift.
  uint64_t z = x + 0x9E3779B97F4A7C15ULL;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

extern "C" int64_t orc_home_slot(int64_t key, int64_t capacity) {
  return (int64_t)(orc_splitmix64((uint64_t)key) % (uint64_t)capacity);
}

// Hash-owner sharding (Memory Layer section 2: the table is sharded across
// devices and the distributed lookup keeps its all-to-all path; MTGR section
// 3.3: ids are exchanged all-to-all between devices).  The owning shard takes
// the upper 32 bits of the same SplitMix64 output, so the shard and the home
// slot inside the shard (lower bits, mod C) come from different bits.
extern "C" int32_t orc_owner(int64_t key, int32_t n_owners) {
  return (int32_t)((orc_splitmix64((uint64_t)key) >> 32) % (uint64_t)n_owners);
}

extern "C" int orc_owners(const int64_t* ids, int64_t n, int32_t n_owners, int32_t* out) {
  if (n_owners < 1 || (n > 0 && (!ids || !out))) return ORC_EINVAL;
  for (int64_t i = 0; i < n; ++i) out[i] = orc_owner(ids[i], n_owners);
  return ORC_OK;
}

// The P-slot probe window of a key, in probe order.
static int64_t window_slot(const orc_table* t, int64_t key, int32_t j) {
  return (orc_home_slot(key, t->C) + j) % t->C;
}

// Row holding `key`, or -1.  Every slot of the window is examined.
static int64_t find_row(const orc_table* t, int64_t key) {
  int64_t found = -1;
  for (int32_t j = 0; j < t->P; ++j) {
    int64_t s = window_slot(t, key, j);
    if (t->keys[s] == key && found < 0) found = s;
  }
  return found;
}

static float* row_ptr(orc_table* t, int64_t r) {
  if (t->track_all) return &t->M[(size_t)r * t->D];
  auto it = t->tracked.find((int32_t)r);
  return it == t->tracked.end() ? nullptr : it->second.data();
}
static const float* row_ptr(const orc_table* t, int64_t r) {
  return row_ptr(const_cast<orc_table*>(t), r);
}

extern "C" int orc_create(int64_t capacity, int32_t dim, int32_t probes, int32_t track_all,
                          orc_table** out) {
  if (!out || capacity <= 0 || capacity > 0x7fffffffLL || dim <= 0 || probes <= 0 ||
      probes > capacity)
    return ORC_EINVAL;
  orc_table* t = new (std::nothrow) orc_table;
  if (!t) return ORC_ENOMEM;
  try {
    t->C = capacity;
    t->D = dim;
    t->P = probes;
    t->track_all = track_all != 0;
    t->keys.assign((size_t)capacity, -1);
    t->last.assign((size_t)capacity, -1);
    if (t->track_all) t->M.assign((size_t)capacity * dim, 0.0f);
    t->last_step = -1;
    t->eta = 1.0f;
  } catch (...) {
    delete t;
    return ORC_ENOMEM;
  }
  *out = t;
  return ORC_OK;
}

extern "C" void orc_destroy(orc_table* t) { delete t; }

extern "C" int orc_track_rows(orc_table* t, const int32_t* rows, int64_t n) {
  if (!t || (n > 0 && !rows)) return ORC_EINVAL;
  for (int64_t i = 0; i < n; ++i) {
    if (rows[i] < 0 || rows[i] >= t->C) return ORC_EINVAL;
    if (!t->track_all && !t->tracked.count(rows[i]))
      t->tracked.emplace(rows[i], std::vector<float>((size_t)t->D, 0.0f));
  }
  return ORC_OK;
}

// Lookup: row of each id (or -1) and the hit flag.  Read-only.
extern "C" int orc_lookup(const orc_table* t, const int64_t* ids, int64_t n, int32_t* rows,
                          uint8_t* hit) {
  if (!t || (n > 0 && (!ids || !rows || !hit))) return ORC_EINVAL;
  int rc = ORC_OK;
  for (int64_t i = 0; i < n; ++i) {
    int64_t r = -1;
    if (ids[i] < 0)
      rc = ORC_EBADKEY;
    else
      r = find_row(t, ids[i]);
    rows[i] = (int32_t)r;
    hit[i] = r >= 0 ? 1 : 0;
  }
  return rc;
}

// Fused read: [hit ? M[row] : +0] ++ ao[ao_rows[i]].
extern "C" int orc_gather_fused(const orc_table* t, const int32_t* rows, const uint8_t* hit,
                                int64_t n, const float* ao, int64_t ao_nrows, int32_t ao_dim,
                                const int32_t* ao_rows, float* out) {
  if (!t || (n > 0 && (!rows || !hit || !out))) return ORC_EINVAL;
  const bool has_ao = ao != nullptr && ao_dim > 0;
  if (has_ao && !ao_rows) return ORC_EINVAL;
  const int64_t W = t->D + (has_ao ? ao_dim : 0);
  for (int64_t i = 0; i < n; ++i) {
    float* o = out + i * W;
    if (hit[i]) {
      if (rows[i] < 0 || rows[i] >= t->C) return ORC_EINVAL;
      const float* m = row_ptr(t, rows[i]);
      if (!m) return ORC_EUNTRACKED;
      for (int32_t d = 0; d < t->D; ++d) o[d] = m[d];
    } else {
      for (int32_t d = 0; d < t->D; ++d) o[d] = 0.0f;
    }
    if (has_ao) {
      if (ao_rows[i] < 0 || ao_rows[i] >= ao_nrows) return ORC_EINVAL;
      const float* a = ao + (int64_t)ao_rows[i] * ao_dim;
      for (int32_t d = 0; d < ao_dim; ++d) o[t->D + d] = a[d];
    }
  }
  return ORC_OK;
}

extern "C" int orc_dedup(const int64_t* ids, int64_t n, int64_t* uniq, int64_t* pos,
                         int64_t* n_unique) {
  if ((n > 0 && (!ids || !uniq || !pos)) || !n_unique) return ORC_EINVAL;
  std::unordered_map<int64_t, int64_t> first;
  first.reserve((size_t)n * 2 + 1);
  int64_t u = 0;
  for (int64_t i = 0; i < n; ++i) {
    if (ids[i] < 0) continue;
    if (first.emplace(ids[i], i).second) {
      uniq[u] = ids[i];
      pos[u] = i;
      ++u;
    }
  }
  *n_unique = u;
  return ORC_OK;
}

// One training step's table update.
extern "C" int orc_writeback(orc_table* t, const int64_t* ids, const float* e, int64_t n,
                             int64_t step, orc_wb_stats* stats) {
  if (!t || (n > 0 && (!ids || !e))) return ORC_EINVAL;
  if (step <= t->last_step) return ORC_EINVAL;
  int rc = ORC_OK;
  for (int64_t i = 0; i < n; ++i)
    if (ids[i] < 0) rc = ORC_EBADKEY;

  // 1. In-batch dedup; the first occurrence supplies the target e.
  std::vector<int64_t> uniq((size_t)n), pos((size_t)n);
  int64_t U = 0;
  orc_dedup(ids, n, uniq.data(), pos.data(), &U);
  uniq.resize((size_t)U);
  pos.resize((size_t)U);

  // 2. Resident keys: their rows count as accessed at this step (touched
  //    before any miss is inserted).
  std::vector<int64_t> row_of((size_t)U, -1);
  std::vector<int64_t> missing;  // indices into uniq
  int64_t n_hit = 0;
  for (int64_t u = 0; u < U; ++u) {
    int64_t r = find_row(t, uniq[u]);
    if (r >= 0) {
      row_of[u] = r;
      t->last[r] = step;
      ++n_hit;
    } else {
      missing.push_back(u);
    }
  }

  // 3. Missing keys, one at a time in ascending key order: the victim is the
  //    window row with the smallest (last-access step, row index); an empty
  //    row has last-access -1, so empty rows go first, lowest row first.
  std::sort(missing.begin(), missing.end(),
            [&](int64_t a, int64_t b) { return uniq[a] < uniq[b]; });
  int64_t n_evicted = 0;
  for (int64_t u : missing) {
    int64_t best = -1;
    for (int32_t j = 0; j < t->P; ++j) {
      int64_t s = window_slot(t, uniq[u], j);
      if (best < 0 || t->last[s] < t->last[best] || (t->last[s] == t->last[best] && s < best))
        best = s;
    }
    if (t->keys[best] != -1) ++n_evicted;
    t->keys[best] = uniq[u];
    t->last[best] = step;
    row_of[u] = best;
  }

  // 4. Writeback: every key still owning its row gets the SGD step with
  //    gradient g = e_hat - e and learning rate eta,
  //    M[r] <- e_hat - eta * g   (eta = 1: M[r] <- e_hat - (e_hat - e)),
  //    e_hat = the row's content before this step.  A row is owned by at most
  //    one key, so each row is read and written once and reading it here still
  //    gives its pre-step content.
  int64_t n_dropped = 0;
  for (int64_t u = 0; u < U; ++u) {
    int64_t r = row_of[u];
    if (t->keys[r] != uniq[u]) {
      ++n_dropped;  // evicted again later in this same step
      continue;
    }
    float* m = row_ptr(t, r);
    if (!m) continue;  // value row not tracked (identity map still exact)
    const float* ek = e + pos[u] * t->D;
    for (int32_t d = 0; d < t->D; ++d) {
      float e_hat = m[d];
      float g = e_hat - ek[d];  // Writeback gradient
      float step_d = t->eta * g;  // rounded before the subtraction (no FMA)
      m[d] = e_hat - step_d;      // SGD step
    }
  }
  t->last_step = step;

  if (stats) {
    int64_t valid = 0;
    for (int64_t i = 0; i < n; ++i) valid += ids[i] >= 0;
    stats->n_ids = valid;
    stats->n_unique = U;
    stats->n_hit_unique = n_hit;
    stats->n_inserted = (int64_t)missing.size();
    stats->n_evicted = n_evicted;
    stats->n_dropped = n_dropped;
  }
  return rc;
}

extern "C" int orc_set_learning_rate(orc_table* t, float eta) {
  if (!t || !std::isfinite(eta)) return ORC_EINVAL;
  t->eta = eta;
  return ORC_OK;
}

// Rows (ascending) whose key is live and whose last write is at or after `since`.
extern "C" int orc_select_written_since(const orc_table* t, int64_t since, int32_t* rows_out,
                                        int64_t* count) {
  if (!t || !rows_out || !count) return ORC_EINVAL;
  int64_t c = 0;
  for (int64_t r = 0; r < t->C; ++r)
    if (t->keys[r] != -1 && t->last[r] >= since) rows_out[c++] = (int32_t)r;
  *count = c;
  return ORC_OK;
}

// Per-row int8: a = max|x|, scale = a / 127, q = clamp(round_half_even(x / scale), -127, 127);
// an all-zero row has scale 0 and q 0.
extern "C" int orc_quantize_row(const float* x, int32_t dim, int8_t* q, float* scale) {
  if (!x || !q || !scale || dim <= 0) return ORC_EINVAL;
  float a = 0.0f;
  for (int32_t d = 0; d < dim; ++d) a = std::max(a, std::fabs(x[d]));
  if (a == 0.0f) {
    *scale = 0.0f;
    for (int32_t d = 0; d < dim; ++d) q[d] = 0;
    return ORC_OK;
  }
  const float s = a / 127.0f;
  *scale = s;
  for (int32_t d = 0; d < dim; ++d) {
    float v = std::nearbyint(x[d] / s);  // default rounding mode: nearest, ties to even
    if (v > 127.0f) v = 127.0f;
    if (v < -127.0f) v = -127.0f;
    q[d] = (int8_t)v;
  }
  return ORC_OK;
}

extern "C" int orc_export_int8(const orc_table* t, const int32_t* rows, int64_t n, int8_t* q,
                               float* scale, int64_t* keys) {
  if (!t || (n > 0 && (!rows || !q || !scale || !keys))) return ORC_EINVAL;
  for (int64_t i = 0; i < n; ++i) {
    if (rows[i] < 0 || rows[i] >= t->C) return ORC_EINVAL;
    const float* m = row_ptr(t, rows[i]);
    if (!m) return ORC_EUNTRACKED;
    orc_quantize_row(m, t->D, q + i * t->D, scale + i);
    keys[i] = t->keys[rows[i]];
  }
  return ORC_OK;
}

// Serving read from the int8 snapshot: probe the snapshot's identity map, then
// out = hit ? q * scale : +0.
extern "C" int orc_serve_gather(const int64_t* snap_keys, int64_t capacity, int32_t probes,
                                const int8_t* snap_q, const float* snap_scale, int32_t dim,
                                const int64_t* ids, int64_t n, int32_t* rows, uint8_t* hit,
                                float* out) {
  if (!snap_keys || !snap_q || !snap_scale || capacity <= 0 || probes <= 0 || probes > capacity ||
      dim <= 0 || (n > 0 && (!ids || !rows || !hit || !out)))
    return ORC_EINVAL;
  int rc = ORC_OK;
  for (int64_t i = 0; i < n; ++i) {
    int64_t r = -1;
    if (ids[i] < 0) {
      rc = ORC_EBADKEY;
    } else {
      int64_t h = orc_home_slot(ids[i], capacity);
      for (int32_t j = 0; j < probes; ++j) {
        int64_t s = (h + j) % capacity;
        if (snap_keys[s] == ids[i] && r < 0) r = s;
      }
    }
    rows[i] = (int32_t)r;
    hit[i] = r >= 0;
    float* o = out + i * (int64_t)dim;
    for (int32_t d = 0; d < dim; ++d)
      o[d] = r >= 0 ? (float)snap_q[r * (int64_t)dim + d] * snap_scale[r] : 0.0f;
  }
  return rc;
}

extern "C" int orc_state(orc_table* t, int64_t** keys, int64_t** last, int64_t* last_step) {
  if (!t) return ORC_EINVAL;
  if (keys) *keys = t->keys.data();
  if (last) *last = t->last.data();
  if (last_step) *last_step = t->last_step;
  return ORC_OK;
}

extern "C" int orc_get_row(const orc_table* t, int32_t row, float* out) {
  if (!t || !out || row < 0 || row >= t->C) return ORC_EINVAL;
  const float* m = row_ptr(t, row);
  if (!m) return ORC_EUNTRACKED;
  std::memcpy(out, m, sizeof(float) * t->D);
  return ORC_OK;
}

extern "C" int orc_get_rows(const orc_table* t, const int32_t* rows, int64_t n, float* out) {
  if (!t || (n > 0 && (!rows || !out))) return ORC_EINVAL;
  for (int64_t i = 0; i < n; ++i) {
    int rc = orc_get_row(t, rows[i], out + i * t->D);
    if (rc) return rc;
  }
  return ORC_OK;
}

extern "C" int orc_set_row(orc_table* t, int32_t row, const float* in) {
  if (!t || !in || row < 0 || row >= t->C) return ORC_EINVAL;
  float* m = row_ptr(t, row);
  if (!m) return ORC_EUNTRACKED;
  std::memcpy(m, in, sizeof(float) * t->D);
  return ORC_OK;
}

extern "C" int orc_set_state(orc_table* t, const int64_t* keys, const int64_t* last,
                             int64_t last_step) {
  if (!t || !keys || !last) return ORC_EINVAL;
  std::memcpy(t->keys.data(), keys, sizeof(int64_t) * t->C);
  std::memcpy(t->last.data(), last, sizeof(int64_t) * t->C);
  t->last_step = last_step;
  return ORC_OK;
}
