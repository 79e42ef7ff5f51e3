// Streaming export of freshly written rows to a host serving snapshot
// ("Memory Layer: Train the In-Model Cache for Recommendation Models",
// section 2, RES paragraph: every step the new vectors, already in HBM, are
// copied to the host asynchronously; a background stage dedups by id,
// quantises and merges, and vectors + identity map + metadata are pushed
// atomically every 15 s without blocking training; section 5: serving reads
// int8 rows).
//
// Design:
//  * mpzch_res_stream (caller's thread and stream): selects the rows written
//    at or after `since` and exports them (int8 q, scale, key, last-write step)
//    into a free device staging slot, then copies the row count to pinned host
//    memory and records the slot's event.  Nothing waits on the host.  A row
//    written several times since the previous call is exported once, with its
//    latest value: that is the dedup by id.  With every slot busy the call
//    returns MPZCH_EBUSY instead of blocking training; the next call with an
//    earlier `since` covers the skipped rows.
//  * one background host thread per exporter: waits for a slot's event,
//    copies exactly that many rows to pinned host buffers on its own copy
//    stream, merges them into the working snapshot by row index with a few
//    host threads (a row reassigned to a new key simply carries the new key),
//    frees the slot, and every period publishes what has been merged: the
//    working snapshot is copied into the published one under a lock and the
//    version increases.  Readers copy the
//    published snapshot under the same lock, so they always see one whole
//    version.
#include <cuda_runtime.h>

#include <algorithm>
#include <chrono>
#include <condition_variable>
#include <cstring>
#include <deque>
#include <mutex>
#include <new>
#include <thread>
#include <vector>

#include "mpzch.h"
#include "mpzch_internal.h"

namespace {

double now_ms() {
  return std::chrono::duration<double, std::milli>(
             std::chrono::steady_clock::now().time_since_epoch())
      .count();
}

struct Slot {
  // device staging
  int32_t* rows = nullptr;  // C entries (the selection may list every row)
  int8_t* q = nullptr;
  float* scale = nullptr;
  int64_t* keys = nullptr;
  int64_t* last = nullptr;
  int64_t* count_dev = nullptr;
  // pinned host copies
  int64_t* count_host = nullptr;
  int32_t* h_rows = nullptr;
  int8_t* h_q = nullptr;
  float* h_scale = nullptr;
  int64_t* h_keys = nullptr;
  int64_t* h_last = nullptr;
  cudaEvent_t exported = nullptr;
  bool busy = false;
  int64_t upto_step = -1;
  double t_enqueue = 0;
};

}  // namespace

struct mpzch_res {
  mpzch_table* t = nullptr;
  int64_t C = 0, max_rows = 0;
  int32_t D = 0;
  int device = 0;
  double period_ms = 15000;
  std::vector<Slot> slots;
  cudaStream_t copy_stream = nullptr;
  // snapshots: working (merge target, background thread only) and published
  std::vector<int64_t> w_keys, p_keys, w_last, p_last;
  std::vector<int8_t> w_q, p_q;
  std::vector<float> w_scale, p_scale;
  int64_t w_upto = -1, p_upto = -1, version = 0;
  std::vector<double> unpublished;  // enqueue times of merged, not yet published batches
  std::vector<double> latency_ms;   // enqueue -> publish, one per batch
  int64_t overflow_rows = 0;        // rows beyond max_rows in one call (not exported)
  int error = MPZCH_OK;
  std::mutex mu;
  std::condition_variable cv;
  std::deque<int> pending;
  bool stop = false;
  int64_t flush_requests = 0, flushes_done = 0;
  int merge_threads = 1;
  std::thread th;
};

namespace {

template <typename T>
int halloc(T** p, size_t n) {
  *p = nullptr;
  if (n == 0) return MPZCH_OK;
  if (cudaHostAlloc((void**)p, n * sizeof(T), cudaHostAllocDefault) != cudaSuccess) {
    cudaGetLastError();
    *p = nullptr;
    return MPZCH_ENOMEM;
  }
  return MPZCH_OK;
}

template <typename T>
int dalloc(T** p, size_t n) {
  *p = nullptr;
  if (n == 0) return MPZCH_OK;
  if (cudaMalloc((void**)p, n * sizeof(T)) != cudaSuccess) {
    cudaGetLastError();
    *p = nullptr;
    return MPZCH_ENOMEM;
  }
  return MPZCH_OK;
}

void free_slot(Slot& s) {
  cudaFree(s.rows);
  cudaFree(s.q);
  cudaFree(s.scale);
  cudaFree(s.keys);
  cudaFree(s.last);
  cudaFree(s.count_dev);
  cudaFreeHost(s.count_host);
  cudaFreeHost(s.h_rows);
  cudaFreeHost(s.h_q);
  cudaFreeHost(s.h_scale);
  cudaFreeHost(s.h_keys);
  cudaFreeHost(s.h_last);
  if (s.exported) cudaEventDestroy(s.exported);
  s = Slot();
}

void publish_locked(mpzch_res* r) {
  r->p_keys = r->w_keys;
  r->p_q = r->w_q;
  r->p_scale = r->w_scale;
  r->p_last = r->w_last;
  r->p_upto = r->w_upto;
  ++r->version;
  const double t = now_ms();
  for (double t0 : r->unpublished) r->latency_ms.push_back(t - t0);
  r->unpublished.clear();
}

// Copies one exported slot to the host and merges it into the working snapshot.
int merge_slot(mpzch_res* r, Slot& s) {
  if (cudaEventSynchronize(s.exported) != cudaSuccess) return MPZCH_ECUDA;
  int64_t n = *s.count_host;
  if (n > r->max_rows) {
    r->overflow_rows += n - r->max_rows;
    n = r->max_rows;
  }
  const int64_t D = r->D;
  cudaStream_t cs = r->copy_stream;
  if (n > 0) {
    if (cudaMemcpyAsync(s.h_rows, s.rows, n * sizeof(int32_t), cudaMemcpyDeviceToHost, cs) ||
        cudaMemcpyAsync(s.h_q, s.q, n * D, cudaMemcpyDeviceToHost, cs) ||
        cudaMemcpyAsync(s.h_scale, s.scale, n * sizeof(float), cudaMemcpyDeviceToHost, cs) ||
        cudaMemcpyAsync(s.h_keys, s.keys, n * sizeof(int64_t), cudaMemcpyDeviceToHost, cs) ||
        cudaMemcpyAsync(s.h_last, s.last, n * sizeof(int64_t), cudaMemcpyDeviceToHost, cs) ||
        cudaStreamSynchronize(cs))
      return MPZCH_ECUDA;
  }
  // Merge by row index; the rows of one export are distinct, so host threads
  // can take disjoint ranges of it.
  auto merge_range = [&](int64_t i0, int64_t i1) {
    for (int64_t i = i0; i < i1; ++i) {
      const int64_t row = s.h_rows[i];
      r->w_keys[row] = s.h_keys[i];
      r->w_last[row] = s.h_last[i];
      r->w_scale[row] = s.h_scale[i];
      std::memcpy(&r->w_q[row * D], &s.h_q[i * D], D);
    }
  };
  const int64_t per = 65536;
  const int nt = (int)std::min<int64_t>(r->merge_threads, (n + per - 1) / per);
  if (nt <= 1) {
    merge_range(0, n);
  } else {
    std::vector<std::thread> pool;
    pool.reserve(nt);
    const int64_t chunk = (n + nt - 1) / nt;
    for (int k = 0; k < nt; ++k)
      pool.emplace_back(merge_range, std::min(n, k * chunk), std::min(n, (k + 1) * chunk));
    for (auto& th : pool) th.join();
  }
  return MPZCH_OK;
}

void worker(mpzch_res* r) {
  cudaSetDevice(r->device);
  double next_publish = now_ms() + r->period_ms;
  std::unique_lock<std::mutex> lk(r->mu);
  while (true) {
    // Publish on the period whatever is still queued (what has been merged so
    // far); a flush publishes once everything queued before it is merged.
    if (now_ms() >= next_publish) {
      publish_locked(r);
      next_publish = now_ms() + r->period_ms;
      r->cv.notify_all();
    }
    const bool flush_wanted = r->flush_requests > r->flushes_done;
    if (r->pending.empty()) {
      if (r->stop) break;
      if (flush_wanted) {
        publish_locked(r);
        r->flushes_done = r->flush_requests;
        next_publish = now_ms() + r->period_ms;
        r->cv.notify_all();
        continue;
      }
      const double wait = std::max(1.0, next_publish - now_ms());
      r->cv.wait_for(lk, std::chrono::duration<double, std::milli>(std::min(wait, 50.0)));
      continue;
    }
    const int si = r->pending.front();
    Slot& s = r->slots[si];
    lk.unlock();
    const int rc = merge_slot(r, s);
    lk.lock();
    if (rc && !r->error) r->error = rc;
    r->pending.pop_front();
    r->w_upto = std::max(r->w_upto, s.upto_step);
    r->unpublished.push_back(s.t_enqueue);
    s.busy = false;
    r->cv.notify_all();
  }
}

}  // namespace

extern "C" {

int mpzch_res_create(mpzch_table* t, int64_t max_rows, int32_t slots, int32_t period_ms,
                     mpzch_res** out) {
  if (!out) return MPZCH_EINVAL;
  *out = nullptr;
  if (!t || slots < 1 || slots > 16 || period_ms < 1) return MPZCH_EINVAL;
  const int64_t C = mpzch_internal::table_capacity(t);
  if (max_rows <= 0) max_rows = C;
  if (max_rows > C) return MPZCH_EINVAL;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != mpzch_internal::table_device(t))
    return MPZCH_EINVAL;
  mpzch_res* r = new (std::nothrow) mpzch_res;
  if (!r) return MPZCH_ENOMEM;
  r->t = t;
  r->C = C;
  r->D = mpzch_internal::table_dim(t);
  r->max_rows = max_rows;
  r->device = dev;
  r->period_ms = period_ms;
  int rc = MPZCH_OK;
  try {
    r->w_keys.assign(C, -1);
    r->w_last.assign(C, -1);
    r->w_q.assign((size_t)C * r->D, 0);
    r->w_scale.assign(C, 0.0f);
    r->p_keys = r->w_keys;
    r->p_last = r->w_last;
    r->p_q = r->w_q;
    r->p_scale = r->w_scale;
  } catch (...) {
    rc = MPZCH_ENOMEM;
  }
  r->slots.resize(slots);
  for (auto& s : r->slots) {
    if (rc) break;
    rc = dalloc(&s.rows, C);
    if (!rc) rc = dalloc(&s.q, (size_t)max_rows * r->D);
    if (!rc) rc = dalloc(&s.scale, max_rows);
    if (!rc) rc = dalloc(&s.keys, max_rows);
    if (!rc) rc = dalloc(&s.last, max_rows);
    if (!rc) rc = dalloc(&s.count_dev, 1);
    if (!rc) rc = halloc(&s.count_host, 1);
    if (!rc) rc = halloc(&s.h_rows, max_rows);
    if (!rc) rc = halloc(&s.h_q, (size_t)max_rows * r->D);
    if (!rc) rc = halloc(&s.h_scale, max_rows);
    if (!rc) rc = halloc(&s.h_keys, max_rows);
    if (!rc) rc = halloc(&s.h_last, max_rows);
    if (!rc && cudaEventCreateWithFlags(&s.exported, cudaEventDisableTiming) != cudaSuccess)
      rc = MPZCH_ECUDA;
  }
  if (!rc && cudaStreamCreateWithFlags(&r->copy_stream, cudaStreamNonBlocking) != cudaSuccess)
    rc = MPZCH_ECUDA;
  if (rc) {
    cudaGetLastError();
    for (auto& s : r->slots) free_slot(s);
    if (r->copy_stream) cudaStreamDestroy(r->copy_stream);
    delete r;
    return rc;
  }
  r->merge_threads = (int)std::max(1u, std::min(8u, std::thread::hardware_concurrency() / 2));
  r->th = std::thread(worker, r);
  *out = r;
  return MPZCH_OK;
}

int mpzch_res_stream(mpzch_res* r, int64_t since_step, int64_t upto_step, void* stream) {
  if (!r) return MPZCH_EINVAL;
  int si = -1;
  {
    std::lock_guard<std::mutex> lk(r->mu);
    if (r->error) return r->error;
    for (int i = 0; i < (int)r->slots.size(); ++i)
      if (!r->slots[i].busy) {
        si = i;
        break;
      }
    if (si < 0) return MPZCH_EBUSY;
    r->slots[si].busy = true;
  }
  Slot& s = r->slots[si];
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int rc = mpzch_internal::export_since(r->t, since_step, s.rows, s.count_dev, r->max_rows, s.q,
                                        s.scale, s.keys, s.last, st);
  if (!rc && (cudaMemcpyAsync(s.count_host, s.count_dev, sizeof(int64_t), cudaMemcpyDeviceToHost,
                              st) != cudaSuccess ||
              cudaEventRecord(s.exported, st) != cudaSuccess))
    rc = MPZCH_ECUDA;
  std::lock_guard<std::mutex> lk(r->mu);
  if (rc) {
    s.busy = false;
    return rc;
  }
  s.upto_step = upto_step;
  s.t_enqueue = now_ms();
  r->pending.push_back(si);
  r->cv.notify_all();
  return MPZCH_OK;
}

int mpzch_res_flush(mpzch_res* r, int32_t timeout_ms) {
  if (!r || timeout_ms < 0) return MPZCH_EINVAL;
  std::unique_lock<std::mutex> lk(r->mu);
  const int64_t want = ++r->flush_requests;
  r->cv.notify_all();
  const bool ok = r->cv.wait_for(lk, std::chrono::milliseconds(timeout_ms),
                                 [&] { return r->flushes_done >= want || r->error; });
  if (r->error) return r->error;
  return ok ? MPZCH_OK : MPZCH_ETIMEDOUT;
}

int mpzch_res_read(mpzch_res* r, int64_t* keys, int8_t* q, float* scale, int64_t* last,
                   int64_t* version, int64_t* upto_step) {
  if (!r) return MPZCH_EINVAL;
  std::lock_guard<std::mutex> lk(r->mu);
  if (keys) std::memcpy(keys, r->p_keys.data(), r->C * sizeof(int64_t));
  if (q) std::memcpy(q, r->p_q.data(), (size_t)r->C * r->D);
  if (scale) std::memcpy(scale, r->p_scale.data(), r->C * sizeof(float));
  if (last) std::memcpy(last, r->p_last.data(), r->C * sizeof(int64_t));
  if (version) *version = r->version;
  if (upto_step) *upto_step = r->p_upto;
  return r->error;
}

int mpzch_res_latency(mpzch_res* r, double* p50_ms, double* p99_ms, double* max_ms,
                      int64_t* samples, int64_t* overflow_rows) {
  if (!r) return MPZCH_EINVAL;
  std::lock_guard<std::mutex> lk(r->mu);
  std::vector<double> v = r->latency_ms;
  std::sort(v.begin(), v.end());
  auto at = [&](double f) {
    if (v.empty()) return 0.0;
    size_t i = (size_t)(f * (v.size() - 1) + 0.5);
    return v[std::min(i, v.size() - 1)];
  };
  if (p50_ms) *p50_ms = at(0.50);
  if (p99_ms) *p99_ms = at(0.99);
  if (max_ms) *max_ms = v.empty() ? 0.0 : v.back();
  if (samples) *samples = (int64_t)v.size();
  if (overflow_rows) *overflow_rows = r->overflow_rows;
  return MPZCH_OK;
}

int mpzch_res_destroy(mpzch_res* r) {
  if (!r) return MPZCH_OK;
  {
    std::lock_guard<std::mutex> lk(r->mu);
    r->stop = true;
    r->cv.notify_all();
  }
  if (r->th.joinable()) r->th.join();
  cudaDeviceSynchronize();
  for (auto& s : r->slots) free_slot(s);
  if (r->copy_stream) cudaStreamDestroy(r->copy_stream);
  delete r;
  return MPZCH_OK;
}

}  // extern "C"
