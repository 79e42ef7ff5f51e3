// Internal interface between the table library (mpzch.cu) and the streaming
// exporter (mpzch_res.cu).  Not part of the public ABI.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "mpzch.h"

namespace mpzch_internal {

int64_t table_capacity(const mpzch_table* t);
int32_t table_dim(const mpzch_table* t);
int table_device(const mpzch_table* t);

// On stream `st` (joined with the table's other work): rows with a live key and
// last-write step >= since, ascending, into rows[] with their number in
// *dev_count (device memory); then, for the first min(*dev_count, max_rows) of
// them, the int8 export (q, scale, keys) and the last-write steps.
int export_since(mpzch_table* t, int64_t since, int32_t* rows, int64_t* dev_count, int64_t max_rows,
                 int8_t* q, float* scale, int64_t* keys, int64_t* last, cudaStream_t st);

}  // namespace mpzch_internal
