// internal.h -- private declarations shared by the library's translation units.
#pragma once
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/dsq.h"
#include "layout.h"

namespace dsq {

double half_bits_to_double(uint16_t h);
int check_desc(const dsq_desc *d);
void plan_blob(const dsq_desc *d, BlobHeader *h);
int parse_blob(const void *packed, size_t bytes, BlobHeader *out);

// Device view of one packed matrix (pointers into the handle's device copy
// of the blob) plus the per-device schedule.
struct MatrixView {
    int rows, cols, bits, mode, slots, row_words;
    int64_t nnz;
    const uint32_t *dense;   // rows x row_words
    const uint16_t *table;   // LUT: rows x 2^bits fp16
    const int32_t *row_ptr;  // rows+1
    const uint16_t *col;     // nnz
    const uint16_t *val;     // nnz fp16
};

// Row-tile schedule of the batch-1..15 kernels: CTA t owns rows
// [tile_row[t], tile_row[t+1]).
struct Schedule {
    int n_tiles = 0;
    int32_t *tile_row = nullptr;  // device, n_tiles+1
};

}  // namespace dsq

struct dsq_handle_s {
    int device = -1;
    int sm_count = 0;
    dsq::BlobHeader header;
    uint8_t *d_blob = nullptr;
    size_t blob_bytes = 0;
    dsq::MatrixView view;
    dsq::Schedule sched;
    size_t device_bytes = 0;
};

namespace dsq {

// Launchers; each returns a dsq_status and never synchronises.
int launch_gemv_generic(const dsq_handle_s *h, const __half *x, __half *y, int batch,
                        cudaStream_t stream);
int launch_decode(const dsq_handle_s *h, __half *w, cudaStream_t stream);
int gemv_launch_count(const dsq_handle_s *h, int batch);
int launch_zero(__half *y, int64_t n, cudaStream_t stream);

}  // namespace dsq
