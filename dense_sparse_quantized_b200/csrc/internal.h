// internal.h -- private declarations shared by the library's translation units.
#pragma once
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/dsq.h"
#include "layout.h"

namespace dsq {

double half_bits_to_double(uint16_t h);
int check_desc(const dsq_desc *d);
void plan_blob(const dsq_desc *d, BlobHeader *h, uint32_t flags = 0, uint32_t stream_words = 0,
               uint32_t nsym = 0);
int parse_blob(const void *packed, size_t bytes, BlobHeader *out);

// Device view of one packed matrix (pointers into the handle's device copy
// of the blob).
struct MatrixView {
    int rows, cols, bits, mode, slots, row_words;
    int64_t nnz;
    const uint32_t *dense;   // rows x row_words
    const uint16_t *table;   // LUT: rows x 2^bits fp16
    const int32_t *row_ptr;  // rows+1
    const uint32_t *csr;     // nnz: column | fp16 value << 16
    const uint16_t *rscale = nullptr;  // two-axis: fp16 [rows] row scales, else null
    const uint16_t *cscale = nullptr;  // two-axis: fp16 [cols] column scales, else null
    const uint32_t *slot_bits = nullptr;  // INTGRID: [rows][slots] first bit of each slot
    const uint32_t *codebook = nullptr;   // INTGRID: canonical code tables
};

// One CTA's share of the batch-1 work: rows [r0, r1), outlier pieces
// [p0, p1) and the CSR range [k0, k1) those pieces cover.
struct TileDesc {
    int32_t r0, r1, p0, p1, k0, k1, pad0, pad1;
};

// Schedule of the batch-1 kernels, built at create for the device's SM
// count.  Outliers are cut into "pieces": runs of at most kPieceMax entries
// of one row; piece p covers CSR entries [piece_k[p], piece_k[p+1]) and row
// r owns pieces [row_piece[r], row_piece[r+1]).  One lane sums a piece; an
// odd kPieceMax keeps the lanes walking consecutive pieces of a long row on
// distinct shared-memory banks.
constexpr int kPieceMax = 31;
struct Schedule {
    int n_tiles = 0;
    int per_sm = 1;       // CTAs per SM the tiles were cut for (batch-1 affine kernel)
    int max_rows = 0;     // rows of the largest tile
    int max_pieces = 0;   // pieces of the largest tile
    int max_csr = 0;      // CSR entries of the largest tile
    TileDesc *tiles = nullptr;    // device, n_tiles
    int32_t *row_piece = nullptr; // device, rows+1 (+ padding)
    int32_t *piece_k = nullptr;   // device, n_pieces+1 (+ padding)
};

// Tensor-core (batch >= 16) plan: the K split (a thread-block cluster of KS
// CTAs per 128-row tile) and where each split starts in every CSR row.
struct TcPlan {
    bool ready = false;
    int KS = 1, nkb = 0, kb_per_split = 0;
    int min_batch = 3;  // smallest batch sent to the tensor cores
    int32_t *split_start = nullptr;  // device, KS x rows (KS > 1)
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
    dsq::TcPlan tc;
    int *d_status = nullptr;  // sticky error word written by kernels on a timed-out wait
    size_t device_bytes = 0;
    int intgrid_grid[3] = {0, 0, 0};  // integer-grid blocks per launch for 1, 2, 4 activation rows
};

namespace dsq {

// Launchers; each returns a dsq_status and never synchronises.
int launch_gemv_generic(const dsq_handle_s *h, const __half *x, __half *y, int batch,
                        cudaStream_t stream);
int launch_decode(const dsq_handle_s *h, __half *w, cudaStream_t stream);
int gemv_launch_count(const dsq_handle_s *h, int batch);
int launch_zero(__half *y, int64_t n, cudaStream_t stream);
int launch_wait_timeout(const dsq_handle_s *h, cudaStream_t stream);
// Huffman-coded integer grids (huffman.cu).
// 4-bit row tables at 2+ activation rows on warp-level tensor cores (tc_lut.cu).
int tl4_prepare();  // per-device kernel attributes (dsq_create, device current)
bool tl4_covers(const dsq_handle_s *h, int batch);
int tl4_launch_count(const dsq_handle_s *h, int batch);
int launch_gemv_tl4(const dsq_handle_s *h, const __half *x, __half *y, int batch, cudaStream_t stream);
int launch_gemv_intgrid(const dsq_handle_s *h, const __half *x, __half *y, int batch, cudaStream_t stream);
int intgrid_launch_count(const dsq_handle_s *h, int batch);
int intgrid_prepare(dsq_handle_s *h);  // per-device attributes and the launch grids (dsq_create)
int launch_decode_intgrid(const dsq_handle_s *h, __half *w, cudaStream_t stream);
int check_intgrid_contents(const void *packed, const BlobHeader &h);

// Tuned batch-1 path (fused_b1.cu).  launch_gemv_fused returns
// DSQ_ERR_UNSUPPORTED, launching nothing, for shapes it does not cover.
int build_schedule(dsq_handle_s *h, const int32_t *row_ptr_host);
void free_schedule(dsq_handle_s *h);
int fused_prepare(dsq_handle_s *h);
int fused_launch_count(const dsq_handle_s *h, int batch);
int launch_gemv_fused(const dsq_handle_s *h, const __half *x, __half *y, int batch, cudaStream_t stream);
// Table matrices at batch >= 2 (fused_b1.cu), same convention.
int batched_launch_count(const dsq_handle_s *h, int batch);
int launch_gemv_batched(const dsq_handle_s *h, const __half *x, __half *y, int batch, cudaStream_t stream);

// Tensor-core path (tc_b16.cu), same convention.
int tc_prepare(dsq_handle_s *h, const int32_t *row_ptr_host, const uint32_t *csr_host);
void tc_free(dsq_handle_s *h);
bool tc_covers(const dsq_handle_s *h, int batch);
int tc_launch_count(const dsq_handle_s *h, int batch);
int launch_gemv_tc(const dsq_handle_s *h, const __half *x, __half *y, int batch, cudaStream_t stream);

}  // namespace dsq
