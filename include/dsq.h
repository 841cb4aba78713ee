/*
 * dsq.h -- C ABI of libdsq: the dense-and-sparse quantized matrix-vector /
 * skinny-matrix product on one NVIDIA B200 (sm_100a).
 *
 *     y[b][i] = sum_j x[b][j] * What[i][j],   What = W_dense + W_sparse
 *
 * W_dense (SqueezeLLM page, "Dense-and-Sparse decomposition"; SpQR page,
 * "Diagramme de la matrice sparse vs dense") holds one 3- or 4-bit code per
 * weight, decoded either
 *   - DSQ_MODE_LUT_ROW:    w = table[i][q], a per-output-row table of 2^bits
 *                          fp16 centroids (SqueezeLLM page, "Sensitivity-based
 *                          non-uniform quantization"), or
 *   - DSQ_MODE_AFFINE_G16: w = fp16(scale[i][g] * (q - zero[i][g])), g = j/16,
 *                          an fp16 scale and an integral fp16 zero per group
 *                          of 16 inputs (SpQR page, quant_config "wbits",
 *                          "groupsize": 16; the formula is this library's
 *                          reading, the page prints none), or
 *   - DSQ_MODE_BITPLANE:   w = fp16(C0 + sum_{i=1..k} C_i * b_i), k = bits
 *                          bit planes b_i = bit (i-1) of q and k+1 fp16
 *                          coefficients per group of 32 * 2^k inputs
 *                          (BPDQ page, "1. Formulation de la Grille
 *                          Variable"); the sum is exact, rounded once, or
 *   - DSQ_MODE_INTGRID:    w = fp16(scale[i][g] * q), q a signed integer with
 *                          |q| <= 8191, an fp16 scale per group of 16 inputs:
 *                          inliers and outliers on one unconstrained integer
 *                          grid, the integers Huffman coded (gist.science
 *                          2507.18553, the HPTQ bullet); packed by
 *                          dsq_pack_intgrid, bits = 14.
 * At the positions of the outliers the dense part holds "holes" whose codes
 * still decode (to 0 when the encoder chose q = zero).
 * W_sparse holds the outliers as fp16 CSR: values / col_idx / row_ptr (SpQR
 * page, "Le format de stockage sparse"); each outlier is ADDED to the decoded
 * dense weight at its position.
 *
 * Conventions for every call:
 *  - Return value is a dsq_status (0 = DSQ_OK); nothing else reports errors.
 *    No call aborts, traps or throws.  dsq_status_string() names a code.
 *  - "host" pointers are ordinary CPU memory; "device" pointers are CUDA
 *    global memory on the handle's device.  fp16 data is passed as raw IEEE
 *    binary16 bit patterns (uint16_t or void*).
 *  - A cudaStream_t is passed as void* (NULL = the legacy default stream),
 *    so this header needs no CUDA header.
 *  - Work on a stream is asynchronous: a DSQ_OK from dsq_gemv/dsq_decode
 *    means the kernels were launched; a fault inside them shows up at the
 *    caller's next synchronisation, as with any CUDA call.
 */
#ifndef DSQ_H
#define DSQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DSQ_API __attribute__((visibility("default")))
#else
#define DSQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DSQ_OK = 0,
    DSQ_ERR_INVALID_ARG = -1,     /* a NULL pointer, a size or value out of range, a malformed blob */
    DSQ_ERR_UNSUPPORTED = -2,     /* well-formed but outside what the library supports (e.g. cols > 65535) */
    DSQ_ERR_CUDA = -3,            /* a CUDA runtime call or a kernel launch failed */
    DSQ_ERR_OOM = -4,             /* device allocation failed */
    DSQ_ERR_BUFFER_TOO_SMALL = -5,/* output buffer smaller than required; size reported */
    DSQ_ERR_DEVICE = -6,          /* a kernel reported an error through its status word */
    DSQ_ERR_SCRATCH_LIMIT = -7    /* dsq_gemv_noalloc: the problem needs more than its fixed scratch */
} dsq_status;

enum { DSQ_MODE_LUT_ROW = 0, DSQ_MODE_AFFINE_G16 = 1, DSQ_MODE_BITPLANE = 2, DSQ_MODE_INTGRID = 3 };

/* Shape and encoding of one quantized weight matrix (rows = out features M,
 * cols = in features N).  Requirements: rows >= 0; cols >= 0 and
 * cols % 16 == 0; cols <= 65535 (column indices are stored in 16 bits);
 * bits in {3, 4} for DSQ_MODE_LUT_ROW and DSQ_MODE_AFFINE_G16, in {2, 3}
 * for DSQ_MODE_BITPLANE (there also cols % (32 << bits) == 0), 14 for
 * DSQ_MODE_INTGRID;
 * 0 <= nnz <= rows*cols. */
typedef struct {
    int32_t rows;
    int32_t cols;
    int32_t bits;
    int32_t mode;
    int64_t nnz;
} dsq_desc;

typedef struct dsq_handle_s *dsq_handle_t;

/*
 * dsq_pack -- validate the logical (unpacked) weights and write the packed
 * blob that dsq_create uploads.  Host-only; thread-safe; touches no GPU.
 *
 *   d        host; shape and encoding.
 *   codes    host uint8 [rows][cols] row-major, one code per byte, < 2^bits.
 *   table    host fp16.  LUT_ROW: [rows][2^bits] centroids.  AFFINE_G16:
 *            [rows][cols/16] scales.  BITPLANE: [rows][cols/(32<<bits)]
 *            [bits+1] coefficients C0..Ck of each group; every level
 *            C0 + sum_i C_i b_i must round to a finite fp16.  All finite.
 *   zeros    host fp16 [rows][cols/16] (AFFINE_G16: integral values in
 *            [0, 2^bits-1]); must be NULL for LUT_ROW and BITPLANE.  For AFFINE_G16,
 *            |scale| * max(zero, 2^bits-1-zero) must stay below 65520 so
 *            every decoded weight is finite.
 *   row_ptr  host int32 [rows+1]: row_ptr[0] = 0, nondecreasing,
 *            row_ptr[rows] = nnz.
 *   col_idx  host int32 [nnz]: < cols, strictly increasing inside a row.
 *   values   host fp16 [nnz], finite.
 *   out      host buffer of *out_bytes bytes, or NULL to query the size.
 *   out_bytes in: capacity of out; out: bytes required (always written when
 *            the inputs are valid).
 * Returns DSQ_OK, DSQ_ERR_INVALID_ARG (first invalid input; nothing written
 * to out), DSQ_ERR_UNSUPPORTED, or DSQ_ERR_BUFFER_TOO_SMALL (out too small
 * or NULL; *out_bytes holds the size).  The blob is position-independent
 * plain bytes and may be stored and reloaded.  With rows*cols == 0 the
 * pointers of empty arrays may be NULL.
 */
DSQ_API int dsq_pack(const dsq_desc *d, const uint8_t *codes, const uint16_t *table,
             const uint16_t *zeros, const int32_t *row_ptr,
             const int32_t *col_idx, const uint16_t *values, void *out,
             size_t *out_bytes);

/*
 * dsq_pack_two_axis -- dsq_pack for a matrix with two-axis scales (SINQ
 * page, "Mise a l'echelle sur deux axes"): a scale per output row and a
 * scale per input column around the quantized dense part,
 *
 *     What[i][j] = r[i] * c[j] * W_dense[i][j] + W_sparse[i][j],
 *
 * the product evaluated exactly (not rounded to fp16) and the outliers
 * unscaled.  Arguments as for dsq_pack, plus
 *   row_scale  host fp16 [rows], finite (may be NULL when rows == 0);
 *   col_scale  host fp16 [cols], finite (may be NULL when cols == 0).
 * The blob records the scales; dsq_create, dsq_gemv and dsq_decode take it
 * like any other (dsq_decode still writes W_dense, unscaled).  Every mode
 * is accepted; at batch 1 table and bit-plane matrices run the tuned table
 * kernel (x times c formed exactly in fp32 as it is loaded, r applied to
 * each row's dense sum before the outliers are added), other shapes and
 * batches the one-warp-per-row kernel.  Returns as dsq_pack, and
 * DSQ_ERR_INVALID_ARG for a non-finite or missing scale.
 */
DSQ_API int dsq_pack_two_axis(const dsq_desc *d, const uint8_t *codes, const uint16_t *table,
                              const uint16_t *zeros, const int32_t *row_ptr, const int32_t *col_idx,
                              const uint16_t *values, const uint16_t *row_scale,
                              const uint16_t *col_scale, void *out, size_t *out_bytes);

/*
 * dsq_pack_intgrid -- pack a DSQ_MODE_INTGRID matrix: Huffman-code its
 * integers (one canonical code per matrix, codes of at most 20 bits, an
 * MSB-first bitstream with the bit offset of every 32-column slot so slots
 * decode independently) and store its scales and outliers.
 *   d       host; mode DSQ_MODE_INTGRID, bits 14.
 *   q       host int16 [rows][cols], |q| <= 8191.
 *   scales  host fp16 [rows][cols/16], finite.
 *   row_ptr, col_idx, values, out, out_bytes  as for dsq_pack (an outlier
 *           list is optional: the grid holds outliers as large integers).
 * Returns as dsq_pack; DSQ_ERR_UNSUPPORTED when the stream would pass 2^32
 * bits.  dsq_gemv of such a matrix runs the variable-length-decode kernel
 * (one warp per row, lanes decoding whole slots); dsq_decode writes
 * fp16(scale * q).
 */
DSQ_API int dsq_pack_intgrid(const dsq_desc *d, const int16_t *q, const uint16_t *scales,
                             const int32_t *row_ptr, const int32_t *col_idx, const uint16_t *values,
                             void *out, size_t *out_bytes);

/*
 * dsq_blob_desc -- read the shape of a packed blob (host).  Returns
 * DSQ_ERR_INVALID_ARG when the blob is not one dsq_pack wrote.
 */
DSQ_API int dsq_blob_desc(const void *packed, size_t bytes, dsq_desc *out);

/*
 * dsq_create -- upload a packed blob to CUDA device `device` and build the
 * row-tile schedule for that device's SM count.  The handle owns every
 * device allocation it makes (released by dsq_destroy); the blob stays the
 * caller's and may be freed on return.  Synchronous.  The calling thread's
 * current device is left unchanged.
 * The blob's header and its outlier index (row pointers from 0 to nnz, never
 * decreasing; columns below cols and increasing within a row) are checked
 * on the host before any device work; codes, tables and scales are used as
 * they are.
 * Returns DSQ_OK, DSQ_ERR_INVALID_ARG (NULL out, malformed blob, bad
 * device), DSQ_ERR_UNSUPPORTED (not an sm_100 device), DSQ_ERR_OOM or
 * DSQ_ERR_CUDA.
 */
DSQ_API int dsq_create(const void *packed, size_t bytes, int device, dsq_handle_t *out);

/*
 * dsq_gemv -- y[b][i] = sum_j x[b][j] * What[i][j] for b < batch.
 *   x      device fp16 [batch][cols], row-major, 16-byte aligned (may be
 *          NULL only when cols == 0).
 *   y      device fp16 [batch][rows], row-major, 16-byte aligned (may be
 *          NULL only when rows == 0); fully overwritten, each
 *          element written once, rounded to nearest from an fp32 sum.
 *   batch  >= 1.  Affine 3-bit matrices take the tensor-core path from 3
 *          rows on (from 16 when a row holds more than 256 outliers);
 *          4-bit row-table matrices take warp-level tensor-core MMAs from
 *          5 rows on, 8 rows per launch; other table and bit-plane
 *          matrices (and 4-bit tables at 2-4 rows) take a CUDA-core
 *          kernel, 4 rows per launch; integer-grid matrices take the
 *          variable-length-decode kernel, up to 4 rows per launch;
 *          two-axis matrices (affine ones at every batch, the others
 *          from 2 rows) and affine 4-bit matrices take the one-warp-per-
 *          row kernel.
 *   stream cudaStream_t of the handle's device, as void*.
 * x and y are the caller's and must not overlap.  The handle is read-only
 * here, so calls on several streams or threads may run concurrently.
 * The kernels use programmatic dependent launch: they may start while the
 * previous kernel in `stream` is still running, but until it has finished
 * they read only the handle's own device memory; x is read and y written
 * after it, as with plain stream order.
 * Accuracy: |y - y_exact| <= 1e-3 * sum_j |What[i][j]| * |x[b][j]|.
 * Returns DSQ_OK, DSQ_ERR_INVALID_ARG (NULL or misaligned pointer,
 * batch < 1) or DSQ_ERR_CUDA (launch failure).
 */
DSQ_API int dsq_gemv(dsq_handle_t h, const void *x, void *y, int batch, void *stream);

/*
 * dsq_gemv_launches -- number of kernel launches one dsq_gemv call of this
 * batch makes on this handle (0 for an empty matrix); -1 for a NULL handle
 * or batch < 1.  Host-only.
 */
DSQ_API int dsq_gemv_launches(dsq_handle_t h, int batch);

/*
 * dsq_decode -- write W_dense (no outliers added) as fp16
 * [rows][cols] row-major to device memory w_dense_out (caller-owned), bit
 * for bit equal to the definitions above.  A test hook; asynchronous on
 * `stream`.
 */
DSQ_API int dsq_decode(dsq_handle_t h, void *w_dense_out, void *stream);

/*
 * dsq_handle_desc -- shape of the matrix a handle holds (host).
 */
DSQ_API int dsq_handle_desc(dsq_handle_t h, dsq_desc *out);

/*
 * dsq_device_bytes -- device bytes the handle holds (packed weights, CSR,
 * schedule), for accounting.  Returns 0 for NULL.
 */
DSQ_API size_t dsq_device_bytes(dsq_handle_t h);

/*
 * dsq_check -- synchronise the handle's device and report whether any
 * kernel launched for this handle gave up a bounded wait (its pipelines
 * never wait forever: a wait that runs out of iterations abandons the call
 * and sets a status word).  Returns DSQ_OK, DSQ_ERR_DEVICE (the word was set;
 * it is cleared, and the y of the affected calls is undefined) or
 * DSQ_ERR_CUDA.  Host-side; blocks until the device is idle.
 */
DSQ_API int dsq_check(dsq_handle_t h);

/*
 * dsq_selftest_wait_timeout -- test hook for the failure path of the bounded
 * waits: launches on `stream` one small kernel that waits on a barrier
 * nothing ever arrives on, through the same bounded wait (about 2 s) the
 * product kernels use; the wait gives up, sets the handle's status word and
 * the kernel returns, leaving the context usable.  A following dsq_check
 * then returns DSQ_ERR_DEVICE (and clears the word).  No product call makes
 * such a launch.  Returns DSQ_OK (launched), DSQ_ERR_INVALID_ARG or
 * DSQ_ERR_CUDA.
 */
DSQ_API int dsq_selftest_wait_timeout(dsq_handle_t h, void *stream);

/* dsq_destroy -- free the handle's device memory; NULL is a no-op.  The
 * caller must make sure no work using the handle is still in flight. */
DSQ_API int dsq_destroy(dsq_handle_t h);

/*
 * dsq_gemv_noalloc -- the product of dsq_gemv for a caller that may not
 * allocate device memory: y[b][i] = sum_j x[b][j] * What[i][j], b < batch.
 * The paper has no counterpart; this entry point exists for integration.
 *
 * Who needs it: code whose device memory all belongs to a host program --
 * a plugin that runs inside an inference engine or framework that hands out
 * every device buffer from its own pool (a cudaMalloc there would fragment
 * or escape the pool, or be forbidden outright), and code that runs where
 * cudaMalloc's implicit device synchronisation is not allowed.  Such a caller
 * cannot create a handle (dsq_create allocates), so it uploads the blob from
 * dsq_pack into memory it owns and calls this function with no handle.
 *
 * d             host; the blob's shape (as dsq_blob_desc reports it).
 * packed_device device; the dsq_pack blob copied verbatim, `bytes` long
 *               (exactly the size dsq_pack reported), 256-byte aligned.
 *               Read only; the caller owns it.  Being on the device, its
 *               contents are not checked as dsq_create checks them: pass
 *               only blobs that dsq_pack wrote.
 * x, y, batch, stream  as for dsq_gemv (fp16 [batch][cols] / [batch][rows],
 *               16-byte aligned, on the current device).
 *
 * Covers what the tensor-core path covers: 3-bit affine (DSQ_MODE_AFFINE_G16)
 * matrices with cols <= 32768 and batch >= 16; anything else returns
 * DSQ_ERR_UNSUPPORTED and launches nothing.  Results equal dsq_gemv's for the
 * same inputs on the same device.
 *
 * Memory: no device allocation of any kind.  The scratch the kernels need
 * (a status word and the start of every CSR row in each K split) is one
 * fixed 256 KiB array of the library that every GPU which loads it holds
 * until the process exits.  At most 65472 split-start entries fit: a
 * matrix whose K split needs more (split count x rows) is refused with
 * DSQ_ERR_SCRATCH_LIMIT before any launch.  Each call first clears the
 * status word and rewrites the split starts, so nothing of an earlier call
 * leaks into it; but every call on a device shares that one array, so calls
 * whose kernels overlap on the GPU (other streams, other host threads) race
 * and give undefined y: order them on one stream or with events.
 *
 * The first call on each device, with that device current, does a one-time
 * set-up (looks up the array's device address, sets the kernels' shared-
 * memory limit); make that first call before any stream capture.  A bounded
 * wait that runs out inside the kernels (a broken device, never a normal
 * call) leaves y of that call undefined; this entry point has no status
 * read-back.
 *
 * Returns DSQ_OK, DSQ_ERR_INVALID_ARG (NULL or misaligned pointer, batch <
 * 1, bytes not the blob's size, malformed desc), DSQ_ERR_UNSUPPORTED,
 * DSQ_ERR_SCRATCH_LIMIT or DSQ_ERR_CUDA.  Asynchronous on `stream`.
 */
DSQ_API int dsq_gemv_noalloc(const dsq_desc *d, const void *packed_device, size_t bytes, const void *x, void *y,
                             int batch, void *stream);

/*
 * dsq_decompose -- the step before dsq_pack, on the device: split dense fp32
 * weights into outliers and a quantized dense part (SqueezeLLM page,
 * "Dense-and-Sparse decomposition"; SpQR page, "Diagramme de la matrice
 * sparse vs dense" and "Quantification d'un modele").
 *   - outliers: the d->nnz largest |w| of the whole matrix (equal |w| taken
 *     in row-major order), as CSR with fp16 values (rounded to nearest);
 *   - dense part, outlier positions counting as 0:
 *     AFFINE_G16: per group of 16 inputs, the range [min, max] widened to
 *       contain 0; scale = fp16((max - min) / (2^bits - 1)) -- scale 1 and
 *       zero 0 when that is not a positive finite number --, zero =
 *       rint(-min / scale) and q = rint(w / scale) + zero, both clipped to
 *       [0, 2^bits - 1] (rint: nearest, ties to even; fp64 arithmetic);
 *     LUT_ROW: per row, the centroids are the fp16 roundings of the linear
 *       quantiles (2k+1)/2^(bits+1) of the row's dense weights (0 for a row
 *       of outliers only); every weight takes the nearest centroid, the
 *       lower index on a tie.
 * The outputs are exactly the logical arrays dsq_pack takes.
 *   d          host; rows, cols, bits, mode (LUT_ROW or AFFINE_G16, bits 3
 *              or 4), nnz = the number of outliers to keep.
 *   w          device fp32 [rows][cols], finite, 16-byte aligned; read only.
 *   codes      device uint8 [rows][cols], 16-byte aligned.
 *   table      device fp16: LUT_ROW [rows][2^bits] centroids, AFFINE_G16
 *              [rows][cols/16] scales.
 *   zeros      device fp16 [rows][cols/16] (AFFINE_G16); NULL for LUT_ROW.
 *   row_ptr    device int32 [rows+1]; col_idx device int32 [nnz]; values
 *              device fp16 [nnz].
 *   workspace  device scratch, 256-byte aligned, *workspace_bytes long, the
 *              caller's; with workspace NULL (or too small) the call only
 *              writes the size it needs to *workspace_bytes and returns
 *              DSQ_ERR_BUFFER_TOO_SMALL.  About rows*cols/8 bytes.
 *   stream     cudaStream_t as void*.  Asynchronous; nothing is allocated.
 * Limits: rows*cols < 2^31; LUT_ROW needs cols <= 32768 (one row is sorted
 * in shared memory).  Returns DSQ_OK, DSQ_ERR_INVALID_ARG (NULL or
 * misaligned pointer, bad desc), DSQ_ERR_UNSUPPORTED (BITPLANE mode, sizes
 * past the limits), DSQ_ERR_BUFFER_TOO_SMALL or DSQ_ERR_CUDA.
 */
DSQ_API int dsq_decompose(const dsq_desc *d, const float *w, void *codes, void *table, void *zeros,
                          int32_t *row_ptr, int32_t *col_idx, void *values, void *workspace,
                          size_t *workspace_bytes, void *stream);

/* Static, never-NULL text for a status code. */
DSQ_API const char *dsq_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* DSQ_H */
