// api.cu -- the C ABI entry points that touch a device: create, gemv,
// decode, destroy, plus status strings.
#include <string.h>

#include <new>
#include <vector>

#include "internal.h"

using namespace dsq;

namespace dsq {
int check_blob_contents(const void *packed, const BlobHeader &h);  // pack.cu
}

namespace {

// Makes `device` current for the scope and restores the caller's device.
struct DeviceGuard {
    int prev = -1;
    bool ok = false;
    explicit DeviceGuard(int device) {
        if (cudaGetDevice(&prev) != cudaSuccess) return;
        ok = prev == device || cudaSetDevice(device) == cudaSuccess;
    }
    ~DeviceGuard() {
        int cur = -1;
        if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
    }
};

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace

extern "C" const char *dsq_status_string(int status) {
    switch (status) {
        case DSQ_OK: return "DSQ_OK";
        case DSQ_ERR_INVALID_ARG: return "DSQ_ERR_INVALID_ARG: invalid argument";
        case DSQ_ERR_UNSUPPORTED: return "DSQ_ERR_UNSUPPORTED: outside what the library supports";
        case DSQ_ERR_CUDA: return "DSQ_ERR_CUDA: CUDA runtime or launch failure";
        case DSQ_ERR_OOM: return "DSQ_ERR_OOM: device allocation failed";
        case DSQ_ERR_BUFFER_TOO_SMALL: return "DSQ_ERR_BUFFER_TOO_SMALL: output buffer too small";
        case DSQ_ERR_DEVICE: return "DSQ_ERR_DEVICE: a kernel reported an error";
        case DSQ_ERR_SCRATCH_LIMIT:
            return "DSQ_ERR_SCRATCH_LIMIT: the matrix needs more than dsq_gemv_noalloc's fixed scratch";
        default: return "unknown dsq status";
    }
}

extern "C" int dsq_create(const void *packed, size_t bytes, int device, dsq_handle_t *out) {
    if (!out) return DSQ_ERR_INVALID_ARG;
    *out = nullptr;
    BlobHeader hd;
    int rc = parse_blob(packed, bytes, &hd);
    if (rc == DSQ_OK) rc = check_blob_contents(packed, hd);
    if (rc == DSQ_OK && hd.mode == DSQ_MODE_INTGRID) rc = check_intgrid_contents(packed, hd);
    if (rc != DSQ_OK) return rc;
    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess) return DSQ_ERR_CUDA;
    if (device < 0 || device >= ndev) return DSQ_ERR_INVALID_ARG;
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, device) != cudaSuccess) return DSQ_ERR_CUDA;
    if (prop.major != 10 || prop.minor != 0) return DSQ_ERR_UNSUPPORTED;
    DeviceGuard guard(device);
    if (!guard.ok) return DSQ_ERR_CUDA;

    dsq_handle_s *h = new (std::nothrow) dsq_handle_s();
    if (!h) return DSQ_ERR_OOM;
    h->device = device;
    h->sm_count = prop.multiProcessorCount;
    h->header = hd;
    h->blob_bytes = hd.total;
    if (cudaMalloc(&h->d_blob, hd.total) != cudaSuccess) {
        cudaGetLastError();
        delete h;
        return DSQ_ERR_OOM;
    }
    h->device_bytes = hd.total;
    if (cudaMemcpy(h->d_blob, packed, hd.total, cudaMemcpyHostToDevice) != cudaSuccess) {
        dsq_destroy(h);
        return DSQ_ERR_CUDA;
    }
    MatrixView &m = h->view;
    m.rows = hd.rows;
    m.cols = hd.cols;
    m.bits = hd.bits;
    m.mode = hd.mode;
    m.slots = hd.slots;
    m.row_words = hd.row_words;
    m.nnz = hd.nnz;
    m.dense = (const uint32_t *)(h->d_blob + hd.off_dense);
    m.table = (const uint16_t *)(h->d_blob + hd.off_table);
    m.row_ptr = (const int32_t *)(h->d_blob + hd.off_row_ptr);
    m.csr = (const uint32_t *)(h->d_blob + hd.off_csr);
    if (hd.mode == DSQ_MODE_INTGRID) {
        m.slot_bits = (const uint32_t *)(h->d_blob + hd.off_index);
        m.codebook = (const uint32_t *)(h->d_blob + hd.off_codebook);
    }
    if (hd.flags & kFlagTwoAxis) {
        m.rscale = (const uint16_t *)(h->d_blob + hd.off_rscale);
        m.cscale = (const uint16_t *)(h->d_blob + hd.off_cscale);
    }
    if (cudaMalloc(&h->d_status, sizeof(int)) != cudaSuccess) {
        cudaGetLastError();
        dsq_destroy(h);
        return DSQ_ERR_OOM;
    }
    h->device_bytes += sizeof(int);
    if (cudaMemset(h->d_status, 0, sizeof(int)) != cudaSuccess) {
        dsq_destroy(h);
        return DSQ_ERR_CUDA;
    }
    const int32_t *rp_host = (const int32_t *)((const uint8_t *)packed + hd.off_row_ptr);
    rc = build_schedule(h, rp_host);
    if (rc == DSQ_OK) rc = fused_prepare(h);
    if (rc == DSQ_OK) rc = tl4_prepare();
    if (rc == DSQ_OK && hd.mode == DSQ_MODE_INTGRID) rc = intgrid_prepare(h);
    if (rc == DSQ_OK) rc = tc_prepare(h, rp_host, (const uint32_t *)((const uint8_t *)packed + hd.off_csr));
    if (rc != DSQ_OK) {
        dsq_destroy(h);
        return rc;
    }
    *out = h;
    return DSQ_OK;
}

extern "C" int dsq_gemv(dsq_handle_t h, const void *x, void *y, int batch, void *stream) {
    if (!h || batch < 1) return DSQ_ERR_INVALID_ARG;
    if ((!x && h->view.cols > 0) || (!y && h->view.rows > 0)) return DSQ_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(y)) return DSQ_ERR_INVALID_ARG;
    DeviceGuard guard(h->device);
    if (!guard.ok) return DSQ_ERR_CUDA;
    const __half *xh = (const __half *)x;
    __half *yh = (__half *)y;
    const cudaStream_t st = (cudaStream_t)stream;
    if (h->view.mode == DSQ_MODE_INTGRID) return launch_gemv_intgrid(h, xh, yh, batch, st);
    // tensor cores where they cover the shape and batch; else the tuned
    // batch-1 kernel once per activation row; else the generic kernel
    int rc = launch_gemv_tc(h, xh, yh, batch, st);
    if (rc == DSQ_ERR_UNSUPPORTED && batch > 1) rc = launch_gemv_batched(h, xh, yh, batch, st);
    if (rc == DSQ_ERR_UNSUPPORTED && fused_launch_count(h, 1) > 0) {
        rc = DSQ_OK;
        for (int b = 0; b < batch && rc == DSQ_OK; b++)
            rc = launch_gemv_fused(h, xh + (size_t)b * h->view.cols, yh + (size_t)b * h->view.rows, 1, st);
    }
    if (rc == DSQ_ERR_UNSUPPORTED) rc = launch_gemv_generic(h, xh, yh, batch, st);
    return rc;
}

extern "C" int dsq_gemv_launches(dsq_handle_t h, int batch) {
    if (!h || batch < 1) return -1;
    if (h->view.mode == DSQ_MODE_INTGRID) return intgrid_launch_count(h, batch);
    int n = tc_launch_count(h, batch);
    if (n < 0 && batch > 1) n = batched_launch_count(h, batch);
    if (n < 0 && fused_launch_count(h, 1) > 0) n = batch * fused_launch_count(h, 1);
    return n >= 0 ? n : gemv_launch_count(h, batch);
}

extern "C" int dsq_decode(dsq_handle_t h, void *w_dense_out, void *stream) {
    if (!h || !w_dense_out) return DSQ_ERR_INVALID_ARG;
    DeviceGuard guard(h->device);
    if (!guard.ok) return DSQ_ERR_CUDA;
    if (h->view.mode == DSQ_MODE_INTGRID) return launch_decode_intgrid(h, (__half *)w_dense_out, (cudaStream_t)stream);
    return launch_decode(h, (__half *)w_dense_out, (cudaStream_t)stream);
}

extern "C" int dsq_selftest_wait_timeout(dsq_handle_t h, void *stream) {
    if (!h) return DSQ_ERR_INVALID_ARG;
    DeviceGuard guard(h->device);
    if (!guard.ok) return DSQ_ERR_CUDA;
    return launch_wait_timeout(h, (cudaStream_t)stream);
}

extern "C" int dsq_handle_desc(dsq_handle_t h, dsq_desc *out) {
    if (!h || !out) return DSQ_ERR_INVALID_ARG;
    out->rows = h->header.rows;
    out->cols = h->header.cols;
    out->bits = h->header.bits;
    out->mode = h->header.mode;
    out->nnz = h->header.nnz;
    return DSQ_OK;
}

extern "C" size_t dsq_device_bytes(dsq_handle_t h) { return h ? h->device_bytes : 0; }

extern "C" int dsq_destroy(dsq_handle_t h) {
    if (!h) return DSQ_OK;
    DeviceGuard guard(h->device);
    int rc = DSQ_OK;
    if (h->d_blob && cudaFree(h->d_blob) != cudaSuccess) rc = DSQ_ERR_CUDA;
    if (h->d_status && cudaFree(h->d_status) != cudaSuccess) rc = DSQ_ERR_CUDA;
    free_schedule(h);
    tc_free(h);
    delete h;
    return rc;
}

extern "C" int dsq_check(dsq_handle_t h) {
    if (!h) return DSQ_ERR_INVALID_ARG;
    DeviceGuard guard(h->device);
    if (!guard.ok) return DSQ_ERR_CUDA;
    if (cudaDeviceSynchronize() != cudaSuccess) return DSQ_ERR_CUDA;
    int word = 0;
    if (cudaMemcpy(&word, h->d_status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return DSQ_ERR_CUDA;
    if (word == 0) return DSQ_OK;
    const int zero = 0;
    if (cudaMemcpy(h->d_status, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return DSQ_ERR_CUDA;
    return DSQ_ERR_DEVICE;
}
