// decompose.cu -- the step before the product, on the device: outlier
// selection, the CSR of the outliers, and the quantization of the dense part
// into the logical arrays dsq_pack takes (SqueezeLLM page, "Dense-and-Sparse
// decomposition"; SpQR page, "Diagramme de la matrice sparse vs dense" and
// "Quantification d'un modele").
//
// Outliers: the nnz largest |w| of the whole matrix, equal |w| taken in
// row-major order.  |w| of a finite fp32 as its 31 low bits is an unsigned
// key in the same order, so the nnz-th largest key T comes from a 3-pass
// radix select (11 + 11 + 10 bits, one histogram per pass, no host round
// trip); then every key above T is an outlier, and of the keys equal to T
// the first nnz - #(keys > T) in row-major order.  One block per row counts
// its keys above and equal to T, a one-block scan gives every row its first
// equal-key rank and its CSR start, and one block per row writes its
// outliers (columns ascending, values rounded to fp16) and a per-row bit mask
// of the holes with warp ballots.
//
// Dense part, holes counting as 0:
//   affine (groups of 16): one thread per group -- the range widened to
//     contain 0, scale = fp16((max - min) / (2^b - 1)) (scale 1 / zero 0
//     when that is not a positive finite number), zero = rint(-min / scale)
//     clipped, q = rint(w / scale) + zero clipped, all in fp64 from the fp32
//     weights and the fp16 scale;
//   row table: one block per row sorts the row's dense weights in shared
//     memory (bitonic), takes the linear quantiles at (2k+1)/2^(b+1) in fp64
//     (explicitly rounded operations: no fused multiply-add, so the value is
//     the textbook expression's), rounds them to fp16 and gives every weight
//     the nearest centroid, the lower index on a tie.
#include <cuda_fp16.h>

#include <algorithm>

#include "internal.h"

namespace dsq {

namespace {

// radix digits, most significant first: bits 21..31, 10..20, 0..9
__host__ __device__ constexpr int digit_width(int pass) { return pass < 2 ? 11 : 10; }
__host__ __device__ constexpr int digit_shift(int pass) { return pass == 0 ? 21 : pass == 1 ? 10 : 0; }
constexpr int kBins = 2048;
constexpr int kRowThreads = 256;
constexpr int kLutThreads = 1024;
constexpr int kLutMaxCols = 32768;   // a row's dense weights sorted in shared memory

// Select state in the workspace.
struct SelState {
    uint32_t prefix;       // key bits fixed so far
    uint32_t remaining;    // rank still to find among keys with that prefix (1-based)
    uint32_t above;        // keys strictly above the prefix's range
    uint32_t pad;
};

__device__ __forceinline__ uint32_t key_of(float v) { return __float_as_uint(v) & 0x7fffffffu; }

// Histogram of digit `pass` of the keys whose higher digits equal the prefix.
__global__ void radix_hist_kernel(const float *__restrict__ w, int64_t n, int pass, const SelState *st,
                                  uint32_t *__restrict__ hist) {
    __shared__ uint32_t h[kBins];
    for (int b = threadIdx.x; b < kBins; b += blockDim.x) h[b] = 0;
    __syncthreads();
    const int shift = digit_shift(pass), width = digit_width(pass);
    const uint32_t mask = (1u << width) - 1u;
    const int hi_shift = shift + width;
    const uint32_t prefix = pass == 0 ? 0u : st->prefix;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const uint32_t k = key_of(__ldg(w + i));
        if (pass == 0 || (k >> hi_shift) == prefix) atomicAdd(&h[(k >> shift) & mask], 1u);
    }
    __syncthreads();
    for (int b = threadIdx.x; b < kBins; b += blockDim.x)
        if (h[b]) atomicAdd(&hist[b], h[b]);
}

// One thread: the digit holding the wanted rank (counted from the largest),
// appended to the prefix; the histogram is cleared for the next pass.
__global__ void radix_pick_kernel(int pass, uint32_t nnz, SelState *st, uint32_t *hist) {
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    if (pass == 0) {
        st->prefix = 0;
        st->remaining = nnz;
        st->above = 0;
    }
    const int width = digit_width(pass);
    uint32_t rem = st->remaining, cum = 0, pick = 0;
    for (int b = (1 << width) - 1; b >= 0; b--) {
        const uint32_t c = hist[b];
        if (cum + c >= rem) {
            pick = (uint32_t)b;
            break;
        }
        cum += c;
    }
    st->prefix = (st->prefix << width) | pick;
    st->remaining = rem - cum;
    st->above += cum;
    for (int b = 0; b < (1 << width); b++) hist[b] = 0;
}

// Per row: keys above T and keys equal to T.
__global__ void row_count_kernel(const float *__restrict__ w, int rows, int cols, const SelState *st, bool any,
                                 int32_t *__restrict__ gt, int32_t *__restrict__ eq) {
    const int r = blockIdx.x;
    const uint32_t T = st->prefix;
    int a = 0, e = 0;
    if (any)
        for (int j = threadIdx.x; j < cols; j += blockDim.x) {
            const uint32_t k = key_of(__ldg(w + (size_t)r * cols + j));
            a += k > T;
            e += k == T;
        }
    __shared__ int sa[kRowThreads / 32], se[kRowThreads / 32];
    for (int o = 16; o > 0; o >>= 1) {
        a += __shfl_xor_sync(0xffffffffu, a, o);
        e += __shfl_xor_sync(0xffffffffu, e, o);
    }
    if ((threadIdx.x & 31) == 0) {
        sa[threadIdx.x >> 5] = a;
        se[threadIdx.x >> 5] = e;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int ta = 0, te = 0;
        for (int i = 0; i < kRowThreads / 32; i++) {
            ta += sa[i];
            te += se[i];
        }
        gt[r] = ta;
        eq[r] = te;
    }
}

// Exclusive scan of n values by one block (thread t sums a contiguous chunk).
__device__ void block_exclusive_scan(const int32_t *in, int32_t *out, int n, int32_t *total) {
    __shared__ int32_t part[1024];
    const int per = (n + blockDim.x - 1) / blockDim.x;
    const int b0 = threadIdx.x * per, b1 = min(n, b0 + per);
    int32_t s = 0;
    for (int i = b0; i < b1; i++) s += in[i];
    part[threadIdx.x] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
        int32_t run = 0;
        for (int i = 0; i < (int)blockDim.x; i++) {
            const int32_t v = part[i];
            part[i] = run;
            run += v;
        }
        *total = run;
    }
    __syncthreads();
    int32_t run = part[threadIdx.x];
    for (int i = b0; i < b1; i++) {
        const int32_t v = in[i];
        out[i] = run;
        run += v;
    }
    __syncthreads();
}

// Row r takes all its keys above T and, of its keys equal to T, those whose
// row-major rank among the equal keys is below the number still wanted.
__global__ void row_scan_kernel(int rows, const SelState *st, bool any, const int32_t *gt, const int32_t *eq,
                                int32_t *eq_base, int32_t *outc, int32_t *row_ptr) {
    __shared__ int32_t total;
    block_exclusive_scan(eq, eq_base, rows, &total);
    const int32_t need = any ? (int32_t)st->remaining : 0;
    for (int r = threadIdx.x; r < rows; r += blockDim.x)
        outc[r] = (any ? gt[r] : 0) + max(0, min(eq[r], need - eq_base[r]));
    __syncthreads();
    block_exclusive_scan(outc, row_ptr, rows, &total);
    if (threadIdx.x == 0) row_ptr[rows] = total;
}

// Block-wide exclusive prefix of a flag over one chunk of blockDim columns;
// returns the prefix and writes the chunk's count to *count.
__device__ __forceinline__ int chunk_prefix(bool f, int *count) {
    __shared__ int wsum[kRowThreads / 32];
    const unsigned b = __ballot_sync(0xffffffffu, f);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) wsum[warp] = __popc(b);
    __syncthreads();
    int before = 0, all = 0;
    for (int i = 0; i < kRowThreads / 32; i++) {
        before += i < warp ? wsum[i] : 0;
        all += wsum[i];
    }
    __syncthreads();
    *count = all;
    return before + __popc(b & ((1u << lane) - 1u));
}

// One block per row: the row's outliers into CSR (columns ascending) and the
// row's hole mask (bit j % 32 of word j / 32).
__global__ void emit_kernel(const float *__restrict__ w, int rows, int cols, const SelState *st, bool any,
                            const int32_t *eq_base, const int32_t *row_ptr, int32_t *__restrict__ col_idx,
                            __half *__restrict__ values, uint32_t *__restrict__ holes, int mask_words) {
    const int r = blockIdx.x;
    const uint32_t T = st->prefix;
    const int32_t need = any ? (int32_t)st->remaining : 0;
    int eq_run = eq_base[r], out_run = row_ptr[r];
    for (int j0 = 0; j0 < cols; j0 += kRowThreads) {
        const int j = j0 + threadIdx.x;
        float v = 0.f;
        uint32_t k = 0;
        if (j < cols) {
            v = __ldg(w + (size_t)r * cols + j);
            k = key_of(v);
        }
        const bool is_eq = any && j < cols && k == T;
        int n_eq;
        const int eq_rank = eq_run + chunk_prefix(is_eq, &n_eq);
        const bool out = any && j < cols && (k > T || (is_eq && eq_rank < need));
        int n_out;
        const int pos = out_run + chunk_prefix(out, &n_out);
        if (out) {
            col_idx[pos] = j;
            values[pos] = __float2half_rn(v);
        }
        const unsigned m = __ballot_sync(0xffffffffu, out);
        if ((threadIdx.x & 31) == 0 && j < cols) holes[(size_t)r * mask_words + j / 32] = m;
        eq_run += n_eq;
        out_run += n_out;
    }
}

__device__ __forceinline__ bool is_hole(const uint32_t *holes, int mask_words, int r, int j) {
    return (holes[(size_t)r * mask_words + (j >> 5)] >> (j & 31)) & 1u;
}

// One thread per group of 16: scale, zero and codes.
__global__ void affine_kernel(const float *__restrict__ w, int rows, int cols, int bits,
                              const uint32_t *__restrict__ holes, int mask_words, uint8_t *__restrict__ codes,
                              __half *__restrict__ scales, __half *__restrict__ zeros) {
    const int G = cols / kGroup;
    const double qmax = (double)((1 << bits) - 1);
    for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < (int64_t)rows * G;
         t += (int64_t)gridDim.x * blockDim.x) {
        const int r = (int)(t / G), g = (int)(t % G);
        const float4 *src = reinterpret_cast<const float4 *>(w + (size_t)r * cols + (size_t)g * kGroup);
        float v[kGroup];
#pragma unroll
        for (int q = 0; q < 4; q++) {
            const float4 f = __ldg(src + q);
            v[4 * q] = f.x;
            v[4 * q + 1] = f.y;
            v[4 * q + 2] = f.z;
            v[4 * q + 3] = f.w;
        }
        const uint32_t hm = (holes[(size_t)r * mask_words + (g * kGroup >> 5)] >> ((g * kGroup) & 31)) & 0xffffu;
        double mn = 0.0, mx = 0.0;
#pragma unroll
        for (int c = 0; c < kGroup; c++) {
            const double x = (hm >> c) & 1u ? 0.0 : (double)v[c];
            mn = x < mn ? x : mn;
            mx = x > mx ? x : mx;
        }
        __half s16 = __double2half(__ddiv_rn(__dsub_rn(mx, mn), qmax));
        double sv = (double)__half2float(s16), z = 0.0;
        if (isfinite(sv) && sv > 0.0) {
            z = rint(__ddiv_rn(-mn, sv));
            z = z < 0.0 ? 0.0 : (z > qmax ? qmax : z);
        } else {
            s16 = __ushort_as_half(0x3C00);
            sv = 1.0;
        }
        scales[t] = s16;
        zeros[t] = __double2half(z);
        uint32_t packed[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int c = 0; c < kGroup; c++) {
            const double x = (hm >> c) & 1u ? 0.0 : (double)v[c];
            double q = __dadd_rn(rint(__ddiv_rn(x, sv)), z);
            q = q < 0.0 ? 0.0 : (q > qmax ? qmax : q);
            packed[c >> 2] |= (uint32_t)q << (8 * (c & 3));
        }
        uint4 *dst = reinterpret_cast<uint4 *>(codes + (size_t)r * cols + (size_t)g * kGroup);
        *dst = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    }
}

// One block per row: sorted dense weights, quantile centroids, nearest codes.
__global__ void __launch_bounds__(kLutThreads) lut_kernel(const float *__restrict__ w, int cols, int bits,
                                                          const uint32_t *__restrict__ holes, int mask_words,
                                                          uint8_t *__restrict__ codes, __half *__restrict__ table) {
    extern __shared__ float sv[];  // P floats, P a power of two >= the row's dense count
    __shared__ double cent[16];
    __shared__ int wcount[kLutThreads / 32];
    const int r = blockIdx.x, K = 1 << bits;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // compact the dense weights (order does not matter: they are sorted next)
    int base = 0;
    for (int j0 = 0; j0 < cols; j0 += kLutThreads) {
        const int j = j0 + threadIdx.x;
        const bool keep = j < cols && !is_hole(holes, mask_words, r, j);
        const unsigned b = __ballot_sync(0xffffffffu, keep);
        if (lane == 0) wcount[warp] = __popc(b);
        __syncthreads();
        int before = 0, all = 0;
        for (int i = 0; i < kLutThreads / 32; i++) {
            before += i < warp ? wcount[i] : 0;
            all += wcount[i];
        }
        if (keep) sv[base + before + __popc(b & ((1u << lane) - 1u))] = __ldg(w + (size_t)r * cols + j);
        base += all;
        __syncthreads();
    }
    const int m = base;
    int P = 1;
    while (P < m) P <<= 1;
    for (int i = m + threadIdx.x; i < P; i += kLutThreads) sv[i] = __int_as_float(0x7f800000);  // +inf
    __syncthreads();
    // bitonic sort, ascending
    for (int k = 2; k <= P; k <<= 1)
        for (int jj = k >> 1; jj > 0; jj >>= 1) {
            for (int i = threadIdx.x; i < P; i += kLutThreads) {
                const int l = i ^ jj;
                if (l > i) {
                    const float a = sv[i], b = sv[l];
                    const bool up = (i & k) == 0;
                    if ((a > b) == up) {
                        sv[i] = b;
                        sv[l] = a;
                    }
                }
            }
            __syncthreads();
        }
    if (threadIdx.x < K) {
        const int q = threadIdx.x;
        double c = 0.0;
        if (m > 0) {
            const double p = (2.0 * q + 1.0) / (2.0 * K);
            const double h = (double)(m - 1) * p;  // exact: a dyadic p times an integer below 2^24
            const int lo = (int)floor(h), hi = lo + 1 < m ? lo + 1 : m - 1;
            const double xl = (double)sv[lo], xh = (double)sv[hi];
            c = __dadd_rn(xl, __dmul_rn(__dsub_rn(h, (double)lo), __dsub_rn(xh, xl)));
        }
        const __half c16 = __double2half(c);
        table[(size_t)r * K + q] = c16;
        cent[q] = (double)__half2float(c16);
    }
    __syncthreads();
    for (int j = threadIdx.x; j < cols; j += kLutThreads) {
        const double v = is_hole(holes, mask_words, r, j) ? 0.0 : (double)__ldg(w + (size_t)r * cols + j);
        int best = 0;
        double bd = fabs(__dsub_rn(v, cent[0]));
        for (int q = 1; q < K; q++) {
            const double d = fabs(__dsub_rn(v, cent[q]));
            if (d < bd) {
                bd = d;
                best = q;
            }
        }
        codes[(size_t)r * cols + j] = (uint8_t)best;
    }
}

size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

// Workspace map: select state, histogram, four per-row int arrays, hole mask.
struct Ws {
    size_t st, hist, gt, eq, eqb, outc, holes, total;
};
Ws ws_map(int rows, int cols) {
    Ws m;
    size_t off = 0;
    m.st = off;
    off = align256(off + sizeof(SelState));
    m.hist = off;
    off = align256(off + kBins * 4);
    m.gt = off;
    off = align256(off + (size_t)rows * 4);
    m.eq = off;
    off = align256(off + (size_t)rows * 4);
    m.eqb = off;
    off = align256(off + (size_t)rows * 4);
    m.outc = off;
    off = align256(off + (size_t)rows * 4);
    m.holes = off;
    off = align256(off + (size_t)rows * ((cols + 31) / 32) * 4);
    m.total = off;
    return m;
}

}  // namespace

}  // namespace dsq

using namespace dsq;

extern "C" int dsq_decompose(const dsq_desc *d, const float *w, void *codes, void *table, void *zeros,
                             int32_t *row_ptr, int32_t *col_idx, void *values, void *workspace,
                             size_t *workspace_bytes, void *stream) {
    if (!d || !workspace_bytes) return DSQ_ERR_INVALID_ARG;
    int rc = check_desc(d);
    if (rc != DSQ_OK) return rc;
    if (d->mode == DSQ_MODE_BITPLANE) return DSQ_ERR_UNSUPPORTED;
    const int rows = d->rows, cols = d->cols, bits = d->bits;
    const int64_t n = (int64_t)rows * cols;
    if (n >= ((int64_t)1 << 31)) return DSQ_ERR_UNSUPPORTED;
    if (d->mode == DSQ_MODE_LUT_ROW && cols > kLutMaxCols) return DSQ_ERR_UNSUPPORTED;
    const Ws m = ws_map(rows, cols);
    if (!workspace || *workspace_bytes < m.total) {
        *workspace_bytes = m.total;
        return DSQ_ERR_BUFFER_TOO_SMALL;
    }
    if (rows == 0) return DSQ_OK;
    if (!row_ptr || (n > 0 && (!w || !codes || !table)) || (d->nnz > 0 && (!col_idx || !values)) ||
        (d->mode == DSQ_MODE_AFFINE_G16 && n > 0 && !zeros) || (d->mode == DSQ_MODE_LUT_ROW && zeros))
        return DSQ_ERR_INVALID_ARG;
    if (((uintptr_t)w & 15u) || ((uintptr_t)codes & 15u) || ((uintptr_t)workspace & 255u))
        return DSQ_ERR_INVALID_ARG;
    const cudaStream_t st = (cudaStream_t)stream;
    unsigned char *ws = (unsigned char *)workspace;
    SelState *sel = (SelState *)(ws + m.st);
    uint32_t *hist = (uint32_t *)(ws + m.hist);
    int32_t *gt = (int32_t *)(ws + m.gt), *eq = (int32_t *)(ws + m.eq);
    int32_t *eqb = (int32_t *)(ws + m.eqb), *outc = (int32_t *)(ws + m.outc);
    uint32_t *holes = (uint32_t *)(ws + m.holes);
    const int mask_words = (cols + 31) / 32;
    const bool any = d->nnz > 0;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (cudaMemsetAsync(ws, 0, m.total, st) != cudaSuccess) return DSQ_ERR_CUDA;
    if (any && n > 0)
        for (int pass = 0; pass < 3; pass++) {
            radix_hist_kernel<<<4 * sms, 512, 0, st>>>(w, n, pass, sel, hist);
            radix_pick_kernel<<<1, 32, 0, st>>>(pass, (uint32_t)d->nnz, sel, hist);
        }
    row_count_kernel<<<rows, kRowThreads, 0, st>>>(w, rows, cols, sel, any && n > 0, gt, eq);
    row_scan_kernel<<<1, 1024, 0, st>>>(rows, sel, any && n > 0, gt, eq, eqb, outc, row_ptr);
    if (n > 0) {
        emit_kernel<<<rows, kRowThreads, 0, st>>>(w, rows, cols, sel, any, eqb, row_ptr, col_idx,
                                                  (__half *)values, holes, mask_words);
        if (d->mode == DSQ_MODE_AFFINE_G16) {
            const int64_t groups = n / kGroup;
            const unsigned grid = (unsigned)std::min<int64_t>((groups + 255) / 256, 16 * sms);
            affine_kernel<<<grid, 256, 0, st>>>(w, rows, cols, bits, holes, mask_words, (uint8_t *)codes,
                                                (__half *)table, (__half *)zeros);
        } else {
            int P = 1;
            while (P < cols) P <<= 1;
            const size_t smem = (size_t)P * 4;
            if (cudaFuncSetAttribute(lut_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
                cudaSuccess)
                return DSQ_ERR_CUDA;
            lut_kernel<<<rows, kLutThreads, smem, st>>>(w, cols, bits, holes, mask_words, (uint8_t *)codes,
                                                        (__half *)table);
        }
    }
    return cudaGetLastError() == cudaSuccess ? DSQ_OK : DSQ_ERR_CUDA;
}
