// generic.cu -- the reference-quality CUDA path: one warp per output row,
// every weight decoded to its fp16 value exactly as dsq_decode writes it
// (table entry, fp16(scale * (q - zero)), or the bit-plane group level),
// fp32 accumulation, CSR outliers added by the same warp, y written once.
// Serves every shape, mode and batch; the tuned kernels replace it on the
// shapes they cover.  Also dsq_decode's kernel.
#include "internal.h"
#include "ptx.h"

namespace dsq {

// Code of column c (0..31) of a slot from its code words w[0..BITS-1].
template <int BITS>
__device__ __forceinline__ uint32_t slot_code(const uint32_t (&w)[4], int c) {
    uint32_t q = 0;
#pragma unroll
    for (int k = 0; k < BITS; k++) {
        int wi, pos;
        code_bit_place(BITS, c, k, &wi, &pos);
        q |= ((w[wi] >> pos) & 1u) << k;
    }
    return q;
}

template <int BITS, int MODE>
__device__ __forceinline__ void load_slot(const MatrixView &m, const uint32_t *rec, int s,
                                          uint32_t (&w)[4], uint32_t &scales, uint32_t &zb) {
#pragma unroll
    for (int p = 0; p < BITS; p++) w[p] = __ldg(rec + code_word_index(BITS, MODE, m.slots, s, p));
    if (MODE == DSQ_MODE_AFFINE_G16) {
        scales = __ldg(rec + scale_word_index(BITS, m.slots, s));
        zb = __ldg((const uint8_t *)rec + zero_byte_index(BITS, m.slots, s));
    }
}

// fp16 value of the decoded dense weight of column c of slot s.  row_table:
// the row's centroids (LUT_ROW) or its per-group levels (BITPLANE: the 2^BITS
// levels of every group of 2^BITS slots, one after the other).
template <int BITS, int MODE>
__device__ __forceinline__ __half decode_weight(const __half *row_table, uint32_t q,
                                                uint32_t scales, uint32_t zb, int c, int s) {
    if (MODE == DSQ_MODE_LUT_ROW) return row_table[q];
    if (MODE == DSQ_MODE_BITPLANE) return row_table[((s >> BITS) << BITS) + q];
    int e = c >> 4;  // group inside the slot
    __half sc = __ushort_as_half((unsigned short)(scales >> (16 * e)));
    int z = (int)((zb >> (4 * e)) & 15u);
    // (q - z) is a small integer and sc has an 11-bit significand: the fp32
    // product is exact, so this is the single rounding of sc*(q-z) to fp16.
    return __float2half_rn(__half2float(sc) * (float)((int)q - z));
}

template <int BITS, int MODE>
__device__ __forceinline__ const __half *row_table_of(const MatrixView &m, int row) {
    if (MODE == DSQ_MODE_LUT_ROW) return (const __half *)m.table + ((size_t)row << BITS);
    if (MODE == DSQ_MODE_BITPLANE) return (const __half *)m.table + (size_t)row * m.slots;
    return nullptr;
}

// TWO: two-axis scales -- the dense weights multiply c_j x_j (exact in fp32)
// and the row's dense sum is multiplied by r_i before the outliers, which use
// the unscaled x, are added.
template <int BITS, int MODE, int BC, bool TWO>
__global__ void __launch_bounds__(256) gemv_generic_kernel(MatrixView m, const __half *__restrict__ x,
                                                           __half *__restrict__ y, int batch, int b0) {
    const int lane = threadIdx.x & 31;
    const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (row >= m.rows) return;
    const int nb = min(BC, batch - b0);
    const int N = m.cols;
    const uint32_t *rec = m.dense + (size_t)row * m.row_words;
    const __half *row_table = row_table_of<BITS, MODE>(m, row);
    float acc[BC], aco[BC];  // dense and (two-axis only) outlier sums
#pragma unroll
    for (int b = 0; b < BC; b++) acc[b] = aco[b] = 0.f;

    for (int s = lane; s < m.slots; s += 32) {
        uint32_t w[4] = {0, 0, 0, 0}, scales = 0, zb = 0;
        load_slot<BITS, MODE>(m, rec, s, w, scales, zb);
#pragma unroll
        for (int c = 0; c < 32; c++) {
            const int j = s * 32 + c;
            if (j < N) {
                float wv = __half2float(decode_weight<BITS, MODE>(row_table, slot_code<BITS>(w, c), scales, zb, c, s));
                const float cj = TWO ? __half2float(__ushort_as_half(m.cscale[j])) : 1.0f;
#pragma unroll
                for (int b = 0; b < BC; b++)
                    if (b < nb) acc[b] = fmaf(wv, __half2float(x[(size_t)(b0 + b) * N + j]) * cj, acc[b]);
            }
        }
    }
    const int k0 = m.row_ptr[row], k1 = m.row_ptr[row + 1];
    for (int k = k0 + lane; k < k1; k += 32) {
        const uint32_t e = __ldg(m.csr + k);
        const float v = __half2float(__ushort_as_half((unsigned short)(e >> 16)));
        const int j = (int)(e & 0xffffu);
#pragma unroll
        for (int b = 0; b < BC; b++)
            if (b < nb) {
                if (TWO) aco[b] = fmaf(v, __half2float(x[(size_t)(b0 + b) * N + j]), aco[b]);
                else acc[b] = fmaf(v, __half2float(x[(size_t)(b0 + b) * N + j]), acc[b]);
            }
    }
    const float rs = TWO ? __half2float(__ushort_as_half(m.rscale[row])) : 1.0f;
#pragma unroll
    for (int b = 0; b < BC; b++) {
        float a = acc[b], o = aco[b];
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) {
            a += __shfl_xor_sync(0xffffffffu, a, d);
            if (TWO) o += __shfl_xor_sync(0xffffffffu, o, d);
        }
        if (lane == 0 && b < nb) y[(size_t)(b0 + b) * m.rows + row] = __float2half_rn(TWO ? fmaf(a, rs, o) : a);
    }
}

template <int BITS, int MODE>
__global__ void decode_kernel(MatrixView m, __half *__restrict__ w_out) {
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= (int64_t)m.rows * m.slots) return;
    const int row = (int)(t / m.slots), s = (int)(t % m.slots);
    const uint32_t *rec = m.dense + (size_t)row * m.row_words;
    const __half *row_table = row_table_of<BITS, MODE>(m, row);
    uint32_t w[4] = {0, 0, 0, 0}, scales = 0, zb = 0;
    load_slot<BITS, MODE>(m, rec, s, w, scales, zb);
#pragma unroll
    for (int c = 0; c < 32; c++) {
        const int j = s * 32 + c;
        if (j < m.cols)
            w_out[(size_t)row * m.cols + j] = decode_weight<BITS, MODE>(row_table, slot_code<BITS>(w, c), scales, zb, c, s);
    }
}

__global__ void zero_kernel(__half *y, int64_t n) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        y[i] = __ushort_as_half(0);
}

template <int BITS, int MODE, bool TWO>
static void launch_generic_tt(const MatrixView &m, const __half *x, __half *y, int batch, cudaStream_t st) {
    const int warps = 8;
    dim3 grid((m.rows + warps - 1) / warps);
    for (int b0 = 0; b0 < batch; b0 += 8) {
        int nb = batch - b0;
        if (nb == 1)
            gemv_generic_kernel<BITS, MODE, 1, TWO><<<grid, warps * 32, 0, st>>>(m, x, y, batch, b0);
        else if (nb <= 4)
            gemv_generic_kernel<BITS, MODE, 4, TWO><<<grid, warps * 32, 0, st>>>(m, x, y, batch, b0);
        else
            gemv_generic_kernel<BITS, MODE, 8, TWO><<<grid, warps * 32, 0, st>>>(m, x, y, batch, b0);
    }
}

template <int BITS, int MODE>
static void launch_generic_t(const MatrixView &m, const __half *x, __half *y, int batch, cudaStream_t st) {
    if (m.cscale) launch_generic_tt<BITS, MODE, true>(m, x, y, batch, st);
    else launch_generic_tt<BITS, MODE, false>(m, x, y, batch, st);
}

int launch_gemv_generic(const dsq_handle_s *h, const __half *x, __half *y, int batch, cudaStream_t st) {
    const MatrixView &m = h->view;
    if (m.rows == 0) return DSQ_OK;
    if (m.cols == 0) return launch_zero(y, (int64_t)batch * m.rows, st);
    if (m.mode == DSQ_MODE_BITPLANE) {
        if (m.bits == 2) launch_generic_t<2, 2>(m, x, y, batch, st);
        else launch_generic_t<3, 2>(m, x, y, batch, st);
    } else if (m.bits == 3 && m.mode == 0) launch_generic_t<3, 0>(m, x, y, batch, st);
    else if (m.bits == 4 && m.mode == 0) launch_generic_t<4, 0>(m, x, y, batch, st);
    else if (m.bits == 3) launch_generic_t<3, 1>(m, x, y, batch, st);
    else launch_generic_t<4, 1>(m, x, y, batch, st);
    return cudaGetLastError() == cudaSuccess ? DSQ_OK : DSQ_ERR_CUDA;
}

int gemv_launch_count(const dsq_handle_s *h, int batch) {
    if (h->view.rows == 0) return 0;
    if (h->view.cols == 0) return 1;
    return (batch + 7) / 8;
}

int launch_decode(const dsq_handle_s *h, __half *w, cudaStream_t st) {
    const MatrixView &m = h->view;
    const int64_t n = (int64_t)m.rows * m.slots;
    if (n == 0) return DSQ_OK;
    const int threads = 256;
    const unsigned grid = (unsigned)((n + threads - 1) / threads);
    if (m.mode == DSQ_MODE_BITPLANE) {
        if (m.bits == 2) decode_kernel<2, 2><<<grid, threads, 0, st>>>(m, w);
        else decode_kernel<3, 2><<<grid, threads, 0, st>>>(m, w);
    } else if (m.bits == 3 && m.mode == 0) decode_kernel<3, 0><<<grid, threads, 0, st>>>(m, w);
    else if (m.bits == 4 && m.mode == 0) decode_kernel<4, 0><<<grid, threads, 0, st>>>(m, w);
    else if (m.bits == 3) decode_kernel<3, 1><<<grid, threads, 0, st>>>(m, w);
    else decode_kernel<4, 1><<<grid, threads, 0, st>>>(m, w);
    return cudaGetLastError() == cudaSuccess ? DSQ_OK : DSQ_ERR_CUDA;
}

// One CTA waits on an mbarrier that nothing ever arrives on, through the same
// bounded wait every pipeline uses; when the wait gives up it records the
// timeout in the status word and returns.
__global__ void wait_timeout_kernel(int *status) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (!mbar_wait_warp(&bar, 0) && threadIdx.x == 0) report(status, kStatusTimeout);
}

int launch_wait_timeout(const dsq_handle_s *h, cudaStream_t st) {
    wait_timeout_kernel<<<1, 32, 0, st>>>(h->d_status);
    return cudaGetLastError() == cudaSuccess ? DSQ_OK : DSQ_ERR_CUDA;
}

int launch_zero(__half *y, int64_t n, cudaStream_t st) {
    if (n <= 0) return DSQ_OK;
    zero_kernel<<<(unsigned)std::min<int64_t>((n + 255) / 256, 4096), 256, 0, st>>>(y, n);
    return cudaGetLastError() == cudaSuccess ? DSQ_OK : DSQ_ERR_CUDA;
}

}  // namespace dsq
