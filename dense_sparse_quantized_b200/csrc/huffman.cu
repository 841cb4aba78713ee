// huffman.cu -- Huffman-coded integer grids (gist.science 2507.18553, the
// HPTQ bullet: inliers and outliers on one unconstrained integer grid, the
// integers Huffman coded): the host encoder behind dsq_pack_intgrid and the
// variable-length-decode kernels of the product and of dsq_decode.
//
// Format.  Every weight is a signed integer q (|q| <= 8191) and every group
// of 16 inputs an fp16 scale; w = scale * q.  One canonical Huffman code per
// matrix (lengths at most 20 bits) codes the integers of all rows, row after
// row, slot after slot, into one MSB-first bitstream (bit p is bit 31 - p%32
// of word p/32).  The bit offset of every 32-column slot's first code is
// stored, so the 32 codes of a slot decode independently: a lane reads the
// 32-bit window at its offset with one funnel shift, one table read decodes
// codes of at most 10 bits, longer ones walk the per-length first codes.
//
// The product: one block per output row, one thread per slot, weights
// scale * q formed exactly in fp32 (|q| < 2^13, an 11-bit scale), fp32 FMAs,
// the CSR outliers by the same block, a fixed-order block sum, one fp16
// store.
#include <string.h>

#include <algorithm>
#include <functional>
#include <queue>
#include <vector>

#include "internal.h"

namespace dsq {

namespace {

constexpr size_t kIntGridXsMax = 132 * 1024;  // transposed x of the launch's activation rows (cols <= 65535: one row fits)

__device__ __forceinline__ uint32_t window32(const uint32_t *__restrict__ stream, uint32_t p) {
    const uint32_t hi = __ldg(stream + (p >> 5)), lo = __ldg(stream + (p >> 5) + 1);
    return __funnelshift_l(lo, hi, p & 31u);
}

// Decodes the code at bit p: returns the integer and advances p.  fast: the
// codebook's fast table (in shared memory), whose entry for a code of at most
// kHuffFastBits bits holds its length and the integer itself.
__device__ __forceinline__ int decode_one(const uint32_t *__restrict__ stream, const uint32_t *cb,
                                          const uint32_t *fast, uint32_t &p) {
    const uint32_t win = window32(stream, p);
    const uint32_t f = fast[win >> (32 - kHuffFastBits)];
    uint32_t len = f >> 16;
    int value = (int)(int16_t)(f & 0xffffu);
    if (len == 0) {
        const uint32_t maxl = __ldg(cb + 1);
        uint32_t sym = 0;
        len = maxl;
        for (uint32_t l = kHuffFastBits + 1; l <= maxl; l++) {
            const uint32_t code = win >> (32 - l);
            const uint32_t d = code - __ldg(cb + kCbFirst + l);
            if (d < __ldg(cb + kCbCount + l)) {
                len = l;
                sym = __ldg(cb + kCbOffset + l) + d;
                break;
            }
        }
        value = (int)(int16_t)__ldg(reinterpret_cast<const uint16_t *>(cb + kCbSyms) + sym);
    }
    p += len;
    return value;
}

// The fast table into shared memory (every thread of the block helps).
__device__ __forceinline__ void load_fast(uint32_t *fast, const uint32_t *cb) {
    for (int i = threadIdx.x; i < (1 << kHuffFastBits); i += blockDim.x) fast[i] = __ldg(cb + kCbFast + i);
}

// Long codes, counted against left-justified limits: with the canonical
// code, a window `top` starts a code longer than l bits exactly when top >=
// lim[l] = (first code of length l + count of length l) << (32 - l), so the
// length of a code longer than kHuffFastBits is kHuffFastBits + 1 plus the
// number of lengths l in (kHuffFastBits, maxl) with top >= lim[l].  lim and
// first come from the per-length counts alone (a running code), the symbol
// index is clamped to the symbol table.
struct LongCodes {
    uint32_t lim[kHuffMaxLen + 1];
    uint32_t first[kHuffMaxLen + 1];
    uint32_t offset[kHuffMaxLen + 1];
    uint32_t maxl, nsym;
};

__device__ void load_long_codes(LongCodes &lc, const uint32_t *cb) {
    if (threadIdx.x == 0) {
        const uint32_t maxl = min(__ldg(cb + 1), (uint32_t)kHuffMaxLen);
        uint32_t code = 0;
        for (int l = 1; l <= kHuffMaxLen; l++) {
            const uint32_t n = l <= (int)maxl ? __ldg(cb + kCbCount + l) : 0u;
            lc.first[l] = code;
            lc.offset[l] = __ldg(cb + kCbOffset + l);
            code += n;
            lc.lim[l] = l < 32 ? code << (32 - l) : code;
            code <<= 1;
        }
        lc.maxl = maxl;
        lc.nsym = max(__ldg(cb), 1u);
    }
}

// Per lane: a 64-bit bit buffer, most significant bit first, holding nb >= 20
// valid bits before every code (a refill adds one stream word when nb < 32).
struct BitReader {
    uint64_t buf;
    int nb;
    const uint32_t *next;
    __device__ __forceinline__ void start(const uint32_t *stream, uint32_t p) {
        const uint32_t *w = stream + (p >> 5);
        buf = ((((uint64_t)__ldg(w)) << 32) | __ldg(w + 1)) << (p & 31u);
        nb = 64 - (int)(p & 31u);
        next = w + 2;
    }
    __device__ __forceinline__ int decode(const uint32_t *fast, const LongCodes &lc, const uint16_t *syms) {
        const uint32_t top = (uint32_t)(buf >> 32);
        const uint32_t f = fast[top >> (32 - kHuffFastBits)];
        uint32_t len = f >> 16;
        int v = (int)(int16_t)(f & 0xffffu);
        if (len == 0) {
            len = kHuffFastBits + 1;
            for (uint32_t l = kHuffFastBits + 1; l < lc.maxl; l++) len += top >= lc.lim[l] ? 1u : 0u;
            const uint32_t sym = min(lc.offset[len] + (top >> (32 - len)) - lc.first[len], lc.nsym - 1);
            v = (int)(int16_t)__ldg(syms + sym);
        }
        buf <<= len;
        nb -= (int)len;
        if (nb < 32) {
            buf |= (uint64_t)__ldg(next++) << (32 - nb);
            nb += 32;
        }
        return v;
    }
};

// Persistent warps, one output row at a time: lane l decodes slots l, l+32,
// ... of the row, each slot's 32 codes from its own bit offset; a group of
// 16 codes accumulates sum q * x in fp32 and is scaled once by its fp16
// scale; the row's CSR outliers are spread over the lanes; one fixed
// shuffle tree sums the lanes and lane b stores y[b][row].
// Shared memory: the fast table, the long-code limits and x of nb activation
// rows transposed to [row b][column pair pc of the slot][slot] (one padding
// word per line), so the lanes -- on consecutive slots -- read consecutive
// words, staged once per block.
template <int BC>
__global__ void __launch_bounds__(256) intgrid_gemv_kernel(MatrixView m, const __half *__restrict__ x,
                                                           __half *__restrict__ y, int batch, int b0) {
    extern __shared__ uint32_t xs[];
    __shared__ uint32_t fast[1 << kHuffFastBits];
    __shared__ LongCodes lc;
    const int N = m.cols, S = m.slots, SP = S + 1;
    const int nb = min(BC, batch - b0);
    load_fast(fast, m.codebook);
    load_long_codes(lc, m.codebook);
    for (int i = threadIdx.x; i < BC * 16 * S; i += blockDim.x) {
        const int b = i / (16 * S), r = i - b * 16 * S, s = r >> 4, pc = r & 15, col = 32 * s + 2 * pc;
        uint32_t v = 0;
        if (b < nb && col < N) v = __ldg(reinterpret_cast<const uint32_t *>(x + (size_t)(b0 + b) * N + col));
        xs[(b * 16 + pc) * SP + s] = v;
    }
    __syncthreads();
    const uint16_t *syms = reinterpret_cast<const uint16_t *>(m.codebook + kCbSyms);
    const int lane = threadIdx.x & 31;
    const int warps = gridDim.x * (blockDim.x >> 5);
    for (int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); row < m.rows; row += warps) {
        const __half *scales = reinterpret_cast<const __half *>(m.table) + (size_t)row * (N / kGroup);
        float acc[BC];
#pragma unroll
        for (int b = 0; b < BC; b++) acc[b] = 0.f;
        for (int s = lane; s < S; s += 32) {
            BitReader br;
            br.start(m.dense, __ldg(m.slot_bits + (size_t)row * S + s));
            const int ngroups = min(32, N - 32 * s) / kGroup;  // 1 or 2
            for (int g = 0; g < ngroups; g++) {
                const float sc = __half2float(scales[2 * s + g]);
                float ag[BC];
#pragma unroll
                for (int b = 0; b < BC; b++) ag[b] = 0.f;
#pragma unroll
                for (int pc = 8 * g; pc < 8 * g + 8; pc++) {
                    const float q0 = (float)br.decode(fast, lc, syms);
                    const float q1 = (float)br.decode(fast, lc, syms);
#pragma unroll
                    for (int b = 0; b < BC; b++) {
                        const uint32_t xv = xs[(b * 16 + pc) * SP + s];
                        const float2 xf = __half22float2(*reinterpret_cast<const __half2 *>(&xv));
                        ag[b] = fmaf(q1, xf.y, fmaf(q0, xf.x, ag[b]));
                    }
                }
#pragma unroll
                for (int b = 0; b < BC; b++) acc[b] = fmaf(sc, ag[b], acc[b]);
            }
        }
        for (int k = m.row_ptr[row] + lane; k < m.row_ptr[row + 1]; k += 32) {
            const uint32_t e = __ldg(m.csr + k);
            const float v = __half2float(__ushort_as_half((unsigned short)(e >> 16)));
            const int j = (int)(e & 0xffffu), s = j >> 5, c = j & 31;
#pragma unroll
            for (int b = 0; b < BC; b++) {
                const uint32_t xv = xs[(b * 16 + (c >> 1)) * SP + s];
                acc[b] = fmaf(v, __half2float(__ushort_as_half((unsigned short)(xv >> (16 * (c & 1))))), acc[b]);
            }
        }
#pragma unroll
        for (int b = 0; b < BC; b++) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc[b] += __shfl_xor_sync(0xffffffffu, acc[b], o);
        }
#pragma unroll
        for (int b = 0; b < BC; b++)
            if (lane == b && b < nb) y[(size_t)(b0 + b) * m.rows + row] = __float2half_rn(acc[b]);
    }
}

// One thread per slot: W_dense = fp16(scale * q).
__global__ void intgrid_decode_kernel(MatrixView m, __half *__restrict__ w_out) {
    __shared__ uint32_t fast[1 << kHuffFastBits];
    load_fast(fast, m.codebook);
    __syncthreads();
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= (int64_t)m.rows * m.slots) return;
    const int row = (int)(t / m.slots), s = (int)(t % m.slots), N = m.cols;
    const __half *scales = reinterpret_cast<const __half *>(m.table) + (size_t)row * (N / kGroup);
    uint32_t p = __ldg(m.slot_bits + t);
    const int ncol = min(32, N - 32 * s);
    for (int c = 0; c < ncol; c++) {
        const int q = decode_one(m.dense, m.codebook, fast, p);
        w_out[(size_t)row * N + 32 * s + c] = __float2half_rn((float)q * __half2float(scales[2 * s + c / kGroup]));
    }
}

// ---------------------------------------------------------------- host encoder

struct Code {
    uint32_t bits = 0, len = 0;
};

// Huffman code lengths of the symbol frequencies, at most kHuffMaxLen bits
// (frequencies are halved until the longest code fits).
std::vector<uint32_t> code_lengths(std::vector<uint64_t> freq) {
    const size_t n = freq.size();
    std::vector<uint32_t> len(n, 0);
    if (n == 1) {
        len[0] = 1;
        return len;
    }
    for (;;) {
        // nodes: leaves 0..n-1, internal n..2n-2
        std::vector<int> parent(2 * n - 1, -1);
        using Item = std::pair<uint64_t, int>;
        std::priority_queue<Item, std::vector<Item>, std::greater<Item>> pq;
        for (size_t i = 0; i < n; i++) pq.push({freq[i], (int)i});
        int next = (int)n;
        while (pq.size() > 1) {
            const Item a = pq.top();
            pq.pop();
            const Item b = pq.top();
            pq.pop();
            parent[a.second] = next;
            parent[b.second] = next;
            pq.push({a.first + b.first, next});
            next++;
        }
        uint32_t maxl = 0;
        for (size_t i = 0; i < n; i++) {
            uint32_t l = 0;
            for (int v = (int)i; parent[v] >= 0; v = parent[v]) l++;
            len[i] = l;
            maxl = std::max(maxl, l);
        }
        if (maxl <= (uint32_t)kHuffMaxLen) return len;
        for (auto &f : freq) f = std::max<uint64_t>(1, f / 2);
    }
}

void put_bits(std::vector<uint32_t> &stream, uint64_t &pos, uint32_t bits, uint32_t len) {
    // MSB-first: the code's first bit lands at bit 31 - pos % 32 of word pos / 32
    for (uint32_t i = 0; i < len; i++) {
        const uint32_t b = (bits >> (len - 1 - i)) & 1u;
        if (b) stream[pos >> 5] |= 1u << (31 - (pos & 31));
        pos++;
    }
}

}  // namespace

// Host checks of an INTGRID blob's index and codebook (dsq_create): every
// slot offset inside the stream, a well-formed canonical code.
int check_intgrid_contents(const void *packed, const BlobHeader &h) {
    const uint8_t *b = (const uint8_t *)packed;
    const uint32_t *cb = (const uint32_t *)(b + h.off_codebook);
    const uint32_t nsym = cb[0], maxl = cb[1];
    if (nsym != h.nsym || nsym == 0 || nsym > 2 * kIntGridMax + 1 || maxl < 1 || maxl > (uint32_t)kHuffMaxLen)
        return DSQ_ERR_INVALID_ARG;
    uint64_t total = 0;
    for (uint32_t l = 1; l <= maxl; l++) {
        if (cb[kCbOffset + l] != total) return DSQ_ERR_INVALID_ARG;
        total += cb[kCbCount + l];
    }
    if (total != nsym) return DSQ_ERR_INVALID_ARG;
    for (int i = 0; i < (1 << kHuffFastBits); i++) {
        const uint32_t f = cb[kCbFast + i];
        const int v = (int)(int16_t)(f & 0xffffu);
        if ((f >> 16) > (uint32_t)kHuffFastBits || v < -kIntGridMax || v > kIntGridMax) return DSQ_ERR_INVALID_ARG;
    }
    const uint64_t stream_bits = (uint64_t)h.stream_words * 32;
    const uint32_t *idx = (const uint32_t *)(b + h.off_index);
    for (int64_t t = 0; t < (int64_t)h.rows * h.slots; t++)
        if (idx[t] > stream_bits) return DSQ_ERR_INVALID_ARG;
    return DSQ_OK;
}

// Activation rows per launch: x of BC rows, transposed, in shared memory
// (BC = 4 when the batch has 3 or more rows and 4 fit, else 2, else 1).
int intgrid_bc(int cols, int batch) {
    const size_t per_row = (size_t)16 * (slots_of(cols) + 1) * 4;
    const int cap = 4 * per_row <= kIntGridXsMax ? 4 : 2 * per_row <= kIntGridXsMax ? 2 : 1;
    return std::min(cap, batch >= 3 ? 4 : batch);
}

template <int BC>
size_t intgrid_smem(const MatrixView &m) {
    return (size_t)BC * 16 * (m.slots + 1) * 4;
}

// Blocks per launch for BC activation rows: every block resident at once
// (one pass of persistent warps), at most one per 8 rows.
template <int BC>
int intgrid_grid_of(const dsq_handle_s *h, int *grid) {
    const MatrixView &m = h->view;
    if (cudaFuncSetAttribute(intgrid_gemv_kernel<BC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kIntGridXsMax) != cudaSuccess)
        return DSQ_ERR_CUDA;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, intgrid_gemv_kernel<BC>, 256, intgrid_smem<BC>(m)) !=
        cudaSuccess)
        return DSQ_ERR_CUDA;
    *grid = (int)std::min<int64_t>((m.rows + 7) / 8, (int64_t)std::max(per_sm, 0) * h->sm_count);
    return DSQ_OK;
}

template <int BC>
int launch_intgrid_bc(const dsq_handle_s *h, const __half *x, __half *y, int batch, int b0, cudaStream_t st) {
    const MatrixView &m = h->view;
    const int grid = h->intgrid_grid[BC == 1 ? 0 : BC == 2 ? 1 : 2];
    if (grid < 1) return DSQ_ERR_UNSUPPORTED;  // the shape leaves no room for a block (x of BC rows)
    intgrid_gemv_kernel<BC><<<grid, 256, intgrid_smem<BC>(m), st>>>(m, x, y, batch, b0);
    return cudaGetLastError() == cudaSuccess ? DSQ_OK : DSQ_ERR_CUDA;
}

int intgrid_prepare(dsq_handle_s *h) {
    if (h->view.rows == 0 || h->view.cols == 0) return DSQ_OK;
    const int cap = intgrid_bc(h->view.cols, 4);  // activation rows whose x fits the stage
    int rc = intgrid_grid_of<1>(h, &h->intgrid_grid[0]);
    if (rc == DSQ_OK && cap >= 2) rc = intgrid_grid_of<2>(h, &h->intgrid_grid[1]);
    if (rc == DSQ_OK && cap >= 4) rc = intgrid_grid_of<4>(h, &h->intgrid_grid[2]);
    return rc;
}

int intgrid_launch_count(const dsq_handle_s *h, int batch) {
    if (h->view.rows == 0) return 0;
    if (h->view.cols == 0) return 1;
    const int bc = intgrid_bc(h->view.cols, batch);
    return (batch + bc - 1) / bc;
}

int launch_gemv_intgrid(const dsq_handle_s *h, const __half *x, __half *y, int batch, cudaStream_t st) {
    const MatrixView &m = h->view;
    if (m.rows == 0) return DSQ_OK;
    if (m.cols == 0) return launch_zero(y, (int64_t)batch * m.rows, st);
    const int bc = intgrid_bc(m.cols, batch);
    int rc = DSQ_OK;
    for (int b0 = 0; b0 < batch && rc == DSQ_OK; b0 += bc) {
        if (bc == 4) rc = launch_intgrid_bc<4>(h, x, y, batch, b0, st);
        else if (bc == 2) rc = launch_intgrid_bc<2>(h, x, y, batch, b0, st);
        else rc = launch_intgrid_bc<1>(h, x, y, batch, b0, st);
    }
    return rc;
}

int launch_decode_intgrid(const dsq_handle_s *h, __half *w, cudaStream_t st) {
    const MatrixView &m = h->view;
    const int64_t n = (int64_t)m.rows * m.slots;
    if (n == 0) return DSQ_OK;
    intgrid_decode_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(m, w);
    return cudaGetLastError() == cudaSuccess ? DSQ_OK : DSQ_ERR_CUDA;
}

}  // namespace dsq

using namespace dsq;

extern "C" int dsq_pack_intgrid(const dsq_desc *d, const int16_t *q, const uint16_t *scales,
                                const int32_t *row_ptr, const int32_t *col_idx, const uint16_t *values,
                                void *out, size_t *out_bytes) {
    if (!out_bytes || !d || d->mode != kModeIntGrid) return DSQ_ERR_INVALID_ARG;
    int rc = check_desc(d);
    if (rc != DSQ_OK) return rc;
    const int64_t M = d->rows, N = d->cols, nnz = d->nnz, G = N / kGroup;
    const int S = slots_of((int)N);
    if (M * N > 0 && (!q || !scales)) return DSQ_ERR_INVALID_ARG;
    if (M > 0 && !row_ptr) return DSQ_ERR_INVALID_ARG;
    if (nnz > 0 && (!col_idx || !values)) return DSQ_ERR_INVALID_ARG;
    for (int64_t t = 0; t < M * N; t++)
        if (q[t] < -kIntGridMax || q[t] > kIntGridMax) return DSQ_ERR_INVALID_ARG;
    for (int64_t t = 0; t < M * G; t++)
        if (!isfinite(half_bits_to_double(scales[t]))) return DSQ_ERR_INVALID_ARG;
    if (M > 0) {
        if (row_ptr[0] != 0 || row_ptr[M] != nnz) return DSQ_ERR_INVALID_ARG;
        for (int64_t i = 0; i < M; i++) {
            if (row_ptr[i + 1] < row_ptr[i]) return DSQ_ERR_INVALID_ARG;
            for (int64_t k = row_ptr[i]; k < row_ptr[i + 1]; k++)
                if (col_idx[k] < 0 || col_idx[k] >= N || (k > row_ptr[i] && col_idx[k] <= col_idx[k - 1]))
                    return DSQ_ERR_INVALID_ARG;
        }
    } else if (nnz != 0) {
        return DSQ_ERR_INVALID_ARG;
    }
    for (int64_t k = 0; k < nnz; k++)
        if (!isfinite(half_bits_to_double(values[k]))) return DSQ_ERR_INVALID_ARG;

    // the code: symbols = the distinct integers, canonical order (length, value)
    std::vector<uint64_t> count(2 * kIntGridMax + 1, 0);
    for (int64_t t = 0; t < M * N; t++) count[q[t] + kIntGridMax]++;
    std::vector<int> value;
    std::vector<uint64_t> freq;
    for (int v = 0; v < 2 * kIntGridMax + 1; v++)
        if (count[v]) {
            value.push_back(v - kIntGridMax);
            freq.push_back(count[v]);
        }
    if (value.empty()) {  // empty matrix: one dummy symbol keeps the codebook well formed
        value.push_back(0);
        freq.push_back(1);
    }
    const std::vector<uint32_t> len = code_lengths(freq);
    std::vector<int> order(value.size());
    for (size_t i = 0; i < order.size(); i++) order[i] = (int)i;
    std::sort(order.begin(), order.end(), [&](int a, int b) {
        return len[a] != len[b] ? len[a] < len[b] : value[a] < value[b];
    });
    const uint32_t nsym = (uint32_t)value.size();
    std::vector<uint32_t> cb(kCbSyms + (nsym + 1) / 2, 0);
    uint32_t maxl = 0;
    for (uint32_t l : len) maxl = std::max(maxl, l);
    cb[0] = nsym;
    cb[1] = maxl;
    std::vector<Code> code_of(2 * kIntGridMax + 1);
    uint32_t code = 0, prev_len = 0;
    for (uint32_t r = 0; r < nsym; r++) {
        const int i = order[r];
        code <<= (len[i] - prev_len);
        prev_len = len[i];
        if (cb[kCbCount + len[i]] == 0) {
            cb[kCbFirst + len[i]] = code;
            cb[kCbOffset + len[i]] = r;
        }
        cb[kCbCount + len[i]]++;
        code_of[value[i] + kIntGridMax] = {code, len[i]};
        if (len[i] <= (uint32_t)kHuffFastBits) {  // the entry holds the length and the integer
            const uint32_t lo = code << (kHuffFastBits - len[i]), hi = (code + 1) << (kHuffFastBits - len[i]);
            for (uint32_t e = lo; e < hi; e++) cb[kCbFast + e] = (len[i] << 16) | (uint16_t)(int16_t)value[i];
        }
        reinterpret_cast<uint16_t *>(cb.data() + kCbSyms)[r] = (uint16_t)(int16_t)value[i];
        code++;
    }
    // offsets of lengths with no code: the running symbol index (checked by
    // check_intgrid_contents)
    for (uint32_t l = 1, run = 0; l <= (uint32_t)kHuffMaxLen; l++) {
        cb[kCbOffset + l] = run;
        run += cb[kCbCount + l];
    }
    // the bitstream and the slot offsets
    uint64_t bits_total = 0;
    for (int64_t t = 0; t < M * N; t++) bits_total += code_of[q[t] + kIntGridMax].len;
    if (bits_total > 0xffffffffull - 64) return DSQ_ERR_UNSUPPORTED;
    const uint32_t words = (uint32_t)((bits_total + 31) / 32);

    BlobHeader h;
    plan_blob(d, &h, 0, words, nsym);
    if (!out || *out_bytes < h.total) {
        *out_bytes = h.total;
        return DSQ_ERR_BUFFER_TOO_SMALL;
    }
    *out_bytes = h.total;
    uint8_t *blob = (uint8_t *)out;
    memset(blob, 0, h.total);
    memcpy(blob, &h, sizeof(h));
    std::vector<uint32_t> stream((size_t)words + kStreamPad, 0);
    uint32_t *idx = (uint32_t *)(blob + h.off_index);
    uint64_t pos = 0;
    for (int64_t i = 0; i < M; i++)
        for (int s = 0; s < S; s++) {
            idx[i * S + s] = (uint32_t)pos;
            for (int c = 0; c < 32 && 32 * s + c < N; c++) {
                const Code &cd = code_of[q[i * N + 32 * s + c] + kIntGridMax];
                put_bits(stream, pos, cd.bits, cd.len);
            }
        }
    memcpy(blob + h.off_dense, stream.data(), stream.size() * 4);
    if (M * G > 0) memcpy(blob + h.off_table, scales, (size_t)(M * G) * 2);
    memcpy(blob + h.off_codebook, cb.data(), cb.size() * 4);
    if (M > 0) memcpy(blob + h.off_row_ptr, row_ptr, (size_t)(M + 1) * 4);
    uint32_t *csr = (uint32_t *)(blob + h.off_csr);
    for (int64_t k = 0; k < nnz; k++) csr[k] = (uint32_t)(uint16_t)col_idx[k] | ((uint32_t)values[k] << 16);
    return DSQ_OK;
}
