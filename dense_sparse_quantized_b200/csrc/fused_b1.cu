// fused_b1.cu -- batch-1 dense+sparse GEMV: 3-bit affine group-16 rows and
// 3/4-bit row-LUT rows, one pass, y written once.
//
// One CTA per row tile (contiguous rows of about equal cost, one tile per
// SM, from a host schedule built at create).  Warp 0 is the producer: one
// thread streams, with 1-D bulk copies completing on shared-memory
// mbarriers,
//   * x, the tile's CSR entries, its piece list and (LUT) its table rows,
//   * then the tile's row records -- contiguous in HBM -- through a ring of
//     NS stages of R rows each.
// The other warps are consumers: warp (rg, cw) owns slot s = 32*cw + lane
// and, in every stage, row rg of the stage.  Each lane reads its 16-byte slot
// record from shared memory, decodes 32 weights against x held in registers,
// and the warp reduces the row's partial into shared memory.  After the
// ring, consumer warps reduce the outlier pieces (runs of <= 256 CSR entries
// of one row) from shared memory; then one thread per row adds the column
// partials and the row's piece sums, in a fixed order, and stores y.
//
// Affine decode.  A 3-bit field at bit p (p + 2 <= 22) of a 32-bit word,
// masked with AND and read as an fp32, is a subnormal equal to q * 2^(p-149)
// exactly.  Each lane keeps x[c] * 2^(111-p_c) in registers, so one AND and
// one FFMA add q * x * 2^-38 exactly (FFMA takes subnormal operands at full
// rate; nothing here flushes them).  Per group g of 16 columns:
//     t_g = sum_c q_c x_c - zero_g * X_g        (X_g = sum of the group's x)
//     acc += scale_g * t_g
// i.e. scale*(q - zero) factored out of the group sum; 2^-38 is removed once
// per row.
//
// Table decode.  Every lane of a 2^b-lane segment holds one centroid of the
// current row (fp32); shfl.idx over that segment reads only the low b bits of
// its index, so a code needs a shift but no mask.
#include <algorithm>
#include <vector>

#include "internal.h"
#include "ptx.h"

namespace dsq {

namespace {

constexpr int kThreads = 1024;
constexpr int kMaxConsumerWarps = kThreads / 32 - 1;
constexpr unsigned kFull = 0xffffffffu;
constexpr size_t kSmemBudget = 225 * 1024;
constexpr int kTileCsrCap = 12288;  // CSR entries per tile (48 KB), unless one row needs more

struct B1Params {
    MatrixView m;
    const TileDesc *tiles;
    const int32_t *row_piece;
    const int32_t *piece_k;
    int *status;
    int C, R, NS;
    int row_bytes, stage_bytes;
    // shared-memory offsets, bytes
    int off_x, off_ring, off_csr, off_rp, off_pk, off_part, off_psum, off_table;
};

// ---- 3-bit field placement (see layout.h) for column c < 30
__host__ __device__ constexpr int raw_pos3(int c) { return ((c % 10) & 1 ? 16 : 0) + 3 * ((c % 10) >> 1); }
// masked in the word itself (true) or in the word >> 9 (false)
__host__ __device__ constexpr bool direct3(int c) { return raw_pos3(c) <= 20; }
__host__ __device__ constexpr int pos3(int c) { return direct3(c) ? raw_pos3(c) : raw_pos3(c) - 9; }

__device__ __forceinline__ float fld(uint32_t w, uint32_t mask) { return __uint_as_float(w & mask); }

__device__ __forceinline__ uint4 lds128(const unsigned char *p) { return *reinterpret_cast<const uint4 *>(p); }

// ---------------------------------------------------------------- producer

template <bool LUT, int K>
__device__ void produce(const B1Params &p, const TileDesc &td, unsigned char *smem, uint64_t *full,
                        uint64_t *empty, uint64_t *aux, const __half *x) {
    const MatrixView &m = p.m;
    const int nrows = td.r1 - td.r0;
    // aux: x, CSR entries, piece and row->piece slices (16-byte aligned spans)
    const int ka = td.k0 & ~3, kb = (td.k1 + 3) & ~3;
    const int ra = td.r0 & ~3, rb = (td.r1 + 1 + 3) & ~3;
    const int pa = td.p0 & ~3, pb = (td.p1 + 1 + 3) & ~3;
    uint32_t aux_bytes = (uint32_t)m.cols * 2 + (uint32_t)(kb - ka) * 4 + (uint32_t)(rb - ra) * 4 +
                         (uint32_t)(pb - pa) * 4;
    if (LUT) aux_bytes += (uint32_t)nrows * K * 2;
    mbar_arrive_expect_tx(aux, aux_bytes);
    if (m.cols > 0) bulk_g2s(smem + p.off_x, x, (uint32_t)m.cols * 2, aux);
    if (kb > ka) bulk_g2s(smem + p.off_csr, m.csr + ka, (uint32_t)(kb - ka) * 4, aux);
    bulk_g2s(smem + p.off_rp, p.row_piece + ra, (uint32_t)(rb - ra) * 4, aux);
    bulk_g2s(smem + p.off_pk, p.piece_k + pa, (uint32_t)(pb - pa) * 4, aux);
    if (LUT) bulk_g2s(smem + p.off_table, m.table + (size_t)td.r0 * K, (uint32_t)nrows * K * 2, aux);

    const int n_st = (nrows + p.R - 1) / p.R;
    const unsigned char *src = reinterpret_cast<const unsigned char *>(m.dense) + (size_t)td.r0 * p.row_bytes;
    int issued = 0;
    for (int st = 0; st < n_st; st++) {
        const int slot = st % p.NS;
        if (st >= p.NS && !mbar_wait(&empty[slot], ((st / p.NS) - 1) & 1)) {
            report(p.status, kStatusTimeout);
            break;
        }
        const int rows_here = min(p.R, nrows - st * p.R);
        const uint32_t bytes = (uint32_t)rows_here * p.row_bytes;
        mbar_arrive_expect_tx(&full[slot], bytes);
        bulk_g2s(smem + p.off_ring + (size_t)slot * p.stage_bytes, src + (size_t)st * p.R * p.row_bytes, bytes,
                 &full[slot]);
        issued = st + 1;
    }
    // Copies still in flight must land before the CTA may exit.
    for (int st = max(0, issued - p.NS); st < issued; st++)
        if (!mbar_wait(&full[st % p.NS], (st / p.NS) & 1)) report(p.status, kStatusTimeout);
    if (!mbar_wait(aux, 0)) report(p.status, kStatusTimeout);
}

// ---------------------------------------------------------------- outliers

// Consumer warp `cw` of `ncw`: reduce pieces cw, cw + ncw, ... of the tile.
__device__ __forceinline__ void reduce_pieces(const TileDesc &td, const unsigned char *smem, const B1Params &p,
                                              int cw, int ncw, int lane) {
    const __half *xs = reinterpret_cast<const __half *>(smem + p.off_x);
    const uint32_t *csr = reinterpret_cast<const uint32_t *>(smem + p.off_csr);
    const int32_t *pk = reinterpret_cast<const int32_t *>(smem + p.off_pk);
    float *psum = reinterpret_cast<float *>(const_cast<unsigned char *>(smem) + p.off_psum);
    const int ka = td.k0 & ~3, pa = td.p0 & ~3;
    for (int q = td.p0 + cw; q < td.p1; q += ncw) {
        const int kb = pk[q - pa], ke = pk[q + 1 - pa];
        float acc = 0.f;
        for (int k = kb + lane; k < ke; k += 32) {
            const uint32_t e = csr[k - ka];
            acc = fmaf(__half2float(__ushort_as_half((unsigned short)(e >> 16))),
                       __half2float(xs[e & 0xffffu]), acc);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(kFull, acc, o);
        if (lane == 0) psum[q - td.p0] = acc;
    }
}

// y[r] = fp16(dense_scale * sum_c part[i][c] + sum of the row's piece sums).
__device__ __forceinline__ void finalize(const TileDesc &td, const unsigned char *smem, const B1Params &p,
                                         float dense_scale, __half *y) {
    const float *part = reinterpret_cast<const float *>(smem + p.off_part);
    const float *psum = reinterpret_cast<const float *>(smem + p.off_psum);
    const int32_t *rp = reinterpret_cast<const int32_t *>(smem + p.off_rp);
    const int ra = td.r0 & ~3;
    const int nrows = td.r1 - td.r0;
    for (int i = threadIdx.x; i < nrows; i += blockDim.x) {
        float acc = 0.f;
        for (int c = 0; c < p.C; c++) acc += part[(size_t)i * p.C + c];
        float o = 0.f;
        const int q0 = rp[td.r0 + i - ra], q1 = rp[td.r0 + i + 1 - ra];
        for (int q = q0; q < q1; q++) o += psum[q - td.p0];
        y[td.r0 + i] = __float2half_rn(fmaf(acc, dense_scale, o));
    }
}

// ---------------------------------------------------------------- kernel

template <int KIND>  // 0: affine 3-bit, 3: LUT 3-bit, 4: LUT 4-bit
__global__ void __launch_bounds__(kThreads, 1)
b1_kernel(B1Params p, const __half *__restrict__ x, __half *__restrict__ y) {
    constexpr bool LUT = KIND != 0;
    constexpr int BITS = KIND == 4 ? 4 : 3;
    constexpr int K = 1 << BITS;
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem);
    uint64_t *full = bars, *empty = bars + p.NS, *aux = bars + 2 * p.NS;
    const MatrixView &m = p.m;
    const int S = m.slots, C = p.C;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ncw = C * p.R;
    const TileDesc td = p.tiles[blockIdx.x];
    const int nrows = td.r1 - td.r0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < p.NS; i++) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], ncw);
        }
        mbar_init(aux, 1);
        fence_mbar_init();
    }
    // zero the padding columns of x (the bulk copy fills columns < N)
    for (int i = m.cols / 8 + threadIdx.x; i < S * 4; i += blockDim.x)
        reinterpret_cast<uint4 *>(smem + p.off_x)[i] = make_uint4(0u, 0u, 0u, 0u);
    __syncthreads();

    if (warp == 0) {
        if (lane == 0) produce<LUT, K>(p, td, smem, full, empty, aux, x);
    } else if (warp <= ncw) {
        const int cwarp = warp - 1;
        const int cw = cwarp % C, rg = cwarp / C;
        const int s = cw * 32 + lane;
        const bool valid = s < S;
        // this lane's 32 columns of x, straight from global memory (coalesced
        // 16-byte loads; chunks past N read as 0), while the ring fills
        float xv[32];
#pragma unroll
        for (int k = 0; k < 4; k++) {
            uint4 q = make_uint4(0u, 0u, 0u, 0u);
            if (valid && s * 32 + 8 * k < m.cols) q = __ldg(reinterpret_cast<const uint4 *>(x + (size_t)s * 32) + k);
            const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int t = 0; t < 4; t++) {
                const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&qw[t]));
                xv[8 * k + 2 * t] = f.x;
                xv[8 * k + 2 * t + 1] = f.y;
            }
        }
        bool ok = mbar_wait(aux, 0);
        if (!ok) report(p.status, kStatusTimeout);
        float *part = reinterpret_cast<float *>(smem + p.off_part);
        const int n_st = (nrows + p.R - 1) / p.R;

        if (!LUT) {
            float xr[32];
            float XA = 0.f, XB = 0.f;
#pragma unroll
            for (int c = 0; c < 32; c++) {
                const float v = xv[c];
                if (c < 16) XA += v; else XB += v;
                const int pc = c < 30 ? pos3(c) : (c == 30 ? 15 : 22);
                xr[c] = v * __uint_as_float((uint32_t)(127 + 111 - pc) << 23);
            }
            const float XAt = XA * 0x1p-38f, XBt = XB * 0x1p-38f;
            for (int st = 0; ok && st < n_st; st++) {
                const int slot = st % p.NS;
                if (!mbar_wait(&full[slot], (st / p.NS) & 1)) {
                    report(p.status, kStatusTimeout);
                    ok = false;
                    break;
                }
                const int i = st * p.R + rg;
                if (i < nrows) {
                    const unsigned char *rec = smem + p.off_ring + (size_t)slot * p.stage_bytes + (size_t)rg * p.row_bytes;
                    const uint4 v = valid ? lds128(rec + 16 * s) : make_uint4(0u, 0u, 0u, 0u);
                    const uint32_t zb = valid ? rec[16 * S + s] : 0u;
                    const uint32_t a[3] = {v.x, v.y, v.z};
                    const uint32_t b[3] = {a[0] >> 9, a[1] >> 9, a[2] >> 9};
                    float pa0 = 0.f, pa1 = 0.f, pb0 = 0.f, pb1 = 0.f;
#pragma unroll
                    for (int c = 0; c < 30; c++) {
                        const uint32_t w = direct3(c) ? a[c / 10] : b[c / 10];
                        const float f = fld(w, 7u << pos3(c));
                        if (c < 16) {
                            if (c & 1) pa1 = fmaf(f, xr[c], pa1); else pa0 = fmaf(f, xr[c], pa0);
                        } else {
                            if (c & 1) pb1 = fmaf(f, xr[c], pb1); else pb0 = fmaf(f, xr[c], pb0);
                        }
                    }
                    // columns 30, 31 (group B): bit k at bit 15 / bit 31 of word k
                    pb0 = fmaf(fld(a[0], 1u << 15), xr[30], pb0);
                    pb1 = fmaf(fld(a[1], 1u << 15), xr[30] * 2.f, pb1);
                    pb0 = fmaf(fld(a[2], 1u << 15), xr[30] * 4.f, pb0);
                    pb1 = fmaf(fld(b[0], 1u << 22), xr[31], pb1);
                    pb0 = fmaf(fld(b[1], 1u << 22), xr[31] * 2.f, pb0);
                    pb1 = fmaf(fld(b[2], 1u << 22), xr[31] * 4.f, pb1);
                    const float sA = __half2float(__ushort_as_half((unsigned short)(v.w & 0xffffu)));
                    const float sB = __half2float(__ushort_as_half((unsigned short)(v.w >> 16)));
                    const float zA = (float)(zb & 15u), zB = (float)(zb >> 4);
                    float r = sA * fmaf(-zA, XAt, pa0 + pa1);
                    r = fmaf(sB, fmaf(-zB, XBt, pb0 + pb1), r);
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) r += __shfl_xor_sync(kFull, r, o);
                    if (lane == 0) part[(size_t)i * C + cw] = r;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[slot]);
            }
        } else {
            float (&xr)[32] = xv;
            const __half *tab = reinterpret_cast<const __half *>(smem + p.off_table);
            for (int st = 0; ok && st < n_st; st++) {
                const int slot = st % p.NS;
                if (!mbar_wait(&full[slot], (st / p.NS) & 1)) {
                    report(p.status, kStatusTimeout);
                    ok = false;
                    break;
                }
                const int i = st * p.R + rg;
                if (i < nrows) {
                    const unsigned char *rec = smem + p.off_ring + (size_t)slot * p.stage_bytes + (size_t)rg * p.row_bytes;
                    const float tv = __half2float(tab[(size_t)i * K + (lane & (K - 1))]);
                    uint32_t w[4] = {0u, 0u, 0u, 0u};
                    if (valid) {
                        if (BITS == 4) {
                            const uint4 q = lds128(rec + 16 * s);
                            w[0] = q.x; w[1] = q.y; w[2] = q.z; w[3] = q.w;
                        } else {
                            const uint32_t *r32 = reinterpret_cast<const uint32_t *>(rec);
                            w[0] = r32[s]; w[1] = r32[S + s]; w[2] = r32[2 * S + s];
                        }
                    }
                    float acc[4] = {0.f, 0.f, 0.f, 0.f};
                    if (BITS == 4) {
#pragma unroll
                        for (int c = 0; c < 32; c++) {
                            const uint32_t wd = w[c >> 3];
                            const int sh = 4 * (c & 7);
                            acc[c & 3] = fmaf(__shfl_sync(kFull, tv, sh ? (int)(wd >> sh) : (int)wd, 16), xr[c],
                                              acc[c & 3]);
                        }
                    } else {
#pragma unroll
                        for (int c = 0; c < 30; c++) {
                            const uint32_t wd = w[c / 10];
                            const int sh = raw_pos3(c);
                            acc[c & 3] = fmaf(__shfl_sync(kFull, tv, sh ? (int)(wd >> sh) : (int)wd, 8), xr[c],
                                              acc[c & 3]);
                        }
                        const int q30 = (int)(((w[0] >> 15) & 1u) | ((w[1] >> 14) & 2u) | ((w[2] >> 13) & 4u));
                        const int q31 = (int)((w[0] >> 31) | ((w[1] >> 30) & 2u) | ((w[2] >> 29) & 4u));
                        acc[2] = fmaf(__shfl_sync(kFull, tv, q30, 8), xr[30], acc[2]);
                        acc[3] = fmaf(__shfl_sync(kFull, tv, q31, 8), xr[31], acc[3]);
                    }
                    float r = (acc[0] + acc[1]) + (acc[2] + acc[3]);
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) r += __shfl_xor_sync(kFull, r, o);
                    if (lane == 0) part[(size_t)i * C + cw] = r;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[slot]);
            }
        }
        if (ok) reduce_pieces(td, smem, p, cwarp, ncw, lane);
    }
    __syncthreads();
    finalize(td, smem, p, LUT ? 1.0f : 0x1p38f, y);
}

enum Kind { kNone = -1, kAff3 = 0, kLut3 = 3, kLut4 = 4 };

Kind b1_kind(const MatrixView &m, int batch) {
    if (batch != 1 || m.rows <= 0 || m.cols <= 0) return kNone;
    if ((m.slots + 31) / 32 > kMaxConsumerWarps) return kNone;
    if (m.mode == DSQ_MODE_AFFINE_G16) return m.bits == 3 ? kAff3 : kNone;
    return m.bits == 3 ? kLut3 : kLut4;
}

size_t align_sz(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Launch geometry and shared-memory map for a handle; false when the shape
// does not fit.
bool plan_b1(const dsq_handle_s *h, B1Params *out, size_t *smem_bytes) {
    const MatrixView &m = h->view;
    const Schedule &sc = h->sched;
    B1Params p;
    p.m = m;
    p.tiles = sc.tiles;
    p.row_piece = sc.row_piece;
    p.piece_k = sc.piece_k;
    p.status = h->d_status;
    p.C = (m.slots + 31) / 32;
    p.R = std::max(1, kMaxConsumerWarps / p.C);
    p.row_bytes = m.row_words * 4;
    p.stage_bytes = p.R * p.row_bytes;
    const int K = 1 << m.bits;
    size_t off = 256;  // mbarriers
    p.off_x = (int)off;
    off = align_sz(off + (size_t)m.slots * 64, 128);
    const size_t fixed_after = align_sz((size_t)(sc.max_csr + 8) * 4, 16) + align_sz((size_t)(sc.max_rows + 9) * 4, 16) +
                               align_sz((size_t)(sc.max_pieces + 9) * 4, 16) +
                               align_sz((size_t)sc.max_rows * p.C * 4, 16) + align_sz((size_t)(sc.max_pieces + 1) * 4, 16) +
                               (m.mode == DSQ_MODE_LUT_ROW ? align_sz((size_t)sc.max_rows * K * 2, 16) : 0);
    if (off + fixed_after + p.stage_bytes * 2 > kSmemBudget) return false;
    p.NS = (int)std::min<size_t>(8, (kSmemBudget - off - fixed_after) / p.stage_bytes);
    if (p.NS < 2) return false;
    p.off_ring = (int)off;
    off += (size_t)p.NS * p.stage_bytes;
    p.off_csr = (int)off;
    off = align_sz(off + (size_t)(sc.max_csr + 8) * 4, 16);
    p.off_rp = (int)off;
    off = align_sz(off + (size_t)(sc.max_rows + 9) * 4, 16);
    p.off_pk = (int)off;
    off = align_sz(off + (size_t)(sc.max_pieces + 9) * 4, 16);
    p.off_part = (int)off;
    off = align_sz(off + (size_t)sc.max_rows * p.C * 4, 16);
    p.off_psum = (int)off;
    off = align_sz(off + (size_t)(sc.max_pieces + 1) * 4, 16);
    p.off_table = (int)off;
    if (m.mode == DSQ_MODE_LUT_ROW) off = align_sz(off + (size_t)sc.max_rows * K * 2, 16);
    if (off > kSmemBudget) return false;
    *out = p;
    *smem_bytes = off;
    return true;
}

template <typename F>
int set_smem_attr(F f) {
    return cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBudget) == cudaSuccess
               ? DSQ_OK
               : DSQ_ERR_CUDA;
}

template <typename T>
int upload(T **dst, const std::vector<T> &v, size_t pad_elems, size_t *acct) {
    const size_t n = v.size() + pad_elems;
    if (cudaMalloc(dst, n * sizeof(T)) != cudaSuccess) {
        cudaGetLastError();
        *dst = nullptr;
        return DSQ_ERR_OOM;
    }
    *acct += n * sizeof(T);
    if (cudaMemset(*dst, 0, n * sizeof(T)) != cudaSuccess) return DSQ_ERR_CUDA;
    if (!v.empty() && cudaMemcpy(*dst, v.data(), v.size() * sizeof(T), cudaMemcpyHostToDevice) != cudaSuccess)
        return DSQ_ERR_CUDA;
    return DSQ_OK;
}

}  // namespace

// Row tiles of about equal cost (record bytes + a per-outlier charge), each
// holding at most kTileCsrCap CSR entries unless a single row has more, and
// the outlier pieces.  Host-side, at create.
int build_schedule(dsq_handle_s *h, const int32_t *rp) {
    const MatrixView &m = h->view;
    Schedule &sc = h->sched;
    if (m.rows == 0) return DSQ_OK;
    std::vector<int32_t> row_piece(m.rows + 1), piece_k;
    for (int r = 0; r < m.rows; r++) {
        row_piece[r] = (int32_t)piece_k.size();
        for (int32_t k = rp[r]; k < rp[r + 1]; k += kPieceMax) piece_k.push_back(k);
    }
    row_piece[m.rows] = (int32_t)piece_k.size();
    piece_k.push_back(rp[m.rows]);

    const int tiles_target = std::max(1, std::min(h->sm_count, m.rows));
    double total = 0;
    for (int i = 0; i < m.rows; i++) total += 4.0 * m.row_words + 8.0 * (rp[i + 1] - rp[i]) + 64.0;
    std::vector<TileDesc> tiles;
    int r0 = 0;
    double acc = 0, done = 0;
    for (int i = 0; i < m.rows; i++) {
        const double c = 4.0 * m.row_words + 8.0 * (rp[i + 1] - rp[i]) + 64.0;
        const bool over_csr = i > r0 && rp[i + 1] - rp[r0] > kTileCsrCap;
        const bool due = acc > 0 && (done + acc + c / 2) * tiles_target >= total * (tiles.size() + 1);
        if (i > r0 && (over_csr || (due && (int)tiles.size() + 1 < tiles_target))) {
            tiles.push_back({r0, i, row_piece[r0], row_piece[i], rp[r0], rp[i], 0, 0});
            done += acc;
            acc = 0;
            r0 = i;
        }
        acc += c;
    }
    tiles.push_back({r0, m.rows, row_piece[r0], row_piece[m.rows], rp[r0], rp[m.rows], 0, 0});
    sc.n_tiles = (int)tiles.size();
    sc.max_rows = sc.max_pieces = sc.max_csr = 0;
    for (const TileDesc &t : tiles) {
        sc.max_rows = std::max(sc.max_rows, t.r1 - t.r0);
        sc.max_pieces = std::max(sc.max_pieces, t.p1 - t.p0);
        sc.max_csr = std::max(sc.max_csr, t.k1 - t.k0);
    }
    int rc = upload(&sc.tiles, tiles, 0, &h->device_bytes);
    if (rc == DSQ_OK) rc = upload(&sc.row_piece, row_piece, 8, &h->device_bytes);
    if (rc == DSQ_OK) rc = upload(&sc.piece_k, piece_k, 8, &h->device_bytes);
    return rc;
}

void free_schedule(dsq_handle_s *h) {
    Schedule &sc = h->sched;
    if (sc.tiles) cudaFree(sc.tiles);
    if (sc.row_piece) cudaFree(sc.row_piece);
    if (sc.piece_k) cudaFree(sc.piece_k);
    sc.tiles = nullptr;
    sc.row_piece = sc.piece_k = nullptr;
}

// Per-device kernel attributes; called by dsq_create with the device current.
int fused_prepare(dsq_handle_s *) {
    int rc = set_smem_attr(b1_kernel<kAff3>);
    if (rc == DSQ_OK) rc = set_smem_attr(b1_kernel<kLut3>);
    if (rc == DSQ_OK) rc = set_smem_attr(b1_kernel<kLut4>);
    return rc;
}

int fused_launch_count(const dsq_handle_s *h, int batch) {
    B1Params p;
    size_t smem;
    return b1_kind(h->view, batch) != kNone && h->sched.n_tiles > 0 && plan_b1(h, &p, &smem) ? 1 : -1;
}

int launch_gemv_fused(const dsq_handle_s *h, const __half *x, __half *y, int batch, cudaStream_t st) {
    const Kind kind = b1_kind(h->view, batch);
    B1Params p;
    size_t smem;
    if (kind == kNone || h->sched.n_tiles == 0 || !plan_b1(h, &p, &smem)) return DSQ_ERR_UNSUPPORTED;
    const int threads = (1 + p.C * p.R) * 32;
    const int grid = h->sched.n_tiles;
    switch (kind) {
        case kAff3: b1_kernel<kAff3><<<grid, threads, smem, st>>>(p, x, y); break;
        case kLut3: b1_kernel<kLut3><<<grid, threads, smem, st>>>(p, x, y); break;
        default: b1_kernel<kLut4><<<grid, threads, smem, st>>>(p, x, y); break;
    }
    return cudaGetLastError() == cudaSuccess ? DSQ_OK : DSQ_ERR_CUDA;
}

}  // namespace dsq
