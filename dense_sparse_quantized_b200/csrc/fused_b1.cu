// fused_b1.cu -- batch-1 dense+sparse GEMV: 3-bit affine group-16 rows and
// 3/4-bit row-LUT rows, one pass, y written once.
//
// One CTA per row tile (contiguous rows of about equal cost, one tile per
// SM, from a host schedule built at create).  Warp (rg, cw) owns slot
// s = 32*cw + lane of rows r0 + rg, r0 + rg + R, ...: each lane streams that
// slot's 16-byte record (and, for affine rows, the zero byte) straight from
// HBM with 16-byte loads, U rows per batch of loads and two batches in flight
// (register double buffering), decodes 32 weights against x held in
// registers, and the warp reduces the row's partial into shared memory.
// Meanwhile one thread has started a background bulk copy of x, the tile's
// CSR entries and its outlier-piece lists into shared memory; after the dense
// loop the warps reduce the pieces (runs of <= 256 CSR entries of one row)
// from there, and one thread per row adds the column partials and the row's
// piece sums, in a fixed order, and stores y.
//
// (A shared-memory ring fed by bulk copies was measured slower here than
// direct loads: with one CTA per SM streaming its own contiguous range, the
// loads of 24 warps keep more bytes in flight.)
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

constexpr int kMaxWarps = 24;  // worker warps per CTA
constexpr int kThreads = kMaxWarps * 32;
constexpr int kDepth = 4;      // rows each lane has in flight (cp.async ring stages), a power of 2
constexpr int kStageB = 640;   // ring stage of one warp: 32 x 16-byte slot records + 32 x 4-byte words
constexpr unsigned kFull = 0xffffffffu;
constexpr size_t kSmemBudget = 225 * 1024;
constexpr int kTileCsrCap = 12288;  // CSR entries per tile (48 KB), unless one row needs more

struct B1Params {
    MatrixView m;
    const TileDesc *tiles;
    const int32_t *row_piece;
    const int32_t *piece_k;
    int *status;
    int C, R;  // column warps, row groups
    // shared-memory offsets, bytes
    int off_x, off_csr, off_rp, off_pk, off_part, off_psum, off_ring;
};

// ---- 3-bit field placement (see layout.h) for column c < 30
__host__ __device__ constexpr int raw_pos3(int c) { return ((c % 10) & 1 ? 16 : 0) + 3 * ((c % 10) >> 1); }
// masked in the word itself (true) or in the word >> 9 (false)
__host__ __device__ constexpr bool direct3(int c) { return raw_pos3(c) <= 20; }
__host__ __device__ constexpr int pos3(int c) { return direct3(c) ? raw_pos3(c) : raw_pos3(c) - 9; }

__device__ __forceinline__ float fld(uint32_t w, uint32_t mask) { return __uint_as_float(w & mask); }

// ---------------------------------------------------------------- aux copy

// x, the tile's CSR entries and its piece / row->piece slices, as 16-byte
// aligned spans, completing on `aux`.
__device__ void issue_aux(const B1Params &p, const TileDesc &td, unsigned char *smem, uint64_t *aux,
                          const __half *x) {
    const MatrixView &m = p.m;
    const int ka = td.k0 & ~3, kb = (td.k1 + 3) & ~3;
    const int ra = td.r0 & ~3, rb = (td.r1 + 1 + 3) & ~3;
    const int pa = td.p0 & ~3, pb = (td.p1 + 1 + 3) & ~3;
    const uint32_t bytes =
        (uint32_t)m.cols * 2 + (uint32_t)(kb - ka) * 4 + (uint32_t)(rb - ra) * 4 + (uint32_t)(pb - pa) * 4;
    mbar_arrive_expect_tx(aux, bytes);
    bulk_g2s(smem + p.off_x, x, (uint32_t)m.cols * 2, aux);
    if (kb > ka) bulk_g2s(smem + p.off_csr, m.csr + ka, (uint32_t)(kb - ka) * 4, aux);
    bulk_g2s(smem + p.off_rp, p.row_piece + ra, (uint32_t)(rb - ra) * 4, aux);
    bulk_g2s(smem + p.off_pk, p.piece_k + pa, (uint32_t)(pb - pa) * 4, aux);
}

// ---------------------------------------------------------------- outliers

// Warp `w` of `nw`: reduce pieces w, w + nw, ... of the tile.
__device__ __forceinline__ void reduce_pieces(const TileDesc &td, unsigned char *smem, const B1Params &p, int w,
                                              int nw, int lane) {
    const __half *xs = reinterpret_cast<const __half *>(smem + p.off_x);
    const uint32_t *csr = reinterpret_cast<const uint32_t *>(smem + p.off_csr);
    const int32_t *pk = reinterpret_cast<const int32_t *>(smem + p.off_pk);
    float *psum = reinterpret_cast<float *>(smem + p.off_psum);
    const int ka = td.k0 & ~3, pa = td.p0 & ~3;
    for (int q = td.p0 + w; q < td.p1; q += nw) {
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

// ---------------------------------------------------------------- row decoders

// Affine 3-bit slot record v (3 code words + scale pair) and zero byte zb:
// scale_A*(sum_A q x - zA X_A) + scale_B*(...), in units of 2^-38.
__device__ __forceinline__ float decode_aff3(const uint4 v, uint32_t zb, const float (&xr)[32], float XAt,
                                             float XBt) {
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
    const float r = sA * fmaf(-zA, XAt, pa0 + pa1);
    return fmaf(sB, fmaf(-zB, XBt, pb0 + pb1), r);
}

// Table slot: code words w[0..BITS-1], this row's centroid held by the lane.
template <int BITS>
__device__ __forceinline__ float decode_lut(const uint32_t (&w)[4], float tv, const float (&xr)[32]) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    if (BITS == 4) {
#pragma unroll
        for (int c = 0; c < 32; c++) {
            const uint32_t wd = w[c >> 3];
            const int sh = 4 * (c & 7);
            acc[c & 3] = fmaf(__shfl_sync(kFull, tv, sh ? (int)(wd >> sh) : (int)wd, 16), xr[c], acc[c & 3]);
        }
    } else {
#pragma unroll
        for (int c = 0; c < 30; c++) {
            const uint32_t wd = w[c / 10];
            const int sh = raw_pos3(c);
            acc[c & 3] = fmaf(__shfl_sync(kFull, tv, sh ? (int)(wd >> sh) : (int)wd, 8), xr[c], acc[c & 3]);
        }
        const int q30 = (int)(((w[0] >> 15) & 1u) | ((w[1] >> 14) & 2u) | ((w[2] >> 13) & 4u));
        const int q31 = (int)((w[0] >> 31) | ((w[1] >> 30) & 2u) | ((w[2] >> 29) & 4u));
        acc[2] = fmaf(__shfl_sync(kFull, tv, q30, 8), xr[30], acc[2]);
        acc[3] = fmaf(__shfl_sync(kFull, tv, q31, 8), xr[31], acc[3]);
    }
    return (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

__device__ __forceinline__ float warp_sum(float r) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) r += __shfl_xor_sync(kFull, r, o);
    return r;
}

// ---------------------------------------------------------------- kernel

template <int KIND>  // 0: affine 3-bit, 3: LUT 3-bit, 4: LUT 4-bit
__global__ void __launch_bounds__(kThreads, 1)
b1_kernel(B1Params p, const __half *__restrict__ x, __half *__restrict__ y) {
    constexpr bool LUT = KIND != 0;
    constexpr int BITS = KIND == 4 ? 4 : 3;
    constexpr int K = 1 << BITS;
    constexpr int NW = LUT ? BITS : 4;  // 32-bit words loaded per slot and row
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t *aux = reinterpret_cast<uint64_t *>(smem);
    const MatrixView &m = p.m;
    const int S = m.slots, C = p.C, R = p.R;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = blockDim.x >> 5;
    const TileDesc td = p.tiles[blockIdx.x];
    const int nrows = td.r1 - td.r0;
    const int cw = warp % C, rg = warp / C;
    const int s = cw * 32 + lane;
    const bool valid = s < S;

    // Per-lane asynchronous copy pipeline: each lane copies its own slot
    // record (and the word holding its zero byte, or its row's centroid) for
    // the rows kDepth ahead into this warp's ring, and later reads back
    // exactly what it copied -- no barrier, only cp.async.wait_group.  The
    // weights do not depend on the previous kernel in the stream, so the
    // first copies go out before the dependency wait.
    const uint32_t ring = smem_u32(smem + p.off_ring + (size_t)warp * kDepth * kStageB);
    const uint32_t ring_s = ring + 16 * lane, ring_a = ring + 512 + 4 * lane;
    const size_t row_step = (size_t)R * m.row_words * 4;  // bytes between this warp's rows
    const unsigned char *rec = reinterpret_cast<const unsigned char *>(m.dense) +
                               ((size_t)td.r0 + rg) * m.row_words * 4;  // next row to copy
    const unsigned char *tabp = reinterpret_cast<const unsigned char *>(m.table) +
                                ((size_t)(td.r0 + rg) * K + (lane & (K - 1))) * 2 - 2 * (lane & 1);
    const int nj = rg < nrows ? (nrows - rg + R - 1) / R : 0;  // rows of this warp
    int issued = 0;
    auto issue = [&](int d) {
        if (issued < nj) {
            const uint32_t st = ring_s + d * kStageB, sa = ring_a + d * kStageB;
            if (valid) {
                if (NW == 4) {
                    cp_async16(st, rec + 16 * s);
                } else {
#pragma unroll
                    for (int k = 0; k < NW; k++) cp_async4(st + 4 * k, rec + 4 * ((size_t)k * S + s));
                }
                if (!LUT) cp_async4(sa, rec + ((16 * S + s) & ~3));  // word holding the zero byte
            }
            // the 4-byte word holding this lane's centroid (table rows are 16/32-byte aligned)
            if (LUT) cp_async4(sa, tabp);
            rec += row_step;
            tabp += (size_t)R * K * 2;
        }
        issued++;
        cp_async_commit();
    };
#pragma unroll
    for (int d = 0; d < kDepth; d++) issue(d);

    // x (and y) belong to the surrounding program: wait for the previous
    // kernel in the stream before touching them.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (threadIdx.x == 0) {
        mbar_init(aux, 1);
        fence_mbar_init();
    }
    // zero the padding columns of x in shared memory (the bulk copy fills < N)
    for (int i = m.cols / 8 + threadIdx.x; i < S * 4; i += blockDim.x)
        reinterpret_cast<uint4 *>(smem + p.off_x)[i] = make_uint4(0u, 0u, 0u, 0u);
    __syncthreads();
    if (threadIdx.x == 0) issue_aux(p, td, smem, aux, x);
    float *part = reinterpret_cast<float *>(smem + p.off_part);

    // this lane's 32 columns of x from global memory (chunks past N read 0)
    float xr[32];
#pragma unroll
    for (int k = 0; k < 4; k++) {
        uint4 q = make_uint4(0u, 0u, 0u, 0u);
        if (valid && s * 32 + 8 * k < m.cols) q = __ldg(reinterpret_cast<const uint4 *>(x + (size_t)s * 32) + k);
        const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int t = 0; t < 4; t++) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&qw[t]));
            xr[8 * k + 2 * t] = f.x;
            xr[8 * k + 2 * t + 1] = f.y;
        }
    }
    float XAt = 0.f, XBt = 0.f;
    if (!LUT) {
        float XA = 0.f, XB = 0.f;
#pragma unroll
        for (int c = 0; c < 32; c++) {
            if (c < 16) XA += xr[c]; else XB += xr[c];
            const int pc = c < 30 ? pos3(c) : (c == 30 ? 15 : 22);
            xr[c] *= __uint_as_float((uint32_t)(127 + 111 - pc) << 23);
        }
        XAt = XA * 0x1p-38f;
        XBt = XB * 0x1p-38f;
    }

    int i = rg;
    for (int j = 0; j < nj; j++, i += R) {
        const int d = j & (kDepth - 1);
        cp_async_wait<kDepth - 1>();  // this lane's copies for row j have landed
        const uint32_t st = ring_s + d * kStageB, sa = ring_a + d * kStageB;
        float r = 0.f;
        if (!LUT) {
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            uint32_t zb = 0u;
            if (valid) {
                v = lds128(st);
                zb = (lds32(sa) >> (8 * (s & 3))) & 0xffu;
            }
            r = decode_aff3(v, zb, xr, XAt, XBt);
        } else {
            uint32_t w4[4] = {0u, 0u, 0u, 0u};
            if (valid) {
                if (NW == 4) {
                    const uint4 q = lds128(st);
                    w4[0] = q.x; w4[1] = q.y; w4[2] = q.z; w4[3] = q.w;
                } else {
#pragma unroll
                    for (int k = 0; k < NW; k++) w4[k] = lds32(st + 4 * k);
                }
            }
            const float tv = __half2float(__ushort_as_half((unsigned short)(lds32(sa) >> (16 * (lane & 1)))));
            r = decode_lut<BITS>(w4, tv, xr);
        }
        r = warp_sum(r);
        if (lane == 0) part[(size_t)i * C + cw] = r;
        issue(d);  // refill this stage (its data has been consumed)
    }
    cp_async_wait<0>();

    if (mbar_wait_warp(aux, 0)) reduce_pieces(td, smem, p, warp, nwarps, lane);
    else if (lane == 0) report(p.status, kStatusTimeout);
    __syncthreads();
    finalize(td, smem, p, LUT ? 1.0f : 0x1p38f, y);
}

enum Kind { kNone = -1, kAff3 = 0, kLut3 = 3, kLut4 = 4 };

Kind b1_kind(const MatrixView &m, int batch) {
    if (batch != 1 || m.rows <= 0 || m.cols <= 0) return kNone;
    if ((m.slots + 31) / 32 > kMaxWarps) return kNone;
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
    p.R = std::max(1, kMaxWarps / p.C);
    size_t off = 128;  // mbarrier
    p.off_x = (int)off;
    off = align_sz(off + (size_t)m.slots * 64, 128);
    p.off_csr = (int)off;
    off = align_sz(off + (size_t)(sc.max_csr + 8) * 4, 16);
    p.off_rp = (int)off;
    off = align_sz(off + (size_t)(sc.max_rows + 9) * 4, 16);
    p.off_pk = (int)off;
    off = align_sz(off + (size_t)(sc.max_pieces + 9) * 4, 16);
    p.off_part = (int)off;
    off = align_sz(off + (size_t)sc.max_rows * p.C * 4, 16);
    p.off_psum = (int)off;
    off = align_sz(off + (size_t)(sc.max_pieces + 1) * 4, 128);
    p.off_ring = (int)off;
    off += (size_t)p.C * p.R * kDepth * kStageB;
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
    // Programmatic dependent launch: the kernel may start while the previous
    // kernel in the stream drains; it streams weights first and waits
    // (griddepcontrol.wait) before it reads x or writes y.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(h->sched.n_tiles, 1, 1);
    cfg.blockDim = dim3(p.C * p.R * 32, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e;
    switch (kind) {
        case kAff3: e = cudaLaunchKernelEx(&cfg, b1_kernel<kAff3>, p, x, y); break;
        case kLut3: e = cudaLaunchKernelEx(&cfg, b1_kernel<kLut3>, p, x, y); break;
        default: e = cudaLaunchKernelEx(&cfg, b1_kernel<kLut4>, p, x, y); break;
    }
    return e == cudaSuccess ? DSQ_OK : DSQ_ERR_CUDA;
}

}  // namespace dsq
