// fused_b1.cu -- batch-1 dense+sparse GEMV: 3-bit affine group-16 rows,
// 3/4-bit row-LUT rows and 2/3-bit-plane rows (per-group level tables), one
// pass, y written once; and the table kernel for 2-4 activation rows.
//
// One CTA per row tile (contiguous rows of about equal cost, one tile per
// SM, from a host schedule built at create).  Warp (rg, cw) owns slot
// s = 32*cw + lane of rows r0 + rg, r0 + rg + R, ...: each lane streams that
// slot's 16-byte record (and the word holding its zero byte or centroid)
// straight from HBM -- the first rows before the kernel waits on the
// previous one in the stream, since the packed weights never depend on it --
// decodes 32 weights against its 32 columns of x held in registers, and the
// warp reduces the row's partial into shared memory.  Meanwhile one thread
// has started a background bulk copy of x, the tile's CSR entries and its
// outlier-piece lists into shared memory; after the dense loop every thread
// sums whole pieces (runs of <= 31 CSR entries of one row) from there, and
// one thread per row adds the column partials and the row's piece sums, in a
// fixed order, and stores y.
//
// Affine decode.  A pair of 3-bit codes sits at the same bit h (0, 3 or 6)
// of both 16-bit halves of a word, or of the word shifted right by 10.  One
// LOP3 keeps the pair and ORs in the exponent of M_h = 2^(10-h): each half is
// then the fp16 number M_h + q (the code lands in the mantissa in units of
// 1).  One HSUB2 of M_h + zero (exact: both operands lie within a factor of
// two) leaves q - zero, a small integer, and two mixed-precision FMAs (fp32
// += fp16 * fp16, whose product is exact in fp32) add (q - zero) * x to the
// group's fp32 sum; the fp16 scale multiplies each group sum once.  The zero
// point is taken off every code before its product, so the rounding error of
// a group sum follows sum |q - zero| |x|, the weights' own share of the
// error bound, whatever the range of x.  x stays in its fp16 form in
// registers: nothing is rounded but the fp32 sums.
//
// Table decode.  Every lane of a 2^b-lane segment holds one centroid of the
// current row (fp32); shfl.idx over that segment reads only the low b bits of
// its index, so a code needs a shift but no mask.
#include <algorithm>
#include <type_traits>
#include <vector>

#include "internal.h"
#include "ptx.h"

namespace dsq {

namespace {

constexpr int kMaxWarps = 24;  // warps per CTA
constexpr int kThreads = kMaxWarps * 32;
constexpr int kDepth = 4;      // table kernel: rows each lane has in flight (cp.async ring stages), a power of 2
constexpr int kD = 8;          // affine kernel: rows each lane has in flight (cp.async ring stages)
constexpr int kRB = 4;         // affine kernel: rows decoded per step, reduced together (divides kD)
constexpr int kHeavyPieces = 32;  // rows with more pieces are summed by a whole warp
constexpr int kPre = 4;          // affine kernel: ring stages requested before the dependency wait
// shared-memory header: mbarriers of the staged CSR + piece lists and of the
// staged x
constexpr int kBarCsr = 0, kBarX = 8;
constexpr int kStageB = 640;   // table kernel ring stage of one warp: 32 x 16-byte code words + 32 x 4-byte words
constexpr unsigned kFull = 0xffffffffu;
constexpr size_t kSmemBudget = 225 * 1024;
constexpr int kTileCsrCap = 12288;  // CSR entries per tile (48 KB), unless one row needs more
// Affine matrices of at most kWarps2 column groups run two CTAs of kWarps2
// warps per SM over twice as many row tiles: the next call's CTAs then start
// streaming while this call's last CTAs finish their outliers and stores
// (measured 3-7% faster per call than one CTA of 24 warps per SM).  Each
// CTA must fit half of the SM's shared memory.
constexpr int kWarps2 = 14;
constexpr size_t kSmemBudget2 = 112 * 1024;
constexpr int kTileCsrCap2 = 6144;

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

// ---- 3-bit field placement (layout.h) for column c < 30: bit of the word
__host__ __device__ constexpr int raw_pos3(int c) {
    return ((c % 10) & 1 ? 16 : 0) + ((c % 10) >> 1 < 3 ? 3 * ((c % 10) >> 1) : 3 * ((c % 10) >> 1) + 1);
}

// ---------------------------------------------------------------- aux copy

// The tile's CSR entries and piece / row->piece slices, as 16-byte aligned
// spans, completing on the CSR barrier.  They belong to the handle (never
// written by other kernels), so this runs before the dependency wait.
__device__ void issue_csr(const B1Params &p, const TileDesc &td, unsigned char *smem) {
    const MatrixView &m = p.m;
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + kBarCsr);
    const int ka = td.k0 & ~3, kb = (td.k1 + 3) & ~3;
    const int ra = td.r0 & ~3, rb = (td.r1 + 1 + 3) & ~3;
    const int pa = td.p0 & ~3, pb = (td.p1 + 1 + 3) & ~3;
    mbar_arrive_expect_tx(bar, (uint32_t)(kb - ka) * 4 + (uint32_t)(rb - ra) * 4 + (uint32_t)(pb - pa) * 4);
    if (kb > ka) bulk_g2s(smem + p.off_csr, m.csr + ka, (uint32_t)(kb - ka) * 4, bar);
    bulk_g2s(smem + p.off_rp, p.row_piece + ra, (uint32_t)(rb - ra) * 4, bar);
    bulk_g2s(smem + p.off_pk, p.piece_k + pa, (uint32_t)(pb - pa) * 4, bar);
}

// ---------------------------------------------------------------- outliers

// f32 += f16 * f16 (the product is exact in fp32).
__device__ __forceinline__ float mfma(uint16_t a, uint16_t b, float c) {
    float d;
    asm("fma.rn.f32.f16 %0, %1, %2, %3;" : "=f"(d) : "h"(a), "h"(b), "f"(c));
    return d;
}

__device__ __forceinline__ float warp_sum(float r) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) r += __shfl_xor_sync(kFull, r, o);
    return r;
}

// v[0..NB-1] (one value per activation row) summed over the warp in one
// transposed butterfly; afterwards lane l holds the total of activation row
// bn_row<NB>(l), in a fixed order.
template <int NB>
__device__ __forceinline__ float reduce_rows(float (&v)[NB], int lane) {
    int o = 16;
#pragma unroll
    for (int n = NB; n > 1; n >>= 1, o >>= 1) {
        const bool hi = lane & o;
#pragma unroll
        for (int i = 0; i < n / 2; i++) {
            const float send = hi ? v[i] : v[i + n / 2], keep = hi ? v[i + n / 2] : v[i];
            v[i] = keep + __shfl_xor_sync(kFull, send, o);
        }
    }
#pragma unroll
    for (; o >= 1; o >>= 1) v[0] += __shfl_xor_sync(kFull, v[0], o);
    return v[0];
}
// The row whose total reduce_rows leaves in lane l: the halvings at lane
// bits 4, 3, 2 pick it, high bit first; lanes with the remaining low bits
// zero store it.
template <int NB>
__device__ __forceinline__ int bn_row(int lane) {
    return NB == 8 ? (lane >> 2) & 7 : NB == 4 ? (lane >> 3) & 3 : NB == 2 ? (lane >> 4) & 1 : 0;
}
template <int NB>
__device__ __forceinline__ bool bn_store_lane(int lane) {
    return (lane & (NB == 8 ? 3 : NB == 4 ? 7 : NB == 2 ? 15 : 31)) == 0;
}

// Thread t sums pieces t, t + blockDim, ... of the tile (each <= kPieceMax
// entries of one row) from the staged CSR entries and x.
__device__ __forceinline__ void reduce_pieces(const TileDesc &td, unsigned char *smem, const B1Params &p) {
    const uint16_t *xs = reinterpret_cast<const uint16_t *>(smem + p.off_x);
    const uint32_t *csr = reinterpret_cast<const uint32_t *>(smem + p.off_csr);
    const int32_t *pk = reinterpret_cast<const int32_t *>(smem + p.off_pk);
    float *psum = reinterpret_cast<float *>(smem + p.off_psum);
    const int ka = td.k0 & ~3, pa = td.p0 & ~3;
    for (int q = td.p0 + threadIdx.x; q < td.p1; q += blockDim.x) {
        const int kb = pk[q - pa] - ka, ke = pk[q + 1 - pa] - ka;
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
        int k = kb;
        for (; k + 3 < ke; k += 4) {
            const uint32_t e0 = csr[k], e1 = csr[k + 1], e2 = csr[k + 2], e3 = csr[k + 3];
            a0 = mfma((uint16_t)(e0 >> 16), xs[e0 & 0xffffu], a0);
            a1 = mfma((uint16_t)(e1 >> 16), xs[e1 & 0xffffu], a1);
            a2 = mfma((uint16_t)(e2 >> 16), xs[e2 & 0xffffu], a2);
            a3 = mfma((uint16_t)(e3 >> 16), xs[e3 & 0xffffu], a3);
        }
        for (; k < ke; k++) {
            const uint32_t e0 = csr[k];
            a0 = mfma((uint16_t)(e0 >> 16), xs[e0 & 0xffffu], a0);
        }
        psum[q - td.p0] = (a0 + a1) + (a2 + a3);
    }
}

// y[r] = fp16(dense_scale * r_i * sum_c part[i][c] + sum of the row's piece
// sums), in a fixed order per row (r_i = the row scale of a two-axis matrix,
// else 1).  Warp w takes rows 32w + lane, 32w + lane + 32W,
// ...: a lane sums the pieces of a row with <= kHeavyPieces of them, the
// whole warp those of a longer row.
__device__ __forceinline__ void finalize(const TileDesc &td, const unsigned char *smem, const B1Params &p,
                                         float dense_scale, __half *y) {
    const float *part = reinterpret_cast<const float *>(smem + p.off_part);
    const float *psum = reinterpret_cast<const float *>(smem + p.off_psum);
    const int32_t *rp = reinterpret_cast<const int32_t *>(smem + p.off_rp);
    const int ra = td.r0 & ~3;
    const int nrows = td.r1 - td.r0;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    for (int i0 = 32 * warp; i0 < nrows; i0 += 32 * nw) {
        const int i = i0 + lane;
        int q0 = 0, q1 = 0;
        if (i < nrows) {
            q0 = rp[td.r0 + i - ra];
            q1 = rp[td.r0 + i + 1 - ra];
        }
        const bool heavy = q1 - q0 > kHeavyPieces;
        float o = 0.f;
        if (!heavy)
            for (int q = q0; q < q1; q++) o += psum[q - td.p0];
        unsigned hm = __ballot_sync(kFull, heavy);
        while (hm) {
            const int src = __ffs(hm) - 1;
            hm &= hm - 1;
            const int h0 = __shfl_sync(kFull, q0, src), h1 = __shfl_sync(kFull, q1, src);
            float t = 0.f;
            for (int q = h0 + lane; q < h1; q += 32) t += psum[q - td.p0];
            t = warp_sum(t);
            if (lane == src) o = t;
        }
        if (i < nrows) {
            float acc = 0.f;
            for (int c = 0; c < p.C; c++) acc += part[(size_t)i * p.C + c];
            const float rs = p.m.rscale ? __half2float(__ushort_as_half(p.m.rscale[td.r0 + i])) : 1.0f;
            y[td.r0 + i] = __float2half_rn(fmaf(acc, dense_scale * rs, o));
        }
    }
}

// ---------------------------------------------------------------- row decoders

// lo += the low halves' product, hi += the high halves' (fp16 pairs p, x).
__device__ __forceinline__ void mfma_pair(float &lo, float &hi, uint32_t p, uint32_t xh) {
    asm("{\n\t.reg .f16 pl, ph, xl, xh;\n\t"
        "mov.b32 {pl, ph}, %2;\n\tmov.b32 {xl, xh}, %3;\n\t"
        "fma.rn.f32.f16 %0, pl, xl, %0;\n\tfma.rn.f32.f16 %1, ph, xh, %1;\n\t}"
        : "+f"(lo), "+f"(hi)
        : "r"(p), "r"(xh));
}

// fp16 exponent pattern of M_h = 2^(10-h) in both halves, for a code field
// at bit h = 3k of each half (1024, 128, 16).
__host__ __device__ constexpr uint32_t magic_of(int k) {
    return k == 0 ? 0x64006400u : k == 1 ? 0x58005800u : 0x4C004C00u;
}

// (a & mask) | c in one LOP3.
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t mask, uint32_t c) {
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(a), "r"(mask), "r"(c));
    return r;
}

// Both halves of a - b in fp16 (used where the difference is exact).
__device__ __forceinline__ uint32_t hsub2_bits(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// Affine 3-bit slot record v (3 code words + scale pair), zero byte zb and
// the lane's 32 columns of x as fp16 pairs xh[m] = (x[2m], x[2m+1]):
// returns scale_A * sum_A (q - zA) x + scale_B * sum_B (q - zB) x.
__device__ __forceinline__ float decode_aff3(const uint4 v, uint32_t zb, const uint32_t (&xh)[16]) {
    const uint32_t w[3] = {v.x, v.y, v.z};
    const uint32_t sh[3] = {v.x >> 10, v.y >> 10, v.z >> 10};
    const uint32_t z[2] = {zb & 15u, (zb >> 4) & 15u};
    uint32_t mz[2][3];  // M_h + zero in both halves, per group and field class
#pragma unroll
    for (int g = 0; g < 2; g++)
#pragma unroll
        for (int k = 0; k < 3; k++) mz[g][k] = z[g] * (0x00010001u << (3 * k)) + magic_of(k);
    float acc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};  // [group][low, high half]
#pragma unroll
    for (int m = 0; m < 15; m++) {  // pair m = columns 2m, 2m+1: word m/5, slot j = m%5
        const int i = m / 5, j = m % 5, k = j < 3 ? j : j - 3, g = m < 8 ? 0 : 1;
        const uint32_t pr = and_or(j < 3 ? w[i] : sh[i], 0x00070007u << (3 * k), magic_of(k));
        mfma_pair(acc[g][0], acc[g][1], hsub2_bits(pr, mz[g][k]), xh[m]);
    }
    // columns 30 (low half) and 31 (high half): bit k is bit 9 / 25 of word k
    const uint32_t t15 = ((w[0] >> 9) & 0x00010001u) | ((w[1] >> 8) & 0x00020002u) | ((w[2] >> 7) & 0x00040004u);
    mfma_pair(acc[1][0], acc[1][1], hsub2_bits(t15 | magic_of(0), mz[1][0]), xh[15]);
    const float sA = __half2float(__ushort_as_half((unsigned short)(v.w & 0xffffu)));
    const float sB = __half2float(__ushort_as_half((unsigned short)(v.w >> 16)));
    return fmaf(sB, acc[1][0] + acc[1][1], sA * (acc[0][0] + acc[0][1]));
}

// Table slot: code words w[0..BITS-1], the table entry held by the lane (a
// centroid of the row, or a level of the lane's bit-plane group).
template <int BITS>
__device__ __forceinline__ float decode_lut(const uint32_t (&w)[4], float tv, const float (&xr)[32]) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    if (BITS == 2) {
#pragma unroll
        for (int c = 0; c < 32; c++) {
            const uint32_t wd = w[c >> 4];
            const int sh = 2 * (c & 15);
            acc[c & 3] = fmaf(__shfl_sync(kFull, tv, sh ? (int)(wd >> sh) : (int)wd, 4), xr[c], acc[c & 3]);
        }
    } else if (BITS == 4) {
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
        const int q30 = (int)(((w[0] >> 9) & 1u) | ((w[1] >> 8) & 2u) | ((w[2] >> 7) & 4u));
        const int q31 = (int)(((w[0] >> 25) & 1u) | ((w[1] >> 24) & 2u) | ((w[2] >> 23) & 4u));
        acc[2] = fmaf(__shfl_sync(kFull, tv, q30, 8), xr[30], acc[2]);
        acc[3] = fmaf(__shfl_sync(kFull, tv, q31, 8), xr[31], acc[3]);
    }
    return (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

// ---------------------------------------------------------------- kernels

// Before the dependency wait: one thread sets up the barriers and starts the
// CSR staging copy.
__device__ __forceinline__ void begin(const B1Params &p, const TileDesc &td, unsigned char *smem) {
    if (threadIdx.x == 0) {
        mbar_init(reinterpret_cast<uint64_t *>(smem + kBarCsr), 1);
        mbar_init(reinterpret_cast<uint64_t *>(smem + kBarX), p.C);  // one arrival per column warp
        fence_mbar_init();
        issue_csr(p, td, smem);
    }
    __syncthreads();
}

// The warps of row group 0 cover every slot: they stage x (with its zero
// tail) in shared memory for the outlier pass and arrive on its barrier.
__device__ __forceinline__ void stage_x(unsigned char *smem, const B1Params &p, int s, const uint32_t (&xh)[16]) {
    if (s < p.m.slots) {
        uint4 *dst = reinterpret_cast<uint4 *>(smem + p.off_x + 64 * s);
#pragma unroll
        for (int k = 0; k < 4; k++) dst[k] = make_uint4(xh[4 * k], xh[4 * k + 1], xh[4 * k + 2], xh[4 * k + 3]);
    }
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(reinterpret_cast<uint64_t *>(smem + kBarX));
}

// Wait (warp-wide, bounded) for a staged copy; a timeout is reported.
__device__ __forceinline__ bool wait_stage(unsigned char *smem, int bar, const B1Params &p) {
    if (mbar_wait_warp(reinterpret_cast<uint64_t *>(smem + bar), 0)) return true;
    if ((threadIdx.x & 31) == 0) report(p.status, kStatusTimeout);
    return false;
}

// This lane's 32 columns of x (slot s) as 16 fp16 pairs, straight from
// global memory through the read-only path (x is not written while the
// kernel runs; the row-group warps of an SM share its lines in L1); columns
// past N read 0.
__device__ __forceinline__ void x_pairs(const __half *x, int s, int cols, uint32_t (&xh)[16]) {
#pragma unroll
    for (int k = 0; k < 4; k++) {
        uint4 q = make_uint4(0u, 0u, 0u, 0u);
        if (s * 32 + 8 * k < cols) q = __ldg(reinterpret_cast<const uint4 *>(x + (size_t)s * 32) + k);
        xh[4 * k] = q.x;
        xh[4 * k + 1] = q.y;
        xh[4 * k + 2] = q.z;
        xh[4 * k + 3] = q.w;
    }
}

// Calls f(std::integral_constant<int, D>) for D = B .. E-1 (compile-time stage indices).
template <int B, int E, typename F>
__device__ __forceinline__ void unroll(F &&f) {
    if constexpr (B < E) {
        f(std::integral_constant<int, B>{});
        unroll<B + 1, E>(f);
    }
}

// Affine 3-bit: ring stage of one warp = the 32 slot records of its group
// (512 bytes) + the group's 32 zero bytes.
constexpr int kAffStageB = 544;

// One row of this lane's ring: its slot record (all lanes; source lb + 32)
// and, on lanes 0 and 1, half of the group's zero bytes (source lb), into
// stage OFF; predicated on `more`.  One commit group.  (Per-lane copies on
// the L1 path measured faster here than one bulk copy per warp and row.)
template <int OFF>
__device__ __forceinline__ void copy_row(uint32_t rs, uint32_t rz, const unsigned char *lb, int more, int zl) {
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.b32 p, %2, 0;\n\t"
        "setp.ne.and.b32 q, %3, 0, p;\n\t"
        "@p cp.async.cg.shared.global [%0+%5], [%1+32], 16;\n\t"
        "@q cp.async.cg.shared.global [%4+%5], [%1], 16;\n\t"
        "cp.async.commit_group;\n\t}" ::"r"(rs),
        "l"(lb), "r"(more), "r"(zl), "r"(rz), "n"(OFF)
        : "memory");
}

template <int OFF>
__device__ __forceinline__ void read_row(uint32_t rs, uint32_t rb, uint4 &v, uint32_t &zb) {
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4+%5];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(rs), "n"(OFF));
    asm volatile("ld.shared.u8 %0, [%1+%2];" : "=r"(zb) : "r"(rb), "n"(OFF + 512));
}

// Affine 3-bit rows.  The lanes of warp (rg, cw) stream group cw of rows
// r0 + rg, r0 + rg + R, ...: each lane copies its slot's 16-byte record and
// lanes 0, 1 the group's zero bytes, kD rows ahead, into the warp's ring
// (cp.async, one commit group per row); each lane reads back its record and
// zero byte.  A lane's wait covers only its own copies, so a warp barrier
// follows each wait before the zero bytes are read.  Rows go kRB at a time:
// each lane decodes its slot of kRB rows, one transposed butterfly sums the
// kRB partials over the warp (4 rows: 7 shuffles instead of 20), and the
// stages are refilled after it, when every lane has read them.
template <int NT, int PER_SM>
__global__ void __launch_bounds__(NT, PER_SM)
b1_aff3_kernel(B1Params p, const __half *__restrict__ x, __half *__restrict__ y) {
    static_assert(kD % kRB == 0, "ring depth");
    extern __shared__ __align__(128) unsigned char smem[];
    const MatrixView &m = p.m;
    const int S = m.slots, C = p.C, R = p.R;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const TileDesc td = p.tiles[blockIdx.x];
    const int nrows = td.r1 - td.r0;
    const int cw = warp % C, rg = warp / C;
    const int s = cw * 32 + lane;
    const int nslot = min(32, S - 32 * cw);  // slots in this warp's group
    const int nj = rg < nrows ? (nrows - rg + R - 1) / R : 0;  // rows of this warp
    const size_t step = (size_t)R * m.row_words * 4;            // bytes between this warp's rows
    // lanes past the group's last slot copy that slot again (same sectors); their x is 0
    const unsigned char *lb = reinterpret_cast<const unsigned char *>(m.dense) +
                              ((size_t)td.r0 + rg) * m.row_words * 4 + 4 * kAff3GroupWords * cw +
                              16 * min(lane, nslot - 1);
    const int zl = lane < 2;
    const uint32_t ring = smem_u32(smem + p.off_ring + (size_t)warp * kD * kAffStageB);
    const uint32_t rs = ring + 16 * lane, rz = ring + 512 + 16 * lane, rb = ring + lane;
    begin(p, td, smem);
    unroll<0, kPre>([&](auto dc) {
        constexpr int d = decltype(dc)::value;
        copy_row<d * kAffStageB>(rs, rz, lb, d < nj, zl);
        lb += step;
    });

    // x (and y) belong to the surrounding program: wait for the previous
    // kernel in the stream before touching them.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    {
        uint32_t xh[16];
        x_pairs(x, s, m.cols, xh);  // requested ahead of the rest of the ring
        unroll<kPre, kD>([&](auto dc) {
            constexpr int d = decltype(dc)::value;
            copy_row<d * kAffStageB>(rs, rz, lb, d < nj, zl);
            lb += step;
        });
        if (rg == 0) stage_x(smem, p, s, xh);

        // partial of this warp's row jj at part + jj * pstep
        const uint32_t part = smem_u32(smem + p.off_part) + 4 * (rg * C + cw);
        const uint32_t pstep = 4 * R * C;
        const int my_row = bn_row<kRB>(lane);
        const bool stores = bn_store_lane<kRB>(lane);
        int j = 0;
        for (; j + kD <= nj; j += kD) {
            unroll<0, kD / kRB>([&](auto ec) {
                constexpr int e = decltype(ec)::value;
                cp_async_wait<kD - kRB>();  // this lane's copies of rows j + kRB e .. have landed ...
                __syncwarp();               // ... and every lane's (lanes 0, 1 copy the zero bytes)
                float v[kRB];
                unroll<0, kRB>([&](auto rc) {
                    constexpr int d = kRB * e + decltype(rc)::value;
                    uint4 rec;
                    uint32_t zb;
                    read_row<d * kAffStageB>(rs, rb, rec, zb);
                    v[decltype(rc)::value] = decode_aff3(rec, zb, xh);
                });
                const float t = reduce_rows<kRB>(v, lane);
                if (stores)
                    asm volatile("st.shared.f32 [%0], %1;" ::"r"(part + (j + kRB * e + my_row) * pstep), "f"(t)
                                 : "memory");
                // every lane has read the stages before they are refilled: lane 0's
                // shuffles above waited for every lane's, which consumed its loads
                unroll<0, kRB>([&](auto rc) {
                    constexpr int d = kRB * e + decltype(rc)::value;
                    copy_row<d * kAffStageB>(rs, rz, lb, j + d + kD < nj, zl);
                    lb += step;
                });
            });
        }
        cp_async_wait<0>();
        __syncwarp();
        // the last nj - j < kD rows, all landed: kRB at a time, missing rows as 0
        for (int d0 = 0; j + d0 < nj; d0 += kRB) {
            float v[kRB];
#pragma unroll
            for (int r = 0; r < kRB; r++) {
                v[r] = 0.f;
                if (j + d0 + r < nj) {
                    uint4 rec;
                    uint32_t zb;
                    read_row<0>(rs + (d0 + r) * kAffStageB, rb + (d0 + r) * kAffStageB, rec, zb);
                    v[r] = decode_aff3(rec, zb, xh);
                }
            }
            const float t = reduce_rows<kRB>(v, lane);
            if (stores && j + d0 + my_row < nj)
                asm volatile("st.shared.f32 [%0], %1;" ::"r"(part + (j + d0 + my_row) * pstep), "f"(t) : "memory");
        }
    }
    // the outliers, from the staged CSR entries and x
    if (wait_stage(smem, kBarX, p) && wait_stage(smem, kBarCsr, p)) reduce_pieces(td, smem, p);
    __syncthreads();
    finalize(td, smem, p, 1.0f, y);
}

// Table lookup by shfl.idx over 2^BITS-lane segments.  Row tables (GT
// false): every segment holds the row's 2^BITS centroids.  Bit-plane groups
// (GT true): a group spans 2^BITS slots, i.e. exactly one segment, whose lanes
// hold that group's 2^BITS levels -- the lane of slot s holds level s % 2^BITS
// of group s / 2^BITS -- so the same lookup reads the lane's own group.
template <int BITS, bool GT>
__global__ void __launch_bounds__(kThreads, 1)
b1_lut_kernel(B1Params p, const __half *__restrict__ x, __half *__restrict__ y) {
    constexpr int K = 1 << BITS;
    constexpr int NW = BITS;  // 32-bit code words per slot and row
    extern __shared__ __align__(128) unsigned char smem[];
    const MatrixView &m = p.m;
    const int S = m.slots, C = p.C, R = p.R;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const TileDesc td = p.tiles[blockIdx.x];
    const int nrows = td.r1 - td.r0;
    const int cw = warp % C, rg = warp / C;
    const int s = cw * 32 + lane;
    const bool valid = s < S;

    // Per-lane asynchronous copy pipeline: each lane copies its own slot's
    // code words (and the word holding its row's centroid) for the rows
    // kDepth ahead into this warp's ring, and later reads back exactly what
    // it copied -- no barrier, only cp.async.wait_group.
    const uint32_t ring = smem_u32(smem + p.off_ring + (size_t)warp * kDepth * kStageB);
    const uint32_t ring_s = ring + 16 * lane, ring_a = ring + 512 + 4 * lane;
    const size_t row_step = (size_t)R * m.row_words * 4;
    const unsigned char *rec = reinterpret_cast<const unsigned char *>(m.dense) +
                               ((size_t)td.r0 + rg) * m.row_words * 4;
    const int te = GT ? min(s, S - 1) : (lane & (K - 1));  // this lane's entry of the row's table
    const unsigned char *tabp = reinterpret_cast<const unsigned char *>(m.table) +
                                ((size_t)(td.r0 + rg) * (GT ? S : K) + te) * 2 - 2 * (te & 1);
    const size_t tab_step = (size_t)R * (GT ? S : K) * 2;
    const int nj = rg < nrows ? (nrows - rg + R - 1) / R : 0;
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
            }
            // the 4-byte word holding this lane's entry (table rows are 4-byte aligned)
            cp_async4(sa, tabp);
            rec += row_step;
            tabp += tab_step;
        }
        issued++;
        cp_async_commit();
    };
    begin(p, td, smem);
#pragma unroll
    for (int d = 0; d < kDepth; d++) issue(d);

    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    {
        float xr[32];
        {
            uint32_t xh[16];
            x_pairs(x, s, m.cols, xh);
#pragma unroll
            for (int i = 0; i < 16; i++) {
                const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&xh[i]));
                xr[2 * i] = f.x;
                xr[2 * i + 1] = f.y;
            }
            if (m.cscale) {
                // two-axis: the dense part sees c_j x_j, exact in fp32; the
                // outliers keep the staged, unscaled x
                uint32_t ch[16];
                x_pairs(reinterpret_cast<const __half *>(m.cscale), s, m.cols, ch);
#pragma unroll
                for (int i = 0; i < 16; i++) {
                    const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&ch[i]));
                    xr[2 * i] *= f.x;
                    xr[2 * i + 1] *= f.y;
                }
            }
            if (rg == 0) stage_x(smem, p, s, xh);
        }
        float *part = reinterpret_cast<float *>(smem + p.off_part);
        int i = rg;
        for (int j = 0; j < nj; j++, i += R) {
            const int d = j & (kDepth - 1);
            cp_async_wait<kDepth - 1>();  // this lane's copies for row j have landed
            const uint32_t st = ring_s + d * kStageB, sa = ring_a + d * kStageB;
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
            const float tv = __half2float(__ushort_as_half((unsigned short)(lds32(sa) >> (16 * (te & 1)))));
            float r = decode_lut<BITS>(w4, tv, xr);
            r = warp_sum(r);
            if (lane == 0) part[(size_t)i * C + cw] = r;
            issue(d);  // refill this stage (its data has been consumed)
        }
        cp_async_wait<0>();
    }
    if (wait_stage(smem, kBarX, p) && wait_stage(smem, kBarCsr, p)) reduce_pieces(td, smem, p);
    __syncthreads();
    finalize(td, smem, p, 1.0f, y);
}

// ---------------------------------------------------------------- small batches

constexpr int kMaxWarpsN = 12;  // batched table kernel: fewer warps, room for x of 4 rows in registers
constexpr int kThreadsN = kMaxWarpsN * 32;

// Table rows, NB activation rows at once (NB = 2 or 4; nb <= NB real).
// As the batch-1 table kernel, but each lane keeps its 32 columns of x for
// every activation row as fp16 pairs, looks each weight up once (shfl.idx,
// fp16 centroid) and adds weight * x for every row with mixed-precision
// FMAs.  Outliers: one lane per piece after the dense loop, x read from L2.
template <int BITS, bool GT, int NB>
__global__ void __launch_bounds__(kThreadsN, 1)
bn_lut_kernel(B1Params p, const __half *__restrict__ x, __half *__restrict__ y, int nb) {
    constexpr int K = 1 << BITS;
    constexpr int NW = BITS;
    extern __shared__ __align__(128) unsigned char smem[];
    const MatrixView &m = p.m;
    const int S = m.slots, C = p.C, R = p.R, N = m.cols;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const TileDesc td = p.tiles[blockIdx.x];
    const int nrows = td.r1 - td.r0;
    const int cw = warp % C, rg = warp / C;
    const int s = cw * 32 + lane;
    const bool valid = s < S;

    const uint32_t ring = smem_u32(smem + p.off_ring + (size_t)warp * kDepth * kStageB);
    const uint32_t ring_s = ring + 16 * lane, ring_a = ring + 512 + 4 * lane;
    const size_t row_step = (size_t)R * m.row_words * 4;
    const unsigned char *rec = reinterpret_cast<const unsigned char *>(m.dense) +
                               ((size_t)td.r0 + rg) * m.row_words * 4;
    const int te = GT ? min(s, S - 1) : (lane & (K - 1));  // as in b1_lut_kernel
    const unsigned char *tabp = reinterpret_cast<const unsigned char *>(m.table) +
                                ((size_t)(td.r0 + rg) * (GT ? S : K) + te) * 2 - 2 * (te & 1);
    const size_t tab_step = (size_t)R * (GT ? S : K) * 2;
    const int nj = rg < nrows ? (nrows - rg + R - 1) / R : 0;
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
            }
            cp_async4(sa, tabp);
            rec += row_step;
            tabp += tab_step;
        }
        issued++;
        cp_async_commit();
    };
    if (threadIdx.x == 0) {
        mbar_init(reinterpret_cast<uint64_t *>(smem + kBarCsr), 1);
        fence_mbar_init();
        issue_csr(p, td, smem);
    }
    __syncthreads();
#pragma unroll
    for (int d = 0; d < kDepth; d++) issue(d);

    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    // x of every activation row: this lane's 32 columns as fp16 pairs (rows past nb read 0)
    uint32_t xh[NB][16];
#pragma unroll
    for (int b = 0; b < NB; b++) {
        if (b < nb) {
            x_pairs(x + (size_t)b * N, s, N, xh[b]);
        } else {
#pragma unroll
            for (int i = 0; i < 16; i++) xh[b][i] = 0u;
        }
    }
    float *part = reinterpret_cast<float *>(smem + p.off_part);  // [row][C][NB]
    int i = rg;
    for (int j = 0; j < nj; j++, i += R) {
        const int d = j & (kDepth - 1);
        cp_async_wait<kDepth - 1>();
        const uint32_t st = ring_s + d * kStageB, sa = ring_a + d * kStageB;
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
        // this lane's table entry as fp16 bits (the word holds two entries)
        const uint32_t tv = (lds32(sa) >> (16 * (te & 1))) & 0xffffu;
        float lo[NB], hi[NB];
#pragma unroll
        for (int b = 0; b < NB; b++) lo[b] = hi[b] = 0.f;
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
            int q0, q1;
            if (BITS == 2) {
                q0 = (int)(w4[c >> 4] >> (2 * (c & 15)));
                q1 = (int)(w4[c >> 4] >> (2 * ((c + 1) & 15)));
            } else if (BITS == 4) {
                q0 = (int)(w4[c >> 3] >> (4 * (c & 7)));
                q1 = (int)(w4[c >> 3] >> (4 * ((c + 1) & 7)));
            } else if (c < 30) {
                q0 = (int)(w4[c / 10] >> raw_pos3(c));
                q1 = (int)(w4[(c + 1) / 10] >> raw_pos3(c + 1));
            } else {
                q0 = (int)(((w4[0] >> 9) & 1u) | ((w4[1] >> 8) & 2u) | ((w4[2] >> 7) & 4u));
                q1 = (int)(((w4[0] >> 25) & 1u) | ((w4[1] >> 24) & 2u) | ((w4[2] >> 23) & 4u));
            }
            // shfl.idx over a 2^b-lane segment reads only the low b bits of the index
            const uint32_t w0 = __shfl_sync(kFull, tv, q0, K), w1 = __shfl_sync(kFull, tv, q1, K);
            const uint32_t wp = w0 | (w1 << 16);  // fp16 pair (column c, c + 1)
#pragma unroll
            for (int b = 0; b < NB; b++) mfma_pair(lo[b], hi[b], wp, xh[b][c >> 1]);
        }
        float v[NB];
#pragma unroll
        for (int b = 0; b < NB; b++) v[b] = lo[b] + hi[b];
        const float t = reduce_rows<NB>(v, lane);
        if (bn_store_lane<NB>(lane)) part[((size_t)i * C + cw) * NB + bn_row<NB>(lane)] = t;
        issue(d);
    }
    cp_async_wait<0>();

    // outliers: thread t sums pieces t, t + blockDim, ... for every activation row
    if (wait_stage(smem, kBarCsr, p)) {
        const uint32_t *csr = reinterpret_cast<const uint32_t *>(smem + p.off_csr);
        const int32_t *pk = reinterpret_cast<const int32_t *>(smem + p.off_pk);
        float *psum = reinterpret_cast<float *>(smem + p.off_psum);  // [piece][NB]
        const int ka = td.k0 & ~3, pa = td.p0 & ~3;
        for (int q = td.p0 + threadIdx.x; q < td.p1; q += blockDim.x) {
            float a[NB];
#pragma unroll
            for (int b = 0; b < NB; b++) a[b] = 0.f;
            for (int k = pk[q - pa] - ka; k < pk[q + 1 - pa] - ka; k++) {
                const uint32_t e = csr[k];
                const uint16_t v = (uint16_t)(e >> 16);
                const int col = (int)(e & 0xffffu);
#pragma unroll
                for (int b = 0; b < NB; b++)
                    if (b < nb) a[b] = mfma(v, __ldg(reinterpret_cast<const uint16_t *>(x) + (size_t)b * N + col), a[b]);
            }
#pragma unroll
            for (int b = 0; b < NB; b++) psum[(size_t)(q - td.p0) * NB + b] = a[b];
        }
    }
    __syncthreads();

    // y[b][r] = sum_c part + the row's piece sums, in a fixed order: a lane per
    // row, or the whole warp for a row with many pieces
    const float *psum = reinterpret_cast<const float *>(smem + p.off_psum);
    const int32_t *rp = reinterpret_cast<const int32_t *>(smem + p.off_rp);
    const int ra = td.r0 & ~3, nw = blockDim.x >> 5;
    for (int i0 = 32 * warp; i0 < nrows; i0 += 32 * nw) {
        const int r = i0 + lane;
        int q0 = 0, q1 = 0;
        if (r < nrows) {
            q0 = rp[td.r0 + r - ra];
            q1 = rp[td.r0 + r + 1 - ra];
        }
        const bool heavy = q1 - q0 > kHeavyPieces;
        float o[NB];
#pragma unroll
        for (int b = 0; b < NB; b++) {
            o[b] = 0.f;
            if (!heavy)
                for (int q = q0; q < q1; q++) o[b] += psum[(size_t)(q - td.p0) * NB + b];
        }
        unsigned hm = __ballot_sync(kFull, heavy);
        while (hm) {
            const int src = __ffs(hm) - 1;
            hm &= hm - 1;
            const int h0 = __shfl_sync(kFull, q0, src), h1 = __shfl_sync(kFull, q1, src);
#pragma unroll
            for (int b = 0; b < NB; b++) {
                float tsum = 0.f;
                for (int q = h0 + lane; q < h1; q += 32) tsum += psum[(size_t)(q - td.p0) * NB + b];
                tsum = warp_sum(tsum);
                if (lane == src) o[b] = tsum;
            }
        }
        if (r < nrows) {
#pragma unroll
            for (int b = 0; b < NB; b++) {
                if (b < nb) {
                    float acc = 0.f;
                    for (int c = 0; c < C; c++) acc += part[((size_t)r * C + c) * NB + b];
                    y[(size_t)b * m.rows + td.r0 + r] = __float2half_rn(acc + o[b]);
                }
            }
        }
    }
}

enum Kind { kNone = -1, kAff3 = 0, kLut3 = 3, kLut4 = 4, kBp2 = 12, kBp3 = 13 };

Kind b1_kind(const MatrixView &m, int batch) {
    if (batch != 1 || m.rows <= 0 || m.cols <= 0 || m.mode == kModeIntGrid) return kNone;
    if ((m.slots + 31) / 32 > kMaxWarps) return kNone;
    // the affine kernel multiplies fp16 x, which cannot hold c_j x_j exactly
    if (m.mode == DSQ_MODE_AFFINE_G16) return m.bits == 3 && !m.cscale ? kAff3 : kNone;
    if (m.mode == DSQ_MODE_BITPLANE) return m.bits == 2 ? kBp2 : kBp3;
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
    p.R = std::max(1, (sc.per_sm == 2 ? kWarps2 : kMaxWarps) / p.C);
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
    off = align_sz(off + (size_t)(sc.max_pieces + 1) * 4, 16);
    off = align_sz(off, 128);
    p.off_ring = (int)off;
    off += (size_t)p.C * p.R * (b1_kind(m, 1) == kAff3 ? kD * kAffStageB : kDepth * kStageB);
    if (off > (sc.per_sm == 2 ? kSmemBudget2 : kSmemBudget)) return false;
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

// Launch geometry and shared-memory map of the batched table kernel.
bool plan_bn(const dsq_handle_s *h, int NB, B1Params *out, size_t *smem_bytes) {
    const MatrixView &m = h->view;
    const Schedule &sc = h->sched;
    B1Params p;
    p.m = m;
    p.tiles = sc.tiles;
    p.row_piece = sc.row_piece;
    p.piece_k = sc.piece_k;
    p.status = h->d_status;
    p.C = (m.slots + 31) / 32;
    p.R = std::max(1, kMaxWarpsN / p.C);
    if (p.C > kMaxWarpsN) return false;
    size_t off = 128;  // mbarrier
    p.off_x = (int)off;  // unused
    p.off_csr = (int)off;
    off = align_sz(off + (size_t)(sc.max_csr + 8) * 4, 16);
    p.off_rp = (int)off;
    off = align_sz(off + (size_t)(sc.max_rows + 9) * 4, 16);
    p.off_pk = (int)off;
    off = align_sz(off + (size_t)(sc.max_pieces + 9) * 4, 16);
    p.off_part = (int)off;
    off = align_sz(off + (size_t)sc.max_rows * p.C * NB * 4, 16);
    p.off_psum = (int)off;
    off = align_sz(off + (size_t)(sc.max_pieces + 1) * NB * 4, 128);
    p.off_ring = (int)off;
    off += (size_t)p.C * p.R * kDepth * kStageB;
    if (off > kSmemBudget) return false;
    *out = p;
    *smem_bytes = off;
    return true;
}

}  // namespace

// Row tiles of about equal cost (record bytes + a per-outlier charge), about
// `target` of them, each holding at most csr_cap CSR entries unless a single
// row has more.  Host-side.
static std::vector<TileDesc> cut_tiles(const MatrixView &m, const int32_t *rp, const std::vector<int32_t> &row_piece,
                                       int target, int csr_cap) {
    const int tiles_target = std::max(1, std::min(target, m.rows));
    double total = 0;
    // Cost of a row: its record bytes plus a charge per outlier.
    auto row_cost = [&](int i) { return 4.0 * m.row_words + 4.0 * (rp[i + 1] - rp[i]) + 64.0; };
    for (int i = 0; i < m.rows; i++) total += row_cost(i);
    std::vector<TileDesc> tiles;
    int r0 = 0;
    double acc = 0, done = 0;
    for (int i = 0; i < m.rows; i++) {
        const double c = row_cost(i);
        const bool over_csr = i > r0 && rp[i + 1] - rp[r0] > csr_cap;
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
    return tiles;
}

static void tile_stats(Schedule &sc, const std::vector<TileDesc> &tiles) {
    sc.n_tiles = (int)tiles.size();
    sc.max_rows = sc.max_pieces = sc.max_csr = 0;
    for (const TileDesc &t : tiles) {
        sc.max_rows = std::max(sc.max_rows, t.r1 - t.r0);
        sc.max_pieces = std::max(sc.max_pieces, t.p1 - t.p0);
        sc.max_csr = std::max(sc.max_csr, t.k1 - t.k0);
    }
}

// The tiles and the outlier pieces of the batch-1 kernels.  Affine 3-bit
// matrices of at most kWarps2 column groups get two tiles per SM when their
// largest tile fits the two-CTA shared-memory budget, else one.
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

    std::vector<TileDesc> tiles;
    sc.per_sm = 1;
    if (b1_kind(m, 1) == kAff3 && (m.slots + 31) / 32 <= kWarps2) {
        tiles = cut_tiles(m, rp, row_piece, 2 * h->sm_count, kTileCsrCap2);
        tile_stats(sc, tiles);
        sc.per_sm = 2;
        B1Params p;
        size_t smem;
        if (!plan_b1(h, &p, &smem)) sc.per_sm = 1;
    }
    if (sc.per_sm == 1) {
        tiles = cut_tiles(m, rp, row_piece, h->sm_count, kTileCsrCap);
        tile_stats(sc, tiles);
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
    int rc = set_smem_attr(b1_aff3_kernel<kThreads, 1>);
    if (rc == DSQ_OK) rc = set_smem_attr(b1_aff3_kernel<kWarps2 * 32, 2>);
    if (rc == DSQ_OK) rc = set_smem_attr(b1_lut_kernel<3, false>);
    if (rc == DSQ_OK) rc = set_smem_attr(b1_lut_kernel<4, false>);
    if (rc == DSQ_OK) rc = set_smem_attr(b1_lut_kernel<2, true>);
    if (rc == DSQ_OK) rc = set_smem_attr(b1_lut_kernel<3, true>);
    if (rc == DSQ_OK) rc = set_smem_attr(bn_lut_kernel<3, false, 2>);
    if (rc == DSQ_OK) rc = set_smem_attr(bn_lut_kernel<3, false, 4>);
    if (rc == DSQ_OK) rc = set_smem_attr(bn_lut_kernel<4, false, 2>);
    if (rc == DSQ_OK) rc = set_smem_attr(bn_lut_kernel<4, false, 4>);
    if (rc == DSQ_OK) rc = set_smem_attr(bn_lut_kernel<2, true, 2>);
    if (rc == DSQ_OK) rc = set_smem_attr(bn_lut_kernel<2, true, 4>);
    if (rc == DSQ_OK) rc = set_smem_attr(bn_lut_kernel<3, true, 2>);
    if (rc == DSQ_OK) rc = set_smem_attr(bn_lut_kernel<3, true, 4>);
    return rc;
}

// Table matrices at batch >= 2: chunks of 4 activation rows, each one
// launch of the batched kernel (2 or 4 rows wide; 8 rows of x in registers
// left too few warps per SM and measured slower than two passes of 4).
int batched_launch_count(const dsq_handle_s *h, int batch) {
    const int n_tc = tl4_launch_count(h, batch);  // 4-bit row tables: tensor cores
    if (n_tc >= 0) return n_tc;
    B1Params p;
    size_t smem;
    const MatrixView &m = h->view;
    if (batch < 2 || m.mode == DSQ_MODE_AFFINE_G16 || m.mode == kModeIntGrid || m.cscale || m.rows <= 0 ||
        m.cols <= 0 || h->sched.n_tiles == 0 ||
        !plan_bn(h, 4, &p, &smem))
        return -1;
    return (batch + 3) / 4;
}

int launch_gemv_batched(const dsq_handle_s *h, const __half *x, __half *y, int batch, cudaStream_t st) {
    if (tl4_covers(h, batch)) return launch_gemv_tl4(h, x, y, batch, st);
    if (batched_launch_count(h, batch) < 0) return DSQ_ERR_UNSUPPORTED;
    const MatrixView &m = h->view;
    for (int b0 = 0; b0 < batch; b0 += 4) {
        const int nb = std::min(4, batch - b0);
        const int NB = nb <= 2 ? 2 : 4;
        B1Params p;
        size_t smem;
        if (!plan_bn(h, NB, &p, &smem)) return DSQ_ERR_UNSUPPORTED;
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
        const __half *xb = x + (size_t)b0 * m.cols;
        __half *yb = y + (size_t)b0 * m.rows;
        cudaError_t e;
        if (m.mode == DSQ_MODE_BITPLANE && m.bits == 2)
            e = NB == 2 ? cudaLaunchKernelEx(&cfg, bn_lut_kernel<2, true, 2>, p, xb, yb, nb)
                        : cudaLaunchKernelEx(&cfg, bn_lut_kernel<2, true, 4>, p, xb, yb, nb);
        else if (m.mode == DSQ_MODE_BITPLANE)
            e = NB == 2 ? cudaLaunchKernelEx(&cfg, bn_lut_kernel<3, true, 2>, p, xb, yb, nb)
                        : cudaLaunchKernelEx(&cfg, bn_lut_kernel<3, true, 4>, p, xb, yb, nb);
        else if (m.bits == 3)
            e = NB == 2 ? cudaLaunchKernelEx(&cfg, bn_lut_kernel<3, false, 2>, p, xb, yb, nb)
                        : cudaLaunchKernelEx(&cfg, bn_lut_kernel<3, false, 4>, p, xb, yb, nb);
        else
            e = NB == 2 ? cudaLaunchKernelEx(&cfg, bn_lut_kernel<4, false, 2>, p, xb, yb, nb)
                        : cudaLaunchKernelEx(&cfg, bn_lut_kernel<4, false, 4>, p, xb, yb, nb);
        if (e != cudaSuccess) return DSQ_ERR_CUDA;
    }
    return DSQ_OK;
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
        case kAff3:
            e = h->sched.per_sm == 2 ? cudaLaunchKernelEx(&cfg, b1_aff3_kernel<kWarps2 * 32, 2>, p, x, y)
                                     : cudaLaunchKernelEx(&cfg, b1_aff3_kernel<kThreads, 1>, p, x, y);
            break;
        case kLut3: e = cudaLaunchKernelEx(&cfg, b1_lut_kernel<3, false>, p, x, y); break;
        case kBp2: e = cudaLaunchKernelEx(&cfg, b1_lut_kernel<2, true>, p, x, y); break;
        case kBp3: e = cudaLaunchKernelEx(&cfg, b1_lut_kernel<3, true>, p, x, y); break;
        default: e = cudaLaunchKernelEx(&cfg, b1_lut_kernel<4, false>, p, x, y); break;
    }
    return e == cudaSuccess ? DSQ_OK : DSQ_ERR_CUDA;
}

}  // namespace dsq
