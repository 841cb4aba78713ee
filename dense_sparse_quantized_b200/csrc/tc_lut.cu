// tc_lut.cu -- row-table matrices with 4-bit codes (one fp16 table of 16
// centroids per output row, SqueezeLLM page, "Sensitivity-based non-uniform
// quantization") at 2 or more activation rows: the centroids are looked up
// straight into the A fragments of warp-level tensor-core MMAs (mma.sync
// m16n8k16, fp16 x fp16 -> fp32), x of up to 8 activation rows forming the
// B operand (more rows: one launch per 8).
//
// The lookup stays in registers.  Each thread keeps the 16 centroids of its
// two fragment rows as a low-byte plane and a high-byte plane (four words
// each), and looks four codes up at once with byte permutes: the low 16 bits
// of a code word are four 4-bit codes, i.e. four byte selectors; two permutes
// over the planes' halves and a third that picks by each code's top bit give
// the four low bytes, the same for the high bytes, and two more interleave
// them into fp16 pairs (about 2.9 instructions per weight, no table reads).
// The MMA's k order inside a slot is free as long as A and B agree: thread t
// (c = t%4) takes columns 8c..8c+7 of every slot -- code word c of the slot,
// and one 16-byte load of x -- columns 8c..8c+3 as k-slots 2c, 2c+1, 2c+8,
// 2c+9 of the first MMA and 8c+4..8c+7 of the second.
//
// One CTA per 16-row tile; its 16 warps split the tile's K steps (a step =
// two slots = 64 columns) round robin.  Each warp streams its steps' code
// records (16 rows x 32 bytes) through a per-warp cp.async ring, reads its x
// fragments with 16-byte loads one step ahead (x is small and every tile
// reads it: L2/L1), and keeps its 16 x 8 partial tile in registers.  The
// tile's outliers go by warp pieces (up to 128 consecutive entries of one
// row, one entry per lane, so a dense run of columns reads x coalesced), a
// round of 256 pieces at a time: the first round before the dense loop
// (warps without a piece start streaming at once, so the pieces' load
// latency hides behind the loop), the rest after it; each round is folded
// into the row sums in piece order.  y = the 16 warps' partials in warp
// order plus the outlier sum: a fixed order, one fp16 store.
//
// Measured on c3 (4096 x 11008, 0.5% Zipf outliers): 44.8 us at 8 activation
// rows against 59.8 us for two launches of the 4-row shuffle kernel, but
// 29.7 / 34.7 us at 2 / 4 rows against 25.2 / 30.3 us, so the product takes
// this kernel from 5 activation rows on.  What bounds it: the byte permutes
// of the lookup load the ALU pipe (half rate), and the SMs holding two tiles
// (or a tile with the matrix's densest outlier rows) set the time.
#include "internal.h"
#include "ptx.h"

namespace dsq {

namespace {

constexpr int kTW = 16;                    // warps per CTA = rows per tile = K split of the tile
constexpr int kTThreads = kTW * 32;
constexpr int kTDepth = 8;                 // ring stages per warp
constexpr int kTStageB = 16 * 32;          // 16 rows x 2 slots x 16 bytes
constexpr int kTRingB = kTW * kTDepth * kTStageB;
constexpr int kRound = 256;                // warp pieces per round of piece sums
constexpr size_t kTSmem = (size_t)kTRingB + (size_t)kRound * 8 * 4 + (size_t)kTW * 16 * 8 * 4 + 16 * 8 * 4 + 32 * 4;
static_assert((kTSmem + 1024) * 2 <= 228 * 1024, "two CTAs per SM");

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The centroids of one row as byte planes: L[i] holds the low bytes of
// entries 4i..4i+3, H[i] their high bytes (zeros for a row past the matrix).
__device__ __forceinline__ void load_planes(const uint16_t *table, int row, bool ok, uint32_t (&L)[4],
                                            uint32_t (&H)[4]) {
    uint4 u0 = make_uint4(0u, 0u, 0u, 0u), u1 = u0;
    if (ok) {
        const uint4 *t = reinterpret_cast<const uint4 *>(table + (size_t)row * 16);
        u0 = __ldg(t);
        u1 = __ldg(t + 1);
    }
    const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
    for (int i = 0; i < 4; i++) {
        L[i] = __byte_perm(w[2 * i], w[2 * i + 1], 0x6420u);
        H[i] = __byte_perm(w[2 * i], w[2 * i + 1], 0x7531u);
    }
}

// The four 4-bit codes in the low 16 bits of v, looked up: fp16 pairs
// (T[n0], T[n1]) and (T[n2], T[n3]).
__device__ __forceinline__ void lut4(uint32_t v, const uint32_t (&L)[4], const uint32_t (&H)[4], uint32_t &p01,
                                     uint32_t &p23) {
    const uint32_t sel = v & 0x7777u;                       // entry mod 8 of each code
    const uint32_t pick = ((v >> 1) & 0x4444u) | 0x3210u;  // byte i of the upper half when code i >= 8
    const uint32_t lo = __byte_perm(__byte_perm(L[0], L[1], sel), __byte_perm(L[2], L[3], sel), pick);
    const uint32_t hi = __byte_perm(__byte_perm(H[0], H[1], sel), __byte_perm(H[2], H[3], sel), pick);
    p01 = __byte_perm(lo, hi, 0x5140u);
    p23 = __byte_perm(lo, hi, 0x7362u);
}

// Warp pieces: runs of up to kWP consecutive CSR entries of one row, lane l
// taking entries l, l + 32, l + 64, l + 96 (a dense run of columns reads x
// coalesced); the 32 lanes' sums meet in a fixed shuffle tree.
constexpr int kWP = 128;

// The tile's rows as warp pieces, computed by every warp on its own: lane r
// (< 16) holds row r's first entry, its entry count and the exclusive start
// of its pieces; returns the tile's piece count.
struct TilePieces {
    int start, count, first;
};
__device__ __forceinline__ int tile_pieces(const MatrixView &m, int r0, int nrows, int lane, TilePieces &tp) {
    tp.start = 0;
    tp.count = 0;
    if (lane < nrows) {
        tp.start = m.row_ptr[r0 + lane];
        tp.count = m.row_ptr[r0 + lane + 1] - tp.start;
    }
    const int np = (tp.count + kWP - 1) / kWP;
    int incl = np;
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    tp.first = incl - np;
    return __shfl_sync(0xffffffffu, incl, 15);
}

// Warp piece q of the tile (warp-uniform q): sum over its entries of v * x[b][col]
// for every activation row, returned to every lane.  Also returns its row.
__device__ __forceinline__ int warp_piece(const MatrixView &m, const TilePieces &tp, int q, int lane,
                                          const __half *__restrict__ x, int nb, float (&a)[8]) {
    const unsigned short *xs = reinterpret_cast<const unsigned short *>(x);
    const int N = m.cols;
    // the row: the last lane whose first piece is <= q
    const unsigned le = __ballot_sync(0xffffffffu, lane < 16 && tp.first <= q && tp.count > 0);
    const int r = 31 - __clz(le);
    const int start = __shfl_sync(0xffffffffu, tp.start, r), count = __shfl_sync(0xffffffffu, tp.count, r);
    const int first = __shfl_sync(0xffffffffu, tp.first, r);
    const int k0 = start + (q - first) * kWP, k1 = min(k0 + kWP, start + count);
    uint32_t e[4];
    float v[4];
#pragma unroll
    for (int u = 0; u < 4; u++) {
        const int k = k0 + lane + 32 * u;
        e[u] = k < k1 ? __ldg(m.csr + k) : 0u;
        v[u] = __half2float(__ushort_as_half((unsigned short)(e[u] >> 16)));
    }
#pragma unroll
    for (int b = 0; b < 8; b++) {
        a[b] = 0.f;
        if (b < nb) {
            float xv[4];
#pragma unroll
            for (int u = 0; u < 4; u++) xv[u] = __half2float(__ushort_as_half(__ldg(xs + (size_t)b * N + (e[u] & 0xffffu))));
#pragma unroll
            for (int u = 0; u < 4; u++)
                if (k0 + lane + 32 * u < k1) a[b] = fmaf(v[u], xv[u], a[b]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) a[b] += __shfl_xor_sync(0xffffffffu, a[b], o);
        }
    }
    return r;
}

// x fragments of step `step` for activation row g: per slot of the step,
// columns 8c..8c+7 in one 16-byte load (zeros past nb or past the last column)
__device__ __forceinline__ void load_xf(const __half *__restrict__ x, int N, int nb, int g, int c, int step,
                                        uint4 (&xf)[2]) {
#pragma unroll
    for (int sl = 0; sl < 2; sl++) {
        const int col = 64 * step + 32 * sl + 8 * c;
        xf[sl] = g < nb && col < N ? __ldg(reinterpret_cast<const uint4 *>(x + (size_t)g * N + col))
                                   : make_uint4(0u, 0u, 0u, 0u);
    }
}

__global__ void __launch_bounds__(kTThreads, 2)
tl4_kernel(MatrixView m, const __half *__restrict__ x, __half *__restrict__ y, int nb) {
    extern __shared__ __align__(128) unsigned char smem[];
    unsigned char *ring = smem;
    float *psum = reinterpret_cast<float *>(ring + kTRingB);          // [piece of the round][8]
    float *red = psum + kRound * 8;                                   // [warp][16 rows][8]
    float *osum = red + kTW * 16 * 8;                                 // [16 rows][8]
    int *pfirst = reinterpret_cast<int *>(osum + 16 * 8);             // [16] first piece, [16] piece count
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int M = m.rows, N = m.cols, S = m.slots;
    const int r0 = blockIdx.x * 16, nrows = min(16, M - r0);
    const int nsteps = (S + 1) >> 1;

    // ring producer: lane l copies slot 2*step + (l & 1) of tile row l >> 1
    const int crow = lane >> 1, cslot = lane & 1;
    const bool crow_ok = crow < nrows;
    const unsigned char *rec =
        reinterpret_cast<const unsigned char *>(m.dense) + (size_t)(r0 + (crow_ok ? crow : 0)) * m.row_words * 4;
    const uint32_t ring_w = smem_u32(ring) + warp * kTDepth * kTStageB;
    const uint32_t dst = ring_w + crow * 32 + cslot * 16;
    int next_step = warp;
    auto issue = [&](int d) {
        if (next_step < nsteps) {
            const int s = 2 * next_step + cslot;
            if (crow_ok && s < S) cp_async16(dst + d * kTStageB, rec + 16 * (size_t)s);
        }
        next_step += kTW;
        cp_async_commit();
    };
#pragma unroll
    for (int d = 0; d < kTDepth; d++) issue(d);

    // the centroids of this thread's fragment rows g and g + 8, as byte planes
    const int g = lane >> 2, c = lane & 3;
    uint32_t Lg[4], Hg[4], L8[4], H8[4];
    load_planes(m.table, r0 + g, g < nrows, Lg, Hg);
    load_planes(m.table, r0 + g + 8, g + 8 < nrows, L8, H8);

    // x is written by the previous kernel in the stream: wait for it here
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    // the first round of outlier pieces, before the dense loop: warps with no
    // piece go straight on, so the pieces' load latency overlaps the loop
    TilePieces tp;
    const int npieces = tile_pieces(m, r0, nrows, lane, tp);
    for (int q = warp; q < min(npieces, kRound); q += kTW) {
        float a[8];
        warp_piece(m, tp, q, lane, x, nb, a);
#pragma unroll
        for (int b = 0; b < 8; b++)
            if (lane == b) psum[(size_t)q * 8 + b] = a[b];
    }

    const uint32_t rg = ring_w + g * 32 + 4 * c, rg8 = ring_w + (g + 8) * 32 + 4 * c;  // code word c
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    uint4 xf[2];
    if (warp < nsteps) load_xf(x, N, nb, g, c, warp, xf);
    int j = 0;
    for (int step = warp; step < nsteps; step += kTW, j++) {
        const int d = j % kTDepth;
        uint4 xn[2];  // the next step's fragments, loaded a step ahead
        if (step + kTW < nsteps) load_xf(x, N, nb, g, c, step + kTW, xn);
        cp_async_wait<kTDepth - 1>();
        __syncwarp();  // every lane's copies of this stage are visible to the warp
        const uint32_t so = d * kTStageB;
        const uint32_t wg[2] = {lds32(rg + so), lds32(rg + so + 16)};
        const uint32_t w8[2] = {lds32(rg8 + so), lds32(rg8 + so + 16)};
        __syncwarp();  // the stage is read: refill it
        issue(d);
#pragma unroll
        for (int sl = 0; sl < 2; sl++) {
            const int s0 = 64 * step + 32 * sl;  // first column of the slot
            if (s0 >= N) continue;              // warp-uniform: past the last slot
            uint32_t ag[4], a8[4];
            lut4(wg[sl], Lg, Hg, ag[0], ag[1]);
            lut4(wg[sl] >> 16, Lg, Hg, ag[2], ag[3]);
            lut4(w8[sl], L8, H8, a8[0], a8[1]);
            lut4(w8[sl] >> 16, L8, H8, a8[2], a8[3]);
            if (s0 + 32 > N) {  // tail slot of 16 columns: no weight past the last column
                if (s0 + 8 * c >= N) {
#pragma unroll
                    for (int i = 0; i < 4; i++) ag[i] = a8[i] = 0u;
                }
            }
            mma16816(acc, ag[0], a8[0], ag[1], a8[1], xf[sl].x, xf[sl].y);
            mma16816(acc, ag[2], a8[2], ag[3], a8[3], xf[sl].z, xf[sl].w);
        }
        xf[0] = xn[0];
        xf[1] = xn[1];
    }
    cp_async_wait<0>();
    // D fragment: acc[0..1] = row g, activation rows 2c, 2c + 1; acc[2..3] = row g + 8
    float *rw = red + (size_t)warp * 16 * 8;
    rw[g * 8 + 2 * c] = acc[0];
    rw[g * 8 + 2 * c + 1] = acc[1];
    rw[(g + 8) * 8 + 2 * c] = acc[2];
    rw[(g + 8) * 8 + 2 * c + 1] = acc[3];
    if (threadIdx.x < 16 * 8) osum[threadIdx.x] = 0.f;
    if (warp == 0 && lane < 16) {
        pfirst[lane] = tp.first;
        pfirst[16 + lane] = (tp.count + kWP - 1) / kWP;
    }
    __syncthreads();

    // fold every round's piece sums into the row sums, in piece order; rounds
    // after the first (tiles with more than kRound pieces) are summed here
    for (int base = 0; base < npieces; base += kRound) {
        if (base != 0) {
            for (int q = base + warp; q < min(npieces, base + kRound); q += kTW) {
                float a[8];
                warp_piece(m, tp, q, lane, x, nb, a);
#pragma unroll
                for (int b = 0; b < 8; b++)
                    if (lane == b) psum[(size_t)(q - base) * 8 + b] = a[b];
            }
            __syncthreads();
        }
        if (threadIdx.x < 16 * 8) {
            const int r = threadIdx.x >> 3, b = threadIdx.x & 7;
            if (r < nrows) {
                const int qa = max(pfirst[r], base), qb = min(pfirst[r] + pfirst[16 + r], base + kRound);
                float o = osum[threadIdx.x];
                for (int qq = qa; qq < qb; qq++) o += psum[(size_t)(qq - base) * 8 + b];
                osum[threadIdx.x] = o;
            }
        }
        __syncthreads();
    }

    if (threadIdx.x < 16 * 8) {
        const int r = threadIdx.x >> 3, b = threadIdx.x & 7;
        if (r < nrows && b < nb) {
            float sum = 0.f;
            for (int w = 0; w < kTW; w++) sum += red[((size_t)w * 16 + r) * 8 + b];
            y[(size_t)b * M + r0 + r] = __float2half_rn(sum + osum[threadIdx.x]);
        }
    }
}

int launch_tl4(const dsq_handle_s *h, const __half *x, __half *y, int nb, cudaStream_t st) {
    const MatrixView &m = h->view;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((m.rows + 15) / 16), 1, 1);
    cfg.blockDim = dim3(kTThreads, 1, 1);
    cfg.dynamicSmemBytes = kTSmem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, tl4_kernel, m, x, y, nb) == cudaSuccess ? DSQ_OK : DSQ_ERR_CUDA;
}

}  // namespace

int tl4_prepare() {
    return cudaFuncSetAttribute(tl4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kTSmem) == cudaSuccess
               ? DSQ_OK
               : DSQ_ERR_CUDA;
}

// 4-bit row tables, no column scales, 5 or more activation rows: 8 per launch.
bool tl4_covers(const dsq_handle_s *h, int batch) {
    const MatrixView &m = h->view;
    return batch >= 5 && m.mode == DSQ_MODE_LUT_ROW && m.bits == 4 && !m.cscale && m.rows > 0 && m.cols > 0;
}

int tl4_launch_count(const dsq_handle_s *h, int batch) { return tl4_covers(h, batch) ? (batch + 7) / 8 : -1; }

int launch_gemv_tl4(const dsq_handle_s *h, const __half *x, __half *y, int batch, cudaStream_t st) {
    if (!tl4_covers(h, batch)) return DSQ_ERR_UNSUPPORTED;
    const MatrixView &m = h->view;
    for (int b0 = 0; b0 < batch; b0 += 8) {
        const int rc = launch_tl4(h, x + (size_t)b0 * m.cols, y + (size_t)b0 * m.rows, std::min(8, batch - b0), st);
        if (rc != DSQ_OK) return rc;
    }
    return DSQ_OK;
}

}  // namespace dsq
