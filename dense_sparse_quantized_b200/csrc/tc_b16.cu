// tc_b16.cu -- batch >= 3: dequantise to fp16, contract on the 5th-gen
// tensor cores (tcgen05, accumulator in tensor memory), outliers in fp32.
//
// At 16+ activation rows the product is a real (skinny) GEMM, so the dense
// part goes through tcgen05.mma: for every 128-row tile and 64-column
// K-block the decoded weights W_dense (bit for bit the fp16 values dsq_decode
// writes) form the A operand and the x tile the B operand.
//
// One CTA per (128-row tile, K split); a K split >1 forms a thread-block
// cluster whose partial tiles are summed over distributed shared memory into
// the cluster's rank-0 CTA, which writes y once.  Warp roles:
//   warp 0       x producer: per K-block, a 2-D TMA load of the x tile
//                [NB rows][64 cols] into the 128-byte-swizzled K-major layout
//                the MMA reads (a deep ring; x is small and stays in L2);
//   warp 1       allocates tensor memory, issues the MMAs (one thread), frees
//                tensor memory;
//   warp 22      record producer: per stage of 4 K-blocks, two 2-D TMA loads
//                of the tile's packed rows -- 128 rows x 128 bytes of slot
//                records (128-byte swizzle) and 128 rows x 16 bytes of their
//                zero bytes -- into a ring of stages;
//   warps 2-17   decode: warp (quarter q = warp%4, K-block j of the stage)
//                reads, for row 32q + lane, its two slot records and zero
//                bytes from the stage (conflict-free thanks to the swizzle),
//                turns each slot's 32 codes into 16 fp16 pairs -- LOP3 places
//                two codes in the two halves of 1024.0, one HFMA2 gives the
//                exact q - zero, one HMUL2 rounds scale*(q - zero) once -- and
//                stores them into tensor memory (tcgen05.st) as the MMA's A
//                operand;
//   warps 18-21  outliers: the tile's CSR slice is brought into shared memory
//                by one bulk copy when it fits; thread (row) then walks its
//                row's entries that fall in each stage and accumulates
//                v * x[b][col] in fp32 (exact products) from the staged x
//                tiles -- at 64 activation rows from a column-major copy of
//                the stage that the four warps write first;
// after the loop warps 2-5 read the accumulator rows (tcgen05.ld), add the
// outlier sums, reduce over the cluster and store y.
//
// Every mbarrier wait is bounded (ptx.h); a wait that runs out sets the
// handle's status word and the CTA abandons the call, still releasing its
// tensor memory.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "internal.h"
#include "ptx.h"

namespace dsq {

namespace {

constexpr int kTM = 128;        // rows per tile (MMA M)
constexpr int kKB = 64;         // columns per K-block (two slots)
constexpr int kKS = 4;          // K-blocks per stage (8 slots: 128 bytes of each packed row)
constexpr int kRecB = kTM * 128;                // record bytes of a stage
constexpr int kStageRB = kRecB + kTM * 16;      // + the zero bytes (16 per row)
constexpr int kWarps = 23;
constexpr int kThreads = kWarps * 32;
constexpr int kTmemCols = 512;  // accumulators from column 0, then the A stages
constexpr uint32_t kMagic = 0x64006400u;  // fp16 1024.0 in both halves
constexpr uint32_t kSentinel = 0xffffffffu;

// Independent accumulators: consecutive MMAs into one accumulator serialise
// on its latency, so MMA number n of the split goes to accumulator
// n % NACC and the epilogue sums them.  Tensor memory: NACC accumulators of
// NB columns, then NA stages of A (4 K-blocks = 128 columns each) -- 512
// columns for every NB.
template <int NB>
__host__ __device__ constexpr int n_acc() { return NB <= 32 ? 8 : 4; }
template <int NB>
__host__ __device__ constexpr int a_col0() { return NB * n_acc<NB>(); }
template <int NB>
__host__ __device__ constexpr int a_stages() { return (kTmemCols - a_col0<NB>()) / 128; }
template <int NB>
__host__ __device__ constexpr int x_stages() { return NB <= 32 ? 3 : 2; }  // of kKS x tiles
template <int NB>
__host__ __device__ constexpr int rec_stages() { return NB <= 32 ? 4 : 2; }
// Shared memory for the tile's CSR entries (all of its rows, every split),
// staged by one bulk copy; a tile with more entries reads them from global
// memory, one row per thread.
template <int NB>
__host__ __device__ constexpr int csr_cap_bytes() { return NB == 16 ? 96 * 1024 : NB == 32 ? 64 * 1024 : 24 * 1024; }
// At 64 activation rows the outlier warps first copy each x stage
// column-major (the NB values of one column NB * 2 contiguous bytes) and read
// an entry's x values with NB / 8 16-byte loads instead of NB 2-byte loads
// from the swizzled tiles.  At 16 and 32 rows the copy and its two extra
// synchronisations per stage cost more than they save (measured: c4 q at 32
// rows 34.7 us without, 48.7 us with; at 64 rows 117 us without, 103 us with).
template <int NB>
__host__ __device__ constexpr bool col_major_x() { return NB >= 64; }
template <int NB>
__host__ __device__ constexpr int xt_bytes() { return col_major_x<NB>() ? kKS * kKB * NB * 2 : 0; }

struct TcParams {
    int rows, cols, S, row_words, nkb, kb_per_split, batch;
    const uint32_t *dense;
    const int32_t *row_ptr;
    const uint32_t *csr;
    const int32_t *split_start;  // [KS][rows] first CSR entry at or past the split's first column; null if KS == 1
    int *status;
};

// ------------------------------------------------------------ tcgen05 / TMA
__device__ __forceinline__ void tma2d(void *dst, const CUtensorMap *map, int c0, int c1, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_st16(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
        "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tc_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; i++) v[i] = __uint_as_float(r[i]);
}

// D[tmem] (+)= A[tmem] * B[smem desc]^T, kind::f16, one CTA.
__device__ __forceinline__ void tc_mma(uint32_t d, uint32_t a, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(d),
        "r"(a), "l"(bdesc), "r"(idesc), "r"(acc), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
        : "memory");
}
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// K-major operand, 128-byte swizzle, 8-row core groups 1024 bytes apart.
__device__ __forceinline__ uint64_t sw128_desc(const void *p) {
    const uint64_t a = (smem_u32(p) >> 4) & 0x3fffu;
    return a | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor: fp16 A and B (K-major), fp32 accumulator, M = 128.
__host__ __device__ constexpr uint32_t idesc_f16(int n) {
    return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kTM >> 4) << 24);
}

__device__ __forceinline__ uint32_t lop_or_and(uint32_t a, uint32_t mask, uint32_t c) {
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(a), "r"(mask), "r"(c));  // (a & mask) | c
    return r;
}
__device__ __forceinline__ uint32_t h2u(__half2 h) { return *reinterpret_cast<uint32_t *>(&h); }
__device__ __forceinline__ __half2 u2h(uint32_t u) { return *reinterpret_cast<__half2 *>(&u); }

// 32 codes of one slot (3 code words + scale pair) -> 16 fp16 pairs equal to
// fp16(scale * (q - zero)) for columns 2P, 2P+1.
__device__ __forceinline__ void decode_slot_f16(uint4 v, uint32_t zb, uint32_t (&o)[16]) {
    const uint32_t zA = zb & 15u, zB = (zb >> 4) & 15u;
    const __half2 nA = __hneg2(u2h((zA | (zA << 16)) | kMagic));  // -(1024 + zA)
    const __half2 nB = __hneg2(u2h((zB | (zB << 16)) | kMagic));
    const __half2 c896 = u2h(0x63006300u), c1008 = u2h(0x63e063e0u);
    const __half2 dA[3] = {nA, __hadd2(nA, c896), __hadd2(nA, c1008)};  // -(1024 * 8^-t + zA)
    const __half2 dB[3] = {nB, __hadd2(nB, c896), __hadd2(nB, c1008)};
    const __half2 cs[3] = {u2h(0x3c003c00u), u2h(0x30003000u), u2h(0x24002400u)};  // 1, 1/8, 1/64
    uint32_t sA, sB;
    asm("prmt.b32 %0, %1, %1, 0x1010;" : "=r"(sA) : "r"(v.w));
    asm("prmt.b32 %0, %1, %1, 0x3232;" : "=r"(sB) : "r"(v.w));
    const uint32_t a[3] = {v.x, v.y, v.z};
    const uint32_t b[3] = {v.x >> 10, v.y >> 10, v.z >> 10};
#pragma unroll
    for (int P = 0; P < 15; P++) {
        const int w = P / 5, j = P % 5;
        const int t = j < 3 ? j : j - 3;  // field at bit 3t of each half
        const uint32_t h = lop_or_and(j < 3 ? a[w] : b[w], 0x00070007u << (3 * t), kMagic);
        const __half2 qz = __hfma2(u2h(h), cs[t], P < 8 ? dA[t] : dB[t]);
        o[P] = h2u(__hmul2(qz, u2h(P < 8 ? sA : sB)));
    }
    // columns 30 (low half) and 31 (high half): bit k at bits 9 / 25 of word k
    const uint32_t t15 = ((a[0] >> 9) & 0x00010001u) | ((a[1] >> 8) & 0x00020002u) | ((a[2] >> 7) & 0x00040004u);
    o[15] = h2u(__hmul2(__hadd2(u2h(t15 | kMagic), nB), u2h(sB)));
}

// Element (row b, column c) of an x tile [NB][64] fp16 stored by TMA with the
// 128-byte swizzle (16-byte chunk index XOR row % 8 inside 1024-byte atoms).
__device__ __forceinline__ int sw128_off(int b, int c) {
    return ((b >> 3) << 10) + ((b & 7) << 7) + ((((c >> 3) ^ (b & 7))) << 4) + ((c & 7) << 1);
}

struct Smem {
    uint64_t *afull, *aempty, *xfull, *xempty, *done, *rfull, *rempty, *csrfull, *xtready, *xtfree;
    uint32_t *tmem_slot;
    unsigned char *x, *rec, *xt;
    float *obuf, *rbuf;
    uint32_t *csr;
};

template <int NB>
__device__ __forceinline__ Smem carve(unsigned char *base) {
    constexpr int NX = x_stages<NB>(), NA = a_stages<NB>(), NR = rec_stages<NB>();
    Smem s;
    uint64_t *bars = reinterpret_cast<uint64_t *>(base);
    s.afull = bars;
    s.aempty = s.afull + NA;
    s.xfull = s.aempty + NA;
    s.xempty = s.xfull + NX;
    s.done = s.xempty + NX;
    s.rfull = s.done + 1;
    s.rempty = s.rfull + NR;
    s.csrfull = s.rempty + NR;
    s.xtready = s.csrfull + 1;
    s.xtfree = s.xtready + 1;
    s.tmem_slot = reinterpret_cast<uint32_t *>(s.xtfree + 1);
    s.x = base + 1024;                  // stages of kKS tiles [NB][64] fp16
    s.rec = s.x + NX * kKS * NB * 128;  // stages of kStageRB bytes
    s.obuf = reinterpret_cast<float *>(s.rec + NR * kStageRB);
    s.rbuf = s.obuf + kTM * NB;
    s.csr = reinterpret_cast<uint32_t *>(s.rbuf + kTM * NB);
    s.xt = reinterpret_cast<unsigned char *>(s.csr) + csr_cap_bytes<NB>();
    return s;
}

// 1 KB alignment slack + barriers + x ring + record ring + outlier sums +
// cluster inbox + staged CSR entries + column-major x stage.
template <int NB>
__host__ __device__ constexpr size_t smem_bytes() {
    return 2048 + (size_t)x_stages<NB>() * kKS * NB * 128 + (size_t)rec_stages<NB>() * kStageRB +
           (size_t)kTM * NB * 4 * 2 + csr_cap_bytes<NB>() + xt_bytes<NB>();
}
static_assert(smem_bytes<16>() <= 232448 && smem_bytes<32>() <= 232448 && smem_bytes<64>() <= 232448,
              "shared memory per CTA");

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void st_cluster_f32(const float *local, uint32_t rank, float v) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(remote), "f"(v) : "memory");
}

template <int NB>
__global__ void __launch_bounds__(kThreads, 1)
tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_rec,
          const __grid_constant__ CUtensorMap tm_zero, TcParams p, int KS, __half *__restrict__ y) {
    static_assert(NB == 16 || NB == 32 || NB == 64, "NB");
    constexpr int NX = x_stages<NB>(), NA = a_stages<NB>(), NR = rec_stages<NB>(), NACC = n_acc<NB>();
    constexpr int XB = kKS * NB * 128;  // bytes of one x stage
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // 1024-byte alignment for the swizzled tiles (1 KB of slack is allocated)
    unsigned char *smem_base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const Smem sm = carve<NB>(smem_base);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rank = KS > 1 ? (int)cluster_rank() : 0;
    const int tile = blockIdx.y;
    const int kb0 = rank * p.kb_per_split;  // a multiple of kKS
    const int nk = max(0, min(p.nkb, kb0 + p.kb_per_split) - kb0);
    const int t0 = kb0 / kKS, nst = (nk + kKS - 1) / kKS;  // stages of this split

    if (threadIdx.x == 0) {
        for (int i = 0; i < NA; i++) {
            mbar_init(&sm.afull[i], 16);  // every decode warp, once per stage
            mbar_init(&sm.aempty[i], 1);
        }
        for (int i = 0; i < NR; i++) {
            mbar_init(&sm.rfull[i], 1);
            mbar_init(&sm.rempty[i], 16);
        }
        for (int i = 0; i < NX; i++) {
            mbar_init(&sm.xfull[i], 1);
            mbar_init(&sm.xempty[i], 1 + 4);  // the MMAs and the four outlier warps (after their transpose)
        }
        mbar_init(sm.done, 1);
        mbar_init(sm.csrfull, 1);
        mbar_init(sm.xtready, 4);  // the four outlier warps, once per stage
        mbar_init(sm.xtfree, 4);
        fence_mbar_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(sm.tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *sm.tmem_slot;
    // The next call may start launching; weights, scales and outliers belong
    // to the handle, so only x (loaded below) and y (stored at the end) wait
    // for the previous kernel in the stream.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (warp == 0) {
        // x producer: per stage, the kKS x tiles [NB][64] (128-byte swizzle)
        if (lane == 0) {
            asm volatile("griddepcontrol.wait;" ::: "memory");
            int issued = 0;
            for (int i = 0; i < nst; i++) {
                const int s = i % NX;
                if (i >= NX && !mbar_wait(&sm.xempty[s], ((i / NX) - 1) & 1)) {
                    report(p.status, kStatusTimeout);
                    break;
                }
                mbar_arrive_expect_tx(&sm.xfull[s], (uint32_t)XB);
                for (int kb = 0; kb < kKS; kb++)
                    tma2d(sm.x + s * XB + kb * NB * 128, &tm_x, kKB * (kb0 + kKS * i + kb), 0, &sm.xfull[s]);
                issued = i + 1;
            }
            for (int i = max(0, issued - NX); i < issued; i++)
                if (!mbar_wait(&sm.xfull[i % NX], (i / NX) & 1)) report(p.status, kStatusTimeout);
        }
    } else if (warp == 1) {
        // MMA issuer: per stage, 4 MMAs (K = 16 each) per K-block into rotating
        // accumulators.  The issuing thread shares its scheduler with busy
        // decode warps, so a full stage is one unrolled run of MMAs with
        // compile-time offsets.
        if (lane == 0) {
            const uint32_t idesc = idesc_f16(NB);
            for (int i = 0; i < nst; i++) {
                const int as = i % NA, s = i % NX;
                if (!mbar_wait(&sm.afull[as], (i / NA) & 1) || !mbar_wait(&sm.xfull[s], (i / NX) & 1)) {
                    report(p.status, kStatusTimeout);
                    break;
                }
                tc_fence_after();
                const uint32_t a0 = tmem + a_col0<NB>() + 128 * as;
                const uint64_t b0 = sw128_desc(sm.x + s * XB);
                const int nkb = min(kKS, nk - kKS * i);  // K-blocks of this stage
                if (nkb == kKS && i > 0) {
#pragma unroll
                    for (int m = 0; m < 4 * kKS; m++)  // m = 4 * kb + k
                        tc_mma(tmem + NB * (m % NACC), a0 + 32 * (m / 4) + 8 * (m % 4),
                               b0 + ((m / 4) * NB * 128 >> 4) + 2 * (m % 4), idesc, 1u);
                } else {
                    for (int m = 0; m < 4 * nkb; m++)
                        tc_mma(tmem + NB * (m % NACC), a0 + 32 * (m / 4) + 8 * (m % 4),
                               b0 + ((m / 4) * NB * 128 >> 4) + 2 * (m % 4), idesc,
                               (i > 0 || m >= NACC) ? 1u : 0u);
                }
                tc_commit(&sm.aempty[as]);
                tc_commit(&sm.xempty[s]);
            }
            tc_commit(sm.done);  // fires once every MMA issued above has completed
        }
    } else if (warp < 18) {
        // decode: warp (quarter q, K-block j of every stage)
        const int q = warp & 3, j = (warp - 2) >> 2;
        const int r = 32 * q + lane;
        const uint32_t tbase = tmem + ((uint32_t)(32 * q) << 16);
        for (int i = 0; i < nst; i++) {
            const int st = i % NR, as = i % NA;
            if (!mbar_wait_warp(&sm.rfull[st], (i / NR) & 1) ||
                (i >= NA && !mbar_wait_warp(&sm.aempty[as], ((i / NA) - 1) & 1))) {
                if (lane == 0) report(p.status, kStatusTimeout);
                break;
            }
            const int t = t0 + i;
            if (kKS * i + j < nk) {
                const unsigned char *rs = sm.rec + st * kStageRB;
                tc_fence_after();
#pragma unroll
                for (int h = 0; h < 2; h++) {
                    const int c = 2 * j + h;  // 16-byte chunk of the row = slot of the stage
                    const uint4 v = *reinterpret_cast<const uint4 *>(rs + r * 128 + ((c ^ (r & 7)) << 4));
                    const uint32_t zb = rs[kRecB + r * 16 + 8 * (t & 1) + c];
                    uint32_t o[16];
                    decode_slot_f16(v, zb, o);  // records past the row's end read as 0 and decode to 0
                    tc_st16(tbase + a_col0<NB>() + 128 * as + 32 * j + 16 * h, o);
                }
                tc_wait_st();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&sm.afull[as]);
                mbar_arrive(&sm.rempty[st]);
            }
        }
    } else if (warp == 22) {
        // record producer
        if (lane == 0) {
            for (int i = 0; i < nst; i++) {
                const int st = i % NR, t = t0 + i;
                if (i >= NR && !mbar_wait(&sm.rempty[st], ((i / NR) - 1) & 1)) {
                    report(p.status, kStatusTimeout);
                    break;
                }
                unsigned char *rs = sm.rec + st * kStageRB;
                const int g = (2 * kKS * t) / 32, u = (2 * kKS * t) % 32;  // group, first slot in it
                mbar_arrive_expect_tx(&sm.rfull[st], (uint32_t)kStageRB);
                tma2d(rs, &tm_rec, kAff3GroupWords * g + 8 + 4 * u, kTM * tile, &sm.rfull[st]);
                tma2d(rs + kRecB, &tm_zero, kAff3GroupWords * g + 4 * (u / 16), kTM * tile, &sm.rfull[st]);
            }
        }
    } else {
        // outliers: thread = row, the entries in this split's columns, stage by stage
        const int r = 32 * (warp & 3) + lane;
        const int grow = kTM * tile + r;
        float acc[NB];
#pragma unroll
        for (int b = 0; b < NB; b++) acc[b] = 0.f;
        // the tile's entries [ka, kz), rounded out to 16 bytes (the blob is padded past the end)
        const int ka = __ldg(p.row_ptr + kTM * tile) & ~3;
        const int kz = (__ldg(p.row_ptr + min(kTM * tile + kTM, p.rows)) + 3) & ~3;
        const bool staged = kz > ka && (kz - ka) * 4 <= csr_cap_bytes<NB>();
        if (staged && warp == 18 && lane == 0) {
            mbar_arrive_expect_tx(sm.csrfull, (uint32_t)(kz - ka) * 4);
            bulk_g2s(sm.csr, p.csr + ka, (uint32_t)(kz - ka) * 4, sm.csrfull);
        }
        int k = 0, kend = 0;
        if (grow < p.rows && nk > 0) {
            k = p.split_start ? p.split_start[(size_t)rank * p.rows + grow] : p.row_ptr[grow];
            kend = p.row_ptr[grow + 1];
        }
        if (staged && !mbar_wait_warp(sm.csrfull, 0)) {
            if (lane == 0) report(p.status, kStatusTimeout);
            kend = k;  // the entries never arrived: none are read
        }
        auto entry = [&](int e) -> uint32_t {
            return e < kend ? (staged ? sm.csr[e - ka] : __ldg(p.csr + e)) : kSentinel;
        };
        uint32_t qv[4];
#pragma unroll
        for (int t = 0; t < 4; t++) qv[t] = entry(k + t);
        const int cend = kKB * (kb0 + nk);  // first column past this split
        for (int i = 0; i < nst && !col_major_x<NB>(); i++) {
            const int s = i % NX;
            if (!mbar_wait_warp(&sm.xfull[s], (i / NX) & 1)) {
                if (lane == 0) report(p.status, kStatusTimeout);
                break;
            }
            const int c0 = kKB * (kb0 + kKS * i);
            const int c1 = min(c0 + kKS * kKB, cend);
            while ((int)(qv[0] & 0xffffu) < c1) {
                const int cs = (int)(qv[0] & 0xffffu) - c0;
                const unsigned char *xt = sm.x + s * XB + (cs >> 6) * NB * 128;
                const int cl = cs & 63;
                const unsigned short vb = (unsigned short)(qv[0] >> 16);
#pragma unroll
                for (int b = 0; b < NB; b++) {
                    const unsigned short xb = *reinterpret_cast<const unsigned short *>(xt + sw128_off(b, cl));
                    asm("fma.rn.f32.f16 %0, %1, %2, %0;" : "+f"(acc[b]) : "h"(vb), "h"(xb));
                }
                qv[0] = qv[1];
                qv[1] = qv[2];
                qv[2] = qv[3];
                k++;
                qv[3] = entry(k + 3);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.xempty[s]);
        }
        // column pair of the stage this thread transposes: K-block kt, columns 2 jp, 2 jp + 1
        const int ot = 32 * (warp - 18) + lane, kt = ot >> 5, jp = ot & 31;
        uint4 *xt0 = reinterpret_cast<uint4 *>(sm.xt + (size_t)(kKB * kt + 2 * jp) * NB * 2);
        for (int i = 0; i < nst && col_major_x<NB>(); i++) {
            const int s = i % NX;
            // the previous stage's column-major copy is free, this stage's x tiles have landed
            if ((i > 0 && !mbar_wait_warp(sm.xtfree, (i - 1) & 1)) || !mbar_wait_warp(&sm.xfull[s], (i / NX) & 1)) {
                if (lane == 0) report(p.status, kStatusTimeout);
                break;
            }
            {
                const unsigned char *tile = sm.x + s * XB + kt * NB * 128;
#pragma unroll
                for (int q = 0; q < NB / 8; q++) {
                    uint32_t w[NB];  // rows 8q .. 8q + 7 used
#pragma unroll
                    for (int b = 8 * q; b < 8 * q + 8; b++)
                        w[b] = *reinterpret_cast<const uint32_t *>(tile + sw128_off(b, 2 * jp));
                    uint4 lo, hi;  // columns 2 jp and 2 jp + 1, rows 8q .. 8q + 7
                    asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(lo.x) : "r"(w[8 * q + 0]), "r"(w[8 * q + 1]));
                    asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(lo.y) : "r"(w[8 * q + 2]), "r"(w[8 * q + 3]));
                    asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(lo.z) : "r"(w[8 * q + 4]), "r"(w[8 * q + 5]));
                    asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(lo.w) : "r"(w[8 * q + 6]), "r"(w[8 * q + 7]));
                    asm("prmt.b32 %0, %1, %2, 0x7632;" : "=r"(hi.x) : "r"(w[8 * q + 0]), "r"(w[8 * q + 1]));
                    asm("prmt.b32 %0, %1, %2, 0x7632;" : "=r"(hi.y) : "r"(w[8 * q + 2]), "r"(w[8 * q + 3]));
                    asm("prmt.b32 %0, %1, %2, 0x7632;" : "=r"(hi.z) : "r"(w[8 * q + 4]), "r"(w[8 * q + 5]));
                    asm("prmt.b32 %0, %1, %2, 0x7632;" : "=r"(hi.w) : "r"(w[8 * q + 6]), "r"(w[8 * q + 7]));
                    xt0[q] = lo;
                    xt0[NB / 8 + q] = hi;
                }
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&sm.xempty[s]);  // this warp is done with the ring stage
                mbar_arrive(sm.xtready);
            }
            if (!mbar_wait_warp(sm.xtready, i & 1)) {
                if (lane == 0) report(p.status, kStatusTimeout);
                break;
            }
            const int c0 = kKB * (kb0 + kKS * i);
            const int c1 = min(c0 + kKS * kKB, cend);
            while ((int)(qv[0] & 0xffffu) < c1) {
                const uint4 *xc = reinterpret_cast<const uint4 *>(sm.xt + (size_t)((int)(qv[0] & 0xffffu) - c0) * NB * 2);
                const unsigned short vb = (unsigned short)(qv[0] >> 16);
#pragma unroll
                for (int q = 0; q < NB / 8; q++) {
                    const uint4 v = xc[q];
                    const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int t = 0; t < 4; t++)
                        asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
                            "fma.rn.f32.f16 %0, %3, l, %0;\n\tfma.rn.f32.f16 %1, %3, h, %1;\n\t}"
                            : "+f"(acc[8 * q + 2 * t]), "+f"(acc[8 * q + 2 * t + 1])
                            : "r"(vv[t]), "h"(vb));
                }
                qv[0] = qv[1];
                qv[1] = qv[2];
                qv[2] = qv[3];
                k++;
                qv[3] = entry(k + 3);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(sm.xtfree);
        }
#pragma unroll
        for (int b = 0; b < NB; b++) sm.obuf[r * NB + b] = acc[b];
    }

    __syncthreads();
    // epilogue: warps 2..5 own accumulator lane quarters 2, 3, 0, 1
    float part[NB];
    const bool epi = warp >= 2 && warp < 6;
    const int q = warp & 3;
    const int r = 32 * q + lane;
    const int grow = kTM * tile + r;
    if (epi) {
        bool have = nk > 0;
        if (have && !mbar_wait_warp(sm.done, 0)) {
            if (lane == 0) report(p.status, kStatusTimeout);
            have = false;
        }
        tc_fence_after();
        // sum the accumulators that received MMAs (all of them once nk >= NACC/4)
        const int nacc = min(4 * nk, n_acc<NB>());
#pragma unroll
        for (int c = 0; c < NB; c += 16) {
            float v[16];
#pragma unroll
            for (int t = 0; t < 16; t++) v[t] = 0.f;
            if (have)
                for (int u = 0; u < nacc; u++) {
                    float w[16];
                    tc_ld16(tmem + ((uint32_t)(32 * q) << 16) + NB * u + c, w);
#pragma unroll
                    for (int t = 0; t < 16; t++) v[t] += w[t];
                }
#pragma unroll
            for (int t = 0; t < 16; t++) part[c + t] = v[t] + sm.obuf[r * NB + c + t];
        }
        if (KS > 1 && rank > 0) {
#pragma unroll
            for (int b = 0; b < NB; b++) st_cluster_f32(sm.rbuf + ((size_t)(rank - 1) * kTM + r) * NB + b, 0, part[b]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
    }
    if (KS > 1) cluster_sync();
    if (epi && rank == 0 && grow < p.rows) {
        asm volatile("griddepcontrol.wait;" ::: "memory");
        for (int j = 0; j < KS - 1; j++)
#pragma unroll
            for (int b = 0; b < NB; b++) part[b] += sm.rbuf[((size_t)j * kTM + r) * NB + b];
#pragma unroll
        for (int b = 0; b < NB; b++)
            if (b < p.batch) y[(size_t)b * p.rows + grow] = __float2half_rn(part[b]);
    }
}

// ------------------------------------------------------------ host side
// The driver's tensor-map encoder, looked up once (a function-local static:
// its initialisation is thread-safe); null when the driver lacks it.
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static const PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        cudaGetLastError();
        return nullptr;
    }();
    return fn;
}

bool encode_2d(CUtensorMap *m, CUtensorMapDataType dt, const void *base, uint64_t d0, uint64_t d1,
               uint64_t stride1_bytes, uint32_t b0, uint32_t b1, CUtensorMapSwizzle sw) {
    PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {d0, d1};
    const cuuint64_t strides[1] = {stride1_bytes};
    const cuuint32_t box[2] = {b0, b1};
    const cuuint32_t es[2] = {1, 1};
    return fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NB>
int launch_nb(const TcParams &p, int KS, const CUtensorMap &tx, const CUtensorMap &trec, const CUtensorMap &tzero,
              __half *y, cudaStream_t st, bool pdl) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(KS, (p.rows + kTM - 1) / kTM, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem_bytes<NB>();
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = KS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, tc_kernel<NB>, tx, trec, tzero, p, KS, y) == cudaSuccess ? DSQ_OK : DSQ_ERR_CUDA;
}

template <int NB>
int set_attr() {
    return cudaFuncSetAttribute(tc_kernel<NB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)smem_bytes<NB>()) == cudaSuccess
               ? DSQ_OK
               : DSQ_ERR_CUDA;
}

int set_attrs() {
    int rc = set_attr<16>();
    if (rc == DSQ_OK) rc = set_attr<32>();
    if (rc == DSQ_OK) rc = set_attr<64>();
    return rc;
}

// K split of a matrix: KS CTAs (one cluster) per 128-row tile, as many as fit
// one CTA per SM, at most 2; a split covers whole stages (kKS K-blocks) and
// none is empty.
struct Split {
    int KS, nkb, kb_per_split;
};
Split plan_split(const MatrixView &m, int sm_count) {
    Split sp;
    const int tiles = (m.rows + kTM - 1) / kTM;
    sp.nkb = (m.slots + 1) / 2;
    const int stages = (sp.nkb + kKS - 1) / kKS;
    sp.KS = 1;
    for (int k = 2; k <= 2; k++)  // the cluster inbox holds one peer's tile
        if (tiles * k <= sm_count && k <= stages) sp.KS = k;
    sp.kb_per_split = kKS * ((stages + sp.KS - 1) / sp.KS);
    sp.KS = (sp.nkb + sp.kb_per_split - 1) / sp.kb_per_split;
    return sp;
}

bool tc_shape_ok(const MatrixView &m) {
    // cols <= 32768 keeps every K-block's end below the sentinel column 0xffff
    return m.rows > 0 && m.cols > 0 && m.cols <= 32768 && m.mode == DSQ_MODE_AFFINE_G16 && m.bits == 3;
}

// All launches of one product (batch in chunks of 64 rows of x).
// pdl: programmatic dependent launch (the kernel reads the packed matrix
// before the previous kernel in the stream has finished) -- only for packed
// data the handle owns.
int run_tc(const MatrixView &m, const Split &sp, const int32_t *split_start, int *status, const __half *x,
           __half *y, int batch, cudaStream_t st, bool pdl) {
    for (int b0 = 0; b0 < batch; b0 += 64) {
        const int nb = std::min(64, batch - b0);
        const int NB = nb <= 16 ? 16 : nb <= 32 ? 32 : 64;
        CUtensorMap tx, trec, tzero;
        if (!encode_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, x + (size_t)b0 * m.cols, m.cols, nb,
                       (uint64_t)m.cols * 2, kKB, NB, CU_TENSOR_MAP_SWIZZLE_128B))
            return DSQ_ERR_CUDA;
        // the packed rows as [rows][row_words] u32: stage boxes of 32 words (records,
        // 128-byte swizzle) and 4 words (zero bytes) by 128 rows; past the row end or
        // the last row the loads fill zeros
        if (!encode_2d(&trec, CU_TENSOR_MAP_DATA_TYPE_UINT32, m.dense, m.row_words, m.rows, (uint64_t)m.row_words * 4,
                       32, kTM, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !encode_2d(&tzero, CU_TENSOR_MAP_DATA_TYPE_UINT32, m.dense, m.row_words, m.rows,
                       (uint64_t)m.row_words * 4, 4, kTM, CU_TENSOR_MAP_SWIZZLE_NONE))
            return DSQ_ERR_CUDA;
        TcParams p;
        p.rows = m.rows;
        p.cols = m.cols;
        p.S = m.slots;
        p.row_words = m.row_words;
        p.nkb = sp.nkb;
        p.kb_per_split = sp.kb_per_split;
        p.batch = nb;
        p.dense = m.dense;
        p.row_ptr = m.row_ptr;
        p.csr = m.csr;
        p.split_start = sp.KS > 1 ? split_start : nullptr;
        p.status = status;
        __half *yb = y + (size_t)b0 * m.rows;
        int rc;
        if (NB == 16) rc = launch_nb<16>(p, sp.KS, tx, trec, tzero, yb, st, pdl);
        else if (NB == 32) rc = launch_nb<32>(p, sp.KS, tx, trec, tzero, yb, st, pdl);
        else rc = launch_nb<64>(p, sp.KS, tx, trec, tzero, yb, st, pdl);
        if (rc != DSQ_OK) return rc;
    }
    return DSQ_OK;
}

}  // namespace

// From 3 activation rows on, one tensor-core pass (the batch padded to 16
// with zero rows by the x loads) beats the batch-1 kernel run per row --
// unless a row carries hundreds of outliers: the outlier warps walk one row
// per thread, so such matrices go to the tensor cores from 16 rows on.
constexpr int kTcMinBatch = 3, kTcMinBatchHeavy = 16, kHeavyRowNnz = 256;

bool tc_covers(const dsq_handle_s *h, int batch) {
    // two-axis matrices need x times the column scales exactly (fp32), which
    // an fp16 B operand cannot hold
    return h->tc.ready && batch >= h->tc.min_batch && tc_shape_ok(h->view) && !h->view.cscale;
}

int tc_launch_count(const dsq_handle_s *h, int batch) { return tc_covers(h, batch) ? (batch + 63) / 64 : -1; }

// K split and the per-split CSR start of every row.  Host-side, at create,
// with the device current.
int tc_prepare(dsq_handle_s *h, const int32_t *rp, const uint32_t *csr_host) {
    const MatrixView &m = h->view;
    TcPlan &tc = h->tc;
    tc.ready = false;
    if (!tc_shape_ok(m)) return DSQ_OK;
    if (!encode_fn()) return DSQ_OK;  // no tensor-map support: the CUDA-core path serves every batch
    const Split sp = plan_split(m, h->sm_count);
    const int KS = sp.KS;
    tc.KS = KS;
    tc.nkb = sp.nkb;
    tc.kb_per_split = sp.kb_per_split;
    int max_nnz = 0;
    for (int r = 0; r < m.rows; r++) max_nnz = std::max(max_nnz, rp[r + 1] - rp[r]);
    tc.min_batch = max_nnz > kHeavyRowNnz ? kTcMinBatchHeavy : kTcMinBatch;
    if (KS > 1) {
        std::vector<int32_t> starts((size_t)KS * m.rows);
        for (int s = 0; s < KS; s++) {
            const int c0 = s * tc.kb_per_split * kKB;
            for (int r = 0; r < m.rows; r++) {
                // first entry of row r with column >= c0 (entries sorted by column)
                int32_t lo = rp[r], hi = rp[r + 1];
                while (lo < hi) {
                    const int32_t mid = lo + (hi - lo) / 2;
                    if ((int)(csr_host[mid] & 0xffffu) < c0) lo = mid + 1; else hi = mid;
                }
                starts[(size_t)s * m.rows + r] = lo;
            }
        }
        if (cudaMalloc(&tc.split_start, starts.size() * 4) != cudaSuccess) {
            cudaGetLastError();
            return DSQ_ERR_OOM;
        }
        h->device_bytes += starts.size() * 4;
        if (cudaMemcpy(tc.split_start, starts.data(), starts.size() * 4, cudaMemcpyHostToDevice) != cudaSuccess)
            return DSQ_ERR_CUDA;
    }
    const int rc = set_attrs();
    if (rc != DSQ_OK) return rc;
    tc.ready = true;
    return DSQ_OK;
}

void tc_free(dsq_handle_s *h) {
    if (h->tc.split_start) cudaFree(h->tc.split_start);
    h->tc.split_start = nullptr;
}

int launch_gemv_tc(const dsq_handle_s *h, const __half *x, __half *y, int batch, cudaStream_t st) {
    if (!tc_covers(h, batch)) return DSQ_ERR_UNSUPPORTED;
    const Split sp = {h->tc.KS, h->tc.nkb, h->tc.kb_per_split};
    return run_tc(h->view, sp, h->tc.split_start, h->d_status, x, y, batch, st, true);
}

}  // namespace dsq

// ---------------------------------------------------------------------------
// dsq_gemv_noalloc: the tensor-core product for callers that cannot allocate
// device memory.  The only memory the kernels need besides the caller's
// buffers -- the status word and the per-split CSR starts -- lives in one
// fixed array that every GPU loading this library holds until exit.
// ---------------------------------------------------------------------------

namespace dsq {

namespace {

// 256 KiB: word 0 is the status word, words [kNoAllocStartsOff, ...) the
// split starts ([KS][rows], KS > 1 only).
constexpr int kNoAllocWords = 65536;
constexpr int kNoAllocStartsOff = 64;
constexpr int kNoAllocMaxStarts = kNoAllocWords - kNoAllocStartsOff;
constexpr int kNoAllocMaxDevices = 64;

static __device__ __align__(256) int32_t g_noalloc_scratch[kNoAllocWords];

// Clears the status word and, for a K split, finds in every row the first CSR
// entry at or past each split's first column (entries sorted by column).
__global__ void noalloc_prep_kernel(int32_t *scratch, const int32_t *row_ptr, const uint32_t *csr, int rows,
                                    int KS, int cols_per_split) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i == 0) scratch[0] = 0;
    if (KS <= 1 || i >= (int64_t)KS * rows) return;
    const int s = (int)(i / rows), r = (int)(i % rows);
    const int c0 = s * cols_per_split;
    int32_t lo = row_ptr[r], hi = row_ptr[r + 1];
    while (lo < hi) {
        const int32_t mid = lo + (hi - lo) / 2;
        if ((int)(csr[mid] & 0xffffu) < c0) lo = mid + 1; else hi = mid;
    }
    scratch[kNoAllocStartsOff + i] = lo;
}

struct NoAllocDevice {
    bool ready = false;
    int sm_count = 0;
    int32_t *scratch = nullptr;  // device address of g_noalloc_scratch on this device
};
std::mutex g_noalloc_mu;
NoAllocDevice g_noalloc_dev[kNoAllocMaxDevices];

// Once per device, with that device current: check the architecture, look up
// the scratch array's device address and set the kernels' shared-memory limit.
int noalloc_setup(int dev, NoAllocDevice *out) {
    if (dev < 0 || dev >= kNoAllocMaxDevices) return DSQ_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    NoAllocDevice &d = g_noalloc_dev[dev];
    if (!d.ready) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return DSQ_ERR_CUDA;
        if (major != 10 || minor != 0 || !encode_fn()) return DSQ_ERR_UNSUPPORTED;
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) {
            cudaGetLastError();
            return DSQ_ERR_CUDA;
        }
        const int rc = set_attrs();
        if (rc != DSQ_OK) return rc;
        d.sm_count = sms;
        d.scratch = (int32_t *)ptr;
        d.ready = true;
    }
    *out = d;
    return DSQ_OK;
}

}  // namespace

}  // namespace dsq

extern "C" int dsq_gemv_noalloc(const dsq_desc *d, const void *packed_device, size_t bytes, const void *x, void *y,
                                int batch, void *stream) {
    using namespace dsq;
    if (!d || batch < 1) return DSQ_ERR_INVALID_ARG;
    int rc = check_desc(d);
    if (rc != DSQ_OK) return rc;
    BlobHeader hd;
    plan_blob(d, &hd);
    if (bytes != hd.total) return DSQ_ERR_INVALID_ARG;
    if (d->rows == 0) return DSQ_OK;
    if (!packed_device || ((uintptr_t)packed_device & 255u) || !y || ((uintptr_t)y & 15u) ||
        (d->cols > 0 && (!x || ((uintptr_t)x & 15u))))
        return DSQ_ERR_INVALID_ARG;
    if (d->mode != DSQ_MODE_AFFINE_G16 || d->bits != 3 || d->cols > 32768 || batch < 16) return DSQ_ERR_UNSUPPORTED;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return DSQ_ERR_CUDA;
    NoAllocDevice nd;
    rc = noalloc_setup(dev, &nd);
    if (rc != DSQ_OK) return rc;
    const cudaStream_t st = (cudaStream_t)stream;
    if (d->cols == 0) return launch_zero((__half *)y, (int64_t)batch * d->rows, st);

    const uint8_t *base = (const uint8_t *)packed_device;
    MatrixView m;
    m.rows = hd.rows;
    m.cols = hd.cols;
    m.bits = hd.bits;
    m.mode = hd.mode;
    m.slots = hd.slots;
    m.row_words = hd.row_words;
    m.nnz = hd.nnz;
    m.dense = (const uint32_t *)(base + hd.off_dense);
    m.table = (const uint16_t *)(base + hd.off_table);
    m.row_ptr = (const int32_t *)(base + hd.off_row_ptr);
    m.csr = (const uint32_t *)(base + hd.off_csr);
    const Split sp = plan_split(m, nd.sm_count);
    const int64_t starts = sp.KS > 1 ? (int64_t)sp.KS * m.rows : 0;
    if (starts > kNoAllocMaxStarts) return DSQ_ERR_SCRATCH_LIMIT;

    const int64_t n_prep = std::max<int64_t>(1, starts);
    noalloc_prep_kernel<<<(unsigned)((n_prep + 255) / 256), 256, 0, st>>>(
        nd.scratch, m.row_ptr, m.csr, m.rows, sp.KS, sp.kb_per_split * kKB);
    if (cudaGetLastError() != cudaSuccess) return DSQ_ERR_CUDA;
    // no programmatic dependent launch: the packed matrix is the caller's and
    // the split starts come from the kernel just launched
    return run_tc(m, sp, nd.scratch + kNoAllocStartsOff, (int *)nd.scratch, (const __half *)x, (__half *)y, batch,
                  st, false);
}
