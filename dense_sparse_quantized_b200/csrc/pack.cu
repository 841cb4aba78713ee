// pack.cu -- dsq_pack / dsq_blob_desc: host-side validation of the logical
// weights and their layout into the packed blob (see layout.h).
#include <math.h>
#include <string.h>

#include <vector>

#include <cuda_fp16.h>

#include "../../include/dsq.h"
#include "layout.h"
#include "internal.h"

namespace dsq {

// IEEE binary16 bit pattern -> double (host; validation only).
double half_bits_to_double(uint16_t h) {
    int e = (h >> 10) & 31, m = h & 1023;
    double v = e == 0 ? ldexp((double)m, -24)
             : e == 31 ? (m ? NAN : INFINITY)
                       : ldexp((double)(1024 + m), e - 25);
    return (h & 0x8000) ? -v : v;
}

static inline uint64_t align_up(uint64_t v, uint64_t a) { return (v + a - 1) / a * a; }

int check_desc(const dsq_desc *d) {
    if (!d) return DSQ_ERR_INVALID_ARG;
    if (d->rows < 0 || d->cols < 0 || d->cols % kGroup != 0) return DSQ_ERR_INVALID_ARG;
    if (d->mode != DSQ_MODE_LUT_ROW && d->mode != DSQ_MODE_AFFINE_G16 && d->mode != DSQ_MODE_BITPLANE &&
        d->mode != DSQ_MODE_INTGRID)
        return DSQ_ERR_INVALID_ARG;
    if (d->mode == DSQ_MODE_INTGRID) {
        if (d->bits != 14) return DSQ_ERR_INVALID_ARG;
    } else if (d->mode == DSQ_MODE_BITPLANE) {
        if (d->bits != 2 && d->bits != 3) return DSQ_ERR_INVALID_ARG;
        if (d->cols % (32 << d->bits) != 0) return DSQ_ERR_INVALID_ARG;
    } else if (d->bits != 3 && d->bits != 4) {
        return DSQ_ERR_INVALID_ARG;
    }
    if (d->nnz < 0 || d->nnz > (int64_t)d->rows * d->cols) return DSQ_ERR_INVALID_ARG;
    if (d->cols > 65535) return DSQ_ERR_UNSUPPORTED;
    return DSQ_OK;
}

void plan_blob(const dsq_desc *d, BlobHeader *h, uint32_t flags, uint32_t stream_words, uint32_t nsym) {
    memset(h, 0, sizeof(*h));
    memcpy(h->magic, kMagic, sizeof(kMagic));
    h->version = kVersion;
    h->header_bytes = kHeaderBytes;
    h->rows = d->rows;
    h->cols = d->cols;
    h->bits = d->bits;
    h->mode = d->mode;
    h->nnz = d->nnz;
    h->slots = slots_of(d->cols);
    h->row_words = row_words_of(d->bits, d->mode, h->slots);
    uint64_t off = kHeaderBytes;
    h->off_dense = off;
    if (d->mode == DSQ_MODE_INTGRID) {
        // bitstream, scales, slot offsets, codebook
        h->stream_words = stream_words;
        h->nsym = nsym;
        off = align_up(off + ((uint64_t)stream_words + kStreamPad) * 4, kSectionAlign);
        h->off_table = off;
        off = align_up(off + (uint64_t)d->rows * (d->cols / kGroup) * 2, kSectionAlign);
        h->off_index = off;
        off = align_up(off + (uint64_t)d->rows * h->slots * 4, kSectionAlign);
        h->off_codebook = off;
        off = align_up(off + ((uint64_t)kCbSyms + (nsym + 1) / 2) * 4, kSectionAlign);
        h->off_row_ptr = off;
        off = align_up(off + (uint64_t)(d->rows + 1) * 4, kSectionAlign);
        h->off_csr = off;
        off = align_up(off + (uint64_t)d->nnz * 4 + 16, kSectionAlign);
        h->flags = flags;
        h->total = off;
        return;
    }
    off = align_up(off + (uint64_t)d->rows * h->row_words * 4, kSectionAlign);
    h->off_table = off;
    if (d->mode == DSQ_MODE_LUT_ROW)
        off = align_up(off + (uint64_t)d->rows * (1u << d->bits) * 2, kSectionAlign);
    else if (d->mode == DSQ_MODE_BITPLANE)
        off = align_up(off + (uint64_t)d->rows * h->slots * 2, kSectionAlign);
    h->off_row_ptr = off;
    off = align_up(off + (uint64_t)(d->rows + 1) * 4, kSectionAlign);
    h->off_csr = off;
    // +16: kernels copy 16-byte-aligned spans, up to 12 bytes past the end
    off = align_up(off + (uint64_t)d->nnz * 4 + 16, kSectionAlign);
    h->flags = flags;
    if (flags & kFlagTwoAxis) {
        h->off_rscale = off;
        off = align_up(off + (uint64_t)d->rows * 2, kSectionAlign);
        h->off_cscale = off;
        off = align_up(off + (uint64_t)d->cols * 2 + 16, kSectionAlign);
    }
    h->total = off;
}

int parse_blob(const void *packed, size_t bytes, BlobHeader *out) {
    if (!packed || bytes < kHeaderBytes) return DSQ_ERR_INVALID_ARG;
    BlobHeader h;
    memcpy(&h, packed, sizeof(h));
    if (memcmp(h.magic, kMagic, sizeof(kMagic)) != 0 || h.version != kVersion ||
        h.header_bytes != kHeaderBytes || (h.flags & ~kFlagTwoAxis) != 0)
        return DSQ_ERR_INVALID_ARG;
    dsq_desc d = {h.rows, h.cols, h.bits, h.mode, h.nnz};
    int rc = check_desc(&d);
    if (rc != DSQ_OK) return rc;
    if (h.mode == DSQ_MODE_INTGRID && (h.flags != 0 || h.nsym == 0 || h.nsym > 2 * kIntGridMax + 1))
        return DSQ_ERR_INVALID_ARG;
    BlobHeader want;
    plan_blob(&d, &want, h.flags, h.stream_words, h.nsym);
    if (want.slots != h.slots || want.row_words != h.row_words || want.off_dense != h.off_dense ||
        want.off_table != h.off_table || want.off_row_ptr != h.off_row_ptr ||
        want.off_csr != h.off_csr || h.reserved0 != 0 || want.off_rscale != h.off_rscale ||
        want.off_cscale != h.off_cscale || want.off_index != h.off_index ||
        want.off_codebook != h.off_codebook || want.total != h.total || h.total > bytes)
        return DSQ_ERR_INVALID_ARG;
    *out = h;
    return DSQ_OK;
}

// The blob contents the kernels index by: row_ptr (from 0 to nnz, never
// decreasing) and the CSR columns (below cols, strictly increasing within a
// row).  Codes, tables, scales and zero points are safe for any bit pattern.
// Host-side, O(rows + nnz); the blob may sit at any host address.
int check_blob_contents(const void *packed, const BlobHeader &h) {
    const uint8_t *b = (const uint8_t *)packed;
    auto rp = [&](int64_t i) {
        int32_t v;
        memcpy(&v, b + h.off_row_ptr + 4 * i, 4);
        return (int64_t)v;
    };
    auto col = [&](int64_t k) {
        uint32_t v;
        memcpy(&v, b + h.off_csr + 4 * k, 4);
        return (int64_t)(v & 0xffffu);
    };
    if (rp(0) != 0 || rp(h.rows) != h.nnz) return DSQ_ERR_INVALID_ARG;
    for (int64_t i = 0; i < h.rows; i++) {
        const int64_t k0 = rp(i), k1 = rp(i + 1);
        if (k1 < k0) return DSQ_ERR_INVALID_ARG;
        int64_t prev = -1;
        for (int64_t k = k0; k < k1; k++) {
            const int64_t c = col(k);
            if (c >= h.cols || c <= prev) return DSQ_ERR_INVALID_ARG;
            prev = c;
        }
    }
    return DSQ_OK;
}

}  // namespace dsq

using namespace dsq;

static int pack_impl(const dsq_desc *d, const uint8_t *codes, const uint16_t *table, const uint16_t *zeros,
                     const int32_t *row_ptr, const int32_t *col_idx, const uint16_t *values,
                     const uint16_t *rscale, const uint16_t *cscale, uint32_t flags, void *out,
                     size_t *out_bytes) {
    if (!out_bytes) return DSQ_ERR_INVALID_ARG;
    int rc = check_desc(d);
    if (rc != DSQ_OK) return rc;
    if (d->mode == DSQ_MODE_INTGRID) return DSQ_ERR_INVALID_ARG;  // integers: dsq_pack_intgrid
    const int64_t M = d->rows, N = d->cols, nnz = d->nnz;
    const int bits = d->bits, mode = d->mode, K = 1 << bits, qmax = K - 1;
    const int64_t G = N / kGroup;
    const int64_t GB = mode == DSQ_MODE_BITPLANE ? N / (32 << bits) : 0;  // bit-plane groups per row
    const bool any = M * N > 0;
    if (any && !codes) return DSQ_ERR_INVALID_ARG;
    if (M > 0 && (mode == DSQ_MODE_LUT_ROW || G > 0) && !table) return DSQ_ERR_INVALID_ARG;
    if (mode != DSQ_MODE_AFFINE_G16 && zeros) return DSQ_ERR_INVALID_ARG;
    if (mode == DSQ_MODE_AFFINE_G16 && any && !zeros) return DSQ_ERR_INVALID_ARG;
    if (M > 0 && !row_ptr) return DSQ_ERR_INVALID_ARG;
    if (nnz > 0 && (!col_idx || !values)) return DSQ_ERR_INVALID_ARG;

    // ---- validate every input before writing anything
    for (int64_t t = 0; t < M * N; t++)
        if (codes[t] > qmax) return DSQ_ERR_INVALID_ARG;
    std::vector<uint16_t> levels;  // BITPLANE: rows x GB x K level table
    if (mode == DSQ_MODE_LUT_ROW) {
        for (int64_t t = 0; t < M * K; t++)
            if (!isfinite(half_bits_to_double(table[t]))) return DSQ_ERR_INVALID_ARG;
    } else if (mode == DSQ_MODE_BITPLANE) {
        levels.resize((size_t)(M * GB * K));
        for (int64_t t = 0; t < M * GB; t++) {
            double c[4];
            for (int i = 0; i <= bits; i++) {
                c[i] = half_bits_to_double(table[t * (bits + 1) + i]);
                if (!isfinite(c[i])) return DSQ_ERR_INVALID_ARG;
            }
            for (int q = 0; q < K; q++) {
                double w = c[0];  // fp16 terms: the sum is exact in fp64
                for (int i = 1; i <= bits; i++)
                    if ((q >> (i - 1)) & 1) w += c[i];
                const uint16_t hb = __half_as_ushort(__double2half(w));  // one round-to-nearest-even
                if ((hb & 0x7C00u) == 0x7C00u) return DSQ_ERR_INVALID_ARG;
                levels[(size_t)(t * K + q)] = hb;
            }
        }
    } else {
        for (int64_t t = 0; t < M * G; t++) {
            double s = half_bits_to_double(table[t]);
            double z = half_bits_to_double(zeros[t]);
            if (!isfinite(s) || !(z >= 0 && z <= qmax) || z != floor(z)) return DSQ_ERR_INVALID_ARG;
            double span = fabs(s) * (z > qmax - z ? z : qmax - z);
            if (!(span < 65520.0)) return DSQ_ERR_INVALID_ARG;
        }
    }
    if (M > 0) {
        if (row_ptr[0] != 0 || row_ptr[M] != nnz) return DSQ_ERR_INVALID_ARG;
        for (int64_t i = 0; i < M; i++) {
            if (row_ptr[i + 1] < row_ptr[i]) return DSQ_ERR_INVALID_ARG;
            for (int64_t k = row_ptr[i]; k < row_ptr[i + 1]; k++) {
                if (col_idx[k] < 0 || col_idx[k] >= N) return DSQ_ERR_INVALID_ARG;
                if (k > row_ptr[i] && col_idx[k] <= col_idx[k - 1]) return DSQ_ERR_INVALID_ARG;
            }
        }
    } else if (nnz != 0) {
        return DSQ_ERR_INVALID_ARG;
    }
    for (int64_t k = 0; k < nnz; k++)
        if (!isfinite(half_bits_to_double(values[k]))) return DSQ_ERR_INVALID_ARG;
    if (flags & kFlagTwoAxis) {
        if ((M > 0 && !rscale) || (N > 0 && !cscale)) return DSQ_ERR_INVALID_ARG;
        for (int64_t i = 0; i < M; i++)
            if (!isfinite(half_bits_to_double(rscale[i]))) return DSQ_ERR_INVALID_ARG;
        for (int64_t j = 0; j < N; j++)
            if (!isfinite(half_bits_to_double(cscale[j]))) return DSQ_ERR_INVALID_ARG;
    }

    BlobHeader h;
    plan_blob(d, &h, flags);
    if (!out || *out_bytes < h.total) {
        *out_bytes = h.total;
        return DSQ_ERR_BUFFER_TOO_SMALL;
    }
    *out_bytes = h.total;
    uint8_t *blob = (uint8_t *)out;
    memset(blob, 0, h.total);
    memcpy(blob, &h, sizeof(h));

    // ---- dense row records
    const int S = h.slots;
    int place_word[32][4], place_pos[32][4];
    for (int c = 0; c < 32; c++)
        for (int k = 0; k < bits; k++) code_bit_place(bits, c, k, &place_word[c][k], &place_pos[c][k]);
    for (int64_t i = 0; i < M; i++) {
        uint32_t *rec = (uint32_t *)(blob + h.off_dense) + i * h.row_words;
        for (int s = 0; s < S; s++) {
            uint32_t w[4] = {0, 0, 0, 0};
            for (int c = 0; c < 32; c++) {
                int64_t j = (int64_t)s * 32 + c;
                if (j >= N) break;
                uint32_t q = codes[i * N + j];
                for (int k = 0; k < bits; k++)
                    w[place_word[c][k]] |= ((q >> k) & 1u) << place_pos[c][k];
            }
            for (int p = 0; p < bits; p++) rec[code_word_index(bits, mode, S, s, p)] = w[p];
            if (mode == DSQ_MODE_AFFINE_G16) {
                uint32_t pair = 0, zb = 0;
                for (int e = 0; e < 2; e++) {
                    int64_t g = 2 * (int64_t)s + e;
                    if (g >= G) break;
                    pair |= (uint32_t)table[i * G + g] << (16 * e);
                    zb |= (uint32_t)half_bits_to_double(zeros[i * G + g]) << (4 * e);
                }
                rec[scale_word_index(bits, S, s)] = pair;
                ((uint8_t *)rec)[zero_byte_index(bits, S, s)] = (uint8_t)zb;
            }
        }
    }
    if (mode == DSQ_MODE_LUT_ROW && M > 0) memcpy(blob + h.off_table, table, (size_t)M * K * 2);
    if (mode == DSQ_MODE_BITPLANE && M > 0) memcpy(blob + h.off_table, levels.data(), levels.size() * 2);
    if (M > 0) memcpy(blob + h.off_row_ptr, row_ptr, (size_t)(M + 1) * 4);
    else memset(blob + h.off_row_ptr, 0, 4);
    uint32_t *csr = (uint32_t *)(blob + h.off_csr);
    for (int64_t k = 0; k < nnz; k++) csr[k] = (uint32_t)(uint16_t)col_idx[k] | ((uint32_t)values[k] << 16);
    if (flags & kFlagTwoAxis) {
        if (M > 0) memcpy(blob + h.off_rscale, rscale, (size_t)M * 2);
        if (N > 0) memcpy(blob + h.off_cscale, cscale, (size_t)N * 2);
    }
    return DSQ_OK;
}

extern "C" int dsq_pack(const dsq_desc *d, const uint8_t *codes, const uint16_t *table,
                        const uint16_t *zeros, const int32_t *row_ptr, const int32_t *col_idx,
                        const uint16_t *values, void *out, size_t *out_bytes) {
    return pack_impl(d, codes, table, zeros, row_ptr, col_idx, values, nullptr, nullptr, 0, out, out_bytes);
}

extern "C" int dsq_pack_two_axis(const dsq_desc *d, const uint8_t *codes, const uint16_t *table,
                                 const uint16_t *zeros, const int32_t *row_ptr, const int32_t *col_idx,
                                 const uint16_t *values, const uint16_t *row_scale, const uint16_t *col_scale,
                                 void *out, size_t *out_bytes) {
    return pack_impl(d, codes, table, zeros, row_ptr, col_idx, values, row_scale, col_scale, kFlagTwoAxis, out,
                     out_bytes);
}

extern "C" int dsq_blob_desc(const void *packed, size_t bytes, dsq_desc *out) {
    if (!out) return DSQ_ERR_INVALID_ARG;
    BlobHeader h;
    int rc = parse_blob(packed, bytes, &h);
    if (rc != DSQ_OK) return rc;
    out->rows = h.rows;
    out->cols = h.cols;
    out->bits = h.bits;
    out->mode = h.mode;
    out->nnz = h.nnz;
    return DSQ_OK;
}
