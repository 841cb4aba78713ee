// layout.h -- the packed blob written by dsq_pack and read by the kernels.
//
// The blob is a 256-byte header followed by 256-byte-aligned sections:
//
//   dense    rows x row_words u32: one "row record" per output row
//   table    LUT_ROW: rows x 2^bits fp16 centroids, as given;
//            BITPLANE: rows x S fp16 levels -- for every group of 2^bits
//            slots (32 * 2^bits columns) its 2^bits levels
//            fp16(C0 + sum_i C_i b_i), entry g * 2^bits + q
//   row_ptr  int32 [rows+1]
//   csr      uint32 [nnz]   one outlier per word: column index in bits 0..15
//                           (cols <= 65535), fp16 value in bits 16..31
//   INTGRID (Huffman-coded integers on one grid) replaces the dense and table
//   sections: dense = the MSB-first bitstream of all rows (stream_words u32
//   + kStreamPad words of padding), table = fp16 scales [rows][cols/16],
//   index = u32 [rows][S] bit offset of each slot's first code, codebook =
//   the canonical code (see huffman.cu)
//   rscale   two-axis blobs only: fp16 [rows], the row scales r
//   cscale   two-axis blobs only: fp16 [cols], the column scales c
//
// Row record.  The columns of a row are cut into S = ceil(cols/32) "slots"
// of 32 consecutive columns; the tail slot is padded with code 0 (and, in
// affine mode, scale 0 / zero 0 for the padded group).  One slot carries
// 32 codes in `bits` u32 code words.  Within a record, per mode:
//
//   LUT_ROW, 3 bit:    3 planes of S words: word p of slot s at [p*S + s]
//   BITPLANE, 2/3 bit: 2/3 planes of S words, as LUT_ROW 3 bit
//   LUT_ROW, 4 bit:    S uint4 (4 code words) at [4s .. 4s+3]
//   AFFINE_G16, 3 bit: groups of 32 slots, 136 words apart: group g holds
//                      the zero bytes of its slots (8 words; byte t =
//                      zero byte of slot 32g + t), then one uint4 per slot
//                      = (code word 0, 1, 2, scale pair) at [136g + 8 + 4t];
//                      the last group holds only its S - 32g slots
//   AFFINE_G16, 4 bit: S uint4 code words, then S scale-pair words at [4S+s],
//                      then S zero bytes starting at word 5S
//
// A zero byte is zero[2s] | zero[2s+1] << 4, a scale pair is
// scale[2s] | scale[2s+1] << 16 (the two groups of 16 in the slot).  Records
// are padded to a multiple of 4 words, so every record and every uint4
// starts on a 16-byte boundary.  (The 3-bit affine grouping gives the 32
// lanes that stream one group a single base address: zero bytes at +0,
// their slot at +32 + 16*lane.)
//
// Code bits inside a slot.  4-bit: column c in word c/8, bits 4(c%8)..+3.
// 2-bit: column c in word c/16, bits 2(c%16)..+1.
// 3-bit: word w (0..2) holds columns 10w..10w+9 as five adjacent pairs; pair
// j (columns 10w+2j, 10w+2j+1) sits at half-word bit h_j of the low half
// (even column) and of the high half (odd column), h = 0, 3, 6, 10, 13.  One
// mask therefore pulls both codes of a pair into the two 16-bit halves of a
// word, and since pairs 0..2 lie in bits 0..9 of each half -- and pairs 3, 4
// do in the word shifted right by 10 -- an AND alone turns a pair into two
// exact fp16 subnormals (q * 2^(h-24)).  Columns 30 and 31 use the spare
// bits: bit k of column 30 is bit 9 of word k, bit k of column 31 is bit 25
// of word k.
#pragma once
#include <stdint.h>

#ifndef __CUDACC__
#define __host__
#define __device__
#endif

namespace dsq {

constexpr char kMagic[8] = {'D', 'S', 'Q', 'B', 'L', 'O', 'B', '1'};
constexpr uint32_t kFlagTwoAxis = 1;  // header flag: the blob holds row and column scales
constexpr int kModeIntGrid = 3;        // dsq mode of Huffman-coded integer grids
constexpr int kHuffMaxLen = 20;        // longest code
constexpr int kHuffFastBits = 10;      // codes this short decode with one table read
constexpr int kStreamPad = 24;         // words after the stream: a slot's 32 codes never read past it
constexpr int kIntGridMax = 8191;      // |q| bound: scale * q is exact in fp32
// codebook words: [0] nsym, [1] max_len, then first code, count and first
// symbol index per length 0..kHuffMaxLen, the fast table (entry = length << 16
// | the integer as int16, length 0 for codes longer than kHuffFastBits), the
// symbols (int16)
constexpr int kCbFirst = 2, kCbCount = kCbFirst + kHuffMaxLen + 1, kCbOffset = kCbCount + kHuffMaxLen + 1;
constexpr int kCbFast = kCbOffset + kHuffMaxLen + 1, kCbSyms = kCbFast + (1 << kHuffFastBits);
constexpr uint32_t kVersion = 1;
constexpr uint32_t kHeaderBytes = 256;
constexpr uint64_t kSectionAlign = 256;
constexpr int kSlotCols = 32;
constexpr int kGroup = 16;

struct BlobHeader {
    char magic[8];
    uint32_t version;
    uint32_t header_bytes;
    int32_t rows, cols, bits, mode;
    int64_t nnz;
    int32_t slots;      // S
    int32_t row_words;  // u32 words per row record (multiple of 4)
    uint64_t off_dense, off_table, off_row_ptr, off_csr, reserved0, total;
    uint64_t off_rscale, off_cscale;  // two-axis blobs; 0 otherwise
    uint32_t flags, pad0;
    // INTGRID blobs (Huffman-coded integers): the slot bit offsets, the
    // codebook, the bitstream length in words and the alphabet size
    uint64_t off_index, off_codebook;
    uint32_t stream_words, nsym;
    uint8_t reserved[kHeaderBytes - 8 - 4 - 4 - 16 - 8 - 8 - 48 - 24 - 24];
};
static_assert(sizeof(BlobHeader) == kHeaderBytes, "header size");

__host__ __device__ inline int slots_of(int cols) { return (cols + kSlotCols - 1) / kSlotCols; }

constexpr int kAff3GroupWords = 136;  // 8 words of zero bytes + 32 slot uint4

__host__ __device__ inline int row_words_of(int bits, int mode, int S) {
    int w;
    if (mode == kModeIntGrid) return 0;  // variable length: the stream has no fixed row records
    if (mode != 1)
        w = bits * S;
    else if (bits == 3)
        w = S == 0 ? 0 : kAff3GroupWords * ((S - 1) / 32) + 8 + 4 * (S - 32 * ((S - 1) / 32));
    else
        w = 5 * S + (S + 3) / 4;
    return (w + 3) & ~3;
}

// Byte offset (inside a record) of the zero byte of slot s (affine only).
__host__ __device__ inline int zero_byte_index(int bits, int S, int s) {
    return bits == 3 ? 4 * kAff3GroupWords * (s / 32) + (s % 32) : 4 * 5 * S + s;
}

// Position of bit k (0 = least significant) of column c's code inside a
// slot: returns the code word index (0..bits-1) and the bit position.
__host__ __device__ inline void code_bit_place(int bits, int c, int k, int *word, int *pos) {
    if (bits == 4) {
        *word = c >> 3;
        *pos = 4 * (c & 7) + k;
        return;
    }
    if (bits == 2) {
        *word = c >> 4;
        *pos = 2 * (c & 15) + k;
        return;
    }
    if (c < 30) {
        const int t = c % 10, j = t >> 1;
        *word = c / 10;
        *pos = (t & 1 ? 16 : 0) + (j < 3 ? 3 * j : 3 * j + 1) + k;
        return;
    }
    *word = k;
    *pos = c == 30 ? 9 : 25;
}

// Word index (inside a record) of code word p of slot s.
__host__ __device__ inline int code_word_index(int bits, int mode, int S, int s, int p) {
    if ((bits == 3 && mode == 0) || mode == 2) return p * S + s;
    if (bits == 3) return kAff3GroupWords * (s / 32) + 8 + 4 * (s % 32) + p;
    return 4 * s + p;
}

// Word index of the scale pair of slot s (affine only).
__host__ __device__ inline int scale_word_index(int bits, int S, int s) {
    return bits == 3 ? code_word_index(3, 1, S, s, 3) : 4 * S + s;
}

}  // namespace dsq
