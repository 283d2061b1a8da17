// blob_format.h -- layout of a serialized entro blob and of its device image.
//
// Blob (little-endian, version 1):
//   [0, 128)    header (BlobHeader below)
//   [128, 384)  code length of each of the 256 symbols, 0 = symbol absent
//   index       (n_chunks + 1) entries of {u64 start, u64 first_symbol};
//               start = bit offset of the chunk (single stream) or word offset
//               of the chunk (lanes); the last entry holds the totals
//   payload     payload_words x u32, codes MSB-first within each word
//
// Lanes format: a chunk of n_c symbols is split over L = 32 or 64 lanes; lane
// l codes the runs of 8 consecutive symbols at chunk positions 8*L*t + 8*l +
// (0..7), t = 0, 1, ...  Every lane of a chunk is padded with zero bits to the
// chunk's longest lane (W_c words), and word j of lane l sits at
// payload[chunk_start + L*j + l], so one row of 4L bytes holds word j of all
// lanes (the interleaved lanes of the LazyWeights abstract; the run of 8
// makes each lane's output 8 adjacent weights).
//
// Row-tile format (a second reading of the interleaved lanes, made for the
// fused matrix-vector product): the [rows, cols] tensor is cut into tiles of
// L rows by Kc = chunk_symbols / L columns, row groups outer and column tiles
// inner, one tile per chunk.  Lane l of a tile codes row l of the tile, its Kc
// codes (fewer in the last column tile) in column order; lanes past the last
// row of a ragged row group are empty.  Padding and word interleave as in the
// lanes format.  cols and Kc are multiples of 8.  The index's first_symbol is
// the number of symbols in earlier tiles.
//
// Row tiles in consumption order (format 4): the tiles and lane bitstreams of
// the row-tile format, each lane keeping only its own n_l = ceil(bits / 32)
// words.  A chunk is [n_l of every lane: one byte each, two (little-endian)
// when ceil(Kc * max_len / 32) > 255, zero-padded to whole words] [words 0-2
// of every lane as three rows of L words (zero past n_l)] [the later words in
// the order a lock-step reference decoder takes them] [zero words up to a
// multiple of 4].  The reference decoder: a lookup takes the longest run of
// whole codes within kCoPeekBits bits, at most kCoCodes4 (4-bit) or kCoCodes8
// (8-bit) codes, or one longer code alone; a refill point precedes every
// even-numbered lookup of a lane (every lookup when the length limit max_len
// is above kCoRefillEachAbove); the bits a lane's lookups take add up in a count
// that, at a refill point, gives back 32 when it has reached 32, and the lane
// then takes its next word if it has one left; the words taken at one refill
// point are stored in lane order.  The decoder of a warp finds its words with
// a ballot and a population count, so no lane is padded.
#pragma once
#include <stdint.h>

#ifdef __CUDACC__
#define ENTRO_HD __host__ __device__
#else
#define ENTRO_HD
#endif

namespace entro {

constexpr uint32_t kMagic = 0x52544E45u;  // "ENTR"
constexpr uint32_t kVersion = 1;
constexpr int kHeaderBytes = 128;
constexpr int kLengthsBytes = 256;
constexpr int kLanes = 32;                   // lanes of a warp, and the default lane count
constexpr int kMaxLanes = 64;
constexpr int kRun = 8;
constexpr int kStepSymbols = kLanes * kRun;  // 256 symbols per lane step with 32 lanes
constexpr int kMaxLutBits = 12;
constexpr int kMaxLenLimit = 24;
constexpr int64_t kMaxLanesChunk = 16384;
constexpr int64_t kMaxSingleChunk = int64_t(1) << 20;
constexpr double kMaxZero = 16777216.0;  // |zero| <= 2^24
constexpr int kCoPeekBits = 12;          // consumption order: the reference lookup's peek
constexpr int kCoCodes4 = 8, kCoCodes8 = 4;
constexpr int kCoRefillEachAbove = 16;

// consumption order: bytes of a lane's word count in the chunk header
ENTRO_HD inline int co_count_bytes(uint64_t kc, uint32_t max_len) { return (kc * max_len + 31) / 32 <= 255 ? 1 : 2; }
ENTRO_HD inline uint64_t co_header_words(uint64_t lanes, int count_bytes) { return (lanes * count_bytes + 3) / 4; }

#pragma pack(push, 1)
struct BlobHeader {
    uint32_t magic, version, bits, scheme, max_len, format, lanes, run;
    uint64_t rows, cols, n, chunk_symbols, n_chunks;
    uint32_t scale_bits;
    int32_t zero;
    uint64_t payload_words;
    uint8_t reserved[40];
};
#pragma pack(pop)
static_assert(sizeof(BlobHeader) == kHeaderBytes, "header size");

// Row-tile geometry of chunk c.
struct TileGeom {
    int64_t row0, col0, width;  // first row, first column, columns
    int nrows;                  // rows (lanes that hold codes)
    uint64_t first;             // symbols in all earlier tiles
};

inline uint64_t tile_count(uint64_t rows, uint64_t cols, uint64_t lanes, uint64_t chunk_symbols) {
    if (rows == 0 || cols == 0) return 0;
    const uint64_t kc = chunk_symbols / lanes;
    return ((rows + lanes - 1) / lanes) * ((cols + kc - 1) / kc);
}

inline TileGeom tile_geom(uint64_t rows, uint64_t cols, uint64_t lanes, uint64_t chunk_symbols, uint64_t c) {
    const uint64_t kc = chunk_symbols / lanes, per_group = (cols + kc - 1) / kc;
    const uint64_t g = c / per_group, j = c % per_group;
    TileGeom t;
    t.row0 = (int64_t)(g * lanes);
    t.col0 = (int64_t)(j * kc);
    t.nrows = (int)(rows - g * lanes < lanes ? rows - g * lanes : lanes);
    t.width = (int64_t)(cols - j * kc < kc ? cols - j * kc : kc);
    t.first = g * lanes * cols + (uint64_t)t.nrows * j * kc;
    return t;
}

inline uint64_t index_offset() { return kHeaderBytes + kLengthsBytes; }
inline uint64_t payload_offset(uint64_t n_chunks) { return index_offset() + 16 * (n_chunks + 1); }

// Device image of one tensor, all sections 256-byte aligned inside the
// caller's allocation.
//   lut      u32[2^lut_bits]: bits 0..4 code length (0 = longer than
//            lut_bits or no code), bits 8..15 symbol; bits 16..31 are filled
//            in shared memory by the kernels with the bf16 dequantized value
//   slow     u32 limit[32] (left-justified to max_len bits), i32 offs[32],
//            u8 sorted_symbols[256]
//   index    copied verbatim from the blob
//   payload  copied verbatim, followed by kPadWords zero words
constexpr int kPadWords = 64;
constexpr int kSlowBytes = 32 * 4 + 32 * 4 + 256;

inline uint64_t align256(uint64_t v) { return (v + 255) & ~uint64_t(255); }

}  // namespace entro
