// Shared constants and helpers of libsherry_b200 (not part of the C ABI).
#pragma once

#include <cstddef>
#include <cstdint>

// Kernel-native weight layout.  Rows are grouped in tiles of 128 (the M of a
// tcgen05 MMA, one TMEM lane per row) and K in chunks of 128 weights
// (32 groups = 160 bits = 5 words per row).  Word j of (row r, chunk c) holds
// canonical stream bytes [20c + 4j, 20c + 4j + 4) of row r, little endian, so
// group g of the chunk sits at bits [5g, 5g+5) of the 160-bit concatenation
// of the 5 words.  Memory order: [row tile][chunk][word j][position p], and
// plane j is rotated by 8j rows: row r's word j sits at position
// (r + 8j) mod 128.  A warp reading one word of 32 consecutive rows, and a
// warp of mma.sync A-fragment lanes reading words c and c+1 of rows g, g+8
// (lane = 4g + c), both touch 32 distinct shared-memory banks.
#define SHERRY_TILE_ROWS 128
#define SHERRY_KCHUNK 128
#define SHERRY_CHUNK_WORDS 5
#define SHERRY_CHUNK_BYTES_PER_TILE (SHERRY_TILE_ROWS * SHERRY_CHUNK_WORDS * 4)

// W4A8 (SINT4 weights) kernel-native layout: the same row tiles and K chunks;
// one (tile, chunk) block is 8192 bytes, [piece q 0..3][row r 0..127][word i
// 0..3] of 32-bit words.  Word i of piece q of row r covers k0 = 32q + 8i
// within the chunk: byte b holds w[k0 + b] in its low nibble and w[k0 + 4 + b]
// in its high nibble.  So (word << 4) & 0xF0F0F0F0 and word & 0xF0F0F0F0 are
// the int8 values 16 w of k0..k0+3 and k0+4..k0+7, and a warp loading the
// 16-byte pieces of 32 consecutive rows reads 512 contiguous bytes.
#define SHERRY_W4_CHUNK_BYTES (SHERRY_TILE_ROWS * SHERRY_KCHUNK / 2)
// Largest K of the W4A8 path: |sum of q * 16 w| <= 127 * 128 * K below 2^31.
#define SHERRY_W4_MAX_K int64_t(132104)

// Largest supported K: keeps |acc| <= 127 * 0.75 * K below 2^31.
#define SHERRY_MAX_K (int64_t(1) << 24)
#define SHERRY_MAX_DIM ((int64_t(1) << 31) - 1)

#ifdef __CUDACC__
#define SHERRY_HD __host__ __device__
#else
#define SHERRY_HD
#endif

inline bool sherry_shape_ok(int64_t M, int64_t N, int64_t K)
{
    return M >= 1 && N >= 1 && K >= 1 && K % 32 == 0 && K <= SHERRY_MAX_K &&
           M <= SHERRY_MAX_DIM && N <= SHERRY_MAX_DIM;
}

SHERRY_HD inline int64_t sherry_row_tiles(int64_t N) { return (N + SHERRY_TILE_ROWS - 1) / SHERRY_TILE_ROWS; }
SHERRY_HD inline int64_t sherry_k_chunks(int64_t K) { return (K + SHERRY_KCHUNK - 1) / SHERRY_KCHUNK; }
// Word index of (word j, row r) inside one (tile, chunk) block.
SHERRY_HD inline int sherry_word_pos(int j, int r)
{
    return j * SHERRY_TILE_ROWS + ((r + 8 * j) & (SHERRY_TILE_ROWS - 1));
}

// Word index of (piece q, row r, word i) inside one W4A8 (tile, chunk) block.
SHERRY_HD inline int sherry_w4_word_index(int q, int r, int i) { return (q * SHERRY_TILE_ROWS + r) * 4 + i; }

// Byte offset of the 16-byte piece p (k = 32p .. 32p+31) of row n in the
// native W4A8 layout: chunk c = p / 4, piece q = p % 4 of that chunk.
SHERRY_HD inline int64_t sherry_w4_piece_offset(int64_t n, int64_t Kc, int64_t p)
{
    const int64_t t = n / SHERRY_TILE_ROWS, r = n % SHERRY_TILE_ROWS;
    return (t * Kc + (p >> 2)) * SHERRY_W4_CHUNK_BYTES + (p & 3) * (SHERRY_TILE_ROWS * 16) + 16 * r;
}

// Native W4A8 word `idx` built from canonical SINT4 rows w4 [N][K/2] (even k
// in the low nibble), K % 32 == 0, Kc = K chunks.  Rows past N and chunks
// past K give 0.
SHERRY_HD inline uint32_t sherry_w4_native_word(const uint8_t* w4, int64_t N, int64_t K, int64_t Kc, int64_t idx)
{
    const int i = (int)(idx & 3);
    const int r = (int)((idx >> 2) & (SHERRY_TILE_ROWS - 1));
    const int q = (int)((idx >> 9) & 3);
    const int64_t blk = idx >> 11;                         // (tile, chunk) block of 2048 words
    const int64_t c = blk % Kc, t = blk / Kc;
    const int64_t n = t * SHERRY_TILE_ROWS + r;
    const int64_t k0 = c * SHERRY_KCHUNK + 32 * q + 8 * i;
    if (n >= N || k0 >= K) return 0u;                      // K % 32 == 0: all 8 weights are in range
    const uint8_t* src = w4 + n * (K / 2) + k0 / 2;
    uint32_t u = 0;                                        // nibble e = w[k0 + e]
    for (int b = 0; b < 4; ++b) u |= (uint32_t)src[b] << (8 * b);
    uint32_t w = 0;
    for (int b = 0; b < 4; ++b) w |= (((u >> (4 * b)) & 0xFu) | (((u >> (16 + 4 * b)) & 0xFu) << 4)) << (8 * b);
    return w;
}

// Codes reported through sherry_last_device_status when a bounded wait runs out.
enum sherry_device_code : unsigned {
    SHERRY_DEV_OK = 0,
    SHERRY_DEV_TIMEOUT_PRODUCER = 0x101,
    SHERRY_DEV_TIMEOUT_DECODER = 0x102,
    SHERRY_DEV_TIMEOUT_MMA = 0x103,
    SHERRY_DEV_TIMEOUT_EPILOGUE = 0x104,
    SHERRY_DEV_TIMEOUT_DRAIN = 0x105,
    SHERRY_DEV_TMEM_ALLOC = 0x106,
    SHERRY_DEV_TIMEOUT_SELFTEST = 0x107,
};
