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

// Codes reported through sherry_last_device_status when a bounded wait runs out.
enum sherry_device_code : unsigned {
    SHERRY_DEV_OK = 0,
    SHERRY_DEV_TIMEOUT_PRODUCER = 0x101,
    SHERRY_DEV_TIMEOUT_DECODER = 0x102,
    SHERRY_DEV_TIMEOUT_MMA = 0x103,
    SHERRY_DEV_TIMEOUT_EPILOGUE = 0x104,
    SHERRY_DEV_TIMEOUT_DRAIN = 0x105,
    SHERRY_DEV_TMEM_ALLOC = 0x106,
};
