// Host check of the W4A8 kernel-native layout (sherry_internal.h): builds the
// native words of random canonical SINT4 rows with sherry_w4_native_word, then
// does what the tensor-core kernel's decoder warps do with them (16-byte piece
// loads per row, (v << 4) & 0xF0F0F0F0 and v & 0xF0F0F0F0 as TMEM columns
// 8q + 2i and 8q + 2i + 1) and checks every int8 against 16 w[n][k], zeros
// past N and K, and that 8 consecutive rows' 16-byte loads cover 128
// contiguous bytes (one shared-memory wavefront per quarter warp).
#include <cstdint>
#include <cstdio>
#include <vector>

#include "sherry_internal.h"

static uint64_t rng = 88172645463325252ull;
static uint32_t next_u32()
{
    rng ^= rng << 13;
    rng ^= rng >> 7;
    rng ^= rng << 17;
    return (uint32_t)rng;
}

static int check(int64_t N, int64_t K)
{
    std::vector<int> w((size_t)(N * K));
    std::vector<uint8_t> canon((size_t)(N * K / 2));
    for (auto& v : w) v = (int)(next_u32() % 16) - 8;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t j = 0; j < K / 2; ++j)
            canon[n * (K / 2) + j] =
                (uint8_t)((w[n * K + 2 * j] & 15) | ((w[n * K + 2 * j + 1] & 15) << 4));
    const int64_t TN = sherry_row_tiles(N), Kc = sherry_k_chunks(K);
    const int64_t words = TN * Kc * SHERRY_W4_CHUNK_BYTES / 4;
    std::vector<uint32_t> nat((size_t)words);
    for (int64_t idx = 0; idx < words; ++idx) nat[idx] = sherry_w4_native_word(canon.data(), N, K, Kc, idx);
    const uint8_t* bytes = reinterpret_cast<const uint8_t*>(nat.data());
    for (int64_t t = 0; t < TN; ++t)
        for (int64_t c = 0; c < Kc; ++c) {
            const uint8_t* blk = bytes + (t * Kc + c) * SHERRY_W4_CHUNK_BYTES;
            for (int row = 0; row < SHERRY_TILE_ROWS; ++row) {
                const int64_t n = t * SHERRY_TILE_ROWS + row;
                for (int q = 0; q < 4; ++q) {
                    const uint8_t* piece = blk + q * SHERRY_TILE_ROWS * 16 + 16 * row;
                    if (piece != blk + 4 * sherry_w4_word_index(q, row, 0)) return 10;
                    // the GEMV kernel's address of the same piece
                    if (piece != bytes + sherry_w4_piece_offset(n, Kc, 4 * c + q)) return 12;
                    for (int i = 0; i < 4; ++i) {
                        uint32_t v = 0;
                        for (int b = 0; b < 4; ++b) v |= (uint32_t)piece[4 * i + b] << (8 * b);
                        const uint32_t col[2] = {(v << 4) & 0xF0F0F0F0u, v & 0xF0F0F0F0u};
                        for (int h = 0; h < 2; ++h) {
                            const int column = 8 * q + 2 * i + h;     // TMEM column = group of 4 k
                            for (int b = 0; b < 4; ++b) {
                                const int64_t k = c * SHERRY_KCHUNK + 4 * column + b;
                                const int got = (int)(int8_t)(uint8_t)(col[h] >> (8 * b));
                                const int want = (n < N && k < K) ? 16 * w[n * K + k] : 0;
                                if (got != want) {
                                    std::printf("mismatch N=%lld K=%lld n=%lld k=%lld got %d want %d\n",
                                                (long long)N, (long long)K, (long long)n, (long long)k, got, want);
                                    return 1;
                                }
                            }
                        }
                    }
                }
            }
            // quarter-warp rows 8j..8j+7 read 128 contiguous bytes per piece
            for (int q = 0; q < 4; ++q)
                for (int r0 = 0; r0 < SHERRY_TILE_ROWS; r0 += 8)
                    if (4 * sherry_w4_word_index(q, r0 + 7, 0) - 4 * sherry_w4_word_index(q, r0, 0) != 7 * 16) return 11;
        }
    return 0;
}

int main()
{
    const int64_t shapes[][2] = {{1, 32}, {128, 128}, {129, 160}, {300, 4096}, {37, 96}, {256, 8192}, {5, 14336}};
    for (auto& s : shapes) {
        const int rc = check(s[0], s[1]);
        if (rc) {
            std::printf("fail %d at N=%lld K=%lld\n", rc, (long long)s[0], (long long)s[1]);
            return rc;
        }
    }
    std::printf("ok\n");
    return 0;
}
