// Host driver for the byte-unpack of the integer tensor-core decode (csrc/i8unpack.cuh), run by
// tests/test_u8unpack.py on the CPU.  Reads "L nrows" and then, per row, W words (decimal) from
// stdin; prints, per row, the 128 operand bytes in operand order, then one line with row_index of
// every operand byte and one with row_pos of every row position.  Table lookups check their index,
// and every block of 8 registers, taken when block_done_word says it is complete, must equal the
// final registers.
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "../../mixed_precision_kv_semkv_b200/csrc/i8unpack.cuh"

using namespace semkv;

template <int L>
static int run(int nrows)
{
    using P = U8Plan<L>;
    std::vector<uint32_t> table(P::ENTRIES > 0 ? P::ENTRIES : 1);
    for (int e = 0; e < P::ENTRIES; ++e) table[e] = u8_entry<L>((uint32_t)e);
    auto lut = [&](uint32_t idx) -> uint32_t {
        if ((int)idx >= P::ENTRIES) {
            std::printf("BAD_INDEX %u\n", idx);
            std::exit(3);
        }
        return table[idx];
    };
    for (int r = 0; r < nrows; ++r) {
        uint32_t wv[64];
        for (int j = 0; j < P::W; ++j) {
            unsigned long v;
            if (std::scanf("%lu", &v) != 1) return 2;
            wv[j] = (uint32_t)v;
        }
        uint32_t out[32];
        uint32_t stored[32];
        int nstored = 0;
        // the unpack's per-word hook: a block of 8 registers is taken when its last word is done
        unpack_row_u8<L>(wv, lut, out, [&](int j) {
            for (int b = 0; b < 4; ++b)
                if (block_done_word<L>(b) == j) {
                    for (int i = 0; i < 8; ++i) stored[8 * b + i] = out[8 * b + i];
                    ++nstored;
                }
        });
        if (nstored != 4) {
            std::printf("BLOCKS %d\n", nstored);
            std::exit(5);
        }
        for (int i = 0; i < 32; ++i)
            if (stored[i] != out[i]) {
                std::printf("EARLY_BLOCK register %d\n", i);
                std::exit(6);
            }
        for (int pos = 0; pos < 128; ++pos) std::printf("%u ", (out[pos >> 2] >> (8 * (pos & 3))) & 0xFFu);
        std::printf("\n");
    }
    for (int pos = 0; pos < 128; ++pos) std::printf("%d ", row_index<L>(pos));
    std::printf("\n");
    for (int t = 0; t < 128; ++t) std::printf("%d ", row_pos<L>(t));
    std::printf("\n");
    return 0;
}

int main()
{
    int L, nrows;
    if (std::scanf("%d %d", &L, &nrows) != 2) return 2;
    switch (L) {
        case 4: return run<4>(nrows);
        case 5: return run<5>(nrows);
        case 6: return run<6>(nrows);
        case 8: return run<8>(nrows);
        case 16: return run<16>(nrows);
        default: return 4;
    }
}
