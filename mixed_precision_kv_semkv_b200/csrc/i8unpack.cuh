// Base-L code words -> one byte per code, for the decode on the integer tensor cores.
//
// SemKV page, Abstract: codes live on L-level grids whose L need not be a power of two, packed as
// base-L radix words (k(L) digits per 32-bit word).  The decode's 8-bit tensor-core operands need
// each code in a byte of its own.  A 128-code row (the K codes of one slot, or the V codes of one
// channel in a 128-slot tile) is held in W = ceil(128/k) words; digit i of word j is row position
// j*k + i.  unpack_row_u8 turns the row into 32 registers of 4 bytes: byte b of register r holds
// the code at row position row_index<L>(4r + b).  That order serves speed; row_index and its
// inverse row_pos let the other operand of each product be laid out to match.
//
//  - L = 4, 16: bit fields, split with masks (no table).
//  - otherwise each word becomes the 32-bit fixed-point fraction f ~ w / L^k (the method of
//    common.cuh; for L = 8 an exact shift), its zero padding digits (row positions past 128, only
//    in the last word) are dropped by one multiply by L^pad, and its digits are taken most
//    significant first, C at a time: one 32x32->64 multiply by L^C gives the next C digits as a
//    table index in the high half and the remaining fraction in the low half.  A per-lane copy of
//    a table in shared memory maps the index to C bytes (digit i of the chunk in byte i): C = 4
//    for L = 5 (625 entries), C = 3 for L = 6 and 8 (216, 512 entries).  Digits that do not fill a
//    chunk are taken one at a time (high half of a multiply by L).
//  - chunk bytes fill the row from position 0 in extraction order; the single digits follow.
#pragma once

#include <stdint.h>

#include "common.cuh"

namespace semkv {

template <int L>
struct U8Plan {
    static constexpr int k = radix_k(L);
    static constexpr int W = ceil_div(128, k);
    static constexpr bool masks = (L == 4 || L == 16);
    static constexpr int C = masks ? 0 : (L <= 5 ? 4 : 3);
    static constexpr int ENTRIES = C ? (int)ipow(L, C) : 0;
    static constexpr uint32_t LC = C ? (uint32_t)ipow(L, C) : 0u;
    static constexpr uint32_t LUT_BYTES = (uint32_t)ENTRIES * 128u;  // 32 lane copies of 4-byte entries
    // the table path needs the fraction method (or L = 8, whose fraction is a shift)
    static constexpr bool ok = masks || L == 5 || L == 6 || L == 8;

    __host__ __device__ static constexpr int real(int j) { return 128 - j * k < k ? 128 - j * k : k; }
    __host__ __device__ static constexpr int chunks(int j) { return C ? real(j) / C : 0; }
    __host__ __device__ static constexpr int singles(int j) { return C ? real(j) % C : 0; }
    // every word but the last has k real digits: positions in closed form
    __host__ __device__ static constexpr int chunk_pos(int j, int c) { return (j * chunks(0) + c) * C; }
    __host__ __device__ static constexpr int chunk_bytes() { return ((W - 1) * chunks(0) + chunks(W - 1)) * C; }
    __host__ __device__ static constexpr int single_pos(int j, int s) { return chunk_bytes() + j * singles(0) + s; }
};

__host__ __device__ __forceinline__ uint32_t mulhi_u32(uint32_t a, uint32_t b)
{
    return (uint32_t)(((unsigned long long)a * (unsigned long long)b) >> 32);
}

// Row position held at operand byte `pos` (0..127).
template <int L>
__host__ __device__ inline int row_index(int pos)
{
    using P = U8Plan<L>;
    const int r = pos >> 2, b = pos & 3;
    if constexpr (L == 16) {
        return (r >> 1) * 8 + 2 * b + (r & 1);
    } else if constexpr (L == 4) {
        return (r >> 2) * 16 + 4 * b + (r & 3);
    } else {
        if (pos < P::chunk_bytes()) {
            const int ci = pos / P::C, i = pos % P::C;
            int j = ci / P::chunks(0), c = ci % P::chunks(0);
            if (j > P::W - 1) {  // (only reached when the last word has fewer chunks)
                j = P::W - 1;
                c = ci - (P::W - 1) * P::chunks(0);
            }
            return j * P::k + P::real(j) - P::C * (c + 1) + i;
        }
        const int si = pos - P::chunk_bytes();
        constexpr int S0 = P::singles(0) > 0 ? P::singles(0) : 1;  // singles of a full word
        int j, s;
        if (P::singles(0) > 0 && si < (P::W - 1) * P::singles(0)) {
            j = si / S0;
            s = si % S0;
        } else {
            j = P::W - 1;
            s = si - (P::W - 1) * P::singles(0);
        }
        return j * P::k + P::singles(j) - 1 - s;
    }
}

// Operand byte that holds row position t (the inverse of row_index).
template <int L>
__host__ __device__ inline int row_pos(int t)
{
    using P = U8Plan<L>;
    if constexpr (L == 16) {
        const int j = t >> 3, i = t & 7;
        return 4 * (2 * j + (i & 1)) + (i >> 1);
    } else if constexpr (L == 4) {
        const int j = t >> 4, i = t & 15;
        return 4 * (4 * j + (i & 3)) + (i >> 2);
    } else {
        const int j = t / P::k, i = t % P::k;
        if (i >= P::singles(j)) {
            const int c = (P::real(j) - 1 - i) / P::C;
            return P::chunk_pos(j, c) + (i - (P::real(j) - P::C * (c + 1)));
        }
        return P::single_pos(j, P::singles(j) - 1 - i);
    }
}

// Table entry e: the C base-L digits of e, digit i in byte i.
template <int L>
__host__ __device__ inline uint32_t u8_entry(uint32_t e)
{
    uint32_t v = 0;
#pragma unroll
    for (int i = 0; i < U8Plan<L>::C; ++i) {
        v |= (e % (uint32_t)L) << (8 * i);
        e /= (uint32_t)L;
    }
    return v;
}

// the bytes of {b, a} (b high) picked by selector s (byte i of the result = byte s_i of the pair)
__host__ __device__ __forceinline__ uint32_t byte_perm(uint32_t a, uint32_t b, uint32_t s)
{
#ifdef __CUDA_ARCH__
    return __byte_perm(a, b, s);
#else
    const unsigned long long x = ((unsigned long long)b << 32) | a;
    uint32_t r = 0;
    for (int i = 0; i < 4; ++i) r |= (uint32_t)((x >> (8 * ((s >> (4 * i)) & 7))) & 0xFFu) << (8 * i);
    return r;
#endif
}

// place NB bytes of v at operand byte `pos` (a compile-time constant after unrolling)
template <int NB>
__host__ __device__ __forceinline__ void place_bytes(uint32_t (&out)[32], int pos, uint32_t v)
{
    const int reg = pos >> 2, off = pos & 3;
    out[reg] |= v << (8 * off);
    if (off + NB > 4) out[reg + 1] |= v >> (8 * (4 - off));
}

// a * b + c (low 32 bits), hi(a * b) + c, and the full 64-bit a * b, as single multiply-adds
__host__ __device__ __forceinline__ uint32_t mad_lo(uint32_t a, uint32_t b, uint32_t c)
{
#ifdef __CUDA_ARCH__
    uint32_t d;
    asm("mad.lo.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
#else
    return a * b + c;
#endif
}
__host__ __device__ __forceinline__ uint32_t mad_hi(uint32_t a, uint32_t b, uint32_t c)
{
#ifdef __CUDA_ARCH__
    uint32_t d;
    asm("mad.hi.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
#else
    return mulhi_u32(a, b) + c;
#endif
}
__host__ __device__ __forceinline__ void mul_wide(uint32_t a, uint32_t b, uint32_t& hi, uint32_t& lo)
{
#ifdef __CUDA_ARCH__
    unsigned long long d;
    asm("mul.wide.u32 %0, %1, %2;" : "=l"(d) : "r"(a), "r"(b));
    hi = (uint32_t)(d >> 32);
    lo = (uint32_t)d;
#else
    const unsigned long long d = (unsigned long long)a * b;
    hi = (uint32_t)(d >> 32);
    lo = (uint32_t)d;
#endif
}

// The 32-bit fixed-point fraction of a word (within one unit of the last digit; exact for L = 8).
template <int L>
__host__ __device__ __forceinline__ uint32_t u8_fraction(uint32_t w)
{
    using R = Radix<L>;
    if constexpr (R::pow2) {
        return w << (32 - R::bits * R::k);
    } else {
        return mad_lo(w, R::r_int, mad_hi(w, R::c_frac, 1u));
    }
}

// The operand registers that a row's unpack completes with word j (for stores in blocks of 8):
// the last word that writes into block b (registers 8b .. 8b + 7).
template <int L>
__host__ __device__ constexpr int block_done_word(int b)
{
    using P = U8Plan<L>;
    int last = 0;
    for (int j = 0; j < P::W; ++j) {
        if (P::masks) {
            const int regs = L == 16 ? 2 : 4;  // registers written by word j
            if (j * regs <= 8 * b + 7 && (j + 1) * regs > 8 * b) last = j;
            continue;
        }
        for (int c = 0; c < P::chunks(j); ++c) {
            if (P::C == 4) {
                const int r = P::chunk_pos(j, c) / 4;
                if (r / 8 == b) last = j;
            } else {  // a group of 4 three-byte chunks writes registers 3g .. 3g + 2 with its last chunk
                const int ci = P::chunk_pos(j, c) / 3, nch = P::chunk_bytes() / 3;
                if ((ci & 3) == 3 || ci == nch - 1) {
                    const int r0 = 3 * (ci >> 2);
                    if (r0 <= 8 * b + 7 && r0 + 2 >= 8 * b) last = j;
                }
            }
        }
        for (int s = 0; s < P::singles(j); ++s)
            if (P::single_pos(j, s) / 32 == b) last = j;
    }
    return last;
}

// block_done_word<L>(B) as a compile-time constant
template <int L, int B>
struct U8BlockDone {
    static constexpr int value = block_done_word<L>(B);
};

// One row: words wv[0..W) -> out[32].  lut(idx) returns table entry idx; done(j) runs after word
// j (its bytes and every earlier word's are in place).
template <int L, class Lut, class Done>
__host__ __device__ __forceinline__ void unpack_row_u8(const uint32_t* wv, Lut lut, uint32_t (&out)[32], Done done)
{
    using P = U8Plan<L>;
    if constexpr (L == 16) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            out[2 * j] = wv[j] & 0x0F0F0F0Fu;
            out[2 * j + 1] = (wv[j] >> 4) & 0x0F0F0F0Fu;
            done(j);
        }
    } else if constexpr (L == 4) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
#pragma unroll
            for (int s = 0; s < 4; ++s) out[4 * j + s] = (wv[j] >> (2 * s)) & 0x03030303u;
            done(j);
        }
    } else {
#pragma unroll
        for (int r = 0; r < 32; ++r) out[r] = 0u;
        uint32_t pend[4] = {0u, 0u, 0u, 0u};  // 3-byte chunks waiting to be joined
#pragma unroll
        for (int j = 0; j < P::W; ++j) {
            uint32_t f = u8_fraction<L>(wv[j]);
            if (P::k - P::real(j) > 0) f *= (uint32_t)ipow(L, P::k - P::real(j));  // drop the zero padding digits
#pragma unroll
            for (int c = 0; c < P::chunks(j); ++c) {
                uint32_t idx;
                if (c + 1 < P::chunks(j) || P::singles(j) > 0) {
                    mul_wide(f, P::LC, idx, f);
                } else {
                    idx = mulhi_u32(f, P::LC);
                }
                if constexpr (P::C == 4) {
                    out[P::chunk_pos(j, c) >> 2] = lut(idx);  // whole registers
                } else {
                    // 3-byte chunks: every 4 consecutive ones fill 3 registers, joined by byte
                    // permutes once the fourth arrives (and the last few at the end of the stream)
                    const int ci = P::chunk_pos(j, c) / 3, r0 = 3 * (ci >> 2);
                    pend[ci & 3] = lut(idx);
                    if ((ci & 3) == 3) {
                        out[r0] = byte_perm(pend[0], pend[1], 0x4210u);
                        out[r0 + 1] = byte_perm(pend[1], pend[2], 0x5421u);
                        out[r0 + 2] = byte_perm(pend[2], pend[3], 0x6542u);
                    } else if (ci == P::chunk_bytes() / 3 - 1) {
                        // the stream's last register shares its upper bytes with single digits that
                        // earlier words may have placed already
                        if ((ci & 3) == 0) {
                            out[r0] |= pend[0];
                        } else if ((ci & 3) == 1) {
                            out[r0] = byte_perm(pend[0], pend[1], 0x4210u);
                            out[r0 + 1] |= pend[1] >> 8;
                        } else {
                            out[r0] = byte_perm(pend[0], pend[1], 0x4210u);
                            out[r0 + 1] = byte_perm(pend[1], pend[2], 0x5421u);
                            out[r0 + 2] |= pend[2] >> 16;
                        }
                    }
                }
            }
#pragma unroll
            for (int s = 0; s < P::singles(j); ++s) {
                uint32_t d;
                if (s + 1 < P::singles(j)) {
                    mul_wide(f, (uint32_t)L, d, f);
                } else {
                    d = mulhi_u32(f, (uint32_t)L);
                }
                const int pos = P::single_pos(j, s);
                out[pos >> 2] = mad_lo(d, 1u << (8 * (pos & 3)), out[pos >> 2]);  // the byte was zero
            }
            done(j);
        }
    }
}

template <int L, class Lut>
__host__ __device__ __forceinline__ void unpack_row_u8(const uint32_t* wv, Lut lut, uint32_t (&out)[32])
{
    unpack_row_u8<L>(wv, lut, out, [](int) {});
}

}  // namespace semkv
