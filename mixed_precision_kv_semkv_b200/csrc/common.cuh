// Device-side helpers shared by the libsemkv kernels (sm_100a).
//
// Radix packing: a 32-bit word holds k(L) = max{k : L^k <= 2^32} base-L digits, value
// sum_i c_i L^i with digit 0 the lowest channel (K) or the lowest slot (V).  Unpacking with a
// compile-time L uses one of three exact methods:
//   * L a power of two: bit fields.
//   * L with r = 2^32 / L^k >= golden ratio: the word w is turned into the 32-bit fixed-point
//     base-L fraction f ~ w / L^k (f = floor(r) w + umulhi(w, ceil(frac(r) 2^32)) + 1, which lies
//     in [w r, w r + r) and so within one unit of the last digit), after which each digit is
//     the high half of one 32x32->64 multiply of the running fraction by L, most significant digit
//     first.  Exactness: with f/2^32 = w/L^k + e, 0 <= e < L^-k, the i-th product is
//     c_{k-1-i} + frac(L^(i+1) w/L^k) + L^(i+1) e and the last two terms stay below 1.
//   * otherwise (L = 3, 9, ...): remainder/quotient by the constant L, least significant first.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>
#include <string.h>

namespace semkv {

constexpr int TILE = 128;

__host__ __device__ constexpr int radix_k(int L)
{
    int k = 0;
    unsigned long long p = 1;
    while (p * (unsigned long long)L <= (1ull << 32)) {
        p *= (unsigned long long)L;
        ++k;
    }
    return k;
}

__host__ __device__ constexpr unsigned long long ipow(int L, int k)
{
    unsigned long long p = 1;
    for (int i = 0; i < k; ++i) p *= (unsigned long long)L;
    return p;
}

__host__ __device__ constexpr int ceil_div(int a, int b) { return (a + b - 1) / b; }

__host__ __device__ constexpr bool is_pow2(int L) { return (L & (L - 1)) == 0; }

__host__ __device__ constexpr int log2_int(int L)
{
    int b = 0;
    while ((1 << b) < L) ++b;
    return b;
}

template <int L>
struct Radix {
    static constexpr int k = radix_k(L);
    static constexpr unsigned long long Lk = ipow(L, k);
    static constexpr bool pow2 = is_pow2(L);
    static constexpr int bits = log2_int(L);
    // r = 2^32 / Lk; the fraction method needs r >= (1 + sqrt 5)/2
    static constexpr double r = 4294967296.0 / (double)Lk;
    static constexpr bool frac_ok = !pow2 && (r * r - r - 1.0 >= 0.0);
    static constexpr uint32_t r_int = (uint32_t)((1ull << 32) / Lk);
    static constexpr uint32_t c_frac = (uint32_t)((((1ull << 32) % Lk) << 32) / Lk + ((((((1ull << 32) % Lk) << 32) % Lk) != 0) ? 1 : 0));
};

// Digits of one word, least significant first: out[i] = digit i, i < k(L).
template <int L>
__device__ __forceinline__ void unpack_word(uint32_t w, int (&out)[Radix<L>::k])
{
    using R = Radix<L>;
    if constexpr (R::pow2) {
#pragma unroll
        for (int i = 0; i < R::k; ++i) out[i] = (int)((w >> (R::bits * i)) & (uint32_t)(L - 1));
    } else if constexpr (R::frac_ok) {
        uint32_t f = w * R::r_int + __umulhi(w, R::c_frac) + 1u;
#pragma unroll
        for (int i = R::k - 1; i >= 0; --i) {
            unsigned long long t = (unsigned long long)f * (unsigned long long)L;
            out[i] = (int)(t >> 32);
            f = (uint32_t)t;
        }
    } else {
#pragma unroll
        for (int i = 0; i < R::k; ++i) {
            out[i] = (int)(w % (uint32_t)L);
            w /= (uint32_t)L;
        }
    }
}

// Runtime-L digit i of a word (slow path for the generic kernels).
__device__ __forceinline__ int digit_rt(uint32_t w, int L, int i)
{
    for (int j = 0; j < i; ++j) w /= (uint32_t)L;
    return (int)(w % (uint32_t)L);
}

// ------------------------------------------------------------------ fp16 helpers

__device__ __forceinline__ float h2f(uint16_t h) { return __half2float(__ushort_as_half(h)); }

// binary16 scale of a group: rounded toward +inf, saturated at the largest finite binary16.
// sf >= 0 by construction; fabsf turns a -0 (from fminf/fmaxf picking differently signed
// zeros) into +0.
__device__ __forceinline__ uint16_t scale_half_ru(float sf)
{
    sf = fabsf(sf);
    if (sf > 65504.0f) return 0x7BFFu;
    return __half_as_ushort(__float2half_ru(sf));
}

// exact binary16 of a value that is itself a binary16 (the group minimum); -0 becomes +0.
__device__ __forceinline__ uint16_t zero_half(float mn) { return __half_as_ushort(__float2half_rn(mn + 0.0f)); }

// fp16 scale and zero of a group with extrema mn, mx on L levels.  clip = 1: s rounded up from
// (mx - mn)/(L - 1), z = mn.  clip < 1 (clipped range, the SKVQ abstract): the extrema are scaled
// by clip, z is the nearest binary16 of clip*mn (-0 as +0) and s is rounded up from
// (clip*mx - z)/(L - 1), at least 0.  Values outside the clipped grid must be clamped by the caller.
__device__ __forceinline__ void group_scale_zero(float mn, float mx, int L, float clip, uint16_t& s16, uint16_t& z16)
{
    if (clip == 1.0f) {
        s16 = scale_half_ru(__fdiv_rn(__fsub_rn(mx, mn), (float)(L - 1)));
        z16 = zero_half(mn);
        return;
    }
    z16 = __half_as_ushort(__float2half_rn(__fmul_rn(clip, mn)));
    if (z16 == 0x8000u) z16 = 0u;
    float sf = __fdiv_rn(__fsub_rn(__fmul_rn(clip, mx), h2f(z16)), (float)(L - 1));
    if (sf < 0.0f) sf = 0.0f;
    s16 = scale_half_ru(sf);
}

// Tiles [t0, t1) of split s when `tiles` tiles are shared by nsplit splits: shares differ by at
// most one tile (every split works when tiles >= nsplit, so each SM carries about the same load),
// and the later splits take the smaller shares (the last tile, where an appended token lands,
// is in the last split).
__device__ __forceinline__ void split_tiles(int tiles, int nsplit, int s, int& t0, int& t1)
{
    t0 = tiles - (int)(((long long)tiles * (nsplit - s)) / nsplit);
    t1 = tiles - (int)(((long long)tiles * (nsplit - 1 - s)) / nsplit);
}

// code of x on the grid (z, s) with L levels: clamp(rint((x - z)/s), 0, L - 1), IEEE fp32
// subtract and divide, round half to even; 0 when s == 0.
__device__ __forceinline__ int quant_code(float x, float z, float s, int L)
{
    if (s == 0.0f) return 0;
    float q = __fdiv_rn(__fsub_rn(x, z), s);
    q = fminf(fmaxf(q, 0.0f), (float)(L - 1));
    return __float2int_rn(q);
}

// ------------------------------------------------------------------ block scans (warp shuffles)

__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t v)
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    return v;
}

// Exclusive scan over the whole block (blockDim.x a multiple of 32, <= 1024).  `tmp` holds 33
// words of shared memory.  Returns the exclusive prefix; *total receives the block sum.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* tmp, uint32_t* total)
{
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
    uint32_t inc = warp_incl_scan(v);
    if (lane == 31) tmp[wid] = inc;
    __syncthreads();
    if (wid == 0) {
        uint32_t t = lane < nw ? tmp[lane] : 0u;
        uint32_t ti = warp_incl_scan(t);
        tmp[lane] = ti - t;
        if (lane == 31) tmp[32] = ti;
    }
    __syncthreads();
    uint32_t r = tmp[wid] + inc - v;
    *total = tmp[32];
    __syncthreads();
    return r;
}

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Order-preserving uint32 image of a score (-0 taken as +0): a > b as floats iff key(a) > key(b)
__host__ __device__ __forceinline__ uint32_t order_key(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7fffffffu) == 0u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

}  // namespace semkv
