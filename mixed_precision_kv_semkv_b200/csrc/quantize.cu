// Affine quantization + base-L radix packing of a prefill into both segments of the cache.
//
// SemKV page, Abstract: every token is kept and stored on a uniform affine grid whose level count
// need not be a power of two.  Per token and group of G channels: s = fp16-round-up of fp32
// (max - min)/(L - 1) (saturated at 65504), z = min, code = clamp(rint((x - z)/s), 0, L - 1),
// with IEEE fp32 subtract and divide and ties to even.
//
// One launch covers both segments; one CTA (4 warps) per 128-slot output tile (the compile-time
// path uses two CTAs per tile, one for its K rows and one for its V rows):
//   1. each warp reads the tokens of its 32 slots from the slot map (written by the precision
//      assignment) and copies their K and V rows (256 B each) into shared memory in 16-byte
//      cp.async pieces (rows of slots past the segment's end are zeroed); no warp waits for
//      another;
//   2. thread t quantizes K row t and packs it along the channels;
//   3. thread t writes the scale/zero of V row t; after a barrier thread d packs channel d of
//      every slot along the tile's slots.
// The quotient (x - z)/s is the IEEE round-to-nearest quotient, computed by Markstein's method
// (P. Markstein, IBM J. Res. Dev. 34(1), 1990): with r = RN(1/s) (one __frcp_rn per group),
// q0 = RN(d r), e = d - s q0 (exact with one FMA), q = RN(q0 + e r) is the correctly rounded d/s
// when no intermediate underflows -- here d is 0 or a multiple of 2^-24 below 2^17 and
// s >= 2^-24, so none does.  rint is the round-to-nearest-even addition of 1.5 * 2^23.
// q >= 0 because x >= z; q <= L - 1 up to one rounding because s >= (max - min)/(L - 1), so only
// the upper clamp (which matters when the scale saturated) is applied.
#include "common.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace semkv {

constexpr int QROW = 136;  // halves per shared row: 128 + 8; rows 272 B apart keep 16-byte loads conflict-free

struct QuantSeg {
    uint32_t *k, *v, *kz, *vz;
    const int32_t* n;
    const int32_t* map;  // slot -> token of unit 0; unit u at + u * map_stride
    int map_stride;
    int L, k_digits, tiles_cap, is_hi;
    int Lv, kv_digits;  // V codes: level count and codes per word
    const uint32_t* kc;  // per-channel K grids of this segment (unit u at + u * 256), or null
};

__device__ __forceinline__ void half8(const uint16_t* p, float (&f)[8])
{
    const uint4 v = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = h2f((uint16_t)(w[i] & 0xffffu));
        f[2 * i + 1] = h2f((uint16_t)(w[i] >> 16));
    }
}

struct Grid {
    float s, r, z;
};

// per-group grid: scale (fp16, rounded up, saturated), its reciprocal, zero (clip < 1: of the
// clipped range)
__device__ __forceinline__ Grid make_grid(float mn, float mx, int L, float clip, uint32_t* packed)
{
    uint16_t s16, z16;
    group_scale_zero(mn, mx, L, clip, s16, z16);
    Grid g;
    g.s = h2f(s16);
    g.z = h2f(z16);
    g.r = g.s != 0.0f ? __frcp_rn(g.s) : 0.0f;  // s = 0: every code is 0 (d * 0 = 0)
    *packed = (uint32_t)s16 | ((uint32_t)z16 << 16);
    return g;
}

// code of x on grid g: rint(RN((x - z)/s)) clamped to [0, L - 1] (below 0 only on a clipped grid)
__device__ __forceinline__ uint32_t code_of(float x, const Grid& g, float top)
{
    const float d = __fsub_rn(x, g.z);
    const float q0 = __fmul_rn(d, g.r);
    const float e = __fmaf_rn(-g.s, q0, d);
    float q = __fmaf_rn(e, g.r, q0);
    q = fmaxf(fminf(q, top), 0.0f);
    return __float_as_uint(__fadd_rn(q, 12582912.0f)) - 0x4B400000u;
}

// This warp's 32 slots of the tile (slots s0 + 32 w .. s0 + 32 w + 31, those past nv empty): their
// tokens from the slot map, and those tokens' K row and V row (256 B each; V/Vs may be null) into
// shared memory in 16-byte cp.async pieces (16 lanes per row, so every instruction reads two
// whole rows); rows of empty slots are zeroed.  Only the calling warp waits: the warps of a CTA
// fetch and start on their rows independently.
__device__ __forceinline__ void gather_rows_warp(uint16_t* Ks, uint16_t* Vs, const QuantSeg& seg, int u, int s0, int nv,
                                                 const uint16_t* __restrict__ K, const uint16_t* __restrict__ V,
                                                 int T)
{
    constexpr int D = 128;
    const int lane = threadIdx.x & 31, r0 = 32 * (threadIdx.x >> 5);
    const int mine = r0 + lane < nv ? __ldg(seg.map + (size_t)u * seg.map_stride + s0 + r0 + lane) : -1;
#pragma unroll 4
    for (int c = lane; c < 32 * (D / 8); c += 32) {
        const int rr = c >> 4, part = (c & 15) * 8;
        const int t = __shfl_sync(0xffffffffu, mine, rr);
        uint16_t* dk = Ks + (r0 + rr) * QROW + part;
        uint16_t* dv = Vs ? Vs + (r0 + rr) * QROW + part : nullptr;
        if (t >= 0 && t < T) {
            const size_t off = ((size_t)u * T + t) * D + part;
            cp_async16(dk, K + off);
            if (dv) cp_async16(dv, V + off);
        } else {
            *reinterpret_cast<uint4*>(dk) = make_uint4(0u, 0u, 0u, 0u);
            if (dv) *reinterpret_cast<uint4*>(dv) = make_uint4(0u, 0u, 0u, 0u);
        }
    }
    cp_async_wait_all();
    __syncwarp();
}

__global__ void __launch_bounds__(128) k_quantize(QuantSeg hi, QuantSeg lo, const uint16_t* __restrict__ K,
                                                   const uint16_t* __restrict__ V,
                                                   int T, int G, float clip,
                                                   int32_t* __restrict__ status)
{
    constexpr int D = 128;
    const int per_unit = hi.tiles_cap + lo.tiles_cap;
    const int u = blockIdx.x / per_unit;
    int tile = blockIdx.x % per_unit;
    const bool is_hi = tile < hi.tiles_cap;
    const QuantSeg& seg = is_hi ? hi : lo;
    if (!is_hi) tile -= hi.tiles_cap;
    const int L = seg.L, k = seg.k_digits, Lv = seg.Lv, kv = seg.kv_digits;
    const int WK = ceil_div(D, k), WV = ceil_div(TILE, kv);
    const int NG = D / G;
    const int tid = threadIdx.x;
    const int n = seg.n[u];
    const int s0 = tile * TILE;
    if (s0 >= n) return;
    const int nv = min(TILE, n - s0);

    extern __shared__ __align__(128) unsigned char smem[];
    uint16_t* Ks = reinterpret_cast<uint16_t*>(smem);
    uint16_t* Vs = Ks + TILE * QROW;
    float4* vgrid = reinterpret_cast<float4*>(Vs + TILE * QROW);  // [TILE][NG] (s, r, z, -)
    float4* cgrid = vgrid + TILE * NG;                             // [128] per-channel K grids
    if (seg.kc) {
        const uint32_t gk = seg.kc[(size_t)u * 256 + tid];
        const float s = h2f((uint16_t)(gk & 0xffffu)), z = h2f((uint16_t)(gk >> 16));
        cgrid[tid] = make_float4(s, s != 0.0f ? __frcp_rn(s) : 0.0f, z, 0.0f);
    }
    gather_rows_warp(Ks, Vs, seg, u, s0, nv, K, V, T);
    __syncthreads();  // the channel grids (the rows are per warp)

    const size_t tile_base = (size_t)u * seg.tiles_cap + tile;
    uint32_t* kw = seg.k + tile_base * WK * TILE;
    uint32_t* vw = seg.v + tile_base * WV * D;
    uint32_t* kz = seg.kz + tile_base * NG * TILE;
    uint32_t* vz = seg.vz + tile_base * NG * TILE;
    const float top = (float)(L - 1), top_v = (float)(Lv - 1);
    bool bad = false;

    // ---- K row `tid`: groups and channels from the top, Horner into words
    {
        const uint16_t* row = Ks + tid * QROW;
        uint32_t w = 0u;
        int widx = (D - 1) / k, dig = (D - 1) % k;
        for (int grp = NG - 1; grp >= 0; --grp) {
            float mn = __int_as_float(0x7f800000), mx = -mn;
            for (int i = 0; i < G; i += 8) {
                float f[8];
                half8(row + grp * G + i, f);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    bad |= !(fabsf(f[j]) <= 65504.0f);
                    mn = fminf(mn, f[j]);
                    mx = fmaxf(mx, f[j]);
                }
            }
            uint32_t packed;
            const Grid g = make_grid(mn, mx, L, clip, &packed);
            kz[grp * TILE + tid] = seg.kc ? 0u : packed;  // per-channel K grids: no per-token grid
            for (int i = G - 8; i >= 0; i -= 8) {
                float f[8];
                half8(row + grp * G + i, f);
#pragma unroll
                for (int j = 7; j >= 0; --j) {
                    uint32_t code;
                    if (seg.kc) {  // slots past the segment's end hold zero codes, as on the plain grids
                        const float4 cg = cgrid[grp * G + i + j];
                        code = tid < nv ? code_of(f[j], Grid{cg.x, cg.y, cg.z}, top) : 0u;
                    } else {
                        code = code_of(f[j], g, top);
                    }
                    w = w * (uint32_t)L + code;
                    if (dig == 0) {
                        kw[widx * TILE + tid] = w;
                        w = 0u;
                        --widx;
                        dig = k - 1;
                    } else {
                        --dig;
                    }
                }
            }
        }
    }

    // ---- V row `tid`: per-group grids to shared memory
    {
        const uint16_t* row = Vs + tid * QROW;
        for (int grp = 0; grp < NG; ++grp) {
            float mn = __int_as_float(0x7f800000), mx = -mn;
            for (int i = 0; i < G; i += 8) {
                float f[8];
                half8(row + grp * G + i, f);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    bad |= !(fabsf(f[j]) <= 65504.0f);
                    mn = fminf(mn, f[j]);
                    mx = fmaxf(mx, f[j]);
                }
            }
            uint32_t packed;
            const Grid g = make_grid(mn, mx, Lv, clip, &packed);
            vgrid[tid * NG + grp] = make_float4(g.s, g.r, g.z, 0.0f);
            vz[grp * TILE + tid] = packed;
        }
    }
    if (bad && tid < nv) atomicOr(status, SEMKV_STATUS_NONFINITE_KV);
    __syncthreads();

    // ---- V channel `tid` across the tile's slots, top slot first
    {
        const int d = tid, grp = d / G;
        uint32_t w = 0u;
        int widx = (TILE - 1) / kv, dig = (TILE - 1) % kv;
        for (int t = TILE - 1; t >= 0; --t) {
            const float4 gg = vgrid[t * NG + grp];
            const Grid g = {gg.x, gg.y, gg.z};
            w = w * (uint32_t)Lv + code_of(h2f(Vs[t * QROW + d]), g, top_v);
            if (dig == 0) {
                vw[widx * D + d] = w;
                w = 0u;
                --widx;
                dig = kv - 1;
            } else {
                --dig;
            }
        }
    }
}

// ------------------------------------------------------------------ compile-time fast path
//
// Same tile work with L and G known at compile time: words are accumulated as sum_i code_i L^i with
// constant powers (no serial Horner chain), codes are the low byte of the round-to-nearest-even
// magic sum 1.5 * 2^23 + q (the offset is removed once per word), group minima and maxima use
// packed fp16 (NaN-propagating, so a non-finite value shows up in the group's range), and the
// quotient runs two lanes at a time in packed fp32.  On the plain grid no clamp is needed for
// L >= 3: q <= L - 1 up to one rounding when the scale did not saturate, and q <= 131008/65504 = 2
// when it did.  The clipped grid clamps on both sides (group_codes).  The V part of a tile may
// use its own level count.

__host__ __device__ constexpr uint32_t upow(int L, int i)
{
    uint32_t p = 1u;
    for (int j = 0; j < i; ++j) p *= (uint32_t)L;
    return p;
}

// magic offset carried by a word of `cnt` digits: 0x4B400000 * sum_{i < cnt} L^i (mod 2^32)
__host__ __device__ constexpr uint32_t magic_sum(int L, int cnt)
{
    uint32_t s = 0u;
    for (int i = 0; i < cnt; ++i) s += 0x4B400000u * upow(L, i);
    return s;
}

__device__ __forceinline__ uint64_t f2_pack(float a, float b)
{
    return ((uint64_t)__float_as_uint(b) << 32) | __float_as_uint(a);
}

// rint(RN((x - z)/s)) + 1.5 * 2^23 as fp32 bits, two lanes at once (Markstein: q0 = d r,
// e = d - s q0, q = q0 + e r)
__device__ __forceinline__ uint64_t code2_bits(uint64_t x2, uint64_t z2, uint64_t r2, uint64_t ns2, uint64_t m2)
{
    uint64_t d, q0, e, q, y;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(x2), "l"(z2));
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(q0) : "l"(d), "l"(r2));
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(e) : "l"(ns2), "l"(q0), "l"(d));
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(q) : "l"(e), "l"(r2), "l"(q0));
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(y) : "l"(q), "l"(m2));
    return y;
}

struct GroupGrid {
    uint64_t z2, r2, ns2;
    uint32_t zh2;  // the zero as a binary16 pair (the clipped grid's lower clamp)
    uint32_t packed;
    bool finite;
};

// running minimum and maximum (as binary16 pairs) over N pairs of values
template <int N>
__device__ __forceinline__ void minmax_pairs(const uint32_t (&h)[N], __half2& mn2, __half2& mx2, bool first)
{
    if (first) mn2 = mx2 = *reinterpret_cast<const __half2*>(&h[0]);
#pragma unroll
    for (int i = first ? 1 : 0; i < N; ++i) {
        const __half2 v = *reinterpret_cast<const __half2*>(&h[i]);
        mn2 = __hmin2_nan(mn2, v);
        mx2 = __hmax2_nan(mx2, v);
    }
}

// CLIP: the clipped-range grid (clip < 1); otherwise the plain min/max grid
template <int L, bool CLIP>
__device__ __forceinline__ GroupGrid group_grid(__half2 mn2, __half2 mx2, float clip)
{
    const float mn = __half2float(__hmin_nan(__low2half(mn2), __high2half(mn2)));
    const float mx = __half2float(__hmax_nan(__low2half(mx2), __high2half(mx2)));
    GroupGrid g;
    g.finite = fabsf(mn) <= 65504.0f && fabsf(mx) <= 65504.0f;
    uint16_t s16, z16;
    if constexpr (CLIP) {
        group_scale_zero(mn, mx, L, clip, s16, z16);
    } else {
        (void)clip;
        s16 = scale_half_ru(__fdiv_rn(__fsub_rn(mx, mn), (float)(L - 1)));
        z16 = zero_half(mn);
    }
    g.zh2 = (uint32_t)z16 | ((uint32_t)z16 << 16);
    const float s = h2f(s16), z = h2f(z16);
    const float r = s != 0.0f ? __frcp_rn(s) : 0.0f;
    g.z2 = f2_pack(z, z);
    g.r2 = f2_pack(r, r);
    g.ns2 = f2_pack(-s, -s);
    g.packed = (uint32_t)s16 | ((uint32_t)z16 << 16);
    return g;
}

// codes (as magic-offset fp32 bits) of N values (N / 2 pairs), two at a time, handed to
// `sink(i, bits)`.  CLIP: values below the zero are raised to it first (exact: the zero is a
// binary16) and the quotient is clamped to L - 1 before the rounding add, so codes are
// clamp(rint(q), 0, L - 1) and the add stays in its exact range.
template <int L, int N, bool CLIP, typename Sink>
__device__ __forceinline__ void group_codes(const uint32_t (&h)[N / 2], const GroupGrid& g, Sink&& sink)
{
    const uint64_t m2 = f2_pack(12582912.0f, 12582912.0f);
#pragma unroll
    for (int i = 0; i < N / 2; ++i) {
        __half2 hv = *reinterpret_cast<const __half2*>(&h[i]);
        if constexpr (CLIP) hv = __hmax2(hv, *reinterpret_cast<const __half2*>(&g.zh2));
        const float2 xf = __half22float2(hv);
        uint64_t y;
        if constexpr (CLIP) {
            uint64_t d, q0, e, q;
            asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2_pack(xf.x, xf.y)), "l"(g.z2));
            asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(q0) : "l"(d), "l"(g.r2));
            asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(e) : "l"(g.ns2), "l"(q0), "l"(d));
            asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(q) : "l"(e), "l"(g.r2), "l"(q0));
            const float qa = fminf(__uint_as_float((uint32_t)q), (float)(L - 1));
            const float qb = fminf(__uint_as_float((uint32_t)(q >> 32)), (float)(L - 1));
            asm("add.rn.f32x2 %0, %1, %2;" : "=l"(y) : "l"(f2_pack(qa, qb)), "l"(m2));
        } else {
            y = code2_bits(f2_pack(xf.x, xf.y), g.z2, g.r2, g.ns2, m2);
        }
        uint32_t b0 = (uint32_t)y, b1 = (uint32_t)(y >> 32);
        if constexpr (L == 2) {  // the only level count whose codes can exceed L - 1 (saturated scale)
            b0 = min(b0, 0x4B400001u);
            b1 = min(b1, 0x4B400001u);
        }
        sink(2 * i, b0);
        sink(2 * i + 1, b1);
    }
}

// One group of G values of a row in shared memory: its grid, and its codes handed to
// `sink(i, bits)` (i = the value's index in the group).  Groups of more than 64 values are read
// twice in chunks of 64 (range, then codes), so that a chunk, not the group, is held in registers;
// the last chunk's codes come first.
template <int L, int G, bool CLIP, typename Sink>
__device__ __forceinline__ GroupGrid quantize_group(const uint16_t* src, float clip, Sink&& sink)
{
    constexpr int CH = G > 64 ? 64 : G, NCH = G / CH;
    uint32_t h[CH / 2];
    auto load = [&](int c) {
#pragma unroll
        for (int i = 0; i < CH / 8; ++i) {
            const uint4 v = *reinterpret_cast<const uint4*>(src + c * CH + 8 * i);
            h[4 * i] = v.x;
            h[4 * i + 1] = v.y;
            h[4 * i + 2] = v.z;
            h[4 * i + 3] = v.w;
        }
    };
    __half2 mn2, mx2;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
        load(c);
        minmax_pairs<CH / 2>(h, mn2, mx2, c == 0);
    }
    const GroupGrid g = group_grid<L, CLIP>(mn2, mx2, clip);
    group_codes<L, CH, CLIP>(h, g, [&](int i, uint32_t bits) { sink((NCH - 1) * CH + i, bits); });
#pragma unroll
    for (int c = 0; c + 1 < NCH; ++c) {
        load(c);
        group_codes<L, CH, CLIP>(h, g, [&](int i, uint32_t bits) { sink(c * CH + i, bits); });
    }
    return g;
}

// K rows of a tile: thread `tid` quantizes row tid and packs it along the channels
template <int L, int G, bool CLIP>
__device__ __forceinline__ void quantize_k_rows(const uint16_t* Ks, uint32_t* kw, uint32_t* kz, int tid, bool& bad,
                                                float clip)
{
    constexpr int D = 128, k = radix_k(L), WK = ceil_div(D, k), NG = D / G;
    {
        uint32_t w[WK];
#pragma unroll
        for (int j = 0; j < WK; ++j) w[j] = 0u;
        const uint16_t* row = Ks + tid * QROW;
#pragma unroll
        for (int grp = 0; grp < NG; ++grp) {
            const GroupGrid g = quantize_group<L, G, CLIP>(row + grp * G, clip, [&](int i, uint32_t bits) {
                const int d = grp * G + i;
                w[d / k] += bits * upow(L, d % k);
            });
            bad |= !g.finite;
            kz[grp * TILE + tid] = g.packed;
        }
#pragma unroll
        for (int j = 0; j < WK; ++j) {
            const int cnt = (j + 1) * k <= D ? k : D - j * k;
            kw[j * TILE + tid] = w[j] - magic_sum(L, cnt);
        }
    }
}

// Per-channel K grids of a segment as channel pairs: (z, z'), (r, r'), (-s, -s') in packed fp32 and
// the zeros as a binary16 pair
struct KpcPair {
    uint64_t z2, r2, ns2;
    uint32_t zh2, pad;
};

// K rows of a tile on per-channel grids (thread `tid` = slot `tid`; slots at or past `nv` get zero
// codes): the value is raised to its channel's zero, the quotient clamped to L - 1 before the
// rounding add, as on the clipped grid
template <int L>
__device__ __forceinline__ void quantize_k_rows_kpc(const uint16_t* Ks, uint32_t* kw, uint32_t* kz, int tid, int nv,
                                                    int NG, const KpcPair* tab, bool& bad)
{
    constexpr int D = 128, k = radix_k(L), WK = ceil_div(D, k);
    const uint64_t m2 = f2_pack(12582912.0f, 12582912.0f);
    const bool live = tid < nv;
    uint32_t w[WK];
#pragma unroll
    for (int j = 0; j < WK; ++j) w[j] = 0u;
    const uint16_t* row = Ks + tid * QROW;
#pragma unroll
    for (int c8 = 0; c8 < D / 8; ++c8) {
        const uint4 v = *reinterpret_cast<const uint4*>(row + 8 * c8);
        const uint32_t hw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int i = 4 * c8 + e;  // channel pair (2i, 2i + 1)
            const KpcPair p = tab[i];
            const __half2 x2 = *reinterpret_cast<const __half2*>(&hw[e]);
            const float2 xr = __half22float2(x2);
            bad |= !(fabsf(xr.x) <= 65504.0f) || !(fabsf(xr.y) <= 65504.0f);
            const float2 xf = __half22float2(__hmax2(x2, *reinterpret_cast<const __half2*>(&p.zh2)));
            uint64_t d, q0, ee, q, y;
            asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2_pack(xf.x, xf.y)), "l"(p.z2));
            asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(q0) : "l"(d), "l"(p.r2));
            asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(ee) : "l"(p.ns2), "l"(q0), "l"(d));
            asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(q) : "l"(ee), "l"(p.r2), "l"(q0));
            const float qa = fminf(__uint_as_float((uint32_t)q), (float)(L - 1));
            const float qb = fminf(__uint_as_float((uint32_t)(q >> 32)), (float)(L - 1));
            asm("add.rn.f32x2 %0, %1, %2;" : "=l"(y) : "l"(f2_pack(qa, qb)), "l"(m2));
            const uint32_t b0 = live ? (uint32_t)y : 0x4B400000u, b1 = live ? (uint32_t)(y >> 32) : 0x4B400000u;
            w[(2 * i) / k] += b0 * upow(L, (2 * i) % k);
            w[(2 * i + 1) / k] += b1 * upow(L, (2 * i + 1) % k);
        }
    }
    for (int grp = 0; grp < NG; ++grp) kz[grp * TILE + tid] = 0u;  // no per-token K grid
#pragma unroll
    for (int j = 0; j < WK; ++j) {
        const int cnt = (j + 1) * k <= D ? k : D - j * k;
        kw[j * TILE + tid] = w[j] - magic_sum(L, cnt);
    }
}

// V rows of a tile: thread `tid` writes the grids of row tid and its codes as bytes over the first
// half of its own row; after a barrier thread `tid` packs channel tid along the tile's slots
template <int L, int G, bool CLIP>
__device__ __forceinline__ void quantize_v_rows(uint16_t* Vs, uint32_t* vw, uint32_t* vz, int tid, bool& bad,
                                                float clip)
{
    constexpr int D = 128, k = radix_k(L), WV = ceil_div(TILE, k), NG = D / G;
    {
        uint16_t* row = Vs + tid * QROW;
        uint32_t packed[NG];
        uint32_t bytes[D / 4];
#pragma unroll
        for (int grp = 0; grp < NG; ++grp) {
            // the low byte of each magic sum is the code: byte i%4 of word i/4 (a chunk of the
            // group covers whole words)
            const GroupGrid g = quantize_group<L, G, CLIP>(row + grp * G, clip, [&](int i, uint32_t b) {
                const int c = grp * G + i;
                constexpr uint32_t sel[4] = {0x3214u, 0x3240u, 0x3410u, 0x4210u};
                bytes[c / 4] = (c % 4 == 0) ? (b & 0xffu) : __byte_perm(bytes[c / 4], b, sel[c % 4]);
            });
            bad |= !g.finite;
            packed[grp] = g.packed;
        }
#pragma unroll
        for (int grp = 0; grp < NG; ++grp) vz[grp * TILE + tid] = packed[grp];
#pragma unroll
        for (int i = 0; i < D / 16; ++i)
            *reinterpret_cast<uint4*>(reinterpret_cast<unsigned char*>(row) + 16 * i) =
                make_uint4(bytes[4 * i], bytes[4 * i + 1], bytes[4 * i + 2], bytes[4 * i + 3]);
    }
    named_sync(1, 128);  // the 128 row threads only
    // ---- V channel `tid` across the tile's slots
    {
        uint32_t w[WV];
#pragma unroll
        for (int j = 0; j < WV; ++j) w[j] = 0u;
        const unsigned char* cb = reinterpret_cast<const unsigned char*>(Vs) + tid;
#pragma unroll
        for (int t = 0; t < TILE; ++t) w[t / k] += (uint32_t)cb[t * QROW * 2] * upow(L, t % k);
#pragma unroll
        for (int j = 0; j < WV; ++j) vw[j * D + tid] = w[j];
    }
}

// LH, LL: level counts of the K codes of the two segments; LHV, LLV: of the V codes; CLIP: the
// clipped-range grid with ratio `clip`; KPC: K on the per-channel grids of seg.kc
template <int LH, int LL, int LHV, int LLV, int G, bool CLIP, bool KPC>
__device__ __forceinline__ void quantize_fast_body(const QuantSeg& hi, const QuantSeg& lo,
                                                   const uint16_t* __restrict__ K, const uint16_t* __restrict__ V,
                                                   int T, float clip, int32_t* __restrict__ status)
{
    constexpr int D = 128, NG = D / G;
    // order: the L_lo segment's K rows, its V rows, then the L_hi segment's K rows and V rows
    // (every unit's tiles in each): the CTAs resident at any time mostly run one code path,
    // which keeps instruction fetch local
    const int units = (int)(gridDim.x / 2) / (hi.tiles_cap + lo.tiles_cap);
    const int n_lo = units * lo.tiles_cap;  // CTAs of one part of the L_lo segment
    int item = blockIdx.x;
    const bool is_hi = item >= 2 * n_lo;
    if (is_hi) item -= 2 * n_lo;
    const QuantSeg& seg = is_hi ? hi : lo;
    const int n_seg = units * seg.tiles_cap;
    const int part = item >= n_seg ? 1 : 0;  // 0: K rows, 1: V rows of the tile
    if (part) item -= n_seg;
    const int u = item / seg.tiles_cap;
    const int tile = item % seg.tiles_cap;
    const int tid = threadIdx.x;
    const int n = seg.n[u];
    const int s0 = tile * TILE;
    if (s0 >= n) return;

    extern __shared__ __align__(128) unsigned char smem[];
    uint16_t* Xs = reinterpret_cast<uint16_t*>(smem);  // this CTA's rows: K rows or V rows
    gather_rows_warp(Xs, nullptr, seg, u, s0, min(TILE, n - s0), part ? V : K, nullptr, T);

    const size_t tile_base = (size_t)u * seg.tiles_cap + tile;
    bool bad = false;
    if (part == 0) {
        const int Wk = is_hi ? ceil_div(D, radix_k(LH)) : ceil_div(D, radix_k(LL));
        uint32_t* kw = seg.k + tile_base * Wk * TILE;
        uint32_t* kz = seg.kz + tile_base * NG * TILE;
        if constexpr (KPC) {
            KpcPair* tab = reinterpret_cast<KpcPair*>(smem + (size_t)TILE * QROW * 2);  // [64]
            if (tid < 64) {
                float z[2], r[2], sv[2];
                uint16_t zh[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const uint32_t gk = seg.kc[(size_t)u * 256 + 2 * tid + e];
                    sv[e] = h2f((uint16_t)(gk & 0xffffu));
                    zh[e] = (uint16_t)(gk >> 16);
                    z[e] = h2f(zh[e]);
                    r[e] = sv[e] != 0.0f ? __frcp_rn(sv[e]) : 0.0f;
                }
                tab[tid] = KpcPair{f2_pack(z[0], z[1]), f2_pack(r[0], r[1]), f2_pack(-sv[0], -sv[1]),
                                   (uint32_t)zh[0] | ((uint32_t)zh[1] << 16), 0u};
            }
            __syncthreads();  // uniform: every thread of a K-part CTA
            const int nv = min(TILE, n - s0);
            if (is_hi) quantize_k_rows_kpc<LH>(Xs, kw, kz, tid, nv, NG, tab, bad);
            else quantize_k_rows_kpc<LL>(Xs, kw, kz, tid, nv, NG, tab, bad);
        } else {
            if (is_hi) quantize_k_rows<LH, G, CLIP>(Xs, kw, kz, tid, bad, clip);
            else quantize_k_rows<LL, G, CLIP>(Xs, kw, kz, tid, bad, clip);
        }
    } else {
        const int Wv = is_hi ? ceil_div(TILE, radix_k(LHV)) : ceil_div(TILE, radix_k(LLV));
        uint32_t* vw = seg.v + tile_base * Wv * D;
        uint32_t* vz = seg.vz + tile_base * NG * TILE;
        if (is_hi) quantize_v_rows<LHV, G, CLIP>(Xs, vw, vz, tid, bad, clip);
        else quantize_v_rows<LLV, G, CLIP>(Xs, vw, vz, tid, bad, clip);
    }
    if (bad && tid < n - s0) atomicOr(status, SEMKV_STATUS_NONFINITE_KV);
}

template <int LH, int LL, int LHV, int LLV, int G, bool CLIP, bool KPC>
__global__ void __launch_bounds__(128) k_quantize_fast(QuantSeg hi, QuantSeg lo, const uint16_t* __restrict__ K,
                                                        const uint16_t* __restrict__ V, int T, float clip,
                                                        int32_t* __restrict__ status)
{
    quantize_fast_body<LH, LL, LHV, LLV, G, CLIP, KPC>(hi, lo, K, V, T, clip, status);
}

// groups of 128: registers capped for 6 CTAs per SM (the compiler would otherwise take ~100,
// leaving 4 CTAs and fewer rows in flight; the cap costs a few spilled bytes)
template <int LH, int LL, int LHV, int LLV, int G, bool CLIP, bool KPC>
__global__ void __launch_bounds__(128, 6) k_quantize_fast_wide(QuantSeg hi, QuantSeg lo,
                                                                const uint16_t* __restrict__ K,
                                                                const uint16_t* __restrict__ V, int T, float clip,
                                                                int32_t* __restrict__ status)
{
    quantize_fast_body<LH, LL, LHV, LLV, G, CLIP, KPC>(hi, lo, K, V, T, clip, status);
}

template <int LH, int LL, int LHV, int LLV, int G, bool CLIP, bool KPC = false>
static auto quantize_fast_kernel()
{
    if constexpr (G > 64) return k_quantize_fast_wide<LH, LL, LHV, LLV, G, CLIP, KPC>;
    else return k_quantize_fast<LH, LL, LHV, LLV, G, CLIP, KPC>;
}

static size_t quantize_smem(int G)
{
    return (size_t)2 * TILE * QROW * 2 + (size_t)TILE * (128 / G) * 16 + 128 * 16;
}

void launch_quantize(const SegView& shi, const SegView& slo, const uint16_t* K, const uint16_t* V,
                     const int32_t* slot_token, int units, int T, int D, int G, float clip,
                     const uint32_t* kc, int32_t* status, cudaStream_t st)
{
    (void)D;
    const int per_unit = shi.tiles_cap + slo.tiles_cap;
    if (per_unit == 0 || units == 0) return;
    const int map_stride = (shi.tiles_cap + slo.tiles_cap) * TILE;
    auto conv = [&](const SegView& s, const int32_t* map) {
        QuantSeg q;
        q.k = s.k;
        q.v = s.v;
        q.kz = s.kz;
        q.vz = s.vz;
        q.n = s.n;
        q.L = s.L;
        q.k_digits = radix_k(s.L);
        q.Lv = s.Lv;
        q.kv_digits = radix_k(s.Lv);
        q.kc = kc ? kc + (s.is_hi ? 0 : 128) : nullptr;
        q.tiles_cap = s.tiles_cap;
        q.is_hi = s.is_hi;
        q.map = map;
        q.map_stride = map_stride;
        return q;
    };
    const unsigned grid = (unsigned)units * per_unit;
    const QuantSeg qh = conv(shi, slot_token), ql = conv(slo, slot_token + shi.tiles_cap * TILE);
    // compile-time level pairs and group sizes of the common configurations
    // compile-time level counts and group sizes of the common configurations; the quantizer
    // variants (a clip, V level counts of their own) for a few of them, the rest on k_quantize
    const bool clipped = clip != 1.0f;
#define SEMKV_QK(LH, LL, GG)                                                                                  \
    if (kc && !clipped && shi.L == LH && slo.L == LL && shi.Lv == LH && slo.Lv == LL && G == GG) {            \
        const size_t sm = (size_t)TILE * QROW * 2 + 64 * sizeof(KpcPair);                                     \
        const auto kern = quantize_fast_kernel<LH, LL, LH, LL, GG, false, true>();                            \
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);                    \
        kern<<<2 * grid, 128, sm, st>>>(qh, ql, K, V, T, clip, status);                                       \
        return;                                                                                               \
    }
    SEMKV_QK(8, 5, 64) SEMKV_QK(6, 5, 64) SEMKV_QK(8, 6, 64) SEMKV_QK(16, 8, 64) SEMKV_QK(5, 4, 64)
#undef SEMKV_QK
    if (!kc) {
#define SEMKV_QF(LH, LL, LHV, LLV, GG, CL)                                                                    \
    if (clipped == CL && shi.L == LH && slo.L == LL && shi.Lv == LHV && slo.Lv == LLV && G == GG) {           \
        const size_t sm = (size_t)TILE * QROW * 2;                                                            \
        const auto kern = quantize_fast_kernel<LH, LL, LHV, LLV, GG, CL>();                                   \
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);                    \
        kern<<<2 * grid, 128, sm, st>>>(qh, ql, K, V, T, clip, status);                                       \
        return;                                                                                               \
    }
#define SEMKV_QF_G(LH, LL) SEMKV_QF(LH, LL, LH, LL, 32, false) SEMKV_QF(LH, LL, LH, LL, 64, false) \
    SEMKV_QF(LH, LL, LH, LL, 128, false) SEMKV_QF(LH, LL, LH, LL, 64, true)
    SEMKV_QF_G(8, 5) SEMKV_QF_G(6, 5) SEMKV_QF_G(8, 6) SEMKV_QF_G(16, 8) SEMKV_QF_G(5, 4)
    SEMKV_QF(8, 5, 4, 2, 64, false) SEMKV_QF(6, 5, 4, 3, 64, false) SEMKV_QF(8, 6, 4, 2, 64, false)
    SEMKV_QF(16, 8, 8, 4, 64, false)
#undef SEMKV_QF_G
#undef SEMKV_QF
    }  // per-channel K grids: the runtime-L kernel below
    const size_t sm = quantize_smem(G);
    cudaFuncSetAttribute(k_quantize, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    k_quantize<<<grid, 128, sm, st>>>(qh, ql, K, V, T, G, clip, status);
}

}  // namespace semkv
