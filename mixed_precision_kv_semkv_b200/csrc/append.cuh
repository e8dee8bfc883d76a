// Writing one generated token into a unit's cache: the row (by one CTA of 128 threads, thread d =
// channel d) and the unit's bookkeeping (by one thread).  Used by the append kernel and by the
// decode kernels that append and attend in one pass.
//
// SemKV page, Abstract: the quality cliff also appears for tokens quantized as they are generated.
// The token is quantized alone with the prefill's affine rule (and clip) and written at slot n_seg
// of its segment.  K: the row's W words are written whole.  V: each channel's word that holds the slot
// gets its digit -- a fresh word at the first slot of a word, otherwise the word plus
// code * L^position (the digit was zero: slots are filled in order and the prefill wrote zero
// digits past the segment's end).
#pragma once

#include "common.cuh"
#include "kernels.cuh"

namespace semkv {

// Row of the new token of unit u (grid hi; nh, nl: the unit's counts before it; kx, vx: channel d
// of the new K and V rows), written by 128 threads (d = 0..127) that synchronize with sync() and
// OR a flag over themselves with sync_or(flag).  kc: 160 ints of shared scratch; gmn, gmx: per-warp
// partial extrema of groups wider than a warp.  Returns true on every thread if a K or V value of
// the row is not finite.
template <class Sync, class SyncOr>
__device__ __forceinline__ bool append_row_impl(const semkv_cache_t& c, int u, bool hi, int nh, int nl, float kx,
                                                float vx, int d, int* kc, float (*gmn)[4], float (*gmx)[4], Sync sync,
                                                SyncOr sync_or)
{
    constexpr int D = 128;
    const int lane = d & 31, warp = d >> 5;
    const int G = c.G, NG = D / G;
    const int slot = hi ? nh : nl;
    const int L = hi ? c.L_hi : c.L_lo, Lv = level_v(c, hi);
    const int k = radix_k(L), kv = radix_k(Lv);
    const int WK = ceil_div(D, k), WV = ceil_div(TILE, kv);
    const int tile = slot / TILE, tt = slot % TILE;
    const int tiles_cap = (hi ? c.cap_hi : c.cap_lo) / TILE;
    const size_t tb = (size_t)u * tiles_cap + tile;
    uint32_t* kw = (hi ? c.k_hi : c.k_lo) + tb * WK * TILE;
    uint32_t* vw = (hi ? c.v_hi : c.v_lo) + tb * WV * D;
    uint32_t* kz = (hi ? c.kz_hi : c.kz_lo) + tb * NG * TILE;
    uint32_t* vz = (hi ? c.vz_hi : c.vz_lo) + tb * NG * TILE;
    if (d < 32) kc[D + d] = 0;  // padding digits of the last K word

    // group extrema: butterfly over the group's lanes (min and max are exact in any order)
    const int width = G < 32 ? G : 32;
    float kmn = kx, kmx = kx, vmn = vx, vmx = vx;
    for (int o = width >> 1; o > 0; o >>= 1) {
        kmn = fminf(kmn, __shfl_xor_sync(0xffffffffu, kmn, o));
        kmx = fmaxf(kmx, __shfl_xor_sync(0xffffffffu, kmx, o));
        vmn = fminf(vmn, __shfl_xor_sync(0xffffffffu, vmn, o));
        vmx = fmaxf(vmx, __shfl_xor_sync(0xffffffffu, vmx, o));
    }
    if (G > 32) {  // combine the group's warps
        if (lane == 0) {
            gmn[0][warp] = kmn;
            gmx[0][warp] = kmx;
            gmn[1][warp] = vmn;
            gmx[1][warp] = vmx;
        }
        sync();
        const int w0 = (d / G) * (G / 32);
        for (int i = 0; i < G / 32; ++i) {
            kmn = fminf(kmn, gmn[0][w0 + i]);
            kmx = fmaxf(kmx, gmx[0][w0 + i]);
            vmn = fminf(vmn, gmn[1][w0 + i]);
            vmx = fmaxf(vmx, gmx[1][w0 + i]);
        }
    }
    const float clip = clip_ratio(c);
    uint16_t ks16, kz16, vs16, vz16;
    group_scale_zero(kmn, kmx, L, clip, ks16, kz16);
    group_scale_zero(vmn, vmx, Lv, clip, vs16, vz16);
    const int grp = d / G;
    if (d % G == 0) {
        // per-channel K grids: no per-token K grid
        kz[grp * TILE + tt] = c.k_per_channel ? 0u : (uint32_t)ks16 | ((uint32_t)kz16 << 16);
        vz[grp * TILE + tt] = (uint32_t)vs16 | ((uint32_t)vz16 << 16);
    }
    if (c.k_per_channel) {  // the channel's grid of this segment, fitted at prefill (clamped)
        const uint32_t gk = c.kc[(size_t)u * 2 * D + (hi ? 0 : D) + d];
        kc[d] = quant_code(kx, h2f((uint16_t)(gk >> 16)), h2f((uint16_t)(gk & 0xffffu)), L);
    } else {
        kc[d] = quant_code(kx, h2f(kz16), h2f(ks16), L);
    }
    const uint32_t cv = (uint32_t)quant_code(vx, h2f(vz16), h2f(vs16), Lv);
    const bool bad = !isfinite(kx) || !isfinite(vx);
    sync();

    if (d < WK) {  // K word d: Horner over its k digits, top digit first
        uint32_t w = 0u;
        for (int i = k - 1; i >= 0; --i) w = w * (uint32_t)L + (uint32_t)kc[d * k + i];
        kw[d * TILE + tt] = w;
    }
    {
        // V channel d: a fresh word at the first slot of a word; otherwise the digit is added in
        // place (it was zero), with a reduction that needs no read
        const int pos = tt % kv;
        uint32_t* p = vw + (size_t)(tt / kv) * D + d;
        if (pos == 0) {
            *p = cv;
        } else {
            uint32_t pw = 1u;
            for (int i = 0; i < pos; ++i) pw *= (uint32_t)Lv;
            atomicAdd(p, cv * pw);
        }
    }
    return sync_or(bad);
}

// append_row_impl by every thread of a 128-thread CTA (thread d = channel d)
__device__ __forceinline__ bool append_row(const semkv_cache_t& c, int u, bool hi, int nh, int nl, float kx, float vx)
{
    __shared__ int kc[128 + 32];
    __shared__ float gmn[2][4], gmx[2][4];
    return append_row_impl(
        c, u, hi, nh, nl, kx, vx, (int)threadIdx.x, kc, gmn, gmx, [] { __syncthreads(); },
        [](bool b) { return __syncthreads_or(b) != 0; });
}

// The unit's bookkeeping after its new token went in (one thread): bitmap bit, rank directory,
// segment count, score key.
__device__ __forceinline__ void append_state(const semkv_cache_t& c, int u, bool hi, int nh, int nl, float sc)
{
    if (isnan(sc)) atomicOr(c.status, SEMKV_STATUS_NAN_SCORE);
    const int T = nh + nl;
    const int words_cap = c.T_cap / 32;
    uint32_t* bm = c.bitmap + (size_t)u * words_cap;
    uint32_t* rk = c.rank + (size_t)u * words_cap;
    const int w = T / 32;
    if (T % 32 == 0) {
        bm[w] = hi ? 1u : 0u;
        rk[w] = (uint32_t)nh;
    } else if (hi) {
        atomicOr(bm + w, 1u << (T % 32));
    }
    if (hi) c.n_hi[u] = nh + 1;
    else c.n_lo[u] = nl + 1;
    c.score_keys[(size_t)u * c.T_cap + T] = order_key(sc);
}

// Whether the new token of unit u fits (fixed-threshold rule): its grid and room in its segment.
__device__ __forceinline__ bool append_fits(const semkv_cache_t& c, bool hi, int nh, int nl)
{
    return (hi ? nh < c.cap_hi : nl < c.cap_lo) && nh + nl < c.T_cap;
}

}  // namespace semkv
