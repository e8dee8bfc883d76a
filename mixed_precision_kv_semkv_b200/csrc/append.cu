// Quantization at generation time: one new token per unit (SemKV page, Abstract: the quality
// cliff is reported for tokens quantized as they are generated, too).
//
// The token is on the L_hi grid iff its score > tau of its unit (strict: the newest token loses
// ties), is quantized alone with the same affine rule as the prefill, and is written at slot
// n_seg of its segment.  K: the row's W words are written whole.  V: each channel's word that
// holds the slot gets its digit -- a fresh word at the first slot of a word, otherwise the word
// plus code * L^position (the digit was zero: slots are filled in order and the prefill wrote
// zero digits past the segment's end).  One CTA of 128 threads (thread d = channel d) per unit.
#include "common.cuh"
#include "kernels.cuh"

namespace semkv {

__global__ void __launch_bounds__(128) k_append(semkv_cache_t c, const uint16_t* __restrict__ knew,
                                                 const uint16_t* __restrict__ vnew, const float* __restrict__ score)
{
    constexpr int D = 128;
    const int u = blockIdx.x, d = threadIdx.x;
    const int G = c.G, NG = D / G;
    __shared__ float kr[D], vr[D];
    __shared__ int kc[D + 32];
    __shared__ float gs[2][16], gz[2][16];

    const float sc = score[u];
    const bool hi = sc > c.tau[u];  // NaN compares false: the token goes lo
    const int nh = c.n_hi[u], nl = c.n_lo[u];
    const int T = nh + nl;
    const int slot = hi ? nh : nl;
    const int cap = hi ? c.cap_hi : c.cap_lo;
    if (slot >= cap || T >= c.T_cap) {
        if (d == 0) atomicOr(c.status, SEMKV_STATUS_APPEND_OVERFLOW | (isnan(sc) ? SEMKV_STATUS_NAN_SCORE : 0));
        return;
    }
    const int L = hi ? c.L_hi : c.L_lo;
    const int k = radix_k(L);
    const int WK = ceil_div(D, k), WV = ceil_div(TILE, k);
    const int tile = slot / TILE, tt = slot % TILE;
    const int tiles_cap = (hi ? c.cap_hi : c.cap_lo) / TILE;
    const size_t tb = (size_t)u * tiles_cap + tile;
    uint32_t* kw = (hi ? c.k_hi : c.k_lo) + tb * WK * TILE;
    uint32_t* vw = (hi ? c.v_hi : c.v_lo) + tb * WV * D;
    uint32_t* kz = (hi ? c.kz_hi : c.kz_lo) + tb * NG * TILE;
    uint32_t* vz = (hi ? c.vz_hi : c.vz_lo) + tb * NG * TILE;

    kr[d] = h2f(knew[(size_t)u * D + d]);
    vr[d] = h2f(vnew[(size_t)u * D + d]);
    if (d < 32) kc[D + d] = 0;  // padding digits of the last K word
    __syncthreads();

    bool bad = !isfinite(kr[d]) || !isfinite(vr[d]);
    if (d < 2 * NG) {  // threads 0..NG-1: K groups, NG..2NG-1: V groups
        const int which = d / NG, grp = d % NG;
        const float* x = which ? vr : kr;
        float mn = __int_as_float(0x7f800000), mx = -mn;
        for (int i = 0; i < G; ++i) {
            mn = fminf(mn, x[grp * G + i]);
            mx = fmaxf(mx, x[grp * G + i]);
        }
        uint16_t s16 = scale_half_ru(__fdiv_rn(__fsub_rn(mx, mn), (float)(L - 1)));
        uint16_t z16 = zero_half(mn);
        gs[which][grp] = h2f(s16);
        gz[which][grp] = h2f(z16);
        (which ? vz : kz)[grp * TILE + tt] = (uint32_t)s16 | ((uint32_t)z16 << 16);
    }
    __syncthreads();
    const int grp = d / G;
    kc[d] = quant_code(kr[d], gz[0][grp], gs[0][grp], L);
    const uint32_t cv = (uint32_t)quant_code(vr[d], gz[1][grp], gs[1][grp], L);
    __syncthreads();

    if (d < WK) {  // K word d: Horner over its k digits, top digit first
        uint32_t w = 0u;
        for (int i = k - 1; i >= 0; --i) w = w * (uint32_t)L + (uint32_t)kc[d * k + i];
        kw[d * TILE + tt] = w;
    }
    {
        const int pos = tt % k;
        uint32_t* p = vw + (size_t)(tt / k) * D + d;
        if (pos == 0) {
            *p = cv;
        } else {
            uint32_t pw = 1u;
            for (int i = 0; i < pos; ++i) pw *= (uint32_t)L;
            *p = *p + cv * pw;
        }
    }
    if (__syncthreads_or(bad) && d == 0) atomicOr(c.status, SEMKV_STATUS_NONFINITE_KV);
    if (d == 0) {
        if (isnan(sc)) atomicOr(c.status, SEMKV_STATUS_NAN_SCORE);
        const int words_cap = c.T_cap / 32;
        uint32_t* bm = c.bitmap + (size_t)u * words_cap;
        uint32_t* rk = c.rank + (size_t)u * words_cap;
        const int w = T / 32;
        if (T % 32 == 0) {
            bm[w] = hi ? 1u : 0u;
            rk[w] = (uint32_t)nh;
        } else if (hi) {
            bm[w] |= 1u << (T % 32);
        }
        if (hi) c.n_hi[u] = nh + 1;
        else c.n_lo[u] = nl + 1;
    }
}

void launch_append(const semkv_cache_t& c, const uint16_t* k, const uint16_t* v, const float* score, cudaStream_t st)
{
    k_append<<<c.B * c.H, 128, 0, st>>>(c, k, v, score);
}

}  // namespace semkv
