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

// p < 0: the token goes on the L_hi grid iff score > tau.  p >= 0 (running top-p): iff fewer than
// floor(p (T+1)) earlier tokens have a score >= its score (the newest token loses ties).
__global__ void __launch_bounds__(128) k_append(semkv_cache_t c, const uint16_t* __restrict__ knew,
                                                 const uint16_t* __restrict__ vnew, const float* __restrict__ score,
                                                 float p)
{
    constexpr int D = 128;
    const int u = blockIdx.x, d = threadIdx.x, lane = d & 31, warp = d >> 5;
    const int G = c.G, NG = D / G;
    __shared__ int kc[D + 32];
    __shared__ float gmn[2][4], gmx[2][4];  // per-warp partial extrema of groups wider than a warp

    // every independent load first: the unit's state and this thread's channel of the new rows
    const float sc = score[u];
    const float tau = c.tau[u];
    const int nh = c.n_hi[u], nl = c.n_lo[u];
    const float kx = h2f(knew[(size_t)u * D + d]);
    const float vx = h2f(vnew[(size_t)u * D + d]);
    const int T = nh + nl;
    const uint32_t key = order_key(sc);
    bool hi;
    if (p < 0.0f) {
        hi = sc > tau;  // NaN compares false: the token goes lo
    } else {
        // rank of the new token among all T + 1 scores: earlier keys >= its key, 4 per load
        __shared__ int cnt_s[4];
        const uint32_t* keys = c.score_keys + (size_t)u * c.T_cap;
        int cnt = 0;
#pragma unroll 8
        for (int t = 4 * d; t < T; t += 4 * 128) {  // t + 3 < T_cap: T < T_cap, T_cap % 32 == 0
            const uint4 k4 = *reinterpret_cast<const uint4*>(keys + t);
            cnt += (k4.x >= key) + (t + 1 < T && k4.y >= key) + (t + 2 < T && k4.z >= key) + (t + 3 < T && k4.w >= key);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
        if (lane == 0) cnt_s[warp] = cnt;
        __syncthreads();
        const int total = cnt_s[0] + cnt_s[1] + cnt_s[2] + cnt_s[3];
        const double target = floor((double)p * (double)(T + 1));
        hi = !isnan(sc) && (double)total < target;
    }
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
        __syncthreads();
        const int w0 = (d / G) * (G / 32);
        for (int i = 0; i < G / 32; ++i) {
            kmn = fminf(kmn, gmn[0][w0 + i]);
            kmx = fmaxf(kmx, gmx[0][w0 + i]);
            vmn = fminf(vmn, gmn[1][w0 + i]);
            vmx = fmaxf(vmx, gmx[1][w0 + i]);
        }
    }
    const uint16_t ks16 = scale_half_ru(__fdiv_rn(__fsub_rn(kmx, kmn), (float)(L - 1))), kz16 = zero_half(kmn);
    const uint16_t vs16 = scale_half_ru(__fdiv_rn(__fsub_rn(vmx, vmn), (float)(L - 1))), vz16 = zero_half(vmn);
    const int grp = d / G;
    if (d % G == 0) {
        kz[grp * TILE + tt] = (uint32_t)ks16 | ((uint32_t)kz16 << 16);
        vz[grp * TILE + tt] = (uint32_t)vs16 | ((uint32_t)vz16 << 16);
    }
    kc[d] = quant_code(kx, h2f(kz16), h2f(ks16), L);
    const uint32_t cv = (uint32_t)quant_code(vx, h2f(vz16), h2f(vs16), L);
    const bool bad = !isfinite(kx) || !isfinite(vx);
    __syncthreads();

    if (d < WK) {  // K word d: Horner over its k digits, top digit first
        uint32_t w = 0u;
        for (int i = k - 1; i >= 0; --i) w = w * (uint32_t)L + (uint32_t)kc[d * k + i];
        kw[d * TILE + tt] = w;
    }
    {
        // V channel d: a fresh word at the first slot of a word; otherwise the digit is added in
        // place (it was zero), with a reduction that needs no read
        const int pos = tt % k;
        uint32_t* p = vw + (size_t)(tt / k) * D + d;
        if (pos == 0) {
            *p = cv;
        } else {
            uint32_t pw = 1u;
            for (int i = 0; i < pos; ++i) pw *= (uint32_t)L;
            atomicAdd(p, cv * pw);
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
            atomicOr(bm + w, 1u << (T % 32));
        }
        if (hi) c.n_hi[u] = nh + 1;
        else c.n_lo[u] = nl + 1;
        c.score_keys[(size_t)u * c.T_cap + T] = key;
    }
}

void launch_append(const semkv_cache_t& c, const uint16_t* k, const uint16_t* v, const float* score, float p,
                   cudaStream_t st)
{
    k_append<<<c.B * c.H, 128, 0, st>>>(c, k, v, score, p);
}

}  // namespace semkv
