// Quantization at generation time: one new token per unit (SemKV page, Abstract: the quality
// cliff is reported for tokens quantized as they are generated, too).
//
// The token is on the L_hi grid iff its score > tau of its unit (strict: the newest token loses
// ties), is quantized alone with the same affine rule as the prefill, and is written at slot
// n_seg of its segment.  K: the row's W words are written whole.  V: each channel's word that
// holds the slot gets its digit -- a fresh word at the first slot of a word, otherwise the word
// plus code * L^position (the digit was zero: slots are filled in order and the prefill wrote
// zero digits past the segment's end).  One CTA of 128 threads (thread d = channel d) per unit.
#include "append.cuh"

namespace semkv {

// p < 0: the token goes on the L_hi grid iff score > tau.  p >= 0 (running top-p): iff fewer than
// floor(p (T+1)) earlier tokens have a score >= its score (the newest token loses ties).
__global__ void __launch_bounds__(128) k_append(semkv_cache_t c, const uint16_t* __restrict__ knew,
                                                 const uint16_t* __restrict__ vnew, const float* __restrict__ score,
                                                 float p)
{
    constexpr int D = 128;
    const int u = blockIdx.x, d = threadIdx.x, lane = d & 31, warp = d >> 5;

    // every independent load first: the unit's state and this thread's channel of the new rows
    const float sc = score[u];
    const float tau = c.tau[u];
    const int nh = c.n_hi[u], nl = c.n_lo[u];
    const float kx = h2f(knew[(size_t)u * D + d]);
    const float vx = h2f(vnew[(size_t)u * D + d]);
    const int T = nh + nl;
    bool hi;
    if (p < 0.0f) {
        hi = sc > tau;  // NaN compares false: the token goes lo
    } else {
        // rank of the new token among all T + 1 scores: earlier keys >= its key, 4 per load
        const uint32_t key = order_key(sc);
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
    if (!append_fits(c, hi, nh, nl)) {
        if (d == 0) atomicOr(c.status, SEMKV_STATUS_APPEND_OVERFLOW | (isnan(sc) ? SEMKV_STATUS_NAN_SCORE : 0));
        return;
    }
    const bool bad = append_row(c, u, hi, nh, nl, kx, vx);
    if (d == 0) {
        if (bad) atomicOr(c.status, SEMKV_STATUS_NONFINITE_KV);
        append_state(c, u, hi, nh, nl, sc);
    }
}

void launch_append(const semkv_cache_t& c, const uint16_t* k, const uint16_t* v, const float* score, float p,
                   cudaStream_t st)
{
    k_append<<<c.B * c.H, 128, 0, st>>>(c, k, v, score, p);
}

}  // namespace semkv
