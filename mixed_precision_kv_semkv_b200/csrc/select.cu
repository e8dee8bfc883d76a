// Precision assignment: per unit, the n_hi largest of T fp32 scores get the L_hi grid.
//
// SemKV page, Abstract: tokens are ordered by an importance score from inside the model and the
// top fraction is stored at the finer of two neighbouring precisions.  Ties: equal scores are
// taken in increasing token order (-0 and +0 are equal).
//
// One CTA of 1024 threads per unit.  The n_hi-th largest key K* is found by a most-significant-
// digit radix select over the order-preserving uint32 image of the scores (4 passes of 8 bits,
// shared-memory histograms; the scores stay in L2 between passes).  A final pass forms each
// bitmap word from warp ballots (key > K*, key == K*), takes the first (n_hi - #greater) ties in
// token order with a block-wide exclusive scan, and writes the rank directory with a second scan.
#include "common.cuh"
#include "kernels.cuh"

namespace semkv {

__device__ __forceinline__ uint32_t score_key(float f)
{
    uint32_t u = __float_as_uint(f);
    if ((u & 0x7fffffffu) == 0u) u = 0u;  // -0 -> +0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_score(uint32_t k)
{
    uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
    return __uint_as_float(u);
}

__global__ void __launch_bounds__(1024) k_select(const float* __restrict__ scores, int T, int n_hi, int words_cap,
                                                  uint32_t* __restrict__ bitmap, uint32_t* __restrict__ rank,
                                                  int32_t* __restrict__ n_hi_out, int32_t* __restrict__ n_lo_out,
                                                  float* __restrict__ tau_out, int32_t* __restrict__ status)
{
    const int u = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const float* s = scores + (size_t)u * T;
    uint32_t* bm = bitmap + (size_t)u * words_cap;
    uint32_t* rk = rank + (size_t)u * words_cap;

    __shared__ uint32_t hist[256];
    __shared__ uint32_t scan_tmp[33];
    __shared__ uint32_t sh_prefix, sh_remaining;

    // NaN scores: flag; their keys sort above +inf (order unspecified, as documented)
    {
        bool bad = false;
        for (int t = tid; t < T; t += blockDim.x) bad |= isnan(s[t]);
        if (__syncthreads_or(bad) && tid == 0) atomicOr(status, SEMKV_STATUS_NAN_SCORE);
    }

    uint32_t prefix = 0u, mask = 0u, remaining = (uint32_t)n_hi;
    if (n_hi > 0) {
        for (int shift = 24; shift >= 0; shift -= 8) {
            if (tid < 256) hist[tid] = 0u;
            __syncthreads();
            for (int t = tid; t < T; t += blockDim.x) {
                uint32_t key = score_key(s[t]);
                if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
            }
            __syncthreads();
            if (wid == 0) {
                // lane l owns bins 255-8l .. 248-8l (descending); find the bin where the count
                // of keys from the top reaches `remaining`
                uint32_t cnt[8], sum = 0u;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    cnt[j] = hist[255 - 8 * lane - j];
                    sum += cnt[j];
                }
                uint32_t inc = warp_incl_scan(sum);
                uint32_t exc = inc - sum;
                if (exc < remaining && remaining <= inc) {
                    uint32_t cum = exc;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        if (cum + cnt[j] >= remaining) {
                            sh_prefix = prefix | ((uint32_t)(255 - 8 * lane - j) << shift);
                            sh_remaining = remaining - cum;
                            break;
                        }
                        cum += cnt[j];
                    }
                }
            }
            __syncthreads();
            prefix = sh_prefix;
            remaining = sh_remaining;
            mask |= 255u << shift;
            __syncthreads();
        }
    } else {
        prefix = 0xffffffffu;  // no key is greater; ties are not taken (remaining = 0)
        remaining = 0u;
    }
    const uint32_t kstar = prefix, take = remaining;

    // bitmap and rank, 1024 words (32768 tokens) per round; warp wid forms words c+32*wid+j
    const int nwords = (T + 31) / 32;
    uint32_t carry_ties = 0u, carry_ones = 0u;
    for (int c = 0; c < nwords; c += 1024) {
        uint32_t my_gt = 0u, my_eq = 0u;
        for (int j = 0; j < 32; ++j) {
            int w = c + 32 * wid + j;
            if (w >= nwords) break;  // uniform across the warp
            int t = 32 * w + lane;
            uint32_t key = t < T ? score_key(s[t]) : 0u;
            bool valid = t < T;
            uint32_t gt = __ballot_sync(0xffffffffu, valid && key > kstar);
            uint32_t eq = __ballot_sync(0xffffffffu, valid && key == kstar);
            if (lane == j) {
                my_gt = gt;
                my_eq = eq;
            }
        }
        const int w = c + tid;
        uint32_t tot;
        uint32_t ties_before = carry_ties + block_excl_scan((uint32_t)__popc(my_eq), scan_tmp, &tot);
        carry_ties += tot;
        uint32_t take_mask = 0u;
        if (ties_before < take) {
            uint32_t need = take - ties_before;
            if (need >= (uint32_t)__popc(my_eq)) {
                take_mask = my_eq;
            } else {
                uint32_t pos = __fns(my_eq, 0u, (int)need);  // position of the need-th set bit
                take_mask = my_eq & (0xffffffffu >> (31u - pos));
            }
        }
        uint32_t word = my_gt | take_mask;
        uint32_t ones_before = carry_ones + block_excl_scan((uint32_t)__popc(word), scan_tmp, &tot);
        carry_ones += tot;
        if (w < nwords) {
            bm[w] = word;
            rk[w] = ones_before;
        }
    }
    for (int w = nwords + tid; w < words_cap; w += blockDim.x) {
        bm[w] = 0u;
        rk[w] = (uint32_t)n_hi;
    }
    if (tid == 0) {
        n_hi_out[u] = n_hi;
        n_lo_out[u] = T - n_hi;
        tau_out[u] = n_hi > 0 ? key_score(kstar) : __int_as_float(0x7f800000);
    }
}

void launch_select(const float* scores, int units, int T, int n_hi, int words_cap, uint32_t* bitmap, uint32_t* rank,
                   int32_t* n_hi_out, int32_t* n_lo_out, float* tau, int32_t* status, cudaStream_t st)
{
    k_select<<<units, 1024, 0, st>>>(scores, T, n_hi, words_cap, bitmap, rank, n_hi_out, n_lo_out, tau, status);
}

}  // namespace semkv
