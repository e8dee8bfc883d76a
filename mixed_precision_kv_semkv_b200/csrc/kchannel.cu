// Per-channel K grids (a quantizer variant: keys quantized per channel, as the KVQuant blog page on
// the same pages names it).  For every unit and channel d, the grid is fitted over the channel's T
// prefill values: min and max (NaN skipped), then the plain or clipped rule of the per-token groups
// (scale rounded up to binary16, zero the binary16 of the minimum), once with L_hi and once with
// L_lo levels.  kc[u][0][d] and kc[u][1][d] hold the two grids (fp16 scale | fp16 zero << 16).
//
// Three small launches: the buffer is seeded with the order-preserving uint32 image of +max and
// -max (k_kc_init); CTAs over slices of the tokens reduce their slice per channel in shared memory
// and fold it in with atomicMin / atomicMax on those images (k_kc_range; one 256-byte K row per warp
// per step, lane l holding channels 4l..4l+3); the images then become the two grids in place
// (k_kc_finalize).
#include "common.cuh"
#include "kernels.cuh"

namespace semkv {

__device__ __forceinline__ float key_to_float(uint32_t k)
{
    const uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
    return __uint_as_float(u);
}

__global__ void k_kc_init(uint32_t* __restrict__ kc, int n)
{
    const int i = blockIdx.x * blockDim.x + threadIdx.x;  // over units * 2 * 128
    if (i < n) kc[i] = ((i / 128) & 1) ? 0u : 0xffffffffu;  // [u][0][d]: min image, [u][1][d]: max image
}

constexpr int KC_THREADS = 256, KC_WARPS = KC_THREADS / 32;

__global__ void __launch_bounds__(KC_THREADS) k_kc_range(const uint16_t* __restrict__ K, int T, int slices,
                                                          uint32_t* __restrict__ kc, int32_t* __restrict__ status)
{
    constexpr int D = 128;
    const int u = blockIdx.y, slice = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int t0 = (int)(((long long)T * slice) / slices), t1 = (int)(((long long)T * (slice + 1)) / slices);
    const float inf = __int_as_float(0x7f800000);
    float mn[4] = {inf, inf, inf, inf}, mx[4] = {-inf, -inf, -inf, -inf};
    bool bad = false;
    const uint16_t* base = K + (size_t)u * T * D + 4 * lane;
#pragma unroll 4
    for (int t = t0 + warp; t < t1; t += KC_WARPS) {
        const uint2 w = *reinterpret_cast<const uint2*>(base + (size_t)t * D);
        const float f[4] = {h2f((uint16_t)(w.x & 0xffffu)), h2f((uint16_t)(w.x >> 16)), h2f((uint16_t)(w.y & 0xffffu)),
                            h2f((uint16_t)(w.y >> 16))};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            bad |= !(fabsf(f[j]) <= 65504.0f);
            mn[j] = fminf(mn[j], f[j]);  // NaN is skipped
            mx[j] = fmaxf(mx[j], f[j]);
        }
    }
    __shared__ float smn[KC_WARPS][D], smx[KC_WARPS][D];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        smn[warp][4 * lane + j] = mn[j];
        smx[warp][4 * lane + j] = mx[j];
    }
    if (__syncthreads_or(bad) && threadIdx.x == 0) atomicOr(status, SEMKV_STATUS_NONFINITE_KV);
    if (threadIdx.x < D) {
        const int d = threadIdx.x;
        float a = smn[0][d], b = smx[0][d];
#pragma unroll
        for (int w = 1; w < KC_WARPS; ++w) {
            a = fminf(a, smn[w][d]);
            b = fmaxf(b, smx[w][d]);
        }
        if (a <= b) {  // the slice held a number in this channel
            atomicMin(kc + (size_t)u * 2 * D + d, order_key(a));
            atomicMax(kc + (size_t)u * 2 * D + D + d, order_key(b));
        }
    }
}

__global__ void k_kc_finalize(uint32_t* __restrict__ kc, int units, int L_hi, int L_lo, float clip)
{
    constexpr int D = 128;
    const int i = blockIdx.x * blockDim.x + threadIdx.x;  // over units * 128
    if (i >= units * D) return;
    const int u = i / D, d = i % D;
    uint32_t* p = kc + (size_t)u * 2 * D + d;
    const uint32_t kmin = p[0], kmax = p[D];
    uint32_t ghi = 0u, glo = 0u;
    if (kmin <= kmax) {  // at least one token (and not every value NaN)
        const float mn = key_to_float(kmin), mx = key_to_float(kmax);
        uint16_t s16, z16;
        group_scale_zero(mn, mx, L_hi, clip, s16, z16);
        ghi = (uint32_t)s16 | ((uint32_t)z16 << 16);
        group_scale_zero(mn, mx, L_lo, clip, s16, z16);
        glo = (uint32_t)s16 | ((uint32_t)z16 << 16);
    }
    p[0] = ghi;
    p[D] = glo;
}

void launch_kc_grids(const semkv_cache_t& c, const uint16_t* K, int T, int sms, cudaStream_t st)
{
    const int units = c.B * c.H, n = units * 2 * 128;
    k_kc_init<<<(n + 255) / 256, 256, 0, st>>>(c.kc, n);
    if (T > 0) {
        // about four CTAs per SM over all units, at least 32 tokens per slice
        int slices = (4 * sms + units - 1) / units;
        slices = min(slices, (T + 31) / 32);
        slices = max(slices, 1);
        k_kc_range<<<dim3((unsigned)slices, (unsigned)units), KC_THREADS, 0, st>>>(K, T, slices, c.kc, c.status);
    }
    k_kc_finalize<<<(units * 128 + 127) / 128, 128, 0, st>>>(c.kc, units, c.L_hi, c.L_lo, clip_ratio(c));
}

}  // namespace semkv
