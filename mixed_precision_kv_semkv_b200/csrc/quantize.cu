// Affine quantization + base-L radix packing of a prefill into one segment of the cache.
//
// SemKV page, Abstract: every token is kept and stored on a uniform affine grid whose level count
// need not be a power of two.  Per token and group of G channels: s = fp16-round-up of fp32
// (max - min)/(L - 1) (saturated at 65504), z = min, code = clamp(rint((x - z)/s), 0, L - 1).
//
// One CTA (4 warps) per 128-slot output tile of one segment of one unit:
//   1. warp 0 maps the tile's slots to token indices: a 32-ary search of the rank directory for
//      the first bitmap word, then a ballot scan of the following words;
//   2. all warps gather the tile's K and V rows (fp16, 256 B each, coalesced 8-byte lane loads)
//      into shared memory;
//   3. thread t quantizes K row t and packs it along the channels (Horner, top digit first);
//   4. thread t computes the per-group scale/zero of V row t; after a barrier thread d quantizes
//      channel d of every slot and packs it along the slots of the tile.
// Slots past the segment's length get zero rows, hence zero codes and zero scale/zero.
#include "common.cuh"
#include "kernels.cuh"

namespace semkv {

constexpr int QROW = 136;  // halves per shared row: 128 + 8 keeps 16-byte lane loads conflict-free

__device__ __forceinline__ void half8(const uint16_t* p, float (&f)[8])
{
    uint4 v = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = h2f((uint16_t)(w[i] & 0xffffu));
        f[2 * i + 1] = h2f((uint16_t)(w[i] >> 16));
    }
}

template <int LC>
__global__ void __launch_bounds__(128) k_quantize(SegView seg, const uint16_t* __restrict__ K,
                                                   const uint16_t* __restrict__ V, const uint32_t* __restrict__ bitmap,
                                                   const uint32_t* __restrict__ rank, int T, int G, int words_cap,
                                                   int L_rt, int32_t* __restrict__ status)
{
    constexpr int D = 128;
    const int L = LC ? LC : L_rt;
    const int k = LC ? radix_k(LC) : radix_k(L_rt);
    const int WK = ceil_div(D, k), WV = ceil_div(TILE, k);
    const int NG = D / G;
    const int tile = blockIdx.x, u = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n = seg.n[u];
    const int s0 = tile * TILE;
    if (s0 >= n) return;
    const int nv = min(TILE, n - s0);

    extern __shared__ __align__(16) unsigned char smem[];
    uint16_t* Ks = reinterpret_cast<uint16_t*>(smem);
    uint16_t* Vs = Ks + TILE * QROW;
    int* tok = reinterpret_cast<int*>(Vs + TILE * QROW);
    float* vs_s = reinterpret_cast<float*>(tok + TILE);
    float* vs_z = vs_s + TILE * NG;

    const uint32_t* bm = bitmap + (size_t)u * words_cap;
    const uint32_t* rk = rank + (size_t)u * words_cap;
    const int nwords = (T + 31) / 32;

    // ---- 1. slots [s0, s0 + nv) -> token indices (-1 = not found: bitmap/rank inconsistent with n)
    tok[tid] = -1;
    __syncthreads();
    if (warp == 0) {
        auto before = [&](int w) -> int { return seg.is_hi ? (int)rk[w] : 32 * w - (int)rk[w]; };
        int lo = 0, hi = nwords;  // before(lo) <= s0; the last word with before <= s0 is in [lo, hi)
        while (hi - lo > 1) {
            int step = (hi - lo + 31) / 32;
            int probe = lo + lane * step;
            bool ok = probe < hi && before(probe) <= s0;
            unsigned m = __ballot_sync(0xffffffffu, ok);
            int last = 31 - __clz(m);
            lo = lo + last * step;
            hi = min(hi, lo + step);
        }
        int cur = lo, base = before(lo);
        while (true) {
            int w = cur + lane;
            uint32_t m = 0u;
            if (w < nwords) {
                uint32_t b = bm[w];
                uint32_t valid = (32 * (w + 1) <= T) ? 0xffffffffu : ((1u << (T - 32 * w)) - 1u);
                m = seg.is_hi ? b : (~b & valid);
            }
            int cnt = __popc(m);
            int inc = (int)warp_incl_scan((uint32_t)cnt);
            int my = base + inc - cnt;
            while (m) {
                int bit = __ffs(m) - 1;
                m &= m - 1u;
                if (my >= s0 && my < s0 + nv) tok[my - s0] = 32 * w + bit;
                ++my;
            }
            base += __shfl_sync(0xffffffffu, inc, 31);
            cur += 32;
            if (base >= s0 + nv || cur >= nwords) break;
        }
    }
    __syncthreads();

    // ---- 2. gather rows
#pragma unroll 4
    for (int r = warp; r < TILE; r += 4) {
        uint2 kv = make_uint2(0u, 0u), vv = make_uint2(0u, 0u);
        const int t = r < nv ? tok[r] : -1;
        if (t >= 0 && t < T) {
            size_t base = ((size_t)u * T + t) * D + lane * 4;
            kv = __ldg(reinterpret_cast<const uint2*>(K + base));
            vv = __ldg(reinterpret_cast<const uint2*>(V + base));
        }
        *reinterpret_cast<uint2*>(Ks + r * QROW + lane * 4) = kv;
        *reinterpret_cast<uint2*>(Vs + r * QROW + lane * 4) = vv;
    }
    __syncthreads();

    const size_t tile_base = (size_t)u * seg.tiles_cap + tile;
    uint32_t* kw = seg.k + tile_base * WK * TILE;
    uint32_t* vw = seg.v + tile_base * WV * D;
    uint32_t* kz = seg.kz + tile_base * NG * TILE;
    uint32_t* vz = seg.vz + tile_base * NG * TILE;
    bool bad = false;

    // ---- 3. K row `tid`: groups and channels from the top, Horner into words
    {
        const uint16_t* row = Ks + tid * QROW;
        uint32_t w = 0u;
        for (int grp = NG - 1; grp >= 0; --grp) {
            float mn = __int_as_float(0x7f800000), mx = -mn;
            for (int i = 0; i < G; i += 8) {
                float f[8];
                half8(row + grp * G + i, f);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    bad |= !isfinite(f[j]);
                    mn = fminf(mn, f[j]);
                    mx = fmaxf(mx, f[j]);
                }
            }
            uint16_t s16 = scale_half_ru(__fdiv_rn(__fsub_rn(mx, mn), (float)(L - 1)));
            uint16_t z16 = zero_half(mn);
            const float s = h2f(s16), z = h2f(z16);
            kz[grp * TILE + tid] = (uint32_t)s16 | ((uint32_t)z16 << 16);
            for (int i = G - 8; i >= 0; i -= 8) {
                float f[8];
                half8(row + grp * G + i, f);
#pragma unroll
                for (int j = 7; j >= 0; --j) {
                    const int d = grp * G + i + j;
                    w = w * (uint32_t)L + (uint32_t)quant_code(f[j], z, s, L);
                    if (d % k == 0) {
                        kw[(d / k) * TILE + tid] = w;
                        w = 0u;
                    }
                }
            }
        }
    }

    // ---- 4a. V row `tid`: per-group scale and zero
    {
        const uint16_t* row = Vs + tid * QROW;
        for (int grp = 0; grp < NG; ++grp) {
            float mn = __int_as_float(0x7f800000), mx = -mn;
            for (int i = 0; i < G; i += 8) {
                float f[8];
                half8(row + grp * G + i, f);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    bad |= !isfinite(f[j]);
                    mn = fminf(mn, f[j]);
                    mx = fmaxf(mx, f[j]);
                }
            }
            uint16_t s16 = scale_half_ru(__fdiv_rn(__fsub_rn(mx, mn), (float)(L - 1)));
            uint16_t z16 = zero_half(mn);
            vs_s[tid * NG + grp] = h2f(s16);
            vs_z[tid * NG + grp] = h2f(z16);
            vz[grp * TILE + tid] = (uint32_t)s16 | ((uint32_t)z16 << 16);
        }
    }
    if (bad) atomicOr(status, SEMKV_STATUS_NONFINITE_KV);
    __syncthreads();

    // ---- 4b. V channel `tid` across the tile's slots, top slot first
    {
        const int d = tid, grp = d / G;
        uint32_t w = 0u;
        for (int t = TILE - 1; t >= 0; --t) {
            const float x = h2f(Vs[t * QROW + d]);
            w = w * (uint32_t)L + (uint32_t)quant_code(x, vs_z[t * NG + grp], vs_s[t * NG + grp], L);
            if (t % k == 0) {
                vw[(t / k) * D + d] = w;
                w = 0u;
            }
        }
    }
}

static size_t quantize_smem(int G) { return (size_t)2 * TILE * QROW * 2 + TILE * 4 + (size_t)2 * TILE * (128 / G) * 4; }

template <int LC>
static void launch_q(const SegView& seg, const uint16_t* K, const uint16_t* V, const uint32_t* bitmap,
                     const uint32_t* rank, int units, int T, int G, int words_cap, int32_t* status, cudaStream_t st)
{
    size_t sm = quantize_smem(G);
    cudaFuncSetAttribute(k_quantize<LC>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    dim3 grid(seg.tiles_cap, units);
    k_quantize<LC><<<grid, 128, sm, st>>>(seg, K, V, bitmap, rank, T, G, words_cap, seg.L, status);
}

void launch_quantize(const SegView& seg, const uint16_t* K, const uint16_t* V, const uint32_t* bitmap,
                     const uint32_t* rank, int units, int T, int D, int G, int words_cap, int32_t* status,
                     cudaStream_t st)
{
    (void)D;
    if (seg.tiles_cap == 0 || units == 0) return;
    switch (seg.L) {
#define SEMKV_Q(LL) \
    case LL: launch_q<LL>(seg, K, V, bitmap, rank, units, T, G, words_cap, status, st); break;
        SEMKV_Q(2) SEMKV_Q(3) SEMKV_Q(4) SEMKV_Q(5) SEMKV_Q(6) SEMKV_Q(7) SEMKV_Q(8) SEMKV_Q(9)
        SEMKV_Q(10) SEMKV_Q(11) SEMKV_Q(12) SEMKV_Q(13) SEMKV_Q(14) SEMKV_Q(15) SEMKV_Q(16)
#undef SEMKV_Q
        default: launch_q<0>(seg, K, V, bitmap, rank, units, T, G, words_cap, status, st); break;
    }
}

}  // namespace semkv
