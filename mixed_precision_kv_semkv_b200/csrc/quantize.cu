// Affine quantization + base-L radix packing of a prefill into both segments of the cache.
//
// SemKV page, Abstract: every token is kept and stored on a uniform affine grid whose level count
// need not be a power of two.  Per token and group of G channels: s = fp16-round-up of fp32
// (max - min)/(L - 1) (saturated at 65504), z = min, code = clamp(rint((x - z)/s), 0, L - 1),
// with IEEE fp32 subtract and divide and ties to even.
//
// One launch covers both segments; one CTA (4 warps) per 128-slot output tile:
//   1. warp 0 maps the tile's slots to token indices (32-ary search of the rank directory for the
//      first bitmap word, then a ballot scan), and fetches each token's K and V row (256 B each)
//      with one cp.async.bulk per row into shared memory, completing on an mbarrier; the other
//      warps zero the rows of slots past the segment's end meanwhile;
//   2. thread t quantizes K row t and packs it along the channels (Horner, top digit first);
//   3. thread t writes the scale/zero of V row t; after a barrier thread d quantizes channel d of
//      every slot and packs it along the tile's slots.
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
    int L, k_digits, tiles_cap, is_hi;
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

// per-group grid: scale (fp16, rounded up, saturated), its reciprocal, zero
__device__ __forceinline__ Grid make_grid(float mn, float mx, int L, uint32_t* packed)
{
    const uint16_t s16 = scale_half_ru(__fdiv_rn(__fsub_rn(mx, mn), (float)(L - 1)));
    const uint16_t z16 = zero_half(mn);
    Grid g;
    g.s = h2f(s16);
    g.z = h2f(z16);
    g.r = g.s != 0.0f ? __frcp_rn(g.s) : 0.0f;  // s = 0: every code is 0 (d * 0 = 0)
    *packed = (uint32_t)s16 | ((uint32_t)z16 << 16);
    return g;
}

// code of x on grid g: rint(RN((x - z)/s)) clamped to L - 1
__device__ __forceinline__ uint32_t code_of(float x, const Grid& g, float top)
{
    const float d = __fsub_rn(x, g.z);
    const float q0 = __fmul_rn(d, g.r);
    const float e = __fmaf_rn(-g.s, q0, d);
    float q = __fmaf_rn(e, g.r, q0);
    q = fminf(q, top);
    return __float_as_uint(__fadd_rn(q, 12582912.0f)) - 0x4B400000u;
}

__global__ void __launch_bounds__(128) k_quantize(QuantSeg hi, QuantSeg lo, const uint16_t* __restrict__ K,
                                                   const uint16_t* __restrict__ V,
                                                   const uint32_t* __restrict__ bitmap,
                                                   const uint32_t* __restrict__ rank, int T, int G, int words_cap,
                                                   int32_t* __restrict__ status)
{
    constexpr int D = 128;
    const int per_unit = hi.tiles_cap + lo.tiles_cap;
    const int u = blockIdx.x / per_unit;
    int tile = blockIdx.x % per_unit;
    const bool is_hi = tile < hi.tiles_cap;
    const QuantSeg& seg = is_hi ? hi : lo;
    if (!is_hi) tile -= hi.tiles_cap;
    const int L = seg.L, k = seg.k_digits;
    const int WK = ceil_div(D, k), WV = ceil_div(TILE, k);
    const int NG = D / G;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n = seg.n[u];
    const int s0 = tile * TILE;
    if (s0 >= n) return;
    const int nv = min(TILE, n - s0);

    extern __shared__ __align__(128) unsigned char smem[];
    uint16_t* Ks = reinterpret_cast<uint16_t*>(smem);
    uint16_t* Vs = Ks + TILE * QROW;
    int* tok = reinterpret_cast<int*>(Vs + TILE * QROW);
    float4* vgrid = reinterpret_cast<float4*>(tok + TILE);  // [TILE][NG] (s, r, z, -)
    __shared__ __align__(8) uint64_t bar;

    if (tid == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    tok[tid] = -1;
    __syncthreads();

    const uint32_t* bm = bitmap + (size_t)u * words_cap;
    const uint32_t* rk = rank + (size_t)u * words_cap;
    const int nwords = (T + 31) / 32;

    if (warp == 0) {
        // ---- slots [s0, s0 + nv) -> token indices
        auto before = [&](int w) -> int { return is_hi ? (int)rk[w] : 32 * w - (int)rk[w]; };
        int lo_w = 0, hi_w = nwords;  // the last word with before() <= s0 lies in [lo_w, hi_w)
        while (hi_w - lo_w > 1) {
            const int step = (hi_w - lo_w + 31) / 32;
            const int probe = lo_w + lane * step;
            const bool ok = probe < hi_w && before(probe) <= s0;
            const unsigned m = __ballot_sync(0xffffffffu, ok);
            lo_w += (31 - __clz(m)) * step;
            hi_w = min(hi_w, lo_w + step);
        }
        int cur = lo_w, base = before(lo_w);
        while (true) {
            const int w = cur + lane;
            uint32_t m = 0u;
            if (w < nwords) {
                const uint32_t b = bm[w];
                const uint32_t valid = (32 * (w + 1) <= T) ? 0xffffffffu : ((1u << (T - 32 * w)) - 1u);
                m = is_hi ? b : (~b & valid);
            }
            const int cnt = __popc(m);
            const int inc = (int)warp_incl_scan((uint32_t)cnt);
            int my = base + inc - cnt;
            while (m) {
                const int bit = __ffs(m) - 1;
                m &= m - 1u;
                if (my >= s0 && my < s0 + nv) tok[my - s0] = 32 * w + bit;
                ++my;
            }
            base += __shfl_sync(0xffffffffu, inc, 31);
            cur += 32;
            if (base >= s0 + nv || cur >= nwords) break;
        }
        __syncwarp();
        // ---- row fetch: one bulk copy per row; rows of unmapped slots are zeroed instead
        int valid_rows = 0;
        for (int r = lane; r < nv; r += 32) valid_rows += (tok[r] >= 0 && tok[r] < T);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) valid_rows += __shfl_xor_sync(0xffffffffu, valid_rows, o);
        if (lane == 0) mbar_arrive_expect_tx(&bar, (uint32_t)valid_rows * 2u * D * 2u);
        __syncwarp();
        for (int r = lane; r < nv; r += 32) {
            const int t = tok[r];
            if (t >= 0 && t < T) {
                const size_t off = ((size_t)u * T + t) * D;
                bulk_g2s(Ks + r * QROW, K + off, D * 2, &bar);
                bulk_g2s(Vs + r * QROW, V + off, D * 2, &bar);
            } else {
                for (int i = 0; i < D; i += 8) {
                    *reinterpret_cast<uint4*>(Ks + r * QROW + i) = make_uint4(0u, 0u, 0u, 0u);
                    *reinterpret_cast<uint4*>(Vs + r * QROW + i) = make_uint4(0u, 0u, 0u, 0u);
                }
            }
        }
    } else {
        for (int r = nv + (tid - 32); r < TILE; r += 96) {
            for (int i = 0; i < D; i += 8) {
                *reinterpret_cast<uint4*>(Ks + r * QROW + i) = make_uint4(0u, 0u, 0u, 0u);
                *reinterpret_cast<uint4*>(Vs + r * QROW + i) = make_uint4(0u, 0u, 0u, 0u);
            }
        }
    }
    const bool arrived = mbar_wait(&bar, 0);
    __syncthreads();
    if (!arrived) {  // copies did not land in time: report, wait once more for them, and stop
        if (tid == 0) atomicOr(status, SEMKV_STATUS_TIMEOUT);
        mbar_wait(&bar, 0);
        return;
    }

    const size_t tile_base = (size_t)u * seg.tiles_cap + tile;
    uint32_t* kw = seg.k + tile_base * WK * TILE;
    uint32_t* vw = seg.v + tile_base * WV * D;
    uint32_t* kz = seg.kz + tile_base * NG * TILE;
    uint32_t* vz = seg.vz + tile_base * NG * TILE;
    const float top = (float)(L - 1);
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
            const Grid g = make_grid(mn, mx, L, &packed);
            kz[grp * TILE + tid] = packed;
            for (int i = G - 8; i >= 0; i -= 8) {
                float f[8];
                half8(row + grp * G + i, f);
#pragma unroll
                for (int j = 7; j >= 0; --j) {
                    w = w * (uint32_t)L + code_of(f[j], g, top);
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
            const Grid g = make_grid(mn, mx, L, &packed);
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
        int widx = (TILE - 1) / k, dig = (TILE - 1) % k;
        for (int t = TILE - 1; t >= 0; --t) {
            const float4 gg = vgrid[t * NG + grp];
            const Grid g = {gg.x, gg.y, gg.z};
            w = w * (uint32_t)L + code_of(h2f(Vs[t * QROW + d]), g, top);
            if (dig == 0) {
                vw[widx * D + d] = w;
                w = 0u;
                --widx;
                dig = k - 1;
            } else {
                --dig;
            }
        }
    }
}

static size_t quantize_smem(int G)
{
    return (size_t)2 * TILE * QROW * 2 + TILE * 4 + (size_t)TILE * (128 / G) * 16;
}

void launch_quantize(const SegView& shi, const SegView& slo, const uint16_t* K, const uint16_t* V,
                     const uint32_t* bitmap, const uint32_t* rank, int units, int T, int D, int G, int words_cap,
                     int32_t* status, cudaStream_t st)
{
    (void)D;
    const int per_unit = shi.tiles_cap + slo.tiles_cap;
    if (per_unit == 0 || units == 0) return;
    auto conv = [](const SegView& s) {
        QuantSeg q;
        q.k = s.k;
        q.v = s.v;
        q.kz = s.kz;
        q.vz = s.vz;
        q.n = s.n;
        q.L = s.L;
        q.k_digits = radix_k(s.L);
        q.tiles_cap = s.tiles_cap;
        q.is_hi = s.is_hi;
        return q;
    };
    const size_t sm = quantize_smem(G);
    cudaFuncSetAttribute(k_quantize, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    k_quantize<<<(unsigned)units * per_unit, 128, sm, st>>>(conv(shi), conv(slo), K, V, bitmap, rank, T, G, words_cap,
                                                             status);
}

}  // namespace semkv
