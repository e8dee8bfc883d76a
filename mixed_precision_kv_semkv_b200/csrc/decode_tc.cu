// GQA decode attention over the packed cache on the 5th-generation tensor cores (tcgen05).
//
// SemKV page, Abstract: the cache stores each token on one of two uniform grids (L_hi or L_lo
// levels); the KVQuant blog page (section on the memory bottleneck) notes that decoding long
// sequences is bound by reading the KV cache.  The packed words are therefore read from HBM once
// and dequantized on chip; the g = Hq/H query heads of a kv head share every read.
//
// One CTA = one warpgroup (128 threads) streams a range of 128-slot tiles of one segment of one
// unit.  Thread i owns TMEM lane i, which is slot i of the tile for the K side and channel i for
// the V side (K words are packed along the channels of a slot, V words along the slots of a
// channel, so each thread unpacks whole words of its own row):
//   unpack   each word is turned into the fixed-point base-L fraction (see common.cuh); one
//            32x32->64 multiply by L^2 yields the next two digits as one index P < L^2, and a
//            per-lane copy of a table in shared memory maps P to the two centred codes
//            (c - (L-1)/2) as an fp16 pair.  The pairs go to TMEM with tcgen05.st.
//   q.k      D_K[slot][(group,head)] = sum over the group's channels of (c - m) q_head, one
//            tcgen05.mma chain (M=128 slots, N = groups x heads, K = code slots) with A (codes) in
//            TMEM and B (the fp16 queries, zero outside each group) in shared memory.
//   softmax  logit = scale * sum_group [ s_K D_K + (z_K + m s_K) sum_{group} q ]; online softmax
//            in the log2 domain across tiles (warp shuffles + one shared exchange per tile).
//   p.V      D_V[channel][(group,limb,head)] = sum_slots (c - m) P', with P' = p s_V split into two
//            fp16 limbs (P' = hi + lo) so the product keeps ~22 bits; A = V codes in TMEM, B = P'
//            in shared memory (written by the slot threads).  The zero terms sum_t p (z_V + m s_V)
//            and the softmax denominators are accumulated on the CUDA cores.
// Each CTA writes (max, sum, unnormalized o) per query head to the workspace; k_decode_merge
// combines the splits.  Every mbarrier wait is bounded; a timeout sets SEMKV_STATUS_TIMEOUT.
#include "common.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace semkv {

constexpr int TC_GMAX = 8;   // query heads per kv head
constexpr int TC_NGMAX = 4;  // channel groups per row (G >= 32)

template <int L>
struct TcShape {
    using R = Radix<L>;
    static constexpr int k = R::k;
    static constexpr int W = ceil_div(128, k);       // words per row (K) = per channel per tile (V)
    static constexpr int NPAIR = (k + 1) / 2;        // digit pairs (TMEM columns) per word
    static constexpr int KC = W * NPAIR;             // TMEM columns of one unpacked row
    static constexpr int KCP = (KC + 7) / 8 * 8;     // padded to whole MMA K-steps (16 fp16)
    static constexpr int KSTEPS = KCP / 8;
    static constexpr int KSLOTS = 2 * KCP;           // fp16 elements along K
    static constexpr bool ok = (R::pow2 || R::frac_ok) && KCP <= 80;
};

// 32-bit fixed-point fraction ~ w / L^k, accurate to less than one unit of the last digit
template <int L>
__device__ __forceinline__ uint32_t to_fraction(uint32_t w)
{
    using R = Radix<L>;
    if constexpr (R::pow2) {
        return w << (32 - R::bits * R::k);
    } else {
        return w * R::r_int + __umulhi(w, R::c_frac) + 1u;
    }
}

// position (0 = least significant digit) of the digit that lands in half `h` of pair `p`
__host__ __device__ constexpr int pair_digit(int k, int p, int h) { return k - 1 - 2 * p - h; }

__host__ __device__ constexpr uint32_t bq_off(int n, int ks, uint32_t lbo, uint32_t sbo)
{
    return (uint32_t)(n >> 3) * sbo + (uint32_t)(ks >> 3) * lbo + (uint32_t)(n & 7) * 16u + (uint32_t)(ks & 7) * 2u;
}

template <int L>
struct TcSmem {
    using S = TcShape<L>;
    static constexpr uint32_t LBO_Q = 128, SBO_Q = (S::KSLOTS / 8) * 128;
    static constexpr uint32_t LBO_P = 144, SBO_P = (S::KSLOTS / 8) * 144;  // 144: conflict-free slot writes
    static constexpr uint32_t LUT_BYTES = (uint32_t)L * L * 32 * 4;
    static constexpr uint32_t BQ = (LUT_BYTES + 127) / 128 * 128;
    static constexpr uint32_t BQ_BYTES = 4 * SBO_Q;   // N_K <= 32 rows
    static constexpr uint32_t BP = BQ + BQ_BYTES;
    static constexpr uint32_t BP_BYTES = 8 * SBO_P;   // N_V <= 64 rows
    static constexpr uint32_t QSUM = (BP + BP_BYTES + 15) / 16 * 16;
    static constexpr uint32_t RED = QSUM + TC_NGMAX * TC_GMAX * 4;
    static constexpr uint32_t FIN = RED + 4 * 48 * 4;
    static constexpr uint32_t TOTAL = FIN + 48 * 4;
};

template <int L>
__global__ void __launch_bounds__(128, 1) k_decode_tc(SegView seg, const uint16_t* __restrict__ q, int H, int g,
                                                       int G, float scale_log2, int nsplit, int split_off,
                                                       int nsplit_total, float* __restrict__ ws,
                                                       int32_t* __restrict__ status, int wait_for_prior)
{
    using S = TcShape<L>;
    using M = TcSmem<L>;
    constexpr int D = 128, W = S::W, NPAIR = S::NPAIR, KC = S::KC, KSTEPS = S::KSTEPS;
    constexpr int KSLOTS = S::KSLOTS, k = S::k;
    constexpr float MID = 0.5f * (float)(L - 1);
    constexpr uint32_t COL_AK = 0, COL_AV = 80, COL_DK = 160, COL_DV = 192, TMEM_COLS = 256;

    // let a dependent launch (the other segment) start on free SMs right away
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    const int NG = D / G;
    const int NK = (NG * g + 15) / 16 * 16;
    const int GSTR = 2 * g <= 8 ? 8 : 16;  // D_V columns per group: limb-major, head-minor, padded
    const int NV = NG * GSTR < 16 ? 16 : NG * GSTR;
    const int split = blockIdx.x, u = blockIdx.y, b = u / H, hk = u % H, Hq = H * g;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    extern __shared__ __align__(1024) unsigned char smem[];
    uint32_t* lut = reinterpret_cast<uint32_t*>(smem);
    unsigned char* bq = smem + M::BQ;
    unsigned char* bp = smem + M::BP;
    float* qsum = reinterpret_cast<float*>(smem + M::QSUM);  // [NG][8]
    float* red = reinterpret_cast<float*>(smem + M::RED);    // [4][48]
    float* fin = reinterpret_cast<float*>(smem + M::FIN);    // [48]
    __shared__ __align__(8) uint64_t mbar[2];
    __shared__ uint32_t tmem_base_s;

    // ---------------- set-up: TMEM, barriers, code table, B_Q (queries), B_P zeroed
    if (warp == 0) {
        tmem_alloc(&tmem_base_s, TMEM_COLS);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(&mbar[0], 1);
        mbar_init(&mbar[1], 1);
        fence_mbar_init();
    }
    for (int i = tid; i < L * L * 32; i += 128) {
        const int P = i >> 5;
        const __half2 pr = __floats2half2_rn((float)(P / L) - MID, (float)(P % L) - MID);  // exact: |x| <= 7.5
        lut[i] = *reinterpret_cast<const uint32_t*>(&pr);
    }
    // the g query rows (g x 128 fp16) staged once in shared memory (reuses the B_P area, zeroed after)
    uint16_t* qs = reinterpret_cast<uint16_t*>(bp);
    {
        const uint16_t* qu = q + ((size_t)b * Hq + (size_t)hk * g) * D;
        for (int i = tid; i < g * D / 8; i += 128)
            reinterpret_cast<uint4*>(qs)[i] = __ldg(reinterpret_cast<const uint4*>(qu) + i);
    }
    __syncthreads();
    // B_Q: row n = (group, head) holds q_head at the K index of each channel of that group
    for (int ks = tid; ks < KSLOTS; ks += 128) {
        const int col = ks >> 1, h2 = ks & 1, j = col / NPAIR, pp = col % NPAIR;
        const int pos = pair_digit(k, pp, h2);
        const int dim = (col < KC && pos >= 0) ? j * k + pos : D;
        const int dgrp = dim < D ? dim / G : -1;
        for (int nrow = 0; nrow < NK; ++nrow) {
            const uint16_t v = (nrow < NG * g && nrow / g == dgrp) ? qs[(nrow % g) * D + dim] : (uint16_t)0;
            *reinterpret_cast<uint16_t*>(bq + bq_off(nrow, ks, M::LBO_Q, M::SBO_Q)) = v;
        }
    }
    if (tid < NG * TC_GMAX) {
        const int grp = tid / TC_GMAX, h = tid % TC_GMAX;
        float s = 0.f;
        if (h < g)
            for (int d = grp * G; d < (grp + 1) * G; ++d) s += h2f(qs[h * D + d]);
        qsum[grp * TC_GMAX + h] = s;
    }
    __syncthreads();
    for (int i = tid; i < (int)(M::BP_BYTES / 16); i += 128) reinterpret_cast<uint4*>(bp)[i] = make_uint4(0, 0, 0, 0);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_s;
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    const uint32_t idesc_k = idesc_f16_f32(128, NK), idesc_v = idesc_f16_f32(128, NV);
    const uint32_t bq_addr = smem_u32(bq), bp_addr = smem_u32(bp);

    // my slot's row of B_P (slot tid -> K index along the unpacked V words)
    const int vrank = k - 1 - (tid % k);
    const int my_ks = 2 * ((tid / k) * NPAIR + (vrank >> 1)) + (vrank & 1);
    unsigned char* bp_my = bp + (uint32_t)(my_ks >> 3) * M::LBO_P + (uint32_t)(my_ks & 7) * 2u;
    const int grp_d = tid / G;  // my channel's group

    const int n = seg.n[u];
    const int tiles = min(ceil_div(n, TILE), seg.tiles_cap);
    const int per = ceil_div(tiles, nsplit);
    const int t0 = split * per, t1 = min(tiles, t0 + per);

    float m[TC_GMAX], O[TC_GMAX], lacc[TC_GMAX], zacc[TC_NGMAX][TC_GMAX];
#pragma unroll
    for (int h = 0; h < TC_GMAX; ++h) {
        m[h] = -__int_as_float(0x7f800000);
        O[h] = lacc[h] = 0.f;
#pragma unroll
        for (int gg = 0; gg < TC_NGMAX; ++gg) zacc[gg][h] = 0.f;
    }
    uint32_t ph_k = 0, ph_v = 0;
    bool timeout = false;

    uint32_t kw[W], vw[W], kzv[TC_NGMAX], vzv[TC_NGMAX];
    auto load_tile = [&](int tile, uint32_t(&kw_)[W], uint32_t(&vw_)[W], uint32_t(&kz_)[TC_NGMAX],
                         uint32_t(&vz_)[TC_NGMAX]) {
        const size_t tb = (size_t)u * seg.tiles_cap + tile;
        const uint32_t* pk = seg.k + tb * W * TILE;
        const uint32_t* pv = seg.v + tb * W * D;
        const uint32_t* pkz = seg.kz + tb * NG * TILE;
        const uint32_t* pvz = seg.vz + tb * NG * TILE;
#pragma unroll
        for (int j = 0; j < W; ++j) {
            kw_[j] = __ldg(pk + j * TILE + tid);
            vw_[j] = __ldg(pv + j * D + tid);
        }
#pragma unroll
        for (int gg = 0; gg < TC_NGMAX; ++gg) {
            kz_[gg] = gg < NG ? __ldg(pkz + gg * TILE + tid) : 0u;
            vz_[gg] = gg < NG ? __ldg(pvz + gg * TILE + tid) : 0u;
        }
    };
    // unpack W words into KCP TMEM columns starting at `col0` of this thread's lane
    auto unpack_to_tmem = [&](const uint32_t(&w_)[W], uint32_t col0) {
        uint32_t chunk[8];
        int ci = 0;
        uint32_t cbase = col0;
#pragma unroll
        for (int j = 0; j < W; ++j) {
            uint32_t f = to_fraction<L>(w_[j]);
#pragma unroll
            for (int pp = 0; pp < NPAIR; ++pp) {
                const unsigned long long t = (unsigned long long)f * (unsigned long long)(L * L);
                f = (uint32_t)t;
                chunk[ci++] = lut[((uint32_t)(t >> 32) << 5) + lane];
                if (ci == 8) {
                    tmem_st8(lane_base + cbase, chunk);
                    cbase += 8;
                    ci = 0;
                }
            }
        }
        if (KC % 8) {
#pragma unroll
            for (int i = KC % 8; i < 8; ++i) chunk[i] = 0u;
            tmem_st8(lane_base + cbase, chunk);
        }
    };

    if (t0 < t1) load_tile(t0, kw, vw, kzv, vzv);
    for (int tile = t0; tile < t1; ++tile) {
        uint32_t kwn[W], vwn[W], kzn[TC_NGMAX], vzn[TC_NGMAX];
        if (tile + 1 < t1) load_tile(tile + 1, kwn, vwn, kzn, vzn);

        // ---- codes -> TMEM (A operands of both products)
        unpack_to_tmem(kw, COL_AK);
        unpack_to_tmem(vw, COL_AV);
        tc_wait_st();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int s = 0; s < KSTEPS; ++s)
                mma_ts_f16(tmem + COL_DK, tmem + COL_AK + 8 * s,
                           smem_desc(bq_addr + s * 2 * M::LBO_Q, M::LBO_Q, M::SBO_Q), idesc_k, s > 0);
            mma_commit(&mbar[0]);
        }
        const bool valid = tile * TILE + tid < n;
        float sk[TC_NGMAX], zk[TC_NGMAX], sv[TC_NGMAX], zv[TC_NGMAX];
#pragma unroll
        for (int gg = 0; gg < TC_NGMAX; ++gg) {
            sk[gg] = h2f((uint16_t)(kzv[gg] & 0xffffu));
            zk[gg] = __fmaf_rn(MID, sk[gg], h2f((uint16_t)(kzv[gg] >> 16)));
            sv[gg] = h2f((uint16_t)(vzv[gg] & 0xffffu));
            zv[gg] = __fmaf_rn(MID, sv[gg], h2f((uint16_t)(vzv[gg] >> 16)));
        }

        // ---- logits of my slot
        if (!mbar_wait(&mbar[0], ph_k)) timeout = true;
        ph_k ^= 1u;
        tc_fence_after();
        uint32_t dk[32];
        {
            uint32_t* d0 = dk;
            tmem_ld16(lane_base + COL_DK, *reinterpret_cast<uint32_t(*)[16]>(d0));
            if (NK > 16) tmem_ld16(lane_base + COL_DK + 16, *reinterpret_cast<uint32_t(*)[16]>(d0 + 16));
        }
        tc_wait_ld();
        float lg[TC_GMAX];
#pragma unroll
        for (int h = 0; h < TC_GMAX; ++h) {
            float acc = 0.f;
#pragma unroll
            for (int gg = 0; gg < TC_NGMAX; ++gg)
                if (gg < NG && h < g)
                    acc += sk[gg] * __uint_as_float(dk[gg * g + h]) + zk[gg] * qsum[gg * TC_GMAX + h];
            lg[h] = (valid && h < g) ? acc * scale_log2 : -__int_as_float(0x7f800000);
            const float mx = warp_max(lg[h]);
            if (lane == 0) red[warp * 48 + h] = mx;
        }
        // slots past n may hold stale words (after appends): their p, P' and zero terms are exact zeros
        __syncthreads();
        float alpha[TC_GMAX], p[TC_GMAX];
#pragma unroll
        for (int h = 0; h < TC_GMAX; ++h) {
            const float mt = fmaxf(fmaxf(red[h], red[48 + h]), fmaxf(red[96 + h], red[144 + h]));
            const float mn = fmaxf(m[h], mt);
            alpha[h] = h < g ? exp2f(m[h] - mn) : 0.f;
            m[h] = mn;
            p[h] = (valid && h < g) ? exp2f(lg[h] - mn) : 0.f;
            lacc[h] = lacc[h] * alpha[h] + p[h];
#pragma unroll
            for (int gg = 0; gg < TC_NGMAX; ++gg)  // a stale slot's scale/zero may be NaN: never multiply it
                zacc[gg][h] = zacc[gg][h] * alpha[h] + (valid ? p[h] * zv[gg] : 0.f);
        }
        // ---- P' = p s_V as two fp16 limbs, into my slot's row of B_P
#pragma unroll
        for (int gg = 0; gg < TC_NGMAX; ++gg) {
            if (gg < NG) {
#pragma unroll
                for (int h = 0; h < TC_GMAX; ++h) {
                    if (h < g) {
                        const float pv = valid ? p[h] * sv[gg] : 0.f;
                        const __half hi = __float2half_rn(pv);
                        const __half lo = __float2half_rn(pv - __half2float(hi));
                        const int n0 = gg * GSTR + h, n1 = gg * GSTR + g + h;
                        *reinterpret_cast<__half*>(bp_my + (uint32_t)(n0 >> 3) * M::SBO_P + (uint32_t)(n0 & 7) * 16u) = hi;
                        *reinterpret_cast<__half*>(bp_my + (uint32_t)(n1 >> 3) * M::SBO_P + (uint32_t)(n1 & 7) * 16u) = lo;
                    }
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int s = 0; s < KSTEPS; ++s)
                mma_ts_f16(tmem + COL_DV, tmem + COL_AV + 8 * s,
                           smem_desc(bp_addr + s * 2 * M::LBO_P, M::LBO_P, M::SBO_P), idesc_v, s > 0);
            mma_commit(&mbar[1]);
        }
        if (!mbar_wait(&mbar[1], ph_v)) timeout = true;
        ph_v ^= 1u;
        tc_fence_after();
        uint32_t dv[16];
        if (GSTR == 8) {
            tmem_ld8(lane_base + COL_DV + grp_d * 8, *reinterpret_cast<uint32_t(*)[8]>(dv));
        } else {
            tmem_ld16(lane_base + COL_DV + grp_d * 16, dv);
        }
        tc_wait_ld();
#pragma unroll
        for (int h = 0; h < TC_GMAX; ++h)
            if (h < g) O[h] = O[h] * alpha[h] + __uint_as_float(dv[h]) + __uint_as_float(dv[g + h]);
        tc_fence_before();

#pragma unroll
        for (int j = 0; j < W; ++j) {
            kw[j] = kwn[j];
            vw[j] = vwn[j];
        }
#pragma unroll
        for (int gg = 0; gg < TC_NGMAX; ++gg) {
            kzv[gg] = kzn[gg];
            vzv[gg] = vzn[gg];
        }
    }

    // ---------------- epilogue: block sums of the denominators and zero terms, partial state out
    {
        float vals[48];
        int nvals = 0;
#pragma unroll
        for (int h = 0; h < TC_GMAX; ++h) vals[nvals++] = lacc[h];
#pragma unroll
        for (int gg = 0; gg < TC_NGMAX; ++gg)
#pragma unroll
            for (int h = 0; h < TC_GMAX; ++h) vals[nvals++] = zacc[gg][h];
#pragma unroll
        for (int i = 0; i < 40; ++i) {
            float v = vals[i];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == 0) red[warp * 48 + i] = v;
        }
    }
    __syncthreads();
    if (tid < 40) fin[tid] = red[tid] + red[48 + tid] + red[96 + tid] + red[144 + tid];
    __syncthreads();
    float* out = ws + ((size_t)u * nsplit_total + split_off + split) * g * (D + 2);
    for (int h = 0; h < g; ++h) {
        out[h * (D + 2) + tid] = O[h] + fin[TC_GMAX + grp_d * TC_GMAX + h];
        if (tid == 0) {
            out[h * (D + 2) + D] = m[h];
            out[h * (D + 2) + D + 1] = fin[h];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
    if (timeout) atomicOr(status, SEMKV_STATUS_TIMEOUT);
    // the merge reads this launch's and the previous launch's partials: finish only after it
    if (wait_for_prior) asm volatile("griddepcontrol.wait;" ::: "memory");
}

template <int L>
static size_t tc_smem() { return TcSmem<L>::TOTAL; }

bool decode_tc_supported(int L, int G, int g)
{
    if (G < 32 || g < 1 || g > TC_GMAX) return false;
    switch (L) {
#define SEMKV_TCOK(LL) \
    case LL: return TcShape<LL>::ok;
        SEMKV_TCOK(2) SEMKV_TCOK(4) SEMKV_TCOK(5) SEMKV_TCOK(6) SEMKV_TCOK(7) SEMKV_TCOK(8)
        SEMKV_TCOK(10) SEMKV_TCOK(11) SEMKV_TCOK(12) SEMKV_TCOK(13) SEMKV_TCOK(14) SEMKV_TCOK(15) SEMKV_TCOK(16)
#undef SEMKV_TCOK
        default: return false;
    }
}

template <int L>
static void launch_tc(const SegView& seg, const uint16_t* q, int units, int H, int g, int G, float scale_log2,
                      int nsplit, int split_off, int nsplit_total, float* ws, int32_t* status, bool dependent,
                      cudaStream_t st)
{
    // at most two CTAs per SM: each holds 256 of the SM's 512 TMEM columns
    const size_t sm = tc_smem<L>() > 100u * 1024u ? tc_smem<L>() : 100u * 1024u;
    cudaFuncSetAttribute(k_decode_tc<L>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)nsplit, (unsigned)units);
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = sm;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = dependent ? 1 : 0;
    cudaLaunchKernelEx(&cfg, k_decode_tc<L>, seg, q, H, g, G, scale_log2, nsplit, split_off, nsplit_total, ws, status,
                       dependent ? 1 : 0);
}

void launch_decode_tc(const SegView& seg, const uint16_t* q, int units, int H, int g, int G, float scale_log2,
                      int nsplit, int split_off, int nsplit_total, float* ws, int32_t* status, bool dependent,
                      cudaStream_t st)
{
    if (nsplit == 0 || units == 0) return;
    switch (seg.L) {
#define SEMKV_TC(LL)                                                                                                 \
    case LL:                                                                                                         \
        launch_tc<LL>(seg, q, units, H, g, G, scale_log2, nsplit, split_off, nsplit_total, ws, status, dependent, st); \
        break;
        SEMKV_TC(2) SEMKV_TC(4) SEMKV_TC(5) SEMKV_TC(6) SEMKV_TC(7) SEMKV_TC(8)
        SEMKV_TC(10) SEMKV_TC(11) SEMKV_TC(12) SEMKV_TC(13) SEMKV_TC(14) SEMKV_TC(15) SEMKV_TC(16)
#undef SEMKV_TC
        default: break;
    }
}

}  // namespace semkv
