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
//   fetch    a tile's words and scale/zero pairs are four contiguous chunks; one thread moves them
//            into a two-stage shared-memory ring with cp.async.bulk (no multicast), two tiles ahead.
//   unpack   each word becomes the fixed-point base-L fraction (see common.cuh); one 32x32->64
//            multiply by L^2 yields the next two digits as one index P < L^2, and a per-lane copy
//            of a table in shared memory maps P to the two centred codes (c - (L-1)/2) as an fp16
//            pair, stored to TMEM with tcgen05.st.
//   q.k      D_K[slot][(group,head)] = sum over the group's channels of (c - m) q_head: a chain of
//            tcgen05.mma (M=128 slots, N = groups x heads, K = code slots), A (codes) in TMEM and
//            B (the fp16 queries, zero outside each group) in shared memory.
//   (per-channel K grids: B holds q_hd s_d as two fp16 limbs instead, and the zero terms are one
//   constant per head: logit = scale * (D_K[hi limb] + D_K[lo limb] + sum_d q_hd (z_d + m s_d)))
//   softmax  logit = scale * sum_group [ s_K D_K + (z_K + m s_K) sum_{group} q ]; online softmax
//            in the log2 domain across tiles (warp shuffles + one shared exchange per tile).
//   p.V      D_V[channel][(group,limb,head)] = sum_slots (c - m) P', P' = p s_V split into two
//            fp16 limbs (P' = hi + lo, ~22 bits kept); A = V codes in the same TMEM columns (the
//            q.k product has completed), B = P' in shared memory written by the slot threads.
//            The zero terms sum_t p (z_V + m s_V) and the denominators stay on the CUDA cores.
// K and V may use different level counts (a radix configuration per tensor, TcRadix).
// Each CTA writes (max, sum, unnormalized o) per query head to the workspace; k_decode_merge
// combines the splits.  Every mbarrier wait is bounded; a timeout sets SEMKV_STATUS_TIMEOUT.
#include "append.cuh"
#include "common.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace semkv {

// One tensor's codes in TMEM: words per row (K) or per 128-slot column (V), digit pairs per word
// (TMEM columns), and the MMA K-steps of 16 fp16 elements that cover them.
template <int L>
struct TcRadix {
    using R = Radix<L>;
    static constexpr int k = R::k;
    static constexpr int W = ceil_div(128, k);     // words per slot row (K) = per channel per tile (V)
    static constexpr int NPAIR = (k + 1) / 2;      // digit pairs (TMEM columns) per word
    static constexpr int KC = W * NPAIR;           // TMEM columns of one unpacked row
    static constexpr int KCP = (KC + 7) / 8 * 8;   // padded to whole MMA K-steps (16 fp16)
    static constexpr int KSTEPS = KCP / 8;
    static constexpr int KSLOTS = 2 * KCP;         // fp16 elements along K
    static constexpr bool ok = (R::pow2 || R::frac_ok) && KCP <= 80;
    static constexpr uint32_t LUT_BYTES = (uint32_t)L * L * 32 * 4;
};

// LK, LV: level counts of the K and the V codes of the segment (equal unless V has its own)
template <int LK, int LV, int GQ, int NG>
struct Tc {
    using RK = TcRadix<LK>;
    using RV = TcRadix<LV>;
    static constexpr int D = 128;
    static constexpr int G = D / NG;
    static constexpr int NK = (NG * GQ + 15) / 16 * 16;  // N of q.k
    static constexpr int GSTR = 2 * GQ <= 8 ? 8 : 16;    // D_V columns per group: limb-major, head-minor
    static constexpr int NV = NG * GSTR < 16 ? 16 : NG * GSTR;
    static constexpr uint32_t COL_A = 0, COL_DK = 80, COL_DV = 96, TMEM_COLS = 128;
    static constexpr bool ok = RK::ok && RV::ok && NK <= 16 && NV <= 32 && G >= 32;
    // shared memory
    static constexpr uint32_t LBO_Q = 128, SBO_Q = (RK::KSLOTS / 8) * 128;
    static constexpr uint32_t LBO_P = 144, SBO_P = (RV::KSLOTS / 8) * 144;  // 144: conflict-free slot writes
    static constexpr uint32_t STAGE_K = 0, STAGE_V = RK::W * 512, STAGE_KZ = STAGE_V + RV::W * 512,
                              STAGE_VZ = STAGE_KZ + NG * 512, STAGE_BYTES = STAGE_VZ + NG * 512;
    static constexpr uint32_t LUT_K = 0, LUT_V = LK == LV ? 0u : (RK::LUT_BYTES + 127) / 128 * 128;
    static constexpr uint32_t STAGES = (LUT_V + (LK == LV ? RK::LUT_BYTES : RV::LUT_BYTES) + 127) / 128 * 128;
    static constexpr uint32_t BQ = STAGES + 2 * STAGE_BYTES;
    static constexpr uint32_t BP = BQ + (NK / 8) * SBO_Q;
    static constexpr uint32_t QSUM = BP + (NV / 8) * SBO_P;
    static constexpr uint32_t RED = QSUM + NG * GQ * 4;
    static constexpr uint32_t TOTAL = RED + 4 * 32 * 4;
};

// 32-bit fixed-point fraction ~ w / L^k, within one unit of the last digit
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

__host__ __device__ constexpr uint32_t core_off(int n, int ks, uint32_t lbo, uint32_t sbo)
{
    return (uint32_t)(n >> 3) * sbo + (uint32_t)(ks >> 3) * lbo + (uint32_t)(n & 7) * 16u + (uint32_t)(ks & 7) * 2u;
}

// One thread's row of codes -> TMEM: the tensor's W words (shared address `words` + 4 tid, stride
// 512 B) become KCP columns of fp16 code pairs at `taddr` (this thread's lane), through the code
// table whose lane copy starts at `lut_lane` (entry P at + 128 P bytes).
template <int L>
__device__ __forceinline__ void unpack_to_tmem(uint32_t words, uint32_t lut_lane, uint32_t taddr, int tid)
{
    using RC = TcRadix<L>;
    constexpr int W = RC::W, NPAIR = RC::NPAIR, KC = RC::KC;
    uint32_t wv[W];
#pragma unroll
    for (int j = 0; j < W; ++j) wv[j] = lds_u32_after_wait(words + (uint32_t)(j * 512 + 4 * tid));
    uint32_t chunk[8];
    int ci = 0;
    uint32_t cbase = 0;
#pragma unroll
    for (int j = 0; j < W; ++j) {
        uint32_t f = to_fraction<L>(wv[j]);
#pragma unroll
        for (int pp = 0; pp < NPAIR; ++pp) {
            const unsigned long long t = (unsigned long long)f * (unsigned long long)(L * L);
            f = (uint32_t)t;
            chunk[ci++] = lds_u32(lut_lane + ((uint32_t)(t >> 32) << 7));
            if (ci == 8) {
                tmem_st8(taddr + cbase, chunk);
                cbase += 8;
                ci = 0;
            }
        }
    }
    if (KC % 8) {
#pragma unroll
        for (int i = KC % 8; i < 8; ++i) chunk[i] = 0u;
        tmem_st8(taddr + cbase, chunk);
    }
}

// KPC: per-channel K grids (seg.kc): B_Q holds q_hd s_d as two fp16 limbs per head (rows h and
// GQ + h), and the zero terms sum_d q_hd (z_d + m s_d) are one constant per head
template <int LK, int LV, int GQ, int NG, bool APP, bool KPC>
__global__ void __launch_bounds__(128, 4) k_decode_tc(SegView seg, const uint16_t* __restrict__ q, int H,
                                                       float scale_log2, int nsplit, int split_off, int nsplit_total,
                                                       float* __restrict__ ws, int32_t* __restrict__ status,
                                                       int wait_for_prior, semkv_cache_t cache,
                                                       const uint16_t* __restrict__ knew,
                                                       const uint16_t* __restrict__ vnew,
                                                       const float* __restrict__ snew)
{
    using C = Tc<LK, LV, GQ, NG>;
    using RK = typename C::RK;
    using RV = typename C::RV;
    constexpr int D = 128, G = C::G, NK = C::NK, NV = C::NV, GSTR = C::GSTR;
    constexpr float MID_K = 0.5f * (float)(LK - 1), MID_V = 0.5f * (float)(LV - 1);
    constexpr float NEG_INF = -__builtin_huge_valf();

    // a dependent launch (the other segment) may start on free SMs right away
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    const int split = blockIdx.x, u = blockIdx.y, b = u / H, hk = u % H, Hq = H * GQ;
    // the warp index through a shuffle from lane 0: the compiler then keeps the addresses derived
    // from it (TMEM lanes, MMA operands) in uniform registers
    const int tid = threadIdx.x, lane = tid & 31, warp = __shfl_sync(0xffffffffu, tid >> 5, 0);

    extern __shared__ __align__(1024) unsigned char smem[];
    uint32_t* lut = reinterpret_cast<uint32_t*>(smem + C::LUT_K);
    uint32_t* lut_v = reinterpret_cast<uint32_t*>(smem + C::LUT_V);
    unsigned char* stage0 = smem + C::STAGES;
    unsigned char* bq = smem + C::BQ;
    unsigned char* bp = smem + C::BP;
    float* qsum = reinterpret_cast<float*>(smem + C::QSUM);  // [NG][GQ]
    float* red = reinterpret_cast<float*>(smem + C::RED);    // [4][32]
    __shared__ __align__(8) uint64_t mbar[4];                // 0: q.k done, 1: p.V done, 2/3: stage full
    __shared__ uint32_t tmem_base_s;

    // append and attend in one pass (APP; knew != nullptr): every CTA works out the new token's grid
    // and its segment's new length from the inputs alone (the counts are updated by the merge,
    // after every CTA has read them); the CTA whose tiles hold the new slot writes the row first
    int n = seg.n[u];
    int append_tile = -1;
    bool app_hi = false;
    int app_nh = 0, app_nl = 0;
    if constexpr (APP) {
        app_nh = cache.n_hi[u];
        app_nl = cache.n_lo[u];
        app_hi = snew[u] > cache.tau[u];  // NaN compares false: the token goes lo
        if (append_fits(cache, app_hi, app_nh, app_nl) && app_hi == (seg.is_hi != 0)) append_tile = n++ / TILE;
    }
    const int tiles = min(ceil_div(n, TILE), seg.tiles_cap);
    int t0, t1;
    split_tiles(tiles, nsplit, split, t0, t1);
    if (APP && append_tile >= t0 && append_tile < t1) {
        const bool bad = append_row(cache, u, app_hi, app_nh, app_nl, h2f(knew[(size_t)u * D + tid]),
                                    h2f(vnew[(size_t)u * D + tid]));
        if (bad && tid == 0) atomicOr(status, SEMKV_STATUS_NONFINITE_KV);
        // the row's words (plain stores and reductions) before this CTA's bulk copies read the tile
        asm volatile("fence.proxy.async.global;" ::: "memory");
        __syncthreads();
    }

    auto issue_fetch = [&](int tile, int stg) {  // one thread
        unsigned char* dst = stage0 + stg * C::STAGE_BYTES;
        const size_t tb = (size_t)u * seg.tiles_cap + tile;
        mbar_arrive_expect_tx(&mbar[2 + stg], C::STAGE_BYTES);
        bulk_g2s(dst + C::STAGE_K, seg.k + tb * RK::W * TILE, RK::W * 512, &mbar[2 + stg]);
        bulk_g2s(dst + C::STAGE_V, seg.v + tb * RV::W * D, RV::W * 512, &mbar[2 + stg]);
        bulk_g2s(dst + C::STAGE_KZ, seg.kz + tb * NG * TILE, NG * 512, &mbar[2 + stg]);
        bulk_g2s(dst + C::STAGE_VZ, seg.vz + tb * NG * TILE, NG * 512, &mbar[2 + stg]);
    };

    // ---------------- set-up: TMEM, barriers, first fetches, code table, B_Q, B_P zeroed
    if (warp == 0) {
        tmem_alloc(&tmem_base_s, C::TMEM_COLS);
        tmem_relinquish();
    }
    if (tid == 0) {
#pragma unroll
        for (int i = 0; i < 4; ++i) mbar_init(&mbar[i], 1);
        fence_mbar_init();
        if (t0 < t1) issue_fetch(t0, 0);
        if (t0 + 1 < t1) issue_fetch(t0 + 1, 1);
    }
    // the GQ query rows: loads issued first, their latency hidden behind the table build; staged in
    // the B_P area (zeroed once B_Q is built)
    uint16_t* qs = reinterpret_cast<uint16_t*>(bp);
    constexpr int QV = GQ * D / 8;  // 16-byte pieces of the query rows
    uint4 qv[(QV + 127) / 128];
    {
        const uint4* qu = reinterpret_cast<const uint4*>(q + ((size_t)b * Hq + (size_t)hk * GQ) * D);
#pragma unroll
        for (int e = 0; e < (QV + 127) / 128; ++e)
            if (tid + 128 * e < QV) qv[e] = __ldg(qu + tid + 128 * e);
    }
    for (int i = tid; i < LK * LK * 32; i += 128) {
        const int P = i >> 5;
        const __half2 pr = __floats2half2_rn((float)(P / LK) - MID_K, (float)(P % LK) - MID_K);  // exact: |x| <= 7.5
        lut[i] = *reinterpret_cast<const uint32_t*>(&pr);
    }
    if constexpr (LV != LK) {
        for (int i = tid; i < LV * LV * 32; i += 128) {
            const int P = i >> 5;
            const __half2 pr = __floats2half2_rn((float)(P / LV) - MID_V, (float)(P % LV) - MID_V);
            lut_v[i] = *reinterpret_cast<const uint32_t*>(&pr);
        }
    }
#pragma unroll
    for (int e = 0; e < (QV + 127) / 128; ++e)
        if (tid + 128 * e < QV) reinterpret_cast<uint4*>(qs)[tid + 128 * e] = qv[e];
    __syncthreads();
    for (int ks = tid; ks < RK::KSLOTS; ks += 128) {
        const int col = ks >> 1, h2 = ks & 1, j = col / RK::NPAIR, pp = col % RK::NPAIR;
        const int pos = pair_digit(RK::k, pp, h2);
        const int dim = (col < RK::KC && pos >= 0) ? j * RK::k + pos : D;
        const int dgrp = dim < D ? dim / G : -1;
        if constexpr (KPC) {
            static_assert(2 * GQ <= NK, "two limbs per head must fit the q.k columns");
            const float sd = dim < D ? h2f((uint16_t)(seg.kc[(size_t)u * 256 + dim] & 0xffffu)) : 0.f;
#pragma unroll
            for (int nrow = 0; nrow < NK; ++nrow) {
                uint16_t v = 0;
                if (nrow < 2 * GQ && dim < D) {
                    const float x = h2f(qs[(nrow % GQ) * D + dim]) * sd;
                    const __half hi = __float2half_rn(x);
                    v = __half_as_ushort(nrow < GQ ? hi : __float2half_rn(x - __half2float(hi)));
                }
                *reinterpret_cast<uint16_t*>(bq + core_off(nrow, ks, C::LBO_Q, C::SBO_Q)) = v;
            }
        } else {
#pragma unroll
            for (int nrow = 0; nrow < NK; ++nrow) {
                const uint16_t v = (nrow < NG * GQ && nrow / GQ == dgrp) ? qs[(nrow % GQ) * D + dim] : (uint16_t)0;
                *reinterpret_cast<uint16_t*>(bq + core_off(nrow, ks, C::LBO_Q, C::SBO_Q)) = v;
            }
        }
    }
    if constexpr (KPC) {
        // zero term of each head: 8 threads per head, 16 channels each
        const int h = tid >> 3, part = tid & 7;
        float a = 0.f;
        if (h < GQ) {
#pragma unroll 4
            for (int e = 0; e < 16; ++e) {
                const int d = part * 16 + e;
                const uint32_t gk = seg.kc[(size_t)u * 256 + d];
                const float sd = h2f((uint16_t)(gk & 0xffffu));
                a += h2f(qs[h * D + d]) * __fmaf_rn(MID_K, sd, h2f((uint16_t)(gk >> 16)));
            }
        }
        a += __shfl_xor_sync(0xffffffffu, a, 4);
        a += __shfl_xor_sync(0xffffffffu, a, 2);
        a += __shfl_xor_sync(0xffffffffu, a, 1);
        if (h < GQ && part == 0) qsum[h] = a;
    } else {
        // per-group query sums: 8 threads per (group, head), G/8 channels each
        const int si = tid >> 3, part = tid & 7;
        float a = 0.f;
        if (si < NG * GQ) {
            const int grp = si / GQ, h = si % GQ;
            const __half2* qp = reinterpret_cast<const __half2*>(qs + h * D + grp * G + part * (G / 8));
#pragma unroll
            for (int e = 0; e < G / 16; ++e) {
                const float2 f2 = __half22float2(qp[e]);
                a += f2.x + f2.y;
            }
        }
        a += __shfl_xor_sync(0xffffffffu, a, 4);
        a += __shfl_xor_sync(0xffffffffu, a, 2);
        a += __shfl_xor_sync(0xffffffffu, a, 1);
        if (si < NG * GQ && part == 0) qsum[si] = a;
    }
    __syncthreads();
    for (int i = tid; i < (int)((NV / 8) * C::SBO_P / 16); i += 128) reinterpret_cast<uint4*>(bp)[i] = make_uint4(0, 0, 0, 0);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = __shfl_sync(0xffffffffu, tmem_base_s, 0);
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    constexpr uint32_t idesc_k = idesc_f16_f32(128, NK), idesc_v = idesc_f16_f32(128, NV);
    const uint32_t bq_addr = smem_u32(bq), bp_addr = smem_u32(bp);

    // my slot's row of B_P (slot tid -> K index along the unpacked V words)
    const int vrank = RV::k - 1 - (tid % RV::k);
    const int my_ks = 2 * ((tid / RV::k) * RV::NPAIR + (vrank >> 1)) + (vrank & 1);
    unsigned char* bp_my = bp + (uint32_t)(my_ks >> 3) * C::LBO_P + (uint32_t)(my_ks & 7) * 2u;
    const int grp_d = tid / G;  // my channel's group (uniform over a warp: G >= 32)

    float m[GQ], O[GQ], lacc[GQ], zacc[NG][GQ];
#pragma unroll
    for (int h = 0; h < GQ; ++h) {
        m[h] = NEG_INF;
        O[h] = lacc[h] = 0.f;
#pragma unroll
        for (int gg = 0; gg < NG; ++gg) zacc[gg][h] = 0.f;
    }
    uint32_t ph_k = 0, ph_v = 0;
    bool timeout = false;

    // this lane's copies of the code tables: entry P at + 128 P bytes
    const uint32_t lut_lane_k = smem_u32(lut + lane), lut_lane_v = smem_u32(lut_v + lane);
    const uint32_t taddr_a = lane_base + C::COL_A;

    for (int tile = t0, it = 0; tile < t1; ++tile, ++it) {
        const int stg = it & 1;
        const unsigned char* sb = stage0 + stg * C::STAGE_BYTES;
        if (!mbar_wait(&mbar[2 + stg], (uint32_t)(it >> 1) & 1u)) timeout = true;

        // ---- K codes -> TMEM, q.k
        unpack_to_tmem<LK>(smem_u32(sb + C::STAGE_K), lut_lane_k, taddr_a, tid);
        tc_wait_st();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int s = 0; s < RK::KSTEPS; ++s)
                mma_ts_f16(tmem + C::COL_DK, tmem + C::COL_A + 8 * s,
                           smem_desc(bq_addr + s * 2 * C::LBO_Q, C::LBO_Q, C::SBO_Q), idesc_k, s > 0);
            mma_commit(&mbar[0]);
        }
        const bool valid = tile * TILE + tid < n;
        float sk[NG], zk[NG], sv[NG], zv[NG];
#pragma unroll
        for (int gg = 0; gg < NG; ++gg) {
            const uint32_t kzv = reinterpret_cast<const uint32_t*>(sb + C::STAGE_KZ)[gg * 128 + tid];
            const uint32_t vzv = reinterpret_cast<const uint32_t*>(sb + C::STAGE_VZ)[gg * 128 + tid];
            sk[gg] = h2f((uint16_t)(kzv & 0xffffu));
            zk[gg] = __fmaf_rn(MID_K, sk[gg], h2f((uint16_t)(kzv >> 16)));
            sv[gg] = h2f((uint16_t)(vzv & 0xffffu));
            zv[gg] = __fmaf_rn(MID_V, sv[gg], h2f((uint16_t)(vzv >> 16)));
        }
        if (!mbar_wait(&mbar[0], ph_k)) timeout = true;
        ph_k ^= 1u;
        tc_fence_after();
        uint32_t dk[16];
        tmem_ld16(lane_base + C::COL_DK, dk);
        tc_wait_ld();

        // ---- online softmax over the tile (log2 domain)
        float lg[GQ];
#pragma unroll
        for (int h = 0; h < GQ; ++h) {
            float acc = 0.f;
            if constexpr (KPC) {
                acc = __uint_as_float(dk[h]) + __uint_as_float(dk[GQ + h]) + qsum[h];
            } else {
#pragma unroll
                for (int gg = 0; gg < NG; ++gg)
                    acc += sk[gg] * __uint_as_float(dk[gg * GQ + h]) + zk[gg] * qsum[gg * GQ + h];
            }
            lg[h] = valid ? acc * scale_log2 : NEG_INF;
            const float mx = warp_max_redux(lg[h]);
            if (lane == 0) red[warp * 32 + h] = mx;
        }
        __syncthreads();
        float alpha[GQ], p[GQ];
#pragma unroll
        for (int h = 0; h < GQ; ++h) {
            const float mt = fmaxf(fmaxf(red[h], red[32 + h]), fmaxf(red[64 + h], red[96 + h]));
            const float mn = fmaxf(m[h], mt);
            alpha[h] = ex2_approx(m[h] - mn);
            m[h] = mn;
            // slots past n may hold stale words (after appends): exact zeros, never a product
            p[h] = valid ? ex2_approx(lg[h] - mn) : 0.f;
            lacc[h] = lacc[h] * alpha[h] + p[h];
#pragma unroll
            for (int gg = 0; gg < NG; ++gg) zacc[gg][h] = zacc[gg][h] * alpha[h] + (valid ? p[h] * zv[gg] : 0.f);
        }
        // ---- P' = p s_V as two fp16 limbs, into my slot's row of B_P
#pragma unroll
        for (int gg = 0; gg < NG; ++gg) {
#pragma unroll
            for (int h = 0; h < GQ; ++h) {
                const float pv = valid ? p[h] * sv[gg] : 0.f;
                const __half hi = __float2half_rn(pv);
                const __half lo = __float2half_rn(pv - __half2float(hi));
                const int n0 = gg * GSTR + h, n1 = gg * GSTR + GQ + h;
                *reinterpret_cast<__half*>(bp_my + (uint32_t)(n0 >> 3) * C::SBO_P + (uint32_t)(n0 & 7) * 16u) = hi;
                *reinterpret_cast<__half*>(bp_my + (uint32_t)(n1 >> 3) * C::SBO_P + (uint32_t)(n1 & 7) * 16u) = lo;
            }
        }
        // ---- V codes -> TMEM (same columns: the q.k product has completed), p.V
        unpack_to_tmem<LV>(smem_u32(sb + C::STAGE_V), lut_lane_v, taddr_a, tid);
        tc_wait_st();
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int s = 0; s < RV::KSTEPS; ++s)
                mma_ts_f16(tmem + C::COL_DV, tmem + C::COL_A + 8 * s,
                           smem_desc(bp_addr + s * 2 * C::LBO_P, C::LBO_P, C::SBO_P), idesc_v, s > 0);
            mma_commit(&mbar[1]);
            // this stage has been read by every thread: refill it two tiles ahead
            if (tile + 2 < t1) {
                fence_async_smem();
                issue_fetch(tile + 2, stg);
            }
        }
        if (!mbar_wait(&mbar[1], ph_v)) timeout = true;
        ph_v ^= 1u;
        tc_fence_after();
        uint32_t dv[16];
        if constexpr (GSTR == 8) {
            tmem_ld8(lane_base + C::COL_DV + grp_d * 8, *reinterpret_cast<uint32_t(*)[8]>(dv));
        } else {
            tmem_ld16(lane_base + C::COL_DV + grp_d * 16, dv);
        }
        tc_wait_ld();
#pragma unroll
        for (int h = 0; h < GQ; ++h) O[h] = O[h] * alpha[h] + __uint_as_float(dv[h]) + __uint_as_float(dv[GQ + h]);
        tc_fence_before();
    }

    // ---------------- epilogue: block sums of the denominators and zero terms, partial state out
    constexpr int NVAL = GQ + NG * GQ;  // <= 32
    float vals[NVAL];
#pragma unroll
    for (int h = 0; h < GQ; ++h) vals[h] = lacc[h];
#pragma unroll
    for (int gg = 0; gg < NG; ++gg)
#pragma unroll
        for (int h = 0; h < GQ; ++h) vals[GQ + gg * GQ + h] = zacc[gg][h];
    __syncthreads();  // every thread is past its last read of red[]
#pragma unroll
    for (int i = 0; i < NVAL; ++i) {
        float v = vals[i];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) red[warp * 32 + i] = v;
    }
    __syncthreads();
    float* out = ws + ((size_t)u * nsplit_total + split_off + split) * GQ * (D + 2);
#pragma unroll
    for (int h = 0; h < GQ; ++h) {
        const int zi = GQ + grp_d * GQ + h;
        const float zsum = red[zi] + red[32 + zi] + red[64 + zi] + red[96 + zi];
        out[h * (D + 2) + tid] = O[h] + zsum;
        if (tid == 0) {
            out[h * (D + 2) + D] = m[h];
            out[h * (D + 2) + D + 1] = red[h] + red[32 + h] + red[64 + h] + red[96 + h];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
    if (timeout) atomicOr(status, SEMKV_STATUS_TIMEOUT);
    // the merge reads this launch's and the previous launch's partials: finish only after it
    if (wait_for_prior) asm volatile("griddepcontrol.wait;" ::: "memory");
}

template <int LK, int LV, int GQ, int NG, bool KPC>
static void launch_tc(const SegView& seg, const uint16_t* q, int units, int H, float scale_log2, int nsplit,
                      int split_off, int nsplit_total, float* ws, int32_t* status, bool dependent,
                      const AppendIn& app, cudaStream_t st)
{
    using C = Tc<LK, LV, GQ, NG>;
    // at most four CTAs per SM: each holds 128 of the SM's 512 TMEM columns
    const size_t sm = C::TOTAL > 48u * 1024u ? C::TOTAL : 48u * 1024u;
    // the plain decode and the one that appends first are separate instantiations, so that the
    // plain one carries no append code
    const auto kern = app.k ? k_decode_tc<LK, LV, GQ, NG, true, KPC> : k_decode_tc<LK, LV, GQ, NG, false, KPC>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
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
    cudaLaunchKernelEx(&cfg, kern, seg, q, H, scale_log2, nsplit, split_off, nsplit_total, ws,
                       status, dependent ? 1 : 0, app.cache, app.k, app.v, app.score);
}

// instantiated shapes: K and V level counts (equal: L in {4, 5, 6, 8, 16}; V with its own count:
// six common pairs) x (g, groups) whose accumulators fit 128 TMEM columns; per-channel K grids for
// the equal counts on the common shapes
#define SEMKV_TC_SHAPES(X, LK, LV) X(LK, LV, 2, 1, false) X(LK, LV, 2, 2, false) X(LK, LV, 2, 4, false) \
    X(LK, LV, 4, 1, false) X(LK, LV, 4, 2, false) X(LK, LV, 4, 4, false) X(LK, LV, 8, 1, false) X(LK, LV, 8, 2, false) \
    X(LK, LV, 4, 1, true) X(LK, LV, 4, 2, true) X(LK, LV, 8, 1, true) X(LK, LV, 8, 2, true)
#define SEMKV_TC_SHAPES_KV(X, LK, LV) X(LK, LV, 2, 2, false) X(LK, LV, 4, 1, false) X(LK, LV, 4, 2, false) \
    X(LK, LV, 8, 1, false) X(LK, LV, 8, 2, false)
#define SEMKV_TC_LEVELS(X) SEMKV_TC_SHAPES(X, 4, 4) SEMKV_TC_SHAPES(X, 5, 5) SEMKV_TC_SHAPES(X, 6, 6) \
    SEMKV_TC_SHAPES(X, 8, 8) SEMKV_TC_SHAPES(X, 16, 16) SEMKV_TC_SHAPES_KV(X, 8, 4) SEMKV_TC_SHAPES_KV(X, 5, 2) \
    SEMKV_TC_SHAPES_KV(X, 8, 5) SEMKV_TC_SHAPES_KV(X, 6, 4) SEMKV_TC_SHAPES_KV(X, 5, 4) SEMKV_TC_SHAPES_KV(X, 16, 8)

bool decode_tc_supported(int Lk, int Lv, int G, int g, bool kpc)
{
    if (G <= 0 || 128 % G) return false;
    const int ng = 128 / G;
#define SEMKV_TC_OK(LK, LV, GG, NN, KP) \
    if (Lk == LK && Lv == LV && g == GG && ng == NN && kpc == KP) return Tc<LK, LV, GG, NN>::ok;
    SEMKV_TC_LEVELS(SEMKV_TC_OK)
#undef SEMKV_TC_OK
    return false;
}

void launch_decode_tc(const SegView& seg, const uint16_t* q, int units, int H, int g, int G, float scale_log2,
                      int nsplit, int split_off, int nsplit_total, float* ws, int32_t* status, bool dependent,
                      const AppendIn& app, cudaStream_t st)
{
    if (nsplit == 0 || units == 0) return;
    const int ng = 128 / G;
    const bool kpc = seg.kc != nullptr;
#define SEMKV_TC_GO(LK, LV, GG, NN, KP)                                                                             \
    if (seg.L == LK && seg.Lv == LV && g == GG && ng == NN && kpc == KP) {                                       \
        launch_tc<LK, LV, GG, NN, KP>(seg, q, units, H, scale_log2, nsplit, split_off, nsplit_total, ws, status,  \
                                      dependent, app, st);                                                      \
        return;                                                                                                 \
    }
    SEMKV_TC_LEVELS(SEMKV_TC_GO)
#undef SEMKV_TC_GO
}

}  // namespace semkv
