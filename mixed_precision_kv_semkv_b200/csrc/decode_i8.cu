// GQA decode attention over the packed cache on the integer tensor cores (tcgen05, kind::i8).
//
// SemKV page, Abstract: tokens are stored on L-level grids (L need not be a power of two); the
// KVQuant blog page (section on the memory bottleneck) notes that long-sequence decoding is bound
// by reading the KV cache.  The packed words are read from HBM once and turned into one byte per
// code on chip (i8unpack.cuh); both products then run on the tensor cores with exact integer
// accumulation, so the codes are never converted to floating point:
//   q.k   D_K[slot][n] = sum_k A_K[slot][k] B_Q[n][k]: A = the slot's K codes (u8, in TMEM),
//         B = the unit's queries as three signed 8-bit limbs of a 22-bit fixed-point image
//         q * 2^F (s8, shared memory; one column per (group, limb, head), zero outside the group).
//         logit = scale * [ sum_group s_K (D_0 + 2^8 D_1 + 2^16 D_2) 2^-F + z_K sum_group q ].
//   p.V   D_V[channel][n] = sum_slots A_V[channel][k] B_P[k][n]: A = the channel's V codes (u8,
//         TMEM), B = P' = p s_V of each slot as a 22-bit fixed-point integer split into three
//         unsigned bytes (one 4-byte column group per (group, head); the tile's own power-of-two
//         scale per (group, head) keeps 22 bits relative to the tile's largest P').  The zero
//         terms sum_t p z_V and the denominators stay in fp32 on the CUDA cores.
//
// Work: one CTA per SM (512 threads = 4 warpgroups).  The tiles of one segment of all units form a
// line of units x tiles_cap tiles; worker w (one warpgroup) takes the tiles x with
// floor(x workers / line) = w, i.e. a contiguous range that may cross a unit boundary; each unit it
// touches gets one partial softmax state (max, sum, unnormalized o) in the workspace, at slot
// w - (first worker of the unit), and k_decode_merge combines them.  Per warpgroup: a two-stage
// shared-memory ring filled by cp.async.bulk (no multicast) one tile ahead, its own 128 TMEM
// columns (K codes, V codes, D_K, D_V), its own mbarriers and named barrier; the 4 warpgroups
// share the code table.  Every wait is bounded; a timeout sets SEMKV_STATUS_TIMEOUT.
#include "append.cuh"
#include "common.cuh"
#include "i8unpack.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace semkv {
namespace {

constexpr int round16(int x) { return (x + 15) / 16 * 16; }

template <int L, int GQ, int NG>
struct I8 {
    using P = U8Plan<L>;
    static constexpr int D = 128, G = D / NG;
    static constexpr int NK = round16(3 * NG * GQ);  // q.k columns: (group, limb, head)
    static constexpr int NV = round16(4 * NG * GQ);  // p.V columns: (group, head, byte)
    static constexpr bool ok = P::ok && NK <= 32 && NV <= 32 && G >= 32;
    // TMEM columns of a warpgroup (relative to its 128)
    static constexpr uint32_t COL_AK = 0, COL_AV = 32, COL_DK = 64, COL_DV = 96;
    // one tile in shared memory: K words [W][128], V words [W][128], K and V scale/zero [NG][128]
    static constexpr uint32_t ST_K = 0, ST_V = P::W * 512, ST_KZ = 2 * P::W * 512, ST_VZ = ST_KZ + NG * 512,
                              STAGE = ST_VZ + NG * 512;
    static constexpr uint32_t LUT_SPAN = (P::LUT_BYTES + 1023) / 1024 * 1024;
    // per warpgroup: 2 stages, B_Q, B_P, reduction scratch, mbarriers (0/1 stage full, 2 q.k done,
    // 3 p.V done).  At the start of a chunk, before its first p.V, the B_P area holds the query rows
    // (while B_Q is built) and then the append scratch.
    static constexpr uint32_t BP_SPAN = NV * 128 > GQ * 256 ? (NV * 128 > 704 ? NV * 128 : 704)
                                                            : (GQ * 256 > 704 ? GQ * 256 : 704);
    static constexpr uint32_t W_BQ = 2 * STAGE, W_BP = W_BQ + NK * 128, W_QS = W_BP, W_APP = W_BP,
                              W_RED = W_BP + (BP_SPAN + 127) / 128 * 128, W_BAR = W_RED + 4 * 16 * 4,
                              WG_SPAN = (W_BAR + 32 + 127) / 128 * 128;
    static constexpr uint32_t TOTAL = LUT_SPAN + 4 * WG_SPAN + 16;
    static constexpr uint32_t SMEM_MAX = 232448;  // per-block opt-in maximum on sm_100
    // B_Q: K-major core matrices (8 rows x 16 bytes); B_P: MN-major core matrices (16 bytes x 8 rows)
    static constexpr uint32_t LBO_Q = 128, SBO_Q = 1024;
    static constexpr uint32_t SBO_P = 128, LBO_P = (NV / 16) * 128;
    static constexpr uint32_t IDESC_QK = idesc_i8_s32(128, NK, true, false);
    static constexpr uint32_t IDESC_PV = idesc_i8_s32(128, NV, false, true);
};

__device__ __forceinline__ int exponent_of(float x) { return (int)((__float_as_uint(x) >> 23) & 0xFFu) - 127; }
__device__ __forceinline__ float pow2f(int e) { return __uint_as_float((uint32_t)(e + 127) << 23); }  // e in [-126, 127]

}  // namespace

struct I8Params {
    SegView seg;
    const uint16_t* q;
    int H, units, workers;
    float scale_log2;
    int slots, slot_off, slots_total;  // partial slots per unit of this segment, their offset, all segments'
    float* ws;
    int32_t* status;
    int wait_for_prior;
    semkv_cache_t cache;  // the appended token (knew != nullptr): fixed-threshold rule
    const uint16_t* knew;
    const uint16_t* vnew;
    const float* snew;
};

template <int L, int GQ, int NG, bool APP>
__global__ void __launch_bounds__(512, 1) k_decode_i8(const I8Params pr)
{
    using C = I8<L, GQ, NG>;
    using P = typename C::P;
    constexpr int D = 128, G = C::G, NK = C::NK, NV = C::NV;
    constexpr float NEG_INF = -__builtin_huge_valf();
    static_assert(C::TOTAL <= C::SMEM_MAX, "shared memory of one CTA");

    // a dependent launch (the other segment, then the merge) may start on free SMs right away
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    extern __shared__ __align__(1024) unsigned char smem[];
    // the warpgroup index through a shuffle from lane 0: the compiler then knows it is the same in
    // every lane and keeps the shared-memory and TMEM addresses derived from it (the MMA operands)
    // in uniform registers
    const int tid = threadIdx.x, wg = __shfl_sync(0xffffffffu, tid >> 7, 0), t = tid & 127, lane = tid & 31,
              wl = __shfl_sync(0xffffffffu, (tid >> 5) & 3, 0);
    const uint32_t bar_id = 1 + (uint32_t)wg;
    auto wg_sync = [&] { named_sync(bar_id, 128); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::LUT_SPAN + 4 * C::WG_SPAN);
    unsigned char* wsm = smem + C::LUT_SPAN + wg * C::WG_SPAN;
    uint64_t* bar = reinterpret_cast<uint64_t*>(wsm + C::W_BAR);
    uint16_t* qs = reinterpret_cast<uint16_t*>(wsm + C::W_QS);
    float* red = reinterpret_cast<float*>(wsm + C::W_RED);  // [4 warps][16]
    const uint32_t bq_addr = smem_u32(wsm + C::W_BQ), bp_addr = smem_u32(wsm + C::W_BP);
    const uint32_t lut_lane = smem_u32(smem) + 4u * (uint32_t)lane;

    // ---------------- set-up: TMEM (4 x 128 columns), code table, barriers
    if (tid < 32) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    if constexpr (P::C > 0) {
        // entry e: 32 lane copies at (e * 32 + lane) * 4; each warp computes 32 entries (one per
        // lane) and stores them lane by lane
        uint32_t* lut = reinterpret_cast<uint32_t*>(smem);
        for (int e0 = (tid >> 5) * 32; e0 < P::ENTRIES; e0 += 16 * 32) {
            const uint32_t v = (e0 + lane < P::ENTRIES) ? u8_entry<L>((uint32_t)(e0 + lane)) : 0u;
            const int n = P::ENTRIES - e0 < 32 ? P::ENTRIES - e0 : 32;
            for (int j = 0; j < n; ++j) lut[(e0 + j) * 32 + lane] = __shfl_sync(0xffffffffu, v, j);
        }
    }
    if (t == 0) {
#pragma unroll
        for (int i = 0; i < 4; ++i) mbar_init(&bar[i], 1);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = __shfl_sync(0xffffffffu, *tmem_slot, 0) + (uint32_t)(wg * 128);
    const uint32_t lane_base = tmem + ((uint32_t)(wl * 32) << 16);

    // operand orders: K position t holds channel kch; slot t's V code sits at K position vpos
    const int kch = row_index<L>(t), vpos = row_pos<L>(t);
    const int grp_d = wl * 32 / G;  // group of channel t (the same in every lane of the warp: G >= 32)

    const int T = pr.seg.tiles_cap, U = pr.units, NW = pr.workers;
    const long long line = (long long)U * T;
    const int worker = blockIdx.x * 4 + wg;
    const long long x_begin = (line * worker + NW - 1) / NW, x_end = (line * (worker + 1) + NW - 1) / NW;
    const int Hq = pr.H * GQ;

    uint32_t fetched = 0;  // tiles fetched so far by this warpgroup: stage = n & 1, parity = (n >> 1) & 1
    uint32_t ph_qk = 0, ph_pv = 0;
    bool timeout = false;
    int cur_unit = -1;
    // per-head values are kept as pairs of heads (h, h + 1) for the packed FP32 instructions
    constexpr int GP = GQ / 2;
    static_assert(GQ % 2 == 0, "heads per kv head come in pairs");
    float cK = 0.f;
    uint64_t zq[NG][GP];
#pragma unroll
    for (int g2 = 0; g2 < NG; ++g2)
#pragma unroll
        for (int h = 0; h < GP; ++h) zq[g2][h] = 0ull;

    auto fetch = [&](int unit, int tile, uint32_t n) {  // one thread
        const uint32_t stg = n & 1u;
        unsigned char* dst = wsm + stg * C::STAGE;
        const size_t tb = (size_t)unit * T + tile;
        mbar_arrive_expect_tx(&bar[stg], C::STAGE);
        bulk_g2s(dst + C::ST_K, pr.seg.k + tb * P::W * TILE, P::W * 512, &bar[stg]);
        bulk_g2s(dst + C::ST_V, pr.seg.v + tb * P::W * D, P::W * 512, &bar[stg]);
        bulk_g2s(dst + C::ST_KZ, pr.seg.kz + tb * NG * TILE, NG * 512, &bar[stg]);
        bulk_g2s(dst + C::ST_VZ, pr.seg.vz + tb * NG * TILE, NG * 512, &bar[stg]);
    };
    // one row of codes (K words of slot t, or V words of channel t) -> 32 TMEM columns
    auto unpack_to_tmem = [&](uint32_t words_saddr, uint32_t taddr) {
        uint32_t wv[P::W];
#pragma unroll
        for (int j = 0; j < P::W; ++j) wv[j] = lds_u32_after_wait(words_saddr + (uint32_t)(j * 512 + 4 * t));
        uint32_t out[32];
        // each block of 8 registers goes to TMEM as soon as its bytes are complete
        unpack_row_u8<L>(
            wv, [&](uint32_t idx) { return lds_u32(lut_lane + (idx << 7)); }, out,
            [&](int j) {
                if (j == U8BlockDone<L, 0>::value) tmem_st8(taddr, *reinterpret_cast<const uint32_t(*)[8]>(&out[0]));
                if (j == U8BlockDone<L, 1>::value) tmem_st8(taddr + 8, *reinterpret_cast<const uint32_t(*)[8]>(&out[8]));
                if (j == U8BlockDone<L, 2>::value)
                    tmem_st8(taddr + 16, *reinterpret_cast<const uint32_t(*)[8]>(&out[16]));
                if (j == U8BlockDone<L, 3>::value)
                    tmem_st8(taddr + 24, *reinterpret_cast<const uint32_t(*)[8]>(&out[24]));
            });
    };

    for (long long x = x_begin; x < x_end;) {
        const int u = (int)(x / T);
        const int a = (int)(x - (long long)u * T);
        const long long ue = (long long)(u + 1) * T;
        const int b = (int)((x_end < ue ? x_end : ue) - (long long)u * T);  // this chunk: tiles [a, b) of unit u
        x = (long long)u * T + b;

        // the segment's tokens (with the appended one), and where the appended token lands
        int n = pr.seg.n[u];
        int app_tile = -1;
        bool app_hi = false;
        int app_nh = 0, app_nl = 0;
        if constexpr (APP) {
            app_nh = pr.cache.n_hi[u];
            app_nl = pr.cache.n_lo[u];
            app_hi = pr.snew[u] > pr.cache.tau[u];  // NaN compares false: the token goes lo
            if (append_fits(pr.cache, app_hi, app_nh, app_nl) && app_hi == (pr.seg.is_hi != 0)) app_tile = n++ / TILE;
        }
        const int tiles_n = min(ceil_div(n, TILE), T);
        const int e = min(b, tiles_n);  // tiles [a, e) hold tokens
        const int nt = e > a ? e - a : 0;
        // the first two tiles' copies overlap the query set-up, unless the appended token is written
        // into one of them first
        const bool fetch_early = !(APP && app_tile >= a && app_tile < a + 2);
        auto fetch_first = [&] {
            if (t == 0 && nt > 0) {
                fence_async_smem();
                fetch(u, a, fetched);
                if (nt > 1) fetch(u, a + 1, fetched + 1);
            }
        };
        if (fetch_early) fetch_first();

        // ---------------- the unit's queries: B_Q limbs, group sums, fixed-point scale
        if (u != cur_unit) {
            cur_unit = u;
            const int bb = u / pr.H, hk = u % pr.H;
            const uint16_t* qrow = pr.q + ((size_t)bb * Hq + (size_t)hk * GQ) * D;
            float amax = 0.f;
#pragma unroll
            for (int h = 0; h < GQ; ++h) {
                const uint16_t qv = qrow[h * D + t];
                qs[h * D + t] = qv;
                const float f = h2f(qv);
                amax = fmaxf(amax, fabsf(f));
                float sgrp = f;  // channel t's group sum over the warp's 32 channels
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) sgrp += __shfl_xor_sync(0xffffffffu, sgrp, o);
                if (lane == 0) red[wl * 16 + h] = sgrp;
            }
            const uint32_t am = warp_max_u32(__float_as_uint(amax));
            if (lane == 0) red[wl * 16 + 15] = __uint_as_float(am);
            wg_sync();
            amax = fmaxf(fmaxf(red[15], red[16 + 15]), fmaxf(red[32 + 15], red[48 + 15]));
            // 2^F: the largest power of two with amax 2^F < 2^20 (so that the three limb sums of a
            // group combine exactly in 32-bit integers: 128 channels x 15 x 2^20 < 2^31)
            const int F = amax > 0.f ? 19 - exponent_of(amax) : 0;
            cK = pr.scale_log2 * pow2f(-F < -126 ? -126 : -F);
            float qsm[NG][GQ];
#pragma unroll
            for (int g2 = 0; g2 < NG; ++g2)
#pragma unroll
                for (int h = 0; h < GQ; ++h) {
                    float s = 0.f;
#pragma unroll
                    for (int w2 = 0; w2 < G / 32; ++w2) s += red[(g2 * (G / 32) + w2) * 16 + h];
                    qsm[g2][h] = s;
                }
            // B_Q column n = group * 3 GQ + limb * GQ + head; this thread writes K position t
            const int gch = kch / G;
            uint8_t col[NK];
#pragma unroll
            for (int i = 0; i < NK; ++i) col[i] = 0;
            const float scaleF = pow2f(F > 127 ? 127 : F);
#pragma unroll
            for (int h = 0; h < GQ; ++h) {
                const int qi = __float2int_rn(h2f(qs[h * D + kch]) * scaleF);
                const int l0 = (int)(int8_t)(qi & 0xff);
                const int r1 = (qi - l0) >> 8;
                const int l1 = (int)(int8_t)(r1 & 0xff);
                const int l2 = (r1 - l1) >> 8;
#pragma unroll
                for (int g2 = 0; g2 < NG; ++g2) {
                    if (g2 == gch) {
                        col[g2 * 3 * GQ + h] = (uint8_t)l0;
                        col[g2 * 3 * GQ + GQ + h] = (uint8_t)l1;
                        col[g2 * 3 * GQ + 2 * GQ + h] = (uint8_t)l2;
                    }
                }
            }
            unsigned char* bq = wsm + C::W_BQ;
#pragma unroll
            for (int nn = 0; nn < NK; ++nn)
                bq[(nn >> 3) * C::SBO_Q + (t >> 4) * C::LBO_Q + (nn & 7) * 16 + (t & 15)] = col[nn];
            fence_async_smem();
#pragma unroll
            for (int g2 = 0; g2 < NG; ++g2)
#pragma unroll
                for (int h = 0; h < GP; ++h)
                    zq[g2][h] = f2(qsm[g2][2 * h] * pr.scale_log2, qsm[g2][2 * h + 1] * pr.scale_log2);
            wg_sync();  // B_Q complete; red[] free again
        }

        // ---------------- the appended token first, if it lands in this chunk's tiles
        if (APP && app_tile >= a && app_tile < e) {
            const size_t r = (size_t)u * D + t;
            const bool bad = append_row_impl(
                pr.cache, u, app_hi, app_nh, app_nl, h2f(pr.knew[r]), h2f(pr.vnew[r]), t,
                reinterpret_cast<int*>(wsm + C::W_APP), reinterpret_cast<float(*)[4]>(wsm + C::W_APP + 160 * 4),
                reinterpret_cast<float(*)[4]>(wsm + C::W_APP + 168 * 4), [&] { wg_sync(); },
                [&](bool f) { return named_sync_or(bar_id, 128, f); });
            if (bad && t == 0) atomicOr(pr.status, SEMKV_STATUS_NONFINITE_KV);
            // the row's words (plain stores and reductions) before this warpgroup's bulk copies read it
            asm volatile("fence.proxy.async.global;" ::: "memory");
            wg_sync();
        }

        // ---------------- the chunk's tiles
        // running maximum of head h in lane h; every thread keeps the sums of its slot and the
        // output of its channel
        float m_l = NEG_INF;
        uint64_t lsum[GP], O[GP], zacc[NG][GP], pa[GP], pb[GP];
#pragma unroll
        for (int h = 0; h < GP; ++h) {
            lsum[h] = O[h] = 0ull;
            pa[h] = pb[h] = 0ull;
#pragma unroll
            for (int g2 = 0; g2 < NG; ++g2) zacc[g2][h] = 0ull;
        }
        float psa = 0.f;  // 2^-a of channel t's group for the tile whose p.V is in flight
        if (!fetch_early) fetch_first();

        // D_V of the finished p.V -> O (after waiting for it)
        auto take_pv = [&] {
            if (!mbar_wait(&bar[3], ph_pv)) timeout = true;
            ph_pv ^= 1u;
            tc_fence_after();
            uint32_t dv[32];
            tmem_ld_n<4 * GQ>(lane_base + C::COL_DV + (uint32_t)(grp_d * 4 * GQ), dv);
            tc_wait_ld();
            const uint64_t psa2 = f2(psa, psa), c16 = f2(65536.f, 65536.f);
#pragma unroll
            for (int h = 0; h < GP; ++h) {
                const int a0 = (int)dv[8 * h] + ((int)dv[8 * h + 1] << 8);
                const int a1 = (int)dv[8 * h + 4] + ((int)dv[8 * h + 5] << 8);
                const uint64_t v = fma2(f2((float)(int)dv[8 * h + 2], (float)(int)dv[8 * h + 6]), c16,
                                        f2((float)a0, (float)a1));
                O[h] = fma2(mul2(v, psa2), pb[h], mul2(O[h], pa[h]));
            }
        };
        auto wait_stage = [&](uint32_t nfetch) {
            if (!mbar_wait(&bar[nfetch & 1u], (nfetch >> 1) & 1u)) timeout = true;
        };
        auto issue_qk = [&] {  // every thread: after its A_K stores
            tc_wait_st();
            tc_fence_before();
            wg_sync();
            if (t == 0) {
                tc_fence_after();
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_ts_i8(tmem + C::COL_DK, tmem + C::COL_AK + 8 * s,
                              smem_desc(bq_addr + s * 2 * C::LBO_Q, C::LBO_Q, C::SBO_Q), C::IDESC_QK, s > 0);
                mma_commit(&bar[2]);
            }
        };

        if (nt > 0) {
            wait_stage(fetched);
            unpack_to_tmem(smem_u32(wsm + (fetched & 1u) * C::STAGE + C::ST_K), lane_base + C::COL_AK);
            issue_qk();
            for (int i = 0; i < nt; ++i) {
                const uint32_t nf = fetched + (uint32_t)i;
                const unsigned char* sb = wsm + (nf & 1u) * C::STAGE;
                const int tile = a + i;
                if (i > 0) take_pv();  // A_V, B_P and D_V are free again
                unpack_to_tmem(smem_u32(sb + C::ST_V), lane_base + C::COL_AV);
                const bool valid = tile * TILE + t < n;
                float sK[NG], zK[NG], sV[NG], zV[NG];
#pragma unroll
                for (int g2 = 0; g2 < NG; ++g2) {
                    const uint32_t kz = reinterpret_cast<const uint32_t*>(sb + C::ST_KZ)[g2 * 128 + t];
                    const uint32_t vz = reinterpret_cast<const uint32_t*>(sb + C::ST_VZ)[g2 * 128 + t];
                    sK[g2] = h2f((uint16_t)(kz & 0xffffu)) * cK;
                    zK[g2] = h2f((uint16_t)(kz >> 16));
                    sV[g2] = valid ? h2f((uint16_t)(vz & 0xffffu)) : 0.f;
                    zV[g2] = valid ? h2f((uint16_t)(vz >> 16)) : 0.f;
                }
                // ---- logits (log2 domain)
                if (!mbar_wait(&bar[2], ph_qk)) timeout = true;
                ph_qk ^= 1u;
                tc_fence_after();
                uint32_t dk[32];
                tmem_ld_n<NK>(lane_base + C::COL_DK, dk);
                tc_wait_ld();
                float lg[GQ];
#pragma unroll
                for (int h = 0; h < GP; ++h) {
                    uint64_t acc = 0ull;
#pragma unroll
                    for (int g2 = 0; g2 < NG; ++g2) {
                        const int n0 = g2 * 3 * GQ + 2 * h;
                        const int q0 = (int)dk[n0] + ((int)dk[n0 + GQ] << 8) + ((int)dk[n0 + 2 * GQ] << 16);
                        const int q1 = (int)dk[n0 + 1] + ((int)dk[n0 + 1 + GQ] << 8) + ((int)dk[n0 + 1 + 2 * GQ] << 16);
                        acc = fma2(f2(sK[g2], sK[g2]), f2((float)q0, (float)q1),
                                   fma2(f2(zK[g2], zK[g2]), zq[g2][h], acc));
                    }
                    lg[2 * h] = valid ? f2lo(acc) : NEG_INF;
                    lg[2 * h + 1] = valid ? f2hi(acc) : NEG_INF;
                }
                // ---- tile maxima: logits per head, V scales per group
#pragma unroll
                for (int h = 0; h < GQ; ++h) {
                    const float mx = warp_max_redux(lg[h]);
                    if (lane == 0) red[wl * 16 + h] = mx;
                }
#pragma unroll
                for (int g2 = 0; g2 < NG; ++g2) {
                    const uint32_t sm = warp_max_u32(__float_as_uint(sV[g2]));
                    if (lane == 0) red[wl * 16 + 8 + g2] = __uint_as_float(sm);
                }
                wg_sync();
                // one lane per head (lanes 0..GQ-1: tile maximum of the logits) or per group (lanes
                // 8..8+NG-1: tile maximum of the V scales) works out that item's uniform values, then
                // every thread reads them with shuffles
                const int li = lane & 15;
                const float it = fmaxf(fmaxf(red[li], red[16 + li]), fmaxf(red[32 + li], red[48 + li]));
                const float mn = fmaxf(m_l, it);
                const bool live = mn != NEG_INF;  // some slot of the chunk so far is valid
                const float al = live ? ex2_approx(m_l - mn) : 1.f;
                const float pmax = live ? ex2_approx(it - mn) : 0.f;
                int eb = pmax > 0.f ? 10 - exponent_of(pmax) : 0;  // p 2^b < 2^11
                eb = eb > 120 ? 120 : (eb < 0 ? 0 : eb);
                int ea = it > 0.f ? 10 - exponent_of(it) : 0;  // s_V 2^a < 2^11
                ea = ea > 120 ? 120 : (ea < -120 ? -120 : ea);
                if (lane < GQ) m_l = mn;
                const float x0 = lane < 8 ? mn : pow2f(ea), x1 = lane < 8 ? al : pow2f(-ea);
                const float x2 = pow2f(eb), x3 = pow2f(-eb);
                float sVa[NG];
#pragma unroll
                for (int g2 = 0; g2 < NG; ++g2) sVa[g2] = sV[g2] * __shfl_sync(0xffffffffu, x0, 8 + g2);
                psa = __shfl_sync(0xffffffffu, x1, 8 + grp_d);
                // ---- online softmax; P' = p s_V as 22-bit integers
                uint32_t wd[NV / 4];
#pragma unroll
                for (int i2 = 0; i2 < NV / 4; ++i2) wd[i2] = 0u;
                const uint64_t magic = f2(8388608.f, 8388608.f);
#pragma unroll
                for (int h = 0; h < GP; ++h) {
                    const uint64_t mh = f2(__shfl_sync(0xffffffffu, x0, 2 * h), __shfl_sync(0xffffffffu, x0, 2 * h + 1));
                    const uint64_t alh = f2(__shfl_sync(0xffffffffu, x1, 2 * h), __shfl_sync(0xffffffffu, x1, 2 * h + 1));
                    const uint64_t d = sub2(f2(lg[2 * h], lg[2 * h + 1]), mh);
                    const uint64_t p = f2(valid ? ex2_approx(f2lo(d)) : 0.f, valid ? ex2_approx(f2hi(d)) : 0.f);
                    lsum[h] = fma2(lsum[h], alh, p);
#pragma unroll
                    for (int g2 = 0; g2 < NG; ++g2) zacc[g2][h] = fma2(p, f2(zV[g2], zV[g2]), mul2(zacc[g2][h], alh));
                    const uint64_t p2 =
                        mul2(p, f2(__shfl_sync(0xffffffffu, x2, 2 * h), __shfl_sync(0xffffffffu, x2, 2 * h + 1)));
#pragma unroll
                    for (int g2 = 0; g2 < NG; ++g2) {
                        const uint64_t y = fma2(p2, f2(sVa[g2], sVa[g2]), magic);
                        wd[g2 * GQ + 2 * h] = (uint32_t)y & 0x7FFFFFu;
                        wd[g2 * GQ + 2 * h + 1] = (uint32_t)(y >> 32) & 0x7FFFFFu;
                    }
                    pa[h] = alh;
                    pb[h] = f2(__shfl_sync(0xffffffffu, x3, 2 * h), __shfl_sync(0xffffffffu, x3, 2 * h + 1));
                }
                // my slot's row of B_P (K position vpos), 16 bytes per MN core-matrix row
#pragma unroll
                for (int nb = 0; nb < NV / 16; ++nb)
                    sts128(bp_addr + (uint32_t)((vpos >> 3) * C::LBO_P + nb * C::SBO_P + (vpos & 7) * 16),
                           wd[4 * nb], wd[4 * nb + 1], wd[4 * nb + 2], wd[4 * nb + 3]);
                // ---- p.V (q.k is issued by warp 0, p.V and the copies by warp 2)
                tc_wait_st();
                fence_async_smem();
                tc_fence_before();
                wg_sync();
                if (t == 64) {
                    tc_fence_after();
#pragma unroll
                    for (int s = 0; s < 4; ++s)
                        mma_ts_i8(tmem + C::COL_DV, tmem + C::COL_AV + 8 * s,
                                  smem_desc(bp_addr + s * 4 * C::LBO_P, C::LBO_P, C::SBO_P), C::IDESC_PV, s > 0);
                    mma_commit(&bar[3]);
                    // every thread has read this stage (K codes last iteration, V codes and scales
                    // above): refill it two tiles ahead
                    if (i + 2 < nt) fetch(u, tile + 2, nf + 2);
                }
                // ---- next tile's K codes and q.k, overlapping this p.V
                if (i + 1 < nt) {
                    wait_stage(nf + 1);
                    unpack_to_tmem(smem_u32(wsm + ((nf + 1) & 1u) * C::STAGE + C::ST_K), lane_base + C::COL_AK);
                    issue_qk();
                }
            }
            take_pv();
            fetched += (uint32_t)nt;
        }

        // ---------------- the chunk's partial state -> its workspace slot
        float vals[GQ + NG * GQ];
#pragma unroll
        for (int h = 0; h < GQ; ++h) vals[h] = h & 1 ? f2hi(lsum[h >> 1]) : f2lo(lsum[h >> 1]);
#pragma unroll
        for (int g2 = 0; g2 < NG; ++g2)
#pragma unroll
            for (int h = 0; h < GQ; ++h) vals[GQ + g2 * GQ + h] = h & 1 ? f2hi(zacc[g2][h >> 1]) : f2lo(zacc[g2][h >> 1]);
        tc_fence_before();
        wg_sync();  // every thread is past its reads of red[]
#pragma unroll
        for (int i2 = 0; i2 < GQ + NG * GQ; ++i2) {
            float v = vals[i2];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == 0) red[wl * 16 + i2] = v;
        }
        wg_sync();
        const long long first = (long long)u * NW / U;  // the unit's first worker: floor(u T NW / line)
        const long long last = (((long long)u + 1) * T - 1) * NW / line;
        const int slot = worker - (int)first;
        float* rec = pr.ws + ((size_t)u * pr.slots_total + pr.slot_off + slot) * GQ * (D + 2);
#pragma unroll
        for (int h = 0; h < GQ; ++h) {
            const int zi = GQ + grp_d * GQ + h;
            const float zs = red[zi] + red[16 + zi] + red[32 + zi] + red[48 + zi];
            rec[h * (D + 2) + t] = (h & 1 ? f2hi(O[h >> 1]) : f2lo(O[h >> 1])) + zs;
            const float mh = __shfl_sync(0xffffffffu, m_l, h);
            if (t == 0) {
                rec[h * (D + 2) + D] = mh;
                rec[h * (D + 2) + D + 1] = red[h] + red[16 + h] + red[32 + h] + red[48 + h];
            }
        }
        if (worker == (int)last) {
            // the unit's slots that no chunk writes (slots past its last worker, and workers in
            // between whose tile range is empty when there are fewer tiles than workers): empty
            // states
            for (int s = 0; s < pr.slots; ++s) {
                const long long w2 = first + s;
                if (w2 <= last && (line * w2 + NW - 1) / NW < (line * (w2 + 1) + NW - 1) / NW) continue;
                float* r2 = pr.ws + ((size_t)u * pr.slots_total + pr.slot_off + s) * GQ * (D + 2);
#pragma unroll
                for (int h = 0; h < GQ; ++h) {
                    r2[h * (D + 2) + t] = 0.f;
                    if (t == 0) {
                        r2[h * (D + 2) + D] = NEG_INF;
                        r2[h * (D + 2) + D + 1] = 0.f;
                    }
                }
            }
        }
        wg_sync();  // red[] is rewritten by the next chunk
    }

    // ---------------- teardown
    if (timeout) {
        // a wait gave up: wait once more (bounded) for this warpgroup's last copies and products,
        // so that nothing lands in shared or tensor memory after the CTA has let them go
        if (fetched >= 1) mbar_wait(&bar[(fetched - 1) & 1u], ((fetched - 1) >> 1) & 1u);
        if (fetched >= 2) mbar_wait(&bar[(fetched - 2) & 1u], ((fetched - 2) >> 1) & 1u);
        mbar_wait(&bar[2], ph_qk ^ 1u);
        mbar_wait(&bar[3], ph_pv ^ 1u);
    }
    tc_fence_before();
    __syncthreads();
    if (tid < 32) {
        tc_fence_after();
        tmem_dealloc(*tmem_slot, 512);
    }
    if (timeout) atomicOr(pr.status, SEMKV_STATUS_TIMEOUT);
    // the merge reads this launch's and the previous launch's partials: finish only after it
    if (pr.wait_for_prior) asm volatile("griddepcontrol.wait;" ::: "memory");
}

// ------------------------------------------------------------------ host side

template <int L, int GQ, int NG>
static void launch_i8(const I8Params& pr, int ctas, bool dependent, cudaStream_t st)
{
    using C = I8<L, GQ, NG>;
    const auto kern = pr.knew ? k_decode_i8<L, GQ, NG, true> : k_decode_i8<L, GQ, NG, false>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::TOTAL);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)ctas);
    cfg.blockDim = dim3(512);
    cfg.dynamicSmemBytes = C::TOTAL;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = dependent ? 1 : 0;
    cudaLaunchKernelEx(&cfg, kern, pr);
}

// instantiated: L in {4, 5, 6, 8, 16} (K and V on the same level count, per-token K grids) x
// (g, groups) whose accumulators fit a warpgroup's 128 TMEM columns
#define SEMKV_I8_SHAPES(X, L) X(L, 2, 1) X(L, 2, 2) X(L, 4, 1) X(L, 4, 2) X(L, 8, 1)
#define SEMKV_I8_LEVELS(X) SEMKV_I8_SHAPES(X, 4) SEMKV_I8_SHAPES(X, 5) SEMKV_I8_SHAPES(X, 6) \
    SEMKV_I8_SHAPES(X, 8) SEMKV_I8_SHAPES(X, 16)

bool decode_i8_supported(int Lk, int Lv, int G, int g, bool kpc)
{
    if (kpc || Lk != Lv || G <= 0 || 128 % G) return false;
    const int ng = 128 / G;
#define SEMKV_I8_OK(LL, GG, NN) \
    if (Lk == LL && g == GG && ng == NN) return I8<LL, GG, NN>::ok;
    SEMKV_I8_LEVELS(SEMKV_I8_OK)
#undef SEMKV_I8_OK
    return false;
}

void launch_decode_i8(const SegView& seg, const uint16_t* q, int units, int H, int g, int G, float scale_log2,
                      int ctas, int slots, int slot_off, int slots_total, float* ws, int32_t* status, bool dependent,
                      const AppendIn& app, cudaStream_t st)
{
    if (ctas == 0 || units == 0) return;
    I8Params pr = {};
    pr.seg = seg;
    pr.q = q;
    pr.H = H;
    pr.units = units;
    pr.workers = 4 * ctas;
    pr.scale_log2 = scale_log2;
    pr.slots = slots;
    pr.slot_off = slot_off;
    pr.slots_total = slots_total;
    pr.ws = ws;
    pr.status = status;
    pr.wait_for_prior = dependent ? 1 : 0;
    pr.cache = app.cache;
    pr.knew = app.k;
    pr.vnew = app.v;
    pr.snew = app.score;
    const int ng = 128 / G;
#define SEMKV_I8_GO(LL, GG, NN)                                   \
    if (seg.L == LL && g == GG && ng == NN) {                     \
        launch_i8<LL, GG, NN>(pr, ctas, dependent, st);           \
        return;                                                   \
    }
    SEMKV_I8_LEVELS(SEMKV_I8_GO)
#undef SEMKV_I8_GO
}

}  // namespace semkv
