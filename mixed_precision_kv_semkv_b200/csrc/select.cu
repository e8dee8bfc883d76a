// Precision assignment: per unit, the n_sel largest of T fp32 scores get the L_hi grid (and, in the
// recent-window variant, the last `window` tokens too; n_hi counts both).
//
// SemKV page, Abstract: tokens are ordered by an importance score from inside the model and the
// top fraction is stored at the finer of two neighbouring precisions.  Ties: equal scores are
// taken in increasing token order (-0 and +0 are equal).
//
// The n_hi-th largest key K* is found by a most-significant-
// digit radix select over the order-preserving uint32 image of the scores (4 passes of 8 bits,
// shared-memory histograms).  A final pass forms each
// bitmap word from warp ballots (key > K*, key == K*), takes the first (n_hi - #greater) ties in
// token order with a block-wide exclusive scan, and writes the rank directory with a second scan.
// The window (the SKVQ abstract on the same pages: recent tokens kept at high precision) only ORs
// a suffix of tokens into the words; the selection, its ties and tau do not see it.
#include <cooperative_groups.h>

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

// bits of bitmap word w that hold tokens of the window [win_lo, T)
__device__ __forceinline__ uint32_t window_bits(int w, int T, int win_lo)
{
    const int a = win_lo - 32 * w, b = T - 32 * w;  // the window's bit range [a, b) in this word
    if (b <= 0 || a >= 32 || a >= b) return 0u;
    const uint32_t below_b = b >= 32 ? 0xffffffffu : ((1u << b) - 1u);
    const uint32_t from_a = a <= 0 ? 0xffffffffu : ~((1u << a) - 1u);
    return below_b & from_a;
}

// One CTA of 1024 threads per unit.  CACHED: the keys are first copied into shared memory (T up to
// 48K tokens), otherwise every pass streams them from global memory (L2).
// The slot map of a warp's 32 consecutive bitmap words (lane l holds word w0 + l, its bits and the
// number of L_hi tokens before it): for each word in turn, lane i places token 32 w + i at its slot,
// rank within its class, so each word gives two contiguous runs of stores.  Words at or past
// `w_end` are not this warp's (or hold no token).
__device__ __forceinline__ void emit_slot_tokens(int32_t* __restrict__ st_hi, int32_t* __restrict__ st_lo, int w0,
                                                 int w_end, uint32_t word, uint32_t ones_before, int T)
{
    const int lane = threadIdx.x & 31;
    const uint32_t below = (1u << lane) - 1u;
    for (int j = 0; j < 32; ++j) {
        const int w = w0 + j;
        if (w >= w_end) break;  // uniform over the warp
        const uint32_t bits = __shfl_sync(0xffffffffu, word, j);
        const uint32_t ob = __shfl_sync(0xffffffffu, ones_before, j);
        const int t = 32 * w + lane;
        if (t < T) {
            if ((bits >> lane) & 1u) st_hi[ob + __popc(bits & below)] = t;
            else st_lo[32 * w - (int)ob + __popc(~bits & below)] = t;
        }
    }
}

template <bool CACHED>
__global__ void __launch_bounds__(1024) k_select(const float* __restrict__ scores, int T, int n_hi, int window,
                                                  int words_cap,
                                                  uint32_t* __restrict__ bitmap, uint32_t* __restrict__ rank,
                                                  int32_t* __restrict__ n_hi_out, int32_t* __restrict__ n_lo_out,
                                                  float* __restrict__ tau_out, int32_t* __restrict__ status,
                 int32_t* __restrict__ slot_token, int cap_hi, int cap_lo, uint32_t* __restrict__ score_keys)
{
    const int u = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const float* s = scores + (size_t)u * T;
    uint32_t* bm = bitmap + (size_t)u * words_cap;
    uint32_t* rk = rank + (size_t)u * words_cap;
    int32_t* st_hi = slot_token + (size_t)u * (cap_hi + cap_lo);

    __shared__ uint32_t hist[256];
    __shared__ uint32_t scan_tmp[33];
    __shared__ uint32_t sh_prefix, sh_remaining;
    extern __shared__ uint32_t kcache[];  // [T] when CACHED

    // NaN scores: flag; their keys sort above +inf (order unspecified, as documented)
    {
        bool bad = false;
        uint32_t* sk = score_keys + (size_t)u * 32 * words_cap;
#pragma unroll 8
        for (int t = tid; t < T; t += blockDim.x) {
            const float f = s[t];
            bad |= isnan(f);
            sk[t] = score_key(f);
            if (CACHED) kcache[t] = score_key(f);
        }
        if (__syncthreads_or(bad) && tid == 0) atomicOr(status, SEMKV_STATUS_NAN_SCORE);
    }
    auto key_at = [&](int t) -> uint32_t { return CACHED ? kcache[t] : score_key(s[t]); };

    uint32_t prefix = 0u, mask = 0u, remaining = (uint32_t)n_hi;
    if (n_hi > 0) {
        for (int shift = 24; shift >= 0; shift -= 8) {
            if (tid < 256) hist[tid] = 0u;
            __syncthreads();
#pragma unroll 4
            for (int t0 = 0; t0 < T; t0 += blockDim.x) {  // warp-uniform trip count: match_any needs full warps
                const int t = t0 + tid;
                const uint32_t key = t < T ? key_at(t) : 0u;
                const bool in = t < T && (key & mask) == prefix;
                const uint32_t bin = in ? (key >> shift) & 255u : 256u;
                const uint32_t peers = __match_any_sync(0xffffffffu, bin);
                if (in && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
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
            uint32_t key = t < T ? key_at(t) : 0u;
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
        uint32_t word = my_gt | take_mask | (w < nwords ? window_bits(w, T, T - window) : 0u);
        uint32_t ones_before = carry_ones + block_excl_scan((uint32_t)__popc(word), scan_tmp, &tot);
        carry_ones += tot;
        if (w < nwords) {
            bm[w] = word;
            rk[w] = ones_before;
        }
        emit_slot_tokens(st_hi, st_hi + cap_hi, c + (tid & ~31), nwords, w < nwords ? word : 0u, ones_before, T);
    }
    for (int w = nwords + tid; w < words_cap; w += blockDim.x) {
        bm[w] = 0u;
        rk[w] = carry_ones;
    }
    if (tid == 0) {
        n_hi_out[u] = (int)carry_ones;  // n_hi (selected) plus the window's other tokens
        n_lo_out[u] = T - (int)carry_ones;
        tau_out[u] = n_hi > 0 ? key_score(kstar) : __int_as_float(0x7f800000);
    }
}

// ------------------------------------------------------------------ cluster version
//
// The same selection spread over a cluster of SEL_CS CTAs (512 threads each) per unit.  CTA c owns
// a contiguous range of bitmap words; each thread keeps its KPT keys in registers.
//   * the bits every key shares (cluster-wide AND / OR of the keys) are taken as known: the radix
//     passes start at the highest bit where keys differ, so their digits are spread and plain
//     shared-memory atomics see little contention;
//   * every pass builds per-CTA histograms (two buffers, alternating); after one cluster barrier
//     each CTA sums all SEL_CS histograms through distributed shared memory and finds the same bin,
//     so nothing is broadcast;
//   * the bitmap pass takes the tie and one counts of the earlier CTAs from distributed shared
//     memory for its prefix sums; the four per-CTA counts share one 64-bit block scan.

constexpr int SEL_CS = 8, SEL_THREADS = 512, SEL_WARPS = SEL_THREADS / 32;

// Exclusive scan of 64-bit values over the block (blockDim.x = SEL_THREADS); `tmp` holds 33 words.
__device__ __forceinline__ uint64_t block_excl_scan64(uint64_t v, uint64_t* tmp, uint64_t* total)
{
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    uint64_t inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint64_t n = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += n;
    }
    if (lane == 31) tmp[wid] = inc;
    __syncthreads();
    if (wid == 0) {
        const uint64_t t = lane < SEL_WARPS ? tmp[lane] : 0ull;
        uint64_t ti = t;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint64_t n = __shfl_up_sync(0xffffffffu, ti, o);
            if (lane >= o) ti += n;
        }
        tmp[lane] = ti - t;
        if (lane == 31) tmp[32] = ti;
    }
    __syncthreads();
    const uint64_t r = tmp[wid] + inc - v;
    *total = tmp[32];
    __syncthreads();
    return r;
}

template <int KPT>
__global__ void __cluster_dims__(SEL_CS, 1, 1) __launch_bounds__(SEL_THREADS)
    k_select_cluster(const float* __restrict__ scores, int T, int n_hi, int window, int words_cap,
                     uint32_t* __restrict__ bitmap,
                     uint32_t* __restrict__ rank, int32_t* __restrict__ n_hi_out, int32_t* __restrict__ n_lo_out,
                     float* __restrict__ tau_out, int32_t* __restrict__ status,
                 int32_t* __restrict__ slot_token, int cap_hi, int cap_lo, uint32_t* __restrict__ score_keys)
{
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    const int c = (int)cluster.block_rank();
    const int u = blockIdx.x / SEL_CS;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const float* s = scores + (size_t)u * T;
    const int nwords = (T + 31) / 32;
    const int wpc = (nwords + SEL_CS - 1) / SEL_CS;  // words per CTA
    const int w0 = min(nwords, c * wpc), w1 = min(nwords, w0 + wpc);
    const int tok0 = 32 * w0;

    __shared__ uint32_t hist[2][256], merged[256];
    __shared__ uint32_t gtm[KPT * SEL_WARPS], eqm[KPT * SEL_WARPS];
    __shared__ uint32_t scan_tmp[33];
    __shared__ uint64_t scan_tmp64[33];
    __shared__ uint32_t andor[2];   // this CTA's AND and OR of its keys
    __shared__ __align__(16) uint32_t totals[4];  // ties, strictly-greater, window-and-not-greater, window ties
    __shared__ uint32_t sh_prefix, sh_remaining, red_and[SEL_WARPS], red_or[SEL_WARPS];

    // my keys: tokens tok0 + j*512 + tid (j < KPT) that fall in my CTA's range and below T
    uint32_t key[KPT];
    bool bad = false;
    uint32_t kand = 0xffffffffu, kor = 0u;
    uint32_t* sk = score_keys + (size_t)u * 32 * words_cap;
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
        const int t = tok0 + j * SEL_THREADS + tid;
        const bool in = t < 32 * w1 && t < T;
        const float f = in ? s[t] : 0.f;
        bad |= in && isnan(f);
        key[j] = in ? score_key(f) : 0u;
        if (in) sk[t] = key[j];
        if (in) {
            kand &= key[j];
            kor |= key[j];
        }
    }
    if (__syncthreads_or(bad) && tid == 0) atomicOr(status, SEMKV_STATUS_NAN_SCORE);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        kand &= __shfl_xor_sync(0xffffffffu, kand, o);
        kor |= __shfl_xor_sync(0xffffffffu, kor, o);
    }
    if (lane == 0) {
        red_and[wid] = kand;
        red_or[wid] = kor;
    }
    if (tid < 256) {
        hist[0][tid] = 0u;
        hist[1][tid] = 0u;
    }
    __syncthreads();
    if (tid == 0) {
        uint32_t a = 0xffffffffu, o = 0u;
        for (int i = 0; i < SEL_WARPS; ++i) {
            a &= red_and[i];
            o |= red_or[i];
        }
        andor[0] = a;
        andor[1] = o;
    }
    cluster.sync();
    uint32_t gand = 0xffffffffu, gor = 0u;
    for (int r = 0; r < SEL_CS; ++r) {
        const uint32_t* ro = cluster.map_shared_rank(andor, r);
        gand &= ro[0];
        gor |= ro[1];
    }
    const uint32_t diff = gand ^ gor;  // bits where some keys differ (gand > gor only if T == 0)
    const int top = diff ? 31 - __clz(diff) : -1;

    uint32_t prefix, mask, remaining = (uint32_t)n_hi;
    if (n_hi > 0) {
        mask = top >= 31 ? 0u : (0xffffffffu << (top + 1));
        prefix = gand & mask;  // the shared leading bits
        int pass = 0;
        for (int hi = top; hi >= 0; hi -= 8, ++pass) {
            const int lo = hi >= 7 ? hi - 7 : 0;
            const uint32_t dmask = (2u << (hi - lo)) - 1u;
            uint32_t* hcur = hist[pass & 1];
#pragma unroll
            for (int j = 0; j < KPT; ++j) {
                const int t = tok0 + j * SEL_THREADS + tid;
                if (t < 32 * w1 && t < T && (key[j] & mask) == prefix) atomicAdd(&hcur[(key[j] >> lo) & dmask], 1u);
            }
            cluster.sync();  // this pass's histograms are complete everywhere, and last pass's reads are done
            if (tid < 256) {
                hist[(pass + 1) & 1][tid] = 0u;  // free now: nobody reads it any more
                uint32_t v = 0u;                 // bin tid summed over the cluster (independent remote loads)
#pragma unroll
                for (int r = 0; r < SEL_CS; ++r) v += cluster.map_shared_rank(hcur, r)[tid];
                merged[tid] = v;
            }
            __syncthreads();
            if (wid == 0) {
                uint32_t cnt[8], sum = 0u;
#pragma unroll
                for (int j = 0; j < 8; ++j) cnt[j] = merged[255 - 8 * lane - j];
#pragma unroll
                for (int j = 0; j < 8; ++j) sum += cnt[j];
                const uint32_t inc = warp_incl_scan(sum);
                const uint32_t exc = inc - sum;
                if (exc < remaining && remaining <= inc) {
                    uint32_t cum = exc;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        if (cum + cnt[j] >= remaining) {
                            sh_prefix = prefix | ((uint32_t)(255 - 8 * lane - j) << lo);
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
            mask |= dmask << lo;
        }
    } else {
        prefix = 0xffffffffu;
        remaining = 0u;
    }
    const uint32_t kstar = prefix, take = remaining;

    // ---- word masks of my range (word w0 + j*SEL_WARPS + wid is formed by warp wid at step j)
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
        const int t = tok0 + j * SEL_THREADS + tid;
        const bool in = t < 32 * w1 && t < T;
        const uint32_t gt = __ballot_sync(0xffffffffu, in && key[j] > kstar);
        const uint32_t eq = __ballot_sync(0xffffffffu, in && key[j] == kstar);
        if (lane == 0) {
            gtm[j * SEL_WARPS + wid] = gt;
            eqm[j * SEL_WARPS + wid] = eq;
        }
    }
    __syncthreads();
    const int nw = w1 - w0;  // <= KPT * SEL_WARPS
    uint32_t my_gt = 0u, my_eq = 0u;
    if (tid < nw) {
        my_gt = gtm[tid];
        my_eq = eqm[tid];
    }
    const uint32_t my_win = tid < nw ? window_bits(w0 + tid, T, T - window) : 0u;
    // the four counts of my word as 16-bit fields of one scan (a CTA holds at most
    // KPT * SEL_THREADS <= 16384 tokens)
    const uint64_t packed = (uint64_t)__popc(my_eq) | ((uint64_t)__popc(my_gt) << 16) |
                            ((uint64_t)__popc(my_win & ~my_gt) << 32) | ((uint64_t)__popc(my_win & my_eq) << 48);
    uint64_t tot4;
    const uint64_t before4 = block_excl_scan64(packed, scan_tmp64, &tot4);
    uint32_t ties_before = (uint32_t)(before4 & 0xffffu);
    if (tid == 0) {
        totals[0] = (uint32_t)(tot4 & 0xffffu);
        totals[1] = (uint32_t)((tot4 >> 16) & 0xffffu);
        totals[2] = (uint32_t)((tot4 >> 32) & 0xffffu);
        totals[3] = (uint32_t)(tot4 >> 48);
    }
    cluster.sync();
    // ones (L_hi tokens) of the earlier CTAs, and of all: CTA r holds gt_r greater keys and takes
    // the ties at global tie positions below `take`; the window is a suffix of the tokens, so its
    // ties in CTA r are r's last wt_r ties, and the window adds its tokens that are neither
    // greater nor taken ties.
    // Lane r < SEL_CS of every warp fetches CTA r's four counts (one 16-byte remote load) and the
    // warp combines them with scans over the ranks.
    uint4 tr = make_uint4(0u, 0u, 0u, 0u);
    if (lane < SEL_CS) tr = *reinterpret_cast<const uint4*>(cluster.map_shared_rank(totals, lane));
    uint32_t ties_inc = tr.x;
#pragma unroll
    for (int o = 1; o < SEL_CS; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, ties_inc, o);
        if (lane >= o) ties_inc += v;
    }
    const uint32_t ties_acc = ties_inc - tr.x;  // ties of the CTAs before rank `lane`
    const uint32_t taken = ties_acc >= take ? 0u : min(tr.x, take - ties_acc);
    const uint32_t first_wt = ties_acc + tr.x - tr.w;  // global tie position of rank lane's first window tie
    const uint32_t taken_w = take <= first_wt ? 0u : min(tr.w, take - first_wt);
    const uint32_t ones = lane < SEL_CS ? tr.y + taken + (tr.z - taken_w) : 0u;
    uint32_t ones_inc = ones;
#pragma unroll
    for (int o = 1; o < SEL_CS; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, ones_inc, o);
        if (lane >= o) ones_inc += v;
    }
    const uint32_t cta_ties_before = __shfl_sync(0xffffffffu, ties_acc, c);
    const uint32_t cta_ones_before = __shfl_sync(0xffffffffu, ones_inc - ones, c);
    const uint32_t ones_total = __shfl_sync(0xffffffffu, ones_inc, SEL_CS - 1);
    ties_before += cta_ties_before;
    uint32_t take_mask = 0u;
    if (ties_before < take) {
        const uint32_t need = take - ties_before;
        if (need >= (uint32_t)__popc(my_eq)) {
            take_mask = my_eq;
        } else {
            const uint32_t pos = __fns(my_eq, 0u, (int)need);
            take_mask = my_eq & (0xffffffffu >> (31u - pos));
        }
    }
    const uint32_t word = my_gt | take_mask | my_win;
    uint32_t tot_ones;
    const uint32_t ones_before = cta_ones_before + block_excl_scan((uint32_t)__popc(word), scan_tmp, &tot_ones);
    uint32_t* bm = bitmap + (size_t)u * words_cap;
    uint32_t* rk = rank + (size_t)u * words_cap;
    if (tid < nw) {
        bm[w0 + tid] = word;
        rk[w0 + tid] = ones_before;
    }
    // slot map: every thread places the tokens of its own keys (bitmap words and their counts of
    // L_hi tokens before them staged in shared memory; gtm/eqm are free again)
    if (tid < nw) {
        gtm[tid] = word;
        eqm[tid] = ones_before;
    }
    __syncthreads();
    {
        int32_t* st_hi = slot_token + (size_t)u * (cap_hi + cap_lo);
        int32_t* st_lo = st_hi + cap_hi;
        const uint32_t below = (1u << lane) - 1u;
#pragma unroll
        for (int j = 0; j < KPT; ++j) {
            const int t = tok0 + j * SEL_THREADS + tid;
            if (t < 32 * w1 && t < T) {
                const int wl = j * SEL_WARPS + wid;  // the word of token t, within this CTA
                const uint32_t wd = gtm[wl], ob = eqm[wl];
                if ((wd >> lane) & 1u) st_hi[ob + __popc(wd & below)] = t;
                else st_lo[32 * (w0 + wl) - (int)ob + __popc(~wd & below)] = t;
            }
        }
    }
    for (int w = nwords + c * SEL_THREADS + tid; w < words_cap; w += SEL_CS * SEL_THREADS) {
        bm[w] = 0u;
        rk[w] = ones_total;
    }
    if (c == 0 && tid == 0) {
        n_hi_out[u] = (int)ones_total;
        n_lo_out[u] = T - (int)ones_total;
        tau_out[u] = n_hi > 0 ? key_score(kstar) : __int_as_float(0x7f800000);
    }
    cluster.sync();  // no CTA leaves while another may still read its shared memory
}

// ------------------------------------------------------------------ one CTA, keys in registers
//
// For T <= 32768 one CTA of 1024 threads per unit holds every key in registers (KPT per thread):
// the radix passes re-read nothing and need no cross-CTA exchange.  Thread tid holds tokens
// j*1024 + tid; warp w at step j forms bitmap word j*32 + w.

constexpr int SELR_THREADS = 1024, SELR_WARPS = SELR_THREADS / 32;

template <int KPT>
__global__ void __launch_bounds__(SELR_THREADS)
    k_select_reg(const float* __restrict__ scores, int T, int n_hi, int window, int words_cap,
                 uint32_t* __restrict__ bitmap,
                 uint32_t* __restrict__ rank, int32_t* __restrict__ n_hi_out, int32_t* __restrict__ n_lo_out,
                 float* __restrict__ tau_out, int32_t* __restrict__ status,
                 int32_t* __restrict__ slot_token, int cap_hi, int cap_lo, uint32_t* __restrict__ score_keys)
{
    const int u = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const float* s = scores + (size_t)u * T;
    const int nwords = (T + 31) / 32;
    __shared__ uint32_t hist[256];
    __shared__ uint32_t gtm[KPT * SELR_WARPS], eqm[KPT * SELR_WARPS];
    __shared__ uint32_t scan_tmp[33];
    __shared__ uint32_t sh_prefix, sh_remaining;

    uint32_t key[KPT];
    bool bad = false;
    uint32_t* sk = score_keys + (size_t)u * 32 * words_cap;
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
        const int t = j * SELR_THREADS + tid;
        const float f = t < T ? s[t] : 0.f;
        bad |= t < T && isnan(f);
        key[j] = score_key(f);
        if (t < T) sk[t] = key[j];
    }
    if (__syncthreads_or(bad) && tid == 0) atomicOr(status, SEMKV_STATUS_NAN_SCORE);

    uint32_t prefix = 0u, mask = 0u, remaining = (uint32_t)n_hi;
    if (n_hi > 0) {
        for (int shift = 24; shift >= 0; shift -= 8) {
            if (tid < 256) hist[tid] = 0u;
            __syncthreads();
#pragma unroll
            for (int j = 0; j < KPT; ++j) {
                const bool in = j * SELR_THREADS + tid < T && (key[j] & mask) == prefix;
                const uint32_t bin = in ? (key[j] >> shift) & 255u : 256u;
                const uint32_t peers = __match_any_sync(0xffffffffu, bin);
                if (in && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
            }
            __syncthreads();
            if (wid == 0) {
                uint32_t cnt[8], sum = 0u;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    cnt[j] = hist[255 - 8 * lane - j];
                    sum += cnt[j];
                }
                const uint32_t inc = warp_incl_scan(sum);
                const uint32_t exc = inc - sum;
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
        }
    } else {
        prefix = 0xffffffffu;
        remaining = 0u;
    }
    const uint32_t kstar = prefix, take = remaining;
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
        const bool in = j * SELR_THREADS + tid < T;
        const uint32_t gt = __ballot_sync(0xffffffffu, in && key[j] > kstar);
        const uint32_t eq = __ballot_sync(0xffffffffu, in && key[j] == kstar);
        if (lane == 0) {
            gtm[j * SELR_WARPS + wid] = gt;
            eqm[j * SELR_WARPS + wid] = eq;
        }
    }
    __syncthreads();
    const uint32_t my_gt = tid < nwords ? gtm[tid] : 0u, my_eq = tid < nwords ? eqm[tid] : 0u;
    uint32_t tot;
    const uint32_t ties_before = block_excl_scan((uint32_t)__popc(my_eq), scan_tmp, &tot);
    uint32_t take_mask = 0u;
    if (ties_before < take) {
        const uint32_t need = take - ties_before;
        if (need >= (uint32_t)__popc(my_eq)) {
            take_mask = my_eq;
        } else {
            const uint32_t pos = __fns(my_eq, 0u, (int)need);
            take_mask = my_eq & (0xffffffffu >> (31u - pos));
        }
    }
    const uint32_t word = my_gt | take_mask | (tid < nwords ? window_bits(tid, T, T - window) : 0u);
    const uint32_t ones_before = block_excl_scan((uint32_t)__popc(word), scan_tmp, &tot);  // tot: all ones
    uint32_t* bm = bitmap + (size_t)u * words_cap;
    uint32_t* rk = rank + (size_t)u * words_cap;
    if (tid < nwords) {
        bm[tid] = word;
        rk[tid] = ones_before;
    }
    {
        int32_t* st_hi = slot_token + (size_t)u * (cap_hi + cap_lo);
        emit_slot_tokens(st_hi, st_hi + cap_hi, tid & ~31, nwords, tid < nwords ? word : 0u, ones_before, T);
    }
    for (int w = nwords + tid; w < words_cap; w += SELR_THREADS) {
        bm[w] = 0u;
        rk[w] = tot;
    }
    if (tid == 0) {
        n_hi_out[u] = (int)tot;
        n_lo_out[u] = T - (int)tot;
        tau_out[u] = n_hi > 0 ? key_score(kstar) : __int_as_float(0x7f800000);
    }
}

void launch_select(const float* scores, int units, int T, int n_hi, int window, int words_cap, uint32_t* bitmap,
                   uint32_t* rank, int32_t* n_hi_out, int32_t* n_lo_out, float* tau, int32_t* status,
                   int32_t* slot_token, int cap_hi, int cap_lo, uint32_t* score_keys, cudaStream_t st)
{
    if (T <= SELR_THREADS) {  // one key per thread: a single CTA
        k_select_reg<1><<<units, SELR_THREADS, 0, st>>>(scores, T, n_hi, window, words_cap, bitmap, rank, n_hi_out,
                                                        n_lo_out, tau, status, slot_token, cap_hi, cap_lo, score_keys);
        return;
    }
    const int nwords = (T + 31) / 32;
    const int wpc = (nwords + SEL_CS - 1) / SEL_CS;
    const int kpt = (wpc * 32 + SEL_THREADS - 1) / SEL_THREADS;  // keys per thread in the cluster kernel
    const dim3 grid((unsigned)(units * SEL_CS));
#define SEMKV_SEL(K)                                                                                           \
    if (kpt <= K) {                                                                                            \
        k_select_cluster<K><<<grid, SEL_THREADS, 0, st>>>(scores, T, n_hi, window, words_cap, bitmap, rank, n_hi_out, \
                                                          n_lo_out, tau, status, slot_token, cap_hi, cap_lo, score_keys);                             \
        return;                                                                                                \
    }
    SEMKV_SEL(1) SEMKV_SEL(2) SEMKV_SEL(4) SEMKV_SEL(8) SEMKV_SEL(16) SEMKV_SEL(32)
#undef SEMKV_SEL
    // more keys than a cluster holds in registers: one CTA per unit streams the scores from L2
    k_select<false><<<units, 1024, 0, st>>>(scores, T, n_hi, window, words_cap, bitmap, rank, n_hi_out, n_lo_out, tau,
                                            status, slot_token, cap_hi, cap_lo, score_keys);
}

}  // namespace semkv
