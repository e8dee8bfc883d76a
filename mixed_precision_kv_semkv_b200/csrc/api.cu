// C ABI of libsemkv: argument validation, buffer sizes, split-K choice and kernel launches.
// Every entry point is documented in include/semkv.h.
#include <cmath>
#include <cstdlib>
#include <cstring>

#include "common.cuh"
#include "kernels.cuh"

using namespace semkv;

namespace {

constexpr int D_SUPPORTED = 128;

bool level_ok(int L) { return L >= 2 && L <= 256; }

int validate_shape(const semkv_cache_t* c)
{
    if (!c) return SEMKV_ERR_INVALID_ARG;
    if (c->B < 1 || c->H < 1 || c->Hq < 1 || c->D < 1 || c->G < 1) return SEMKV_ERR_INVALID_ARG;
    if (c->Hq % c->H != 0 || c->D % c->G != 0) return SEMKV_ERR_INVALID_ARG;
    if (c->cap_hi < 0 || c->cap_lo < 0 || c->cap_hi % TILE || c->cap_lo % TILE) return SEMKV_ERR_INVALID_ARG;
    if (c->T_cap < 0 || c->T_cap % 32) return SEMKV_ERR_INVALID_ARG;
    if (c->D != D_SUPPORTED) return SEMKV_ERR_UNSUPPORTED;
    if (!level_ok(c->L_hi) || !level_ok(c->L_lo)) return SEMKV_ERR_UNSUPPORTED;
    if (c->G != 8 && c->G != 16 && c->G != 32 && c->G != 64 && c->G != 128) return SEMKV_ERR_UNSUPPORTED;
    if (c->Hq / c->H > 8) return SEMKV_ERR_UNSUPPORTED;
    if (c->window < 0 || !(c->clip == 0.0f || (c->clip > 0.0f && c->clip <= 1.0f))) return SEMKV_ERR_INVALID_ARG;
    if ((c->L_hi_v && !level_ok(c->L_hi_v)) || (c->L_lo_v && !level_ok(c->L_lo_v))) return SEMKV_ERR_UNSUPPORTED;
    if (c->k_per_channel != 0 && c->k_per_channel != 1) return SEMKV_ERR_INVALID_ARG;
    return SEMKV_OK;
}

int validate_ptrs(const semkv_cache_t* c)
{
    const void* p[] = {c->k_hi, c->v_hi, c->kz_hi, c->vz_hi, c->k_lo, c->v_lo, c->kz_lo, c->vz_lo,
                       c->bitmap, c->rank, c->n_hi, c->n_lo, c->tau, c->status, c->slot_token,
                       c->score_keys, c->kc};
    for (const void* x : p)
        if (!x) return SEMKV_ERR_INVALID_ARG;
    return SEMKV_OK;
}

int validate(const semkv_cache_t* c)
{
    int r = validate_shape(c);
    return r != SEMKV_OK ? r : validate_ptrs(c);
}

int words_row(int L) { return ceil_div(D_SUPPORTED, radix_k(L)); }
int words_col(int L) { return ceil_div(TILE, radix_k(L)); }

int sm_count()
{
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return 148;
    }
    if (dev >= 0 && dev < 64 && cache[dev]) return cache[dev];
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        n = 148;
    }
    if (dev >= 0 && dev < 64) cache[dev] = n;
    return n;
}

// Split-K factor per segment: one wave of four CTAs per SM over the whole decode, shared between
// the segments in proportion to their capacity in tiles (rounded down, so that the two grids
// together never need a second wave), at least one and at most one split per tile.
void decode_splits(const semkv_cache_t* c, int* ns_hi, int* ns_lo)
{
    const int units = c->B * c->H;
    const int th = c->cap_hi / TILE, tl = c->cap_lo / TILE, total = th + tl;
    const long target = 4L * sm_count();
    auto pick = [&](int tiles) -> int {
        if (tiles == 0) return 0;
        long s = (target * tiles) / ((long)units * total);
        if (s < 1) s = 1;
        if (s > tiles) s = tiles;
        return (int)s;
    };
    *ns_hi = pick(th);
    *ns_lo = pick(tl);
}

// How a decode of this shape runs on the current device.  The integer tensor-core decode (when it
// covers both segments): one CTA per SM, the SMs shared by the segments in proportion to their
// work (capacity tiles x a per-tile cost that grows with the words per row: the decode issues
// instructions faster than HBM delivers bytes), at least 8 tiles per CTA, and
// 4 * ctas / units + 2 partial slots per unit and segment (the most workers that can touch one
// unit).  Otherwise the split-K factors of the other decode kernels.
constexpr int I8_MIN_TILES = 8;

// Relative time of one tile of the integer-MMA decode per level count (B200, tiles per SM-second
// measured with all tokens on one grid, 64 units x 32768 tokens, G64): the code table's digits
// per lookup and the words per row set it.  The SMs are split between the two segments' grids in
// proportion to tiles x this cost, so that both grids end together.
double i8_tile_cost(int L)
{
    switch (L) {
    case 4: return 0.70;
    case 6: return 1.10;
    case 8: return 1.02;
    case 16: return 0.70;
    default: return 1.0;
    }
}

// SEMKV_DECODE=i8: the integer-MMA decode wherever it serves the shape; =tc: never it (the fp16-MMA
// or CUDA-core decode); unset or anything else: chosen by the tile count.  Read at every call.
int decode_path_override()
{
    const char* e = std::getenv("SEMKV_DECODE");
    if (!e) return 0;
    if (std::strcmp(e, "i8") == 0) return 1;
    if (std::strcmp(e, "tc") == 0) return 2;
    return 0;
}

struct DecodePlan {
    bool i8;
    int ctas_hi, ctas_lo, slots_hi, slots_lo;  // i8
    int ns_hi, ns_lo;                          // otherwise
    int slots() const { return i8 ? slots_hi + slots_lo : ns_hi + ns_lo; }
};

DecodePlan decode_plan(const semkv_cache_t* c)
{
    DecodePlan p = {};
    const int g = c->Hq / c->H, units = c->B * c->H;
    const bool kpc = c->k_per_channel != 0;
    const int th = c->cap_hi / TILE, tl = c->cap_lo / TILE;
    const bool hi_ok = th == 0 || decode_i8_supported(c->L_hi, level_v(*c, true), c->G, g, kpc);
    const bool lo_ok = tl == 0 || decode_i8_supported(c->L_lo, level_v(*c, false), c->G, g, kpc);
    // Fewer than I8_MIN_TILES tiles per warpgroup of the integer-MMA decode: its fixed cost per
    // warpgroup (query operand, pipeline fill, partial record) outweighs its faster tiles, and the
    // fp16-MMA decode (one warpgroup per CTA, four CTAs per SM) is faster when it serves the shape
    // (measured on B200: 2048 and 4096 tiles favour it, 8192 and more the integer decode).
    const bool tc_ok = (th == 0 || decode_tc_supported(c->L_hi, level_v(*c, true), c->G, g, kpc)) &&
                       (tl == 0 || decode_tc_supported(c->L_lo, level_v(*c, false), c->G, g, kpc));
    const bool few = (long long)units * (th + tl) < (long long)I8_MIN_TILES * 4 * sm_count();
    const int force = decode_path_override();
    const bool use_i8 = force == 1 ? true : (force == 2 ? false : !(few && tc_ok));
    if (hi_ok && lo_ok && th + tl > 0 && use_i8) {
        p.i8 = true;
        const int sms = sm_count();
        const double bh = (double)th * i8_tile_cost(c->L_hi), bl = (double)tl * i8_tile_cost(c->L_lo);
        int ch = 0, cl = 0;
        if (th && tl) {
            ch = (int)std::lround(sms * bh / (bh + bl));
            ch = ch < 1 ? 1 : (ch > sms - 1 ? sms - 1 : ch);
            cl = sms - ch;
        } else {
            ch = th ? sms : 0;
            cl = tl ? sms : 0;
        }
        const long long mh = ((long long)units * th + 7) / 8, ml = ((long long)units * tl + 7) / 8;
        if (ch > mh) ch = (int)mh;
        if (cl > ml) cl = (int)ml;
        p.ctas_hi = ch;
        p.ctas_lo = cl;
        p.slots_hi = ch ? 4 * ch / units + 2 : 0;
        p.slots_lo = cl ? 4 * cl / units + 2 : 0;
    } else {
        decode_splits(c, &p.ns_hi, &p.ns_lo);
    }
    return p;
}

SegView seg_view(const semkv_cache_t* c, bool hi)
{
    SegView s;
    s.k = hi ? c->k_hi : c->k_lo;
    s.v = hi ? c->v_hi : c->v_lo;
    s.kz = hi ? c->kz_hi : c->kz_lo;
    s.vz = hi ? c->vz_hi : c->vz_lo;
    s.n = hi ? c->n_hi : c->n_lo;
    s.L = hi ? c->L_hi : c->L_lo;
    s.Lv = level_v(*c, hi);
    s.tiles_cap = (hi ? c->cap_hi : c->cap_lo) / TILE;
    s.is_hi = hi ? 1 : 0;
    s.kc = c->k_per_channel ? c->kc + (hi ? 0 : 128) : nullptr;
    return s;
}

int launch_status()
{
    return cudaGetLastError() == cudaSuccess ? SEMKV_OK : SEMKV_ERR_CUDA;
}

}  // namespace

namespace {

// host checks of a decode call, before anything is launched
static int decode_args(const semkv_cache_t* c, const uint16_t* q, float softmax_scale, const float* out,
                       const void* workspace, size_t workspace_bytes)
{
    int r = validate(c);
    if (r != SEMKV_OK) return r;
    if (!q || !out || !std::isfinite(softmax_scale)) return SEMKV_ERR_INVALID_ARG;
    if (((uintptr_t)q) & 15u) return SEMKV_ERR_INVALID_ARG;  // query rows are read 16 bytes at a time
    size_t need = 0;
    semkv_workspace_bytes(c, &need);
    if (workspace_bytes < need || (need > 0 && !workspace)) return SEMKV_ERR_INVALID_ARG;
    return SEMKV_OK;
}

// decode, with an appended token first when app.k is set (both segments on the tensor-core kernel)
static int decode_impl(const semkv_cache_t* c, const uint16_t* q, float softmax_scale, float* out, void* workspace,
                       size_t workspace_bytes, const AppendIn& app, cudaStream_t st)
{
    const int r = decode_args(c, q, softmax_scale, out, workspace, workspace_bytes);
    if (r != SEMKV_OK) return r;
    const DecodePlan plan = decode_plan(c);
    const int units = c->B * c->H, g = c->Hq / c->H;
    const float scale_log2 = softmax_scale * 1.4426950408889634f;
    float* ws = static_cast<float*>(workspace);
    if (plan.i8) {
        const SegView hs = seg_view(c, true), ls = seg_view(c, false);
        launch_decode_i8(hs, q, units, c->H, g, c->G, scale_log2, plan.ctas_hi, plan.slots_hi, 0, plan.slots(), ws,
                         c->status, false, app, st);
        launch_decode_i8(ls, q, units, c->H, g, c->G, scale_log2, plan.ctas_lo, plan.slots_lo, plan.slots_hi,
                         plan.slots(), ws, c->status, plan.ctas_hi > 0, app, st);
        launch_decode_merge(ws, units, c->H, g, c->D, plan.slots(), out, app, st);
        return launch_status();
    }
    const int nh = plan.ns_hi, nl = plan.ns_lo;
    bool dependent = false;
    for (int hi = 1; hi >= 0; --hi) {
        const SegView sv = seg_view(c, hi != 0);
        const int ns = hi ? nh : nl, off = hi ? 0 : nh;
        if (ns == 0) continue;
        if (decode_tc_supported(sv.L, sv.Lv, c->G, g, c->k_per_channel != 0)) {
            launch_decode_tc(sv, q, units, c->H, g, c->G, scale_log2, ns, off, nh + nl, ws, c->status, dependent, app,
                             st);
        } else {
            launch_decode_split(sv, q, units, c->H, g, c->D, c->G, scale_log2, ns, off, nh + nl, ws, st);
        }
        dependent = true;
    }
    launch_decode_merge(ws, units, c->H, g, c->D, nh + nl, out, app, st);
    return launch_status();
}

}  // namespace

extern "C" {

int32_t semkv_radix_digits(int32_t L) { return level_ok(L) ? radix_k(L) : 0; }

int semkv_capacities(int32_t T, float p, int32_t window, int32_t extra, int32_t* n_sel, int32_t* cap_hi,
                     int32_t* cap_lo, int32_t* T_cap)
{
    if (T < 0 || window < 0 || extra < 0 || !(p >= 0.0f && p <= 1.0f)) return SEMKV_ERR_INVALID_ARG;
    const long long ns = (long long)std::floor((double)p * (double)T);
    const long long win = window < T ? window : T;
    auto up = [](long long x, long long m) { return (x + m - 1) / m * m; };
    const long long ch = up(ns + win + extra, TILE), cl = up((long long)T - ns + extra, TILE),
                    tc = up((long long)T + extra, 32);
    if (ch > INT32_MAX || cl > INT32_MAX || tc > INT32_MAX) return SEMKV_ERR_INVALID_ARG;
    if (n_sel) *n_sel = (int32_t)ns;
    if (cap_hi) *cap_hi = (int32_t)ch;
    if (cap_lo) *cap_lo = (int32_t)cl;
    if (T_cap) *T_cap = (int32_t)tc;
    return SEMKV_OK;
}

int semkv_p_for_ratio(int32_t D, int32_t G, int32_t L_hi, int32_t L_lo, double ratio, double* p)
{
    return semkv_p_for_ratio_kv(D, G, L_hi, L_lo, L_hi, L_lo, ratio, p);
}

int semkv_p_for_ratio_kv(int32_t D, int32_t G, int32_t L_hi, int32_t L_lo, int32_t L_hi_v, int32_t L_lo_v,
                         double ratio, double* p)
{
    if (!p || !(ratio > 0.0) || !std::isfinite(ratio) || D < 1 || G < 1 || D % G) return SEMKV_ERR_INVALID_ARG;
    if (!level_ok(L_hi) || !level_ok(L_lo) || !level_ok(L_hi_v) || !level_ok(L_lo_v)) return SEMKV_ERR_UNSUPPORTED;
    // bits(p) = a + b p, linear in p; the budget is 16 / ratio bits per value
    auto seg_bits = [&](int Lk, int Lv) {  // K words per row and V words per 128-slot column, averaged
        return 16.0 * ceil_div(D, radix_k(Lk)) / D + 16.0 * ceil_div(TILE, radix_k(Lv)) / TILE;
    };
    const double b_hi = seg_bits(L_hi, L_hi_v), b_lo = seg_bits(L_lo, L_lo_v);
    const double a = b_lo + 32.0 / G + 1.0 / (2.0 * D), b = b_hi - b_lo;
    const double budget = 16.0 / ratio;
    if (a + b <= budget) {  // p = 1 fits (also every b <= 0 case that fits at all)
        *p = 1.0;
        return SEMKV_OK;
    }
    if (b <= 0.0 || a > budget) return SEMKV_ERR_CAPACITY;
    const double x = (budget - a) / b;  // in [0, 1) here
    *p = x < 0.0 ? 0.0 : x;
    return SEMKV_OK;
}

int semkv_cache_bytes(const semkv_cache_t* c, size_t sizes[SEMKV_NBUF])
{
    int r = validate_shape(c);
    if (r != SEMKV_OK) return r;
    if (!sizes) return SEMKV_ERR_INVALID_ARG;
    const size_t units = (size_t)c->B * c->H, ng = (size_t)(c->D / c->G);
    const size_t th = (size_t)c->cap_hi / TILE, tl = (size_t)c->cap_lo / TILE;
    sizes[SEMKV_BUF_K_HI] = units * th * words_row(c->L_hi) * TILE * 4;
    sizes[SEMKV_BUF_V_HI] = units * th * words_col(level_v(*c, true)) * c->D * 4;
    sizes[SEMKV_BUF_KZ_HI] = units * th * ng * TILE * 4;
    sizes[SEMKV_BUF_VZ_HI] = sizes[SEMKV_BUF_KZ_HI];
    sizes[SEMKV_BUF_K_LO] = units * tl * words_row(c->L_lo) * TILE * 4;
    sizes[SEMKV_BUF_V_LO] = units * tl * words_col(level_v(*c, false)) * c->D * 4;
    sizes[SEMKV_BUF_KZ_LO] = units * tl * ng * TILE * 4;
    sizes[SEMKV_BUF_VZ_LO] = sizes[SEMKV_BUF_KZ_LO];
    sizes[SEMKV_BUF_BITMAP] = units * (size_t)(c->T_cap / 32) * 4;
    sizes[SEMKV_BUF_RANK] = sizes[SEMKV_BUF_BITMAP];
    sizes[SEMKV_BUF_N_HI] = units * 4;
    sizes[SEMKV_BUF_N_LO] = units * 4;
    sizes[SEMKV_BUF_TAU] = units * 4;
    sizes[SEMKV_BUF_STATUS] = 4;
    sizes[SEMKV_BUF_SLOT_TOKEN] = units * (size_t)(c->cap_hi + c->cap_lo) * 4;
    sizes[SEMKV_BUF_SCORE_KEYS] = units * (size_t)c->T_cap * 4;
    sizes[SEMKV_BUF_KC] = units * 2 * (size_t)c->D * 4;
    return SEMKV_OK;
}

int semkv_workspace_bytes(const semkv_cache_t* c, size_t* bytes)
{
    int r = validate_shape(c);
    if (r != SEMKV_OK) return r;
    if (!bytes) return SEMKV_ERR_INVALID_ARG;
    *bytes = (size_t)c->B * c->H * (size_t)decode_plan(c).slots() * (c->Hq / c->H) * (c->D + 2) * sizeof(float);
    return SEMKV_OK;
}

int semkv_assign_precision(const semkv_cache_t* c, const float* scores, int32_t T, float p, void* stream)
{
    int r = validate(c);
    if (r != SEMKV_OK) return r;
    if (T < 0 || T > c->T_cap || !(p >= 0.0f && p <= 1.0f) || (!scores && T > 0)) return SEMKV_ERR_INVALID_ARG;
    const int n_sel = (int)std::floor((double)p * (double)T);
    const int win = c->window < T ? c->window : T;  // the recent tokens also put on the L_hi grid
    if (n_sel + win > c->cap_hi || T - n_sel > c->cap_lo) return SEMKV_ERR_CAPACITY;
    launch_select(scores, c->B * c->H, T, n_sel, win, c->T_cap / 32, c->bitmap, c->rank, c->n_hi, c->n_lo, c->tau,
                  c->status, c->slot_token, c->cap_hi, c->cap_lo, c->score_keys, (cudaStream_t)stream);
    return launch_status();
}

int semkv_quantize_pack(const semkv_cache_t* c, const uint16_t* K, const uint16_t* V, int32_t T, void* stream)
{
    int r = validate(c);
    if (r != SEMKV_OK) return r;
    if (T < 0 || T > c->T_cap || ((!K || !V) && T > 0)) return SEMKV_ERR_INVALID_ARG;
    if (T == 0) {  // nothing to place; per-channel K grids of an empty prefill are zero
        if (c->k_per_channel) launch_kc_grids(*c, K, 0, sm_count(), (cudaStream_t)stream);
        return launch_status();
    }
    if ((((uintptr_t)K) | ((uintptr_t)V)) & 15u) return SEMKV_ERR_INVALID_ARG;  // rows are fetched by bulk copies
    if (c->k_per_channel) launch_kc_grids(*c, K, T, sm_count(), (cudaStream_t)stream);  // grids first: the codes use them
    launch_quantize(seg_view(c, true), seg_view(c, false), K, V, c->slot_token, c->B * c->H, T, c->D, c->G,
                    clip_ratio(*c), c->k_per_channel ? c->kc : nullptr, c->status, (cudaStream_t)stream);
    return launch_status();
}

int semkv_append_token(const semkv_cache_t* c, const uint16_t* k, const uint16_t* v, const float* score,
                       void* stream)
{
    int r = validate(c);
    if (r != SEMKV_OK) return r;
    if (!k || !v || !score) return SEMKV_ERR_INVALID_ARG;
    launch_append(*c, k, v, score, -1.0f, (cudaStream_t)stream);
    return launch_status();
}

int semkv_append_token_running(const semkv_cache_t* c, const uint16_t* k, const uint16_t* v, const float* score,
                               float p, void* stream)
{
    int r = validate(c);
    if (r != SEMKV_OK) return r;
    if (!k || !v || !score || !(p >= 0.0f && p <= 1.0f)) return SEMKV_ERR_INVALID_ARG;
    launch_append(*c, k, v, score, p, (cudaStream_t)stream);
    return launch_status();
}


int semkv_decode_attention(const semkv_cache_t* c, const uint16_t* q, float softmax_scale, float* out,
                           void* workspace, size_t workspace_bytes, void* stream)
{
    const AppendIn none = {};
    return decode_impl(c, q, softmax_scale, out, workspace, workspace_bytes, none, (cudaStream_t)stream);
}

int semkv_append_decode(const semkv_cache_t* c, const uint16_t* k, const uint16_t* v, const float* score,
                        const uint16_t* q, float softmax_scale, float* out, void* workspace, size_t workspace_bytes,
                        void* stream)
{
    // every argument is checked before anything is launched, on both paths below
    int r = decode_args(c, q, softmax_scale, out, workspace, workspace_bytes);
    if (r != SEMKV_OK) return r;
    if (!k || !v || !score) return SEMKV_ERR_INVALID_ARG;
    const int g = c->Hq / c->H;
    if (!decode_plan(c).i8 && (!decode_tc_supported(c->L_hi, level_v(*c, true), c->G, g, c->k_per_channel != 0) ||
                               !decode_tc_supported(c->L_lo, level_v(*c, false), c->G, g, c->k_per_channel != 0))) {
        // shapes the fused path does not cover: the two calls, in order
        launch_append(*c, k, v, score, -1.0f, (cudaStream_t)stream);
        r = launch_status();
        if (r != SEMKV_OK) return r;
        return semkv_decode_attention(c, q, softmax_scale, out, workspace, workspace_bytes, stream);
    }
    const AppendIn app = {*c, k, v, score};
    return decode_impl(c, q, softmax_scale, out, workspace, workspace_bytes, app, (cudaStream_t)stream);
}

int semkv_dequantize(const semkv_cache_t* c, float* K, float* V, int32_t T, void* stream)
{
    int r = validate(c);
    if (r != SEMKV_OK) return r;
    if (T < 0 || T > c->T_cap || ((!K || !V) && T > 0)) return SEMKV_ERR_INVALID_ARG;
    if (T == 0) return SEMKV_OK;
    launch_dequantize(*c, T, K, V, (cudaStream_t)stream);
    return launch_status();
}

const char* semkv_status_string(int code)
{
    switch (code) {
        case SEMKV_OK: return "SEMKV_OK";
        case SEMKV_ERR_INVALID_ARG: return "SEMKV_ERR_INVALID_ARG";
        case SEMKV_ERR_UNSUPPORTED: return "SEMKV_ERR_UNSUPPORTED";
        case SEMKV_ERR_CAPACITY: return "SEMKV_ERR_CAPACITY";
        case SEMKV_ERR_CUDA: return "SEMKV_ERR_CUDA";
        default: return "SEMKV_ERR_UNKNOWN";
    }
}

}  // extern "C"
