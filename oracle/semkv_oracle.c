/*
 * semkv_oracle.c -- plain, slow CPU oracle for the SemKV mixed-precision KV-cache hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or call this file:
 * only tests/, __graft_entry__.smoke() and bench.py (its cpu_baseline leg and its
 * "--impl reference" arm) use it.  It shares no code, header, table or constant generator
 * with the CUDA library; the two meet only through the seeded input generator.
 *
 * What it computes, and where the method states it
 * ------------------------------------------------
 * The method is the one given in the Abstract of the page "SemKV: Semantic Mixed-Precision KV
 * Cache Quantization Guided by the Quality Cliff for Long-Context LLM Inference" (arXiv
 * 2608.28911v1).  In short: no token is dropped; tokens are ordered by an importance score that
 * the model supplies; the top fraction gets the higher of two neighbouring precisions that both
 * sit above the quality cliff, the rest the lower one; each precision is a uniform affine grid
 * whose level count need not be a power of two (5 levels = 2.322 code bits per value, 4 levels =
 * 2.0 bits).  The Abstract fixes neither the quantizer's rounding, the packing, nor the tie rule;
 * every such choice below is a reading, marked [reading].
 *
 *   select      order the tokens of one (batch, kv-head) unit by score; the n_hi = floor(p*T) with
 *               the largest scores get L_hi levels, the rest L_lo.  [reading: floor; equal scores
 *               are ordered by lower token index first (-0 and +0 are equal); tau = the n_hi-th
 *               largest score (a zero stored as +0), +inf if n_hi = 0.]  Done here with a full
 *               sort -- no selection algorithm.
 *   quantize    per token, per group of G channels: mn = min x, mx = max x;
 *               s = (mx - mn)/(L - 1) in fp32, then rounded UP to fp16 [reading: rounding up keeps
 *               the grid z + c*s, c = 0..L-1, over [mn, mx]; saturates at 65504];  z = mn (exact
 *               in fp16); c = clamp(rint((x - z)/s), 0, L - 1) with fp32 subtract and divide and
 *               round-half-even, c = 0 when s = 0.
 *   pack        base-L radix words: k(L) = max{k : L^k <= 2^32} codes per uint32 word,
 *               word = sum_i c_i * L^i, lowest index in the least significant digit.
 *               K codes are packed along the channel axis of a token row (the axis q.k sums
 *               over); V codes are packed along the token axis of one channel inside a 128-slot
 *               tile (the axis p.V sums over).  [reading: the Abstract fixes no packing axis.]
 *   place       a token goes to the hi or lo segment of its unit, at slot = number of earlier
 *               tokens of the same class; every token is kept, so n_hi + n_lo = T.
 *   append      a token produced during generation (the Abstract reports the cliff for
 *               quantization at generation time too) is hi iff its score > tau of its unit
 *               (strict) [reading]; it is quantized alone and placed at the next slot.
 *   dequantize  x^ = fmaf((float)c, s, z).
 *   variants    three quantizer variants of prior art that the pages summarise (the SKVQ abstract):
 *               a clip ratio that shrinks each group's range before the grid is fitted; a window
 *               of the most recent tokens forced onto the finer grid at selection; and level
 *               counts of their own for V (keys and values at different bit widths): each segment
 *               has a K level count and a V level count, and each tensor's codes, scale and radix
 *               words use its own; and per-channel K grouping (the KVQuant blog page: keys quantized
 *               per channel): each channel of a unit's K gets one grid, fitted over all prefill
 *               tokens, and every token of the unit (appended ones too) is coded on it.  All are off
 *               by default; the formulas are readings, given at oracle_quantize_group_clip,
 *               oracle_select and oracle_k_channel_grid.
 *   attention   fp64: o = sum_t softmax_t(sigma * q.k^_t) v^_t over all tokens of the unit, for
 *               each of the g query heads that share the kv head (GQA); no mask.
 *
 * Physical layout (shared with nothing: it is written out here from the layout's definition so
 * that buffers compare byte for byte):
 *   tile          = 128 slots of one segment
 *   K words       [tile][j < WK][slot in tile]        WK = ceil(D / k)
 *   V words       [tile][w < WV][channel d]           WV = ceil(128 / k)
 *   scale/zero    [tile][group][slot in tile]         uint32 = fp16 scale | fp16 zero << 16
 *   bitmap        bit t of word t/32 (LSB first) = 1 iff token t is in the hi segment
 *   rank          rank[w] = number of 1 bits in bitmap words 0..w-1
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_TILE 128

/* status bits, same meaning as the device status word of the library (defined independently) */
#define OR_NAN_SCORE 1
#define OR_NONFINITE_KV 2
#define OR_OVERFLOW 4
#define OR_BAD_ARG 256

/* ------------------------------------------------------------------ radix parameters */

/* k(L): the largest k with L^k <= 2^32, found by counting. */
int oracle_radix_digits(int L)
{
    uint64_t p = 1;
    int k = 0;
    while (p * (uint64_t)L <= 4294967296ull) {
        p *= (uint64_t)L;
        k++;
    }
    return k;
}

static int ceil_div(int a, int b) { return (a + b - 1) / b; }

int oracle_words_per_row(int L, int D) { return ceil_div(D, oracle_radix_digits(L)); }
int oracle_words_per_tile_column(int L) { return ceil_div(OR_TILE, oracle_radix_digits(L)); }

/* ------------------------------------------------------------------ IEEE binary16 */

/* binary16 -> binary32, exact: sign, 5-bit biased exponent, 10-bit fraction. */
float oracle_half_to_float(uint16_t h)
{
    int sign = h >> 15, e = (h >> 10) & 31, m = h & 1023;
    float v;
    if (e == 0)
        v = ldexpf((float)m, -24); /* subnormal: m * 2^-24 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexpf((float)(m + 1024), e - 25); /* (1 + m/1024) * 2^(e-15) */
    return sign ? -v : v;
}

/* encode a magnitude v that is exactly representable in binary16 (0 <= v <= 65504) */
static uint16_t encode_half(int neg, double v)
{
    uint16_t s = neg ? 0x8000 : 0;
    if (v == 0.0) return s;
    int e;
    frexp(v, &e); /* v in [2^(e-1), 2^e) */
    int E = e - 1;
    if (E < -14) return (uint16_t)(s | (uint16_t)ldexp(v, 24)); /* subnormal */
    uint32_t frac = (uint32_t)ldexp(v, 10 - E) - 1024u;
    return (uint16_t)(s | (uint16_t)((E + 15) << 10) | (uint16_t)frac);
}

/* binary32 -> binary16 rounded toward +infinity (the smallest binary16 >= f). */
uint16_t oracle_float_to_half_up(float f)
{
    if (isnan(f)) return 0x7E00;
    if (f == 0.0f) return signbit(f) ? 0x8000 : 0x0000;
    int neg = f < 0.0f;
    double a = fabs((double)f);
    if (a > 65504.0) return neg ? 0xFBFF : 0x7C00; /* RU: -65504 below, +inf above */
    int e;
    frexp(a, &e);
    int E = e - 1; /* a in [2^E, 2^(E+1)) */
    if (E < -14) E = -14; /* subnormal spacing 2^-24 */
    double ulp = ldexp(1.0, E - 10);
    double n = a / ulp; /* exact: scaling by a power of two */
    double k = neg ? floor(n) : ceil(n); /* toward +inf: up in magnitude if positive */
    return encode_half(neg, k * ulp);
}

/* binary32 -> binary16 rounded to nearest, ties to the even significand (IEEE 754 default
 * rounding).  Only finite |f| <= 65504 is asked of it here (the clipped zero); larger magnitudes
 * give infinity, NaN gives the quiet NaN. */
uint16_t oracle_float_to_half_rn(float f)
{
    if (isnan(f)) return 0x7E00;
    if (f == 0.0f) return signbit(f) ? 0x8000 : 0x0000;
    int neg = f < 0.0f;
    double a = fabs((double)f);
    if (a >= 65520.0) return neg ? 0xFC00 : 0x7C00; /* halfway to 2^16 and beyond: infinity */
    int e;
    frexp(a, &e);
    int E = e - 1; /* a in [2^E, 2^(E+1)) */
    if (E < -14) E = -14;
    double ulp = ldexp(1.0, E - 10);
    double n = a / ulp; /* exact */
    double k = floor(n);
    double rem = n - k;
    if (rem > 0.5 || (rem == 0.5 && fmod(k, 2.0) != 0.0)) k += 1.0; /* nearest; a tie goes to even */
    return encode_half(neg, k * ulp);
}

/* the fp16 scale of a group: rounded up, saturated at the largest finite binary16 [reading] */
uint16_t oracle_scale_half(float sf)
{
    if (sf > 65504.0f) return 0x7BFF;
    return oracle_float_to_half_up(sf);
}

/* ------------------------------------------------------------------ select */

typedef struct {
    float s;
    int32_t t;
} scored_t;

static int cmp_desc(const void* a, const void* b)
{
    const scored_t* x = (const scored_t*)a;
    const scored_t* y = (const scored_t*)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->t < y->t) ? -1 : (x->t > y->t); /* equal scores: lower token index first */
}

/* n_hi for a fraction p of T tokens [reading: floor of p*T in double]. */
int32_t oracle_n_hi(float p, int32_t T) { return (int32_t)floor((double)p * (double)T); }

/*
 * Order the T scores of one unit and assign the two precisions (SemKV page, Abstract: tokens
 * are ordered by a model-internal score and split between two neighbouring precisions).
 * Writes bitmap[0..ceil(T/32)) and rank[0..ceil(T/32)).  Returns status bits.
 *
 * window (prior-art variant, the SKVQ abstract on the same pages: the most recent tokens are
 * kept at high precision) [reading]: after the selection by score, the last min(window, T)
 * tokens are put on the finer grid too; n_hi is then the number of tokens on it.  tau stays the
 * score threshold of the selection by score.  window = 0 is the plain method.
 */
int oracle_select(const float* score, int32_t T, float p, int32_t window, uint32_t* bitmap, uint32_t* rank,
                  int32_t* n_hi_out, float* tau_out)
{
    if (T < 0 || !(p >= 0.0f && p <= 1.0f) || window < 0) return OR_BAD_ARG;
    int status = 0;
    int32_t nw = (T + 31) / 32;
    scored_t* v = (scored_t*)malloc(sizeof(scored_t) * (size_t)(T > 0 ? T : 1));
    for (int32_t t = 0; t < T; t++) {
        if (isnan(score[t])) status |= OR_NAN_SCORE;
        v[t].s = score[t];
        v[t].t = t;
    }
    qsort(v, (size_t)T, sizeof(scored_t), cmp_desc);
    int32_t n_hi = oracle_n_hi(p, T);
    memset(bitmap, 0, sizeof(uint32_t) * (size_t)nw);
    for (int32_t i = 0; i < n_hi; i++) bitmap[v[i].t / 32] |= 1u << (v[i].t % 32);
    for (int32_t t = (window < T ? T - window : 0); t < T; t++) bitmap[t / 32] |= 1u << (t % 32);
    uint32_t acc = 0;
    for (int32_t w = 0; w < nw; w++) {
        rank[w] = acc;
        uint32_t x = bitmap[w];
        while (x) { /* popcount by clearing the lowest set bit */
            x &= x - 1;
            acc++;
        }
    }
    *n_hi_out = (int32_t)acc; /* = n_hi when window = 0 */
    /* -0 and +0 are the same score; the threshold is stored as +0 */
    *tau_out = n_hi > 0 ? v[n_hi - 1].s + 0.0f : INFINITY;
    free(v);
    return status;
}

/* ------------------------------------------------------------------ quantize and pack */

/* code of one fp16 value on the grid (s16, z16) with L levels: clamp(rint((x - z)/s), 0, L - 1) in
 * binary32 (RN subtract and divide, ties to even); 0 when s = 0 */
int oracle_code_on_grid(uint16_t x, uint16_t s16, uint16_t z16, int L)
{
    float v = oracle_half_to_float(x), s = oracle_half_to_float(s16), z = oracle_half_to_float(z16);
    if (s == 0.0f) return 0;
    float q = (v - z) / s;
    float r = rintf(q); /* round half to even in the default rounding mode */
    if (!(r >= 0.0f)) r = 0.0f;
    if (r > (float)(L - 1)) r = (float)(L - 1);
    return (int)r;
}

/*
 * Affine quantization of one group of G fp16 values to L levels (SemKV page, Abstract: a uniform
 * affine grid whose level count need not be a power of two).  Writes G codes, the fp16 scale and
 * the fp16 zero.
 *
 * clip (prior-art variant, the SKVQ abstract on the same pages: clipped dynamic quantization of
 * each group): clip = 1 is the plain grid over [mn, mx].  For 0 < clip < 1 [reading -- the pages
 * give neither the formula nor a value]: the extrema are first scaled by clip in fp32
 * (mn' = clip*mn, mx' = clip*mx); z = the binary16 nearest to mn' (ties to even, -0 stored as
 * +0); s = fp16 rounded up of (mx' - z)/(L - 1), taken as 0 if that is negative; values outside
 * the clipped range get the end codes through the clamp below.
 */
int oracle_quantize_group_clip(const uint16_t* x, int G, int L, float clip, uint8_t* code, uint16_t* scale_out,
                               uint16_t* zero_out)
{
    int status = 0;
    float mn = INFINITY, mx = -INFINITY;
    for (int i = 0; i < G; i++) {
        float v = oracle_half_to_float(x[i]);
        if (!isfinite(v)) status |= OR_NONFINITE_KV;
        if (v < mn) mn = v;
        if (v > mx) mx = v;
    }
    uint16_t s16, z16;
    if (clip == 1.0f) {
        float sf = (mx - mn) / (float)(L - 1);
        s16 = oracle_scale_half(sf);
        float z0 = mn + 0.0f;                   /* -0 becomes +0: one zero for both signs */
        z16 = oracle_float_to_half_up(z0);      /* exact: mn is a binary16 value */
    } else {
        float mnc = clip * mn, mxc = clip * mx; /* one fp32 multiply each */
        z16 = oracle_float_to_half_rn(mnc);
        if (z16 == 0x8000) z16 = 0x0000;        /* -0 becomes +0 */
        float sf = (mxc - oracle_half_to_float(z16)) / (float)(L - 1);
        if (sf < 0.0f) sf = 0.0f;               /* mn == mx and z rounded above clip*mx */
        s16 = oracle_scale_half(sf);
    }
    float s = oracle_half_to_float(s16);
    float z = oracle_half_to_float(z16);
    for (int i = 0; i < G; i++) code[i] = (uint8_t)oracle_code_on_grid(x[i], s16, z16, L);
    (void)s;
    (void)z;
    *scale_out = s16;
    *zero_out = z16;
    return status;
}

int oracle_quantize_group(const uint16_t* x, int G, int L, uint8_t* code, uint16_t* scale_out,
                          uint16_t* zero_out)
{
    return oracle_quantize_group_clip(x, G, L, 1.0f, code, scale_out, zero_out);
}

/*
 * Per-channel K grids of one unit (prior-art variant; the KVQuant blog page on the same pages names
 * per-channel key quantization) [reading]: channel d's T prefill values form one group, fitted as
 * in oracle_quantize_group_clip (same clip) once with L_hi and once with L_lo levels.
 * kc[d] = hi grid, kc[D + d] = lo grid, each fp16 scale | fp16 zero << 16.  Tokens appended later
 * are coded on the same grids (clamped), since the pages give no rule for refitting them.
 */
int oracle_k_channel_grid(const uint16_t* K, int32_t T, int D, int L_hi, int L_lo, float clip, uint32_t* kc)
{
    int status = 0;
    uint16_t* col = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)(T > 0 ? T : 1));
    uint8_t* codes = (uint8_t*)malloc((size_t)(T > 0 ? T : 1));
    for (int d = 0; d < D; d++) {
        for (int32_t t = 0; t < T; t++) col[t] = K[(size_t)t * D + d];
        uint16_t s16 = 0, z16 = 0;
        if (T > 0) status |= oracle_quantize_group_clip(col, T, L_hi, clip, codes, &s16, &z16);
        kc[d] = (uint32_t)s16 | ((uint32_t)z16 << 16);
        if (T > 0) status |= oracle_quantize_group_clip(col, T, L_lo, clip, codes, &s16, &z16);
        kc[D + d] = (uint32_t)s16 | ((uint32_t)z16 << 16);
    }
    free(col);
    free(codes);
    return status;
}

/* word = sum_i c_i L^i over k codes (base-L positional notation, lowest index least significant) */
uint32_t oracle_pack_word(const uint8_t* c, int k, int L)
{
    uint64_t w = 0, pw = 1;
    for (int i = 0; i < k; i++) {
        w += (uint64_t)c[i] * pw;
        pw *= (uint64_t)L;
    }
    return (uint32_t)w;
}

void oracle_unpack_word(uint32_t w, int k, int L, uint8_t* c)
{
    for (int i = 0; i < k; i++) {
        c[i] = (uint8_t)(w % (uint32_t)L);
        w /= (uint32_t)L;
    }
}

static size_t k_word_index(int tile, int j, int t, int WK)
{
    return ((size_t)tile * WK + j) * OR_TILE + t;
}
static size_t v_word_index(int tile, int w, int d, int WV, int D)
{
    return ((size_t)tile * WV + w) * D + d;
}
static size_t sz_index(int tile, int grp, int t, int NG)
{
    return ((size_t)tile * NG + grp) * OR_TILE + t;
}

/* Pack one segment from its per-slot codes (zero codes past n_seg) into the tile layout: K words
 * in base Lk, V words in base Lv. */
static void pack_segment(const uint8_t* ck, const uint8_t* cv, int tiles, int D, int Lk, int Lv, uint32_t* kw,
                         uint32_t* vw)
{
    int kk = oracle_radix_digits(Lk), kv = oracle_radix_digits(Lv);
    int WK = ceil_div(D, kk), WV = ceil_div(OR_TILE, kv);
    uint8_t* buf = (uint8_t*)malloc((size_t)(kk > kv ? kk : kv));
    for (int tile = 0; tile < tiles; tile++) {
        for (int t = 0; t < OR_TILE; t++) {
            const uint8_t* row = ck + ((size_t)tile * OR_TILE + t) * D;
            for (int j = 0; j < WK; j++) {
                for (int i = 0; i < kk; i++) buf[i] = (j * kk + i < D) ? row[j * kk + i] : 0;
                kw[k_word_index(tile, j, t, WK)] = oracle_pack_word(buf, kk, Lk);
            }
        }
        for (int d = 0; d < D; d++) {
            for (int w = 0; w < WV; w++) {
                for (int i = 0; i < kv; i++) {
                    int slot = w * kv + i;
                    buf[i] = slot < OR_TILE ? cv[((size_t)tile * OR_TILE + slot) * D + d] : 0;
                }
                vw[v_word_index(tile, w, d, WV, D)] = oracle_pack_word(buf, kv, Lv);
            }
        }
    }
    free(buf);
}

/*
 * Quantize and place every token of one unit.  K, V: [T][D] fp16 bits.  bitmap from select.
 * Segment buffers must hold tiles_hi (tiles_lo) tiles; slots past n_seg are written as zeros.
 */
int oracle_quantize_pack_unit(const uint16_t* K, const uint16_t* V, int32_t T, int D, int G, int L_hi,
                              int L_lo, int L_hi_v, int L_lo_v, float clip, const uint32_t* bitmap, int tiles_hi,
                              int tiles_lo,
                              uint32_t* k_hi, uint32_t* v_hi, uint32_t* kz_hi, uint32_t* vz_hi,
                              uint32_t* k_lo, uint32_t* v_lo, uint32_t* kz_lo, uint32_t* vz_lo, const uint32_t* kc)
{
    /* kc: per-channel K grids (oracle_k_channel_grid), or NULL for per-token K groups */
    if (D <= 0 || G <= 0 || D % G != 0 || L_hi < 2 || L_lo < 2 || L_hi > 256 || L_lo > 256 ||
        L_hi_v < 2 || L_lo_v < 2 || L_hi_v > 256 || L_lo_v > 256 || !(clip > 0.0f && clip <= 1.0f))
        return OR_BAD_ARG;
    int status = 0, NG = D / G;
    int tiles[2] = {tiles_hi, tiles_lo};
    int Ls[2] = {L_hi, L_lo};
    int Lvs[2] = {L_hi_v, L_lo_v};
    uint32_t* kw[2] = {k_hi, k_lo};
    uint32_t* vw[2] = {v_hi, v_lo};
    uint32_t* kz[2] = {kz_hi, kz_lo};
    uint32_t* vz[2] = {vz_hi, vz_lo};
    uint8_t* ck[2];
    uint8_t* cv[2];
    for (int s = 0; s < 2; s++) {
        size_t slots = (size_t)tiles[s] * OR_TILE;
        ck[s] = (uint8_t*)calloc(slots * D + 1, 1);
        cv[s] = (uint8_t*)calloc(slots * D + 1, 1);
        memset(kz[s], 0, sizeof(uint32_t) * slots * NG);
        memset(vz[s], 0, sizeof(uint32_t) * slots * NG);
    }
    int32_t next[2] = {0, 0};
    for (int32_t t = 0; t < T; t++) {
        int seg = ((bitmap[t / 32] >> (t % 32)) & 1u) ? 0 : 1;
        int32_t slot = next[seg]++;
        if (slot >= tiles[seg] * OR_TILE) {
            status |= OR_OVERFLOW;
            continue;
        }
        int tile = slot / OR_TILE, tt = slot % OR_TILE;
        for (int grp = 0; grp < NG; grp++) {
            uint16_t s16, z16;
            if (kc) { /* K on its channels' grids; the per-token K scale/zero stay 0 */
                for (int d = grp * G; d < (grp + 1) * G; d++) {
                    uint32_t g = kc[(size_t)seg * D + d];
                    uint16_t x = K[(size_t)t * D + d];
                    if (!isfinite(oracle_half_to_float(x))) status |= OR_NONFINITE_KV;
                    ck[seg][(size_t)slot * D + d] =
                        (uint8_t)oracle_code_on_grid(x, (uint16_t)(g & 0xFFFF), (uint16_t)(g >> 16), Ls[seg]);
                }
                kz[seg][sz_index(tile, grp, tt, NG)] = 0;
            } else {
                status |= oracle_quantize_group_clip(K + (size_t)t * D + grp * G, G, Ls[seg], clip,
                                                     ck[seg] + (size_t)slot * D + grp * G, &s16, &z16);
                kz[seg][sz_index(tile, grp, tt, NG)] = (uint32_t)s16 | ((uint32_t)z16 << 16);
            }
            status |= oracle_quantize_group_clip(V + (size_t)t * D + grp * G, G, Lvs[seg], clip,
                                                 cv[seg] + (size_t)slot * D + grp * G, &s16, &z16);
            vz[seg][sz_index(tile, grp, tt, NG)] = (uint32_t)s16 | ((uint32_t)z16 << 16);
        }
    }
    for (int s = 0; s < 2; s++) {
        pack_segment(ck[s], cv[s], tiles[s], D, Ls[s], Lvs[s], kw[s], vw[s]);
        free(ck[s]);
        free(cv[s]);
    }
    return status;
}

/* ------------------------------------------------------------------ dequantize */

/* code of (slot, channel d) of a segment, read back from its packed words */
static void segment_codes(const uint32_t* kw, const uint32_t* vw, int D, int Lk, int Lv, int32_t slot, uint8_t* kc,
                          uint8_t* vc)
{
    int kk = oracle_radix_digits(Lk), kv = oracle_radix_digits(Lv);
    int WK = ceil_div(D, kk), WV = ceil_div(OR_TILE, kv);
    int tile = slot / OR_TILE, tt = slot % OR_TILE;
    uint8_t* buf = (uint8_t*)malloc((size_t)(kk > kv ? kk : kv));
    for (int j = 0; j < WK; j++) {
        oracle_unpack_word(kw[k_word_index(tile, j, tt, WK)], kk, Lk, buf);
        for (int i = 0; i < kk && j * kk + i < D; i++) kc[j * kk + i] = buf[i];
    }
    for (int d = 0; d < D; d++) {
        oracle_unpack_word(vw[v_word_index(tile, tt / kv, d, WV, D)], kv, Lv, buf);
        vc[d] = buf[tt % kv];
    }
    free(buf);
}

/* x^ = fmaf(c, s, z) for every token of a unit, in original token order.  Khat, Vhat: [T][D]. */
void oracle_dequantize_unit(int32_t T, int D, int G, int L_hi, int L_lo, int L_hi_v, int L_lo_v,
                            const uint32_t* bitmap,
                            const uint32_t* k_hi, const uint32_t* v_hi, const uint32_t* kz_hi,
                            const uint32_t* vz_hi, const uint32_t* k_lo, const uint32_t* v_lo,
                            const uint32_t* kz_lo, const uint32_t* vz_lo, float* Khat, float* Vhat,
                            const uint32_t* kgrid)
{
    int NG = D / G;
    const uint32_t* kw[2] = {k_hi, k_lo};
    const uint32_t* vw[2] = {v_hi, v_lo};
    const uint32_t* kz[2] = {kz_hi, kz_lo};
    const uint32_t* vz[2] = {vz_hi, vz_lo};
    int Ls[2] = {L_hi, L_lo};
    int Lvs[2] = {L_hi_v, L_lo_v};
    uint8_t* kc = (uint8_t*)malloc((size_t)D);
    uint8_t* vc = (uint8_t*)malloc((size_t)D);
    int32_t next[2] = {0, 0};
    for (int32_t t = 0; t < T; t++) {
        int seg = ((bitmap[t / 32] >> (t % 32)) & 1u) ? 0 : 1;
        int32_t slot = next[seg]++;
        int tile = slot / OR_TILE, tt = slot % OR_TILE;
        segment_codes(kw[seg], vw[seg], D, Ls[seg], Lvs[seg], slot, kc, vc);
        for (int d = 0; d < D; d++) {
            int grp = d / G;
            uint32_t kzv = kgrid ? kgrid[(size_t)seg * D + d] : kz[seg][sz_index(tile, grp, tt, NG)];
            uint32_t vzv = vz[seg][sz_index(tile, grp, tt, NG)];
            float ks = oracle_half_to_float((uint16_t)(kzv & 0xFFFF));
            float kz0 = oracle_half_to_float((uint16_t)(kzv >> 16));
            float vs = oracle_half_to_float((uint16_t)(vzv & 0xFFFF));
            float vz0 = oracle_half_to_float((uint16_t)(vzv >> 16));
            Khat[(size_t)t * D + d] = fmaf((float)kc[d], ks, kz0);
            Vhat[(size_t)t * D + d] = fmaf((float)vc[d], vs, vz0);
        }
    }
    free(kc);
    free(vc);
}

/* ------------------------------------------------------------------ append */

/*
 * Quantization at generation time of one new token of one unit (SemKV page, Abstract: the same
 * cliff is reported when tokens are quantized as they are generated).  hi iff score > tau
 * [reading].  The token is quantized alone (with the prefill's clip) and written at the next
 * slot of its segment; older tokens are untouched.
 * State (bitmap, rank, n_hi, n_lo) is updated in place.  Returns status bits.
 */
int oracle_append_unit(const uint16_t* k, const uint16_t* v, float score, float tau, int D, int G,
                       int L_hi, int L_lo, int L_hi_v, int L_lo_v, float clip, int32_t T_cap, uint32_t* bitmap, uint32_t* rank,
                       int32_t* n_hi, int32_t* n_lo, int tiles_hi, int tiles_lo, uint32_t* k_hi,
                       uint32_t* v_hi, uint32_t* kz_hi, uint32_t* vz_hi, uint32_t* k_lo,
                       uint32_t* v_lo, uint32_t* kz_lo, uint32_t* vz_lo,
                       const uint32_t* kgrid)
{
    int status = 0;
    if (isnan(score)) status |= OR_NAN_SCORE;
    int hi = score > tau;
    int seg = hi ? 0 : 1;
    int32_t T = *n_hi + *n_lo;
    int32_t slot = hi ? *n_hi : *n_lo;
    int tiles = hi ? tiles_hi : tiles_lo;
    if (slot >= tiles * OR_TILE || T >= T_cap) return status | OR_OVERFLOW;
    int L = hi ? L_hi : L_lo, Lv = hi ? L_hi_v : L_lo_v;
    int NG = D / G;
    int kdig = oracle_radix_digits(L), vdig = oracle_radix_digits(Lv);
    int WK = ceil_div(D, kdig), WV = ceil_div(OR_TILE, vdig);
    uint32_t* kw = hi ? k_hi : k_lo;
    uint32_t* vw = hi ? v_hi : v_lo;
    uint32_t* kz = hi ? kz_hi : kz_lo;
    uint32_t* vz = hi ? vz_hi : vz_lo;
    (void)seg;
    uint8_t* kc = (uint8_t*)calloc((size_t)WK * kdig, 1);
    uint8_t* vc = (uint8_t*)calloc((size_t)D, 1);
    uint8_t* buf = (uint8_t*)malloc((size_t)vdig);
    int tile = slot / OR_TILE, tt = slot % OR_TILE;
    for (int grp = 0; grp < NG; grp++) {
        uint16_t s16, z16;
        if (kgrid) { /* per-channel K grids fitted at prefill (clamped) */
            for (int d = grp * G; d < (grp + 1) * G; d++) {
                uint32_t g = kgrid[(size_t)seg * D + d];
                if (!isfinite(oracle_half_to_float(k[d]))) status |= OR_NONFINITE_KV;
                kc[d] = (uint8_t)oracle_code_on_grid(k[d], (uint16_t)(g & 0xFFFF), (uint16_t)(g >> 16), L);
            }
            kz[sz_index(tile, grp, tt, NG)] = 0;
        } else {
            status |= oracle_quantize_group_clip(k + grp * G, G, L, clip, kc + grp * G, &s16, &z16);
            kz[sz_index(tile, grp, tt, NG)] = (uint32_t)s16 | ((uint32_t)z16 << 16);
        }
        status |= oracle_quantize_group_clip(v + grp * G, G, Lv, clip, vc + grp * G, &s16, &z16);
        vz[sz_index(tile, grp, tt, NG)] = (uint32_t)s16 | ((uint32_t)z16 << 16);
    }
    for (int j = 0; j < WK; j++) kw[k_word_index(tile, j, tt, WK)] = oracle_pack_word(kc + j * kdig, kdig, L);
    for (int d = 0; d < D; d++) {
        /* rewrite the word that holds this slot with its digit set; other digits unchanged */
        size_t idx = v_word_index(tile, tt / vdig, d, WV, D);
        if (tt % vdig == 0) memset(buf, 0, (size_t)vdig); /* first slot of a word: fresh word */
        else oracle_unpack_word(vw[idx], vdig, Lv, buf);
        buf[tt % vdig] = vc[d];
        vw[idx] = oracle_pack_word(buf, vdig, Lv);
    }
    if (T % 32 == 0) {
        bitmap[T / 32] = 0;
        rank[T / 32] = (uint32_t)*n_hi;
    }
    if (hi) bitmap[T / 32] |= 1u << (T % 32);
    if (hi) (*n_hi)++;
    else (*n_lo)++;
    free(kc);
    free(vc);
    free(buf);
    return status;
}

/* ------------------------------------------------------------------ attention */

/*
 * fp64 decode attention for one unit: g query heads share one kv head (GQA).
 * q: [g][D] fp16 bits; Khat, Vhat: [T][D] fp32 (dequantized); out: [g][D] fp64.
 * logit_t = sm_scale * sum_d q_d k^_{t,d};  o = sum_t e^(logit_t - max) v^_t / sum_t e^(logit_t - max).
 * An empty unit (T = 0) gives o = 0.
 */
void oracle_attention_fp64(const uint16_t* q, int g, const float* Khat, const float* Vhat, int32_t T, int D,
                           float sm_scale, double* out)
{
    double* logit = (double*)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    double* qd = (double*)malloc(sizeof(double) * (size_t)D);
    for (int h = 0; h < g; h++) {
        for (int d = 0; d < D; d++) qd[d] = (double)oracle_half_to_float(q[h * D + d]);
        double mx = -INFINITY;
        for (int32_t t = 0; t < T; t++) {
            double acc = 0.0;
            for (int d = 0; d < D; d++) acc += qd[d] * (double)Khat[(size_t)t * D + d];
            logit[t] = (double)sm_scale * acc;
            if (logit[t] > mx) mx = logit[t];
        }
        double l = 0.0;
        for (int d = 0; d < D; d++) out[h * D + d] = 0.0;
        for (int32_t t = 0; t < T; t++) {
            double w = exp(logit[t] - mx);
            l += w;
            for (int d = 0; d < D; d++) out[h * D + d] += w * (double)Vhat[(size_t)t * D + d];
        }
        for (int d = 0; d < D; d++) out[h * D + d] = (l > 0.0) ? out[h * D + d] / l : 0.0;
    }
    free(logit);
    free(qd);
}

/*
 * The same decode attention of one unit with binary32 arithmetic and binary32 accumulation: the
 * timed CPU baseline of the attention (the fp64 routine above is the one parity is taken
 * against).  SemKV page, Abstract: attention over the compressed cache, whose dequantized values
 * Khat, Vhat are exact in binary32.  Plain loops in the order of the fp64 routine: logits
 * l_t = sm_scale * sum_d q_d Khat[t][d], then out = sum_t exp(l_t - max) Vhat[t] / sum_t exp(l_t - max).
 */
void oracle_attention_f32(const uint16_t* q, int g, const float* Khat, const float* Vhat, int32_t T, int D,
                          float sm_scale, float* out)
{
    float* logit = (float*)malloc(sizeof(float) * (size_t)(T > 0 ? T : 1));
    float* qf = (float*)malloc(sizeof(float) * (size_t)D);
    for (int h = 0; h < g; h++) {
        for (int d = 0; d < D; d++) qf[d] = oracle_half_to_float(q[h * D + d]);
        float mx = -INFINITY;
        for (int32_t t = 0; t < T; t++) {
            float acc = 0.0f;
            for (int d = 0; d < D; d++) acc += qf[d] * Khat[(size_t)t * D + d];
            logit[t] = sm_scale * acc;
            if (logit[t] > mx) mx = logit[t];
        }
        float l = 0.0f;
        for (int d = 0; d < D; d++) out[h * D + d] = 0.0f;
        for (int32_t t = 0; t < T; t++) {
            float w = expf(logit[t] - mx);
            l += w;
            for (int d = 0; d < D; d++) out[h * D + d] += w * Vhat[(size_t)t * D + d];
        }
        for (int d = 0; d < D; d++) out[h * D + d] = (l > 0.0f) ? out[h * D + d] / l : 0.0f;
    }
    free(logit);
    free(qf);
}

/* ------------------------------------------------------------------ array helpers for the tests */

void oracle_half_to_float_array(const uint16_t* h, float* f, int64_t n)
{
    for (int64_t i = 0; i < n; i++) f[i] = oracle_half_to_float(h[i]);
}

void oracle_float_to_half_up_array(const float* f, uint16_t* h, int64_t n)
{
    for (int64_t i = 0; i < n; i++) h[i] = oracle_float_to_half_up(f[i]);
}
