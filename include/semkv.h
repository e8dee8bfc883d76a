/*
 * semkv.h -- C ABI of libsemkv: the hot path of SemKV-style semantic mixed-precision KV-cache
 * quantization on NVIDIA B200 (sm_100a).
 *
 * The method is the one stated in the Abstract of the page "SemKV: Semantic Mixed-Precision KV
 * Cache Quantization Guided by the Quality Cliff for Long-Context LLM Inference" (arXiv
 * 2608.28911v1): every cached token is kept; tokens are ordered by an importance score taken from
 * inside the model; a fraction p of them is stored on the finer of two neighbouring uniform grids
 * (L_hi levels) and the rest on the coarser one (L_lo levels), both above the quality cliff; the
 * level counts need not be powers of two (5 levels = 2.322 code bits per value), so the average
 * precision interpolates between the two grids.  The Abstract also reports the cliff when tokens
 * are quantized during generation, which is what semkv_append_token does.  Decode attention over
 * the compressed cache is the consumer; the KVQuant blog page (section on the memory bottleneck)
 * notes that for long sequences the KV cache is the dominant memory traffic of decoding.
 *
 * Conventions for every entry point
 *   - All array pointers are DEVICE pointers (cudaMalloc'd or torch tensors), owned by the caller.
 *     The library allocates nothing and never synchronizes; work is enqueued on `stream`
 *     (a cudaStream_t passed as void*; NULL = the legacy default stream).
 *   - fp16 data are IEEE binary16 bit patterns (uint16_t).  Scores are IEEE binary32.
 *   - The return value is a host-side status (SEMKV_OK or SEMKV_ERR_*), known before any launch
 *     except SEMKV_ERR_CUDA (launch failure).  Problems only the device can see (NaN score,
 *     non-finite K/V, append past capacity) are OR-ed into the device word *status as
 *     SEMKV_STATUS_* bits; the caller reads it when it chooses.  No kernel traps or asserts.
 *   - A "unit" is one (batch row b, kv head h) pair, u = b*H + h.  Units are independent.
 *
 * Data layout of one layer's cache (all uint32 words; tile = 128 slots of one segment):
 *   k_seg   [B*H][cap_seg/128][WK][128]   K codes of one token row, base-L radix words:
 *                                          word j holds channels j*k .. j*k+k-1 of the slot,
 *                                          value sum_i code_i * L^i  (k = max{k: L^k <= 2^32},
 *                                          WK = ceil(D/k); channels past D are zero digits)
 *   v_seg   [B*H][cap_seg/128][WV][D]     V codes of one channel, packed along the slots of a
 *                                          tile: word w of channel d holds slots w*k .. w*k+k-1,
 *                                          value sum_i code_i * L^i  (WV = ceil(128/k); with V
 *                                          level counts of their own, L and k are the V ones)
 *   kz_seg, vz_seg [B*H][cap_seg/128][D/G][128]   per (slot, channel group): fp16 scale in the
 *                                          low half, fp16 zero in the high half
 *   bitmap  [B*H][T_cap/32]  bit t%32 of word t/32 = 1 iff token t is on the L_hi grid
 *   rank    [B*H][T_cap/32]  rank[w] = number of L_hi tokens in words 0..w-1 (valid for words
 *                            that hold at least one token)
 *   n_hi, n_lo [B*H] int32   tokens in each segment (a token's slot is its rank in its class)
 *                            Slots past n of a segment hold unspecified words, except that after
 *                            semkv_quantize_pack the rest of the last tile is zero, and a V word
 *                            that holds a live slot always has zero digits at the slots past n.
 *   tau     [B*H] float      precision threshold of the unit (the n_hi-th largest score)
 *   status  [1] int32        device status word (SEMKV_STATUS_* bits)
 *   slot_token [B*H][cap_hi + cap_lo] int32   token index of each prefill slot (L_hi segment
 *                            first, then L_lo): the inverse of the slot map, written by
 *                            semkv_assign_precision for slots < n and read by
 *                            semkv_quantize_pack; appends do not update it
 *   score_keys [B*H][T_cap] uint32   every token's score as an order-preserving key (-0 as +0;
 *                            key order = score order), written by semkv_assign_precision and by
 *                            every append; semkv_append_token_running ranks a new token by it
 *   kc      [B*H][2][D] uint32   per-channel K grids of the L_hi and L_lo segments (fp16 scale |
 *                            fp16 zero << 16), written by semkv_quantize_pack when k_per_channel
 *                            is set (then the per-token K scale/zero in kz_seg are 0)
 * Code c of value x on a group with scale s and zero z dequantizes to fmaf((float)c, s, z).
 */
#ifndef SEMKV_H
#define SEMKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define SEMKV_API __attribute__((visibility("default")))
#else
#define SEMKV_API
#endif

#define SEMKV_TILE 128

/* host-side return codes */
#define SEMKV_OK 0
#define SEMKV_ERR_INVALID_ARG 1 /* null pointer, bad shape (Hq % H, D % G, T > T_cap, p outside [0,1]) */
#define SEMKV_ERR_UNSUPPORTED 2 /* D != 128, L outside [2, 256], G not in {8,16,32,64,128}, Hq/H > 8 */
#define SEMKV_ERR_CAPACITY 3    /* the host can already see that a segment or T_cap is too small */
#define SEMKV_ERR_CUDA 4        /* a kernel launch failed (cudaGetLastError) */

/* device status word bits */
#define SEMKV_STATUS_NAN_SCORE 1       /* a score was NaN: its place in the order is unspecified */
#define SEMKV_STATUS_NONFINITE_KV 2    /* a K or V value was inf/NaN: its codes are unspecified */
#define SEMKV_STATUS_APPEND_OVERFLOW 4 /* an appended token found its segment (or T_cap) full and
                                          was dropped; that unit's state is unchanged */
#define SEMKV_STATUS_LENGTH_MISMATCH 8 /* semkv_dequantize: a unit's n_hi + n_lo != T */
#define SEMKV_STATUS_TIMEOUT 16        /* a kernel gave up a bounded wait (asynchronous copy or tensor-core
                                          result); that call's outputs are incomplete */

/* One layer's packed cache.  Shape fields are set by the caller; the pointers are device
 * buffers of the sizes semkv_cache_bytes() reports, in the order of the SEMKV_BUF_* indices. */
typedef struct semkv_cache {
    int32_t B, H, Hq, D, G; /* batch, kv heads, query heads (GQA group g = Hq/H), head dim, group */
    int32_t L_hi, L_lo;     /* level counts of the two grids (L_hi is used for the top fraction p) */
    int32_t cap_hi, cap_lo; /* slot capacity of each segment per unit, multiples of 128 */
    int32_t T_cap;          /* token capacity per unit (bitmap/rank length), multiple of 32 */
    /* Quantizer variants of prior art (the SKVQ abstract on the same pages); zero-initialised
     * fields give the plain method.
     *   window: semkv_assign_precision also puts the last min(window, T) tokens of each unit on
     *           the L_hi grid (recent tokens at high precision); >= 0.
     *   clip:   0 or 1 = the plain min/max grid.  In (0, 1): each group's min and max are first
     *           scaled by clip in fp32 (clipped range), the zero is the nearest binary16 of the
     *           scaled min (-0 stored as +0), the scale is fp16 rounded up of
     *           (clip*max - zero)/(L - 1) (at least 0); values outside take the end codes.  Used by
     *           semkv_quantize_pack and every append.  Other values: SEMKV_ERR_INVALID_ARG.
     *   L_hi_v, L_lo_v: level counts of the V codes of each segment (keys and values at different
     *           bit widths); 0 = the K level count (L_hi, L_lo), else in [2, 256].  The V words of a
     *           segment then hold k(L_v) codes each.  The tensor-core decode serves equal K and V
     *           counts; other segments run on the CUDA-core decode.
     *   k_per_channel: 0 = K grids per token and group of G channels (the plain method); 1 = one K
     *           grid per channel of each unit (keys quantized per channel), fitted by
     *           semkv_quantize_pack over all T prefill tokens (min and max of the channel, the clip
     *           applied), once on the L_hi and once on the L_lo levels, and kept in the `kc` buffer;
     *           every K code of the unit, appended tokens included, is coded on its channel's grid
     *           of its segment, clamped to [0, L-1]; the per-token K scale/zero are 0.  The decode
     *           folds each channel's scale into the query. */
    int32_t window;
    float clip;
    int32_t L_hi_v, L_lo_v;
    int32_t k_per_channel;
    uint32_t *k_hi, *v_hi, *kz_hi, *vz_hi;
    uint32_t *k_lo, *v_lo, *kz_lo, *vz_lo;
    uint32_t *bitmap, *rank;
    int32_t *n_hi, *n_lo;
    float *tau;
    int32_t *status;
    int32_t *slot_token;  /* [B*H][cap_hi + cap_lo], see the layout above */
    uint32_t *score_keys; /* [B*H][T_cap], see the layout above */
    uint32_t *kc;         /* [B*H][2][D] per-channel K grids (hi, lo): fp16 scale | fp16 zero << 16 */
} semkv_cache_t;

enum {
    SEMKV_BUF_K_HI = 0, SEMKV_BUF_V_HI, SEMKV_BUF_KZ_HI, SEMKV_BUF_VZ_HI,
    SEMKV_BUF_K_LO, SEMKV_BUF_V_LO, SEMKV_BUF_KZ_LO, SEMKV_BUF_VZ_LO,
    SEMKV_BUF_BITMAP, SEMKV_BUF_RANK, SEMKV_BUF_N_HI, SEMKV_BUF_N_LO, SEMKV_BUF_TAU, SEMKV_BUF_STATUS,
    SEMKV_BUF_SLOT_TOKEN, SEMKV_BUF_SCORE_KEYS, SEMKV_BUF_KC, SEMKV_NBUF
};

/* Byte size of each of the SEMKV_NBUF buffers of a cache with the shape fields of `shape`
 * (pointers ignored).  Pure host function.  Returns SEMKV_OK or a validation error. */
SEMKV_API int semkv_cache_bytes(const semkv_cache_t* shape, size_t sizes[SEMKV_NBUF]);

/* Sizing of a cache for a prefill (SemKV page, Abstract: the top fraction p of the tokens goes on
 * the finer grid).  Pure host function.  For a prefill of T tokens at fraction p with the last
 * min(window, T) tokens also on the finer grid, and room for `extra` appended tokens per unit:
 *   *n_sel  = floor(p*T), computed in double from the binary32 p (the count semkv_assign_precision
 *             puts on the finer grid by score),
 *   *cap_hi = n_sel + min(window, T) + extra, *cap_lo = T - n_sel + extra (each rounded up to a
 *             multiple of SEMKV_TILE), *T_cap = T + extra rounded up to a multiple of 32.
 * Any output pointer may be NULL.  Returns SEMKV_ERR_INVALID_ARG for T < 0, window < 0,
 * extra < 0, p outside [0, 1], or capacities that overflow int32. */
SEMKV_API int semkv_capacities(int32_t T, float p, int32_t window, int32_t extra, int32_t* n_sel, int32_t* cap_hi,
                               int32_t* cap_lo, int32_t* T_cap);

/* Bytes of device workspace semkv_decode_attention needs for this shape on the current device
 * (it depends on the device's SM count, which sets the split-K factor). */
SEMKV_API int semkv_workspace_bytes(const semkv_cache_t* shape, size_t* bytes);

/* Precision assignment (SemKV page, Abstract: tokens ranked by an internal score; the top fraction
 * gets the finer of two neighbouring grids).  scores: device fp32 [B][H][T].  For every unit:
 * n_sel = floor(p*T) (p in [0,1], computed in double); the n_sel tokens with the largest scores
 * (equal scores: lower token index first; -0 == +0) get bit 1 in the bitmap, and so do the last
 * min(window, T) tokens; n_hi = the number of 1 bits (n_sel when window = 0); rank[] and
 * slot_token[] are filled; n_lo = T - n_hi; tau = the n_sel-th largest score (+inf if
 * n_sel = 0).  Requires T <= T_cap, n_sel + min(window, T) <= cap_hi and T - n_sel <= cap_lo
 * (else SEMKV_ERR_CAPACITY).  NaN scores set SEMKV_STATUS_NAN_SCORE.  Bitmap words past the last
 * token are cleared. */
SEMKV_API int semkv_assign_precision(const semkv_cache_t* cache, const float* scores, int32_t T, float p,
                           void* stream);

/* Affine quantization and radix packing of a whole prefill (SemKV page, Abstract: uniform affine
 * grids with a level count that need not be a power of two).  K, V: device fp16 [B][H][T][D];
 * semkv_assign_precision must have run for this T.  Per token and group of G channels:
 * mn, mx = min, max; s = fp16 rounded up of fp32 (mx - mn)/(L - 1) (saturated at 65504);
 * z = mn; code = clamp(rint((x - z)/s), 0, L - 1) (fp32 subtract and divide, ties to even; 0 if
 * s = 0).  With the clip variant set in the cache, s and z are those of the clipped range (see
 * semkv_cache_t).  K and V must be 16-byte aligned (rows are fetched with bulk copies).  Codes are packed and placed as described at the top of this file; slots past the
 * segment's length inside its last tile get zero codes and zero scale/zero.  Non-finite inputs
 * set SEMKV_STATUS_NONFINITE_KV. */
SEMKV_API int semkv_quantize_pack(const semkv_cache_t* cache, const uint16_t* K, const uint16_t* V, int32_t T,
                        void* stream);

/* Quantization at generation time (SemKV page, Abstract): one new token per unit.  k, v: device
 * fp16 [B][H][D]; score: device fp32 [B][H].  The token is on the L_hi grid iff score > tau of
 * its unit (strict); it is quantized alone and written at slot n_seg of its segment; bitmap,
 * rank and n_hi/n_lo advance.  A full segment (or n_hi + n_lo = T_cap) drops the token and sets
 * SEMKV_STATUS_APPEND_OVERFLOW; a NaN score sets SEMKV_STATUS_NAN_SCORE (the token goes lo). */
SEMKV_API int semkv_append_token(const semkv_cache_t* cache, const uint16_t* k, const uint16_t* v, const float* score,
                       void* stream);

/* semkv_append_token with the exact running top-p rule instead of the fixed threshold tau: the
 * new token goes on the L_hi grid iff it is among the floor(p*(T+1)) largest of the unit's T+1
 * scores (equal scores: lower token index first, so the new token loses ties), i.e. iff fewer than
 * floor(p*(T+1)) earlier tokens have a score >= its score.  Earlier tokens keep their grid (their
 * original values are gone), so n_hi may differ from floor(p*(T+1)).  p in [0,1] (else
 * SEMKV_ERR_INVALID_ARG); reads the unit's score_keys (4 B per token); otherwise as
 * semkv_append_token. */
SEMKV_API int semkv_append_token_running(const semkv_cache_t* cache, const uint16_t* k, const uint16_t* v,
                                         const float* score, float p, void* stream);

/* GQA decode attention over the packed cache.  q: device fp16 [B][Hq][D]; out: device fp32
 * [B][Hq][D].  Query head qh attends with kv head qh / (Hq/H) over all n_hi + n_lo tokens of its
 * unit (no mask): out = sum_t softmax_t(softmax_scale * q.k^_t) v^_t with k^, v^ the dequantized
 * codes (dequantized in registers; the packed words are read once from HBM).  Split-K over token
 * tiles, then a log-sum-exp merge.  q must be 16-byte aligned (its rows are read 16 bytes at a
 * time).  workspace: device buffer of at least semkv_workspace_bytes() bytes (partial softmax
 * states), contents need not be initialized.
 * A unit with no tokens gives zeros.
 * Kernels: the integer tensor-core decode (codes as bytes, queries and p s_V as fixed-point limbs)
 * for level counts 4, 5, 6, 8, 16 with equal K and V counts and at least 8 tiles per warpgroup;
 * otherwise the fp16 tensor-core decode or, for shapes neither serves, the CUDA-core decode.  The
 * environment variable SEMKV_DECODE (read at every call, and by semkv_workspace_bytes) overrides
 * the tile-count rule: "i8" takes the integer decode wherever it serves the shape, "tc" never
 * takes it.  Size the workspace under the same setting as the call. */
SEMKV_API int semkv_decode_attention(const semkv_cache_t* cache, const uint16_t* q, float softmax_scale, float* out,
                           void* workspace, size_t workspace_bytes, void* stream);

/* semkv_append_token (fixed threshold) followed by semkv_decode_attention, in one pass over the
 * cache (SemKV page, Abstract: generation-time quantization): the decode CTA whose tiles hold the new
 * token's slot quantizes and writes the token before it reads that tile, and the merge then updates
 * the unit's counts, bitmap, rank and score key.  Results (cache state, out, status) are those of
 * the two calls in order.  Shapes the tensor-core decode does not cover run the two calls.  Every
 * argument (the decode's too) is checked first: an error returns before anything is enqueued, so
 * a failed call leaves the cache as it was.  k, v: device fp16 [B][H][D]; score: device fp32
 * [B][H]; the rest as semkv_decode_attention. */
SEMKV_API int semkv_append_decode(const semkv_cache_t* cache, const uint16_t* k, const uint16_t* v, const float* score,
                                  const uint16_t* q, float softmax_scale, float* out, void* workspace,
                                  size_t workspace_bytes, void* stream);

/* Bytes of the fixed device scratch that semkv_decode_attention_noalloc uses (per GPU). */
#define SEMKV_NOALLOC_SCRATCH_BYTES (4u << 20)

/* semkv_decode_attention without a workspace argument, for callers that cannot allocate device
 * memory when they decode (for example a plugin in a server whose process has already given all
 * device memory to its own pool allocator, or a service that forbids allocator calls after
 * start-up).  There is no counterpart on the SemKV page: this is a deployment convenience.
 * The split-K partials live in a fixed array of SEMKV_NOALLOC_SCRATCH_BYTES in device memory that
 * is part of the library image; every GPU that loads the library holds one until the process
 * exits.  Same arguments and results as semkv_decode_attention otherwise.
 *   - Allocates nothing: no cudaMalloc/cudaFree and no allocating library routine is called.
 *   - The first call on a device looks up the array's device address for that device
 *     (cudaGetSymbolAddress, with that device current); make that first call before any stream
 *     capture on the device.
 *   - Under CUDA's default lazy module loading, that first call is also when the driver loads the
 *     array into device memory (SEMKV_NOALLOC_SCRATCH_BYTES of it).  A caller whose pool allocator
 *     later takes all free device memory must therefore make the first call at start-up, before the
 *     pool is created (or run with CUDA_MODULE_LOADING=EAGER, which loads it with the library);
 *     otherwise that first call can fail with SEMKV_ERR_CUDA.
 *   - Shapes whose workspace (semkv_workspace_bytes) exceeds SEMKV_NOALLOC_SCRATCH_BYTES are
 *     rejected with SEMKV_ERR_CAPACITY before any launch.
 *   - All calls on a device share the one array and it keeps the last call's contents; nothing in
 *     it needs clearing (every partial is written before it is read), but two calls whose work
 *     overlaps on the GPU (different streams, no ordering between them) race on it. */
SEMKV_API int semkv_decode_attention_noalloc(const semkv_cache_t* cache, const uint16_t* q, float softmax_scale,
                                             float* out, void* stream);

/* Dequantize every token back to original token order (test and inspection path, not tuned).
 * K, V: device fp32 [B][H][T][D] outputs; T = n_hi + n_lo of every unit (else
 * SEMKV_STATUS_LENGTH_MISMATCH and the unit's rows are left as they were). */
SEMKV_API int semkv_dequantize(const semkv_cache_t* cache, float* K, float* V, int32_t T, void* stream);

/* Self-test of the bounded waits (test hook; the SemKV page has no counterpart).  Every wait in
 * the library's kernels gives up after a bounded number of tests and then sets
 * SEMKV_STATUS_TIMEOUT, frees the tensor memory it holds and returns; those waits cannot be made to
 * fail without breaking a copy or a product, so this call launches one small kernel (one warp)
 * whose wait nothing completes: one thread arrives on an mbarrier that expects two arrivals and
 * waits for the phase with at most `tests` tests (1 <= tests <= 65536; each sleeps at most
 * ~20 us).  use_tmem = 1: the warp allocates 32 tensor-memory columns before the wait and frees
 * them after it, as the decode kernels do.  On return of the kernel, *status (device int32) has
 * SEMKV_STATUS_TIMEOUT set.  Returns SEMKV_ERR_INVALID_ARG (null status, tests or use_tmem out of
 * range) or SEMKV_ERR_CUDA (launch failure). */
SEMKV_API int semkv_selftest_wait_timeout(int32_t* status, int32_t tests, int32_t use_tmem, void* stream);

/* Name of a host return code (SEMKV_OK ... SEMKV_ERR_CUDA). */
SEMKV_API const char* semkv_status_string(int code);

/* Radix parameters for L levels: digits per 32-bit word k(L) and words per D-channel row.
 * Pure host function; returns 0 for L outside [2, 256]. */
SEMKV_API int32_t semkv_radix_digits(int32_t L);

/* Fraction of tokens the finer grid can take under a storage budget (SemKV page, Abstract: measure
 * the quality cliff, then interpolate above it).  Physical bits per cached value (K and V
 * averaged) are
 *   bits(p) = p*B(L_hi, L_hi_v) + (1-p)*B(L_lo, L_lo_v) + 32/G + 1/(2D),
 *   B(Lk, Lv) = 16*ceil(D/k(Lk))/D + 16*ceil(128/k(Lv))/128
 * (K code words per row, V code words per 128-slot column, fp16 scale + zero per group, the
 * precision bitmap shared by K and V).  semkv_p_for_ratio uses L_hi_v = L_hi, L_lo_v = L_lo.  *p receives the largest p in [0,1] with 16/bits(p) >= ratio,
 * to be passed to semkv_assign_precision (which puts floor(p*T) tokens on the finer grid, never
 * more).  Pure host function.  Returns SEMKV_ERR_INVALID_ARG (null p, ratio not > 0, D or G not
 * positive, G not dividing D), SEMKV_ERR_UNSUPPORTED (L outside [2, 256]) or SEMKV_ERR_CAPACITY
 * (even p = 0 gives a smaller reduction than `ratio`). */
SEMKV_API int semkv_p_for_ratio(int32_t D, int32_t G, int32_t L_hi, int32_t L_lo, double ratio, double* p);
SEMKV_API int semkv_p_for_ratio_kv(int32_t D, int32_t G, int32_t L_hi, int32_t L_lo, int32_t L_hi_v, int32_t L_lo_v,
                                   double ratio, double* p);

#ifdef __cplusplus
}
#endif

#endif /* SEMKV_H */
