// Host-side launchers of the libsemkv kernels (defined in the .cu files of this directory).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/semkv.h"

namespace semkv {

// The V level count of a segment: 0 (unset) means the K level count.
__host__ __device__ __forceinline__ int level_v(const semkv_cache_t& c, bool hi)
{
    return hi ? (c.L_hi_v ? c.L_hi_v : c.L_hi) : (c.L_lo_v ? c.L_lo_v : c.L_lo);
}

// The clip ratio a cache asks for: 0 (unset) means 1, the plain min/max grid.
__host__ __device__ __forceinline__ float clip_ratio(const semkv_cache_t& c) { return c.clip == 0.0f ? 1.0f : c.clip; }

// One segment (hi or lo) of one layer's cache, as the kernels see it.
struct SegView {
    uint32_t* k;    // [units][tiles_cap][WK][128]
    uint32_t* v;    // [units][tiles_cap][WV][D]
    uint32_t* kz;   // [units][tiles_cap][NG][128]
    uint32_t* vz;   // [units][tiles_cap][NG][128]
    int32_t* n;     // [units] tokens in the segment
    int L;          // levels of the K codes
    int Lv;         // levels of the V codes
    int tiles_cap;  // capacity in tiles of 128 slots
    int is_hi;      // 1: L_hi segment (bitmap bit 1), 0: L_lo segment
    const uint32_t* kc;  // per-channel K grids of this segment (unit u at + u * 256), or null
};

// A generated token to append while decoding (k == nullptr: none); the fixed-threshold rule.
struct AppendIn {
    semkv_cache_t cache;
    const uint16_t* k;
    const uint16_t* v;
    const float* score;
};

// also writes slot_token [units][cap_hi + cap_lo]: the token index of every prefill slot
// n_sel tokens by score, then the last `window` tokens (window <= T) also get the L_hi grid
void launch_select(const float* scores, int units, int T, int n_sel, int window, int words_cap, uint32_t* bitmap,
                   uint32_t* rank, int32_t* n_hi_out, int32_t* n_lo_out, float* tau, int32_t* status,
                   int32_t* slot_token, int cap_hi, int cap_lo, uint32_t* score_keys, cudaStream_t st);

// reads the slot map (slot_token) that launch_select wrote
void launch_quantize(const SegView& hi, const SegView& lo, const uint16_t* K, const uint16_t* V,
                     const int32_t* slot_token, int units, int T, int D, int G, float clip, const uint32_t* kc,
                     int32_t* status, cudaStream_t st);

// per-channel K grids of every unit from the prefill's K (kchannel.cu)
void launch_kc_grids(const semkv_cache_t& c, const uint16_t* K, int T, int sms, cudaStream_t st);

// p < 0: the fixed threshold rule (score > tau); p in [0, 1]: the running top-p rule
void launch_append(const semkv_cache_t& c, const uint16_t* k, const uint16_t* v, const float* score, float p,
                   cudaStream_t st);

// decode: split partials of one segment go to splits [split_off, split_off + nsplit) of each unit
void launch_decode_split(const SegView& seg, const uint16_t* q, int units, int H, int g, int D, int G,
                         float scale_log2, int nsplit, int split_off, int nsplit_total, float* ws, cudaStream_t st);
// with app.k != nullptr the merge also does the appended tokens' bookkeeping (counts, bitmap, rank,
// score keys, status), once every decode CTA has read the counts
void launch_decode_merge(const float* ws, int units, int H, int g, int D, int nsplit_total, float* out,
                         const AppendIn& app, cudaStream_t st);

// tcgen05 decode (decode_tc.cu): the instantiated (K levels, V levels, g, groups, per-channel K), G >= 32.
bool decode_tc_supported(int Lk, int Lv, int G, int g, bool kpc);
// `dependent`: launched as a programmatic dependent of the previous kernel in the stream (it may
// start while that kernel drains, and waits for it to complete before it exits).
void launch_decode_tc(const SegView& seg, const uint16_t* q, int units, int H, int g, int G, float scale_log2,
                      int nsplit, int split_off, int nsplit_total, float* ws, int32_t* status, bool dependent,
                      const AppendIn& app, cudaStream_t st);

// integer tensor-core decode (decode_i8.cu): one CTA of 4 warpgroups per SM; `ctas` CTAs share the
// segment's units x tiles_cap tiles in contiguous ranges; unit u's partial states go to slots
// [slot_off, slot_off + slots) of its slots_total.  Covers equal K/V level counts in {4, 5, 6, 8,
// 16}, per-token K grids, and (g, groups) in {(2,1), (2,2), (4,1), (4,2), (8,1)}.
bool decode_i8_supported(int Lk, int Lv, int G, int g, bool kpc);
void launch_decode_i8(const SegView& seg, const uint16_t* q, int units, int H, int g, int G, float scale_log2,
                      int ctas, int slots, int slot_off, int slots_total, float* ws, int32_t* status, bool dependent,
                      const AppendIn& app, cudaStream_t st);

void launch_dequantize(const semkv_cache_t& c, int T, float* K, float* V, cudaStream_t st);

}  // namespace semkv
