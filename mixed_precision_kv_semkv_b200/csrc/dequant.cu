// Dequantization back to original token order (inspection and test path; not on the timed path).
//
// Token t of unit u is in the hi segment iff bitmap bit t is set; its slot is its rank within
// its class (rank directory + popcount of the lower bits of its word).  x^ = fmaf(c, s, z).
// One thread per token; K codes come from the slot's row words, V codes from the channel words
// of the slot's tile.
#include "common.cuh"
#include "kernels.cuh"

namespace semkv {

__global__ void __launch_bounds__(128) k_dequantize(semkv_cache_t c, int T, float* __restrict__ Kout,
                                                     float* __restrict__ Vout)
{
    constexpr int D = 128;
    const int u = blockIdx.y;
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    const int nh = c.n_hi[u], nl = c.n_lo[u];
    if (nh + nl != T) {
        if (t == 0) atomicOr(c.status, SEMKV_STATUS_LENGTH_MISMATCH);
        return;
    }
    if (t >= T) return;
    const int G = c.G, NG = D / G;
    const int words_cap = c.T_cap / 32;
    const uint32_t word = c.bitmap[(size_t)u * words_cap + t / 32];
    const uint32_t r = c.rank[(size_t)u * words_cap + t / 32];
    const bool hi = (word >> (t % 32)) & 1u;
    const int below = (int)r + __popc(word & ((1u << (t % 32)) - 1u));
    const int slot = hi ? below : t - below;
    const int L = hi ? c.L_hi : c.L_lo, Lv = level_v(c, hi);
    const int k = radix_k(L), kv = radix_k(Lv);
    const int WK = ceil_div(D, k), WV = ceil_div(TILE, kv);
    const int tiles_cap = (hi ? c.cap_hi : c.cap_lo) / TILE;
    if (slot >= tiles_cap * TILE) {  // state inconsistent with the capacity: leave the row
        atomicOr(c.status, SEMKV_STATUS_LENGTH_MISMATCH);
        return;
    }
    const int tile = slot / TILE, tt = slot % TILE;
    const size_t tb = (size_t)u * tiles_cap + tile;
    const uint32_t* kw = (hi ? c.k_hi : c.k_lo) + tb * WK * TILE;
    const uint32_t* vw = (hi ? c.v_hi : c.v_lo) + tb * WV * D;
    const uint32_t* kz = (hi ? c.kz_hi : c.kz_lo) + tb * NG * TILE;
    const uint32_t* vz = (hi ? c.vz_hi : c.vz_lo) + tb * NG * TILE;
    float* ko = Kout + ((size_t)u * T + t) * D;
    float* vo = Vout + ((size_t)u * T + t) * D;
    for (int d = 0; d < D; ++d) {
        const uint32_t kzv = c.k_per_channel ? c.kc[(size_t)u * 2 * D + (hi ? 0 : D) + d] : kz[(d / G) * TILE + tt];
        const uint32_t vzv = vz[(d / G) * TILE + tt];
        const int ck = digit_rt(kw[(d / k) * TILE + tt], L, d % k);
        const int cv = digit_rt(vw[(tt / kv) * D + d], Lv, tt % kv);
        ko[d] = __fmaf_rn((float)ck, h2f((uint16_t)(kzv & 0xffffu)), h2f((uint16_t)(kzv >> 16)));
        vo[d] = __fmaf_rn((float)cv, h2f((uint16_t)(vzv & 0xffffu)), h2f((uint16_t)(vzv >> 16)));
    }
}

void launch_dequantize(const semkv_cache_t& c, int T, float* K, float* V, cudaStream_t st)
{
    dim3 grid((unsigned)ceil_div(T > 0 ? T : 1, 128), (unsigned)(c.B * c.H));
    k_dequantize<<<grid, 128, 0, st>>>(c, T, K, V);
}

}  // namespace semkv
