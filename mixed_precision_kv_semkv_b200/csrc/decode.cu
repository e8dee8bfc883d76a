// GQA decode attention over the packed mixed-precision cache: split-K partials + LSE merge.
//
// The cache is read once: each CTA streams its share of one segment's 128-slot tiles of one
// unit, unpacks the radix words in registers and folds the per-group scale and zero into the
// dot products (the KVQuant blog page notes that decoding long sequences is bound by reading the
// KV cache, so the packed words are the only large traffic).
//
// Per tile (4 warps, thread t = slot t for K, thread d = channel d for V):
//   logit_h(t) = sum_grp [ s_grp * sum_{d in grp} q_hd (c_d - m) + (z_grp + m s_grp) * sum_{d in grp} q_hd ]
// with m = (L - 1)/2: codes are centred so that the fp32 sums over channels and over tokens do
// not grow a common offset that would later cancel.  Online softmax in the log2 domain; the
// tile's probabilities p_h(t) times the V scale go to shared memory; thread d then accumulates
// sum_t p_h(t) s_V(t) (c_td - m), and the zero terms sum_t p_h(t) (z_V + m s_V) are summed per
// (group, head).  Each CTA writes (m_h, l_h, o_h[D]) to the workspace; a second kernel merges the
// splits with log-sum-exp weights.
#include "append.cuh"
#include "common.cuh"
#include "kernels.cuh"

namespace semkv {

constexpr int GMAX = 8;  // query heads per kv head supported by this kernel

template <int LC>
__device__ __forceinline__ void digits_of(uint32_t w, int L, int k, int (&out)[32])
{
    if constexpr (LC > 0) {
        int tmp[Radix<LC>::k];
        unpack_word<LC>(w, tmp);
#pragma unroll
        for (int i = 0; i < Radix<LC>::k; ++i) out[i] = tmp[i];
    } else {
        for (int i = 0; i < k; ++i) {
            out[i] = (int)(w % (uint32_t)L);
            w /= (uint32_t)L;
        }
    }
}

template <int LC>
__global__ void __launch_bounds__(128) k_decode_split(SegView seg, const uint16_t* __restrict__ q, int H, int g, int G,
                                                       float scale_log2, int nsplit, int split_off, int nsplit_total,
                                                       float* __restrict__ ws)
{
    constexpr int D = 128;
    const int L = LC ? LC : seg.L, Lv = LC ? LC : seg.Lv;  // LC > 0 only when K and V share it
    const int k = LC ? radix_k(LC) : radix_k(seg.L), kv = LC ? radix_k(LC) : radix_k(seg.Lv);
    const int WK = ceil_div(D, k), WV = ceil_div(TILE, kv);
    const int NG = D / G, NGg = NG * g;
    const int split = blockIdx.x, u = blockIdx.y;
    const int b = u / H, hk = u % H, Hq = H * g;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const float mid = 0.5f * (float)(L - 1), mid_v = 0.5f * (float)(Lv - 1);

    extern __shared__ __align__(16) float dsm[];
    float* qs = dsm;                 // [D][GMAX]
    float* qsum = qs + D * GMAX;     // [NG][GMAX]
    float* red = qsum + 16 * GMAX;   // [4][GMAX]
    float* zs = red + 4 * GMAX;      // [NG*g]
    float* ls = zs + 16 * GMAX;      // [GMAX]
    float* Pv = ls + GMAX;           // [TILE][NG*g]
    float* part = Pv + TILE * NGg;   // [TILE][NG*g]
    float* lpart = part + TILE * NGg;  // [TILE][GMAX]

    for (int i = tid; i < g * D; i += blockDim.x) {
        const int h = i / D, d = i % D;
        qs[d * GMAX + h] = h2f(q[((size_t)b * Hq + hk * g + h) * D + d]);
    }
    __syncthreads();
    for (int i = tid; i < NGg; i += blockDim.x) {
        const int grp = i / g, h = i % g;
        float s = 0.f;
        for (int d = grp * G; d < (grp + 1) * G; ++d) s += qs[d * GMAX + h];
        qsum[grp * GMAX + h] = s;
    }
    __syncthreads();
    // per-channel K grids: q_hd s_d replaces q_hd (the scale folds into the query) and the zero
    // terms sum_d q_hd (z_d + m s_d) become one constant per head
    __shared__ float kzt[GMAX];
    if (seg.kc) {
        float v[GMAX];
        {
            const uint32_t gk = seg.kc[(size_t)u * 256 + tid];  // thread = channel (128 threads)
            const float s = h2f((uint16_t)(gk & 0xffffu));
            const float zc = __fmaf_rn(mid, s, h2f((uint16_t)(gk >> 16)));
#pragma unroll
            for (int h = 0; h < GMAX; ++h) {
                v[h] = h < g ? qs[tid * GMAX + h] * zc : 0.f;
                if (h < g) qs[tid * GMAX + h] *= s;
            }
        }
#pragma unroll
        for (int h = 0; h < GMAX; ++h) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v[h] += __shfl_xor_sync(0xffffffffu, v[h], o);
            if (lane == 0) red[warp * GMAX + h] = v[h];
        }
        __syncthreads();
        if (tid < GMAX) kzt[tid] = red[tid] + red[GMAX + tid] + red[2 * GMAX + tid] + red[3 * GMAX + tid];
        __syncthreads();
    }

    const int n = seg.n[u];
    const int tiles = min(ceil_div(n, TILE), seg.tiles_cap);  // never past the segment's capacity
    int t0, t1;
    split_tiles(tiles, nsplit, split, t0, t1);

    float m[GMAX], acc[GMAX], zacc = 0.f, lacc = 0.f;
#pragma unroll
    for (int h = 0; h < GMAX; ++h) {
        m[h] = -__int_as_float(0x7f800000);
        acc[h] = 0.f;
    }
    const int grp_d = tid / G;

    for (int tile = t0; tile < t1; ++tile) {
        const size_t tb = (size_t)u * seg.tiles_cap + tile;
        const uint32_t* kw = seg.k + tb * WK * TILE;
        const uint32_t* vw = seg.v + tb * WV * D;
        const uint32_t* kz = seg.kz + tb * NG * TILE;
        const uint32_t* vz = seg.vz + tb * NG * TILE;
        const bool valid = tile * TILE + tid < n;

        // ---- K side: thread = slot
        float logit[GMAX], a[GMAX];
#pragma unroll
        for (int h = 0; h < GMAX; ++h) {
            logit[h] = seg.kc ? kzt[h] : 0.f;
            a[h] = 0.f;
        }
        int cur = 0;
        auto flush = [&](int grp) {
            if (seg.kc) {  // the channel scales are in qs
#pragma unroll
                for (int h = 0; h < GMAX; ++h)
                    if (h < g) logit[h] += a[h];
            } else {
                const uint32_t zz = kz[grp * TILE + tid];
                const float s = h2f((uint16_t)(zz & 0xffffu));
                const float zc = __fmaf_rn(mid, s, h2f((uint16_t)(zz >> 16)));
#pragma unroll
                for (int h = 0; h < GMAX; ++h)
                    if (h < g) logit[h] += s * a[h] + zc * qsum[grp * GMAX + h];
            }
#pragma unroll
            for (int h = 0; h < GMAX; ++h) a[h] = 0.f;
        };
        for (int j = 0; j < WK; ++j) {
            int dg[32];
            digits_of<LC>(kw[j * TILE + tid], L, k, dg);
#pragma unroll
            for (int i = 0; i < (LC ? Radix<(LC ? LC : 2)>::k : 32); ++i) {
                if (i >= k) break;
                const int d = j * k + i;
                if (d >= D) break;
                const int grp = d / G;
                if (grp != cur) {
                    flush(cur);
                    cur = grp;
                }
                const float cf = (float)dg[i] - mid;
#pragma unroll
                for (int h = 0; h < GMAX; ++h)
                    if (h < g) a[h] += qs[d * GMAX + h] * cf;
            }
        }
        flush(cur);

        // ---- online softmax (log2 domain)
        float alpha[GMAX], p[GMAX];
#pragma unroll
        for (int h = 0; h < GMAX; ++h) {
            if (h < g) {
                logit[h] = valid ? logit[h] * scale_log2 : -__int_as_float(0x7f800000);
                const float mx = warp_max(logit[h]);
                if (lane == 0) red[warp * GMAX + h] = mx;
            }
        }
        __syncthreads();
#pragma unroll
        for (int h = 0; h < GMAX; ++h) {
            if (h < g) {
                const float mt = fmaxf(fmaxf(red[h], red[GMAX + h]), fmaxf(red[2 * GMAX + h], red[3 * GMAX + h]));
                const float mn = fmaxf(m[h], mt);
                alpha[h] = exp2f(m[h] - mn);
                m[h] = mn;
                p[h] = valid ? exp2f(logit[h] - mn) : 0.f;
            } else {
                alpha[h] = p[h] = 0.f;
            }
        }
        for (int grp = 0; grp < NG; ++grp) {
            const uint32_t zz = vz[grp * TILE + tid];
            const float s = h2f((uint16_t)(zz & 0xffffu));
            const float zc = __fmaf_rn(mid_v, s, h2f((uint16_t)(zz >> 16)));
            for (int h = 0; h < g; ++h) {  // slots past n may hold stale scale/zero bits: write zeros
                Pv[tid * NGg + grp * g + h] = valid ? p[h] * s : 0.f;
                part[tid * NGg + grp * g + h] = valid ? p[h] * zc : 0.f;
            }
        }
#pragma unroll
        for (int h = 0; h < GMAX; ++h) lpart[tid * GMAX + h] = p[h];
        __syncthreads();

        // ---- V side: thread = channel
#pragma unroll
        for (int h = 0; h < GMAX; ++h) acc[h] *= alpha[h];
        for (int w = 0; w < WV; ++w) {
            int dg[32];
            digits_of<LC>(vw[w * D + tid], Lv, kv, dg);
#pragma unroll
            for (int i = 0; i < (LC ? Radix<(LC ? LC : 2)>::k : 32); ++i) {
                if (i >= kv) break;
                const int t = w * kv + i;
                if (t >= TILE) break;
                const float cf = (float)dg[i] - mid_v;
                const float* pv = Pv + t * NGg + grp_d * g;
#pragma unroll
                for (int h = 0; h < GMAX; ++h)
                    if (h < g) acc[h] += pv[h] * cf;
            }
        }
        if (tid < NGg) {
            float s = 0.f;
            for (int t = 0; t < TILE; ++t) s += part[t * NGg + tid];
            zacc = zacc * alpha[tid % g] + s;
        }
        if (tid < g) {
            float s = 0.f;
            for (int t = 0; t < TILE; ++t) s += lpart[t * GMAX + tid];
            lacc = lacc * alpha[tid] + s;
        }
        __syncthreads();
    }

    if (tid < NGg) zs[tid] = zacc;
    if (tid < g) ls[tid] = lacc;
    __syncthreads();
    float* out = ws + ((size_t)u * nsplit_total + split_off + split) * g * (D + 2);
    for (int h = 0; h < g; ++h) {
        out[h * (D + 2) + tid] = acc[h] + zs[grp_d * g + h];
        if (tid == 0) {
            out[h * (D + 2) + D] = m[h];
            out[h * (D + 2) + D + 1] = ls[h];
        }
    }
}

// Log-sum-exp merge of the split partials of one (unit, query head): all splits' maxima are read
// in parallel, the weights 2^(m_s - M) go to shared memory, then four slices of 128 threads each
// sum a quarter of the splits of o_s[d] with independent loads, and the slices are added.
// Merge of the split-K partials: one CTA per (unit, query head, 32-channel slice); its 512 threads
// first reduce the splits' maxima and denominators, then each of 16 warps sums a 16th of the
// splits for the slice's 32 channels, so every thread makes only a few independent loads.
constexpr int MERGE_CH = 32, MERGE_PARTS = 16;

__global__ void __launch_bounds__(32 * MERGE_PARTS) k_decode_merge(const float* __restrict__ ws, int g,
                                                                  int nsplit_total, float* __restrict__ out,
                                                                  semkv_cache_t cache,
                                                                  const uint16_t* __restrict__ knew,
                                                                  const float* __restrict__ snew)
{
    constexpr int D = 128, NT = 32 * MERGE_PARTS;
    // launched as a programmatic dependent of the split kernels: wait for them (and their writes)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int u = blockIdx.x / g, h = blockIdx.x % g;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (knew && h == 0 && blockIdx.y == 0 && tid == 0) {
        // the appended token's bookkeeping: every decode CTA has read the counts by now
        const float sc = snew[u];
        const int nh = cache.n_hi[u], nl = cache.n_lo[u];
        const bool hi = sc > cache.tau[u];
        if (append_fits(cache, hi, nh, nl)) append_state(cache, u, hi, nh, nl, sc);
        else atomicOr(cache.status, SEMKV_STATUS_APPEND_OVERFLOW | (isnan(sc) ? SEMKV_STATUS_NAN_SCORE : 0));
    }
    const float* base = ws + (size_t)u * nsplit_total * g * (D + 2) + h * (D + 2);
    const size_t stride = (size_t)g * (D + 2);
    extern __shared__ float wts[];  // [nsplit_total]: the splits' maxima, then their weights
    __shared__ float red[MERGE_PARTS], redl[MERGE_PARTS], part[MERGE_PARTS][MERGE_CH];
    const float NEG = -__int_as_float(0x7f800000);
    float M = NEG;
    for (int s = tid; s < nsplit_total; s += NT) {
        const float m = base[s * stride + D];
        wts[s] = m;
        M = fmaxf(M, m);
    }
    M = warp_max(M);
    if (lane == 0) red[warp] = M;
    __syncthreads();
    M = NEG;
#pragma unroll
    for (int i = 0; i < MERGE_PARTS; ++i) M = fmaxf(M, red[i]);
    float l = 0.f;
    for (int s = tid; s < nsplit_total; s += NT) {
        const float w = M == NEG ? 0.f : exp2f(wts[s] - M);
        wts[s] = w;
        l += w * base[s * stride + D + 1];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    if (lane == 0) redl[warp] = l;
    __syncthreads();
    float Ls = 0.f;
#pragma unroll
    for (int i = 0; i < MERGE_PARTS; ++i) Ls += redl[i];
    const int d = blockIdx.y * MERGE_CH + lane;
    float O = 0.f;
    for (int s = warp; s < nsplit_total; s += MERGE_PARTS) O += wts[s] * base[s * stride + d];
    part[warp][lane] = O;
    __syncthreads();
    if (warp == 0) {
        float t = 0.f;
#pragma unroll
        for (int i = 0; i < MERGE_PARTS; ++i) t += part[i][lane];
        out[((size_t)u * g + h) * D + d] = Ls > 0.f ? t / Ls : 0.f;
    }
}

// The same merge for few splits per unit (at most MERGE_FEW): one CTA of 128 threads per (unit,
// query head), thread d owns output channel d.  Every thread reads the splits' maxima and
// denominators (the same addresses in all lanes: one transaction per warp) and its channel of each
// split's output, so there is no barrier and a many-unit grid is resident at once (its tail is on
// the step's critical path).  With many splits the serial loop is slower than the kernel above
// (measured on B200: 8 splits per unit over 128 units favour this kernel, 11 and more the other).
constexpr int MERGE_FEW = 8;

__global__ void __launch_bounds__(128) k_decode_merge_few(const float* __restrict__ ws, int g, int nsplit_total,
                                                      float* __restrict__ out, semkv_cache_t cache,
                                                      const uint16_t* __restrict__ knew,
                                                      const float* __restrict__ snew)
{
    constexpr int D = 128;
    // launched as a programmatic dependent of the split kernels: wait for them (and their writes)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int u = blockIdx.x / g, h = blockIdx.x % g, d = threadIdx.x;
    if (knew && h == 0 && d == 0) {
        // the appended token's bookkeeping: every decode CTA has read the counts by now
        const float sc = snew[u];
        const int nh = cache.n_hi[u], nl = cache.n_lo[u];
        const bool hi = sc > cache.tau[u];
        if (append_fits(cache, hi, nh, nl)) append_state(cache, u, hi, nh, nl, sc);
        else atomicOr(cache.status, SEMKV_STATUS_APPEND_OVERFLOW | (isnan(sc) ? SEMKV_STATUS_NAN_SCORE : 0));
    }
    const float* base = ws + (size_t)u * nsplit_total * g * (D + 2) + h * (D + 2);
    const size_t stride = (size_t)g * (D + 2);
    const float NEG = -__int_as_float(0x7f800000);
    float M = NEG;
#pragma unroll 4
    for (int s = 0; s < nsplit_total; ++s) M = fmaxf(M, base[s * stride + D]);
    float L = 0.f, O = 0.f;
    if (M != NEG) {  // every split empty: the unit has no tokens, its output is 0
#pragma unroll 4
        for (int s = 0; s < nsplit_total; ++s) {
            const float* r = base + s * stride;
            const float w = exp2f(r[D] - M);
            L = fmaf(w, r[D + 1], L);
            O = fmaf(w, r[d], O);
        }
    }
    out[((size_t)u * g + h) * D + d] = L > 0.f ? O / L : 0.f;
}

static size_t decode_smem(int NGg)
{
    return sizeof(float) * ((size_t)128 * GMAX + 16 * GMAX + 4 * GMAX + 16 * GMAX + GMAX + (size_t)2 * TILE * NGg +
                            (size_t)TILE * GMAX);
}

template <int LC>
static void launch_ds(const SegView& seg, const uint16_t* q, int units, int H, int g, int G, float scale_log2,
                      int nsplit, int split_off, int nsplit_total, float* ws, cudaStream_t st)
{
    const size_t sm = decode_smem((128 / G) * g);
    cudaFuncSetAttribute(k_decode_split<LC>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    dim3 grid(nsplit, units);
    k_decode_split<LC><<<grid, 128, sm, st>>>(seg, q, H, g, G, scale_log2, nsplit, split_off, nsplit_total, ws);
}

void launch_decode_split(const SegView& seg, const uint16_t* q, int units, int H, int g, int D, int G,
                         float scale_log2, int nsplit, int split_off, int nsplit_total, float* ws, cudaStream_t st)
{
    (void)D;
    if (nsplit == 0 || units == 0) return;
    if (seg.Lv != seg.L) {  // V level count of its own: both radixes at run time
        launch_ds<0>(seg, q, units, H, g, G, scale_log2, nsplit, split_off, nsplit_total, ws, st);
        return;
    }
    switch (seg.L) {
#define SEMKV_D(LL) \
    case LL: launch_ds<LL>(seg, q, units, H, g, G, scale_log2, nsplit, split_off, nsplit_total, ws, st); break;
        SEMKV_D(2) SEMKV_D(3) SEMKV_D(4) SEMKV_D(5) SEMKV_D(6) SEMKV_D(7) SEMKV_D(8) SEMKV_D(9)
        SEMKV_D(10) SEMKV_D(11) SEMKV_D(12) SEMKV_D(13) SEMKV_D(14) SEMKV_D(15) SEMKV_D(16)
#undef SEMKV_D
        default: launch_ds<0>(seg, q, units, H, g, G, scale_log2, nsplit, split_off, nsplit_total, ws, st); break;
    }
}

void launch_decode_merge(const float* ws, int units, int H, int g, int D, int nsplit_total, float* out,
                         const AppendIn& app, cudaStream_t st)
{
    (void)H;
    (void)D;
    const bool few = nsplit_total <= MERGE_FEW;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = few ? dim3((unsigned)(units * g)) : dim3((unsigned)(units * g), 128 / MERGE_CH);
    cfg.blockDim = dim3(few ? 128 : 32 * MERGE_PARTS);
    cfg.dynamicSmemBytes = few ? 0 : (size_t)(nsplit_total > 0 ? nsplit_total : 1) * sizeof(float);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, few ? k_decode_merge_few : k_decode_merge, ws, g, nsplit_total, out, app.cache, app.k,
                       app.score);
}

}  // namespace semkv
