// Decode attention without a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they decode: for example a plugin
// inside an inference server whose host process has already handed the whole device memory to its
// own pool allocator, so a cudaMalloc there would fail or fragment that pool, or a service that
// forbids allocator calls after start-up to keep its latency predictable.  For them this file
// keeps the split-K partials of semkv_decode_attention in a fixed array in device memory that is
// part of the library image (SEMKV_NOALLOC_SCRATCH_BYTES per GPU that loads the library, held
// until the process exits), and semkv_decode_attention_noalloc hands that array to the ordinary
// decode path as its workspace.  Nothing in it allocates.  With CUDA's lazy module loading the
// driver places the array in device memory when the first call looks up its address, so a caller
// whose pool will take all free device memory makes that first call at start-up.
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"

namespace {

// file-scope scratch: one copy per device that loads the library
static __device__ __align__(256) unsigned char g_scratch[SEMKV_NOALLOC_SCRATCH_BYTES];

constexpr int MAX_DEVICES = 64;
std::mutex g_mu;
void* g_scratch_addr[MAX_DEVICES] = {};

// Device address of g_scratch on the current device.  In host code `g_scratch` names a host-side
// stand-in, never a device address, so the address is asked for once per device (with that device
// current) and remembered.
int scratch_address(void** out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) {
        cudaGetLastError();
        return SEMKV_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return SEMKV_ERR_CUDA;
        }
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return SEMKV_OK;
}

}  // namespace

extern "C" int semkv_decode_attention_noalloc(const semkv_cache_t* cache, const uint16_t* q, float softmax_scale,
                                              float* out, void* stream)
{
    size_t need = 0;
    const int r = semkv_workspace_bytes(cache, &need);
    if (r != SEMKV_OK) return r;
    if (need > SEMKV_NOALLOC_SCRATCH_BYTES) return SEMKV_ERR_CAPACITY;  // shape too large for the fixed scratch
    void* scratch = nullptr;
    const int a = scratch_address(&scratch);
    if (a != SEMKV_OK) return a;
    return semkv_decode_attention(cache, q, softmax_scale, out, scratch, SEMKV_NOALLOC_SCRATCH_BYTES, stream);
}
