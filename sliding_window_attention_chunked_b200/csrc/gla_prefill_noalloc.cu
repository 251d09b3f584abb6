// gla_prefill_noalloc.cu -- rod_gla_prefill for callers that cannot allocate device memory.
//
// Some callers have no way to obtain device scratch per call: code that runs inside a host
// runtime whose memory pool they do not control, plug-ins that must not call cudaMalloc or a
// framework allocator (an allocation can synchronise the device, fail under memory pressure,
// or is simply not offered by the host program), and real-time paths that must never allocate
// after start-up. For them this file keeps the chunkwise prefill's scratch in one fixed
// device array that is part of the library's image, so the call itself allocates nothing.
//
// Properties a user of rod_gla_prefill_noalloc relies on:
//  * The scratch is a file-scope device array of ROD_GLA_PREFILL_NOALLOC_MAX_SCRATCH bytes
//    (48 MiB). Every GPU on which this code is used holds it until the process exits.
//  * Its device address is looked up once per device, on the first call made with that
//    device current (cudaGetSymbolAddress). That first call should come before any stream
//    capture begins.
//  * A problem whose scratch need (rod_gla_prefill_workspace_size) exceeds that size is
//    rejected with ROD_ERR_WORKSPACE before anything is launched. A failed address lookup
//    returns ROD_ERR_CUDA.
//  * All calls on a device share the one array, and it keeps whatever the last call left in
//    it. No part of it needs to start at zero: every scratch byte a call reads is written
//    earlier in that same call. Calls whose work overlaps on the GPU (different streams
//    without ordering between them, or several host threads) race on the array and give
//    wrong results; callers must serialise them.
// The kernels are exactly those of rod_gla_prefill; only where the scratch lives differs.
#include <math.h>
#include <stdint.h>

#include <mutex>

#include "../../include/rod.h"
#include "kernels.h"

namespace {

constexpr size_t kScratchBytes = ROD_GLA_PREFILL_NOALLOC_MAX_SCRATCH;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once per device).
int scratch_address(void** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ROD_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p) return ROD_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return ROD_OK;
}

bool dim_ok(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" {

int rod_gla_prefill_noalloc(const void* q, const void* k, const void* v, const float* g,
                            float* state, void* o, int B, int H, int T, int dk, int dv, int chunk,
                            int dtype, void* stream) {
    if (dtype != ROD_BF16 && dtype != ROD_FP32) return ROD_ERR_DTYPE;
    if (B < 0 || H < 0 || T < 0 || !dim_ok(dk) || !dim_ok(dv)) return ROD_ERR_SHAPE;
    if (chunk < 16 || chunk > 128 || chunk % 16 != 0) return ROD_ERR_SHAPE;
    if ((int64_t)B * H == 0 || T == 0) return ROD_OK;
    if (!q || !k || !v || !g || !state || !o) return ROD_ERR_NULL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) || !aligned16(state) ||
        !aligned16(o))
        return ROD_ERR_ALIGN;
    const size_t need = rod_gla_prefill_workspace_size(B, H, T, dk, dv, chunk, dtype);
    if (need > kScratchBytes) return ROD_ERR_WORKSPACE;  // larger than the fixed scratch
    void* scratch = nullptr;
    if (need > 0) {
        const int st = scratch_address(&scratch);
        if (st != ROD_OK) return st;
    }
    return rod_gla_prefill(q, k, v, g, state, o, B, H, T, dk, dv, chunk, dtype, scratch, need,
                           stream);
}

}  // extern "C"
