// rod_api.cu -- the C ABI of librod.so (declared in include/rod.h): host-side argument
// validation, then dispatch to the kernels. Nothing here computes on the data.
#include <math.h>
#include <stdint.h>

#include <atomic>

#include "../../include/rod.h"
#include "kernels.h"

namespace rod {
static std::atomic<uint64_t> g_launches{0};
void note_launches(unsigned n) { g_launches.fetch_add(n, std::memory_order_relaxed); }
}  // namespace rod

namespace {

thread_local int t_last_cuda_error = 0;

bool dim_ok(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool dtype_ok(int dt) { return dt == ROD_BF16 || dt == ROD_FP32; }

int from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return ROD_OK;
    t_last_cuda_error = (int)e;
    return ROD_ERR_CUDA;
}

float resolve_scale(float scale, int dk) { return scale > 0.f ? scale : 1.0f / sqrtf((float)dk); }

}  // namespace

extern "C" {

const char* rod_status_string(int status) {
    switch (status) {
        case ROD_OK: return "ok";
        case ROD_ERR_NULL: return "null pointer argument";
        case ROD_ERR_SHAPE: return "unsupported or out-of-range size";
        case ROD_ERR_ALIGN: return "pointer not 16-byte aligned";
        case ROD_ERR_DTYPE: return "unsupported dtype";
        case ROD_ERR_WORKSPACE: return "workspace missing or too small";
        case ROD_ERR_CUDA: return "CUDA error";
        case ROD_ERR_TIMEOUT: return "a bounded device wait expired";
    }
    return "unknown status";
}

int rod_last_cuda_error(void) { return t_last_cuda_error; }

int rod_abi_version(void) { return 1; }

int rod_test_expire_waits(uint32_t probes) {
    rod::gla_prefill_tc_arm_wait_expiry(probes);
    return ROD_OK;
}

uint64_t rod_launch_count(void) { return rod::g_launches.load(std::memory_order_relaxed); }

int rod_check(void* stream) {
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return from_cuda(e);
    const unsigned flags = rod::swska_decode_take_timeout_flag() |
                           rod::swska_decode_warp_take_timeout_flag() |
                           rod::swska_prefill_tc_take_timeout_flag() |
                           rod::gla_prefill_tc_take_timeout_flag() |
                           rod::gla_backward_tc_take_timeout_flag() |
                           rod::swska_backward_tc_take_timeout_flag();
    if (flags) return ROD_ERR_TIMEOUT;
    return from_cuda(cudaGetLastError());
}

size_t rod_gla_prefill_workspace_size(int B, int H, int T, int dk, int dv, int chunk, int dtype) {
    if (B < 0 || H < 0 || T < 0 || !dim_ok(dk) || !dim_ok(dv) || !dtype_ok(dtype)) return 0;
    if (chunk < 16 || chunk > 128 || chunk % 16 != 0) return 0;
    if (dtype == ROD_BF16 && rod::gla_prefill_tc_supported(dk, dv, chunk))
        return rod::gla_prefill_tc_workspace_size(B, H, T);
    return 0;
}

int rod_gla_prefill(const void* q, const void* k, const void* v, const float* g, float* state,
                    void* o, int B, int H, int T, int dk, int dv, int chunk, int dtype,
                    void* workspace, size_t ws_bytes, void* stream) {
    if (!dtype_ok(dtype)) return ROD_ERR_DTYPE;
    if (B < 0 || H < 0 || T < 0 || !dim_ok(dk) || !dim_ok(dv)) return ROD_ERR_SHAPE;
    if (chunk < 16 || chunk > 128 || chunk % 16 != 0) return ROD_ERR_SHAPE;
    if ((int64_t)B * H == 0 || T == 0) return ROD_OK;
    if (!q || !k || !v || !g || !state || !o) return ROD_ERR_NULL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) || !aligned16(state) ||
        !aligned16(o))
        return ROD_ERR_ALIGN;
    const size_t need = rod_gla_prefill_workspace_size(B, H, T, dk, dv, chunk, dtype);
    if (need > 0 && (!workspace || ws_bytes < need)) return ROD_ERR_WORKSPACE;
    if (need > 0 && !aligned16(workspace)) return ROD_ERR_ALIGN;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    // bf16 with 128-wide heads and 64-token chunks runs the chunkwise tensor-core kernels;
    // fp32 (exact FMA) and the other shapes run the sequential-in-time CUDA-core kernel
    if (dtype == ROD_BF16 && rod::gla_prefill_tc_supported(dk, dv, chunk))
        return from_cuda(rod::gla_prefill_tc_launch(q, k, v, g, state, o, B, H, T, workspace, s));
    return from_cuda(rod::gla_prefill_recurrent_launch(q, k, v, g, state, o, B, H, T, dk, dv,
                                                       dtype == ROD_BF16, s));
}

int rod_gla_decode_step(const void* q, const void* k, const void* v, const float* g,
                        float* state, void* o, int N, int H, int dk, int dv, int dtype,
                        void* stream) {
    if (!dtype_ok(dtype)) return ROD_ERR_DTYPE;
    if (N < 0 || H < 0 || !dim_ok(dk) || !dim_ok(dv)) return ROD_ERR_SHAPE;
    if ((int64_t)N * H == 0) return ROD_OK;
    if (!q || !k || !v || !g || !state || !o) return ROD_ERR_NULL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) || !aligned16(state) ||
        !aligned16(o))
        return ROD_ERR_ALIGN;
    return from_cuda(rod::gla_decode_launch(q, k, v, g, state, o, N, H, dk, dv,
                                            dtype == ROD_BF16, static_cast<cudaStream_t>(stream)));
}

int rod_swska_prefill(const void* q, const void* k, const void* v, void* o, int B, int H,
                      int T, int dk, int dv, int window, float scale, int dtype, void* stream) {
    if (!dtype_ok(dtype)) return ROD_ERR_DTYPE;
    if (B < 0 || H < 0 || T < 0 || H > 64 || window < 1 || !dim_ok(dk) || !dim_ok(dv))
        return ROD_ERR_SHAPE;
    if (!(scale == scale) || isinf(scale)) return ROD_ERR_SHAPE;
    if ((int64_t)B * H == 0 || T == 0) return ROD_OK;
    if (!q || !k || !v || !o) return ROD_ERR_NULL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return ROD_ERR_ALIGN;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    // bf16 with 128-wide heads runs on the tensor cores; fp32 (exact FMA) and the small head
    // dims run on the CUDA-core kernel
    if (dtype == ROD_BF16 && rod::swska_prefill_tc_supported(H, T, dk, dv))
        return from_cuda(rod::swska_prefill_tc_launch(q, k, v, o, B, H, T, window,
                                                      resolve_scale(scale, dk), s));
    return from_cuda(rod::swska_prefill_simt_launch(q, k, v, o, B, H, T, dk, dv, window,
                                                    resolve_scale(scale, dk), dtype == ROD_BF16, s));
}

int rod_swska_prefill_lse(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                          int T, int dk, int dv, int window, float scale, int dtype, void* stream) {
    if (!dtype_ok(dtype)) return ROD_ERR_DTYPE;
    if (B < 0 || H < 0 || T < 0 || H > 64 || window < 1 || !dim_ok(dk) || !dim_ok(dv))
        return ROD_ERR_SHAPE;
    if (!(scale == scale) || isinf(scale)) return ROD_ERR_SHAPE;
    if ((int64_t)B * H == 0 || T == 0) return ROD_OK;
    if (!q || !k || !v || !o || !lse) return ROD_ERR_NULL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || reinterpret_cast<uintptr_t>(lse) % 4)
        return ROD_ERR_ALIGN;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the routes of rod_swska_prefill; the tensor-core kernel runs its statistics instantiation,
    // which stores the output and each row's log-sum-exp (times ln 2: natural log)
    if (dtype == ROD_BF16 && rod::swska_prefill_tc_supported(H, T, dk, dv))
        return from_cuda(rod::swska_prefill_tc_stats_launch(q, k, v, o, nullptr, lse, nullptr, T, B, H, T, window,
                                                            resolve_scale(scale, dk), s, 0.6931471805599453f));
    return from_cuda(rod::swska_prefill_simt_launch(q, k, v, o, B, H, T, dk, dv, window,
                                                    resolve_scale(scale, dk), dtype == ROD_BF16, s, lse));
}

int rod_swska_decode(const void* q, const void* k_new, const void* v_new, void* k_cache,
                     void* v_cache, const int64_t* pos, void* o, int N, int H, int dk, int dv,
                     int window, float scale, int dtype, void* stream) {
    if (!dtype_ok(dtype)) return ROD_ERR_DTYPE;
    if (N < 0 || H < 1 || H > 64 || window < 1 || !dim_ok(dk) || !dim_ok(dv))
        return ROD_ERR_SHAPE;
    if (!(scale == scale) || isinf(scale)) return ROD_ERR_SHAPE;
    if (N == 0) return ROD_OK;
    if (!q || !k_new || !v_new || !k_cache || !v_cache || !pos || !o) return ROD_ERR_NULL;
    if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) ||
        !aligned16(v_cache) || !aligned16(pos) || !aligned16(o))
        return ROD_ERR_ALIGN;
    return from_cuda(rod::swska_decode_launch(q, k_new, v_new, k_cache, v_cache, pos, o, N, H, dk,
                                              dv, window, resolve_scale(scale, dk),
                                              dtype == ROD_BF16,
                                              static_cast<cudaStream_t>(stream)));
}

size_t rod_gla_backward_workspace_size(int B, int H, int T, int dk, int dv) {
    if (B < 0 || H < 0 || T < 0 || !dim_ok(dk) || !dim_ok(dv)) return 0;
    // the size does not depend on dtype: enough for either route (tensor cores for bf16 at
    // d = 128, CUDA cores otherwise)
    size_t need = rod::gla_backward_workspace_size(B, H, T, dk, dv);
    if (rod::gla_backward_tc_supported(dk, dv)) {
        const size_t tc = rod::gla_backward_tc_workspace_size(B, H, T);
        if (tc > need) need = tc;
    }
    return need;
}

int rod_gla_backward(const void* q, const void* k, const void* v, const float* g, const float* state0,
                     const void* dO, const float* dstate_final, void* dq, void* dk, void* dv, float* dg,
                     float* dstate0, int B, int H, int T, int dk_dim, int dv_dim, int dtype,
                     void* workspace, size_t ws_bytes, void* stream) {
    if (!dtype_ok(dtype)) return ROD_ERR_DTYPE;
    if (B < 0 || H < 0 || T < 0 || !dim_ok(dk_dim) || !dim_ok(dv_dim)) return ROD_ERR_SHAPE;
    if ((int64_t)B * H == 0) return ROD_OK;
    if (!state0 || !dstate0) return ROD_ERR_NULL;
    if (!aligned16(state0) || !aligned16(dstate0) || (dstate_final && !aligned16(dstate_final)))
        return ROD_ERR_ALIGN;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t state_bytes = (size_t)B * H * dk_dim * dv_dim * sizeof(float);
    if (T == 0) {  // nothing in between: the initial state's gradient is the final state's
        return from_cuda(dstate_final
                             ? cudaMemcpyAsync(dstate0, dstate_final, state_bytes, cudaMemcpyDeviceToDevice, s)
                             : cudaMemsetAsync(dstate0, 0, state_bytes, s));
    }
    if (!q || !k || !v || !g || !dO || !dq || !dk || !dv || !dg) return ROD_ERR_NULL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) || !aligned16(dO) ||
        !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(dg))
        return ROD_ERR_ALIGN;
    const bool tc = dtype == ROD_BF16 && rod::gla_backward_tc_supported(dk_dim, dv_dim);
    const size_t need = tc ? rod::gla_backward_tc_workspace_size(B, H, T)
                           : rod::gla_backward_workspace_size(B, H, T, dk_dim, dv_dim);
    if (!workspace || ws_bytes < need) return ROD_ERR_WORKSPACE;
    if (!aligned16(workspace)) return ROD_ERR_ALIGN;
    rod::GlaBackwardArgs a{q, k, v, g, state0, dO, dstate_final, dq, dk, dv, dg, dstate0,
                           B, H, T, dk_dim, dv_dim, workspace};
    // bf16 with 128-wide heads runs the chunkwise tensor-core backward; fp32 (exact FMA) and
    // the other head dims run the step-by-step CUDA-core sweeps
    if (tc) return from_cuda(rod::gla_backward_tc_launch(a, s));
    return from_cuda(rod::gla_backward_launch(a, dtype == ROD_BF16, s));
}

size_t rod_swska_backward_workspace_size(int B, int H, int T) {
    if (B < 0 || H < 0 || T < 0) return 0;
    return rod::swska_backward_workspace_size(B, H, T);
}

int rod_swska_backward(const void* q, const void* k, const void* v, const void* dO, void* dq, void* dk,
                       void* dv, int B, int H, int T, int dk_dim, int dv_dim, int window, float scale,
                       int dtype, void* workspace, size_t ws_bytes, void* stream) {
    if (!dtype_ok(dtype)) return ROD_ERR_DTYPE;
    if (B < 0 || H < 0 || T < 0 || H > 64 || window < 1 || !dim_ok(dk_dim) || !dim_ok(dv_dim))
        return ROD_ERR_SHAPE;
    if (!(scale == scale) || isinf(scale)) return ROD_ERR_SHAPE;
    if ((int64_t)B * H == 0 || T == 0) return ROD_OK;
    if (!q || !k || !v || !dO || !dq || !dk || !dv) return ROD_ERR_NULL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dO) || !aligned16(dq) ||
        !aligned16(dk) || !aligned16(dv))
        return ROD_ERR_ALIGN;
    if (!workspace || ws_bytes < rod::swska_backward_workspace_size(B, H, T)) return ROD_ERR_WORKSPACE;
    if (!aligned16(workspace)) return ROD_ERR_ALIGN;
    rod::SkaBackwardArgs a{q, k, v, dO, dq, dk, dv, B, H, T, dk_dim, dv_dim, window,
                           resolve_scale(scale, dk_dim), workspace};
    return from_cuda(rod::swska_backward_launch(a, dtype == ROD_BF16, static_cast<cudaStream_t>(stream)));
}

int rod_swska_backward_lse(const void* q, const void* k, const void* v, const void* o, const float* lse,
                           const void* dO, void* dq, void* dk, void* dv, int B, int H, int T, int dk_dim,
                           int dv_dim, int window, float scale, int dtype, void* workspace, size_t ws_bytes,
                           void* stream) {
    if (!dtype_ok(dtype)) return ROD_ERR_DTYPE;
    if (B < 0 || H < 0 || T < 0 || H > 64 || window < 1 || !dim_ok(dk_dim) || !dim_ok(dv_dim))
        return ROD_ERR_SHAPE;
    if (!(scale == scale) || isinf(scale)) return ROD_ERR_SHAPE;
    if ((int64_t)B * H == 0 || T == 0) return ROD_OK;
    if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv) return ROD_ERR_NULL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || reinterpret_cast<uintptr_t>(lse) % 4 ||
        !aligned16(dO) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
        return ROD_ERR_ALIGN;
    if (!workspace || ws_bytes < rod::swska_backward_workspace_size(B, H, T)) return ROD_ERR_WORKSPACE;
    if (!aligned16(workspace)) return ROD_ERR_ALIGN;
    rod::SkaBackwardArgs a{q, k, v, dO, dq, dk, dv, B, H, T, dk_dim, dv_dim, window,
                           resolve_scale(scale, dk_dim), workspace, o, lse};
    return from_cuda(rod::swska_backward_launch(a, dtype == ROD_BF16, static_cast<cudaStream_t>(stream)));
}

int rod_swska_decode_paged(const void* q, const void* k_new, const void* v_new, void* k_pool,
                           void* v_pool, const int32_t* block_table, int page_size, int pages_per_seq,
                           const int64_t* pos, void* o, int N, int H, int dk, int dv, int window,
                           float scale, int dtype, void* stream) {
    if (!dtype_ok(dtype)) return ROD_ERR_DTYPE;
    if (dtype != ROD_BF16) return ROD_ERR_DTYPE;
    if (N < 0 || !rod::swska_decode_warp_supported(H, dk, dv) || page_size < 8 || page_size % 8 != 0 ||
        pages_per_seq < 1 || pages_per_seq > ROD_MAX_PAGES_PER_SEQ || window < 1 ||
        (int64_t)page_size * pages_per_seq != window)
        return ROD_ERR_SHAPE;
    if (!(scale == scale) || isinf(scale)) return ROD_ERR_SHAPE;
    if (N == 0) return ROD_OK;
    if (!q || !k_new || !v_new || !k_pool || !v_pool || !block_table || !pos || !o) return ROD_ERR_NULL;
    if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(k_pool) ||
        !aligned16(v_pool) || !aligned16(pos) || !aligned16(o) ||
        (reinterpret_cast<uintptr_t>(block_table) & 3u) != 0)
        return ROD_ERR_ALIGN;
    return from_cuda(rod::swska_decode_paged_launch(q, k_new, v_new, k_pool, v_pool, block_table,
                                                    page_size, pages_per_seq, pos, o, N, H, window,
                                                    resolve_scale(scale, dk),
                                                    static_cast<cudaStream_t>(stream)));
}

int rod_swska_cache_fill(const void* k, const void* v, void* k_cache, void* v_cache, int B, int H,
                         int T, int dk, int dv, int window, int dtype, void* stream) {
    if (!dtype_ok(dtype)) return ROD_ERR_DTYPE;
    if (B < 0 || H < 1 || H > 64 || T < 0 || window < 1 || !dim_ok(dk) || !dim_ok(dv))
        return ROD_ERR_SHAPE;
    if (B == 0 || T == 0) return ROD_OK;
    if (!k || !v || !k_cache || !v_cache) return ROD_ERR_NULL;
    if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache))
        return ROD_ERR_ALIGN;
    return from_cuda(rod::swska_cache_fill_launch(k, v, k_cache, v_cache, B, H, T, dk, dv, window,
                                                  dtype == ROD_BF16 ? 2 : 4,
                                                  static_cast<cudaStream_t>(stream)));
}

static bool scale_ok(float s) { return s > 0.f && !isinf(s) && s == s; }

int rod_swska_decode_fp8(const void* q, const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                         const int64_t* pos, void* o, int N, int H, int dk, int dv, int window, float scale,
                         float k_scale, float v_scale, void* stream) {
    if (N < 0 || !rod::swska_decode_warp_supported(H, dk, dv) || window < 1) return ROD_ERR_SHAPE;
    if (!(scale == scale) || isinf(scale) || !scale_ok(k_scale) || !scale_ok(v_scale)) return ROD_ERR_SHAPE;
    if (N == 0) return ROD_OK;
    if (!q || !k_new || !v_new || !k_cache || !v_cache || !pos || !o) return ROD_ERR_NULL;
    if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) ||
        !aligned16(v_cache) || !aligned16(pos) || !aligned16(o))
        return ROD_ERR_ALIGN;
    return from_cuda(rod::swska_decode_fp8_launch(q, k_new, v_new, k_cache, v_cache, pos, o, N, H, window,
                                                  resolve_scale(scale, dk), k_scale, v_scale,
                                                  static_cast<cudaStream_t>(stream)));
}

int rod_swska_cache_fill_fp8(const void* k, const void* v, void* k_cache, void* v_cache, int B, int H, int T,
                             int dk, int dv, int window, float k_scale, float v_scale, void* stream) {
    if (B < 0 || T < 0 || window < 1 || !rod::swska_decode_warp_supported(H, dk, dv)) return ROD_ERR_SHAPE;
    if (!scale_ok(k_scale) || !scale_ok(v_scale)) return ROD_ERR_SHAPE;
    if (B == 0 || T == 0) return ROD_OK;
    if (!k || !v || !k_cache || !v_cache) return ROD_ERR_NULL;
    if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache)) return ROD_ERR_ALIGN;
    return from_cuda(rod::swska_cache_fill_fp8_launch(k, v, k_cache, v_cache, B, H, T, dk, dv, window, k_scale,
                                                      v_scale, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
