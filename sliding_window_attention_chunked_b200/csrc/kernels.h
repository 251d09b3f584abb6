// kernels.h -- internal launch interface between the C ABI (rod_api.cu) and the kernels.
// Every launcher validates nothing (rod_api.cu has done it), enqueues on `stream` and
// returns the launch status.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace rod {

// host-side count of kernel launches enqueued by this library (reported by rod_launch_count)
void note_launches(unsigned n);

// gated linear recurrence, one decode step (fused, HBM-bound)
cudaError_t gla_decode_launch(const void* q, const void* k, const void* v, const float* g,
                              float* state, void* o, int N, int H, int dk, int dv, bool bf16,
                              cudaStream_t stream);

// gated linear recurrence prefill, sequential-in-time form on CUDA cores (exact fp32 FMA)
cudaError_t gla_prefill_recurrent_launch(const void* q, const void* k, const void* v,
                                         const float* g, float* state, void* o, int B, int H,
                                         int T, int dk, int dv, bool bf16, cudaStream_t stream);

// chunkwise gated-recurrence prefill on tcgen05 tensor cores (bf16, dk = dv = 128, chunk 64)
bool gla_prefill_tc_supported(int dk, int dv, int chunk);
size_t gla_prefill_tc_workspace_size(int B, int H, int T);
cudaError_t gla_prefill_tc_launch(const void* q, const void* k, const void* v, const float* g,
                                  float* state, void* o, int B, int H, int T, void* workspace,
                                  cudaStream_t stream);
unsigned gla_prefill_tc_take_timeout_flag();
// test only: the next gla_prefill_tc_launch runs with `probes` as its wait limit and issues no
// copies, so that its bounded waits expire (probes = 0 disarms)
void gla_prefill_tc_arm_wait_expiry(uint32_t probes);

// SW-SKA prefill on CUDA cores (fp32 FMA, online softmax); lse (optional, [B,H,T] fp32): the
// natural log-sum-exp of each row's scaled scores
cudaError_t swska_prefill_simt_launch(const void* q, const void* k, const void* v, void* o,
                                      int B, int H, int T, int dk, int dv, int window,
                                      float scale, bool bf16, cudaStream_t stream, float* lse = nullptr);

// SW-SKA prefill on tcgen05 tensor cores (bf16, dk = dv = 128, T >= 128)
bool swska_prefill_tc_supported(int H, int T, int dk, int dv);
cudaError_t swska_prefill_tc_launch(const void* q, const void* k, const void* v, void* o, int B,
                                    int H, int T, int window, float scale, cudaStream_t stream);
unsigned swska_prefill_tc_take_timeout_flag();
// the same kernel with per-row statistics: lse_mul * (base-2 log-sum-exp) into row bh * Tpad + t
// of `lse` (-1 gives the backward's negated base-2 form, ln 2 the natural log-sum-exp; rows past
// T, up to Tpad, get -inf) and, with dO given, D = dO . o into the same row of dbuf. o may be
// null (the output is then not stored), and so may dO and dbuf.
cudaError_t swska_prefill_tc_stats_launch(const void* q, const void* k, const void* v, void* o,
                                          const void* dO, float* lse, float* dbuf, int64_t Tpad, int B,
                                          int H, int T, int window, float scale, cudaStream_t stream,
                                          float lse_mul = -1.f);


// TMA descriptors for a 3-D tensor [d2][d1][d0] loaded as boxes of box1 x box0 elements
cudaError_t make_tmap_3d(CUtensorMap* map, const void* base, bool fp32, uint64_t d0, uint64_t d1,
                         uint64_t d2, uint32_t box0, uint32_t box1, bool swizzle128);
cudaError_t make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1,
                              uint64_t d2, uint32_t box0, uint32_t box1);

// SW-SKA decode: ring-buffer write + split-window attention combined across a cluster
cudaError_t swska_decode_launch(const void* q, const void* k_new, const void* v_new,
                                void* k_cache, void* v_cache, const int64_t* pos, void* o,
                                int N, int H, int dk, int dv, int window, float scale, bool bf16,
                                cudaStream_t stream);
// read and clear the "bounded wait expired" flag of the decode attention kernel
unsigned swska_decode_take_timeout_flag();
// bf16, d_k = d_v = 128, H <= 16: one warp per head, producer warp, mbarrier ring
bool swska_decode_warp_supported(int H, int dk, int dv);
cudaError_t swska_decode_warp_launch(const void* q, const void* k_new, const void* v_new,
                                     void* k_cache, void* v_cache, const int64_t* pos, void* o,
                                     int N, int H, int window, float scale, cudaStream_t stream);
unsigned swska_decode_warp_take_timeout_flag();
// the same decode over a paged window cache (pools + block table)
cudaError_t swska_decode_paged_launch(const void* q, const void* k_new, const void* v_new, void* k_pool,
                                      void* v_pool, const int32_t* block_table, int page_size,
                                      int pages_per_seq, const int64_t* pos, void* o, int N, int H,
                                      int window, float scale, cudaStream_t stream);

// backward of the recurrence (CUDA cores): gradients of q, k, v, g and of the initial state
struct GlaBackwardArgs {
    const void *q, *k, *v;
    const float* g;
    const float* state0;        // [B,H,dk,dv]
    const void* dO;             // [B,H,T,dv]
    const float* dstate_final;  // [B,H,dk,dv] or nullptr
    void *dq, *dk, *dv;         // dtype
    float* dg;                  // [B,H,T,dk]
    float* dstate0;             // [B,H,dk,dv]
    int B, H, T, d_k, d_v;
    void* workspace;
};
size_t gla_backward_workspace_size(int B, int H, int T, int dk, int dv);
// the chunkwise tensor-core backward (bf16, d_k = d_v = 128): contributions, scans, gradients
bool gla_backward_tc_supported(int dk, int dv);
size_t gla_backward_tc_workspace_size(int B, int H, int T);
cudaError_t gla_backward_tc_launch(const GlaBackwardArgs& a, cudaStream_t stream);
unsigned gla_backward_tc_take_timeout_flag();

// backward of SW-SKA prefill: gradients of q, the shared k, and v (tensor cores for bf16 with
// head dim 128 and T >= 128, CUDA cores otherwise)
struct SkaBackwardArgs {
    const void *q, *k, *v, *dO;  // [B,H,T,dk], [B,T,dk], [B,H,T,dv], [B,H,T,dv]
    void *dq, *dk, *dv;          // same layouts as q, k, v
    int B, H, T, d_k, d_v, W;
    float scale;                 // resolved (> 0)
    void* workspace;             // swska_backward_workspace_size bytes, 16-byte aligned
    const void* o = nullptr;     // optional: the forward's output [B,H,T,dv] ...
    const float* lse = nullptr;  // ... and natural log-sum-exp [B,H,T]: the row statistics are then
                                 // taken from them instead of recomputing the forward
};
size_t swska_backward_workspace_size(int B, int H, int T);
cudaError_t swska_backward_launch(const SkaBackwardArgs& a, bool bf16, cudaStream_t stream);
size_t swska_backward_tc_workspace_size(int B, int H, int T);
bool swska_backward_tc_supported(int H, int T, int dk, int dv);
int swska_backward_tc_groups(int B, int H, int T);
cudaError_t swska_backward_tc_launch(const SkaBackwardArgs& a, cudaStream_t stream);
unsigned swska_backward_tc_take_timeout_flag();
cudaError_t gla_backward_launch(const GlaBackwardArgs& a, bool bf16, cudaStream_t stream);

// SW-SKA decode with FP8 (E4M3) ring caches: k_cache [N,W,128], v_cache [N,H,W,128] codes,
// value = code * scale; q, k_new, v_new, o bf16
cudaError_t swska_decode_fp8_launch(const void* q, const void* k_new, const void* v_new, void* k_cache,
                                    void* v_cache, const int64_t* pos, void* o, int N, int H, int window,
                                    float scale, float k_scale, float v_scale, cudaStream_t stream);
// hand-off into FP8 rings (bf16 prefill rows quantized as e4m3(x / scale))
cudaError_t swska_cache_fill_fp8_launch(const void* k, const void* v, void* k_cache, void* v_cache, int B,
                                        int H, int T, int dk, int dv, int window, float k_scale, float v_scale,
                                        cudaStream_t stream);

// SW-SKA prefill -> decode hand-off: the last W tokens' K / V rows into the ring buffers
cudaError_t swska_cache_fill_launch(const void* k, const void* v, void* k_cache, void* v_cache, int B,
                                    int H, int T, int dk, int dv, int window, size_t elem_bytes,
                                    cudaStream_t stream);

}  // namespace rod
