// gla_prefill_recurrent.cu -- prefill of the Rodimus gated linear recurrence in its
// sequential-in-time form, on CUDA cores with fp32 FMA.
//
//   S_t = diag(g_t) S_{t-1} + k_t^T v_t,   o_t = q_t S_t     (CodeFuse Rodimus* article,
//   Rodimus block: fixed-size state updated recurrently; SALA blog §2.2 state form, §4.3
//   decay of the old state)
//
// This is the exact-fp32 instantiation used for ROD_FP32 inputs (every product an fp32 FMA;
// no tensor-core rounding), so the fp32 path meets a 1e-4 relative bound. One CTA owns one
// (batch, head) and one slice of DVS state columns; thread j keeps column j of S (dk values)
// in registers for the whole sequence, so the state never leaves the SM. Tokens are staged
// through shared memory TT at a time. The readout sum over dk uses four independent partial
// sums to shorten the dependent FMA chain.
#include "common.cuh"
#include "kernels.h"

namespace rod {
namespace {

constexpr int TT = 16;  // tokens staged per shared-memory tile

template <typename T, int DK>
__global__ void __launch_bounds__(128)
gla_prefill_rec_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                       const float* __restrict__ g, float* __restrict__ state, T* __restrict__ o,
                       int T_len, int dv) {
    __shared__ __align__(16) float s_q[TT][DK], s_k[TT][DK], s_g[TT][DK];
    const int ncb = (dv + blockDim.x - 1) / blockDim.x;   // column blocks per (batch, head)
    const int64_t bh = blockIdx.x / ncb;
    const int j = (blockIdx.x % ncb) * blockDim.x + threadIdx.x;  // state column of this thread
    const bool live = j < dv;
    const int64_t tok0 = bh * (int64_t)T_len;

    float S[DK];
    float* Sg = state + bh * (int64_t)DK * dv;
#pragma unroll
    for (int c = 0; c < DK; ++c) S[c] = live ? Sg[(size_t)c * dv + j] : 0.f;

    for (int t0 = 0; t0 < T_len; t0 += TT) {
        const int nt = T_len - t0 < TT ? T_len - t0 : TT;
        __syncthreads();
        for (int i = threadIdx.x; i < nt * DK; i += blockDim.x) {
            const int tt = i / DK, c = i % DK;
            const int64_t idx = (tok0 + t0 + tt) * DK + c;
            s_q[tt][c] = to_f32(q[idx]);
            s_k[tt][c] = to_f32(k[idx]);
            s_g[tt][c] = g[idx];
        }
        __syncthreads();
        for (int tt = 0; tt < nt; ++tt) {
            const float vj = live ? to_f32(v[(tok0 + t0 + tt) * dv + j]) : 0.f;
            float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
            for (int c = 0; c < DK; c += 4) {
                const float4 gg = *reinterpret_cast<const float4*>(&s_g[tt][c]);
                const float4 kk = *reinterpret_cast<const float4*>(&s_k[tt][c]);
                const float4 qq = *reinterpret_cast<const float4*>(&s_q[tt][c]);
                S[c + 0] = fmaf(gg.x, S[c + 0], kk.x * vj);
                S[c + 1] = fmaf(gg.y, S[c + 1], kk.y * vj);
                S[c + 2] = fmaf(gg.z, S[c + 2], kk.z * vj);
                S[c + 3] = fmaf(gg.w, S[c + 3], kk.w * vj);
                a0 = fmaf(qq.x, S[c + 0], a0);
                a1 = fmaf(qq.y, S[c + 1], a1);
                a2 = fmaf(qq.z, S[c + 2], a2);
                a3 = fmaf(qq.w, S[c + 3], a3);
            }
            if (live) o[(tok0 + t0 + tt) * dv + j] = from_f32<T>((a0 + a1) + (a2 + a3));
        }
    }
    if (live) {
#pragma unroll
        for (int c = 0; c < DK; ++c) Sg[(size_t)c * dv + j] = S[c];
    }
}

template <typename T, int DK>
cudaError_t launch_t(const void* q, const void* k, const void* v, const float* g, float* state,
                     void* o, int B, int H, int T_len, int dv, cudaStream_t s) {
    const int threads = dv < 128 ? 32 * ((dv + 31) / 32) : 128;
    const int64_t ncb = (dv + threads - 1) / threads;
    dim3 grid((unsigned)(ncb * B * H));
    gla_prefill_rec_kernel<T, DK><<<grid, threads, 0, s>>>(
        static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), g, state,
        static_cast<T*>(o), T_len, dv);
    note_launches(1);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_dk(int dk, const void* q, const void* k, const void* v, const float* g,
                      float* state, void* o, int B, int H, int T_len, int dv, cudaStream_t s) {
    switch (dk) {
        case 16: return launch_t<T, 16>(q, k, v, g, state, o, B, H, T_len, dv, s);
        case 32: return launch_t<T, 32>(q, k, v, g, state, o, B, H, T_len, dv, s);
        case 64: return launch_t<T, 64>(q, k, v, g, state, o, B, H, T_len, dv, s);
        case 128: return launch_t<T, 128>(q, k, v, g, state, o, B, H, T_len, dv, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t gla_prefill_recurrent_launch(const void* q, const void* k, const void* v,
                                         const float* g, float* state, void* o, int B, int H,
                                         int T, int dk, int dv, bool bf16, cudaStream_t stream) {
    if ((int64_t)B * H == 0 || T == 0) return cudaSuccess;
    if ((int64_t)B * H * 8 > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    return bf16 ? launch_dk<__nv_bfloat16>(dk, q, k, v, g, state, o, B, H, T, dv, stream)
                : launch_dk<float>(dk, q, k, v, g, state, o, B, H, T, dv, stream);
}

}  // namespace rod
