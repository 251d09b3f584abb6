// swska_backward.cu -- backward of SW-SKA prefill on CUDA cores (fp32 arithmetic).
//
// Forward (CodeFuse Rodimus* article, Fig. 4 / SKA paragraph: one K shared by all heads,
// per-head V; setup blog §3: a window of the most recent W tokens):
//   s_tj = scale q_t . k_j (j in [t-W+1, t]),  p_t = softmax(s_t),  o_t = sum_j p_tj v_j.
// For the loss gradient dO of every output row:
//   D_t = dO_t . o_t = sum_j p_tj (dO_t . v_j),   dS_tj = p_tj (dO_t . v_j - D_t)
//   dq_t = scale sum_j dS_tj k_j,   dv_j = sum_t p_tj dO_t (per head),
//   dk_j = scale sum_h sum_t dS_tj q_t (the shared key gathers every head's contribution).
// Two kernels, lanes of a warp spread over the channels (lane l: channels l, l+32, ...):
//   1. one warp per query row (b, h, t): the row's base-2 log-sum-exp and D_t in one online
//      pass over its window, stored for kernel 2, then dq_t in a second pass;
//   2. one warp per key position (b, j): for every head, the queries t in [j, j+W-1] that see
//      it give dv_j of that head and their share of dk_j, which is complete when the warp has
//      gone through all heads (no atomics).
// These kernels serve fp32 inputs and head dims other than 128 (every dot product in fp32);
// bf16 with head dim 128 runs on the tensor cores (swska_backward_tc.cu).
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace rod {
namespace {

constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
}

template <typename T, int N>
__device__ __forceinline__ void load_row(const T* row, int d, int lane, float* r) {
#pragma unroll
    for (int i = 0; i < N; ++i) {
        const int c = lane + 32 * i;
        r[i] = c < d ? to_f32(row[c]) : 0.f;
    }
}

template <int N>
__device__ __forceinline__ float dot_part(const float* a, const float* b) {
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < N; ++i) s = fmaf(a[i], b[i], s);
    return s;
}

// ---- kernel 1: per query row --------------------------------------------------------------
template <typename T, int NK, int NV>
__global__ void __launch_bounds__(256)
ska_bwd_rows(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
             const T* __restrict__ dO, T* __restrict__ dq, float* __restrict__ lse2,
             float* __restrict__ Dbuf, int64_t n_rows, int H, int T_len, int dk, int dv, int W,
             float scale) {
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);  // (b h) * T + t
    if (row >= n_rows) return;  // whole warp: the grid is rounded up to full blocks
    const int64_t bh = row / T_len;
    const int t = (int)(row % T_len);
    const int64_t b = bh / H;
    float qr[NK], dor[NV];
    load_row<T, NK>(q + row * dk, dk, lane, qr);
    load_row<T, NV>(dO + row * dv, dv, lane, dor);
    const float sl = scale * kLog2e;
    const int j0 = t - W + 1 > 0 ? t - W + 1 : 0;
    // pass 1: base-2 log-sum-exp of the row and D_t, online over the window
    float m = -INFINITY, l = 0.f, Dacc = 0.f;
    for (int j = j0; j <= t; ++j) {
        float kr[NK], vr[NV];
        load_row<T, NK>(k + (b * T_len + j) * dk, dk, lane, kr);
        load_row<T, NV>(v + (bh * T_len + j) * dv, dv, lane, vr);
        const float s = warp_sum(dot_part<NK>(qr, kr)) * sl;
        const float dp = warp_sum(dot_part<NV>(dor, vr));
        if (s > m) {
            const float alpha = exp2f(m - s);  // m = -inf gives 0
            l *= alpha;
            Dacc *= alpha;
            m = s;
        }
        const float p = exp2f(s - m);
        l += p;
        Dacc = fmaf(p, dp, Dacc);
    }
    const float L2 = m + log2f(l), D = Dacc / l;
    if (lane == 0) {
        lse2[row] = L2;
        Dbuf[row] = D;
    }
    // pass 2: dq_t = scale sum_j p_tj (dO_t . v_j - D_t) k_j
    float acc[NK];
#pragma unroll
    for (int i = 0; i < NK; ++i) acc[i] = 0.f;
    for (int j = j0; j <= t; ++j) {
        float kr[NK], vr[NV];
        load_row<T, NK>(k + (b * T_len + j) * dk, dk, lane, kr);
        load_row<T, NV>(v + (bh * T_len + j) * dv, dv, lane, vr);
        const float p = exp2f(warp_sum(dot_part<NK>(qr, kr)) * sl - L2);
        const float dS = p * (warp_sum(dot_part<NV>(dor, vr)) - D);
#pragma unroll
        for (int i = 0; i < NK; ++i) acc[i] = fmaf(dS, kr[i], acc[i]);
    }
#pragma unroll
    for (int i = 0; i < NK; ++i) {
        const int c = lane + 32 * i;
        if (c < dk) dq[row * dk + c] = from_f32<T>(acc[i] * scale);
    }
}

// ---- kernel 2: per key position -------------------------------------------------------------
template <typename T, int NK, int NV>
__global__ void __launch_bounds__(256)
ska_bwd_keys(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
             const T* __restrict__ dO, const float* __restrict__ lse2, const float* __restrict__ Dbuf,
             T* __restrict__ dkout, T* __restrict__ dvout, int64_t n_keys, int H, int T_len, int dk,
             int dv, int W, float scale) {
    const int lane = threadIdx.x & 31;
    const int64_t key = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);  // b * T + j
    if (key >= n_keys) return;  // whole warp
    const int64_t b = key / T_len;
    const int j = (int)(key % T_len);
    const float sl = scale * kLog2e;
    const int t1 = j + W - 1 < T_len - 1 ? j + W - 1 : T_len - 1;  // queries j .. t1 see key j
    float kr[NK], dk_acc[NK];
    load_row<T, NK>(k + key * dk, dk, lane, kr);
#pragma unroll
    for (int i = 0; i < NK; ++i) dk_acc[i] = 0.f;
    for (int h = 0; h < H; ++h) {
        const int64_t bh = b * H + h;
        float vr[NV], dv_acc[NV];
        load_row<T, NV>(v + (bh * T_len + j) * dv, dv, lane, vr);
#pragma unroll
        for (int i = 0; i < NV; ++i) dv_acc[i] = 0.f;
        for (int t = j; t <= t1; ++t) {
            const int64_t row = bh * T_len + t;
            float qr[NK], dor[NV];
            load_row<T, NK>(q + row * dk, dk, lane, qr);
            load_row<T, NV>(dO + row * dv, dv, lane, dor);
            const float p = exp2f(warp_sum(dot_part<NK>(qr, kr)) * sl - lse2[row]);
            const float dS = p * (warp_sum(dot_part<NV>(dor, vr)) - Dbuf[row]);
#pragma unroll
            for (int i = 0; i < NK; ++i) dk_acc[i] = fmaf(dS, qr[i], dk_acc[i]);
#pragma unroll
            for (int i = 0; i < NV; ++i) dv_acc[i] = fmaf(p, dor[i], dv_acc[i]);
        }
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            const int c = lane + 32 * i;
            if (c < dv) dvout[(bh * T_len + j) * dv + c] = from_f32<T>(dv_acc[i]);
        }
    }
#pragma unroll
    for (int i = 0; i < NK; ++i) {
        const int c = lane + 32 * i;
        if (c < dk) dkout[key * dk + c] = from_f32<T>(dk_acc[i] * scale);
    }
}

template <typename T, int NK, int NV>
cudaError_t launch_t(const SkaBackwardArgs& a, cudaStream_t s) {
    constexpr int WARPS = 8;
    float* lse2 = static_cast<float*>(a.workspace);
    float* Dbuf = lse2 + (size_t)a.B * a.H * a.T;
    const int64_t rows = (int64_t)a.B * a.H * a.T, keys = (int64_t)a.B * a.T;
    ska_bwd_rows<T, NK, NV><<<(unsigned)((rows + WARPS - 1) / WARPS), 32 * WARPS, 0, s>>>(
        static_cast<const T*>(a.q), static_cast<const T*>(a.k), static_cast<const T*>(a.v),
        static_cast<const T*>(a.dO), static_cast<T*>(a.dq), lse2, Dbuf, rows, a.H, a.T, a.d_k, a.d_v,
        a.W, a.scale);
    ska_bwd_keys<T, NK, NV><<<(unsigned)((keys + WARPS - 1) / WARPS), 32 * WARPS, 0, s>>>(
        static_cast<const T*>(a.q), static_cast<const T*>(a.k), static_cast<const T*>(a.v),
        static_cast<const T*>(a.dO), lse2, Dbuf, static_cast<T*>(a.dk), static_cast<T*>(a.dv), keys,
        a.H, a.T, a.d_k, a.d_v, a.W, a.scale);
    note_launches(2);
    return cudaGetLastError();
}

template <typename T, int NK>
cudaError_t launch_nv(const SkaBackwardArgs& a, cudaStream_t s) {
    switch ((a.d_v + 31) / 32) {
        case 1: return launch_t<T, NK, 1>(a, s);
        case 2: return launch_t<T, NK, 2>(a, s);
        case 4: return launch_t<T, NK, 4>(a, s);
    }
    return cudaErrorInvalidValue;
}

template <typename T>
cudaError_t launch_nk(const SkaBackwardArgs& a, cudaStream_t s) {
    switch ((a.d_k + 31) / 32) {
        case 1: return launch_nv<T, 1>(a, s);
        case 2: return launch_nv<T, 2>(a, s);
        case 4: return launch_nv<T, 4>(a, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

size_t swska_backward_workspace_size(int B, int H, int T) {
    // the tensor-core path's need covers the 2 B H T floats used here
    return swska_backward_tc_workspace_size(B, H, T);
}

cudaError_t swska_backward_launch(const SkaBackwardArgs& a, bool bf16, cudaStream_t stream) {
    if ((int64_t)a.B * a.H == 0 || a.T == 0) return cudaSuccess;
    if (bf16 && swska_backward_tc_supported(a.H, a.T, a.d_k, a.d_v)) return swska_backward_tc_launch(a, stream);
    return bf16 ? launch_nk<__nv_bfloat16>(a, stream) : launch_nk<float>(a, stream);
}

}  // namespace rod
