// swska_prefill_simt.cu -- SW-SKA prefill on CUDA cores (fp32 FMA, online softmax).
//
//   o[b,h,t] = sum_{j=max(0,t-W+1)}^{t} softmax_j(scale * q[b,h,t] . k[b,j]) v[b,h,j]
// (CodeFuse Rodimus* article, Fig. 4 / SKA paragraph: one key matrix shared by all heads,
// per-head values; setup blog §3: the window holds the most recent W tokens; SALA blog §2.1.)
//
// This is the exact-fp32 instantiation for ROD_FP32 inputs. A CTA owns BQ = 64 queries of
// one (batch, head); four threads share a query row, each holding a quarter of q (for the
// score, reduced with two shuffles) and a quarter of the output columns. Key tiles of BK
// keys covering the window of the CTA's rows are staged through shared memory as fp32; tiles
// outside every row's window are never visited. The softmax runs in base 2 on scores
// pre-scaled by scale*log2(e), with the running maximum rescaled once per group of 8 keys.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace rod {
namespace {

constexpr int BQ = 64;
constexpr int BK = 32;

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(256)
swska_prefill_simt_kernel(const T* __restrict__ q, const T* __restrict__ k,
                          const T* __restrict__ v, T* __restrict__ o, float* __restrict__ lse, int H,
                          int T_len, int W, float scale_log2) {
    constexpr int QP = DK / 4, VP = DV / 4;  // per-thread quarter of q and of the output
    __shared__ __align__(16) float sK[BK][DK];
    __shared__ __align__(16) float sV[BK][DV];
    const int qtiles = (T_len + BQ - 1) / BQ;
    const int64_t bh = blockIdx.x / qtiles;
    const int t0 = (int)(blockIdx.x % qtiles) * BQ;
    const int64_t b = bh / H;
    const int row = threadIdx.x / 4, part = threadIdx.x % 4;
    const int t = t0 + row;
    const bool live = t < T_len;

    float qr[QP];
    {
        const T* qp = q + (bh * T_len + (live ? t : 0)) * (int64_t)DK + part * QP;
#pragma unroll
        for (int c = 0; c < QP; ++c) qr[c] = live ? to_f32(qp[c]) * scale_log2 : 0.f;
    }
    float acc[VP];
#pragma unroll
    for (int i = 0; i < VP; ++i) acc[i] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;

    const int t_hi = (t0 + BQ < T_len ? t0 + BQ : T_len) - 1;
    const int k_lo = t0 - W + 1 > 0 ? t0 - W + 1 : 0;
    const T* kb = k + b * (int64_t)T_len * DK;
    const T* vb = v + bh * (int64_t)T_len * DV;

    for (int kt = (k_lo / BK) * BK; kt <= t_hi; kt += BK) {
        __syncthreads();
        for (int i = threadIdx.x; i < BK * DK; i += blockDim.x) {
            const int j = i / DK, c = i % DK;
            sK[j][c] = kt + j < T_len ? to_f32(kb[(int64_t)(kt + j) * DK + c]) : 0.f;
        }
        for (int i = threadIdx.x; i < BK * DV; i += blockDim.x) {
            const int j = i / DV, c = i % DV;
            sV[j][c] = kt + j < T_len ? to_f32(vb[(int64_t)(kt + j) * DV + c]) : 0.f;
        }
        __syncthreads();
        for (int j0 = 0; j0 < BK; j0 += 8) {
            float s[8];
            float gmax = -INFINITY;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int j = j0 + u, kj = kt + j;
                float d = 0.f;
#pragma unroll
                for (int c = 0; c < QP; ++c) d = fmaf(qr[c], sK[j][part * QP + c], d);
                d += __shfl_xor_sync(0xffffffffu, d, 1);
                d += __shfl_xor_sync(0xffffffffu, d, 2);
                const bool ok = live && kj <= t && kj >= t - W + 1;
                s[u] = ok ? d : -INFINITY;
                gmax = fmaxf(gmax, s[u]);
            }
            if (gmax > m_run) {
                const float alpha = exp2f(m_run - gmax);
                l_run *= alpha;
#pragma unroll
                for (int i = 0; i < VP; ++i) acc[i] *= alpha;
                m_run = gmax;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const float p = s[u] == -INFINITY ? 0.f : exp2f(s[u] - m_run);  // masked -> 0
                l_run += p;
#pragma unroll
                for (int i = 0; i < VP; ++i) acc[i] = fmaf(p, sV[j0 + u][part * VP + i], acc[i]);
            }
        }
    }
    if (live) {
        T* op = o + (bh * T_len + t) * (int64_t)DV + part * VP;
        const float inv = 1.f / l_run;
#pragma unroll
        for (int i = 0; i < VP; ++i) op[i] = from_f32<T>(acc[i] * inv);
        // natural log-sum-exp of the row's scaled scores: the base-2 one times ln 2
        if (lse != nullptr && part == 0) lse[bh * T_len + t] = (m_run + log2f(l_run)) * 0.6931471805599453f;
    }
}

template <typename T, int DK, int DV>
cudaError_t launch_t(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                     int T_len, int W, float scale, cudaStream_t s) {
    const int64_t qtiles = (T_len + BQ - 1) / BQ;
    const int64_t grid = qtiles * B * H;
    if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    swska_prefill_simt_kernel<T, DK, DV><<<(unsigned)grid, 256, 0, s>>>(
        static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v),
        static_cast<T*>(o), lse, H, T_len, W, scale * 1.4426950408889634f);
    note_launches(1);
    return cudaGetLastError();
}

template <typename T, int DK>
cudaError_t launch_dv(int dv, const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                      int T_len, int W, float scale, cudaStream_t s) {
    switch (dv) {
        case 16: return launch_t<T, DK, 16>(q, k, v, o, lse, B, H, T_len, W, scale, s);
        case 32: return launch_t<T, DK, 32>(q, k, v, o, lse, B, H, T_len, W, scale, s);
        case 64: return launch_t<T, DK, 64>(q, k, v, o, lse, B, H, T_len, W, scale, s);
        case 128: return launch_t<T, DK, 128>(q, k, v, o, lse, B, H, T_len, W, scale, s);
    }
    return cudaErrorInvalidValue;
}

template <typename T>
cudaError_t launch_dk(int dk, int dv, const void* q, const void* k, const void* v, void* o, float* lse, int B,
                      int H, int T_len, int W, float scale, cudaStream_t s) {
    switch (dk) {
        case 16: return launch_dv<T, 16>(dv, q, k, v, o, lse, B, H, T_len, W, scale, s);
        case 32: return launch_dv<T, 32>(dv, q, k, v, o, lse, B, H, T_len, W, scale, s);
        case 64: return launch_dv<T, 64>(dv, q, k, v, o, lse, B, H, T_len, W, scale, s);
        case 128: return launch_dv<T, 128>(dv, q, k, v, o, lse, B, H, T_len, W, scale, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t swska_prefill_simt_launch(const void* q, const void* k, const void* v, void* o,
                                      int B, int H, int T, int dk, int dv, int window,
                                      float scale, bool bf16, cudaStream_t stream, float* lse) {
    if ((int64_t)B * H == 0 || T == 0) return cudaSuccess;
    return bf16 ? launch_dk<__nv_bfloat16>(dk, dv, q, k, v, o, lse, B, H, T, window, scale, stream)
                : launch_dk<float>(dk, dv, q, k, v, o, lse, B, H, T, window, scale, stream);
}

}  // namespace rod
