// gla_decode.cu -- one decode step of the Rodimus gated linear recurrence, fused.
//
// Per (sequence n, head h), with the fixed-size state S [dk x dv] fp32 resident in HBM
// (CodeFuse Rodimus* article, Rodimus block: O(1)-space recurrent inference; SALA blog §3.3:
// the state is kept on the GPU and accumulated in place each step):
//     S[c][j] <- g[c] * S[c][j] + k[c] * v[j]          (in place)
//     o[j]     = sum_c q[c] * S_new[c][j]
// The step is bound by HBM: S is read once and written once (2 x 64 KB for 128 x 128), while
// q, k, v, g and o are a few hundred bytes. One CTA owns one (n, h) state; thread (rg, cg)
// owns float4 column group cg of rows rg, rg+RG, ...; a warp touches whole contiguous rows,
// so every access is a coalesced 128-bit load or store. All row loads are issued before any
// arithmetic so that each thread keeps DK/RG independent 16-byte loads in flight. The column
// sums of q * S_new are reduced across the RG row groups through shared memory. With few
// (n, h) pairs the columns are split over SPLIT CTAs (each column of o needs only its own column
// of S), so that more CTAs share the latency of the state's round trip.
#include "common.cuh"
#include "kernels.h"

namespace rod {
namespace {

template <typename T, int DK, int DV>
struct DecodeShape {                                    // DV: the columns one CTA handles
    static constexpr int TPC = DV / 4;                  // threads across the columns
    static constexpr int RG0 = 256 / TPC;
    static constexpr int RG = RG0 < DK ? RG0 : DK;      // row groups
    static constexpr int RPT = DK / RG;                 // rows per thread
    static constexpr int THREADS = TPC * RG;
};

// DV: the state's columns; DVC: the columns of this CTA (blockIdx.y selects which)
template <typename T, int DK, int DV, int DVC>
__global__ void __launch_bounds__(256)
gla_decode_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                  const float* __restrict__ g, float* __restrict__ state, T* __restrict__ o) {
    using Sh = DecodeShape<T, DK, DVC>;
    constexpr int TPC = Sh::TPC, RG = Sh::RG, RPT = Sh::RPT;
    __shared__ float s_q[DK], s_k[DK], s_g[DK];
    __shared__ float4 s_red[RG][TPC];

    const int64_t nh = blockIdx.x;
    const int tid = threadIdx.x;
    const int cg = tid % TPC, rg = tid / TPC;
    const int col0 = (int)blockIdx.y * DVC;
    float* S = state + nh * (int64_t)(DK * DV) + col0;

    float4 s4[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i)
        s4[i] = __ldcs(reinterpret_cast<const float4*>(S + (size_t)(rg + i * RG) * DV) + cg);

    for (int c = tid; c < DK; c += Sh::THREADS) {
        s_q[c] = to_f32(q[nh * DK + c]);
        s_k[c] = to_f32(k[nh * DK + c]);
        s_g[c] = g[nh * DK + c];
    }
    const float4 v4 = load4(v + nh * DV + col0 + 4 * cg);
    __syncthreads();

    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int r = rg + i * RG;
        const float gr = s_g[r], kr = s_k[r], qr = s_q[r];
        float4 s = s4[i];
        s.x = fmaf(gr, s.x, kr * v4.x);
        s.y = fmaf(gr, s.y, kr * v4.y);
        s.z = fmaf(gr, s.z, kr * v4.z);
        s.w = fmaf(gr, s.w, kr * v4.w);
        __stcs(reinterpret_cast<float4*>(S + (size_t)r * DV) + cg, s);
        acc.x = fmaf(qr, s.x, acc.x);
        acc.y = fmaf(qr, s.y, acc.y);
        acc.z = fmaf(qr, s.z, acc.z);
        acc.w = fmaf(qr, s.w, acc.w);
    }
    s_red[rg][cg] = acc;
    __syncthreads();
    if (rg == 0) {
        float4 tot = s_red[0][cg];
#pragma unroll
        for (int r = 1; r < RG; ++r) {
            const float4 p = s_red[r][cg];
            tot.x += p.x; tot.y += p.y; tot.z += p.z; tot.w += p.w;
        }
        store4(o + nh * DV + col0 + 4 * cg, tot);
    }
}

template <typename T, int DK, int DV, int DVC = DV>
cudaError_t launch_t(const void* q, const void* k, const void* v, const float* g, float* state,
                     void* o, int64_t NH, cudaStream_t stream) {
    using Sh = DecodeShape<T, DK, DVC>;
    gla_decode_kernel<T, DK, DV, DVC><<<dim3((unsigned)NH, DV / DVC), Sh::THREADS, 0, stream>>>(
        static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), g, state,
        static_cast<T*>(o));
    note_launches(1);
    return cudaGetLastError();
}

template <typename T, int DK>
cudaError_t launch_dv(int dv, const void* q, const void* k, const void* v, const float* g,
                      float* state, void* o, int64_t NH, cudaStream_t s) {
    switch (dv) {
        case 16: return launch_t<T, DK, 16>(q, k, v, g, state, o, NH, s);
        case 32: return launch_t<T, DK, 32>(q, k, v, g, state, o, NH, s);
        case 64: return launch_t<T, DK, 64>(q, k, v, g, state, o, NH, s);
        case 128:
            // few (n, h) pairs: the columns split over 4 or 2 CTAs (N 1, H 16, in CUDA graphs:
            // 2.79 -> 1.86 us; N 4: 2.85 -> 2.31 us)
            if (NH <= 64) return launch_t<T, DK, 128, 32>(q, k, v, g, state, o, NH, s);
            if (NH <= 128) return launch_t<T, DK, 128, 64>(q, k, v, g, state, o, NH, s);
            return launch_t<T, DK, 128>(q, k, v, g, state, o, NH, s);
    }
    return cudaErrorInvalidValue;
}

template <typename T>
cudaError_t launch_dk(int dk, int dv, const void* q, const void* k, const void* v,
                      const float* g, float* state, void* o, int64_t NH, cudaStream_t s) {
    switch (dk) {
        case 16: return launch_dv<T, 16>(dv, q, k, v, g, state, o, NH, s);
        case 32: return launch_dv<T, 32>(dv, q, k, v, g, state, o, NH, s);
        case 64: return launch_dv<T, 64>(dv, q, k, v, g, state, o, NH, s);
        case 128: return launch_dv<T, 128>(dv, q, k, v, g, state, o, NH, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t gla_decode_launch(const void* q, const void* k, const void* v, const float* g,
                              float* state, void* o, int N, int H, int dk, int dv, bool bf16,
                              cudaStream_t stream) {
    const int64_t NH = (int64_t)N * H;
    if (NH == 0) return cudaSuccess;
    if (NH > 0x7fffffffLL) return cudaErrorInvalidValue;
    return bf16 ? launch_dk<__nv_bfloat16>(dk, dv, q, k, v, g, state, o, NH, stream)
                : launch_dk<float>(dk, dv, q, k, v, g, state, o, NH, stream);
}

}  // namespace rod
