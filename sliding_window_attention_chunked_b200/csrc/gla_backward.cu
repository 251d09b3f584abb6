// gla_backward.cu -- backward of the Rodimus gated linear recurrence on CUDA cores (fp32 FMA).
//
// Forward (CodeFuse Rodimus* article, Rodimus block; the chunkwise-parallel algorithm is stated
// for training as well as prefill):  S_t = diag(g_t) S_{t-1} + k_t^T v_t,  o_t = q_t S_t.
// Given dO_t (gradient of every o_t) and dS_T (gradient of the final state, may be absent):
//   dq_t[c] = sum_j dO_t[j] S_t[c][j]
//   dS_t    = q_t^T dO_t + diag(g_{t+1}) dS_{t+1}            (reverse in time, from dS_T)
//   dk_t[c] = sum_j dS_t[c][j] v_t[j],   dv_t[j] = sum_c dS_t[c][j] k_t[c]
//   dg_t[c] = sum_j dS_t[c][j] S_{t-1}[c][j],   d(initial state) = diag(g_1) dS_1.
// Three sweeps per (batch, head), each keeping a state in registers for the whole sequence:
//   1. forward, thread c = state row c: dq, checkpoints of S every 16 steps (stored transposed,
//      element (j, c) at stride 1 in c, so the threads' accesses coalesce);
//   2. reverse, thread c = gradient-state row c: per block of 16 steps the states S_{t-1} are
//      recomputed from the block's checkpoint into a scratch (the forward rows live in padded
//      shared memory meanwhile), then the block is walked backwards for dk, dg and the
//      propagation of dS; the last dS is the initial-state gradient;
//   3. reverse, thread j = gradient-state column j: dv.
// This is the correctness-first form of the training path: O(T d^2) FMAs per (batch, head) in
// sequence, every product in fp32.
#include "common.cuh"
#include "kernels.h"

namespace rod {
namespace {

// Steps between checkpoints. The reverse sweep writes and reads back the BLK states of the
// block it walks (BLK x 64 KB per (batch, head) at d = 128): 16 keeps that scratch in L2 for
// 64 concurrent (batch, head) pairs (with 64 steps it spilled to DRAM: 31 GB of traffic at
// B4 H16 T4096 and 37 ms of the 49 ms backward).
constexpr int BLK = 16;
constexpr int TT = 16;   // tokens staged per shared-memory tile

// workspace per (batch, head): checkpoints [nblk][DV][DK] (state before each block's first
// step), then the block scratch [BLK][DV][DK] (states S_{t-1} of the block being walked)
__host__ __device__ inline size_t ckpt_floats(int T, int dk, int dv) {
    return (size_t)((T + BLK - 1) / BLK) * dk * dv;
}
__host__ __device__ inline size_t per_bh_floats(int T, int dk, int dv) {
    return ckpt_floats(T, dk, dv) + (size_t)BLK * dk * dv;
}

// ---- sweep 1: forward, rows --------------------------------------------------------------
template <typename T, int DK, int DV>
__global__ void __launch_bounds__(128)
gla_bwd_fwd_rows(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                 const float* __restrict__ g, const float* __restrict__ state0, const T* __restrict__ dO,
                 T* __restrict__ dq, float* __restrict__ ws, int T_len) {
    __shared__ __align__(16) float s_v[TT][DV], s_do[TT][DV];
    const int64_t bh = blockIdx.x;
    const int c = threadIdx.x;
    const bool live = c < DK;
    float* ckpt = ws + bh * per_bh_floats(T_len, DK, DV);
    float S[DV];
#pragma unroll
    for (int j = 0; j < DV; ++j) S[j] = live ? state0[(bh * DK + c) * DV + j] : 0.f;
    for (int t0 = 0; t0 < T_len; t0 += TT) {
        const int nt = T_len - t0 < TT ? T_len - t0 : TT;
        __syncthreads();
        for (int i = threadIdx.x; i < nt * DV; i += blockDim.x) {
            const int tt = i / DV, j = i % DV;
            const int64_t idx = (bh * T_len + t0 + tt) * DV + j;
            s_v[tt][j] = to_f32(v[idx]);
            s_do[tt][j] = to_f32(dO[idx]);
        }
        __syncthreads();
        for (int tt = 0; tt < nt; ++tt) {
            const int t = t0 + tt;
            if (t % BLK == 0 && live) {
                float* dst = ckpt + (size_t)(t / BLK) * DV * DK;
#pragma unroll
                for (int j = 0; j < DV; ++j) dst[j * DK + c] = S[j];
            }
            const int64_t tk = (bh * T_len + t) * DK + c;
            const float gc = live ? g[tk] : 0.f, kc = live ? to_f32(k[tk]) : 0.f;
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int j = 0; j < DV; j += 2) {
                S[j] = fmaf(gc, S[j], kc * s_v[tt][j]);
                S[j + 1] = fmaf(gc, S[j + 1], kc * s_v[tt][j + 1]);
                a0 = fmaf(S[j], s_do[tt][j], a0);
                a1 = fmaf(S[j + 1], s_do[tt][j + 1], a1);
            }
            if (live) dq[tk] = from_f32<T>(a0 + a1);
        }
    }
}

// ---- sweep 2: reverse, rows (dk, dg, initial-state gradient) --------------------------------
template <typename T, int DK, int DV>
__global__ void __launch_bounds__(128)
gla_bwd_rev_rows(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                 const float* __restrict__ g, const T* __restrict__ dO, const float* __restrict__ dSf,
                 T* __restrict__ dk, float* __restrict__ dg, float* __restrict__ dstate0,
                 float* __restrict__ ws, int T_len) {
    extern __shared__ __align__(16) float sm[];
    float* s_rows = sm;                    // [DK][DV + 1] forward rows during the recompute
    float* s_v = s_rows + DK * (DV + 1);   // [BLK][DV]
    float* s_do = s_v + BLK * DV;          // [BLK][DV]
    const int64_t bh = blockIdx.x;
    const int c = threadIdx.x;
    const bool live = c < DK;
    float* ckpt = ws + bh * per_bh_floats(T_len, DK, DV);
    float* scratch = ckpt + ckpt_floats(T_len, DK, DV);
    float dS[DV];
#pragma unroll
    for (int j = 0; j < DV; ++j) dS[j] = (live && dSf) ? dSf[(bh * DK + c) * DV + j] : 0.f;
    const int nblk = (T_len + BLK - 1) / BLK;
    for (int blk = nblk - 1; blk >= 0; --blk) {
        const int t0 = blk * BLK, t1 = t0 + BLK < T_len ? t0 + BLK : T_len, nt = t1 - t0;
        __syncthreads();  // the previous block's staged tokens are no longer read
        for (int i = threadIdx.x; i < nt * DV; i += blockDim.x) {
            const int tt = i / DV, j = i % DV;
            const int64_t idx = (bh * T_len + t0 + tt) * DV + j;
            s_v[tt * DV + j] = to_f32(v[idx]);
            s_do[tt * DV + j] = to_f32(dO[idx]);
        }
        // recompute S_{t-1} for t in the block from its checkpoint (row c in shared memory)
        if (live) {
            const float* src = ckpt + (size_t)blk * DV * DK;
#pragma unroll 4
            for (int j = 0; j < DV; ++j) s_rows[c * (DV + 1) + j] = src[j * DK + c];
        }
        __syncthreads();
        for (int tt = 0; tt < nt; ++tt) {
            const int64_t tk = (bh * T_len + t0 + tt) * DK + c;
            const float gc = live ? g[tk] : 0.f, kc = live ? to_f32(k[tk]) : 0.f;
            if (live) {
                float* row = s_rows + c * (DV + 1);
                float* dst = scratch + (size_t)tt * DV * DK;
#pragma unroll 16
                for (int j = 0; j < DV; ++j) {
                    dst[j * DK + c] = row[j];  // S_{t-1}
                    row[j] = fmaf(gc, row[j], kc * s_v[tt * DV + j]);
                }
            }
        }
        __syncthreads();  // (each thread reads back only what it wrote; kept for clarity)
        for (int tt = nt - 1; tt >= 0; --tt) {
            const int64_t tk = (bh * T_len + t0 + tt) * DK + c;
            const float gc = live ? g[tk] : 0.f, qc = live ? to_f32(q[tk]) : 0.f;
            const float* sp = scratch + (size_t)tt * DV * DK;
            float ak0 = 0.f, ak1 = 0.f, ag0 = 0.f, ag1 = 0.f;
#pragma unroll
            for (int j = 0; j < DV; j += 2) {
                dS[j] = fmaf(qc, s_do[tt * DV + j], dS[j]);
                dS[j + 1] = fmaf(qc, s_do[tt * DV + j + 1], dS[j + 1]);
                ak0 = fmaf(dS[j], s_v[tt * DV + j], ak0);
                ak1 = fmaf(dS[j + 1], s_v[tt * DV + j + 1], ak1);
                if (live) {
                    ag0 = fmaf(dS[j], sp[j * DK + c], ag0);
                    ag1 = fmaf(dS[j + 1], sp[(j + 1) * DK + c], ag1);
                }
            }
            if (live) {
                dk[tk] = from_f32<T>(ak0 + ak1);
                dg[tk] = ag0 + ag1;
            }
#pragma unroll
            for (int j = 0; j < DV; ++j) dS[j] *= gc;
        }
    }
    if (live) {
#pragma unroll
        for (int j = 0; j < DV; ++j) dstate0[(bh * DK + c) * DV + j] = dS[j];
    }
}

// ---- sweep 3: reverse, columns (dv) --------------------------------------------------------
template <typename T, int DK, int DV>
__global__ void __launch_bounds__(128)
gla_bwd_rev_cols(const T* __restrict__ q, const T* __restrict__ k, const float* __restrict__ g,
                 const T* __restrict__ dO, const float* __restrict__ dSf, T* __restrict__ dv,
                 int T_len) {
    __shared__ __align__(16) float s_q[TT][DK], s_k[TT][DK], s_g[TT][DK];
    const int64_t bh = blockIdx.x;
    const int j = threadIdx.x;
    const bool live = j < DV;
    float dS[DK];
#pragma unroll
    for (int c = 0; c < DK; ++c) dS[c] = (live && dSf) ? dSf[(bh * DK + c) * DV + j] : 0.f;
    for (int t1 = T_len; t1 > 0; t1 -= TT) {
        const int t0 = t1 - TT > 0 ? t1 - TT : 0, nt = t1 - t0;
        __syncthreads();
        for (int i = threadIdx.x; i < nt * DK; i += blockDim.x) {
            const int tt = i / DK, c = i % DK;
            const int64_t idx = (bh * T_len + t0 + tt) * DK + c;
            s_q[tt][c] = to_f32(q[idx]);
            s_k[tt][c] = to_f32(k[idx]);
            s_g[tt][c] = g[idx];
        }
        __syncthreads();
        for (int tt = nt - 1; tt >= 0; --tt) {
            const int64_t tv = (bh * T_len + t0 + tt) * DV + j;
            const float doj = live ? to_f32(dO[tv]) : 0.f;
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int c = 0; c < DK; c += 2) {
                dS[c] = fmaf(s_q[tt][c], doj, dS[c]);
                dS[c + 1] = fmaf(s_q[tt][c + 1], doj, dS[c + 1]);
                a0 = fmaf(s_k[tt][c], dS[c], a0);
                a1 = fmaf(s_k[tt][c + 1], dS[c + 1], a1);
                dS[c] *= s_g[tt][c];
                dS[c + 1] *= s_g[tt][c + 1];
            }
            if (live) dv[tv] = from_f32<T>(a0 + a1);
        }
    }
}

template <typename T, int DK, int DV>
cudaError_t launch_t(const GlaBackwardArgs& a, cudaStream_t s) {
    const unsigned grid = (unsigned)((int64_t)a.B * a.H);
    const int rows = DK < 32 ? 32 : DK, cols = DV < 32 ? 32 : DV;
    float* ws = static_cast<float*>(a.workspace);
    gla_bwd_fwd_rows<T, DK, DV><<<grid, rows, 0, s>>>(
        static_cast<const T*>(a.q), static_cast<const T*>(a.k), static_cast<const T*>(a.v), a.g, a.state0,
        static_cast<const T*>(a.dO), static_cast<T*>(a.dq), ws, a.T);
    const size_t smem = sizeof(float) * ((size_t)DK * (DV + 1) + 2 * (size_t)BLK * DV);
    cudaError_t e = cudaFuncSetAttribute(gla_bwd_rev_rows<T, DK, DV>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    gla_bwd_rev_rows<T, DK, DV><<<grid, rows, smem, s>>>(
        static_cast<const T*>(a.q), static_cast<const T*>(a.k), static_cast<const T*>(a.v), a.g,
        static_cast<const T*>(a.dO), a.dstate_final, static_cast<T*>(a.dk), a.dg, a.dstate0, ws, a.T);
    gla_bwd_rev_cols<T, DK, DV><<<grid, cols, 0, s>>>(
        static_cast<const T*>(a.q), static_cast<const T*>(a.k), a.g, static_cast<const T*>(a.dO),
        a.dstate_final, static_cast<T*>(a.dv), a.T);
    note_launches(3);
    return cudaGetLastError();
}

template <typename T, int DK>
cudaError_t launch_dv(const GlaBackwardArgs& a, cudaStream_t s) {
    switch (a.d_v) {
        case 16: return launch_t<T, DK, 16>(a, s);
        case 32: return launch_t<T, DK, 32>(a, s);
        case 64: return launch_t<T, DK, 64>(a, s);
        case 128: return launch_t<T, DK, 128>(a, s);
    }
    return cudaErrorInvalidValue;
}

template <typename T>
cudaError_t launch_dk(const GlaBackwardArgs& a, cudaStream_t s) {
    switch (a.d_k) {
        case 16: return launch_dv<T, 16>(a, s);
        case 32: return launch_dv<T, 32>(a, s);
        case 64: return launch_dv<T, 64>(a, s);
        case 128: return launch_dv<T, 128>(a, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

size_t gla_backward_workspace_size(int B, int H, int T, int dk, int dv) {
    return (size_t)B * H * per_bh_floats(T, dk, dv) * sizeof(float);
}

cudaError_t gla_backward_launch(const GlaBackwardArgs& a, bool bf16, cudaStream_t stream) {
    if ((int64_t)a.B * a.H == 0 || a.T == 0) return cudaSuccess;
    return bf16 ? launch_dk<__nv_bfloat16>(a, stream) : launch_dk<float>(a, stream);
}

}  // namespace rod
