// gla_backward.cu -- backward of the Rodimus gated linear recurrence on CUDA cores (fp32 FMA).
//
// Forward (CodeFuse Rodimus* article, Rodimus block; the chunkwise-parallel algorithm is stated
// for training as well as prefill):  S_t = diag(g_t) S_{t-1} + k_t^T v_t,  o_t = q_t S_t.
// Given dO_t (gradient of every o_t) and dS_T (gradient of the final state, may be absent):
//   dq_t[c] = sum_j dO_t[j] S_t[c][j]
//   dS_t    = q_t^T dO_t + diag(g_{t+1}) dS_{t+1}            (reverse in time, from dS_T)
//   dk_t[c] = sum_j dS_t[c][j] v_t[j],   dv_t[j] = sum_c dS_t[c][j] k_t[c]
//   dg_t[c] = sum_j dS_t[c][j] S_{t-1}[c][j],   d(initial state) = diag(g_1) dS_1.
// Both state recurrences act on each column j (S, dS) independently, and on each row c for the
// dv sweep: only the sums over j (dq, dk, dg) and over c (dv) couple them. So each (batch, head)
// is a thread-block cluster of CTAs, each owning CG = 8 state columns (rows in the dv sweep)
// with one thread per state row (column): 16x the CTAs of one CTA per (batch, head) at d = 128,
// and a thread's step is 8 FMAs per product instead of 128. Each CTA writes its partial sums of
// a block of BLK steps to its shared memory; after a cluster barrier every CTA adds up one slice
// of rows over the cluster's CTAs, in rank order (deterministic), reading them through
// distributed shared memory. The partial buffers alternate between blocks, so one barrier per
// block suffices (a CTA writes buffer b % 2 only after every peer has passed the barrier that
// ends the reads of block b - 2).
// Three sweeps:
//   1. forward, rows: dq, and a checkpoint of S before every block of BLK steps;
//   2. reverse, rows: per block, the states S_{t-1} are recomputed from the block's checkpoint
//      into registers (BLK x CG per thread), then the block is walked backwards for dk, dg and
//      the propagation of dS; the last dS is the initial-state gradient;
//   3. reverse, columns: dv.
// Every product is fp32.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace rod {
namespace {

constexpr int BLK = 16;  // steps per block: checkpoint spacing and reduction period
constexpr int CG = 8;    // state columns (rows, in the dv sweep) per CTA

// workspace per (batch, head): checkpoints [nblk][DV][DK], the state before each block's first
// step, element (j, c) at j * DK + c (the threads' accesses coalesce)
__host__ __device__ inline size_t ckpt_floats(int T, int dk, int dv) {
    return (size_t)((T + BLK - 1) / BLK) * dk * dv;
}

// sum of a partial buffer over the cluster's NC CTAs for this CTA's slice of the N columns (rows
// of the state), written through `store(t_in_block, index, value)` for steps below nt; the NC
// remote loads of an element are issued together, then added in rank order
template <int N, int NC, typename Store>
__device__ __forceinline__ void cluster_reduce(cg::cluster_group& cl, const float* part, int nt, Store store) {
    constexpr int per = (N + NC - 1) / NC;
    const int rank = (int)cl.block_rank();
    for (int i = threadIdx.x; i < BLK * per; i += blockDim.x) {
        const int tt = i / per, n = rank * per + i % per;
        if (tt < nt && n < N) {
            float x[NC];
#pragma unroll
            for (int r = 0; r < NC; ++r) x[r] = cl.map_shared_rank(part, r)[tt * N + n];
            float acc = 0.f;
#pragma unroll
            for (int r = 0; r < NC; ++r) acc += x[r];
            store(tt, n, acc);
        }
    }
}

// ---- sweep 1: forward, rows (dq, checkpoints) ------------------------------------------------
template <typename T, int DK, int DV>
__global__ void __launch_bounds__(128)
gla_bwd_fwd_rows(const T* __restrict__ k, const T* __restrict__ v, const float* __restrict__ g,
                 const float* __restrict__ state0, const T* __restrict__ dO, T* __restrict__ dq,
                 float* __restrict__ ws, int T_len) {
    constexpr int NG = DV / CG;
    __shared__ __align__(16) float s_v[BLK][CG], s_do[BLK][CG], s_g[BLK][DK], s_k[BLK][DK];
    __shared__ __align__(16) float part[2][BLK * DK];
    cg::cluster_group cl = cg::this_cluster();
    const int j0 = (int)cl.block_rank() * CG;
    const int64_t bh = blockIdx.x / NG;
    const int c = threadIdx.x;
    const bool live = c < DK;
    float* ckpt = ws + bh * ckpt_floats(T_len, DK, DV);
    float S[CG];
#pragma unroll
    for (int j = 0; j < CG; ++j) S[j] = live ? state0[(bh * DK + c) * DV + j0 + j] : 0.f;
    const int nblk = (T_len + BLK - 1) / BLK;
    for (int b = 0; b < nblk; ++b) {
        const int t0 = b * BLK, nt = T_len - t0 < BLK ? T_len - t0 : BLK;
        __syncthreads();
        for (int i = threadIdx.x; i < BLK * CG; i += blockDim.x) {
            const int tt = i / CG, j = i % CG;
            const int64_t idx = (bh * T_len + t0 + tt) * DV + j0 + j;
            s_v[tt][j] = tt < nt ? to_f32(v[idx]) : 0.f;
            s_do[tt][j] = tt < nt ? to_f32(dO[idx]) : 0.f;
        }
        for (int i = threadIdx.x; i < BLK * DK; i += blockDim.x) {
            const int tt = i / DK, r = i % DK;
            const int64_t idx = (bh * T_len + t0 + tt) * DK + r;
            s_g[tt][r] = tt < nt ? g[idx] : 0.f;
            s_k[tt][r] = tt < nt ? to_f32(k[idx]) : 0.f;
        }
        __syncthreads();
        if (live) {
            float* dst = ckpt + (size_t)b * DV * DK;
#pragma unroll
            for (int j = 0; j < CG; ++j) dst[(j0 + j) * DK + c] = S[j];
        }
        float* pb = part[b & 1];
#pragma unroll
        for (int tt = 0; tt < BLK; ++tt) {
            float acc = 0.f;
            if (tt < nt) {
                const float gc = live ? s_g[tt][c] : 0.f, kc = live ? s_k[tt][c] : 0.f;
#pragma unroll
                for (int j = 0; j < CG; ++j) {
                    S[j] = fmaf(gc, S[j], kc * s_v[tt][j]);
                    acc = fmaf(S[j], s_do[tt][j], acc);
                }
            }
            if (live) pb[tt * DK + c] = acc;
        }
        cl.sync();
        cluster_reduce<DK, NG>(cl, pb, nt, [&](int tt, int n, float x) {
            dq[(bh * T_len + t0 + tt) * DK + n] = from_f32<T>(x);
        });
    }
    cl.sync();  // every peer has read this CTA's partials
}

// ---- sweep 2: reverse, rows (dk, dg, initial-state gradient) --------------------------------
// three CTAs per SM (167 registers, no spills; the block's states take 128 of them)
template <typename T, int DK, int DV>
__global__ void __launch_bounds__(128, 3)
gla_bwd_rev_rows(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                 const float* __restrict__ g, const T* __restrict__ dO, const float* __restrict__ dSf,
                 T* __restrict__ dk, float* __restrict__ dg, float* __restrict__ dstate0,
                 const float* __restrict__ ws, int T_len) {
    constexpr int NG = DV / CG;
    // dynamic shared memory (57 KB at dk = 128): staged rows of the block, then the partial sums
    extern __shared__ __align__(16) float sm[];
    float(*s_v)[CG] = reinterpret_cast<float(*)[CG]>(sm);
    float(*s_do)[CG] = reinterpret_cast<float(*)[CG]>(sm + BLK * CG);
    float(*s_q)[DK] = reinterpret_cast<float(*)[DK]>(sm + 2 * BLK * CG);
    float(*s_k)[DK] = reinterpret_cast<float(*)[DK]>(sm + 2 * BLK * CG + BLK * DK);
    float(*s_g)[DK] = reinterpret_cast<float(*)[DK]>(sm + 2 * BLK * CG + 2 * BLK * DK);
    float* part_k[2] = {sm + 2 * BLK * CG + 3 * BLK * DK, sm + 2 * BLK * CG + 4 * BLK * DK};
    float* part_g[2] = {sm + 2 * BLK * CG + 5 * BLK * DK, sm + 2 * BLK * CG + 6 * BLK * DK};
    cg::cluster_group cl = cg::this_cluster();
    const int j0 = (int)cl.block_rank() * CG;
    const int64_t bh = blockIdx.x / NG;
    const int c = threadIdx.x;
    const bool live = c < DK;
    const float* ckpt = ws + bh * ckpt_floats(T_len, DK, DV);
    float dS[CG];
#pragma unroll
    for (int j = 0; j < CG; ++j) dS[j] = (live && dSf) ? dSf[(bh * DK + c) * DV + j0 + j] : 0.f;
    const int nblk = (T_len + BLK - 1) / BLK;
    for (int b = nblk - 1; b >= 0; --b) {
        const int t0 = b * BLK, nt = T_len - t0 < BLK ? T_len - t0 : BLK;
        __syncthreads();
        for (int i = threadIdx.x; i < BLK * CG; i += blockDim.x) {
            const int tt = i / CG, j = i % CG;
            const int64_t idx = (bh * T_len + t0 + tt) * DV + j0 + j;
            s_v[tt][j] = tt < nt ? to_f32(v[idx]) : 0.f;
            s_do[tt][j] = tt < nt ? to_f32(dO[idx]) : 0.f;
        }
        for (int i = threadIdx.x; i < BLK * DK; i += blockDim.x) {
            const int tt = i / DK, r = i % DK;
            const int64_t idx = (bh * T_len + t0 + tt) * DK + r;
            s_q[tt][r] = tt < nt ? to_f32(q[idx]) : 0.f;
            s_k[tt][r] = tt < nt ? to_f32(k[idx]) : 0.f;
            s_g[tt][r] = tt < nt ? g[idx] : 0.f;
        }
        __syncthreads();
        // the block's states S_{t0 + tt - 1}, recomputed from its checkpoint
        float Sp[BLK][CG];
#pragma unroll
        for (int j = 0; j < CG; ++j) Sp[0][j] = live ? ckpt[(size_t)b * DV * DK + (j0 + j) * DK + c] : 0.f;
#pragma unroll
        for (int tt = 1; tt < BLK; ++tt) {
            // (past the block's last step the staged g, k, v are 0 and these states are unused)
            const float gc = live ? s_g[tt - 1][c] : 0.f, kc = live ? s_k[tt - 1][c] : 0.f;
#pragma unroll
            for (int j = 0; j < CG; ++j) Sp[tt][j] = fmaf(gc, Sp[tt - 1][j], kc * s_v[tt - 1][j]);
        }
        float* pk = part_k[b & 1];
        float* pg = part_g[b & 1];
#pragma unroll
        for (int tt = BLK - 1; tt >= 0; --tt) {
            float ak = 0.f, ag = 0.f;
            if (tt < nt) {
                const float gc = live ? s_g[tt][c] : 0.f, qc = live ? s_q[tt][c] : 0.f;
#pragma unroll
                for (int j = 0; j < CG; ++j) {
                    dS[j] = fmaf(qc, s_do[tt][j], dS[j]);
                    ak = fmaf(dS[j], s_v[tt][j], ak);
                    ag = fmaf(dS[j], Sp[tt][j], ag);
                }
#pragma unroll
                for (int j = 0; j < CG; ++j) dS[j] *= gc;
            }
            if (live) {
                pk[tt * DK + c] = ak;
                pg[tt * DK + c] = ag;
            }
        }
        cl.sync();
        cluster_reduce<DK, NG>(cl, pk, nt, [&](int tt, int n, float x) {
            dk[(bh * T_len + t0 + tt) * DK + n] = from_f32<T>(x);
        });
        cluster_reduce<DK, NG>(cl, pg, nt, [&](int tt, int n, float x) {
            dg[(bh * T_len + t0 + tt) * DK + n] = x;
        });
    }
    if (live) {
#pragma unroll
        for (int j = 0; j < CG; ++j) dstate0[(bh * DK + c) * DV + j0 + j] = dS[j];
    }
    cl.sync();
}

// ---- sweep 3: reverse, columns (dv) --------------------------------------------------------
template <typename T, int DK, int DV>
__global__ void __launch_bounds__(128)
gla_bwd_rev_cols(const T* __restrict__ q, const T* __restrict__ k, const float* __restrict__ g,
                 const T* __restrict__ dO, const float* __restrict__ dSf, T* __restrict__ dv,
                 int T_len) {
    constexpr int NG = DK / CG;
    __shared__ __align__(16) float s_q[BLK][CG], s_k[BLK][CG], s_g[BLK][CG], s_do[BLK][DV];
    __shared__ __align__(16) float part[2][BLK * DV];
    cg::cluster_group cl = cg::this_cluster();
    const int c0 = (int)cl.block_rank() * CG;
    const int64_t bh = blockIdx.x / NG;
    const int j = threadIdx.x;
    const bool live = j < DV;
    float dS[CG];  // column j of the gradient state, rows c0 .. c0 + CG - 1
#pragma unroll
    for (int i = 0; i < CG; ++i) dS[i] = (live && dSf) ? dSf[(bh * DK + c0 + i) * DV + j] : 0.f;
    const int nblk = (T_len + BLK - 1) / BLK;
    for (int b = nblk - 1; b >= 0; --b) {
        const int t0 = b * BLK, nt = T_len - t0 < BLK ? T_len - t0 : BLK;
        __syncthreads();
        for (int i = threadIdx.x; i < BLK * CG; i += blockDim.x) {
            const int tt = i / CG, r = i % CG;
            const int64_t idx = (bh * T_len + t0 + tt) * DK + c0 + r;
            s_q[tt][r] = tt < nt ? to_f32(q[idx]) : 0.f;
            s_k[tt][r] = tt < nt ? to_f32(k[idx]) : 0.f;
            s_g[tt][r] = tt < nt ? g[idx] : 0.f;
        }
        for (int i = threadIdx.x; i < BLK * DV; i += blockDim.x) {
            const int tt = i / DV, n = i % DV;
            s_do[tt][n] = tt < nt ? to_f32(dO[(bh * T_len + t0 + tt) * DV + n]) : 0.f;
        }
        __syncthreads();
        float* pb = part[b & 1];
#pragma unroll
        for (int tt = BLK - 1; tt >= 0; --tt) {
            float a = 0.f;
            if (tt < nt) {
                const float doj = live ? s_do[tt][j] : 0.f;
#pragma unroll
                for (int i = 0; i < CG; ++i) {
                    dS[i] = fmaf(s_q[tt][i], doj, dS[i]);
                    a = fmaf(s_k[tt][i], dS[i], a);
                    dS[i] *= s_g[tt][i];
                }
            }
            if (live) pb[tt * DV + j] = a;
        }
        cl.sync();
        cluster_reduce<DV, NG>(cl, pb, nt, [&](int tt, int n, float x) {
            dv[(bh * T_len + t0 + tt) * DV + n] = from_f32<T>(x);
        });
    }
    cl.sync();
}

template <int DK>
constexpr size_t rev_rows_smem() { return sizeof(float) * (2 * BLK * CG + 7 * BLK * DK); }

template <typename K, typename... Args>
cudaError_t launch_cluster(K kernel, int64_t clusters, int csize, int threads, size_t smem, cudaStream_t s,
                           Args... args) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e == cudaSuccess && smem > 0)
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (clusters * csize > 0x7fffffff) return cudaErrorInvalidConfiguration;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(clusters * csize), 1, 1);
    cfg.blockDim = dim3((unsigned)threads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)csize;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

template <typename T, int DK, int DV>
cudaError_t launch_t(const GlaBackwardArgs& a, cudaStream_t s) {
    static_assert(DK % CG == 0 && DV % CG == 0, "state dims are multiples of the column group");
    const int64_t bhs = (int64_t)a.B * a.H;
    const int rows = DK < 32 ? 32 : DK, cols = DV < 32 ? 32 : DV;
    float* ws = static_cast<float*>(a.workspace);
    cudaError_t e = launch_cluster(gla_bwd_fwd_rows<T, DK, DV>, bhs, DV / CG, rows, 0, s,
                                   static_cast<const T*>(a.k), static_cast<const T*>(a.v), a.g, a.state0,
                                   static_cast<const T*>(a.dO), static_cast<T*>(a.dq), ws, a.T);
    if (e != cudaSuccess) return e;
    e = launch_cluster(gla_bwd_rev_rows<T, DK, DV>, bhs, DV / CG, rows, rev_rows_smem<DK>(), s,
                       static_cast<const T*>(a.q),
                       static_cast<const T*>(a.k), static_cast<const T*>(a.v), a.g, static_cast<const T*>(a.dO),
                       a.dstate_final, static_cast<T*>(a.dk), a.dg, a.dstate0, static_cast<const float*>(ws), a.T);
    if (e != cudaSuccess) return e;
    e = launch_cluster(gla_bwd_rev_cols<T, DK, DV>, bhs, DK / CG, cols, 0, s, static_cast<const T*>(a.q),
                       static_cast<const T*>(a.k), a.g, static_cast<const T*>(a.dO), a.dstate_final,
                       static_cast<T*>(a.dv), a.T);
    note_launches(3);
    return e;
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
    return (size_t)B * H * ckpt_floats(T, dk, dv) * sizeof(float);
}

cudaError_t gla_backward_launch(const GlaBackwardArgs& a, bool bf16, cudaStream_t stream) {
    if ((int64_t)a.B * a.H == 0 || a.T == 0) return cudaSuccess;
    return bf16 ? launch_dk<__nv_bfloat16>(a, stream) : launch_dk<float>(a, stream);
}

}  // namespace rod
