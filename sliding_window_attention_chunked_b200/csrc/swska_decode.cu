// swska_decode.cu -- SW-SKA decode: ring-buffer write + sliding-window attention of one new
// token per sequence over a shared-K / per-head-V window cache.
//
// Semantics (SALA blog §3.3: a self-made circular buffer holds the rolling window; CodeFuse
// Rodimus* article, Fig. 4 / SKA paragraph: one K shared by all heads, per-head V):
//   slot(p) = p mod W;  the new token (position P = pos[n]) is written to slot(P);
//   o[n,h] = softmax over positions p in [max(0,P-W+1), P] of scale * q[n,h] . K[slot(p)],
//            applied to V[h, slot(p)].
// Which slots are valid follows from the ring rule: for P < W the slots 0..P, else all W.
//
// Design (bound by HBM: per sequence 1 K row + H V rows per slot, i.e. 17 MiB at W = 4096,
// H = 16, d = 128 bf16):
//  * a thread-block cluster of SP CTAs serves one sequence; CTA r owns a contiguous run of
//    valid slots, so every K/V byte is read exactly once;
//  * one thread streams KT-slot stages into shared memory with bulk async copies (one copy
//    for the K rows -- shared by all H heads -- and one per head for its V rows; each is
//    contiguous in the cache), into a STAGES-deep ring completed on mbarriers;
//  * phase A: all H x KT scores of a stage, each from the K row held once in shared memory
//    (the shared key is read once for all heads); phase B: thread (h, 8-column group) runs
//    the online softmax (base-2, scores pre-scaled by scale*log2 e) and accumulates p * V;
//  * the SP partial (max, sum, accumulator) triples are combined through distributed shared
//    memory inside the cluster -- no global scratch -- and CTA r writes the heads h = r mod SP;
//  * the new token replaces its slot in shared memory as soon as that stage lands, and is
//    written to the global cache after the CTA has finished reading it.
// All mbarrier waits are bounded (rod::kWaitLimit probes); on expiry the CTA stops, waits
// (bounded) for its outstanding copies, raises the timeout flag and still takes part in the
// cluster barriers, so no thread is left waiting.
#include <cooperative_groups.h>

#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace rod {
namespace {

__device__ unsigned int g_swska_decode_timeout = 0;

struct DecodePlan {
    int KT;       // slots per stage
    int stages;   // ring depth
    int SP;       // CTAs per cluster (split of the window)
    int threads;
    size_t stage_bytes;
    size_t smem_bytes;
};

template <typename T>
__global__ void swska_decode_kernel(const T* __restrict__ q, const T* __restrict__ k_new,
                                    const T* __restrict__ v_new, T* __restrict__ k_cache,
                                    T* __restrict__ v_cache, const int64_t* __restrict__ pos,
                                    T* __restrict__ o, int H, int dk, int dv, int W,
                                    float scale_log2, int KT, int stages) {
    extern __shared__ __align__(128) unsigned char smem[];
    cg::cluster_group cluster = cg::this_cluster();
    const int SP = (int)cluster.num_blocks();
    const int rank = (int)cluster.block_rank();
    const int64_t n = blockIdx.x / SP;
    const int tid = threadIdx.x, nthr = blockDim.x;
    const int CG = dv / 8;                     // 8-column groups per head

    // ---- shared-memory carve-up (all offsets multiples of 16 bytes) ----
    const size_t k_stage = (size_t)KT * dk * sizeof(T);
    const size_t v_head = (size_t)KT * dv * sizeof(T);
    const size_t stage_bytes = k_stage + (size_t)H * v_head;
    unsigned char* p = smem;
    uint64_t* full = reinterpret_cast<uint64_t*>(p);            p += 64;
    float* s_q = reinterpret_cast<float*>(p);                   p += (size_t)H * dk * 4;
    float* s_sc = reinterpret_cast<float*>(p);                  p += (((size_t)H * KT * 4 + 15) / 16) * 16;
    float* s_pm = reinterpret_cast<float*>(p);                  p += (((size_t)H * 4 + 15) / 16) * 16;
    float* s_pl = reinterpret_cast<float*>(p);                  p += (((size_t)H * 4 + 15) / 16) * 16;
    unsigned char* ring = p;
    // the partial accumulators reuse the ring once every stage has been consumed (or drained)
    float* s_pacc = reinterpret_cast<float*>(ring);

    const int64_t P = pos[n];
    const bool bad = P < 0;
    const int64_t cnt = bad ? 0 : (P + 1 < W ? P + 1 : W);      // valid slots 0..cnt-1
    const int64_t s_new = bad ? -1 : P % W;
    const int64_t per = (cnt + SP - 1) / SP;
    const int64_t s_begin = (int64_t)rank * per < cnt ? (int64_t)rank * per : cnt;
    const int64_t s_end = s_begin + per < cnt ? s_begin + per : cnt;
    const int nst = (int)((s_end - s_begin + KT - 1) / KT);

    const T* Kc = k_cache + n * (int64_t)W * dk;
    const T* Vc = v_cache + n * (int64_t)H * W * dv;

    if (tid == 0) {
        for (int s = 0; s < stages; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
    }
    // q for all heads, pre-scaled so that the softmax runs in base 2
    for (int i = tid; i < H * dk; i += nthr) s_q[i] = to_f32(q[n * (int64_t)H * dk + i]) * scale_log2;
    __syncthreads();

    auto issue = [&](int st) {  // thread 0 only
        const int buf = st % stages;
        const int64_t s0 = s_begin + (int64_t)st * KT;
        const int rows = (int)((s_end - s0) < KT ? (s_end - s0) : KT);
        unsigned char* dst = ring + (size_t)buf * stage_bytes;
        const uint32_t kb = (uint32_t)(rows * dk * sizeof(T));
        const uint32_t vb = (uint32_t)(rows * dv * sizeof(T));
        mbar_arrive_expect_tx(&full[buf], kb + (uint32_t)H * vb);
        bulk_g2s(dst, Kc + s0 * dk, kb, &full[buf]);
        for (int h = 0; h < H; ++h)
            bulk_g2s(dst + k_stage + (size_t)h * v_head, Vc + ((int64_t)h * W + s0) * dv, vb, &full[buf]);
    };
    if (tid == 0)
        for (int st = 0; st < nst && st < stages; ++st) issue(st);

    // per-thread online-softmax state for (head h, columns 8*cgi .. 8*cgi+7)
    const int h_mine = tid / CG, cgi = tid % CG;
    const bool owner = h_mine < H;
    float m_run = -INFINITY, l_run = 0.f, acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;

    int issued = nst < stages ? nst : stages;
    bool aborted = false;  // uniform across the CTA (decided by a block-wide vote)
    int st = 0;
    for (; st < nst; ++st) {
        const int buf = st % stages;
        const uint32_t parity = (uint32_t)((st / stages) & 1);
        const bool ok = mbar_wait_bounded(&full[buf], parity, kWaitLimit);
        if (__syncthreads_or(!ok)) {
            aborted = true;
            break;
        }
        const int64_t s0 = s_begin + (int64_t)st * KT;
        const int rows = (int)((s_end - s0) < KT ? (s_end - s0) : KT);
        unsigned char* base = ring + (size_t)buf * stage_bytes;
        T* sK = reinterpret_cast<T*>(base);
        if (s_new >= s0 && s_new < s0 + rows) {  // the new token replaces its slot in this stage
            const int r = (int)(s_new - s0);
            for (int i = tid; i < dk; i += nthr) sK[r * dk + i] = k_new[n * dk + i];
            for (int i = tid; i < H * dv; i += nthr) {
                const int h = i / dv, c = i % dv;
                reinterpret_cast<T*>(base + k_stage + (size_t)h * v_head)[r * dv + c] =
                    v_new[(n * H + h) * (int64_t)dv + c];
            }
            __syncthreads();
        }
        // phase A: scores s[h][j] = (scale*log2e) q_h . K_j, one K row read serves all heads
        const int nchunk = dk / 8;
        for (int pr = tid; pr < H * KT; pr += nthr) {
            const int h = pr / KT, j = pr % KT;
            float sc = -INFINITY;
            if (j < rows) {
                const T* kr = sK + j * dk;
                const float* qh = s_q + h * dk;
                float a0 = 0.f, a1 = 0.f;
                for (int u = 0; u < nchunk; ++u) {
                    const int c = ((u + j) % nchunk) * 8;  // rotate chunks to spread banks
                    float kf[8];
                    load8(kr + c, kf);
                    const float4 q0 = *reinterpret_cast<const float4*>(qh + c);
                    const float4 q1 = *reinterpret_cast<const float4*>(qh + c + 4);
                    a0 = fmaf(q0.x, kf[0], a0); a1 = fmaf(q0.y, kf[1], a1);
                    a0 = fmaf(q0.z, kf[2], a0); a1 = fmaf(q0.w, kf[3], a1);
                    a0 = fmaf(q1.x, kf[4], a0); a1 = fmaf(q1.y, kf[5], a1);
                    a0 = fmaf(q1.z, kf[6], a0); a1 = fmaf(q1.w, kf[7], a1);
                }
                sc = a0 + a1;
            }
            s_sc[h * KT + j] = sc;
        }
        __syncthreads();
        // phase B: online softmax + p * V for (h_mine, column group cgi)
        if (owner) {
            const float* sc = s_sc + h_mine * KT;
            float mx = m_run;
            for (int j = 0; j < rows; ++j) mx = fmaxf(mx, sc[j]);
            if (mx > m_run) {
                const float alpha = exp2f(m_run - mx);  // m_run = -inf gives 0
                l_run *= alpha;
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[i] *= alpha;
                m_run = mx;
            }
            const T* vb = reinterpret_cast<const T*>(base + k_stage + (size_t)h_mine * v_head) + cgi * 8;
            for (int j = 0; j < rows; ++j) {
                const float pj = exp2f(sc[j] - m_run);
                l_run += pj;
                float vf[8];
                load8(vb + j * dv, vf);
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[i] = fmaf(pj, vf[i], acc[i]);
            }
        }
        __syncthreads();  // the stage buffer is free again
        if (tid == 0 && issued < nst) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            issue(issued);
            ++issued;
        }
    }
    if (aborted) {
        // let every copy still in flight land before the CTA's shared memory goes away
        // stages st .. issued-1 are the ones still in flight (each the latest phase of its buffer)
        if (tid == 0) {
            for (int s2 = st; s2 < issued; ++s2)
                mbar_wait_bounded(&full[s2 % stages], (uint32_t)((s2 / stages) & 1), kWaitLimit);
            atomicExch(&g_swska_decode_timeout, 1u);
        }
        m_run = NAN;
    }

    // ---- publish this CTA's partial softmax state to the cluster ----
    __syncthreads();  // every thread is done with the ring before it is overwritten
    if (owner) {
#pragma unroll
        for (int i = 0; i < 8; ++i) s_pacc[h_mine * dv + cgi * 8 + i] = acc[i];
        if (cgi == 0) { s_pm[h_mine] = m_run; s_pl[h_mine] = l_run; }
    }
    cluster.sync();
    // ---- combine: CTA `rank` finalises heads h with h mod SP == rank ----
    for (int idx = tid; idx < H * CG; idx += nthr) {
        const int h = idx / CG, c8 = idx % CG;
        if (h % SP != rank) continue;
        float out[8];
        if (bad) {
#pragma unroll
            for (int i = 0; i < 8; ++i) out[i] = NAN;
        } else {
            float M = -INFINITY;
            for (int r = 0; r < SP; ++r) M = fmaxf(M, cluster.map_shared_rank(s_pm, r)[h]);
            float L = 0.f, a[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) a[i] = 0.f;
            for (int r = 0; r < SP; ++r) {
                const float mr = cluster.map_shared_rank(s_pm, r)[h];
                const float lr = cluster.map_shared_rank(s_pl, r)[h];
                if (!(lr > 0.f) && !isnan(mr)) continue;  // a CTA without slots
                const float w = exp2f(mr - M);
                L = fmaf(w, lr, L);
                const float* pa = cluster.map_shared_rank(s_pacc, r) + h * dv + c8 * 8;
#pragma unroll
                for (int i = 0; i < 8; ++i) a[i] = fmaf(w, pa[i], a[i]);
            }
            const float inv = 1.f / L;
#pragma unroll
            for (int i = 0; i < 8; ++i) out[i] = a[i] * inv;
        }
        store8(o + (n * H + h) * (int64_t)dv + c8 * 8, out);
    }
    // ---- the new token enters the ring buffer (after every read of its slot in this CTA) ----
    if (!bad && s_new >= s_begin && s_new < s_end) {
        T* kdst = k_cache + (n * (int64_t)W + s_new) * dk;
        for (int i = tid; i < dk; i += nthr) kdst[i] = k_new[n * dk + i];
        for (int i = tid; i < H * dv; i += nthr) {
            const int h = i / dv, c = i % dv;
            v_cache[((n * H + h) * (int64_t)W + s_new) * dv + c] = v_new[(n * H + h) * (int64_t)dv + c];
        }
    }
    cluster.sync();  // keep this CTA's shared memory alive until every peer has read it
}

template <typename T>
DecodePlan plan_for(int H, int dk, int dv, int W) {
    DecodePlan pl{};
    pl.KT = 8;
    auto stage = [&](int kt) { return (size_t)kt * dk * sizeof(T) + (size_t)H * kt * dv * sizeof(T); };
    while (pl.KT > 1 && stage(pl.KT) > 48 * 1024) pl.KT /= 2;
    pl.stage_bytes = stage(pl.KT);
    pl.stages = 3;
    pl.SP = W >= 2048 ? 8 : (W >= 1024 ? 4 : (W >= 512 ? 2 : 1));
    pl.threads = ((H * (dv / 8) + 31) / 32) * 32;
    if (pl.threads < 128) pl.threads = 128;
    const size_t fixed = 64 + (size_t)H * dk * 4 + (((size_t)H * pl.KT * 4 + 15) / 16) * 16 +
                         2 * (((size_t)H * 4 + 15) / 16) * 16;
    size_t ring = (size_t)pl.stages * pl.stage_bytes;
    if (ring < (size_t)H * dv * 4) ring = (size_t)H * dv * 4;  // also holds the partials
    pl.smem_bytes = fixed + ring;
    return pl;
}

template <typename T>
cudaError_t launch_t(const void* q, const void* k_new, const void* v_new, void* k_cache,
                     void* v_cache, const int64_t* pos, void* o, int N, int H, int dk, int dv,
                     int W, float scale, cudaStream_t stream) {
    const DecodePlan pl = plan_for<T>(H, dk, dv, W);
    if (pl.threads > 1024 || pl.smem_bytes > 220 * 1024) return cudaErrorInvalidConfiguration;
    cudaError_t e = cudaFuncSetAttribute(swska_decode_kernel<T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)pl.smem_bytes);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((int64_t)N * pl.SP), 1, 1);
    cfg.blockDim = dim3((unsigned)pl.threads, 1, 1);
    cfg.dynamicSmemBytes = pl.smem_bytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)pl.SP;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const float scale_log2 = scale * 1.4426950408889634f;
    note_launches(1);
    return cudaLaunchKernelEx(&cfg, swska_decode_kernel<T>, static_cast<const T*>(q),
                              static_cast<const T*>(k_new), static_cast<const T*>(v_new),
                              static_cast<T*>(k_cache), static_cast<T*>(v_cache), pos,
                              static_cast<T*>(o), H, dk, dv, W, scale_log2, pl.KT, pl.stages);
}

}  // namespace

cudaError_t swska_decode_launch(const void* q, const void* k_new, const void* v_new,
                                void* k_cache, void* v_cache, const int64_t* pos, void* o,
                                int N, int H, int dk, int dv, int window, float scale, bool bf16,
                                cudaStream_t stream) {
    if (N == 0) return cudaSuccess;
    if (bf16 && swska_decode_warp_supported(H, dk, dv))
        return swska_decode_warp_launch(q, k_new, v_new, k_cache, v_cache, pos, o, N, H, window,
                                        scale, stream);
    return bf16 ? launch_t<__nv_bfloat16>(q, k_new, v_new, k_cache, v_cache, pos, o, N, H, dk, dv,
                                          window, scale, stream)
                : launch_t<float>(q, k_new, v_new, k_cache, v_cache, pos, o, N, H, dk, dv,
                                  window, scale, stream);
}

unsigned swska_decode_take_timeout_flag() {
    unsigned v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_swska_decode_timeout, sizeof(v)) != cudaSuccess) return 0;
    cudaMemcpyToSymbol(g_swska_decode_timeout, &zero, sizeof(zero));
    return v;
}

}  // namespace rod
