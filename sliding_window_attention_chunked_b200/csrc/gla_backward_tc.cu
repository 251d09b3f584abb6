// gla_backward_tc.cu -- chunkwise backward of the Rodimus gated linear recurrence on the
// tensor cores (tcgen05 / TMEM / TMA): bf16 q, k, v, dO; fp32 gates, states and gate gradient;
// d_k = d_v = 128; chunks of C = 64 tokens.
//
// Forward (CodeFuse Rodimus* article, Rodimus block; its chunkwise-parallel algorithm serves
// training as well as prefill):  S_t = diag(g_t) S_{t-1} + k_t^T v_t,  o_t = q_t S_t.
// Chunk form of the backward. Inside a chunk with incoming state S_in and E, the gradient that
// reaches the chunk's last state from later chunks, let G_t = prod_{u<=t} g_u (per key channel),
// a = G_{C-1}, q~ = q.G, k~ = k/G, k^ = k.a/G, A2 = dO V^T and QK = q~ k~^T (C x C), M the mask
// s <= t. Then
//     dq = [dO S_in^T + M(A2) k~] . G
//     dk = [M(A2)^T q~] / G + (V E^T) . a/G
//     dv = M(QK)^T dO + k^ E
//     E_prev = diag(a) E + q~^T dO                    (handed to the chunk before; dS_0 at t = 0)
//     dg_t[c] = sum_j D_t[c,j] S_{t-1}[c,j]   (D_t the gradient of S_t)
// and dg in four terms (incoming state or the chunk's earlier keys, paired with E or the chunk's
// later queries), which with X1 = dO S_in^T, X2 = M(A2) k~, X3 = M(A2)^T q~, X4 = V E^T are
//     g_t dg_t = sum_{r>=t} q~_r (X1 + X2)_r - sum_{s>=t} k~_s X3_s
//              + a (sum_{s<t} k~_s X4_s + rho),   rho_c = sum_j E[c,j] S_in[c,j].
// The two sums over X2 and X3 cover the same (query, key) pairs except s < t <= r; they are
// formed from the very bf16 values of q~ and k~ the tensor cores multiplied, so the pairs they
// share cancel to fp32 rounding. Dividing by g_t is the one step the product form cannot do at
// g = 0, so a chunk whose gates reach below 2^-8 (or whose decay a falls below 2^-60) takes the
// exact route: its scores, dq, dk and dg are summed on the CUDA cores from log2-gate prefix sums
// L (log2 g clamped at -126), with every range product prod_{x<=u<=y} g_u = 2^(L_y - L_{x-1})
// taken as one exponent, and the query-key term of dg by the recurrence
// K_{t+1}[r] = g_t K_t[r] + A2[r,t] k_t. (The derivation, both routes, is checked against the
// oracle's step-by-step reverse sweep on the CPU.)
//
// Three launches:
//   1. gla_bwd_contrib_kernel, one CTA per (b, h, chunk): U = k^^T V and U' = q~^T dO (the
//      chunk's contributions to the state and to its gradient) and the chunk decay a;
//   2. gla_bwd_scan_kernel: S_in of every chunk (forward over chunks from the initial state)
//      and E of every chunk (backward from the final-state gradient), stored in bf16; the
//      gradient of the initial state;
//   3. gla_bwd_grad_kernel, one CTA per (b, h, chunk): the eight products above on the tensor
//      cores, every one of them TRANSPOSED (key or value channel in the TMEM lane, token in the
//      column), so that a thread owns one channel over the chunk's 64 tokens and the sums over
//      t that dg needs are plain loops; then dq, dk, dv, dg through shared memory and TMA stores.
#include <cuda.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace rod {
namespace {

__device__ unsigned int g_gla_bwd_timeout = 0;

constexpr int C = 64;
constexpr int D = 128;
constexpr int BOX = C * 128;        // a 64-row box of 128-byte rows (8 KB)
constexpr int BOX128 = D * 128;     // a 128-row box (16 KB)
constexpr float kFastMin = 8.673617e-19f;   // 2^-60: smallest chunk decay of the product form
constexpr float kGateMin = 3.90625e-3f;     // 2^-8: smallest gate the product form divides by
constexpr float kLog2Floor = -126.0f;

// TMEM columns of the gradient kernel
constexpr uint32_t TM_X1 = 0, TM_X2 = 64, TM_X3 = 128, TM_X4 = 192, TM_DV = 256, TM_A2 = 320, TM_QK = 384;

struct BwdArgs {
    int T, NC;                  // tokens, chunks per (b, h)
    float* U;                   // [BH][NC][D][D] fp32  k^^T V
    float* U2;                  // [BH][NC][D][D] fp32  q~^T dO
    float* A;                   // [BH][NC][D]    fp32  chunk decay
    __nv_bfloat16* SIN;         // [BH][NC][D][D] bf16  incoming state S_in[c][j]
    __nv_bfloat16* EE;          // [BH][NC][D][D] bf16  E[c][j]
    const float* state0;        // [BH][D][D]
    const float* dstate_final;  // [BH][D][D] or null
    float* dstate0;             // [BH][D][D]
    // the gradient kernel's inputs, for its L2 prefetch of the chunk one wave ahead
    const __nv_bfloat16 *q, *k, *v, *dO;
    const float* g;
    int wave;                   // CTAs resident at once (0: no prefetch)
};

// ---- small helpers ---------------------------------------------------------------------------
__device__ __forceinline__ uint64_t pk2(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ float2 upk2(uint64_t r) {
    float2 d;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(d.x), "=f"(d.y) : "l"(r));
    return d;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint32_t pack2(uint64_t x) {
    const float2 f = upk2(x);
    return pack_bf16x2(f.x, f.y);
}
__device__ __forceinline__ uint64_t unpack2(uint32_t w) { return pk2(bf16lo(w), bf16hi(w)); }
__device__ __forceinline__ float rcp(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float lg2(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float ldbf(const unsigned char* p) {
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(p));
}
template <typename T> __device__ __forceinline__ T& at(unsigned char* base, uint32_t off) {
    return *reinterpret_cast<T*>(base + off);
}
// byte offset of the 16-byte chunk holding columns [col, col + 8) of row `row` in a K-major
// 128-byte-swizzled bf16 tile whose 64-column boxes hold `rows` rows each (col % 8 == 0)
__device__ __forceinline__ uint32_t sw_off(int row, int col, int rows) {
    const int box = col >> 6, cc = col & 63;
    return (uint32_t)(box * rows * 128 + row * 128 + ((((cc >> 3) ^ (row & 7))) << 4));
}
__device__ __forceinline__ uint32_t sw_off_elem(int row, int col, int rows) {
    return sw_off(row, col & ~7, rows) + ((col & 7) << 1);
}
__device__ __forceinline__ uint4 pack8(const float* f) {
    uint4 u;
    u.x = pack_bf16x2(f[0], f[1]); u.y = pack_bf16x2(f[2], f[3]);
    u.z = pack_bf16x2(f[4], f[5]); u.w = pack_bf16x2(f[6], f[7]);
    return u;
}

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 0) {
            if (*abort_flag) return false;
            if (i >= kWaitLimit) {
                *abort_flag = 1;
                atomicExch(&g_gla_bwd_timeout, 1u);
                return false;
            }
        }
    }
}
__device__ __forceinline__ void bar_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ bool bar_all(int id, int n, bool pred) {
    uint32_t out;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %2, 0;\n\t"
        "bar.red.and.pred q, %1, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(out) : "r"(id), "r"((uint32_t)pred), "r"(n) : "memory");
    return out != 0;
}

// Per-thread part of the chunk's gate products, shared by the contribution and gradient kernels.
// Thread (channel pair p: channels 2p, 2p+1; row quarter qr: rows 16qr .. 16qr+15) of `nthr` =
// 256 operand threads (named barrier `bid`). Loads its 16 gate pairs (rows past nvalid are 1),
// publishes its quarter product through `scan` ([4][128] fp32) and returns the product of the
// quarters before it (pre) and of the whole chunk (a).
struct GateSweep {
    uint64_t g2[16];
    uint64_t pre, a;
};
__device__ __forceinline__ void gate_products(GateSweep& gs, const unsigned char* gsm, float* scan, int p,
                                              int qr, int nvalid, int bid) {
    const int c0 = 2 * p, r0 = 16 * qr;
    uint64_t prod = pk2(1.f, 1.f);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int t = r0 + i;
        gs.g2[i] = t < nvalid ? *reinterpret_cast<const uint64_t*>(gsm + t * 512 + p * 8) : pk2(1.f, 1.f);
        prod = mul2(prod, gs.g2[i]);
    }
    *reinterpret_cast<uint64_t*>(scan + qr * D + c0) = prod;
    bar_sync(bid, 256);
    gs.pre = pk2(1.f, 1.f);
    gs.a = pk2(1.f, 1.f);
#pragma unroll
    for (int q2 = 0; q2 < 4; ++q2) {
        const uint64_t v = *reinterpret_cast<const uint64_t*>(scan + q2 * D + c0);
        if (q2 < qr) gs.pre = mul2(gs.pre, v);
        gs.a = mul2(gs.a, v);
    }
}
// exact route: g2 turned into clamped log2 gates, prefix sums through `scan` (the caller has
// passed a barrier since scan was last read); returns preL (sum of the quarters before) and Ltot
__device__ __forceinline__ void gate_logs(GateSweep& gs, float* scan, int p, int qr, int nvalid, int bid,
                                          uint64_t& preL, uint64_t& Ltot) {
    const int c0 = 2 * p, r0 = 16 * qr;
    uint64_t lsum = pk2(0.f, 0.f);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float2 gg = upk2(gs.g2[i]);
        gs.g2[i] = r0 + i < nvalid ? pk2(fmaxf(lg2(gg.x), kLog2Floor), fmaxf(lg2(gg.y), kLog2Floor))
                                   : pk2(0.f, 0.f);
        lsum = add2(lsum, gs.g2[i]);
    }
    *reinterpret_cast<uint64_t*>(scan + qr * D + c0) = lsum;
    bar_sync(bid, 256);
    preL = pk2(0.f, 0.f);
    Ltot = pk2(0.f, 0.f);
#pragma unroll
    for (int q2 = 0; q2 < 4; ++q2) {
        const uint64_t v = *reinterpret_cast<const uint64_t*>(scan + q2 * D + c0);
        if (q2 < qr) preL = add2(preL, v);
        Ltot = add2(Ltot, v);
    }
}

// ================================================================================================
// 1. chunk contributions: U = k^^T V, U' = q~^T dO, a
// ================================================================================================
constexpr int CA_Q = 0, CA_K = 2 * BOX, CA_V = 4 * BOX, CA_DO = 6 * BOX, CA_G = 8 * BOX;
constexpr int CA_SCAN = 12 * BOX;
constexpr int CA_BAR = CA_SCAN + 4 * D * 4;
constexpr int CA_MISC = CA_BAR + 32;
constexpr int CA_SMEM = CA_MISC + 32 + 1024;
constexpr int CA_STAGE = 32 * 32 * 4;   // one 32 x 32 fp32 tile of U or U' on its way out
static_assert(8 * 2 * CA_STAGE <= CA_G - CA_Q, "two staging tiles per warp fit over q, k, v, dO");

__global__ void __launch_bounds__(256, 2)
gla_bwd_contrib_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                       const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_u,
                       const __grid_constant__ CUtensorMap tm_u2, BwdArgs args) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32, tid = threadIdx.x;
    const int n = blockIdx.x, bh = blockIdx.y;
    const int t0 = n * C;
    const int nvalid = min(C, args.T - t0);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + CA_BAR);
    uint64_t* mma = full + 1;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + CA_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + CA_MISC + 4);
    float* scan = reinterpret_cast<float*>(smem + CA_SCAN);
    if (tid == 0) {
        mbar_init(full, 1);
        mbar_init(mma, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tc::tmem_alloc(tmem_holder, 256);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_holder;
    if (tid == 0) {
        mbar_arrive_expect_tx(full, 12 * BOX);
        for (int h = 0; h < 2; ++h) {
            tc::tma_load_3d(smem + CA_Q + h * BOX, &tm_q, h * 64, t0, bh, full);
            tc::tma_load_3d(smem + CA_K + h * BOX, &tm_k, h * 64, t0, bh, full);
            tc::tma_load_3d(smem + CA_V + h * BOX, &tm_v, h * 64, t0, bh, full);
            tc::tma_load_3d(smem + CA_DO + h * BOX, &tm_do, h * 64, t0, bh, full);
        }
        tc::tma_load_3d(smem + CA_G, &tm_g, 0, t0, bh, full);
    }
    const bool ok = __syncthreads_and(wait_bar(full, 0, abort_flag));
    if (ok) {
        const int p = tid & 63, qr = tid >> 6, c0 = 2 * p, r0 = 16 * qr;
        const uint32_t b16_base = (uint32_t)((p >> 5) * BOX + ((p & 3) * 4));
        const uint32_t b16_chunk = (uint32_t)((p & 31) >> 2);
        auto off16 = [&](int t) { return b16_base + (uint32_t)t * 128u + (((b16_chunk ^ (uint32_t)(t & 7))) << 4); };
        GateSweep gs;
        gate_products(gs, smem + CA_G, scan, p, qr, nvalid, 0);
        float2 af = upk2(gs.a);
        const bool fast = __syncthreads_and(af.x >= kFastMin && af.y >= kFastMin);
        if (fast) {  // k^ = k . a/G over k, q~ = q . G over q
            uint64_t G = gs.pre;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int t = r0 + i;
                G = mul2(G, gs.g2[i]);
                const float2 gf = upk2(G);
                const uint64_t aG = mul2(gs.a, pk2(rcp(gf.x), rcp(gf.y)));
                at<uint32_t>(smem, CA_K + off16(t)) = pack2(mul2(unpack2(at<uint32_t>(smem, CA_K + off16(t))), aG));
                at<uint32_t>(smem, CA_Q + off16(t)) = pack2(mul2(unpack2(at<uint32_t>(smem, CA_Q + off16(t))), G));
            }
        } else {     // k^ = k . 2^(Ltot - L), q~ = q . 2^L
            uint64_t preL, Ltot;
            gate_logs(gs, scan, p, qr, nvalid, 0, preL, Ltot);
            const float2 lt = upk2(Ltot);
            gs.a = pk2(tc::ex2(lt.x), tc::ex2(lt.y));
            uint64_t L = preL;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int t = r0 + i;
                L = add2(L, gs.g2[i]);
                const float2 lf = upk2(L);
                const float2 kf = upk2(unpack2(at<uint32_t>(smem, CA_K + off16(t))));
                const float2 qf = upk2(unpack2(at<uint32_t>(smem, CA_Q + off16(t))));
                at<uint32_t>(smem, CA_K + off16(t)) =
                    pack_bf16x2(kf.x * tc::ex2(lt.x - lf.x), kf.y * tc::ex2(lt.y - lf.y));
                at<uint32_t>(smem, CA_Q + off16(t)) = pack_bf16x2(qf.x * tc::ex2(lf.x), qf.y * tc::ex2(lf.y));
            }
        }
        if (qr == 0)
            *reinterpret_cast<uint64_t*>(args.A + ((int64_t)bh * args.NC + n) * D + c0) = gs.a;
        tc::fence_proxy_async();
    }
    __syncthreads();
    if (ok && warp == 0) {
        tc::fence_after_sync();
        const uint32_t idesc = tc::idesc_bf16_f32(128, 128, 1, 1);
        const uint32_t hi = tc::desc_hi(tc::sdesc_sw128(smem_u32(smem), BOX, 1024));
        const uint32_t k_lo = tc::desc_lo(tc::sdesc_sw128(smem_u32(smem + CA_K), BOX, 1024));
        const uint32_t v_lo = tc::desc_lo(tc::sdesc_sw128(smem_u32(smem + CA_V), BOX, 1024));
        const uint32_t q_lo = tc::desc_lo(tc::sdesc_sw128(smem_u32(smem + CA_Q), BOX, 1024));
        const uint32_t o_lo = tc::desc_lo(tc::sdesc_sw128(smem_u32(smem + CA_DO), BOX, 1024));
#pragma unroll
        for (int k = 0; k < C / 16; ++k)
            tc::mma_ss_lh_warp(tmem, k_lo + 128u * k, hi, v_lo + 128u * k, hi, idesc, k > 0);
#pragma unroll
        for (int k = 0; k < C / 16; ++k)
            tc::mma_ss_lh_warp(tmem + 128, q_lo + 128u * k, hi, o_lo + 128u * k, hi, idesc, k > 0);
        tc::mma_commit_warp(mma);
    }
    if (ok && __syncthreads_and(wait_bar(mma, 0, abort_flag))) {
        tc::fence_after_sync();
        // warps 0-3: U rows, warps 4-7: U' rows (row c = TMEM lane). A warp moves 32 rows x 32
        // columns at a time through shared memory (the operand tiles are free once the MMAs are
        // done): each thread writes its row with the 128-byte swizzle, so the eight 16-byte pieces
        // of a quarter-warp land in distinct banks, and one lane stores the tile with TMA. Direct
        // row-per-thread global stores would touch 32 lines per instruction and back up the
        // load/store queue.
        const int rw = 32 * (warp & 3);
        const uint32_t col0 = warp < 4 ? 0u : 128u;
        const CUtensorMap* tm = warp < 4 ? &tm_u : &tm_u2;
        unsigned char* stage = smem + CA_Q + warp * (2 * CA_STAGE);
        const int z = bh * args.NC + n;
#pragma unroll
        for (int cb = 0; cb < D; cb += 32) {
            unsigned char* buf = stage + ((cb / 32) & 1) * CA_STAGE;
            uint32_t r[32];
            tc::tmem_ld32(tmem + col0 + cb + ((uint32_t)rw << 16), r);
            if (cb >= 64 && lane == 0) tc::bulk_wait_read_1();  // the store two tiles back has read buf
            __syncwarp();
            tc::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 8; ++j)
                *reinterpret_cast<uint4*>(buf + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                    make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
            tc::fence_proxy_async();
            __syncwarp();
            if (lane == 0) {
                tc::tma_store_3d(tm, buf, cb, rw, z);
                tc::bulk_commit();
            }
        }
        if (lane == 0) tc::bulk_wait_read();
        __syncwarp();
    } else if (ok && warp == 0) {
        // the MMAs were issued but did not complete in time: wait once more before TMEM is freed
        mbar_wait_bounded(mma, 0, kWaitLimit);
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 0) tc::tmem_dealloc(tmem, 256);
}

// ================================================================================================
// 2. scans over chunks: S_in (forward), E (backward), dstate0
// ================================================================================================
__global__ void __launch_bounds__(256)
gla_bwd_scan_kernel(BwdArgs args) {
    const int64_t bh = blockIdx.y;
    const int e4 = blockIdx.x * blockDim.x + threadIdx.x;  // float4 index in the D x D state
    if (e4 >= D * D / 4) return;
    const int c = (e4 * 4) / D;
    const int NC = args.NC;
    const size_t slot = (size_t)D * D;
    const int64_t base = bh * NC;
    float4 S = reinterpret_cast<const float4*>(args.state0 + bh * slot)[e4];
    float4 u_next = reinterpret_cast<const float4*>(args.U + base * slot)[e4];
    for (int n = 0; n < NC; ++n) {
        const float4 u = u_next;
        if (n + 1 < NC) u_next = reinterpret_cast<const float4*>(args.U + (base + n + 1) * slot)[e4];
        const float an = args.A[(base + n) * D + c];
        uint2 w;
        w.x = pack_bf16x2(S.x, S.y);
        w.y = pack_bf16x2(S.z, S.w);
        reinterpret_cast<uint2*>(args.SIN + (base + n) * slot)[e4] = w;
        S.x = fmaf(an, S.x, u.x);
        S.y = fmaf(an, S.y, u.y);
        S.z = fmaf(an, S.z, u.z);
        S.w = fmaf(an, S.w, u.w);
    }
    float4 E = args.dstate_final ? reinterpret_cast<const float4*>(args.dstate_final + bh * slot)[e4]
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
    u_next = reinterpret_cast<const float4*>(args.U2 + (base + NC - 1) * slot)[e4];
    for (int n = NC - 1; n >= 0; --n) {
        const float4 u = u_next;
        if (n > 0) u_next = reinterpret_cast<const float4*>(args.U2 + (base + n - 1) * slot)[e4];
        const float an = args.A[(base + n) * D + c];
        uint2 w;
        w.x = pack_bf16x2(E.x, E.y);
        w.y = pack_bf16x2(E.z, E.w);
        reinterpret_cast<uint2*>(args.EE + (base + n) * slot)[e4] = w;
        E.x = fmaf(an, E.x, u.x);
        E.y = fmaf(an, E.y, u.y);
        E.z = fmaf(an, E.z, u.z);
        E.w = fmaf(an, E.w, u.w);
    }
    reinterpret_cast<float4*>(args.dstate0 + bh * slot)[e4] = E;
}

// ================================================================================================
// 3. gradients of one chunk
// ================================================================================================
// shared memory (1024-aligned regions); after the last MMA the staging of the outputs reuses
// regions whose operands are done: dq over V, dk over DO, dv over K, dg over Q|KT, and the two
// partial sums of dg over S_in and E
constexpr int GB_Q = 0;              // q -> q~ (bf16); raw q on the exact route
constexpr int GB_KT = 2 * BOX;       // k~ (bf16); raw k on the exact route
constexpr int GB_K = 4 * BOX;        // k -> k^
constexpr int GB_V = 6 * BOX;
constexpr int GB_DO = 8 * BOX;
constexpr int GB_G = 10 * BOX;       // g (fp32 [64][128]); L over it on the exact route
constexpr int GB_SIN = 14 * BOX;     // S_in bf16 [c][j] (two 128-row boxes)
constexpr int GB_E = 18 * BOX;       // E bf16 [c][j]
constexpr int GB_A2M = 22 * BOX;     // M(A2) bf16 [t][s] (one box)
constexpr int GB_QKM = 23 * BOX;     // M(QK) bf16 [t][s]
constexpr int GB_SCAN = 24 * BOX;    // [4][128] fp32
constexpr int GB_RHO = GB_SCAN + 4 * D * 4;
constexpr int GB_AB = GB_RHO + D * 4;
constexpr int GB_FLAG = GB_AB + D * 4;
constexpr int GB_BAR = GB_FLAG + 16;
constexpr int GB_MISC = GB_BAR + 8 * 8;
constexpr int GB_SMEM = GB_MISC + 32 + 1024;
static_assert(GB_SMEM <= 232448, "shared memory per CTA");

__global__ void __launch_bounds__(512, 1)
gla_bwd_grad_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_sin,
                    const __grid_constant__ CUtensorMap tm_e, const __grid_constant__ CUtensorMap tm_dq,
                    const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                    const __grid_constant__ CUtensorMap tm_dg, BwdArgs args) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32, tid = threadIdx.x;
    const int n = blockIdx.x, bh = blockIdx.y;
    const int t0 = n * C;
    const int nvalid = min(C, args.T - t0);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + GB_BAR);
    uint64_t* full = bars;       // TMA -> everyone
    uint64_t* ops = bars + 1;    // operands ready (8 warps) -> issuer
    uint64_t* mma1 = bars + 2;   // A2, QK, X1, X4 done -> masks
    uint64_t* masks = bars + 3;  // M(A2), M(QK) in shared memory (4 warps) -> issuer
    uint64_t* mma2 = bars + 4;   // every MMA done -> epilogue
    uint64_t* drain = bars + 5;  // issuer: every MMA done before TMEM is freed
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + GB_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + GB_MISC + 4);
    volatile int* flag = reinterpret_cast<volatile int*>(smem + GB_FLAG);
    float* scan = reinterpret_cast<float*>(smem + GB_SCAN);
    float* rho = reinterpret_cast<float*>(smem + GB_RHO);
    float* abuf = reinterpret_cast<float*>(smem + GB_AB);
    if (tid == 0) {
        mbar_init(full, 1);
        mbar_init(ops, 8);
        mbar_init(mma1, 1);
        mbar_init(masks, 4);
        mbar_init(mma2, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tc::tmem_alloc(tmem_holder, 512);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_holder;
    const int zc = bh * args.NC + n;   // chunk index in the S_in / E stacks

    if (warp < 4) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(56));
        if (warp == 0 && lane == 0) {
            mbar_arrive_expect_tx(full, 20 * BOX);
            for (int h = 0; h < 2; ++h) {
                tc::tma_load_3d(smem + GB_Q + h * BOX, &tm_q, h * 64, t0, bh, full);
                tc::tma_load_3d(smem + GB_K + h * BOX, &tm_k, h * 64, t0, bh, full);
                tc::tma_load_3d(smem + GB_V + h * BOX, &tm_v, h * 64, t0, bh, full);
                tc::tma_load_3d(smem + GB_DO + h * BOX, &tm_do, h * 64, t0, bh, full);
                tc::tma_load_3d(smem + GB_SIN + h * BOX128, &tm_sin, h * 64, 0, zc, full);
                tc::tma_load_3d(smem + GB_E + h * BOX128, &tm_e, h * 64, 0, zc, full);
            }
            tc::tma_load_3d(smem + GB_G, &tm_g, 0, t0, bh, full);
            // CTAs start in linear order, one per SM: the chunk one wave later streams into L2
            // while this one computes, so its copies come from L2 instead of waiting on HBM
            const int64_t nxt = (int64_t)blockIdx.y * gridDim.x + blockIdx.x + args.wave;
            if (args.wave > 0 && nxt < (int64_t)gridDim.x * gridDim.y) {
                const int n2 = (int)(nxt % gridDim.x), bh2 = (int)(nxt / gridDim.x);
                const int t2 = n2 * C;
                const uint32_t rows = (uint32_t)min(C, args.T - t2);
                const int64_t row0 = (int64_t)bh2 * args.T + t2;
                const int64_t z2 = (int64_t)bh2 * args.NC + n2;
                tc::prefetch_l2(args.q + row0 * D, rows * D * 2);
                tc::prefetch_l2(args.k + row0 * D, rows * D * 2);
                tc::prefetch_l2(args.v + row0 * D, rows * D * 2);
                tc::prefetch_l2(args.dO + row0 * D, rows * D * 2);
                tc::prefetch_l2(args.g + row0 * D, rows * D * 4);
                tc::prefetch_l2(args.SIN + z2 * D * D, D * D * 2);
                tc::prefetch_l2(args.EE + z2 * D * D, D * D * 2);
            }
            mbar_wait_bounded(full, 0, kWaitLimit);  // copies land before the CTA can leave
        } else if (warp == 1) {
            // ------------------------------ MMA issuer ------------------------------
            auto wait_all = [&](uint64_t* bar) {
                return __all_sync(0xffffffffu, wait_bar(bar, 0, abort_flag)) != 0;
            };
            if (wait_all(ops)) {
                tc::fence_after_sync();
                const bool fast = flag[0] == 0;
                const uint32_t hi = tc::desc_hi(tc::sdesc_sw128(smem_u32(smem), 16, 1024));
                auto dlo = [&](int off, uint32_t lbo) { return tc::desc_lo(tc::sdesc_sw128(smem_u32(smem + off), lbo, 1024)); };
                // K-major koff for a K step of 16 bf16 in 64-row boxes / 128-row boxes
                auto koff64 = [](int k) { return (uint32_t)(((k / 4) * BOX + (k % 4) * 32) >> 4); };
                auto koff128 = [](int k) { return (uint32_t)(((k / 4) * BOX128 + (k % 4) * 32) >> 4); };
                const uint32_t id64 = tc::idesc_bf16_f32(64, 64, 0, 0);
                const uint32_t idKK = tc::idesc_bf16_f32(128, 64, 0, 0);
                const uint32_t idMK = tc::idesc_bf16_f32(128, 64, 1, 0);
                const uint32_t idMM = tc::idesc_bf16_f32(128, 64, 1, 1);
                // group 1: A2 = dO V^T, QK = q~ k~^T (M = 64); X1^T = S_in dO^T, X4^T = E V^T
#pragma unroll
                for (int k = 0; k < D / 16; ++k)
                    tc::mma_ss_lh_warp(tmem + TM_A2, dlo(GB_DO, 16) + koff64(k), hi, dlo(GB_V, 16) + koff64(k), hi, id64, k > 0);
                if (fast) {
#pragma unroll
                    for (int k = 0; k < D / 16; ++k)
                        tc::mma_ss_lh_warp(tmem + TM_QK, dlo(GB_Q, 16) + koff64(k), hi, dlo(GB_KT, 16) + koff64(k), hi, id64,
                                           k > 0);
                }
#pragma unroll
                for (int k = 0; k < D / 16; ++k)
                    tc::mma_ss_lh_warp(tmem + TM_X1, dlo(GB_SIN, 16) + koff128(k), hi, dlo(GB_DO, 16) + koff64(k), hi,
                                       idKK, k > 0);
#pragma unroll
                for (int k = 0; k < D / 16; ++k)
                    tc::mma_ss_lh_warp(tmem + TM_X4, dlo(GB_E, 16) + koff128(k), hi, dlo(GB_V, 16) + koff64(k), hi,
                                       idKK, k > 0);
                tc::mma_commit_warp(mma1);
                if (wait_all(masks)) {
                    tc::fence_after_sync();
                    // group 2 (K = 64 tokens; MN-major operands step 16 rows = 2048 bytes)
                    if (fast) {
                        // X2^T = k~^T M(A2)^T;  X3^T = q~^T M(A2)
#pragma unroll
                        for (int k = 0; k < C / 16; ++k)
                            tc::mma_ss_lh_warp(tmem + TM_X2, dlo(GB_KT, BOX) + 128u * k, hi, dlo(GB_A2M, 16) + 2u * k, hi,
                                               idMK, k > 0);
#pragma unroll
                        for (int k = 0; k < C / 16; ++k)
                            tc::mma_ss_lh_warp(tmem + TM_X3, dlo(GB_Q, BOX) + 128u * k, hi, dlo(GB_A2M, BOX) + 128u * k, hi,
                                               idMM, k > 0);
                    }
                    // dv^T = dO^T M(QK) + E^T k^^T
#pragma unroll
                    for (int k = 0; k < C / 16; ++k)
                        tc::mma_ss_lh_warp(tmem + TM_DV, dlo(GB_DO, BOX) + 128u * k, hi, dlo(GB_QKM, BOX) + 128u * k, hi,
                                           idMM, k > 0);
#pragma unroll
                    for (int k = 0; k < D / 16; ++k)
                        tc::mma_ss_lh_warp(tmem + TM_DV, dlo(GB_E, BOX128) + 128u * k, hi, dlo(GB_K, 16) + koff64(k), hi,
                                           idMK, 1u);
                    tc::mma_commit_warp(mma2);
                }
            }
            tc::mma_commit_warp(drain);
            mbar_wait_bounded(drain, 0, kWaitLimit);
        }
    } else if (warp < 12) {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(152));
        // ------------------------------ operand warps, then dq / dk / dg ------------------------------
        const int ot = tid - 128;
        const int p = ot & 63, qr = ot >> 6;
        const int c0 = 2 * p, r0 = 16 * qr;
        const int wq = warp & 3, half = (warp - 4) >> 2;
        const uint32_t lane_base = (uint32_t)(32 * wq) << 16;
        const uint32_t b16_base = (uint32_t)((p >> 5) * BOX + ((p & 3) * 4));
        const uint32_t b16_chunk = (uint32_t)((p & 31) >> 2);
        auto off16 = [&](int t) { return b16_base + (uint32_t)t * 128u + (((b16_chunk ^ (uint32_t)(t & 7))) << 4); };
        bool ok = bar_all(1, 256, wait_bar(full, 0, abort_flag));
        bool fast = true;
        if (ok) {
            GateSweep gs;
            gate_products(gs, smem + GB_G, scan, p, qr, nvalid, 1);
            const float2 af = upk2(gs.a);
            bool mine = af.x >= kFastMin && af.y >= kFastMin;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float2 gg = upk2(gs.g2[i]);
                mine = mine && gg.x >= kGateMin && gg.y >= kGateMin;
            }
            fast = bar_all(1, 256, mine);
            if (fast) {  // q~ = q.G over q, k~ = k/G beside, k^ = k~.a over k
                uint64_t G = gs.pre;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int t = r0 + i;
                    G = mul2(G, gs.g2[i]);
                    const float2 gf = upk2(G);
                    const uint64_t kt = mul2(unpack2(at<uint32_t>(smem, GB_K + off16(t))), pk2(rcp(gf.x), rcp(gf.y)));
                    at<uint32_t>(smem, GB_KT + off16(t)) = pack2(kt);
                    at<uint32_t>(smem, GB_K + off16(t)) = pack2(mul2(kt, gs.a));
                    at<uint32_t>(smem, GB_Q + off16(t)) = pack2(mul2(unpack2(at<uint32_t>(smem, GB_Q + off16(t))), G));
                }
                if (qr == 0) *reinterpret_cast<uint64_t*>(abuf + c0) = gs.a;
            } else {
                // exact route: L over the gates, exact scores into TMEM, raw k beside, k^ over k
                uint64_t preL, Ltot;
                gate_logs(gs, scan, p, qr, nvalid, 1, preL, Ltot);
                uint64_t L = preL;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    L = add2(L, gs.g2[i]);
                    at<uint64_t>(smem, GB_G + (uint32_t)((r0 + i) * 512 + p * 8)) = L;
                    at<uint32_t>(smem, GB_KT + off16(r0 + i)) = at<uint32_t>(smem, GB_K + off16(r0 + i));
                }
                bar_sync(1, 256);
                const int t = 16 * wq + lane;  // score row (lanes 0-15)
                const float* Lg = reinterpret_cast<const float*>(smem + GB_G);
                float acc[32];
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) acc[jj] = 0.f;
                if (lane < 16) {
                    for (int cc = 0; cc < D; ++cc) {
                        const float qc = ldbf(smem + GB_Q + sw_off_elem(t, cc, C));
                        const float Lt = Lg[t * D + cc];
#pragma unroll
                        for (int jj = 0; jj < 32; ++jj) {
                            const int s = 32 * half + jj;
                            if (s <= t)
                                acc[jj] = fmaf(qc * ldbf(smem + GB_KT + sw_off_elem(s, cc, C)), tc::ex2(Lt - Lg[s * D + cc]),
                                               acc[jj]);
                        }
                    }
                }
                uint32_t ar[32];
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) ar[jj] = __float_as_uint(acc[jj]);
                tc::tmem_st32(tmem + TM_QK + 32u * half + lane_base, ar);
                tc::tmem_wait_st();
                bar_sync(1, 256);  // k read by every thread before k^ overwrites it
                const float2 lt = upk2(Ltot);
                L = preL;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int t2 = r0 + i;
                    L = add2(L, gs.g2[i]);
                    const float2 lf = upk2(L);
                    const float2 kf = upk2(unpack2(at<uint32_t>(smem, GB_KT + off16(t2))));
                    at<uint32_t>(smem, GB_K + off16(t2)) =
                        pack_bf16x2(kf.x * tc::ex2(lt.x - lf.x), kf.y * tc::ex2(lt.y - lf.y));
                }
                if (qr == 0) *reinterpret_cast<uint64_t*>(abuf + c0) = pk2(tc::ex2(lt.x), tc::ex2(lt.y));
            }
            if (ot == 0) flag[0] = fast ? 0 : 1;
            tc::fence_proxy_async();
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(ops);
            ok = bar_all(1, 256, wait_bar(mma2, 0, abort_flag));
        }
        if (ok) {
            bar_sync(3, 384);  // rho, written by warps 12-15 (which arrive here once), is visible
            tc::fence_after_sync();
            // thread = key channel c (TMEM lane), WG1 (half 0): dq and the query sums of dg,
            // WG2 (half 1): dk and the key sums of dg
            const int c = 32 * wq + lane;
            const float ac = abuf[c];
            const float* gcol = reinterpret_cast<const float*>(smem + GB_G) + c;  // g[t][c] (or L) at t * D
            float* T1 = reinterpret_cast<float*>(smem + GB_SIN);  // [t][c] fp32
            float* T2 = reinterpret_cast<float*>(smem + GB_E);
            __nv_bfloat16* stq = reinterpret_cast<__nv_bfloat16*>(smem + GB_V);
            __nv_bfloat16* stk = reinterpret_cast<__nv_bfloat16*>(smem + GB_DO);
            const uint32_t xa = tmem + lane_base + (half == 0 ? TM_X1 : TM_X3);
            const uint32_t xb = tmem + lane_base + (half == 0 ? TM_X2 : TM_X4);
            if (fast) {
                // reverse over t with F_t = prod_{t<u<C} g_u, so G_t = a / F_t and 1/G_t = F_t / a
                float F = 1.f, acc1 = 0.f, acc3 = 0.f;
                const float ra = rcp(ac);
                for (int hh = 1; hh >= 0; --hh) {
                    uint32_t ra_[32], rb_[32];
                    tc::tmem_ld32(xa + 32u * hh, ra_);
                    tc::tmem_ld32(xb + 32u * hh, rb_);
                    tc::tmem_wait_ld();
                    // eight tokens' operands and gates are loaded ahead of their arithmetic: the
                    // compiler cannot move a shared-memory load above the previous token's
                    // shared-memory stores, so a load per token would pay its latency every token
#pragma unroll
                    for (int i0 = 24; i0 >= 0; i0 -= 8) {
                        float opv[8], gv[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const int t = 32 * hh + i0 + j;
                            opv[j] = ldbf(smem + (half == 0 ? GB_Q : GB_KT) + sw_off_elem(t, c, C));
                            gv[j] = t < nvalid ? gcol[t * D] : 1.f;
                        }
#pragma unroll
                        for (int j = 7; j >= 0; --j) {
                            const int i = i0 + j, t = 32 * hh + i;
                            const float x_a = __uint_as_float(ra_[i]), x_b = __uint_as_float(rb_[i]);
                            if (half == 0) {
                                stq[t * D + c] = __float2bfloat16_rn((x_a + x_b) * (ac * rcp(F)));
                                acc1 = fmaf(opv[j], x_a + x_b, acc1);
                                T1[t * D + c] = acc1;
                            } else {
                                stk[t * D + c] = __float2bfloat16_rn(fmaf(ac, x_b, x_a) * (F * ra));
                                acc3 = fmaf(opv[j], x_a, acc3);
                                T2[t * D + c] = -acc3;
                            }
                            F *= gv[j];
                        }
                    }
                }
                if (half == 1) {
                    // forward over t: a . sum_{s<t} k~_s X4_s joins the key sums
                    float ex = 0.f;
                    for (int hh = 0; hh < 2; ++hh) {
                        uint32_t rb_[32];
                        tc::tmem_ld32(xb + 32u * hh, rb_);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int i0 = 0; i0 < 32; i0 += 8) {
                            float t2v[8], kv[8];
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                const int t = 32 * hh + i0 + j;
                                t2v[j] = T2[t * D + c];
                                kv[j] = ldbf(smem + GB_KT + sw_off_elem(t, c, C));
                            }
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                const int t = 32 * hh + i0 + j;
                                T2[t * D + c] = fmaf(ac, ex, t2v[j]);
                                ex = fmaf(kv[j], __uint_as_float(rb_[i0 + j]), ex);
                            }
                        }
                    }
                }
            } else {
                // exact route: every range product 2^(L_y - L_{x-1}) as one exponent
                const float* Lc = gcol;  // L[t][c] at t * D
                const float Ltot = Lc[(C - 1) * D];
                if (half == 0) {
                    uint32_t x1[64];
                    tc::tmem_ld32(xa, x1);
                    tc::tmem_ld32(xa + 32, x1 + 32);
                    tc::tmem_wait_ld();
                    for (int t = 0; t < C; ++t) {
                        const float Lt = Lc[t * D];
                        float acc = __uint_as_float(x1[t]) * tc::ex2(Lt);
                        for (int s = 0; s <= t; ++s)
                            acc = fmaf(ldbf(smem + GB_A2M + sw_off_elem(t, s, C)) * ldbf(smem + GB_KT + sw_off_elem(s, c, C)),
                                       tc::ex2(Lt - Lc[s * D]), acc);
                        stq[t * D + c] = __float2bfloat16_rn(acc);
                        // AE_t + BE_t
                        const float Lp = t > 0 ? Lc[(t - 1) * D] : 0.f;
                        float ae = tc::ex2(Ltot - Lt + Lp) * rho[c];
                        for (int r = t; r < C; ++r)
                            ae = fmaf(tc::ex2(Lp + Lc[r * D] - Lt) * ldbf(smem + GB_Q + sw_off_elem(r, c, C)),
                                      __uint_as_float(x1[r]), ae);
                        T1[t * D + c] = ae;
                    }
                } else {
                    uint32_t x4[64];
                    tc::tmem_ld32(xb, x4);
                    tc::tmem_ld32(xb + 32, x4 + 32);
                    tc::tmem_wait_ld();
                    for (int s = 0; s < C; ++s) {
                        const float Ls = Lc[s * D];
                        float acc = __uint_as_float(x4[s]) * tc::ex2(Ltot - Ls);
                        for (int t = s; t < C; ++t)
                            acc = fmaf(ldbf(smem + GB_A2M + sw_off_elem(t, s, C)) * ldbf(smem + GB_Q + sw_off_elem(t, c, C)),
                                       tc::ex2(Lc[t * D] - Ls), acc);
                        stk[s * D + c] = __float2bfloat16_rn(acc);
                    }
                    for (int t = 0; t < C; ++t) {  // BF_t
                        const float Lt = Lc[t * D], Lp = t > 0 ? Lc[(t - 1) * D] : 0.f;
                        float bf = 0.f;
                        for (int s = 0; s < t; ++s)
                            bf = fmaf(tc::ex2(Ltot - Lt + Lp - Lc[s * D]) * ldbf(smem + GB_KT + sw_off_elem(s, c, C)),
                                      __uint_as_float(x4[s]), bf);
                        T2[t * D + c] = bf;
                    }
                    // AF_t = sum_{r>=t} P(t+1, r) q_r K_t[r], K_{t+1}[r] = g_t K_t[r] + A2[r, t] k_t
                    float Kr[C];
#pragma unroll
                    for (int r = 0; r < C; ++r) Kr[r] = 0.f;
                    for (int t = 0; t < C; ++t) {
                        float af = 0.f, dec = 1.f;
#pragma unroll
                        for (int r = 0; r < C; ++r) {
                            if (r > t) dec *= tc::ex2(Lc[r * D] - Lc[(r - 1) * D]);
                            if (r >= t) af = fmaf(dec * ldbf(smem + GB_Q + sw_off_elem(r, c, C)), Kr[r], af);
                        }
                        T2[t * D + c] += af;
                        const float gt = tc::ex2(Lc[t * D] - (t > 0 ? Lc[(t - 1) * D] : 0.f));
                        const float kt = ldbf(smem + GB_KT + sw_off_elem(t, c, C));
#pragma unroll
                        for (int r = 0; r < C; ++r)
                            Kr[r] = fmaf(gt, Kr[r], r > t ? ldbf(smem + GB_A2M + sw_off_elem(r, t, C)) * kt : 0.f);
                    }
                }
            }
            bar_sync(1, 256);
            // dg[t][c] = (T1 + T2 + a rho) / g_t on the product route, T1 + T2 on the exact one;
            // the 256 threads split the tokens: WG1 rows 0-31, WG2 rows 32-63
            float* dgst = reinterpret_cast<float*>(smem + GB_Q);
            const float rhoc = rho[c];
            for (int i0 = 0; i0 < 32; i0 += 8) {
                float sv[8], gv[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int t = 32 * half + i0 + j;
                    sv[j] = T1[t * D + c] + T2[t * D + c];
                    gv[j] = gcol[t * D];
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int t = 32 * half + i0 + j;
                    float v = sv[j];
                    if (fast) v = (v + ac * rhoc) * (t < nvalid ? rcp(gv[j]) : 1.f);
                    dgst[t * D + c] = v;
                }
            }
        }
        tc::fence_proxy_async();
        bar_sync(1, 256);
        if (ok && ot == 0) {
            tc::tma_store_3d(&tm_dq, smem + GB_V, 0, t0, bh);
            tc::tma_store_3d(&tm_dk, smem + GB_DO, 0, t0, bh);
            tc::tma_store_3d(&tm_dg, smem + GB_Q, 0, t0, bh);
            tc::bulk_commit();
            tc::bulk_wait_read();  // shared memory stays valid until the stores have read it
        }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(152));
        // ------------------------ rho, the masks, dv ------------------------
        const int wq = warp - 12, stid = tid - 384;
        const uint32_t lane_base = (uint32_t)(32 * wq) << 16;
        bool ok = bar_all(2, 128, wait_bar(full, 0, abort_flag));
        if (ok) {
            // rho_c = sum_j E[c,j] S_in[c,j]: row c = stid of both [128][128] tiles
            const int c = stid;
            float acc = 0.f;
#pragma unroll
            for (int b = 0; b < 2; ++b)
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (uint32_t)(b * BOX128 + c * 128 + ((kk ^ (c & 7)) << 4));
                    const uint4 e = at<uint4>(smem, GB_E + off), s = at<uint4>(smem, GB_SIN + off);
                    acc = fmaf(bf16lo(e.x), bf16lo(s.x), acc); acc = fmaf(bf16hi(e.x), bf16hi(s.x), acc);
                    acc = fmaf(bf16lo(e.y), bf16lo(s.y), acc); acc = fmaf(bf16hi(e.y), bf16hi(s.y), acc);
                    acc = fmaf(bf16lo(e.z), bf16lo(s.z), acc); acc = fmaf(bf16hi(e.z), bf16hi(s.z), acc);
                    acc = fmaf(bf16lo(e.w), bf16lo(s.w), acc); acc = fmaf(bf16hi(e.w), bf16hi(s.w), acc);
                }
            rho[c] = acc;
        }
        asm volatile("bar.arrive 3, 384;" ::: "memory");  // rho -> the operand warps' epilogue
        if (ok) ok = bar_all(2, 128, wait_bar(mma1, 0, abort_flag));
        if (ok) {
            tc::fence_after_sync();
            // M(A2), M(QK) in bf16: row t = 16 wq + lane (lanes 0-15)
#pragma unroll
            for (int which = 0; which < 2; ++which) {
                uint32_t r[64];
                const uint32_t src = tmem + (which == 0 ? TM_A2 : TM_QK) + lane_base;
                tc::tmem_ld32(src, r);
                tc::tmem_ld32(src + 32, r + 32);
                tc::tmem_wait_ld();
                if (lane < 16) {
                    const int t = 16 * wq + lane;
#pragma unroll
                    for (int s = 0; s < C; s += 8) {
                        float f[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) f[i] = s + i <= t ? __uint_as_float(r[s + i]) : 0.f;
                        at<uint4>(smem, (which == 0 ? GB_A2M : GB_QKM) + sw_off(t, s, C)) = pack8(f);
                    }
                }
            }
            tc::fence_proxy_async();
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(masks);
            ok = bar_all(2, 128, wait_bar(mma2, 0, abort_flag));
        }
        if (ok) {
            tc::fence_after_sync();
            // dv[s][j] from dv^T (lane j, column s) into the rows over k^
            const int j = 32 * wq + lane;
            __nv_bfloat16* stv = reinterpret_cast<__nv_bfloat16*>(smem + GB_K);
            uint32_t r[64];
            tc::tmem_ld32(tmem + TM_DV + lane_base, r);
            tc::tmem_ld32(tmem + TM_DV + lane_base + 32, r + 32);
            tc::tmem_wait_ld();
#pragma unroll
            for (int s = 0; s < C; ++s) stv[s * D + j] = __float2bfloat16_rn(__uint_as_float(r[s]));
        }
        tc::fence_proxy_async();
        bar_sync(2, 128);
        if (ok && stid == 0) {
            tc::tma_store_3d(&tm_dv, smem + GB_K, 0, t0, bh);
            tc::bulk_commit();
            tc::bulk_wait_read();
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 0) tc::tmem_dealloc(tmem, 512);
}

size_t layout(int B, int H, int T, BwdArgs* a, void* ws) {
    const int64_t BH = (int64_t)B * H;
    const int NC = (T + C - 1) / C;
    const size_t nz = (size_t)BH * NC;
    const size_t fp_slot = (size_t)D * D * 4, bf_slot = (size_t)D * D * 2;
    size_t off = 0;
    unsigned char* base = static_cast<unsigned char*>(ws);
    if (a) a->U = reinterpret_cast<float*>(base + off);
    off += nz * fp_slot;
    if (a) a->U2 = reinterpret_cast<float*>(base + off);
    off += nz * fp_slot;
    if (a) a->SIN = reinterpret_cast<__nv_bfloat16*>(base + off);
    off += nz * bf_slot;
    if (a) a->EE = reinterpret_cast<__nv_bfloat16*>(base + off);
    off += nz * bf_slot;
    if (a) a->A = reinterpret_cast<float*>(base + off);
    off += nz * D * 4;
    if (a) {
        a->T = T;
        a->NC = NC;
    }
    return off;
}

int sm_count() {
    static int sms = 0;
    if (sms == 0) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
            sms = 148;
    }
    return sms;
}

}  // namespace

bool gla_backward_tc_supported(int dk, int dv) { return dk == D && dv == D; }

size_t gla_backward_tc_workspace_size(int B, int H, int T) {
    if ((int64_t)B * H == 0 || T == 0) return 0;
    return layout(B, H, T, nullptr, nullptr);
}

cudaError_t gla_backward_tc_launch(const GlaBackwardArgs& g, cudaStream_t stream) {
    const int B = g.B, H = g.H, T = g.T;
    const int64_t BH = (int64_t)B * H;
    if (BH == 0 || T == 0) return cudaSuccess;
    if (BH > 65535) return cudaErrorInvalidConfiguration;
    BwdArgs a{};
    layout(B, H, T, &a, g.workspace);
    a.state0 = g.state0;
    a.dstate_final = g.dstate_final;
    a.dstate0 = g.dstate0;
    a.q = static_cast<const __nv_bfloat16*>(g.q);
    a.k = static_cast<const __nv_bfloat16*>(g.k);
    a.v = static_cast<const __nv_bfloat16*>(g.v);
    a.dO = static_cast<const __nv_bfloat16*>(g.dO);
    a.g = g.g;
    a.wave = sm_count();
    const int NC = a.NC;
    if ((int64_t)NC * BH > 0x7fffffff) return cudaErrorInvalidConfiguration;
    CUtensorMap mq, mk, mv, mdo, mg, msin, me, mdq, mdk, mdv, mdg, mu, mu2;
    cudaError_t e;
    const uint64_t Tu = (uint64_t)T, BHu = (uint64_t)BH;
    if ((e = make_tmap_3d(&mq, g.q, false, D, Tu, BHu, 64, C, true)) != cudaSuccess) return e;
    if ((e = make_tmap_3d(&mk, g.k, false, D, Tu, BHu, 64, C, true)) != cudaSuccess) return e;
    if ((e = make_tmap_3d(&mv, g.v, false, D, Tu, BHu, 64, C, true)) != cudaSuccess) return e;
    if ((e = make_tmap_3d(&mdo, g.dO, false, D, Tu, BHu, 64, C, true)) != cudaSuccess) return e;
    if ((e = make_tmap_3d(&mg, g.g, true, D, Tu, BHu, D, C, false)) != cudaSuccess) return e;
    if ((e = make_tmap_3d(&msin, a.SIN, false, D, D, BHu * NC, 64, D, true)) != cudaSuccess) return e;
    if ((e = make_tmap_3d(&me, a.EE, false, D, D, BHu * NC, 64, D, true)) != cudaSuccess) return e;
    if ((e = make_tmap_3d(&mdq, g.dq, false, D, Tu, BHu, D, C, false)) != cudaSuccess) return e;
    if ((e = make_tmap_3d(&mdk, g.dk, false, D, Tu, BHu, D, C, false)) != cudaSuccess) return e;
    if ((e = make_tmap_3d(&mdv, g.dv, false, D, Tu, BHu, D, C, false)) != cudaSuccess) return e;
    if ((e = make_tmap_3d(&mdg, g.dg, true, D, Tu, BHu, D, C, false)) != cudaSuccess) return e;
    if ((e = make_tmap_3d(&mu, a.U, true, D, D, BHu * NC, 32, 32, true)) != cudaSuccess) return e;
    if ((e = make_tmap_3d(&mu2, a.U2, true, D, D, BHu * NC, 32, 32, true)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(gla_bwd_contrib_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, CA_SMEM)) !=
        cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(gla_bwd_grad_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, GB_SMEM)) !=
        cudaSuccess)
        return e;
    gla_bwd_contrib_kernel<<<dim3((unsigned)NC, (unsigned)BH), 256, CA_SMEM, stream>>>(mq, mk, mv, mdo, mg, mu, mu2, a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    gla_bwd_scan_kernel<<<dim3((D * D / 4 + 255) / 256, (unsigned)BH), 256, 0, stream>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    gla_bwd_grad_kernel<<<dim3((unsigned)NC, (unsigned)BH), 512, GB_SMEM, stream>>>(mq, mk, mv, mdo, mg, msin, me, mdq,
                                                                                    mdk, mdv, mdg, a);
    note_launches(3);
    return cudaGetLastError();
}

unsigned gla_backward_tc_take_timeout_flag() {
    unsigned v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_gla_bwd_timeout, sizeof(v)) != cudaSuccess) return 0;
    cudaMemcpyToSymbol(g_gla_bwd_timeout, &zero, sizeof(zero));
    return v;
}

}  // namespace rod
