// swska_backward_tc.cu -- backward of SW-SKA prefill on the 5th-generation tensor cores
// (tcgen05 MMAs with bf16 operands and fp32 accumulators in tensor memory), head dim 128.
//
// Forward (CodeFuse Rodimus* article, Fig. 4 / SKA paragraph: one K shared by all heads,
// per-head V; setup blog §3: a window of the most recent W tokens):
//   s_tj = scale q_t . k_j for j in [t-W+1, t],  p_t = softmax(s_t),  o_t = sum_j p_tj v_j.
// For the loss gradient dO of every output row, with dP_tj = dO_t . v_j:
//   D_t = sum_j p_tj dP_tj = dO_t . o_t,   dS_tj = p_tj (dP_tj - D_t),
//   dq_t = scale sum_j dS_tj k_j,   dv_j = sum_t p_tj dO_t (per head),
//   dk_j = scale sum_h sum_t dS_tj q_t   (the shared key gathers every head's share).
//
// Four launches:
//  1. The forward kernel (swska_prefill_tc.cu) in its statistics mode: per row the negated base-2
//     log-sum-exp and D_t = dO_t . o_t from the fp32 output (nothing else is stored).
//  2. Query tiles (one CTA per 128 queries of one head): for each key tile of the window,
//     S = Q K^T and dP = dO V^T, then dS = P (dP - D) in bf16 in tensor memory and
//     dQ += dS K there.
//  3. Key tiles (one CTA per 128 keys and group of heads): for every head of the group and every
//     query tile that sees the key tile, S^T = K Q^T and dP^T = V dO^T; P^T and dS^T go to
//     tensor memory in bf16 and feed dV += P^T dO and dK += dS^T Q. dV is complete per head;
//     dK is a partial per head group, stored in fp32.
//  4. dk = scale * (sum of the groups' partials), summed in group order (deterministic).
// Every MMA is M = 128, N = 128, K = 16 (an N = 64 MMA costs most of an N = 128 one to issue).
// The two softmax warpgroups split each tile's 128 columns (64 each) and work in two phases:
// P from S as soon as S lands, then dS once dP lands; the MMA order lets the tensor core run
// the next products meanwhile. Warp roles (320 threads; 384 in the key-tile kernel):
//   warps 0-3 / 4-7  softmax warpgroups of column halves 0 / 1 (thread = TMEM lane = tile row)
//   warp 8           TMA producer (one lane)
//   warp 9           TMEM allocator; MMA issue (the whole warp runs the loop, one elected lane
//                    issues each tcgen05 instruction)
//   warps 10-11      (key-tile kernel only) idle: they complete the third warpgroup, which gives
//                    its registers to the softmax warpgroups
// Every wait is bounded; a timeout makes all roles stop, drain their copies and MMAs, and
// raise a flag.
#include <cuda.h>
#include <math.h>

#include "common.cuh"
#include "exp2x2.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace rod {
namespace {

__device__ unsigned int g_ska_bwd_tc_timeout = 0;

constexpr int TILE = 128;                   // queries or keys per tile
constexpr int HD = 128;                     // head dim (dk = dv)
constexpr int HALF = 64;                    // score columns per softmax warpgroup
constexpr int TILE_BYTES = TILE * HD * 2;   // 32 KB: one 128 x 128 bf16 tile
constexpr int BOX_BYTES = TILE_BYTES / 2;   // one TMA box: 128 rows x 64 columns
constexpr int NTHREADS = 320;
// The key-tile kernel runs three full warpgroups (warps 10-11 idle) so that it can move registers
// to the softmax warpgroups with setmaxnreg: the register file is split among the SM's four
// sub-partitions and each holds one warp of every warpgroup, so per sub-partition the launch
// provides 3 x 168 = 504 registers per lane, and the split below uses 216 + 216 + 72 = 504.
constexpr int NTHREADS_KEY = 384;
constexpr int kLaunchRegs = 168;
constexpr int kSoftmaxRegs = 216;
constexpr int kControlRegs = 72;
static_assert(2 * kSoftmaxRegs + kControlRegs <= 3 * kLaunchRegs, "register split exceeds launch");
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 0) {
            if (*abort_flag) return false;
            if (i >= kWaitLimit) {
                *abort_flag = 1;
                atomicExch(&g_ska_bwd_tc_timeout, 1u);
                return false;
            }
        }
    }
}

// The same wait executed by a whole warp in lockstep: every lane polls, and the warp leaves
// together (all lanes saw the phase complete, or the abort flag / limit is seen by all), so the
// warp stays converged for the elected MMA issue that follows.
__device__ __forceinline__ bool wait_bar_warp(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    for (uint32_t i = 1;; ++i) {
        if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
        if ((i & 255u) == 0) {
            if (__any_sync(0xffffffffu, *abort_flag != 0)) return false;
            if (i >= kWaitLimit) {
                *abort_flag = 1;
                atomicExch(&g_ska_bwd_tc_timeout, 1u);
                return false;
            }
        }
    }
}

__device__ __forceinline__ unsigned char* align1024(unsigned char* p) {
    return reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Descriptor low words. K-major: K runs along the 128-byte rows (two boxes for K = 128);
// MN-major: K runs down the rows, N across the two boxes (LBO = one box).
__device__ __forceinline__ uint32_t lo_kmajor(uint32_t addr) {
    return tc::desc_lo(tc::sdesc_sw128(addr, 16, 1024));
}
__device__ __forceinline__ uint32_t lo_mnmajor(uint32_t addr) {
    return tc::desc_lo(tc::sdesc_sw128(addr, BOX_BYTES, 1024));
}
// offset (16-byte units) of K step k (16 elements) in a K-major tile of K = 128
__device__ __forceinline__ uint32_t kstep(int k) { return (uint32_t)(((k / 4) * BOX_BYTES + (k % 4) * 32) >> 4); }
// offset of K step k (16 rows) in an MN-major tile
__device__ __forceinline__ uint32_t mnstep(int k) { return (uint32_t)((2048 * k) >> 4); }

using fx::ex2x2_fma;
using fx::f2add;
using fx::f2fma;
using fx::f2mul;
using fx::f2sub;
__device__ __forceinline__ float2 raw2(const uint32_t* r, int e) {
    return make_float2(__uint_as_float(r[e]), __uint_as_float(r[e + 1]));
}
__device__ __forceinline__ float2 ex2x2(float2 x) { return fx::ex2x2_sfu(x); }

// scores outside the window [lo, hi] (column indices of this 32-column chunk) -> -inf
__device__ __forceinline__ void mask_chunk(uint32_t* s, int c, int lo, int hi) {
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        const int col = 32 * c + e;
        if (col < lo || col > hi) s[e] = 0xff800000u;
    }
}
// Which groups of four exponentials in a 32-column chunk go to the FMA pipe (bit g: columns
// 4 g .. 4 g + 3); the rest use the SFU.
constexpr unsigned kPolyGroups = 0xAAu;

// ============================================================================================
// Launch 2: query tiles (dQ)
// ============================================================================================
namespace qa {
constexpr int KSLOT = 3, VSLOT = 2;                 // rings of K and V tiles
constexpr int OFF_Q = 0;
constexpr int OFF_DO = TILE_BYTES;
constexpr int OFF_K = 2 * TILE_BYTES;
constexpr int OFF_V = OFF_K + KSLOT * TILE_BYTES;
constexpr int OFF_BAR = OFF_V + VSLOT * TILE_BYTES;
// kfull[3], kempty[3], vfull[2], vempty[2], qfull, sfull[2], pfull, dsready, done, drain
constexpr int NBAR = 2 * KSLOT + 2 * VSLOT + 7;
constexpr int OFF_MISC = OFF_BAR + 8 * NBAR;
constexpr int SMEM = OFF_MISC + 16 + 1024;
static_assert(SMEM <= 232448, "shared memory");
}  // namespace qa

// TMEM columns: S buffers at 0 and 384 (tile u uses buffer u & 1), dP at 128, dQ at 256.
__device__ __forceinline__ uint32_t s_col(int u) { return (u & 1) ? 384u : 0u; }
// A operand of K step k (16 columns of P or dS) packed by the two warpgroups: warpgroup w's 64
// columns sit, two per 32-bit column, in columns 64 w .. 64 w + 31 of the S buffer
__device__ __forceinline__ uint32_t packed_col(int k) { return (uint32_t)(8 * k + (k >= 4 ? 32 : 0)); }

__global__ void __launch_bounds__(NTHREADS, 1)
ska_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                  const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  __nv_bfloat16* __restrict__ dq, const float* __restrict__ nlse2,
                  const float* __restrict__ dbuf, int T, int Tpad, int H, int W, float scale_log2,
                  float scale, int n_qtiles) {
    using namespace qa;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = align1024(smem_raw);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int qt = n_qtiles - 1 - (int)blockIdx.x;  // full-window tiles first
    const int h = blockIdx.y, b = blockIdx.z;
    const int bh = b * H + h;
    const int t0 = qt * TILE;
    const int kt_lo = (t0 - W + 1 > 0 ? t0 - W + 1 : 0) / TILE;
    const int n_it = qt - kt_lo + 1;  // key tiles of the window

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
    uint64_t* kfull = bars;
    uint64_t* kempty = bars + KSLOT;
    uint64_t* vfull = bars + 2 * KSLOT;
    uint64_t* vempty = vfull + VSLOT;
    uint64_t* qfull = vempty + VSLOT;
    uint64_t* sfull = qfull + 1;
    uint64_t* pfull = sfull + 2;
    uint64_t* dsready = pfull + 1;
    uint64_t* done = dsready + 1;
    uint64_t* drain = done + 1;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);

    if (threadIdx.x == 0) {
        for (int i = 0; i < KSLOT; ++i) {
            mbar_init(&kfull[i], 1);
            mbar_init(&kempty[i], 1);
        }
        for (int i = 0; i < VSLOT; ++i) {
            mbar_init(&vfull[i], 1);
            mbar_init(&vempty[i], 1);
        }
        mbar_init(qfull, 1);
        mbar_init(&sfull[0], 1);
        mbar_init(&sfull[1], 1);
        mbar_init(pfull, 1);
        mbar_init(dsready, 256);
        mbar_init(done, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 9) {
        tc::tmem_alloc(tmem_holder, 512);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_holder;

    if (warp == 8) {
        // ------------------------------- TMA producer -------------------------------
        if (lane == 0) {
            tc::tma_prefetch_desc(&tm_q);
            tc::tma_prefetch_desc(&tm_do);
            tc::tma_prefetch_desc(&tm_k);
            tc::tma_prefetch_desc(&tm_v);
            mbar_arrive_expect_tx(qfull, 2 * TILE_BYTES);
            for (int half = 0; half < 2; ++half) {
                tc::tma_load_3d(smem + OFF_Q + half * BOX_BYTES, &tm_q, half * 64, t0, bh, qfull);
                tc::tma_load_3d(smem + OFF_DO + half * BOX_BYTES, &tm_do, half * 64, t0, bh, qfull);
            }
            int nk = 0, nv = 0;  // loads started
            for (int u = 0; u < n_it; ++u) {  // K(u) then V(u), each into its own ring
                const int key0 = (kt_lo + u) * TILE;
                const int ks = u % KSLOT, vs = u % VSLOT;
                if (u >= KSLOT && !wait_bar(&kempty[ks], (uint32_t)((u / KSLOT - 1) & 1), abort_flag)) break;
                mbar_arrive_expect_tx(&kfull[ks], TILE_BYTES);
                for (int half = 0; half < 2; ++half)
                    tc::tma_load_3d(smem + OFF_K + ks * TILE_BYTES + half * BOX_BYTES, &tm_k, half * 64, key0, b,
                                    &kfull[ks]);
                ++nk;
                if (u >= VSLOT && !wait_bar(&vempty[vs], (uint32_t)((u / VSLOT - 1) & 1), abort_flag)) break;
                mbar_arrive_expect_tx(&vfull[vs], TILE_BYTES);
                for (int half = 0; half < 2; ++half)
                    tc::tma_load_3d(smem + OFF_V + vs * TILE_BYTES + half * BOX_BYTES, &tm_v, half * 64, key0, bh,
                                    &vfull[vs]);
                ++nv;
            }
            // every copy started here has landed before the CTA can leave (an older tile of a
            // ring was consumed by MMAs that completed before its slot was reused)
            mbar_wait_bounded(qfull, 0, kWaitLimit);
            for (int i = (nk > KSLOT ? nk - KSLOT : 0); i < nk; ++i)
                mbar_wait_bounded(&kfull[i % KSLOT], (uint32_t)((i / KSLOT) & 1), kWaitLimit);
            for (int i = (nv > VSLOT ? nv - VSLOT : 0); i < nv; ++i)
                mbar_wait_bounded(&vfull[i % VSLOT], (uint32_t)((i / VSLOT) & 1), kWaitLimit);
        }
    } else if (warp == 9) {
        // ------------------------------- MMA issue (whole warp) -------------------------------
        const uint32_t idesc = tc::idesc_bf16_f32(TILE, TILE, 0, 0);  // S, dP: both K-major
        const uint32_t idesc_g = tc::idesc_bf16_f32(TILE, HD, 0, 1);  // dQ += dS K: K MN-major
        const uint32_t d_hi = tc::desc_hi(tc::sdesc_sw128(0, 16, 1024));
        const uint32_t q_lo = lo_kmajor(smem_u32(smem + OFF_Q));
        const uint32_t do_lo = lo_kmajor(smem_u32(smem + OFF_DO));
        auto kslot = [&](int u) { return smem_u32(smem + OFF_K + (u % KSLOT) * TILE_BYTES); };
        auto vslot = [&](int u) { return smem_u32(smem + OFF_V + (u % VSLOT) * TILE_BYTES); };
        bool ok = true;
        auto acq_k = [&](int u) {
            ok = ok && wait_bar_warp(&kfull[u % KSLOT], (uint32_t)((u / KSLOT) & 1), abort_flag);
            tc::fence_after_sync();
            return ok;
        };
        auto acq_v = [&](int u) {
            ok = ok && wait_bar_warp(&vfull[u % VSLOT], (uint32_t)((u / VSLOT) & 1), abort_flag);
            tc::fence_after_sync();
            return ok;
        };
        auto issue_s = [&](int u) {  // S(u) = Q K(u)^T
            const uint32_t k_lo = lo_kmajor(kslot(u));
#pragma unroll
            for (int k = 0; k < HD / 16; ++k)
                tc::mma_ss_lh_warp(tmem + s_col(u), q_lo + kstep(k), d_hi, k_lo + kstep(k), d_hi, idesc, k > 0);
            tc::mma_commit_warp(&sfull[u & 1]);
        };
        auto issue_dp = [&](int u) {  // dP(u) = dO V(u)^T; V(u) is free once it completes
            const uint32_t v_lo = lo_kmajor(vslot(u));
#pragma unroll
            for (int k = 0; k < HD / 16; ++k)
                tc::mma_ss_lh_warp(tmem + 128u, do_lo + kstep(k), d_hi, v_lo + kstep(k), d_hi, idesc, k > 0);
            tc::mma_commit_warp(pfull);
            tc::mma_commit_warp(&vempty[u % VSLOT]);
        };
        auto issue_dq = [&](int u) {  // dQ += dS(u) K(u); K(u) is free once it completes
            const uint32_t k_lo = lo_mnmajor(kslot(u));
#pragma unroll
            for (int k = 0; k < TILE / 16; ++k)
                tc::mma_ts_lh_warp(tmem + 256u, tmem + s_col(u) + packed_col(k), k_lo + mnstep(k), d_hi, idesc_g,
                                   (u > 0 || k > 0) ? 1u : 0u);
            tc::mma_commit_warp(&kempty[u % KSLOT]);
        };
        ok = wait_bar_warp(qfull, 0, abort_flag);
        tc::fence_after_sync();
        if (ok && acq_k(0)) {
            // order: S(0) dP(0) S(1) | dQ(0) dP(1) S(2) | dQ(1) dP(2) S(3) | ...
            issue_s(0);
            if (acq_v(0)) issue_dp(0);
            if (ok && n_it > 1 && acq_k(1)) issue_s(1);
            for (int u = 0; u < n_it && ok; ++u) {
                if (!wait_bar_warp(dsready, (uint32_t)(u & 1), abort_flag)) { ok = false; break; }
                tc::fence_after_sync();
                issue_dq(u);
                if (u + 1 < n_it) {
                    if (!acq_v(u + 1)) break;
                    issue_dp(u + 1);
                }
                if (u + 2 < n_it) {
                    if (!acq_k(u + 2)) break;
                    issue_s(u + 2);  // into the buffer dQ(u) is reading: the pipe runs in order
                }
            }
            if (ok) tc::mma_commit_warp(done);
        }
        // every MMA this warp issued has completed before TMEM is released
        tc::mma_commit_warp(drain);
        mbar_wait_bounded(drain, 0, kWaitLimit);
    } else {
        // ------------------------------- softmax warpgroups -------------------------------
        const int w = warp / 4;                    // column half (keys 64 w .. 64 w + 63)
        const int row = threadIdx.x % 128;         // query row == TMEM lane
        const uint32_t lane_base = (uint32_t)(32 * (warp % 4)) << 16;
        const uint32_t tP = tmem + lane_base + 128u + 64u * w;
        const uint32_t tQ = tmem + lane_base + 256u + 64u * w;
        const int t = t0 + row;
        const float nL = nlse2[(int64_t)bh * Tpad + t];  // -inf past the end: p = 0
        const float Dr = dbuf[(int64_t)bh * Tpad + t];
        const float2 sl2 = make_float2(scale_log2, scale_log2), nl2 = make_float2(nL, nL);
        const float2 d2 = make_float2(Dr, Dr);
        bool ok = true;
        for (int u = 0; u < n_it; ++u) {
            const uint32_t tS = tmem + lane_base + s_col(u) + 64u * w;
            const int key0 = (kt_lo + u) * TILE + HALF * w;  // first key of this half
            const bool full_tile = key0 >= t0 + TILE - W && key0 + HALF - 1 <= t0;
            const int lo = t - W + 1 - key0, hi = t - key0;   // valid columns [lo, hi]
            // phase 1: P from S
            if (!wait_bar_warp(&sfull[u & 1], (uint32_t)((u >> 1) & 1), abort_flag)) { ok = false; break; }
            tc::fence_after_sync();
            float2 p2[32];
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t s[32];
                tc::tmem_ld32(tS + 32u * c, s);
                tc::tmem_wait_ld();
                if (!full_tile) mask_chunk(s, c, lo, hi);
#pragma unroll
                for (int g = 0; g < 8; ++g) {
                    if ((kPolyGroups >> g) & 1u) {
                        p2[16 * c + 2 * g] = ex2x2_fma(f2fma(raw2(s, 4 * g), sl2, nl2));
                        p2[16 * c + 2 * g + 1] = ex2x2_fma(f2fma(raw2(s, 4 * g + 2), sl2, nl2));
                    } else {
                        p2[16 * c + 2 * g] = ex2x2(f2fma(raw2(s, 4 * g), sl2, nl2));
                        p2[16 * c + 2 * g + 1] = ex2x2(f2fma(raw2(s, 4 * g + 2), sl2, nl2));
                    }
                }
            }
            // phase 2: dS = P (dP - D), packed over this half's first 32 columns of the S buffer
            if (!wait_bar_warp(pfull, (uint32_t)(u & 1), abort_flag)) { ok = false; break; }
            tc::fence_after_sync();
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t dp[32], pk[16];
                tc::tmem_ld32(tP + 32u * c, dp);
                tc::tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float2 ds = f2mul(p2[16 * c + i], f2sub(raw2(dp, 2 * i), d2));
                    pk[i] = pack_bf16x2(ds.x, ds.y);
                }
                tc::tmem_st16(tS + 16u * c, pk);
            }
            tc::tmem_wait_st();
            tc::fence_before_sync();
            mbar_arrive(dsready);
        }
        // epilogue: dq = scale * dQ -> bf16, this half's 64 channels
        if (ok && wait_bar_warp(done, 0, abort_flag)) {
            tc::fence_after_sync();
            __nv_bfloat16* out = dq + ((int64_t)bh * T + t) * HD + HALF * w;
#pragma unroll
            for (int cb = 0; cb < 2; ++cb) {
                uint32_t r[32];
                tc::tmem_ld32(tQ + 32u * cb, r);
                tc::tmem_wait_ld();
                if (t < T) {
#pragma unroll
                    for (int i = 0; i < 32; i += 8) {
                        float f[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(r[i + e]) * scale;
                        store8(out + 32 * cb + i, f);
                    }
                }
            }
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 9) tc::tmem_dealloc(tmem, 512);
}

// ============================================================================================
// Launch 3: key tiles (dV per head, dK partial per head group)
// ============================================================================================
namespace ka {
constexpr int OFF_K = 0;
constexpr int OFF_V = TILE_BYTES;
constexpr int OFF_RING = 2 * TILE_BYTES;             // 2 slots of (Q tile, dO tile)
constexpr int UNIT_BYTES = 2 * TILE_BYTES;
constexpr int OFF_STAT = OFF_RING + 2 * UNIT_BYTES;  // 2 slots of (-lse2[128], D[128]) fp32
constexpr int STAT_BYTES = 2 * TILE * 4;
constexpr int OFF_BAR = OFF_STAT + 2 * STAT_BYTES;
// kfull, vfull, vempty, full[2], empty[2], sfull, pfull, sread, pwritten, dsready, dvdone, dvfree,
// done, drain
constexpr int NBAR = 16;
constexpr int OFF_MISC = OFF_BAR + 8 * NBAR;
constexpr int SMEM = OFF_MISC + 16 + 1024;
static_assert(SMEM <= 232448, "shared memory");
}  // namespace ka

// TMEM columns: S^T [0,128) | dP^T [128,256) | dV [256,384) | dK [384,512). Once a warpgroup has
// read its half of dP^T, that half holds its P^T (packed, first 32 columns) and dS^T (packed,
// last 32 columns), so the S^T region is free as soon as it has been read: the next S^T is
// computed while this pair's gradients are formed.
__global__ void __launch_bounds__(NTHREADS_KEY, 1)
ska_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const float* __restrict__ nlse2, const float* __restrict__ dbuf,
                    __nv_bfloat16* __restrict__ dv, float* __restrict__ dk_part, int B, int T, int Tpad,
                    int H, int HG, int W, float scale_log2, int n_qtiles) {
    using namespace ka;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = align1024(smem_raw);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int kt = blockIdx.x, grp = blockIdx.y, b = blockIdx.z;
    const int j0 = kt * TILE;
    const int qt_lo = kt;  // queries t in [j, j + W - 1] see key j
    const int64_t last_q = (int64_t)j0 + TILE - 1 + W - 1;  // the last query that sees the tile
    const int qt_hi = last_q / TILE < n_qtiles - 1 ? (int)(last_q / TILE) : n_qtiles - 1;
    const int n_q = qt_hi - qt_lo + 1;  // query tiles per head
    const int h0 = grp * HG;
    const int U = HG * n_q;             // (head, query tile) pairs, head-major

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
    uint64_t* kfull = bars;
    uint64_t* vfull = bars + 1;
    uint64_t* vempty = bars + 2;
    uint64_t* full = bars + 3;
    uint64_t* empty = bars + 5;
    uint64_t* sfull = bars + 7;
    uint64_t* pfull = bars + 8;
    uint64_t* sread = bars + 9;      // S^T read by both warpgroups: the region is free
    uint64_t* pwritten = bars + 10;  // P^T written (dP^T read)
    uint64_t* dsready = bars + 11;   // dS^T written
    uint64_t* dvdone = bars + 12;
    uint64_t* dvfree = bars + 13;
    uint64_t* done = bars + 14;
    uint64_t* drain = bars + 15;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);

    if (threadIdx.x == 0) {
        mbar_init(kfull, 1);
        mbar_init(vfull, 1);
        mbar_init(vempty, 1);
        for (int s2 = 0; s2 < 2; ++s2) {
            mbar_init(&full[s2], 1);
            mbar_init(&empty[s2], 1);
        }
        mbar_init(sfull, 1);
        mbar_init(pfull, 1);
        mbar_init(sread, 256);
        mbar_init(pwritten, 256);
        mbar_init(dsready, 256);
        mbar_init(dvdone, 1);
        mbar_init(dvfree, 256);
        mbar_init(done, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 9) {
        tc::tmem_alloc(tmem_holder, 512);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_holder;

    if (warp >= 8) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kControlRegs));
    if (warp == 8) {
        // ------------------------------- TMA producer -------------------------------
        if (lane == 0) {
            tc::tma_prefetch_desc(&tm_q);
            tc::tma_prefetch_desc(&tm_do);
            tc::tma_prefetch_desc(&tm_k);
            tc::tma_prefetch_desc(&tm_v);
            mbar_arrive_expect_tx(kfull, TILE_BYTES);
            for (int half = 0; half < 2; ++half)
                tc::tma_load_3d(smem + OFF_K + half * BOX_BYTES, &tm_k, half * 64, j0, b, kfull);
            int u = 0, nv = 0;
            for (; u < U; ++u) {
                const int hi = u / n_q, qt = qt_lo + u % n_q, bh = b * H + h0 + hi;
                if (u % n_q == 0) {  // a new head: its V tile (once the previous head's is used)
                    if (hi > 0 && !wait_bar(vempty, (uint32_t)((hi - 1) & 1), abort_flag)) break;
                    mbar_arrive_expect_tx(vfull, TILE_BYTES);
                    for (int half = 0; half < 2; ++half)
                        tc::tma_load_3d(smem + OFF_V + half * BOX_BYTES, &tm_v, half * 64, j0, bh, vfull);
                    ++nv;
                }
                const int slot = u % 2, use = u / 2;
                if (use > 0 && !wait_bar(&empty[slot], (uint32_t)((use - 1) & 1), abort_flag)) break;
                unsigned char* dst = smem + OFF_RING + slot * UNIT_BYTES;
                unsigned char* st = smem + OFF_STAT + slot * STAT_BYTES;
                mbar_arrive_expect_tx(&full[slot], 2 * TILE_BYTES + STAT_BYTES);
                for (int half = 0; half < 2; ++half) {
                    tc::tma_load_3d(dst + half * BOX_BYTES, &tm_q, half * 64, qt * TILE, bh, &full[slot]);
                    tc::tma_load_3d(dst + TILE_BYTES + half * BOX_BYTES, &tm_do, half * 64, qt * TILE, bh,
                                    &full[slot]);
                }
                const int64_t srow = (int64_t)bh * Tpad + (int64_t)qt * TILE;
                bulk_g2s(st, nlse2 + srow, TILE * 4, &full[slot]);
                bulk_g2s(st + TILE * 4, dbuf + srow, TILE * 4, &full[slot]);
            }
            // every copy started here has landed before the CTA can leave (a V or unit load
            // older than the latest ones was consumed by MMAs that have completed)
            mbar_wait_bounded(kfull, 0, kWaitLimit);
            if (nv > 0) mbar_wait_bounded(vfull, (uint32_t)((nv - 1) & 1), kWaitLimit);
            for (int ui = (u > 2 ? u - 2 : 0); ui < u; ++ui)
                mbar_wait_bounded(&full[ui % 2], (uint32_t)((ui / 2) & 1), kWaitLimit);
        }
    } else if (warp == 9) {
        // ------------------------------- MMA issue (whole warp) -------------------------------
        const uint32_t idesc = tc::idesc_bf16_f32(TILE, TILE, 0, 0);  // S^T, dP^T: both K-major
        const uint32_t idesc_g = tc::idesc_bf16_f32(TILE, HD, 0, 1);  // dV, dK: B MN-major
        const uint32_t d_hi = tc::desc_hi(tc::sdesc_sw128(0, 16, 1024));
        const uint32_t k_lo = lo_kmajor(smem_u32(smem + OFF_K));
        const uint32_t v_lo = lo_kmajor(smem_u32(smem + OFF_V));
        auto unit = [&](int u) { return smem_u32(smem + OFF_RING + (u % 2) * UNIT_BYTES); };
        bool ok = true;
        auto acquire = [&](uint64_t* bar, uint32_t parity) {
            ok = ok && wait_bar_warp(bar, parity, abort_flag);
            tc::fence_after_sync();
            return ok;
        };
        auto issue_st = [&](int u) {  // S^T(u) = K Q(u)^T
            const uint32_t q_lo = lo_kmajor(unit(u));
#pragma unroll
            for (int k = 0; k < HD / 16; ++k)
                tc::mma_ss_lh_warp(tmem, k_lo + kstep(k), d_hi, q_lo + kstep(k), d_hi, idesc, k > 0);
            tc::mma_commit_warp(sfull);
        };
        auto issue_dpt = [&](int u) {  // dP^T(u) = V dO(u)^T
            const uint32_t o_lo = lo_kmajor(unit(u) + TILE_BYTES);
#pragma unroll
            for (int k = 0; k < HD / 16; ++k)
                tc::mma_ss_lh_warp(tmem + 128u, v_lo + kstep(k), d_hi, o_lo + kstep(k), d_hi, idesc, k > 0);
            tc::mma_commit_warp(pfull);
            if (u % n_q == n_q - 1) tc::mma_commit_warp(vempty);  // the head's last use of V
        };
        auto issue_dv = [&](int u, bool first) {  // dV += P^T(u) dO(u)
            const uint32_t o_lo = lo_mnmajor(unit(u) + TILE_BYTES);
#pragma unroll
            for (int k = 0; k < TILE / 16; ++k)
                tc::mma_ts_lh_warp(tmem + 256u, tmem + 128u + packed_col(k), o_lo + mnstep(k), d_hi, idesc_g,
                                   (first && k == 0) ? 0u : 1u);
        };
        auto issue_dk = [&](int u) {  // dK += dS^T(u) Q(u); the unit's slot is free afterwards
            const uint32_t q_lo = lo_mnmajor(unit(u));
#pragma unroll
            for (int k = 0; k < TILE / 16; ++k)
                tc::mma_ts_lh_warp(tmem + 384u, tmem + 160u + packed_col(k), q_lo + mnstep(k), d_hi, idesc_g,
                                   (u > 0 || k > 0) ? 1u : 0u);
            tc::mma_commit_warp(&empty[u % 2]);
        };
        if (acquire(kfull, 0) && acquire(vfull, 0) && acquire(&full[0], 0)) {
            // order: S^T(0) dP^T(0) | S^T(1) dV(0) dK(0) dP^T(1) | S^T(2) dV(1) dK(1) dP^T(2) | ...
            issue_st(0);
            issue_dpt(0);
            for (int u = 0; u < U && ok; ++u) {
                const int hi = u / n_q;
                const bool first = u % n_q == 0, last = u % n_q == n_q - 1;
                if (u + 1 < U) {  // the next S^T as soon as this one has been read
                    if (!acquire(sread, (uint32_t)(u & 1))) break;
                    if (!acquire(&full[(u + 1) % 2], (uint32_t)(((u + 1) / 2) & 1))) break;
                    issue_st(u + 1);
                }
                if (!acquire(pwritten, (uint32_t)(u & 1))) break;
                if (first && hi > 0 && !acquire(dvfree, (uint32_t)((hi - 1) & 1))) break;
                issue_dv(u, first);
                if (last) tc::mma_commit_warp(dvdone);
                if (!acquire(dsready, (uint32_t)(u & 1))) break;
                issue_dk(u);
                if (u + 1 < U) {  // over P^T(u) and dS^T(u), which dV(u) and dK(u) read first
                    if ((u + 1) % n_q == 0 && !acquire(vfull, (uint32_t)(((u + 1) / n_q) & 1))) break;
                    issue_dpt(u + 1);
                }
            }
            if (ok) tc::mma_commit_warp(done);
        }
        tc::mma_commit_warp(drain);
        mbar_wait_bounded(drain, 0, kWaitLimit);
    } else if (warp < 8) {
        // ------------------------------- softmax warpgroups -------------------------------
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
        const int w = warp / 4;                    // column half (queries 64 w .. 64 w + 63)
        const int row = threadIdx.x % 128;         // key row == TMEM lane
        const uint32_t lane_base = (uint32_t)(32 * (warp % 4)) << 16;
        const uint32_t tS = tmem + lane_base + 64u * w;
        const uint32_t tP = tS + 128u;
        const uint32_t tV = tmem + lane_base + 256u + 64u * w;
        const uint32_t tK = tmem + lane_base + 384u + 64u * w;
        const int key = j0 + row;
        const float2 sl2 = make_float2(scale_log2, scale_log2);
        bool ok = true;
        for (int u = 0; u < U; ++u) {
            const int hi = u / n_q, qt = qt_lo + u % n_q;
            const int tq0 = qt * TILE + HALF * w;  // first query of this half
            const float* st = reinterpret_cast<const float*>(smem + OFF_STAT + (u % 2) * STAT_BYTES) + HALF * w;
            const bool full_tile = tq0 >= j0 + TILE - 1 && tq0 + HALF - 1 <= j0 + W - 1;
            const int lo = key - tq0, hi_e = key + W - 1 - tq0;  // valid columns [lo, hi_e]
            // P^T from S^T (the unit's statistics landed with its tiles); S^T is released as soon
            // as it has been read
            if (!wait_bar_warp(sfull, (uint32_t)(u & 1), abort_flag)) { ok = false; break; }
            tc::fence_after_sync();
            float2 p2[32];
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t s[32];
                tc::tmem_ld32(tS + 32u * c, s);
                tc::tmem_wait_ld();
                if (c == 1) {
                    tc::fence_before_sync();
                    mbar_arrive(sread);
                }
                if (!full_tile) mask_chunk(s, c, lo, hi_e);
#pragma unroll
                for (int e4 = 0; e4 < 32; e4 += 4) {
                    const float4 L4 = *reinterpret_cast<const float4*>(st + 32 * c + e4);  // -lse2
                    const bool fma_pipe = (kPolyGroups >> (e4 / 4)) & 1u;
                    const float2 xa = f2fma(raw2(s, e4), sl2, make_float2(L4.x, L4.y));
                    const float2 xb = f2fma(raw2(s, e4 + 2), sl2, make_float2(L4.z, L4.w));
                    p2[16 * c + e4 / 2] = fma_pipe ? ex2x2_fma(xa) : ex2x2(xa);
                    p2[16 * c + e4 / 2 + 1] = fma_pipe ? ex2x2_fma(xb) : ex2x2(xb);
                }
            }
            // dP^T read; P^T packed over the first 32 columns of this half of it as soon as those
            // have been read (dV may start), then dS^T = P^T (dP^T - D) over the last 32
            if (!wait_bar_warp(pfull, (uint32_t)(u & 1), abort_flag)) { ok = false; break; }
            tc::fence_after_sync();
            {
                uint32_t dp[64], pk[32];
                tc::tmem_ld32(tP, dp);
                tc::tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) pk[i] = pack_bf16x2(p2[i].x, p2[i].y);
                tc::tmem_st32(tP, pk);
                tc::tmem_wait_st();
                tc::fence_before_sync();
                mbar_arrive(pwritten);
                tc::tmem_ld32(tP + 32u, dp + 32);
                tc::tmem_wait_ld();
#pragma unroll
                for (int e4 = 0; e4 < 64; e4 += 4) {
                    const float4 D4 = *reinterpret_cast<const float4*>(st + TILE + e4);
                    const float2 da = f2mul(p2[e4 / 2], f2sub(raw2(dp, e4), make_float2(D4.x, D4.y)));
                    const float2 db = f2mul(p2[e4 / 2 + 1], f2sub(raw2(dp, e4 + 2), make_float2(D4.z, D4.w)));
                    pk[e4 / 2] = pack_bf16x2(da.x, da.y);
                    pk[e4 / 2 + 1] = pack_bf16x2(db.x, db.y);
                }
                tc::tmem_st32(tP + 32u, pk);
                tc::tmem_wait_st();
                tc::fence_before_sync();
                mbar_arrive(dsready);
            }
            if (u % n_q == n_q - 1) {
                // the head's dV rows are complete: store them and release the accumulator
                if (!wait_bar_warp(dvdone, (uint32_t)(hi & 1), abort_flag)) { ok = false; break; }
                tc::fence_after_sync();
                __nv_bfloat16* out = dv + (((int64_t)b * H + h0 + hi) * T + key) * HD + HALF * w;
#pragma unroll
                for (int cb = 0; cb < 2; ++cb) {
                    uint32_t r[32];
                    tc::tmem_ld32(tV + 32u * cb, r);
                    tc::tmem_wait_ld();
                    if (key < T) {
#pragma unroll
                        for (int i = 0; i < 32; i += 8) {
                            float f[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(r[i + e]);
                            store8(out + 32 * cb + i, f);
                        }
                    }
                }
                tc::fence_before_sync();
                mbar_arrive(dvfree);
            }
        }
        // epilogue: this group's dK partial (unscaled fp32), this half's 64 channels
        if (ok && wait_bar_warp(done, 0, abort_flag)) {
            tc::fence_after_sync();
            float* out = dk_part + (((int64_t)grp * B + b) * T + key) * HD + HALF * w;
#pragma unroll
            for (int cb = 0; cb < 2; ++cb) {
                uint32_t r[32];
                tc::tmem_ld32(tK + 32u * cb, r);
                tc::tmem_wait_ld();
                if (key < T) {
#pragma unroll
                    for (int i = 0; i < 32; i += 4)
                        *reinterpret_cast<float4*>(out + 32 * cb + i) =
                            make_float4(__uint_as_float(r[i]), __uint_as_float(r[i + 1]),
                                        __uint_as_float(r[i + 2]), __uint_as_float(r[i + 3]));
                }
            }
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 9) tc::tmem_dealloc(tmem, 512);
}

// ============================================================================================
// Launch 1 when the forward's output and log-sum-exp were kept: one warp per (padded) row,
// lane l holding channels 4l .. 4l + 3, D = dO . o in fp32 and nlse2 = -lse * log2(e); rows
// past T get -inf and 0, as the statistics pass gives them.
__global__ void __launch_bounds__(256)
ska_rowstats_kernel(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dO,
                    const float* __restrict__ lse, float* __restrict__ nlse2, float* __restrict__ dbuf, int T,
                    int Tpad, int64_t rows) {
    const int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (r >= rows) return;
    const int64_t bh = r / Tpad;
    const int t = (int)(r - bh * Tpad);
    if (t >= T) {
        if (lane == 0) {
            nlse2[r] = -INFINITY;
            dbuf[r] = 0.f;
        }
        return;
    }
    const int64_t off = (bh * T + t) * HD + 4 * lane;
    const uint2 ow = *reinterpret_cast<const uint2*>(o + off);
    const uint2 gw = *reinterpret_cast<const uint2*>(dO + off);
    float d = bf16lo(ow.x) * bf16lo(gw.x);
    d = fmaf(bf16hi(ow.x), bf16hi(gw.x), d);
    d = fmaf(bf16lo(ow.y), bf16lo(gw.y), d);
    d = fmaf(bf16hi(ow.y), bf16hi(gw.y), d);
#pragma unroll
    for (int sh = 16; sh > 0; sh >>= 1) d += __shfl_xor_sync(0xffffffffu, d, sh);
    if (lane == 0) {
        dbuf[r] = d;
        nlse2[r] = -lse[bh * T + t] * kLog2e;
    }
}

// Launch 4: dk = scale * sum over head groups of the partials (group order fixed)
// ============================================================================================
__global__ void __launch_bounds__(256)
ska_bwd_dk_reduce(const float* __restrict__ part, __nv_bfloat16* __restrict__ dk, int64_t n4, int G,
                  float scale) {
    const float4* p4 = reinterpret_cast<const float4*>(part);
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
         i += (int64_t)gridDim.x * blockDim.x) {
        float4 a = p4[i];
        for (int g = 1; g < G; ++g) {
            const float4 x = p4[(int64_t)g * n4 + i];
            a.x += x.x;
            a.y += x.y;
            a.z += x.z;
            a.w += x.w;
        }
        store4(dk + 4 * i, make_float4(a.x * scale, a.y * scale, a.z * scale, a.w * scale));
    }
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

int64_t swska_backward_tc_tpad(int T) { return ((int64_t)T + TILE - 1) / TILE * TILE; }

size_t swska_backward_tc_workspace_size(int B, int H, int T) {
    // row statistics (padded rows) + one fp32 dK partial per head group (at most H groups)
    return ((size_t)2 * B * H * swska_backward_tc_tpad(T) + (size_t)H * B * T * HD) * sizeof(float);
}

bool swska_backward_tc_supported(int H, int T, int dk, int dv) {
    return dk == HD && dv == HD && H >= 1 && T >= TILE;
}

int swska_backward_tc_groups(int B, int H, int T) {
    // the fewest head groups that still give every SM several key-tile CTAs
    const int64_t nkt = ((int64_t)T + TILE - 1) / TILE;
    for (int G = 1; G < H; ++G)
        if (H % G == 0 && (int64_t)B * nkt * G >= 4 * (int64_t)sm_count()) return G;
    return H;
}

cudaError_t swska_backward_tc_launch(const SkaBackwardArgs& a, cudaStream_t stream) {
    const int B = a.B, H = a.H, T = a.T;
    const int W = a.W < T ? a.W : T;  // a window longer than the sequence is the whole prefix
    const int64_t Tpad = swska_backward_tc_tpad(T);
    float* nlse2 = static_cast<float*>(a.workspace);
    float* dbuf = nlse2 + (size_t)B * H * Tpad;
    float* part = dbuf + (size_t)B * H * Tpad;
    if (B > 65535 || H > 65535) return cudaErrorInvalidConfiguration;
    // launch 1: the row statistics, from the forward's saved output and log-sum-exp when given,
    // else from the forward in statistics mode (row log-sum-exp and D, no output stored)
    cudaError_t e;
    if (a.o != nullptr && a.lse != nullptr) {
        const int64_t rows = (int64_t)B * H * Tpad;
        ska_rowstats_kernel<<<(unsigned)((rows * 32 + 255) / 256), 256, 0, stream>>>(
            static_cast<const __nv_bfloat16*>(a.o), static_cast<const __nv_bfloat16*>(a.dO), a.lse, nlse2, dbuf,
            T, (int)Tpad, rows);
        note_launches(1);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    } else {
        e = swska_prefill_tc_stats_launch(a.q, a.k, a.v, nullptr, a.dO, nlse2, dbuf, Tpad, B, H, T, W, a.scale,
                                          stream);
        if (e != cudaSuccess) return e;
    }
    CUtensorMap mq, mdo, mk, mv;
    if ((e = make_tmap_bf16_3d(&mq, a.q, HD, (uint64_t)T, (uint64_t)B * H, 64, TILE)) != cudaSuccess) return e;
    if ((e = make_tmap_bf16_3d(&mdo, a.dO, HD, (uint64_t)T, (uint64_t)B * H, 64, TILE)) != cudaSuccess) return e;
    if ((e = make_tmap_bf16_3d(&mk, a.k, HD, (uint64_t)T, (uint64_t)B, 64, TILE)) != cudaSuccess) return e;
    if ((e = make_tmap_bf16_3d(&mv, a.v, HD, (uint64_t)T, (uint64_t)B * H, 64, TILE)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(ska_bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, qa::SMEM)) !=
        cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(ska_bwd_dkdv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, ka::SMEM)) !=
        cudaSuccess)
        return e;
    const int nqt = (int)(Tpad / TILE);
    const float sl = a.scale * kLog2e;
    ska_bwd_dq_kernel<<<dim3((unsigned)nqt, (unsigned)H, (unsigned)B), NTHREADS, qa::SMEM, stream>>>(
        mq, mdo, mk, mv, static_cast<__nv_bfloat16*>(a.dq), nlse2, dbuf, T, (int)Tpad, H, W, sl, a.scale, nqt);
    const int G = swska_backward_tc_groups(B, H, T);
    ska_bwd_dkdv_kernel<<<dim3((unsigned)nqt, (unsigned)G, (unsigned)B), NTHREADS_KEY, ka::SMEM, stream>>>(
        mq, mdo, mk, mv, nlse2, dbuf, static_cast<__nv_bfloat16*>(a.dv), part, B, T, (int)Tpad, H, H / G, W,
        sl, nqt);
    const int64_t n4 = (int64_t)B * T * HD / 4;
    const int64_t want = (n4 + 255) / 256, cap = 8 * (int64_t)sm_count();
    ska_bwd_dk_reduce<<<(unsigned)(want < cap ? want : cap), 256, 0, stream>>>(
        part, static_cast<__nv_bfloat16*>(a.dk), n4, G, a.scale);
    note_launches(3);
    return cudaGetLastError();
}

unsigned swska_backward_tc_take_timeout_flag() {
    unsigned v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_ska_bwd_tc_timeout, sizeof(v)) != cudaSuccess) return 0;
    cudaMemcpyToSymbol(g_ska_bwd_tc_timeout, &zero, sizeof(zero));
    return v;
}

}  // namespace rod
