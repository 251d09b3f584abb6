// gla_prefill_tc.cu -- chunkwise-parallel prefill of the Rodimus gated linear recurrence on the
// 5th-generation tensor cores (tcgen05 / TMEM / TMA), bf16 q, k, v / fp32 gates and state,
// d_k = d_v = 128, chunks of 64 tokens.
//
// Recurrence (CodeFuse Rodimus* article, Rodimus block; SALA blog §2.2 state form, §4.3 decay):
//     S_t = diag(g_t) S_{t-1} + k_t^T v_t,     o_t = q_t S_t.
// Chunk form (the chunkwise-parallel algorithm the Rodimus block paragraph names for training
// and prefill). For a chunk of C tokens with incoming state S_in, per key channel c let
//     G_t = prod_{r<=t} g_r     (prefix product inside the chunk),
//     F_t = prod_{t<r<=C-1} g_r (suffix product),  a = G_{C-1}.
// Then, exactly,
//     o_t   = sum_{s<=t} (sum_c q_tc k_sc G_tc / G_sc) v_s + (q_t . G_t) S_in
//     S_out = diag(a) S_in + sum_s (k_s . F_s)^T v_s.
// With q~ = q.G, k~ = k/G, k^ = k.F the chunk is four dense contractions on the tensor cores:
//     A = q~ k~^T (masked to s <= t, rounded to bf16 as P),  O = P V + q~ S_in,  S += k^^T V
// while the fp32 state lives in tensor memory for the whole segment. k~ needs 1/G, so a chunk
// in which some channel decays below 2^-60 computes A on the CUDA cores from log2-gate sums
// (exact in the limit, g = 0 included) instead; everything else is unchanged.
//
// Parallelism over the sequence: the T tokens are cut into segments of L_seg tokens. Pass A
// (per segment but the last) computes the segment's state contribution U and decay a_seg
// from k, v, g; a scan kernel chains S_in(m+1) = diag(a_seg,m) S_in(m) + U_m per (b, h) with
// each thread walking its state elements through the segments; pass C recomputes every
// segment from its S_in and writes o (and the final state). One segment means pass C alone.
//
// CTA layout (160 threads): warps 0-3 = compute warpgroup, thread c <-> key channel c <->
// TMEM lane c of the state accumulator; warp 4 = TMA producer and TMEM allocator. Thread 0
// issues the MMAs. TMEM: S (128 cols, M=128), O (128 cols) and A (64 cols), both M=64 (rows
// 0-15 of each 32-lane quarter). Every wait is bounded; a timeout stops all roles, drains
// in-flight copies and MMAs, and raises a flag.
#include <cuda.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace rod {
namespace {

__device__ unsigned int g_gla_tc_timeout = 0;

constexpr int C = 64;                    // tokens per chunk
constexpr int D = 128;                   // d_k = d_v
constexpr int NTHREADS = 160;
constexpr int BOX_BYTES = C * 128;       // one 64-row x 64-col bf16 box (128 B rows) = 8 KB
constexpr int OP_BYTES = 2 * BOX_BYTES;  // one 64 x 128 bf16 operand = 16 KB
constexpr int G_BYTES = C * D * 4;       // 64 x 128 fp32 gates = 32 KB
// stage: q | k | v | g
constexpr int ST_Q = 0, ST_K = OP_BYTES, ST_V = 2 * OP_BYTES, ST_G = 3 * OP_BYTES;
constexpr int STAGE_BYTES = 3 * OP_BYTES + G_BYTES;          // 80 KB
constexpr int OFF_KHAT = 2 * STAGE_BYTES;                    // 16 KB
constexpr int OFF_P = OFF_KHAT + OP_BYTES;                   // 8 KB
constexpr int OFF_SBF = OFF_P + BOX_BYTES;                   // 32 KB (128 rows x 128 bf16)
constexpr int OFF_BAR = OFF_SBF + 2 * D * 128;
constexpr int NBAR = 8;                                      // full[2] empty[2] A O drain +1
constexpr int OFF_MISC = OFF_BAR + 8 * NBAR;
constexpr int SMEM_BYTES = OFF_MISC + 32 + 1024;
constexpr float kFastMin = 8.673617e-19f;                    // 2^-60
constexpr float kLog2Floor = -126.0f;                        // log2 of the smallest gate used

// TMEM columns
constexpr uint32_t TM_S = 0, TM_O = 128, TM_A = 256;

enum Mode { PASS_A = 0, PASS_C = 1 };

struct GlaArgs {
    const float* s_in;      // PASS_C: [BH][s_in_slots][D][D] incoming states (slot = segment)
    int s_in_slots;         // 1: every (b,h) reads slot 0 of s_in (initial state, single segment)
    float* state_out;       // PASS_C: [BH][D][D] final state, written by the last segment
    __nv_bfloat16* o;       // PASS_C: [BH][T][D]
    float* u_out;           // PASS_A: [BH][n_seg][D][D] (segment m writes slot m+1)
    float* a_out;           // PASS_A: [BH][n_seg][D]    (segment m writes slot m)
    int T, L_seg, n_seg;
};

// byte offset of element (row, col) of a K-major 128-byte-swizzled bf16 tile whose 64-column
// boxes hold `rows` rows each
__device__ __forceinline__ uint32_t sw_off(int row, int col, int rows) {
    const int box = col >> 6, cc = col & 63;
    return (uint32_t)(box * rows * 128 + row * 128 + ((((cc >> 3) ^ (row & 7))) << 4) + ((cc & 7) << 1));
}

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 0) {
            if (*abort_flag) return false;
            if (i >= kWaitLimit) {
                *abort_flag = 1;
                atomicExch(&g_gla_tc_timeout, 1u);
                return false;
            }
        }
    }
}

// barrier 1 over the 128 threads of the compute warpgroup (the producer warp never joins)
__device__ __forceinline__ void wg_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
__device__ __forceinline__ bool wg_all(bool pred) {
    uint32_t out;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, 1, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(out) : "r"((uint32_t)pred) : "memory");
    return out != 0;
}

__device__ __forceinline__ float bf(const unsigned char* base, uint32_t off) {
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(base + off));
}
__device__ __forceinline__ void put_bf(unsigned char* base, uint32_t off, float x) {
    *reinterpret_cast<__nv_bfloat16*>(base + off) = __float2bfloat16_rn(x);
}

template <int MODE>
__global__ void __launch_bounds__(NTHREADS, 1)
gla_chunk_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                 GlaArgs args) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32, tid = threadIdx.x;
    const int seg = blockIdx.x;
    const int bh = blockIdx.y;
    const int T = args.T;
    const int t_begin = seg * args.L_seg;
    const int t_end = min(T, t_begin + args.L_seg);
    const int n_ch = (t_end - t_begin + C - 1) / C;
    constexpr uint32_t kStageTx = MODE == PASS_C ? STAGE_BYTES : STAGE_BYTES - OP_BYTES;

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
    uint64_t* full = bars;         // [2]
    uint64_t* empty = bars + 2;    // [2]
    uint64_t* barA = bars + 4;
    uint64_t* barO = bars + 5;     // all MMAs of a chunk done
    uint64_t* drain = bars + 6;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);

    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(barA, 1);
        mbar_init(barO, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 4) {
        tc::tmem_alloc(tmem_holder, 512);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_holder;

    if (warp == 4) {
        // ------------------------------- TMA producer -------------------------------
        if (lane == 0) {
            int n = 0;
            for (; n < n_ch; ++n) {
                const int st = n & 1, use = n >> 1;
                if (use > 0 && !wait_bar(&empty[st], (uint32_t)((use - 1) & 1), abort_flag)) break;
                unsigned char* base = smem + st * STAGE_BYTES;
                const int y = t_begin + n * C;
                mbar_arrive_expect_tx(&full[st], kStageTx);
                for (int half = 0; half < 2; ++half) {
                    if (MODE == PASS_C)
                        tc::tma_load_3d(base + ST_Q + half * BOX_BYTES, &tm_q, half * 64, y, bh, &full[st]);
                    tc::tma_load_3d(base + ST_K + half * BOX_BYTES, &tm_k, half * 64, y, bh, &full[st]);
                    tc::tma_load_3d(base + ST_V + half * BOX_BYTES, &tm_v, half * 64, y, bh, &full[st]);
                }
                tc::tma_load_3d(base + ST_G, &tm_g, 0, y, bh, &full[st]);
            }
            for (int ni = (n > 2 ? n - 2 : 0); ni < n; ++ni)  // copies still in flight land first
                mbar_wait_bounded(&full[ni & 1], (uint32_t)((ni >> 1) & 1), kWaitLimit);
        }
    } else {
        // ------------------------------- compute warpgroup -------------------------------
        const int c = tid;                                 // key channel / state row / TMEM lane
        const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
        const uint32_t tS = tmem + TM_S + lane_base;
        const int orow = 16 * warp + lane;                 // row of the M=64 accumulators
        const bool orow_ok = lane < 16;
        float a_seg = 1.f;                                 // PASS_A: decay over the segment
        uint32_t nA = 0;                                   // completed MMA_A phases
        bool ok = true;

        const uint32_t idesc_A = tc::idesc_bf16_f32(64, 64, 0, 0);
        const uint32_t idesc_U = tc::idesc_bf16_f32(128, 128, 1, 1);
        const uint32_t idesc_O = tc::idesc_bf16_f32(64, 128, 0, 1);

        auto epilogue = [&](int n) {  // O rows of chunk n -> bf16 global rows
            const int t0 = t_begin + n * C;
#pragma unroll
            for (int cb = 0; cb < D; cb += 32) {
                uint32_t r[32];
                tc::tmem_ld32(tmem + TM_O + lane_base + cb, r);
                tc::tmem_wait_ld();
                const int t = t0 + orow;
                if (orow_ok && t < t_end) {
                    __nv_bfloat16* dst = args.o + ((int64_t)bh * T + t) * D + cb;
#pragma unroll
                    for (int i = 0; i < 32; i += 8) {
                        uint4 u;
                        u.x = pack_bf16x2(__uint_as_float(r[i + 0]), __uint_as_float(r[i + 1]));
                        u.y = pack_bf16x2(__uint_as_float(r[i + 2]), __uint_as_float(r[i + 3]));
                        u.z = pack_bf16x2(__uint_as_float(r[i + 4]), __uint_as_float(r[i + 5]));
                        u.w = pack_bf16x2(__uint_as_float(r[i + 6]), __uint_as_float(r[i + 7]));
                        *reinterpret_cast<uint4*>(dst + i) = u;
                    }
                }
            }
        };

        for (int n = 0; n < n_ch; ++n) {
            const int st = n & 1;
            unsigned char* base = smem + st * STAGE_BYTES;
            const int t0 = t_begin + n * C;
            const int nvalid = min(C, t_end - t0);
            // every wait of the warpgroup ends in a vote, so all 128 threads leave together
            if (!wg_all(wait_bar(&full[st], (uint32_t)((n >> 1) & 1), abort_flag))) { ok = false; break; }

            // ---- gates: prefix products G_t, suffix products F_t of channel c (rows >= nvalid: g = 1)
            const float* gcol = reinterpret_cast<const float*>(base + ST_G) + c;
            float G[C], F[C];
            float run = 1.f;
#pragma unroll
            for (int t = 0; t < C; ++t) {
                const float gt = t < nvalid ? gcol[t * D] : 1.f;
                run *= gt;
                G[t] = run;
            }
            const float a = run;  // decay of the whole chunk for channel c
            run = 1.f;
#pragma unroll
            for (int t = C - 1; t >= 0; --t) {
                F[t] = run;
                run *= t < nvalid ? gcol[t * D] : 1.f;
            }
            const bool fast = wg_all(a >= kFastMin);

            // ---- the previous chunk's MMAs are complete: its output rows, then its buffers are free
            if (n > 0) {
                if (!wg_all(wait_bar(barO, (uint32_t)((n - 1) & 1), abort_flag))) { ok = false; break; }
                tc::fence_after_sync();
                if (MODE == PASS_C) epilogue(n - 1);
            }

            if (MODE == PASS_C && !fast) {
                // A on the CUDA cores: A[t][s] = sum_c q_tc k_sc 2^(L_tc - L_sc), L = sum log2 g
                float* Lbuf = reinterpret_cast<float*>(smem + OFF_SBF);  // [C][D] fp32, free now
                float L = 0.f;
#pragma unroll 4
                for (int t = 0; t < C; ++t) {
                    const float gt = t < nvalid ? gcol[t * D] : 1.f;
                    L += fmaxf(__log2f(gt), kLog2Floor);
                    Lbuf[t * D + c] = L;
                }
                wg_sync();
                for (int pr = tid; pr < C * C; pr += 128) {
                    const int t = pr / C, s = pr % C;
                    float acc = 0.f;
                    if (s <= t) {
                        for (int cc = 0; cc < D; ++cc) {
                            const float w = exp2f(Lbuf[t * D + cc] - Lbuf[s * D + cc]);
                            acc = fmaf(bf(base + ST_Q, sw_off(t, cc, C)) * bf(base + ST_K, sw_off(s, cc, C)), w, acc);
                        }
                    }
                    put_bf(smem + OFF_P, sw_off(t, s, C), acc);
                }
                wg_sync();
            }

            // ---- operands: q~ = q.G (in place), k~ = k/G (in place), k^ = k.F
#pragma unroll
            for (int t = 0; t < C; ++t) {
                const uint32_t off = sw_off(t, c, C);
                const float kv = bf(base + ST_K, off);
                put_bf(smem + OFF_KHAT, off, kv * F[t]);
                if (MODE == PASS_C) {
                    put_bf(base + ST_Q, off, bf(base + ST_Q, off) * G[t]);
                    if (fast) put_bf(base + ST_K, off, kv * __frcp_rn(G[t]));
                }
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            tc::fence_before_sync();
            wg_sync();
            tc::fence_after_sync();
            if (MODE == PASS_C && fast && tid == 0) {
                const uint32_t qa = smem_u32(base + ST_Q), ka = smem_u32(base + ST_K);
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    const uint32_t koff = (uint32_t)((k / 4) * BOX_BYTES + (k % 4) * 32);
                    tc::mma_ss(tmem + TM_A, tc::sdesc_sw128(qa + koff, 16, 1024),
                               tc::sdesc_sw128(ka + koff, 16, 1024), idesc_A, k > 0);
                }
                tc::mma_commit(barA);
            }

            // ---- state row c: bf16 copy of S_in for the readout, then S <- diag(a) S in TMEM
            {
                uint32_t srow[D];  // fp32 bits of state row c
                if (n == 0) {
                    if (MODE == PASS_C) {
                        const int slot = args.s_in_slots == 1 ? 0 : seg;
                        const float* src = args.s_in + (((int64_t)bh * args.s_in_slots + slot) * D + c) * D;
#pragma unroll
                        for (int j = 0; j < D; j += 4) {
                            const uint4 v4 = *reinterpret_cast<const uint4*>(src + j);
                            srow[j] = v4.x; srow[j + 1] = v4.y; srow[j + 2] = v4.z; srow[j + 3] = v4.w;
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < D; ++j) srow[j] = 0u;
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < D; j += 32) tc::tmem_ld32(tS + j, srow + j);
                    tc::tmem_wait_ld();
                }
                if (MODE == PASS_C) {
                    unsigned char* sb = smem + OFF_SBF;
#pragma unroll
                    for (int j = 0; j < D; j += 8) {
                        uint4 u;
                        u.x = pack_bf16x2(__uint_as_float(srow[j]), __uint_as_float(srow[j + 1]));
                        u.y = pack_bf16x2(__uint_as_float(srow[j + 2]), __uint_as_float(srow[j + 3]));
                        u.z = pack_bf16x2(__uint_as_float(srow[j + 4]), __uint_as_float(srow[j + 5]));
                        u.w = pack_bf16x2(__uint_as_float(srow[j + 6]), __uint_as_float(srow[j + 7]));
                        *reinterpret_cast<uint4*>(sb + sw_off(c, j, D)) = u;
                    }
                }
#pragma unroll
                for (int j = 0; j < D; ++j) srow[j] = __float_as_uint(__uint_as_float(srow[j]) * a);
#pragma unroll
                for (int j = 0; j < D; j += 32) tc::tmem_st32(tS + j, srow + j);
                tc::tmem_wait_st();
            }
            a_seg *= a;
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            tc::fence_before_sync();
            wg_sync();
            tc::fence_after_sync();
            if (tid == 0) {  // S += k^^T V
                const uint32_t kh = smem_u32(smem + OFF_KHAT), va = smem_u32(base + ST_V);
#pragma unroll
                for (int k = 0; k < C / 16; ++k)
                    tc::mma_ss(tmem + TM_S, tc::sdesc_sw128(kh + 2048u * k, BOX_BYTES, 1024),
                               tc::sdesc_sw128(va + 2048u * k, BOX_BYTES, 1024), idesc_U, 1u);
            }

            if (MODE == PASS_C) {
                // ---- P = mask(A) in bf16 (fast path; the slow path wrote P above)
                if (fast) {
                    if (!wg_all(wait_bar(barA, nA & 1, abort_flag))) { ok = false; break; }
                    ++nA;
                    tc::fence_after_sync();
                    uint32_t r[64];
                    tc::tmem_ld32(tmem + TM_A + lane_base, r);
                    tc::tmem_ld32(tmem + TM_A + lane_base + 32, r + 32);
                    tc::tmem_wait_ld();
                    if (orow_ok) {
#pragma unroll
                        for (int s = 0; s < C; s += 8) {
                            uint4 u;
                            float f[8];
#pragma unroll
                            for (int i = 0; i < 8; ++i) f[i] = s + i <= orow ? __uint_as_float(r[s + i]) : 0.f;
                            u.x = pack_bf16x2(f[0], f[1]); u.y = pack_bf16x2(f[2], f[3]);
                            u.z = pack_bf16x2(f[4], f[5]); u.w = pack_bf16x2(f[6], f[7]);
                            *reinterpret_cast<uint4*>(smem + OFF_P + sw_off(orow, s, C)) = u;
                        }
                    }
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    tc::fence_before_sync();
                    wg_sync();
                    tc::fence_after_sync();
                }
                if (tid == 0) {  // O = P V + q~ S_in
                    const uint32_t pa = smem_u32(smem + OFF_P), va = smem_u32(base + ST_V);
                    const uint32_t qa = smem_u32(base + ST_Q), sb = smem_u32(smem + OFF_SBF);
#pragma unroll
                    for (int k = 0; k < C / 16; ++k)
                        tc::mma_ss(tmem + TM_O, tc::sdesc_sw128(pa + 32u * k, 16, 1024),
                                   tc::sdesc_sw128(va + 2048u * k, BOX_BYTES, 1024), idesc_O, k > 0);
#pragma unroll
                    for (int k = 0; k < D / 16; ++k)
                        tc::mma_ss(tmem + TM_O,
                                   tc::sdesc_sw128(qa + (uint32_t)((k / 4) * BOX_BYTES + (k % 4) * 32), 16, 1024),
                                   tc::sdesc_sw128(sb + 2048u * k, D * 128, 1024), idesc_O, 1u);
                }
            }
            if (tid == 0) {
                tc::mma_commit(barO);
                tc::mma_commit(&empty[st]);
            }
        }

        // ---- tail: last chunk's outputs and the segment's state
        if (ok && n_ch > 0 && wg_all(wait_bar(barO, (uint32_t)((n_ch - 1) & 1), abort_flag))) {
            tc::fence_after_sync();
            if (MODE == PASS_C) epilogue(n_ch - 1);
            float* dst = nullptr;
            if (MODE == PASS_C && seg == args.n_seg - 1) dst = args.state_out + ((int64_t)bh * D + c) * D;
            if (MODE == PASS_A) {
                dst = args.u_out + (((int64_t)bh * args.n_seg + seg + 1) * D + c) * D;
                args.a_out[((int64_t)bh * args.n_seg + seg) * D + c] = a_seg;
            }
            for (int j = 0; j < D; j += 32) {
                uint32_t r[32];
                tc::tmem_ld32(tS + j, r);
                tc::tmem_wait_ld();
                if (dst) {
#pragma unroll
                    for (int i = 0; i < 32; i += 4)
                        *reinterpret_cast<float4*>(dst + j + i) =
                            make_float4(__uint_as_float(r[i]), __uint_as_float(r[i + 1]),
                                        __uint_as_float(r[i + 2]), __uint_as_float(r[i + 3]));
                }
            }
        }
        if (tid == 0) {  // every MMA issued has completed before TMEM is released
            tc::mma_commit(drain);
            mbar_wait_bounded(drain, 0, kWaitLimit);
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 4) tc::tmem_dealloc(tmem, 512);
}

// S_in(0) = state; S_in(m+1) = diag(a_m) S_in(m) + U_m in place of U_m, for every (b, h) and
// state element; each thread owns 4 consecutive elements of one state row and walks the
// segments in order, with the next segment's U loaded ahead of the dependent update.
__global__ void __launch_bounds__(256)
gla_segment_scan_kernel(const float* __restrict__ state, float* __restrict__ s_slots,
                        const float* __restrict__ a_seg, int n_seg) {
    const int64_t bh = blockIdx.y;
    const int e4 = blockIdx.x * blockDim.x + threadIdx.x;  // float4 index in the D x D state
    if (e4 >= D * D / 4) return;
    const int row = (e4 * 4) / D;
    const size_t slot_stride = (size_t)D * D;
    float* base = s_slots + bh * (int64_t)n_seg * slot_stride;
    float4 s = reinterpret_cast<const float4*>(state + bh * slot_stride)[e4];
    reinterpret_cast<float4*>(base)[e4] = s;
    float4 u_next = n_seg > 1 ? reinterpret_cast<const float4*>(base + slot_stride)[e4]
                              : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int m = 0; m + 1 < n_seg; ++m) {
        const float4 u = u_next;
        if (m + 2 < n_seg) u_next = reinterpret_cast<const float4*>(base + (m + 2) * slot_stride)[e4];
        const float am = a_seg[(bh * n_seg + m) * D + row];
        s.x = fmaf(am, s.x, u.x);
        s.y = fmaf(am, s.y, u.y);
        s.z = fmaf(am, s.z, u.z);
        s.w = fmaf(am, s.w, u.w);
        reinterpret_cast<float4*>(base + (m + 1) * slot_stride)[e4] = s;
    }
}

struct Plan {
    int L_seg, n_seg;
};

Plan plan(int B, int H, int T) {
    const int64_t BH = (int64_t)B * H;
    const int chunks = (T + C - 1) / C;
    int64_t want = (4 * 148 + BH - 1) / BH;  // about four waves of one-CTA-per-SM units
    if (want < 1) want = 1;
    if (want > chunks) want = chunks;
    const int per = (int)((chunks + want - 1) / want);
    Plan p;
    p.L_seg = per * C;
    p.n_seg = (T + p.L_seg - 1) / p.L_seg;
    return p;
}

}  // namespace

bool gla_prefill_tc_supported(int dk, int dv, int chunk) { return dk == D && dv == D && chunk == C; }

size_t gla_prefill_tc_workspace_size(int B, int H, int T) {
    const Plan p = plan(B, H, T);
    if (p.n_seg <= 1) return 0;
    return (size_t)B * H * p.n_seg * ((size_t)D * D + D) * sizeof(float);
}

cudaError_t gla_prefill_tc_launch(const void* q, const void* k, const void* v, const float* g,
                                  float* state, void* o, int B, int H, int T, void* workspace,
                                  cudaStream_t stream) {
    const Plan p = plan(B, H, T);
    const int64_t BH = (int64_t)B * H;
    if (BH > 65535) return cudaErrorInvalidConfiguration;
    CUtensorMap mq, mk, mv, mg;
    cudaError_t e;
    if ((e = make_tmap_3d(&mq, q, false, D, (uint64_t)T, (uint64_t)BH, 64, C, true)) != cudaSuccess) return e;
    if ((e = make_tmap_3d(&mk, k, false, D, (uint64_t)T, (uint64_t)BH, 64, C, true)) != cudaSuccess) return e;
    if ((e = make_tmap_3d(&mv, v, false, D, (uint64_t)T, (uint64_t)BH, 64, C, true)) != cudaSuccess) return e;
    if ((e = make_tmap_3d(&mg, g, true, D, (uint64_t)T, (uint64_t)BH, D, C, false)) != cudaSuccess) return e;
    for (auto fn : {gla_chunk_kernel<PASS_A>, gla_chunk_kernel<PASS_C>}) {
        e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        if (e != cudaSuccess) return e;
    }
    GlaArgs a{};
    a.T = T;
    a.L_seg = p.L_seg;
    a.n_seg = p.n_seg;
    a.o = static_cast<__nv_bfloat16*>(o);
    a.state_out = state;
    if (p.n_seg == 1) {
        a.s_in = state;
        a.s_in_slots = 1;
    } else {
        float* slots = static_cast<float*>(workspace);
        float* aseg = slots + (size_t)BH * p.n_seg * D * D;
        a.u_out = slots;
        a.a_out = aseg;
        gla_chunk_kernel<PASS_A><<<dim3((unsigned)(p.n_seg - 1), (unsigned)BH), NTHREADS, SMEM_BYTES, stream>>>(
            mq, mk, mv, mg, a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        gla_segment_scan_kernel<<<dim3((D * D / 4 + 255) / 256, (unsigned)BH), 256, 0, stream>>>(
            state, slots, aseg, p.n_seg);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        note_launches(2);
        a.s_in = slots;
        a.s_in_slots = p.n_seg;
    }
    gla_chunk_kernel<PASS_C><<<dim3((unsigned)p.n_seg, (unsigned)BH), NTHREADS, SMEM_BYTES, stream>>>(
        mq, mk, mv, mg, a);
    note_launches(1);
    return cudaGetLastError();
}

unsigned gla_prefill_tc_take_timeout_flag() {
    unsigned v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_gla_tc_timeout, sizeof(v)) != cudaSuccess) return 0;
    cudaMemcpyToSymbol(g_gla_tc_timeout, &zero, sizeof(zero));
    return v;
}

}  // namespace rod
