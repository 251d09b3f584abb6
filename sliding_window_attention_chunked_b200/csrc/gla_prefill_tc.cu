// gla_prefill_tc.cu -- chunkwise-parallel prefill of the Rodimus gated linear recurrence on the
// 5th-generation tensor cores (tcgen05 / TMEM / TMA), bf16 q, k, v / fp32 gates and state,
// d_k = d_v = 128, chunks of 64 tokens.
//
// Recurrence (CodeFuse Rodimus* article, Rodimus block; SALA blog §2.2 state form, §4.3 decay):
//     S_t = diag(g_t) S_{t-1} + k_t^T v_t,     o_t = q_t S_t.
// Chunk form (the chunkwise-parallel algorithm the Rodimus block paragraph names for training
// and prefill). For a chunk of C tokens with incoming state S_in, per key channel c let
//     G_t = prod_{r<=t} g_r     (prefix product inside the chunk),   a = G_{C-1},
//     F_t = prod_{t<r<=C-1} g_r = a / G_t   (suffix product).
// Then, exactly,
//     o_t   = sum_{s<=t} (sum_c q_tc k_sc G_tc / G_sc) v_s + (q_t . G_t) S_in
//     S_out = diag(a) S_in + sum_s (k_s . F_s)^T v_s.
// With q~ = q.G, k~ = k/G, k^ = k.F the chunk is four dense contractions on the tensor cores:
//     A = q~ k~^T (masked to s <= t, rounded to bf16 as P),  O = P V + q~ S_in,  S += k^^T V
// while the fp32 state lives in tensor memory for the whole segment. k~ = k/G needs G well
// inside the fp32/bf16 exponent range, so a chunk in which some channel's product a falls below
// 2^-60 takes the exact route instead: the scores are summed on the CUDA cores from log2-gate
// prefix sums L (log2 g clamped at -126, so g = 0 contributes below fp32 resolution),
// A_ts = sum_c q_tc k_sc 2^(L_tc - L_sc), and written straight into tensor memory, where the
// tensor-core route would have put them; q~ = q.2^L and k^ = k.2^(L_last - L).
// The state is held as S = diag(D) R with a running per-channel decay D: a chunk multiplies D
// by a and adds (k^/D)^T V to R, so R is never read and rewritten per chunk; D is folded into
// q~ for the readout, and R is rescaled (D reset to 1) only when D would fall below 2^-40.
//
// Parallelism over the sequence: the T tokens are cut into segments of L_seg tokens. Pass A
// (per segment but the last) computes the segment's state contribution U and decay a_seg
// from k, v, g; a scan kernel chains S_in(m+1) = diag(a_seg,m) S_in(m) + U_m per (b, h);
// pass C recomputes every segment from its S_in and writes o (and the final state). One
// segment means pass C alone.
//
// CTA (384 threads = 3 warpgroups, setmaxnreg 232 / 216 / 56), a pipeline over the chunks of
// a segment through two 80 KB stages:
//   warp 8        TMA producer (q, k, v, g of chunk n into stage n % 2, L2 prefetch of later
//                 chunks) and TMEM allocator (warps 9-11 idle: they complete the warpgroup
//                 that gives its registers away);
//   warpgroup 0   operands of chunk n: gate prefix products (8 rows x 8 channels per thread,
//                 block products combined through shared memory), q~ and k^ in place over q
//                 and k, k~ over the gates; thread 0 issues A = q~ k~^T into TMEM buffer n % 2;
//   warpgroup 1   state work: P = mask(A) of chunk n into the stage, output rows of chunk n-1,
//                 the state row c (thread c = TMEM lane c) copied to bf16 for the readout, and
//                 thread 128 issues R += k^'^T V and O = P V + q~' R_bf16.
// So the operands of chunk n+1 are built while chunk n's state work and MMAs run.
// TMEM: S (cols 0-127, M=128), O (128-255, M=64: rows in lanes 0-15 of each 32-lane quarter),
// A0 / A1 (256-319 / 320-383, M=64). Every wait is bounded; a timeout stops all roles, drains
// in-flight copies and MMAs, and raises a flag.
#include <cuda.h>
#include <math.h>

#include <atomic>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace rod {
namespace {

__device__ unsigned int g_gla_tc_timeout = 0;

constexpr int C = 64;                    // tokens per chunk
constexpr int D = 128;                   // d_k = d_v
constexpr int NTHREADS = 384;            // 3 warpgroups: operands, state, producer (+3 idle)
// Register split (setmaxnreg). Each of the SM's four sub-partitions holds one warp of every
// warpgroup, so per sub-partition the launch provides 3 x 168 = 504 registers per lane; the split
// 232 (operands) + 216 (state) + 56 (producer warpgroup) = 504 uses exactly that.
constexpr int kLaunchRegs = 168;
constexpr int kOperandRegs = 232;
constexpr int kStateRegs = 216;
constexpr int kControlRegs = 56;
static_assert(kOperandRegs + kStateRegs + kControlRegs <= 3 * kLaunchRegs, "register split exceeds launch");
constexpr int BOX_BYTES = C * 128;       // one 64-row x 64-col bf16 box (128 B rows) = 8 KB
constexpr int OP_BYTES = 2 * BOX_BYTES;  // one 64 x 128 bf16 operand = 16 KB
constexpr int G_BYTES = C * D * 4;       // 64 x 128 fp32 gates = 32 KB
// stage: q | k | v | g      (after warpgroup 0: q~ | k^ | v | k~ (first 16 KB) ...)
constexpr int ST_Q = 0, ST_K = OP_BYTES, ST_V = 2 * OP_BYTES, ST_G = 3 * OP_BYTES;
constexpr int STAGE_BYTES = 3 * OP_BYTES + G_BYTES;          // 80 KB
constexpr int ST_P = ST_G + OP_BYTES;                        // P (64 x 64 bf16) after k~
constexpr int OFF_SBF = 2 * STAGE_BYTES;                     // 32 KB  R in bf16 for the readout
constexpr int OFF_SCAN = OFF_SBF + 2 * D * 128;              // 4 KB   block products [8][128]
constexpr int OFF_ABUF = OFF_SCAN + 8 * D * 4;               // 2 KB   a and D.a per stage
constexpr int OFF_FLAG = OFF_ABUF + 4 * D * 4;               // 16 B   route / rescale flags
constexpr int OFF_BAR = OFF_FLAG + 16;
constexpr int NBAR = 12;
constexpr int OFF_MISC = OFF_BAR + 8 * NBAR;
constexpr int SMEM_BYTES = OFF_MISC + 32 + 1024;
constexpr float kFastMin = 8.673617e-19f;                    // 2^-60: chunk decay for q~ k~^T
constexpr float kRescaleMin = 9.094947e-13f;                 // 2^-40: smallest running decay D
constexpr int kFlagExact = 1, kFlagRescale = 2;
constexpr float kLog2Floor = -126.0f;                        // log2 of the smallest gate used
constexpr int kPrefetchChunks = 3;                           // L2 prefetch distance in chunks

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
    const __nv_bfloat16 *q, *k, *v;  // the inputs again, for L2 prefetches ahead of TMA
    const float* g;
    int T, L_seg, n_seg;
    uint32_t wait_limit;    // probes before a wait gives up (kWaitLimit; smaller only in tests)
    int copies_off;         // nonzero only in the wait-expiry test: the producer issues no copies
};

// byte offset of the 16-byte chunk holding columns [col, col + 8) of row `row` in a K-major
// 128-byte-swizzled bf16 tile whose 64-column boxes hold `rows` rows each (col % 8 == 0)
__device__ __forceinline__ uint32_t sw_off(int row, int col, int rows) {
    const int box = col >> 6, cc = col & 63;
    return (uint32_t)(box * rows * 128 + row * 128 + ((((cc >> 3) ^ (row & 7))) << 4));
}
// byte offset of one bf16 element (row, col) of such a tile
__device__ __forceinline__ uint32_t sw_off_elem(int row, int col, int rows) {
    return sw_off(row, col & ~7, rows) + ((col & 7) << 1);
}

// fp32 pairs in one 64-bit register for the two-wide instructions
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

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                         uint32_t limit) {
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 0) {
            if (*abort_flag) return false;
            if (i >= limit) {
                *abort_flag = 1;
                atomicExch(&g_gla_tc_timeout, 1u);
                return false;
            }
        }
    }
}

// named barriers: id 1 = warpgroup 0, id 2 = warpgroup 1 (128 threads each); the producer warp
// and the other warpgroup never join them
__device__ __forceinline__ void grp_sync(int id) {
    asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory");
}
__device__ __forceinline__ bool grp_all(int id, bool pred) {
    uint32_t out;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %2, 0;\n\t"
        "bar.red.and.pred q, %1, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(out) : "r"(id), "r"((uint32_t)pred) : "memory");
    return out != 0;
}

__device__ __forceinline__ void unpack8(const uint4& u, float* f) {
    f[0] = bf16lo(u.x); f[1] = bf16hi(u.x); f[2] = bf16lo(u.y); f[3] = bf16hi(u.y);
    f[4] = bf16lo(u.z); f[5] = bf16hi(u.z); f[6] = bf16lo(u.w); f[7] = bf16hi(u.w);
}
__device__ __forceinline__ uint4 pack8(const float* f) {
    uint4 u;
    u.x = pack_bf16x2(f[0], f[1]); u.y = pack_bf16x2(f[2], f[3]);
    u.z = pack_bf16x2(f[4], f[5]); u.w = pack_bf16x2(f[6], f[7]);
    return u;
}
// true when no channel's running decay D * a would fall below 2^-40 (no rescale of R needed)
__device__ __forceinline__ bool rescale_vote(const float* Dc, const float* a) {
    bool ok = true;
#pragma unroll
    for (int j = 0; j < 8; ++j) ok = ok && Dc[j] * a[j] >= kRescaleMin;
    return ok;
}

__device__ __forceinline__ float ldbf(const unsigned char* p) {
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(p));
}
__device__ __forceinline__ float rcp(float x) {  // 1/x on the SFU (about 1 ulp)
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float lg2(float x) {  // log2 on the SFU (0 gives -inf)
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
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
    uint64_t* full = bars;         // [2] TMA -> warpgroup 0
    uint64_t* empty = bars + 2;    // [2] chunk MMAs done -> producer
    uint64_t* ops = bars + 4;      // [2] operands ready -> warpgroup 1
    uint64_t* barA = bars + 6;     // [2] A = q~ k~^T done
    uint64_t* barO = bars + 8;     // all MMAs of warpgroup 1 for a chunk done
    uint64_t* drain0 = bars + 9;
    uint64_t* drain1 = bars + 10;
    float* abuf = reinterpret_cast<float*>(smem + OFF_ABUF);
    volatile int* flag = reinterpret_cast<volatile int*>(smem + OFF_FLAG);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);

    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&ops[s], 1);
            mbar_init(&barA[s], 1);
        }
        mbar_init(barO, 1);
        mbar_init(drain0, 1);
        mbar_init(drain1, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 8) {
        tc::tmem_alloc(tmem_holder, 512);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_holder;
    const uint32_t wlim = args.wait_limit;
    bool ok = true;

    if (warp >= 8) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kControlRegs));
    }
    if (warp == 8) {
        // ------------------------------- TMA producer -------------------------------
        if (lane == 0) {
            int n = 0;
            for (; n < n_ch && !args.copies_off; ++n) {
                const int st = n & 1, use = n >> 1;
                if (use > 0 && !wait_bar(&empty[st], (uint32_t)((use - 1) & 1), abort_flag, wlim)) break;
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
                // keep later chunks of the segment streaming into L2 while the two stages turn over
                const int pf = n + kPrefetchChunks;
                if (pf < n_ch) {
                    const int yp = t_begin + pf * C;
                    const uint32_t rows = (uint32_t)min(C, t_end - yp);
                    const int64_t row0 = (int64_t)bh * T + yp;
                    if (MODE == PASS_C) tc::prefetch_l2(args.q + row0 * D, rows * D * 2);
                    tc::prefetch_l2(args.k + row0 * D, rows * D * 2);
                    tc::prefetch_l2(args.v + row0 * D, rows * D * 2);
                    tc::prefetch_l2(args.g + row0 * D, rows * D * 4);
                }
            }
            for (int ni = (n > 2 ? n - 2 : 0); ni < n; ++ni)  // copies still in flight land first
                mbar_wait_bounded(&full[ni & 1], (uint32_t)((ni >> 1) & 1), kWaitLimit);
        }
    } else if (warp < 4) {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kOperandRegs));
        // ------------------------------- warpgroup 0: operands -------------------------------
        // thread = (channel group cg: channels 8cg..8cg+7, row block rb: rows 8rb..8rb+7)
        const int cg = tid & 15, rb = tid >> 4;
        const int c0 = 8 * cg, r0 = 8 * rb;
        const bool rot = ((cg >> 2) & 1) != 0;  // alternate float4 halves: no bank conflicts
        float* scan = reinterpret_cast<float*>(smem + OFF_SCAN);
        const uint32_t idesc_A = tc::idesc_bf16_f32(64, 64, 0, 0);
        // The state is kept as S = diag(D) R with a running per-channel decay D (reset to 1 by a
        // rescale of R when it would drop below 2^-40), so that chunk contributions enter R as
        // k^/D without touching R: D of my 8 channels (same in every row-block thread)
        float Dc[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) Dc[j] = 1.f;
        for (int n = 0; n < n_ch; ++n) {
            const int st = n & 1;
            unsigned char* base = smem + st * STAGE_BYTES;
            float* gsm = reinterpret_cast<float*>(base + ST_G);
            const int nvalid = min(C, t_end - (t_begin + n * C));
            if (!grp_all(1, wait_bar(&full[st], (uint32_t)((n >> 1) & 1), abort_flag, wlim))) { ok = false; break; }

            auto load_gates = [&](int i, float* g8) {  // gates of row r0+i, my 8 channels
                const float4* p = reinterpret_cast<const float4*>(gsm + (r0 + i) * D + c0);
                const float4 x0 = p[rot ? 1 : 0], x1 = p[rot ? 0 : 1];
                const float4 lo = rot ? x1 : x0, hi = rot ? x0 : x1;
                g8[0] = lo.x; g8[1] = lo.y; g8[2] = lo.z; g8[3] = lo.w;
                g8[4] = hi.x; g8[5] = hi.y; g8[6] = hi.z; g8[7] = hi.w;
            };
            // prefix products of the gates: inside my row block, then across row blocks
            float G[8][8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                float g8[8];
                load_gates(i, g8);
                const bool valid = r0 + i < nvalid;  // rows past the sequence end: g = 1
#pragma unroll
                for (int j = 0; j < 8; ++j) G[i][j] = (valid ? g8[j] : 1.f) * (i > 0 ? G[i - 1][j] : 1.f);
            }
            *reinterpret_cast<float4*>(scan + rb * D + c0) = make_float4(G[7][0], G[7][1], G[7][2], G[7][3]);
            *reinterpret_cast<float4*>(scan + rb * D + c0 + 4) = make_float4(G[7][4], G[7][5], G[7][6], G[7][7]);
            grp_sync(1);
            float pre[8], a[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) { pre[j] = 1.f; a[j] = 1.f; }
#pragma unroll
            for (int b2 = 0; b2 < 8; ++b2) {
                const float4 lo = *reinterpret_cast<const float4*>(scan + b2 * D + c0);
                const float4 hi = *reinterpret_cast<const float4*>(scan + b2 * D + c0 + 4);
                const float v[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (b2 < rb) pre[j] *= v[j];
                    a[j] *= v[j];
                }
            }
            bool mine = true;
#pragma unroll
            for (int j = 0; j < 8; ++j) mine = mine && a[j] >= kFastMin;
            // vote (also a barrier: every gate and block product has been read past here)
            const bool fast = grp_all(1, mine);
            // hand a, the rescale factor D.a and the route to warpgroup 1; advance D
            auto publish = [&](bool rmw, const float* dn) {
                if (rb == 0) {
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        abuf[(st * 2 + 0) * D + c0 + j] = a[j];
                        abuf[(st * 2 + 1) * D + c0 + j] = Dc[j] * a[j];
                    }
                }
                if (tid == 0) flag[st] = (fast ? 0 : kFlagExact) | (rmw ? kFlagRescale : 0);
#pragma unroll
                for (int j = 0; j < 8; ++j) Dc[j] = dn[j];
            };

            if (fast) {
                // q~ = q.G.D over q, k^ = k.(a/G)/D' over k, k~ = k/(G.D) over the (consumed) gates
                const bool rmw = !grp_all(1, rescale_vote(Dc, a));
                float dn[8], a_dn[8], inv_d[8];  // per-channel factors, hoisted out of the rows
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    dn[j] = rmw ? 1.f : Dc[j] * a[j];
                    a_dn[j] = a[j] * rcp(dn[j]);
                    inv_d[j] = rcp(Dc[j]);
                }
                // channel pairs in two-wide fp32 registers (mul.rn.f32x2: one instruction per pair)
                uint64_t pre2[4], adn2[4], dc2[4], invd2[4];
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    pre2[p] = pk2(pre[2 * p], pre[2 * p + 1]);
                    adn2[p] = pk2(a_dn[2 * p], a_dn[2 * p + 1]);
                    dc2[p] = pk2(Dc[2 * p], Dc[2 * p + 1]);
                    invd2[p] = pk2(inv_d[2 * p], inv_d[2 * p + 1]);
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint32_t off = sw_off(r0 + i, c0, C);
                    const uint4 kw = *reinterpret_cast<const uint4*>(base + ST_K + off);
                    uint4 qw = make_uint4(0u, 0u, 0u, 0u);
                    if (MODE == PASS_C) qw = *reinterpret_cast<const uint4*>(base + ST_Q + off);
                    const uint32_t kws[4] = {kw.x, kw.y, kw.z, kw.w}, qws[4] = {qw.x, qw.y, qw.z, qw.w};
                    uint32_t khp[4], qtp[4], ktp[4];
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        const uint64_t kf2 = pk2(bf16lo(kws[p]), bf16hi(kws[p]));
                        const uint64_t Gt2 = mul2(pk2(G[i][2 * p], G[i][2 * p + 1]), pre2[p]);
                        const float2 gt = upk2(Gt2);
                        const uint64_t r2 = pk2(rcp(gt.x), rcp(gt.y));
                        const float2 kh = upk2(mul2(kf2, mul2(r2, adn2[p])));
                        khp[p] = pack_bf16x2(kh.x, kh.y);
                        if (MODE == PASS_C) {
                            const float2 qt = upk2(mul2(pk2(bf16lo(qws[p]), bf16hi(qws[p])), mul2(Gt2, dc2[p])));
                            const float2 kt = upk2(mul2(kf2, mul2(r2, invd2[p])));
                            qtp[p] = pack_bf16x2(qt.x, qt.y);
                            ktp[p] = pack_bf16x2(kt.x, kt.y);
                        }
                    }
                    *reinterpret_cast<uint4*>(base + ST_K + off) = make_uint4(khp[0], khp[1], khp[2], khp[3]);
                    if (MODE == PASS_C) {
                        *reinterpret_cast<uint4*>(base + ST_Q + off) = make_uint4(qtp[0], qtp[1], qtp[2], qtp[3]);
                        *reinterpret_cast<uint4*>(base + ST_G + off) = make_uint4(ktp[0], ktp[1], ktp[2], ktp[3]);
                    }
                }
                publish(rmw, dn);
            } else {
                // exact route: L = prefix sums of clamped log2 gates, block sums through shared memory
                float L[8][8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    float g8[8];
                    load_gates(i, g8);
                    const bool valid = r0 + i < nvalid;
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        L[i][j] = (valid ? fmaxf(lg2(g8[j]), kLog2Floor) : 0.f) + (i > 0 ? L[i - 1][j] : 0.f);
                }
                *reinterpret_cast<float4*>(scan + rb * D + c0) = make_float4(L[7][0], L[7][1], L[7][2], L[7][3]);
                *reinterpret_cast<float4*>(scan + rb * D + c0 + 4) = make_float4(L[7][4], L[7][5], L[7][6], L[7][7]);
                grp_sync(1);
                float preL[8], Ltot[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) { preL[j] = 0.f; Ltot[j] = 0.f; }
#pragma unroll
                for (int b2 = 0; b2 < 8; ++b2) {
                    const float4 lo = *reinterpret_cast<const float4*>(scan + b2 * D + c0);
                    const float4 hi = *reinterpret_cast<const float4*>(scan + b2 * D + c0 + 4);
                    const float v[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        if (b2 < rb) preL[j] += v[j];
                        Ltot[j] += v[j];
                    }
                }
                grp_sync(1);  // block sums and gates read before either is overwritten
#pragma unroll
                for (int j = 0; j < 8; ++j) a[j] = tc::ex2(Ltot[j]);
#pragma unroll
                for (int i = 0; i < 8; ++i)
#pragma unroll
                    for (int j = 0; j < 8; ++j) L[i][j] += preL[j];
                if (MODE == PASS_C) {
                    // L over the gates, then the exact scores of row t = 16 w + l into TMEM A[st]
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        *reinterpret_cast<float4*>(gsm + (r0 + i) * D + c0) = make_float4(L[i][0], L[i][1], L[i][2], L[i][3]);
                        *reinterpret_cast<float4*>(gsm + (r0 + i) * D + c0 + 4) = make_float4(L[i][4], L[i][5], L[i][6], L[i][7]);
                    }
                    grp_sync(1);
                    const int w = tid >> 5, l = tid & 31, trow = 16 * w + l;
                    const uint32_t tA = tmem + TM_A + 64u * st + ((uint32_t)(32 * w) << 16);
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        uint32_t ar[32];
#pragma unroll
                        for (int jj = 0; jj < 32; ++jj) {
                            const int s = 32 * half + jj;
                            float acc = 0.f;
                            if (l < 16 && s <= trow) {
                                for (int cc = 0; cc < D; ++cc) {
                                    const float wgt = tc::ex2(gsm[trow * D + cc] - gsm[s * D + cc]);
                                    acc = fmaf(ldbf(base + ST_Q + sw_off_elem(trow, cc, C)) *
                                                   ldbf(base + ST_K + sw_off_elem(s, cc, C)), wgt, acc);
                                }
                            }
                            ar[jj] = __float_as_uint(acc);
                        }
                        tc::tmem_st32(tA + 32u * half, ar);
                    }
                    tc::tmem_wait_st();
                    grp_sync(1);  // q, k and L read by every thread before they are overwritten
                }
                // q~ = q.2^L.D over q, k^ = k.2^(Ltot - L)/D' over k
                const bool rmw = !grp_all(1, rescale_vote(Dc, a));
                float dn[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) dn[j] = rmw ? 1.f : Dc[j] * a[j];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint32_t off = sw_off(r0 + i, c0, C);
                    float qf[8], kf[8], qt[8], kh[8];
                    unpack8(*reinterpret_cast<const uint4*>(base + ST_K + off), kf);
                    if (MODE == PASS_C) unpack8(*reinterpret_cast<const uint4*>(base + ST_Q + off), qf);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        kh[j] = kf[j] * tc::ex2(Ltot[j] - L[i][j]) * rcp(dn[j]);
                        if (MODE == PASS_C) qt[j] = qf[j] * (tc::ex2(L[i][j]) * Dc[j]);
                    }
                    *reinterpret_cast<uint4*>(base + ST_K + off) = pack8(kh);
                    if (MODE == PASS_C) *reinterpret_cast<uint4*>(base + ST_Q + off) = pack8(qt);
                }
                publish(rmw, dn);
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            tc::fence_before_sync();
            grp_sync(1);
            if (warp == 0) {
                // the whole warp issues in lockstep, one lane elected inside each instruction
                tc::fence_after_sync();
                if (MODE == PASS_C && fast) {
                    // descriptors built once; a K step adds its offset (bytes >> 4) to the low word
                    const uint64_t dq = tc::sdesc_sw128(smem_u32(base + ST_Q), 16, 1024);
                    const uint32_t q_lo = tc::desc_lo(dq), hi = tc::desc_hi(dq);
                    const uint32_t k_lo = tc::desc_lo(tc::sdesc_sw128(smem_u32(base + ST_G), 16, 1024));
#pragma unroll
                    for (int k = 0; k < D / 16; ++k) {
                        const uint32_t koff = (uint32_t)(((k / 4) * BOX_BYTES + (k % 4) * 32) >> 4);
                        tc::mma_ss_lh_warp(tmem + TM_A + 64u * st, q_lo + koff, hi, k_lo + koff, hi, idesc_A, k > 0);
                    }
                    tc::mma_commit_warp(&barA[st]);
                }
                if (lane == 0) mbar_arrive(&ops[st]);
            }
        }
        if (warp == 0) {  // every MMA this warp issued has completed before TMEM is released
            tc::mma_commit_warp(drain0);
            mbar_wait_bounded(drain0, 0, kWaitLimit);
        }
    } else if (warp < 8) {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kStateRegs));
        // ------------------------- warpgroup 1: state, P, outputs, MMAs -------------------------
        const int c = tid - 128;                           // state row == TMEM lane
        const int wq = warp - 4;                           // TMEM lane quarter of this warp
        const uint32_t lane_base = (uint32_t)(32 * wq) << 16;
        const uint32_t tS = tmem + TM_S + lane_base;
        const int orow = 16 * wq + lane;                   // row of the M=64 accumulators
        const bool orow_ok = lane < 16;
        const uint32_t idesc_U = tc::idesc_bf16_f32(128, 128, 1, 1);
        const uint32_t idesc_O = tc::idesc_bf16_f32(64, 128, 0, 1);
        float a_seg = 1.f;                                 // PASS_A: decay over the segment
        float Drow = 1.f;                                  // running decay D of state row c
        uint32_t nA0 = 0, nA1 = 0;                         // completed A phases per TMEM buffer

        auto epilogue = [&](int n) {  // O rows of chunk n -> bf16 global rows
            const int t0 = t_begin + n * C;
            uint32_t r[D];
#pragma unroll
            for (int cb = 0; cb < D; cb += 32) tc::tmem_ld32(tmem + TM_O + lane_base + cb, r + cb);
            tc::tmem_wait_ld();
            const int t = t0 + orow;
            if (orow_ok && t < t_end) {
                __nv_bfloat16* dst = args.o + ((int64_t)bh * T + t) * D;
#pragma unroll
                for (int i = 0; i < D; i += 8) {
                    float f[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(r[i + e]);
                    *reinterpret_cast<uint4*>(dst + i) = pack8(f);
                }
            }
        };

        for (int n = 0; n < n_ch; ++n) {
            const int st = n & 1;
            unsigned char* base = smem + st * STAGE_BYTES;
            if (!grp_all(2, wait_bar(&ops[st], (uint32_t)((n >> 1) & 1), abort_flag, wlim))) { ok = false; break; }
            tc::fence_after_sync();
            const int fl = flag[st];
            const bool exact = (fl & kFlagExact) != 0, rmw = (fl & kFlagRescale) != 0;
            const float a_n = abuf[(st * 2 + 0) * D + c];
            const float sig = abuf[(st * 2 + 1) * D + c];  // D_prev * a: R's rescale factor
            if (MODE == PASS_C) {
                // P = mask(A) in bf16 into this stage (A came from the tensor cores or, on the
                // exact route, was stored into TMEM by warpgroup 0 before the operands signal)
                if (!exact) {
                    const uint32_t ph = st == 0 ? nA0 : nA1;
                    if (!grp_all(2, wait_bar(&barA[st], ph & 1, abort_flag, wlim))) { ok = false; break; }
                    if (st == 0) ++nA0; else ++nA1;
                    tc::fence_after_sync();
                }
                uint32_t r[64];
                tc::tmem_ld32(tmem + TM_A + 64u * st + lane_base, r);
                tc::tmem_ld32(tmem + TM_A + 64u * st + lane_base + 32, r + 32);
                tc::tmem_wait_ld();
                if (orow_ok) {
#pragma unroll
                    for (int s = 0; s < C; s += 8) {
                        float f[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) f[i] = s + i <= orow ? __uint_as_float(r[s + i]) : 0.f;
                        *reinterpret_cast<uint4*>(base + ST_P + sw_off(orow, s, C)) = pack8(f);
                    }
                }
            }
            // pass C needs the previous chunk's MMAs done every chunk (its outputs, S_bf reuse);
            // pass A when R is rescaled (S = diag(D) R takes new terms without touching R), and
            // before its last chunk: the tail then waits for the last phase of barO with every
            // earlier phase known complete (a parity wait must not be two phases ahead)
            const bool need_prev = n > 0 && (MODE == PASS_C || rmw || n == n_ch - 1);
            if (need_prev) {
                if (!grp_all(2, wait_bar(barO, (uint32_t)((n - 1) & 1), abort_flag, wlim))) { ok = false; break; }
                tc::fence_after_sync();
                if (MODE == PASS_C) epilogue(n - 1);
            }
            // state row c: bf16 copy of R for the readout (S_in = diag(D) R, D folded into q~),
            // and R <- sig R when the running decay is reset; R starts as S_in (pass C) or 0
            if (MODE == PASS_C || (rmw && n > 0)) {
                uint32_t r[D];
                if (n == 0) {
                    const int slot = args.s_in_slots == 1 ? 0 : seg;
                    const uint4* src = reinterpret_cast<const uint4*>(
                        args.s_in + (((int64_t)bh * args.s_in_slots + slot) * D + c) * D);
#pragma unroll
                    for (int e = 0; e < D / 4; ++e) {
                        const uint4 v4 = src[e];
                        r[4 * e] = v4.x; r[4 * e + 1] = v4.y; r[4 * e + 2] = v4.z; r[4 * e + 3] = v4.w;
                    }
                } else {
#pragma unroll
                    for (int jb = 0; jb < D; jb += 32) tc::tmem_ld32(tS + jb, r + jb);
                    tc::tmem_wait_ld();
                }
                if (MODE == PASS_C) {
#pragma unroll
                    for (int e = 0; e < D; e += 8) {
                        float f[8];
#pragma unroll
                        for (int x = 0; x < 8; ++x) f[x] = __uint_as_float(r[e + x]);
                        *reinterpret_cast<uint4*>(smem + OFF_SBF + sw_off(c, e, D)) = pack8(f);
                    }
                }
                if (n == 0 || rmw) {
                    const float sc = rmw ? sig : 1.f;
#pragma unroll
                    for (int e = 0; e < D; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * sc);
#pragma unroll
                    for (int jb = 0; jb < D; jb += 32) tc::tmem_st32(tS + jb, r + jb);
                    tc::tmem_wait_st();
                }
            }
            a_seg *= a_n;
            Drow = rmw ? 1.f : sig;
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            tc::fence_before_sync();
            grp_sync(2);
            if (warp == 4) {  // the whole warp issues in lockstep, one lane elected inside each instruction
                tc::fence_after_sync();
                // R += k^'^T V (pass A starts from an empty R: the first MMA overwrites)
                // descriptors built once (all share the high word: SBO 1024, SW128); a K step adds
                // its offset (bytes >> 4) to the low word
                const uint64_t dkh = tc::sdesc_sw128(smem_u32(base + ST_K), BOX_BYTES, 1024);
                const uint32_t kh_lo = tc::desc_lo(dkh), hi = tc::desc_hi(dkh);
                const uint32_t va_lo = tc::desc_lo(tc::sdesc_sw128(smem_u32(base + ST_V), BOX_BYTES, 1024));
#pragma unroll
                for (int k = 0; k < C / 16; ++k)
                    tc::mma_ss_lh_warp(tmem + TM_S, kh_lo + 128u * k, hi, va_lo + 128u * k, hi, idesc_U,
                                       (MODE == PASS_A && n == 0 && k == 0) ? 0u : 1u);
                if (MODE == PASS_C) {  // O = P V + q~' R_bf16
                    const uint32_t pa_lo = tc::desc_lo(tc::sdesc_sw128(smem_u32(base + ST_P), 16, 1024));
                    const uint32_t qa_lo = tc::desc_lo(tc::sdesc_sw128(smem_u32(base + ST_Q), 16, 1024));
                    const uint32_t sb_lo = tc::desc_lo(tc::sdesc_sw128(smem_u32(smem + OFF_SBF), D * 128, 1024));
#pragma unroll
                    for (int k = 0; k < C / 16; ++k)
                        tc::mma_ss_lh_warp(tmem + TM_O, pa_lo + 2u * k, hi, va_lo + 128u * k, hi, idesc_O, k > 0);
#pragma unroll
                    for (int k = 0; k < D / 16; ++k)
                        tc::mma_ss_lh_warp(tmem + TM_O, qa_lo + (uint32_t)(((k / 4) * BOX_BYTES + (k % 4) * 32) >> 4),
                                           hi, sb_lo + 128u * k, hi, idesc_O, 1u);
                }
                tc::mma_commit_warp(barO);
                tc::mma_commit_warp(&empty[st]);
            }
        }

        // ---- tail: last chunk's outputs and the segment's state S = diag(D) R
        if (ok && n_ch > 0 && grp_all(2, wait_bar(barO, (uint32_t)((n_ch - 1) & 1), abort_flag, wlim))) {
            tc::fence_after_sync();
            if (MODE == PASS_C) epilogue(n_ch - 1);
            float* dst = nullptr;
            if (MODE == PASS_C && seg == args.n_seg - 1) dst = args.state_out + ((int64_t)bh * D + c) * D;
            if (MODE == PASS_A) {
                dst = args.u_out + (((int64_t)bh * args.n_seg + seg + 1) * D + c) * D;
                args.a_out[((int64_t)bh * args.n_seg + seg) * D + c] = a_seg;
            }
#pragma unroll
            for (int j = 0; j < D; j += 32) {
                uint32_t r[32];
                tc::tmem_ld32(tS + j, r);
                tc::tmem_wait_ld();
                if (dst) {
#pragma unroll
                    for (int i = 0; i < 32; i += 4)
                        *reinterpret_cast<float4*>(dst + j + i) =
                            make_float4(__uint_as_float(r[i]) * Drow, __uint_as_float(r[i + 1]) * Drow,
                                        __uint_as_float(r[i + 2]) * Drow, __uint_as_float(r[i + 3]) * Drow);
                }
            }
        }
        if (warp == 4) {  // every MMA this warp issued has completed before TMEM is released
            tc::mma_commit_warp(drain1);
            mbar_wait_bounded(drain1, 0, kWaitLimit);
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 8) tc::tmem_dealloc(tmem, 512);
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

// one-shot test arming (rod_test_expire_waits): the next launch runs with this wait limit and
// with its producers issuing no copies, so that every consumer's first wait gives up
std::atomic<uint32_t> g_expire_probes{0};

// Segments per (b, h): one wave of the output pass (one CTA per SM), i.e. floor(SMs / (B H)),
// at least 1. Measured on B200 (recurrence layer, d = 128): at B4 H16 T4096 two segments per
// head take 240 us against 271 us for a single segment (the sequential schedule) and 284 us for
// four waves; at B1 H16 T131072 nine segments take 1330 us against 1374 us for four waves.
// Fewer segments also mean fewer k, v, g bytes read twice (segment pass and output pass).
Plan plan(int B, int H, int T) {
    const int64_t BH = (int64_t)B * H;
    const int chunks = (T + C - 1) / C;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1) {
        cudaGetLastError();
        sms = 148;
    }
    int64_t want = BH > 0 ? sms / BH : 1;
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
    const uint32_t expire = g_expire_probes.exchange(0u);
    a.wait_limit = expire ? expire : kWaitLimit;
    a.copies_off = expire ? 1 : 0;
    a.q = static_cast<const __nv_bfloat16*>(q);
    a.k = static_cast<const __nv_bfloat16*>(k);
    a.v = static_cast<const __nv_bfloat16*>(v);
    a.g = g;
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

void gla_prefill_tc_arm_wait_expiry(uint32_t probes) { g_expire_probes.store(probes); }

unsigned gla_prefill_tc_take_timeout_flag() {
    unsigned v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_gla_tc_timeout, sizeof(v)) != cudaSuccess) return 0;
    cudaMemcpyToSymbol(g_gla_tc_timeout, &zero, sizeof(zero));
    return v;
}

}  // namespace rod
