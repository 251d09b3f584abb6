// gla_prefill_tc.cu -- chunkwise-parallel prefill of the Rodimus gated linear recurrence on the
// 5th-generation tensor cores (tcgen05 / TMEM / TMA), bf16 q, k, v / fp32 gates and state,
// d_k = d_v = 128, chunks of 64 tokens.
//
// Recurrence (CodeFuse Rodimus* article, Rodimus block; SALA blog §2.2 state form, §4.3 decay):
//     S_t = diag(g_t) S_{t-1} + k_t^T v_t,     o_t = q_t S_t.
// Chunk form (the chunkwise-parallel algorithm the Rodimus block paragraph names for training
// and prefill). For a chunk of C tokens with incoming state S_in, per key channel c let
//     G_t = prod_{r<=t} g_r     (prefix product inside the chunk),   a = G_{C-1}.
// Then, exactly,
//     o_t   = sum_{s<=t} (sum_c q_tc k_sc G_tc / G_sc) v_s + (q_t . G_t) S_in
//     S_out = diag(a) S_in + sum_s (k_s . a / G_s)^T v_s.
// The state is held as S = diag(D) R with a running per-channel decay D, so that a chunk adds
// its contribution to R without rescaling R: D <- D a, R += (k . a / (G D))^T V; R is rescaled
// (and D reset to 1) only when some channel's D would fall below 2^-64.
//
// Tensor memory holds R TRANSPOSED (R^T: value channel j in lane j, key channel c in column c).
// The readout then takes R^T itself as the A operand of a tf32 MMA -- the fp32 accumulator is
// read in place, with no copy or rounding of the state to 16 bits -- and every product of a
// chunk produces transposed outputs O^T (value channel in the lane, token in the column):
//     A    = q~ k~^T                  bf16,  M=64  N=64  K=128   q~ = q.G, k~ = k/G (scores)
//     O^T  = R^T (q.G.D)^T            tf32,  M=128 N=64  K=128   A operand: R^T in TMEM
//     O^T += V^T P^T                  bf16,  M=128 N=64  K=64    P = A masked to s <= t
//     R^T += V^T (k.a/(G D'))         bf16,  M=128 N=128 K=64
// k~ = k/G needs G well inside the bf16 range, so a chunk in which some channel's product a
// falls below 2^-60 takes the exact route instead: the scores are summed on the CUDA cores from
// log2-gate prefix sums L (log2 g clamped at -126, so g = 0 contributes below fp32 resolution),
// A_ts = sum_c q_tc k_sc 2^(L_tc - L_sc), and stored straight into tensor memory where the
// tensor cores would have put them; q.G becomes q.2^L and a/G becomes 2^(L_last - L).
//
// Parallelism over the sequence: the T tokens are cut into segments of L_seg tokens. Pass A
// (per segment but the last, each cut into `sub` pieces when that fills more SMs) computes each
// piece's state contribution U and decay a from k, v, g; a scan kernel chains
// S(j+1) = diag(a_j) S(j) + U_j per (b, h) over the pieces; pass C recomputes every segment from
// its S_in and writes o (and the final state). One segment means pass C alone.
//
// CTA: 512 threads = 4 warpgroups, setmaxnreg 56 / 152 / 152 / 152, a pipeline over the chunks
// of a segment through two 96 KB stages:
//   warp 0       TMA producer (q, k, v, g of chunk n into stage n % 2, L2 prefetch of later
//                chunks) and TMEM allocator; warps 2-3 idle (they complete the warpgroup);
//   warp 1       MMA issuer: every tcgen05.mma of the chunk, in the order A, readout, P V,
//                state update, issued by the whole warp with one lane elected per MMA;
//   warps 4-11   operands of chunk n (one channel pair x 16 rows per thread): the gate prefix
//                products, q~ (bf16) over q, k^ over k, k~ beside them, q.G.D (fp32, tf32
//                layout) over the consumed gates; the rescale of R^T when voted;
//   warps 12-15  P = mask(A) of chunk n (into the stage), output rows of chunk n-1 (O^T from
//                TMEM, bf16 rows through shared memory, one TMA store per chunk), initial and
//                final state.
// TMEM: R^T (cols 0-127), O^T two buffers (128-255), A two buffers (256-383, M=64: rows in lanes
// 0-15 of each 32-lane quarter). Every wait is bounded; a timeout stops all roles, drains
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
constexpr int NTHREADS = 512;            // 4 warpgroups: control, operands (2), state
constexpr int kOpThreads = 256;          // warps 4-11
// Register split (setmaxnreg). Each of the SM's four sub-partitions holds one warp of every
// warpgroup, so per sub-partition the launch provides 4 x 128 = 512 registers per lane; the split
// 56 (control) + 2 x 152 (operands) + 152 (state) = 512 uses exactly that.
constexpr int kLaunchRegs = 128;
constexpr int kCtlRegs = 56;
constexpr int kOpRegs = 152;
constexpr int kStRegs = 152;
static_assert(kCtlRegs + 2 * kOpRegs + kStRegs <= 4 * kLaunchRegs, "register split exceeds launch");
static_assert(NTHREADS * kLaunchRegs <= 65536, "launch registers exceed the SM's register file");
constexpr int BOX = C * 128;             // one 64-row box of 128-byte rows = 8 KB
// stage layout (every region 1024-aligned)
constexpr int ST_Q = 0;                  // q, two bf16 boxes       -> q.G in bf16 (scores)
constexpr int ST_K = 2 * BOX;            // k, two bf16 boxes       -> k.a/(G D') (state update)
constexpr int ST_V = 4 * BOX;            // v, two bf16 boxes
constexpr int ST_G = 6 * BOX;            // g, fp32 [64][128]       -> q.G.D, four tf32 boxes (readout)
constexpr int ST_KT = 10 * BOX;          // k/G, two bf16 boxes     -> P, one bf16 box, after the scores
constexpr int STAGE = 12 * BOX;          // 96 KB
constexpr int OFF_OST = 2 * STAGE;                 // 16 KB  output rows, bf16 [64][128] unswizzled
constexpr int OFF_SCAN = OFF_OST + 2 * BOX;        // 2 KB   [4][128] fp32 quarter products / sums
constexpr int OFF_ABUF = OFF_SCAN + 4 * D * 4;     // 3 KB   [2][3][128] fp32: a, D.a, D after
constexpr int OFF_FLAG = OFF_ABUF + 2 * 3 * D * 4; // 16 B   route / rescale flag per stage
constexpr int OFF_BAR = OFF_FLAG + 16;
constexpr int NBAR = 18;
constexpr int OFF_MISC = OFF_BAR + 8 * NBAR;
constexpr int SMEM_BYTES = OFF_MISC + 32 + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
constexpr float kFastMin = 8.673617e-19f;          // 2^-60: chunk decay for q~ k~^T
constexpr float kRescaleMin = 5.421011e-20f;       // 2^-64: smallest running decay D
constexpr int kFlagExact = 1, kFlagRescale = 2;
constexpr float kLog2Floor = -126.0f;              // log2 of the smallest gate used
constexpr int kPrefetchChunks = 1;                 // L2 prefetch distance in chunks (measured best of 0-4)

// TMEM columns
constexpr uint32_t TM_R = 0, TM_O = 128, TM_A = 256;

enum Mode { PASS_A = 0, PASS_C = 1 };

struct GlaArgs {
    const float* s_in;      // PASS_C: [BH][s_in_slots][D][D] incoming states (slot = segment)
    int s_in_slots;         // 1: every (b,h) reads slot 0 of s_in (initial state, single segment)
    float* state_out;       // PASS_C: [BH][D][D] final state, written by the last segment
    float* u_out;           // PASS_A: [BH][n_slots][D][D] (sub-segment j writes slot j+1)
    float* a_out;           // PASS_A: [BH][n_slots][D]    (sub-segment j writes slot j)
    const __nv_bfloat16 *q, *k, *v;  // the inputs again, for L2 prefetches ahead of TMA
    const float* g;
    int T, L_seg, n_seg;    // tokens per CTA (a pass A CTA covers a sub-segment); CTAs per (b,h)
    int n_slots;            // workspace slots per (b,h): sub-segments of pass A + 1
    int sub;                // pass C: segment m starts at sub-segment boundary m * sub
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
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint32_t pack2(uint64_t x) {  // fp32 pair -> bf16 pair (RNE)
    const float2 f = upk2(x);
    return pack_bf16x2(f.x, f.y);
}
__device__ __forceinline__ uint64_t unpack2(uint32_t w) {  // bf16 pair -> fp32 pair (exact)
    return pk2(bf16lo(w), bf16hi(w));
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

// named barriers: id 1 = the operand warps (256 threads), id 2 = the state warps (128 threads);
// no other thread ever joins them
constexpr int kBarOp = 1, kBarSt = 2;
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

__device__ __forceinline__ uint4 pack8(const float* f) {
    uint4 u;
    u.x = pack_bf16x2(f[0], f[1]); u.y = pack_bf16x2(f[2], f[3]);
    u.z = pack_bf16x2(f[4], f[5]); u.w = pack_bf16x2(f[6], f[7]);
    return u;
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
template <typename T> __device__ __forceinline__ T& at(unsigned char* base, uint32_t off) {
    return *reinterpret_cast<T*>(base + off);
}

template <int MODE>
__global__ void __launch_bounds__(NTHREADS, 1)
gla_chunk_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                 const __grid_constant__ CUtensorMap tm_o, GlaArgs args) {
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
    constexpr uint32_t kStageTx = (MODE == PASS_C ? 6 : 4) * BOX + 4 * BOX;

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
    uint64_t* full = bars;          // [2] TMA -> operand warps
    uint64_t* empty = bars + 2;     // [2] chunk MMAs done -> producer
    uint64_t* ops = bars + 4;       // [2] operands ready (8 warps) -> issuer
    uint64_t* aready = bars + 6;    // [2] scores in TMEM -> state warps
    uint64_t* pready = bars + 8;    // [2] P in the stage (4 warps) -> issuer
    uint64_t* barO = bars + 10;     // [2] all MMAs of the chunk done -> state warps, operand warps
    uint64_t* barRO = bars + 12;    // readout and P V of a rescale chunk done -> operand warps
    uint64_t* rdone = bars + 13;    // R^T rescaled (8 warps) -> issuer
    uint64_t* rinit = bars + 14;    // R^T loaded with S_in (4 warps) -> issuer
    uint64_t* fin = bars + 15;      // every MMA of the segment done -> state warps
    uint64_t* drain = bars + 16;
    float* abuf = reinterpret_cast<float*>(smem + OFF_ABUF);
    volatile int* flag = reinterpret_cast<volatile int*>(smem + OFF_FLAG);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);

    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&ops[s], 8);
            mbar_init(&aready[s], 1);
            mbar_init(&pready[s], 4);
            mbar_init(&barO[s], 1);
        }
        mbar_init(barRO, 1);
        mbar_init(rdone, 8);
        mbar_init(rinit, 4);
        mbar_init(fin, 1);
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
    const uint32_t wlim = args.wait_limit;

    if (warp < 4) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kCtlRegs));
        if (warp == 0 && lane == 0) {
            // ------------------------------- TMA producer -------------------------------
            int n = 0;
            for (; n < n_ch && !args.copies_off; ++n) {
                const int st = n & 1, use = n >> 1;
                if (use > 0 && !wait_bar(&empty[st], (uint32_t)((use - 1) & 1), abort_flag, wlim)) break;
                unsigned char* base = smem + st * STAGE;
                const int y = t_begin + n * C;
                mbar_arrive_expect_tx(&full[st], kStageTx);
                for (int half = 0; half < 2; ++half) {
                    if (MODE == PASS_C)
                        tc::tma_load_3d(base + ST_Q + half * BOX, &tm_q, half * 64, y, bh, &full[st]);
                    tc::tma_load_3d(base + ST_K + half * BOX, &tm_k, half * 64, y, bh, &full[st]);
                    tc::tma_load_3d(base + ST_V + half * BOX, &tm_v, half * 64, y, bh, &full[st]);
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
        } else if (warp == 1) {
            // -------------------------------- MMA issuer --------------------------------
            // the whole warp runs in lockstep; one lane, elected inside each instruction, issues
            const uint32_t idesc_A = tc::idesc_bf16_f32(64, 64, 0, 0);
            const uint32_t idesc_RO = tc::idesc_tf32_f32(128, 64, 0, 0);
            const uint32_t idesc_PV = tc::idesc_bf16_f32(128, 64, 1, 0);
            const uint32_t idesc_U = tc::idesc_bf16_f32(128, 128, 1, 1);
            auto wait_all = [&](uint64_t* bar, uint32_t par) {
                return __all_sync(0xffffffffu, wait_bar(bar, par, abort_flag, wlim)) != 0;
            };
            bool ok = MODE == PASS_A || wait_all(rinit, 0);
            uint32_t nresc = 0;
            for (int n = 0; ok && n < n_ch; ++n) {
                const int st = n & 1;
                const uint32_t ph = (uint32_t)((n >> 1) & 1);
                unsigned char* base = smem + st * STAGE;
                if (!wait_all(&ops[st], ph)) { ok = false; break; }
                tc::fence_after_sync();
                const int fl = flag[st];
                // descriptors built once per stage (all share the high word: SBO 1024, SW128);
                // a K step adds its offset (bytes >> 4) to the low word
                const uint32_t hi = tc::desc_hi(tc::sdesc_sw128(smem_u32(base), 16, 1024));
                const uint32_t v_lo = tc::desc_lo(tc::sdesc_sw128(smem_u32(base + ST_V), BOX, 1024));
                const uint32_t kh_lo = tc::desc_lo(tc::sdesc_sw128(smem_u32(base + ST_K), BOX, 1024));
                if (MODE == PASS_C) {
                    if (!(fl & kFlagExact)) {  // A = q~ k~^T
                        const uint32_t qa_lo = tc::desc_lo(tc::sdesc_sw128(smem_u32(base + ST_Q), 16, 1024));
                        const uint32_t kt_lo = tc::desc_lo(tc::sdesc_sw128(smem_u32(base + ST_KT), 16, 1024));
#pragma unroll
                        for (int k = 0; k < D / 16; ++k) {
                            const uint32_t koff = (uint32_t)(((k / 4) * BOX + (k % 4) * 32) >> 4);
                            tc::mma_ss_lh_warp(tmem + TM_A + 64u * st, qa_lo + koff, hi, kt_lo + koff, hi,
                                               idesc_A, k > 0);
                        }
                        tc::mma_commit_warp(&aready[st]);
                    } else {  // the operand warps stored the exact scores in TMEM
                        tc::fence_before_sync();
                        if (lane == 0) mbar_arrive(&aready[st]);
                    }
                    if (!wait_all(&pready[st], ph)) { ok = false; break; }
                    tc::fence_after_sync();
                    // O^T = R^T (q.G.D)^T: tf32, A = R^T straight from TMEM (K step of 8 columns)
                    const uint32_t qf_lo = tc::desc_lo(tc::sdesc_sw128(smem_u32(base + ST_G), 16, 1024));
#pragma unroll
                    for (int j = 0; j < D / 8; ++j) {
                        const uint32_t koff = (uint32_t)(((j / 4) * BOX + (j % 4) * 32) >> 4);
                        tc::mma_tf32_ts_lh_warp(tmem + TM_O + 64u * st, tmem + TM_R + 8u * j, qf_lo + koff, hi,
                                                idesc_RO, j > 0);
                    }
                    // O^T += V^T P^T
                    const uint32_t p_lo = tc::desc_lo(tc::sdesc_sw128(smem_u32(base + ST_KT), 16, 1024));
#pragma unroll
                    for (int k = 0; k < C / 16; ++k)
                        tc::mma_ss_lh_warp(tmem + TM_O + 64u * st, v_lo + 128u * k, hi, p_lo + 2u * k, hi,
                                           idesc_PV, 1u);
                    if (fl & kFlagRescale) {  // the operand warps rescale R^T after the readout
                        tc::mma_commit_warp(barRO);
                        if (!wait_all(rdone, nresc & 1u)) { ok = false; break; }
                        ++nresc;
                        tc::fence_after_sync();
                    }
                }
                // R^T += V^T k^ (pass A starts from an empty R: the first MMA overwrites)
#pragma unroll
                for (int k = 0; k < C / 16; ++k)
                    tc::mma_ss_lh_warp(tmem + TM_R, v_lo + 128u * k, hi, kh_lo + 128u * k, hi, idesc_U,
                                       (MODE == PASS_A && n == 0 && k == 0) ? 0u : 1u);
                tc::mma_commit_warp(&barO[st]);
                tc::mma_commit_warp(&empty[st]);
                if (n == n_ch - 1) tc::mma_commit_warp(fin);
            }
            // every MMA this warp issued has completed before TMEM is released
            tc::mma_commit_warp(drain);
            mbar_wait_bounded(drain, 0, kWaitLimit);
        }
    } else if (warp < 12) {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kOpRegs));
        // ------------------------------ operand warps ------------------------------
        // thread = (channel pair p: channels 2p, 2p+1; row quarter qr: rows 16qr .. 16qr+15)
        const int ot = tid - 128;
        const int p = ot & 63, qr = ot >> 6;
        const int c0 = 2 * p, r0 = 16 * qr;
        const int wq = warp & 3;                       // TMEM lane quarter of this warp
        const int half = (warp - 4) >> 2;              // 0: warps 4-7, 1: warps 8-11
        const uint32_t lane_base = (uint32_t)(32 * wq) << 16;
        // byte offsets of my channel pair inside a row: bf16 tiles (two 64-column boxes) and the
        // fp32 tf32 tile (four 32-column boxes), both 128-byte swizzled
        const uint32_t b16_base = (uint32_t)((p >> 5) * BOX + ((p & 3) * 4));
        const uint32_t b16_chunk = (uint32_t)((p & 31) >> 2);
        const uint32_t f32_base = (uint32_t)((p >> 4) * BOX + ((p & 1) * 8));
        const uint32_t f32_chunk = (uint32_t)((p & 15) >> 1);
        auto off16 = [&](int t) { return b16_base + (uint32_t)t * 128u + (((b16_chunk ^ (uint32_t)(t & 7))) << 4); };
        auto off32 = [&](int t) { return f32_base + (uint32_t)t * 128u + (((f32_chunk ^ (uint32_t)(t & 7))) << 4); };
        float* scan = reinterpret_cast<float*>(smem + OFF_SCAN);
        uint64_t Dc = pk2(1.f, 1.f);     // running decay of my two channels
        uint64_t aseg = pk2(1.f, 1.f);   // pass A: decay over the segment
        uint32_t nresc = 0;
        bool ok = true;

        // R^T column c scaled by sig[c] (this warpgroup's 64 columns, this warp's 32 lanes)
        auto rescale_state = [&](const float* sig) {
#pragma unroll
            for (int cb = 0; cb < 2; ++cb) {
                const uint32_t col = (uint32_t)(64 * half + 32 * cb);
                uint32_t r[32];
                tc::tmem_ld32(tmem + TM_R + lane_base + col, r);
                tc::tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * sig[col + i]);
                tc::tmem_st32(tmem + TM_R + lane_base + col, r);
            }
            tc::tmem_wait_st();
            tc::fence_before_sync();
        };

        for (int n = 0; n < n_ch; ++n) {
            const int st = n & 1;
            unsigned char* base = smem + st * STAGE;
            const int nvalid = min(C, t_end - (t_begin + n * C));
            if (!bar_all(kBarOp, kOpThreads, wait_bar(&full[st], (uint32_t)((n >> 1) & 1), abort_flag, wlim))) {
                ok = false;
                break;
            }
            // sweep 1: my 16 gate pairs (rows past the sequence end count as g = 1) and their product
            uint64_t g2[16];
            uint64_t prod = pk2(1.f, 1.f);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int t = r0 + i;
                g2[i] = t < nvalid ? at<uint64_t>(base, ST_G + (uint32_t)(t * 512 + p * 8)) : pk2(1.f, 1.f);
                prod = mul2(prod, g2[i]);
            }
            *reinterpret_cast<uint64_t*>(scan + qr * D + c0) = prod;
            bar_sync(kBarOp, kOpThreads);
            uint64_t pre = pk2(1.f, 1.f), a = pk2(1.f, 1.f);
#pragma unroll
            for (int q2 = 0; q2 < 4; ++q2) {
                const uint64_t v = *reinterpret_cast<const uint64_t*>(scan + q2 * D + c0);
                if (q2 < qr) pre = mul2(pre, v);
                a = mul2(a, v);
            }
            float2 af = upk2(a);
            // route vote (also a barrier: every quarter product has been read past here)
            const bool fast = bar_all(kBarOp, kOpThreads, af.x >= kFastMin && af.y >= kFastMin);
            uint64_t preL = pk2(0.f, 0.f), Ltot = pk2(0.f, 0.f);
            if (!fast) {
                // exact route: L = prefix sums of clamped log2 gates (kept in g2 as log pairs)
                uint64_t lsum = pk2(0.f, 0.f);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float2 gg = upk2(g2[i]);
                    g2[i] = r0 + i < nvalid ? pk2(fmaxf(lg2(gg.x), kLog2Floor), fmaxf(lg2(gg.y), kLog2Floor))
                                            : pk2(0.f, 0.f);
                    lsum = add2(lsum, g2[i]);
                }
                *reinterpret_cast<uint64_t*>(scan + qr * D + c0) = lsum;
                bar_sync(kBarOp, kOpThreads);
#pragma unroll
                for (int q2 = 0; q2 < 4; ++q2) {
                    const uint64_t v = *reinterpret_cast<const uint64_t*>(scan + q2 * D + c0);
                    if (q2 < qr) preL = add2(preL, v);
                    Ltot = add2(Ltot, v);
                }
                const float2 lt = upk2(Ltot);
                a = pk2(tc::ex2(lt.x), tc::ex2(lt.y));
                af = upk2(a);
                if (MODE == PASS_C) {
                    // L over my gates, then the exact scores of row t into TMEM A[st]
                    uint64_t L = preL;
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        L = add2(L, g2[i]);
                        at<uint64_t>(base, ST_G + (uint32_t)((r0 + i) * 512 + p * 8)) = L;
                    }
                    bar_sync(kBarOp, kOpThreads);
                    const int t = 16 * wq + lane;  // row (lanes 0-15 of the quarter)
                    const float* Lg = reinterpret_cast<const float*>(base + ST_G);
                    float acc[32];
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) acc[jj] = 0.f;
                    if (lane < 16) {
                        for (int cc = 0; cc < D; ++cc) {
                            const float qc = ldbf(base + ST_Q + sw_off_elem(t, cc, C));
                            const float Lt = Lg[t * D + cc];
#pragma unroll
                            for (int jj = 0; jj < 32; ++jj) {
                                const int s = 32 * half + jj;
                                if (s <= t)
                                    acc[jj] = fmaf(qc * ldbf(base + ST_K + sw_off_elem(s, cc, C)),
                                                   tc::ex2(Lt - Lg[s * D + cc]), acc[jj]);
                            }
                        }
                    }
                    uint32_t ar[32];
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) ar[jj] = __float_as_uint(acc[jj]);
                    tc::tmem_st32(tmem + TM_A + 64u * st + 32u * half + lane_base, ar);
                    tc::tmem_wait_st();
                    bar_sync(kBarOp, kOpThreads);  // q, k and L read by every thread before overwrites
                }
            }
            // rescale vote: a channel whose running decay would fall below 2^-64 resets D for all
            const float2 dcf = upk2(Dc);
            const bool rmw = !bar_all(kBarOp, kOpThreads,
                                      dcf.x * af.x >= kRescaleMin && dcf.y * af.y >= kRescaleMin);
            const uint64_t dn = rmw ? pk2(1.f, 1.f) : mul2(Dc, a);   // D after this chunk
            const float2 dnf = upk2(dn);
            const uint64_t adn = mul2(a, pk2(rcp(dnf.x), rcp(dnf.y)));  // a / D'
            if (fast) {
                // sweep 2: q~ = q.G (bf16) over q, q.G.D (fp32) over the gates, k~ = k/G beside,
                // k^ = k~ . a / D' over k
                uint64_t G = pre;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int t = r0 + i;
                    G = mul2(G, g2[i]);
                    const float2 gf = upk2(G);
                    const uint64_t kt = mul2(unpack2(at<uint32_t>(base, ST_K + off16(t))), pk2(rcp(gf.x), rcp(gf.y)));
                    at<uint32_t>(base, ST_K + off16(t)) = pack2(mul2(kt, adn));
                    if (MODE == PASS_C) {
                        const uint64_t qg = mul2(unpack2(at<uint32_t>(base, ST_Q + off16(t))), G);
                        at<uint32_t>(base, ST_Q + off16(t)) = pack2(qg);
                        at<uint64_t>(base, ST_G + off32(t)) = mul2(qg, Dc);
                        at<uint32_t>(base, ST_KT + off16(t)) = pack2(kt);
                    }
                }
            } else {
                // exact route: q.2^L.D (fp32) over the gates, k^ = k.2^(Ltot - L) / D' over k
                const float2 ltf = upk2(Ltot);
                const float2 rdn = make_float2(rcp(dnf.x), rcp(dnf.y));
                uint64_t L = preL;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int t = r0 + i;
                    L = add2(L, g2[i]);
                    const float2 lf = upk2(L);
                    const float2 kf = upk2(unpack2(at<uint32_t>(base, ST_K + off16(t))));
                    at<uint32_t>(base, ST_K + off16(t)) =
                        pack_bf16x2(kf.x * tc::ex2(ltf.x - lf.x) * rdn.x, kf.y * tc::ex2(ltf.y - lf.y) * rdn.y);
                    if (MODE == PASS_C) {
                        const float2 qf = upk2(unpack2(at<uint32_t>(base, ST_Q + off16(t))));
                        at<uint64_t>(base, ST_G + off32(t)) =
                            pk2(qf.x * (tc::ex2(lf.x) * dcf.x), qf.y * (tc::ex2(lf.y) * dcf.y));
                    }
                }
            }
            // publish a, the rescale factor D.a and the new D; the route and rescale flags
            if (qr == 0) {
                float* ab = abuf + st * 3 * D + c0;
                *reinterpret_cast<uint64_t*>(ab) = a;
                *reinterpret_cast<uint64_t*>(ab + D) = mul2(Dc, a);
                *reinterpret_cast<uint64_t*>(ab + 2 * D) = dn;
            }
            if (ot == 0) flag[st] = (fast ? 0 : kFlagExact) | (rmw ? kFlagRescale : 0);
            if (MODE == PASS_A) aseg = mul2(aseg, a);
            Dc = dn;
            tc::fence_proxy_async();  // operands written by these threads -> the tensor cores
            const float* sig = abuf + st * 3 * D + D;
            if (MODE == PASS_A) {
                // R^T rescaled before this chunk's update, once the previous chunk's MMAs are done
                if (rmw && n > 0) {
                    if (!bar_all(kBarOp, kOpThreads,
                                 wait_bar(&barO[(n - 1) & 1], (uint32_t)(((n - 1) >> 1) & 1), abort_flag, wlim))) {
                        ok = false;
                        break;
                    }
                    tc::fence_after_sync();
                    rescale_state(sig);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&ops[st]);
            } else {
                tc::fence_before_sync();  // exact-route scores stored to TMEM
                __syncwarp();
                if (lane == 0) mbar_arrive(&ops[st]);
                if (rmw) {  // after this chunk's readout (it reads R^T with the old D)
                    if (!bar_all(kBarOp, kOpThreads, wait_bar(barRO, nresc & 1u, abort_flag, wlim))) {
                        ok = false;
                        break;
                    }
                    ++nresc;
                    tc::fence_after_sync();
                    rescale_state(sig);
                    __syncwarp();
                    if (lane == 0) mbar_arrive(rdone);
                }
            }
        }
        if (MODE == PASS_A && ok && qr == 0)
            *reinterpret_cast<uint64_t*>(args.a_out + ((int64_t)bh * args.n_slots + seg) * D + c0) = aseg;
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kStRegs));
        // ------------------- state warps: P, output rows, initial / final state -------------------
        const int wq = warp - 12;                          // TMEM lane quarter
        const int stid = tid - 384;
        const uint32_t lane_base = (uint32_t)(32 * wq) << 16;
        const int j = 32 * wq + lane;                      // value channel == TMEM lane (R^T, O^T)
        bool ok = true;
        auto all2 = [&](bool x) { return bar_all(kBarSt, 128, x); };

        // state S = diag(D) R out to dst[c][j] (D after the last chunk)
        auto store_state = [&](float* dst, const float* dfin) {
#pragma unroll
            for (int cb = 0; cb < D; cb += 32) {
                uint32_t r[32];
                tc::tmem_ld32(tmem + TM_R + lane_base + cb, r);
                tc::tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) dst[(size_t)(cb + i) * D + j] = __uint_as_float(r[i]) * dfin[cb + i];
            }
        };

        if (MODE == PASS_C) {
            __nv_bfloat16* ost = reinterpret_cast<__nv_bfloat16*>(smem + OFF_OST);
            // O^T of chunk m -> bf16 rows in shared memory -> one TMA store
            auto epilogue = [&](int m) -> bool {
                const int mst = m & 1;
                if (!all2(wait_bar(&barO[mst], (uint32_t)((m >> 1) & 1), abort_flag, wlim))) return false;
                tc::fence_after_sync();
                uint32_t r[64];
                tc::tmem_ld32(tmem + TM_O + 64u * mst + lane_base, r);
                tc::tmem_ld32(tmem + TM_O + 64u * mst + lane_base + 32, r + 32);
                tc::tmem_wait_ld();
                tc::fence_before_sync();
                if (stid == 0) tc::bulk_wait_read();  // the previous store has read the rows
                bar_sync(kBarSt, 128);
#pragma unroll
                for (int t = 0; t < C; ++t) ost[t * D + j] = __float2bfloat16_rn(__uint_as_float(r[t]));
                tc::fence_proxy_async();
                bar_sync(kBarSt, 128);
                if (stid == 0) {
                    tc::tma_store_3d(&tm_o, ost, 0, t_begin + m * C, bh);
                    tc::bulk_commit();
                }
                return true;
            };

            // R^T <- S_in^T with D = 1
            {
                const int slot = args.s_in_slots == 1 ? 0 : seg * args.sub;
                const float* src = args.s_in + ((int64_t)bh * args.s_in_slots + slot) * D * D;
#pragma unroll
                for (int cb = 0; cb < D; cb += 32) {
                    uint32_t r[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(src[(size_t)(cb + i) * D + j]);
                    tc::tmem_st32(tmem + TM_R + lane_base + cb, r);
                }
                tc::tmem_wait_st();
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(rinit);
            }
            for (int n = 0; n < n_ch; ++n) {
                const int st = n & 1;
                unsigned char* base = smem + st * STAGE;
                if (!all2(wait_bar(&aready[st], (uint32_t)((n >> 1) & 1), abort_flag, wlim))) { ok = false; break; }
                tc::fence_after_sync();
                // P = mask(A) in bf16 into the stage (row t = 16 wq + lane, lanes 0-15)
                uint32_t r[64];
                tc::tmem_ld32(tmem + TM_A + 64u * st + lane_base, r);
                tc::tmem_ld32(tmem + TM_A + 64u * st + lane_base + 32, r + 32);
                tc::tmem_wait_ld();
                if (lane < 16) {
                    const int t = 16 * wq + lane;
#pragma unroll
                    for (int s = 0; s < C; s += 8) {
                        float f[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) f[i] = s + i <= t ? __uint_as_float(r[s + i]) : 0.f;
                        *reinterpret_cast<uint4*>(base + ST_KT + sw_off(t, s, C)) = pack8(f);
                    }
                }
                tc::fence_proxy_async();
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&pready[st]);
                if (n > 0 && !epilogue(n - 1)) { ok = false; break; }
            }
            if (ok && epilogue(n_ch - 1) && seg == args.n_seg - 1)
                store_state(args.state_out + (int64_t)bh * D * D, abuf + ((n_ch - 1) & 1) * 3 * D + 2 * D);
            if (stid == 0) tc::bulk_wait_all();
        } else {
            if (all2(wait_bar(fin, 0, abort_flag, wlim))) {
                tc::fence_after_sync();
                store_state(args.u_out + ((int64_t)bh * args.n_slots + seg + 1) * D * D,
                            abuf + ((n_ch - 1) & 1) * 3 * D + 2 * D);
            }
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 0) tc::tmem_dealloc(tmem, 512);
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
    int L_seg, n_seg;   // output pass: segments of L_seg tokens, n_seg per (b, h)
    int sub;            // segment pass: each of the first n_seg - 1 segments in `sub` pieces
    int slots() const { return n_seg > 1 ? (n_seg - 1) * sub + 1 : 0; }
};

// one-shot test arming (rod_test_expire_waits): the next launch runs with this wait limit and
// with its producers issuing no copies, so that every consumer's first wait gives up
std::atomic<uint32_t> g_expire_probes{0};

// Segments per (b, h): one wave of the output pass (one CTA per SM), i.e. floor(SMs / (B H)),
// at least 1. Fewer segments mean fewer k, v, g bytes read twice (segment pass and output pass);
// more than one wave adds segment-pass traffic and a tail. The segment pass has one segment
// fewer per (b, h), so with few segments it would leave SMs idle (B4 H16: 64 CTAs): there each
// segment is split into `sub` equal pieces of whole chunks, as many as still fit one wave, and
// the scan chains the pieces.
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
    p.sub = 1;
    if (p.n_seg > 1) {
        for (int k = per; k > 1; --k)  // the largest divisor of the segment's chunk count that fits
            if (per % k == 0 && BH * (p.n_seg - 1) * k <= sms) { p.sub = k; break; }
    }
    return p;
}

}  // namespace

bool gla_prefill_tc_supported(int dk, int dv, int chunk) { return dk == D && dv == D && chunk == C; }

size_t gla_prefill_tc_workspace_size(int B, int H, int T) {
    const Plan p = plan(B, H, T);
    if (p.n_seg <= 1) return 0;
    return (size_t)B * H * p.slots() * ((size_t)D * D + D) * sizeof(float);
}

cudaError_t gla_prefill_tc_launch(const void* q, const void* k, const void* v, const float* g,
                                  float* state, void* o, int B, int H, int T, void* workspace,
                                  cudaStream_t stream) {
    const Plan p = plan(B, H, T);
    const int64_t BH = (int64_t)B * H;
    if (BH > 65535) return cudaErrorInvalidConfiguration;
    CUtensorMap mq, mk, mv, mg, mo;
    cudaError_t e;
    if ((e = make_tmap_3d(&mq, q, false, D, (uint64_t)T, (uint64_t)BH, 64, C, true)) != cudaSuccess) return e;
    if ((e = make_tmap_3d(&mk, k, false, D, (uint64_t)T, (uint64_t)BH, 64, C, true)) != cudaSuccess) return e;
    if ((e = make_tmap_3d(&mv, v, false, D, (uint64_t)T, (uint64_t)BH, 64, C, true)) != cudaSuccess) return e;
    if ((e = make_tmap_3d(&mg, g, true, D, (uint64_t)T, (uint64_t)BH, D, C, false)) != cudaSuccess) return e;
    if ((e = make_tmap_3d(&mo, o, false, D, (uint64_t)T, (uint64_t)BH, D, C, false)) != cudaSuccess) return e;
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
    a.n_seg = p.n_seg;
    a.sub = p.sub;
    a.n_slots = p.slots();
    a.state_out = state;
    if (p.n_seg == 1) {
        a.s_in = state;
        a.s_in_slots = 1;
    } else {
        float* slots = static_cast<float*>(workspace);
        float* aseg = slots + (size_t)BH * a.n_slots * D * D;
        a.u_out = slots;
        a.a_out = aseg;
        const int n_sub = (p.n_seg - 1) * p.sub;
        a.L_seg = p.L_seg / p.sub;  // a segment-pass CTA covers one piece
        gla_chunk_kernel<PASS_A><<<dim3((unsigned)n_sub, (unsigned)BH), NTHREADS, SMEM_BYTES, stream>>>(
            mq, mk, mv, mg, mo, a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        gla_segment_scan_kernel<<<dim3((D * D / 4 + 255) / 256, (unsigned)BH), 256, 0, stream>>>(
            state, slots, aseg, a.n_slots);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        note_launches(2);
        a.s_in = slots;
        a.s_in_slots = a.n_slots;
    }
    a.L_seg = p.L_seg;
    gla_chunk_kernel<PASS_C><<<dim3((unsigned)p.n_seg, (unsigned)BH), NTHREADS, SMEM_BYTES, stream>>>(
        mq, mk, mv, mg, mo, a);
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
