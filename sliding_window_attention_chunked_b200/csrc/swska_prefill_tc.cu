// swska_prefill_tc.cu -- SW-SKA prefill on the 5th-generation tensor cores (tcgen05, TMEM,
// TMA), bf16 in / fp32 accumulate, head dim 128.
//
//   o[b,h,t] = sum_{j=max(0,t-W+1)}^{t} softmax_j(scale * q[b,h,t] . k[b,j]) v[b,h,j]
// (CodeFuse Rodimus* article, Fig. 4 / SKA paragraph: one key matrix shared by all heads,
// per-head values; setup blog §3: the window holds the most recent W tokens; SALA blog §2.1
// and §3.2: block-wise windowed attention, each query block visiting only the key blocks of its
// window -- here with a per-element causal/window mask on the two edge blocks.)
//
// A work item is a 128-query tile for a PAIR of heads of one sequence (with an odd head count
// the last pair computes its single head twice and stores it once). The kernel is persistent:
// one CTA per SM takes items in turn, so the next item's Q load and first score MMAs overlap
// the current item's last tile and output rows. Each shared key tile
// is brought into shared memory once by TMA and feeds both heads' score MMAs (the pair's
// remaining reuse of K across the other heads goes through L2). Warp roles (384 threads):
//   warps 0-3   softmax warpgroup of head 0 (thread i owns query row i = TMEM lane i)
//   warps 4-7   softmax warpgroup of head 1
//   warp  8     TMA producer: per item Q, then K_j, V0_j, V1_j into a ring of 32 KB slots
//   warp  9     TMEM allocator and MMA issuer
//   warps 10-11 idle (they complete the third warpgroup, which gives its registers away)
// TMEM (512 columns): S0 | O0 | S1 | O1, 128 columns each. S_h = Q_h K_j^T is read by the
// softmax warps, which write P_h (bf16, packed two per column) over the first 64 columns of
// S_h; O_h += P_h V_h,j then reads P_h straight from TMEM (A operand in TMEM). The issue order
//   S0(0) S1(0) | PV0(j) S0(j+1) PV1(j) S1(j+1) | ...
// lets each head's softmax run while the tensor core works on the other head, and each P_h is
// handed over in two halves of 64 keys, so the first half's P V runs while the softmax forms
// the second. The issuing warp runs in lockstep with one elected lane issuing. Softmax is in
// base 2 on scores pre-scaled by scale*log2(e), with lazy rescaling: the running maximum used
// for the exponent only moves when a row's maximum grows by more than 8 (so P <= 256), and
// then the O row is rescaled in TMEM by its owning thread. The row maximum runs as eight
// independent chains of three-input maxima, and the exponent arguments and the row sum use the
// two-wide fp32 instructions (fma.rn.f32x2 / add.rn.f32x2). Every wait is bounded; a timeout
// makes all roles stop, drain their in-flight copies and MMAs, and raise a flag.
#include <cuda.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace rod {
namespace {

__device__ unsigned int g_swska_tc_timeout = 0;

constexpr int BM = 128;                    // queries per tile
constexpr int BN = 128;                    // keys per tile
constexpr int HD = 128;                    // head dim (dk = dv)
constexpr int NSLOT = 4;                   // ring slots
constexpr int TILE_BYTES = BM * HD * 2;    // 32 KB: one 128 x 128 bf16 tile
constexpr int HALF_BYTES = TILE_BYTES / 2; // one 128-row x 64-column TMA box
constexpr int NTHREADS = 384;               // 3 warpgroups
// Register split (setmaxnreg). The register file is divided among the SM's four sub-partitions
// and each holds one warp of every warpgroup here, so per sub-partition the launch provides
// 3 x 168 = 504 registers per lane; the split below uses 216 + 216 + 72 = 504 exactly.
constexpr int kLaunchRegs = 168;
constexpr int kSoftmaxRegs = 216;
constexpr int kControlRegs = 72;
static_assert(2 * kSoftmaxRegs + kControlRegs <= 3 * kLaunchRegs, "register split exceeds launch");
constexpr float kRescaleThreshold = 8.0f;  // log2 units

constexpr int OFF_Q = 0;
constexpr int OFF_RING = 2 * TILE_BYTES;
constexpr int OFF_BAR = OFF_RING + NSLOT * TILE_BYTES;
constexpr int NBAR = 2 * NSLOT + 11;       // full, empty, qfull, qempty, sfull[2], pfull[2], phalf[2], odone[2], drain
constexpr int OFF_MISC = OFF_BAR + 8 * NBAR;
constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + slack for 1024-byte alignment

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 0) {
            if (*abort_flag) return false;
            if (i >= kWaitLimit) {
                *abort_flag = 1;
                atomicExch(&g_swska_tc_timeout, 1u);
                return false;
            }
        }
    }
}

// warp-wide form: every lane of the warp probes together and all leave with the same result
__device__ __forceinline__ bool wait_bar_warp(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    for (uint32_t i = 1;; ++i) {
        if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
        if ((i & 255u) == 0) {
            if (__any_sync(0xffffffffu, *abort_flag != 0)) return false;
            if (i >= kWaitLimit) {
                *abort_flag = 1;
                atomicExch(&g_swska_tc_timeout, 1u);
                return false;
            }
        }
    }
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}
// two-wide fp32 fma / add (one instruction for both lanes of the pair)
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mov.b64 rc, {%6, %7};\n\tfma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// One work item: a 128-query tile of a head pair of one sequence, with the key tiles it visits.
// Two numberings, both with full-window tiles first and short ones last:
//  - qt_slow: all (head pair, sequence) items of a query tile together. With the rounds dealt
//    out boustrophedon (CTA c takes item c of even rounds and G-1-c of odd ones) the CTAs' loads
//    come out within a few percent of each other even over a few rounds, and while HP x B is
//    small every head pair still has several neighbouring query tiles in flight, sharing K and
//    V tiles in L2;
//  - otherwise the query tile fastest, dealt out in plain stride: neighbouring query tiles of
//    a head pair run side by side whatever HP x B is, and over many rounds the loads even out.
struct Item {
    int t0, kt_lo, n_it, hp, b;
};
__device__ __forceinline__ Item item_at(int i, int n_qtiles, int HP, int NHB, int W, bool qt_slow) {
    Item it;
    int qt, rest;
    if (qt_slow) {
        qt = n_qtiles - 1 - i / NHB;
        rest = i % NHB;
    } else {
        qt = n_qtiles - 1 - i % n_qtiles;
        rest = i / n_qtiles;
    }
    it.hp = rest % HP;
    it.b = rest / HP;
    it.t0 = qt * BM;
    it.kt_lo = (it.t0 - W + 1 > 0 ? it.t0 - W + 1 : 0) / BN;
    it.n_it = it.t0 / BN - it.kt_lo + 1;
    return it;
}
// the k-th item of this CTA (round k of gridDim.x items), or -1 past the last
__device__ __forceinline__ int cta_item(int k, int n_items, bool snake) {
    const int G = (int)gridDim.x, base = k * G;
    if (base >= n_items) return -1;
    const int i = base + ((snake && (k & 1)) ? G - 1 - (int)blockIdx.x : (int)blockIdx.x);
    return i < n_items ? i : -1;
}

// STATS: the statistics mode (each row's log-sum-exp times lse_mul, D = dO . o when dO is given,
// output optional); a separate instantiation so the plain forward carries none of its registers
template <bool STATS, bool QT_SLOW>
__global__ void __launch_bounds__(NTHREADS, 1)
swska_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, __nv_bfloat16* __restrict__ o, int T,
                int H, int W, float scale_log2, int n_qtiles, int n_items,
                const __nv_bfloat16* __restrict__ dO,
                float* __restrict__ lse, float* __restrict__ dbuf, int Tpad, float lse_mul) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int HP = (H + 1) / 2, NHB = n_items / n_qtiles;  // NHB: head pairs x sequences
    // persistent: this CTA takes one item per round (cta_item), and every role walks the same
    // sequence

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
    uint64_t* full = bars;
    uint64_t* empty = bars + NSLOT;
    uint64_t* qfull = bars + 2 * NSLOT;
    uint64_t* qempty = qfull + 1;  // the item's last S has read Q: the next item's Q may land
    uint64_t* sfull = qempty + 1;
    uint64_t* pfull = sfull + 2;  // all of P_h stored (and O_h rescaled)
    uint64_t* phalf = pfull + 2;  // the first 64 keys' P_h stored (and O_h rescaled)
    uint64_t* odone = phalf + 2;
    uint64_t* drain = odone + 2;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);

    if (threadIdx.x == 0) {
        for (int s = 0; s < NSLOT; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(qfull, 1);
        mbar_init(qempty, 1);
        for (int h = 0; h < 2; ++h) {
            mbar_init(&sfull[h], 1);
            mbar_init(&pfull[h], 128);
            mbar_init(&phalf[h], 128);
            mbar_init(&odone[h], 1);
        }
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

    if (warp >= 8) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kControlRegs));
    }
    if (warp == 8) {
        // ------------------------------- TMA producer -------------------------------
        if (lane == 0) {
            tc::tma_prefetch_desc(&tm_q);
            tc::tma_prefetch_desc(&tm_k);
            tc::tma_prefetch_desc(&tm_v);
            int L = 0, nq = 0;  // ring loads and Q loads issued so far
            bool ok = true;
            for (int k_item = 0; ok; ++k_item) {
                const int item = cta_item(k_item, n_items, QT_SLOW);
                if (item < 0) break;
                const Item it = item_at(item, n_qtiles, HP, NHB, W, QT_SLOW);
                // the previous item's last S has read its Q
                if (nq > 0 && !wait_bar(qempty, (uint32_t)((nq - 1) & 1), abort_flag)) break;
                mbar_arrive_expect_tx(qfull, 2 * TILE_BYTES);
                for (int h = 0; h < 2; ++h)
                    for (int half = 0; half < 2; ++half)
                        tc::tma_load_3d(smem + OFF_Q + h * TILE_BYTES + half * HALF_BYTES, &tm_q,
                                        half * 64, it.t0, it.b * H + min(2 * it.hp + h, H - 1), qfull);
                ++nq;
                // K_j, V0_j, V1_j for the key tiles j of the item, through the ring
                for (int l = 0; l < 3 * it.n_it; ++l, ++L) {
                    const int slot = L % NSLOT, use = L / NSLOT;
                    if (use > 0 && !wait_bar(&empty[slot], (uint32_t)((use - 1) & 1), abort_flag)) {
                        ok = false;
                        break;
                    }
                    const int j = l / 3, which = l % 3, key0 = (it.kt_lo + j) * BN;
                    unsigned char* dst = smem + OFF_RING + slot * TILE_BYTES;
                    mbar_arrive_expect_tx(&full[slot], TILE_BYTES);
                    for (int half = 0; half < 2; ++half) {
                        if (which == 0)
                            tc::tma_load_3d(dst + half * HALF_BYTES, &tm_k, half * 64, key0, it.b, &full[slot]);
                        else
                            tc::tma_load_3d(dst + half * HALF_BYTES, &tm_v, half * 64, key0,
                                            it.b * H + min(2 * it.hp + which - 1, H - 1), &full[slot]);
                    }
                }
            }
            // every copy this thread started has landed before the CTA can leave: the last Q
            // load, and the last NSLOT ring loads (the latest phase of each slot)
            if (nq > 0) mbar_wait_bounded(qfull, (uint32_t)((nq - 1) & 1), kWaitLimit);
            for (int Li = (L > NSLOT ? L - NSLOT : 0); Li < L; ++Li)
                mbar_wait_bounded(&full[Li % NSLOT], (uint32_t)((Li / NSLOT) & 1), kWaitLimit);
        }
    } else if (warp == 9) {
        // ------------------------------- MMA issuer -------------------------------
        // The whole warp runs the issue loop in lockstep and one lane, elected inside each
        // instruction sequence, issues: the descriptors then stay in uniform registers and no
        // lane waits for another at a branch.
        const uint32_t idesc_s = tc::idesc_bf16_f32(BM, BN, 0, 0);  // Q K^T, both K-major
        const uint32_t idesc_o = tc::idesc_bf16_f32(BM, HD, 0, 1);  // P V, V is MN-major
        const uint32_t q_base = smem_u32(smem + OFF_Q);
        // TMEM columns: S_h at 256 h, O_h at 256 h + 128; Q_h at q_base + h * TILE_BYTES
        auto ring = [&](int L) { return smem_u32(smem + OFF_RING + (L % NSLOT) * TILE_BYTES); };
        auto acquire = [&](int L) {
            const bool ok = wait_bar_warp(&full[L % NSLOT], (uint32_t)((L / NSLOT) & 1), abort_flag);
            tc::fence_after_sync();
            return ok;
        };
        auto handoff = [&](uint64_t* bar, int j) {
            const bool ok = wait_bar_warp(bar, (uint32_t)(j & 1), abort_flag);
            tc::fence_after_sync();
            return ok;
        };
        // descriptors built once; a K step adds its offset (bytes >> 4) to the low word
        const uint64_t dq0 = tc::sdesc_sw128(q_base, 16, 1024);
        const uint64_t dq1 = tc::sdesc_sw128(q_base + TILE_BYTES, 16, 1024);
        const uint32_t dk_hi = tc::desc_hi(tc::sdesc_sw128(q_base, 16, 1024));  // LBO 16, SBO 1024
        const uint32_t dv_hi = tc::desc_hi(tc::sdesc_sw128(q_base, HALF_BYTES, 1024));
        auto issue_s = [&](int h, int L) {
            const uint32_t a_lo = tc::desc_lo(h ? dq1 : dq0), a_hi = tc::desc_hi(h ? dq1 : dq0);
            const uint32_t b_lo = tc::desc_lo(tc::sdesc_sw128(ring(L), 16, 1024));
#pragma unroll
            for (int k = 0; k < HD / 16; ++k) {
                const uint32_t koff = (uint32_t)(((k / 4) * HALF_BYTES + (k % 4) * 32) >> 4);
                tc::mma_ss_lh_warp(tmem + 256u * h, a_lo + koff, a_hi, b_lo + koff, dk_hi, idesc_s, k > 0);
            }
        };
        // O_h += P_h V over the keys 64 * half .. 64 * half + 63 (P_h packed in TMEM columns
        // 32 * half .. 32 * half + 31 of S_h)
        auto issue_pv = [&](int h, int L, bool acc, int half) {
            const uint32_t b_lo = tc::desc_lo(tc::sdesc_sw128(ring(L), HALF_BYTES, 1024));
#pragma unroll
            for (int k = 4 * half; k < 4 * half + 4; ++k)
                tc::mma_ts_lh_warp(tmem + 256u * h + 128u, tmem + 256u * h + 8u * k,
                                   b_lo + (uint32_t)((2048 * k) >> 4), dv_hi, idesc_o, (acc || k > 0) ? 1u : 0u);
        };
        // Per item: S0(0) S1(0) | PV0(j) S0(j+1) PV1(j) S1(j+1) | ... The ring position Lb, the
        // tile count tb (phases of sfull / phalf / pfull) and the item count (phases of qfull /
        // odone / qempty) run on across items. The next item's first S follows the last P V
        // at once: it only needs its Q and K, and its first P V waits for the softmax warps,
        // which finish the previous item's output rows before they hand over that P.
        int Lb = 0, tb = 0, items = 0;
        bool ok = true;
        for (int k_item = 0; ok; ++k_item) {
            const int item = cta_item(k_item, n_items, QT_SLOW);
            if (item < 0) break;
            const int n_it = item_at(item, n_qtiles, HP, NHB, W, QT_SLOW).n_it;
            if (!handoff(qfull, items) || !acquire(Lb)) break;
            issue_s(0, Lb);
            tc::mma_commit_warp(&sfull[0]);
            issue_s(1, Lb);
            tc::mma_commit_warp(&sfull[1]);
            tc::mma_commit_warp(&empty[Lb % NSLOT]);
            if (n_it == 1) tc::mma_commit_warp(qempty);
            for (int j = 0; j < n_it; ++j) {
                const bool more = j + 1 < n_it;
                const int Lj = Lb + 3 * j, tj = tb + j;
                // V0_j first (it landed long ago), then the softmax hand-off in two halves: the
                // first 64 keys' P V runs while the softmax still forms the rest of P. The next
                // key tile is only tested, so PV0 is never delayed by it, and when it is there
                // PV0 and S0 go to the tensor core back to back.
                if (!acquire(Lj + 1) || !handoff(&phalf[0], tj)) { ok = false; break; }
                issue_pv(0, Lj + 1, j > 0, 0);
                if (!handoff(&pfull[0], tj)) { ok = false; break; }
                const bool k_ready =
                    more && __all_sync(0xffffffffu, mbar_test_wait(&full[(Lj + 3) % NSLOT],
                                                                   (uint32_t)(((Lj + 3) / NSLOT) & 1)));
                tc::fence_after_sync();
                issue_pv(0, Lj + 1, j > 0, 1);
                tc::mma_commit_warp(&empty[(Lj + 1) % NSLOT]);
                if (more) {
                    if (!k_ready && !acquire(Lj + 3)) { ok = false; break; }
                    issue_s(0, Lj + 3);
                    tc::mma_commit_warp(&sfull[0]);
                } else {
                    tc::mma_commit_warp(&odone[0]);
                }
                if (!acquire(Lj + 2) || !handoff(&phalf[1], tj)) { ok = false; break; }
                issue_pv(1, Lj + 2, j > 0, 0);
                if (!handoff(&pfull[1], tj)) { ok = false; break; }
                issue_pv(1, Lj + 2, j > 0, 1);
                tc::mma_commit_warp(&empty[(Lj + 2) % NSLOT]);
                if (more) {
                    issue_s(1, Lj + 3);
                    tc::mma_commit_warp(&sfull[1]);
                    tc::mma_commit_warp(&empty[(Lj + 3) % NSLOT]);
                    if (j + 2 == n_it) tc::mma_commit_warp(qempty);  // the item's last S
                } else {
                    tc::mma_commit_warp(&odone[1]);
                }
            }
            Lb += 3 * n_it;
            tb += n_it;
            ++items;
        }
        // every MMA this warp issued has completed before TMEM is released
        tc::mma_commit_warp(drain);
        mbar_wait_bounded(drain, 0, kWaitLimit);
    } else if (warp < 8) {
        // ------------------------------- softmax warpgroups -------------------------------
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
        const int h = warp / 4;                     // head within the pair
        const int row = threadIdx.x % 128;          // query row == TMEM lane
        const uint32_t lane_base = (uint32_t)(32 * (warp % 4)) << 16;
        const uint32_t tS = tmem + 256u * h + lane_base;
        const uint32_t tO = tS + 128u;
        int tb = 0, items = 0;  // tiles and items done: the phases of sfull and odone
        bool ok = true;
        for (int k_item = 0; ok; ++k_item) {
            const int item = cta_item(k_item, n_items, QT_SLOW);
            if (item < 0) break;
            const Item it = item_at(item, n_qtiles, HP, NHB, W, QT_SLOW);
            const int t0 = it.t0, kt_lo = it.kt_lo, n_it = it.n_it, hp = it.hp, b = it.b;
            const int t = t0 + row;
            float m_run = -INFINITY, l_run = 0.f;
            for (int j = 0; j < n_it; ++j) {
                if (!wait_bar(&sfull[h], (uint32_t)((tb + j) & 1), abort_flag)) { ok = false; break; }
                tc::fence_after_sync();
                uint32_t s[BN];  // raw fp32 bits of the score row
                tc::tmem_ld32(tS + 0, s);
                tc::tmem_ld32(tS + 32, s + 32);
                tc::tmem_ld32(tS + 64, s + 64);
                tc::tmem_ld32(tS + 96, s + 96);
                tc::tmem_wait_ld();
                const int key0 = (kt_lo + j) * BN;
                const bool full_tile = key0 >= t0 + BM - W && key0 + BN - 1 <= t0;
                if (!full_tile) {
                    const int lo = t - W + 1 - key0, hi = t - key0;  // valid key columns [lo, hi]
#pragma unroll
                    for (int c = 0; c < BN; ++c)
                        if (c < lo || c > hi) s[c] = 0xff800000u;  // -inf
                }
                // row maximum: 8 independent chains of 3-input maxima over the columns c = 8k + i
                float m8[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    float m = __uint_as_float(s[i]);
#pragma unroll
                    for (int k = 1; k < 15; k += 2)
                        m = fmax3(m, __uint_as_float(s[8 * k + i]), __uint_as_float(s[8 * k + 8 + i]));
                    m8[i] = fmaxf(m, __uint_as_float(s[120 + i]));
                }
                const float mx = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
                const float m_tile = mx * scale_log2;
                const bool need = m_tile > m_run + kRescaleThreshold;
                const float alpha = need ? tc::ex2(m_run - m_tile) : 1.f;  // 0 when m_run = -inf
                l_run *= alpha;
                if (need) m_run = m_tile;
                const float m_use = m_run == -INFINITY ? 0.f : m_run;
                // a row whose maximum moved rescales its O row first (PV of the previous tile is done:
                // this tile's S was committed after it), so that the first half of P can be handed
                // over as soon as it is stored
                if (j > 0 && __any_sync(0xffffffffu, need)) {
#pragma unroll
                    for (int cb = 0; cb < HD; cb += 32) {
                        uint32_t r[32];
                        tc::tmem_ld32(tO + cb, r);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
                        tc::tmem_st32(tO + cb, r);
                    }
                }
                // P = 2^(s * scale * log2 e - m) as bf16 pairs over the first 64 columns of S; the
                // exponent arguments and the row sum use packed two-wide fp32 arithmetic, the sum in
                // four independent accumulators
                const float2 sc2 = make_float2(scale_log2, scale_log2), nm2 = make_float2(-m_use, -m_use);
                float2 l4[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t pk[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int c = 64 * half + 2 * i;
                        const float2 x = ffma2(make_float2(__uint_as_float(s[c]), __uint_as_float(s[c + 1])), sc2, nm2);
                        const float2 p = make_float2(tc::ex2(x.x), tc::ex2(x.y));
                        l4[i & 3] = fadd2(l4[i & 3], p);
                        pk[i] = pack_bf16x2(p.x, p.y);
                    }
                    tc::tmem_st32(tS + 32u * half, pk);
                    tc::tmem_wait_st();
                    tc::fence_before_sync();
                    mbar_arrive(half == 0 ? &phalf[h] : &pfull[h]);
                }
                {
                    const float2 a = fadd2(l4[0], l4[1]), b2 = fadd2(l4[2], l4[3]), t2 = fadd2(a, b2);
                    l_run += t2.x + t2.y;
                }
            }
            // epilogue: O / l -> bf16 rows. With statistics requested (the backward's first step), each
            // row also gets its negated base-2 log-sum-exp and D = dO . o from the fp32 O in TMEM
            // (-inf and 0 for rows past the end of the sequence), and O itself is stored only if asked.
            if (!ok || !wait_bar(&odone[h], (uint32_t)(items & 1), abort_flag)) {
                ok = false;
                break;
            }
            tc::fence_after_sync();
            const float inv = 1.f / l_run;
            const bool live = t < T && 2 * hp + h < H;  // an odd H's last pair computes one head twice
            const int64_t orow_i = ((int64_t)(b * H + 2 * hp + h) * T + t) * HD;
            float dacc = 0.f;
#pragma unroll
            for (int cb = 0; cb < HD; cb += 32) {
                uint32_t r[32];
                tc::tmem_ld32(tO + cb, r);
                tc::tmem_wait_ld();
                if (live && (!STATS || o != nullptr)) {
#pragma unroll
                    for (int i = 0; i < 32; i += 8) {
                        uint4 u;
                        u.x = pack_bf16x2(__uint_as_float(r[i + 0]) * inv, __uint_as_float(r[i + 1]) * inv);
                        u.y = pack_bf16x2(__uint_as_float(r[i + 2]) * inv, __uint_as_float(r[i + 3]) * inv);
                        u.z = pack_bf16x2(__uint_as_float(r[i + 4]) * inv, __uint_as_float(r[i + 5]) * inv);
                        u.w = pack_bf16x2(__uint_as_float(r[i + 6]) * inv, __uint_as_float(r[i + 7]) * inv);
                        *reinterpret_cast<uint4*>(o + orow_i + cb + i) = u;
                    }
                }
                if (STATS && live && dO != nullptr) {
#pragma unroll
                    for (int i = 0; i < 32; i += 8) {
                        float g[8];
                        load8(dO + orow_i + cb + i, g);
#pragma unroll
                        for (int e = 0; e < 8; ++e) dacc = fmaf(g[e], __uint_as_float(r[i + e]) * inv, dacc);
                    }
                }
            }
            // rows past T only where the statistics rows are padded (t < Tpad)
            if (STATS && 2 * hp + h < H && t < Tpad) {
                const int64_t srow = (int64_t)(b * H + 2 * hp + h) * Tpad + t;
                lse[srow] = live ? lse_mul * (m_run + log2f(l_run)) : -INFINITY;
                if (dbuf != nullptr) dbuf[srow] = live ? dacc : 0.f;
            }
            tb += n_it;
            ++items;
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 9) tc::tmem_dealloc(tmem, 512);
}

// streaming multiprocessors of the current device (queried once per device)
int sm_count() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cache[dev] == 0) {
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1) sms = 148;
        cache[dev] = sms;
    }
    return cache[dev];
}

}  // namespace

bool swska_prefill_tc_supported(int H, int T, int dk, int dv) {
    return dk == HD && dv == HD && H >= 1 && T >= BM;
}

cudaError_t swska_prefill_tc_launch(const void* q, const void* k, const void* v, void* o, int B,
                                    int H, int T, int window, float scale, cudaStream_t stream) {
    return swska_prefill_tc_stats_launch(q, k, v, o, nullptr, nullptr, nullptr, 0, B, H, T, window, scale,
                                         stream, -1.f);
}

cudaError_t swska_prefill_tc_stats_launch(const void* q, const void* k, const void* v, void* o,
                                          const void* dO, float* lse, float* dbuf, int64_t Tpad, int B,
                                          int H, int T, int window, float scale, cudaStream_t stream,
                                          float lse_mul) {
    CUtensorMap mq, mk, mv;
    cudaError_t e;
    if ((e = make_tmap_bf16_3d(&mq, q, HD, (uint64_t)T, (uint64_t)B * H, 64, BM)) != cudaSuccess) return e;
    if ((e = make_tmap_bf16_3d(&mk, k, HD, (uint64_t)T, (uint64_t)B, 64, BN)) != cudaSuccess) return e;
    if ((e = make_tmap_bf16_3d(&mv, v, HD, (uint64_t)T, (uint64_t)B * H, 64, BN)) != cudaSuccess) return e;
    const bool stats = lse != nullptr;
    const int n_qtiles = (T + BM - 1) / BM;
    const int64_t n_items = (int64_t)n_qtiles * ((H + 1) / 2) * B;
    if (n_items > INT32_MAX) return cudaErrorInvalidConfiguration;
    // persistent: one CTA per SM (the shared memory allows no second), each taking items in turn.
    // With few rounds of items a plain stride leaves the CTAs' loads uneven (at T 8192, W 4096,
    // 8 head pairs: 3.5 rounds, the busiest CTA 1.39x the mean): there the query-tile-slowest
    // numbering dealt out boustrophedon, while the head pairs x sequences are few enough to keep
    // neighbouring query tiles of each in flight together. With many rounds the stride is within
    // a few percent and keeps the tighter L2 reuse (measured: T 131072 3.4% faster with it).
    const int sms = sm_count();
    const unsigned grid = (unsigned)(n_items < sms ? n_items : sms);
    const bool qt_slow = (int64_t)((H + 1) / 2) * B <= 32 && n_items < 16 * (int64_t)sms;
    auto* kern = stats ? (qt_slow ? swska_tc_kernel<true, true> : swska_tc_kernel<true, false>)
                       : (qt_slow ? swska_tc_kernel<false, true> : swska_tc_kernel<false, false>);
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES)) != cudaSuccess)
        return e;
    kern<<<grid, NTHREADS, SMEM_BYTES, stream>>>(
        mq, mk, mv, static_cast<__nv_bfloat16*>(o), T, H, window, scale * 1.4426950408889634f,
        n_qtiles, (int)n_items, static_cast<const __nv_bfloat16*>(dO), lse, dbuf, (int)Tpad, lse_mul);
    note_launches(1);
    return cudaGetLastError();
}

unsigned swska_prefill_tc_take_timeout_flag() {
    unsigned v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_swska_tc_timeout, sizeof(v)) != cudaSuccess) return 0;
    cudaMemcpyToSymbol(g_swska_tc_timeout, &zero, sizeof(zero));
    return v;
}

}  // namespace rod
