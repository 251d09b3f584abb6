// swska_decode_warp.cu -- SW-SKA decode for bf16 caches with d_k = d_v = 128 and up to 16 heads:
// one warp per head, one producer warp, an mbarrier ring with no block-wide barrier per stage.
//
// Semantics as in swska_decode.cu (SALA blog §3.3: the rolling window is a circular buffer,
// slot(p) = p mod W; CodeFuse Rodimus* article, Fig. 4 / SKA paragraph: one K row per position
// shared by every head, one V row per head):
//   o[n,h] = softmax over p in [max(0, P-W+1), P] of scale * q[n,h] . K[slot(p)], applied to
//            V[h, slot(p)],  with P = pos[n] and the new token stored at slot(P) first.
//
// Bound by HBM: per sequence and slot one 256-byte K row and H 256-byte V rows are read once.
//  * The grid is (N x SP) x (H / HG): a thread-block cluster of SP CTAs (up to 16) splits one
//    sequence's window into contiguous runs of valid slots, and each CTA serves a group of HG
//    heads (the shared K rows are then read once per head group). The host picks SP and HG
//    from the batch: large batches keep all heads in one CTA (K read once), small ones split
//    heads and window so that enough CTAs stream at once.
//  * Warp HG (the producer) moves KT-slot stages into a ring in shared memory with bulk async
//    copies: one for the K rows and one per head for its V rows (each contiguous in the cache).
//    The ring depth is a launch parameter (about 64 KB in flight per CTA). The slot the new
//    token overwrites is never read from the cache: its rows are written into the stage (and
//    into the cache) from k_new / v_new, and the copies skip it.
//  * Warp h (head h), lane l owns channels 4l .. 4l+3. Scores: each lane forms partial dots of
//    q_h with the stage's K rows over its channels; a reduce-scatter across the warp leaves the
//    score of slot j in lanes 4j .. 4j+3. The products are bf16 x bf16 FMAs into fp32
//    (fma.rn.f32.bf16), so the rows are used without unpacking. The online softmax runs in base
//    2 (scores times scale * log2 e); p_j, rounded to bf16 like the probabilities of the
//    tensor-core prefill, is broadcast by shuffle and accumulated into the lane's 4 output
//    columns from V_h. Shared-memory reads are 8 bytes per lane over a 256-byte row: no bank
//    conflicts.
//  * Stage hand-off: full[b] completes when the copies land (transaction bytes), empty[b] when
//    all HG head warps have read the stage.
//  * The SP partial (max, sum, accumulator) triples meet in distributed shared memory; CTA r
//    finalises the heads h with h mod SP == r.
//  * FP8 instance (SALA blog §4.3: the window cache stored in FP8): the rings hold OCP E4M3 codes
//    with one fp32 scale per cache, so a row is 128 bytes and a stage half the bytes. A lane's 4
//    channels are one 32-bit word, converted to f16 (exactly: every E4M3 value is an f16) and
//    multiplied with q (held in f16) by f16 x f16 -> fp32 FMAs; p is rounded to f16 for V. The
//    K scale folds into the score scale and the V scale into the final normalisation. The new
//    token is quantized by the producer: x / scale in fp32, then the nearest E4M3 code (ties to
//    even, saturated at +-448), into the stage and the cache.
// Every wait is bounded. On expiry the waiting warp raises the CTA's abort flag, every role stops
// at its next wait, the producer waits (bounded) for the copies it issued, the timeout flag is
// raised, the affected outputs are NaN, and all threads still meet at the cluster barriers.
#include <cooperative_groups.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include <math.h>

#include <mutex>

#include "common.cuh"
#include "fp8.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace rod {
namespace {

__device__ unsigned int g_swska_decode_warp_timeout = 0;

constexpr int KT = 8;            // slots per stage
constexpr int MAX_STAGES = 16;   // ring depth limit (the depth is a launch parameter)
constexpr int DH = 128;          // d_k = d_v
constexpr int ROW = DH * 2;      // bytes of one bf16 row
constexpr int ROW8 = DH;         // bytes of one E4M3 row
constexpr int MAX_H = 16;        // heads per CTA (one warp each)
template <bool FP8> constexpr int row_bytes() { return FP8 ? ROW8 : ROW; }
constexpr int OFF_FLAG = 256;    // after full[MAX_STAGES] and empty[MAX_STAGES]
constexpr int OFF_PM = 320;      // per-head max   [MAX_H] f32
constexpr int OFF_PL = 384;      // per-head sum   [MAX_H] f32
constexpr int OFF_PACC = 512;    // per-head accumulator [HG][128] f32

// HG: heads served by one CTA; C: head warps per head, each taking every C-th stage from a ring
// of its own (warps 0 .. HG C - 1, head w / C, ring w mod C) next to the producer warp HG C;
// D: stages per ring; row: bytes per row
__host__ __device__ constexpr uint32_t stage_bytes(int HG, int row = ROW) { return (uint32_t)(KT * row * (1 + HG)); }
__host__ __device__ constexpr uint32_t ring_offset(int HG) { return (uint32_t)(OFF_PACC + HG * DH * 4); }
// a CTA's slice of a paged block table: at most pages_per_seq + 1 entries (ROD_MAX_PAGES_PER_SEQ)
constexpr uint32_t kPageSlice = 520;
// with C > 1, each head warp's partial for the in-CTA merge: 128 accumulator columns, then the
// max and the sum, padded so that every partial starts on a 16-byte boundary (float4 accesses)
constexpr int PART = DH + 4;
__host__ __device__ constexpr uint32_t part_bytes(int HG, int C) { return C > 1 ? (uint32_t)(HG * C * PART * 4) : 0u; }
__host__ __device__ constexpr uint32_t smem_total(int HG, int C, int D, int row = ROW) {
    return ring_offset(HG) + (uint32_t)(C * D) * stage_bytes(HG, row) + 4u * kPageSlice + part_bytes(HG, C);
}

__device__ __forceinline__ bool wait_stage(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 0) {
            if (*abort_flag) return false;
            if (i >= kWaitLimit) {
                *abort_flag = 1;
                atomicExch(&g_swska_decode_warp_timeout, 1u);
                return false;
            }
        }
    }
}

__device__ __forceinline__ float ex2_approx(float x) {  // 2^x on the SFU (x = -inf gives 0)
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}



// c + a.lo * b.lo + a.hi * b.hi for two packed bf16 pairs: bf16 operands, fp32 products and sum
__device__ __forceinline__ float dot2_bf16(uint32_t a, uint32_t b, float c) {
    asm("{\n\t.reg .b16 al, ah, bl, bh;\n\tmov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, al, bl, %0;\n\tfma.rn.f32.bf16 %0, ah, bh, %0;\n\t}"
        : "+f"(c) : "r"(a), "r"(b));
    return c;
}
// acc[i] += p * v[i] for the 4 bf16 of w, p a bf16 in the low half of pw; fp32 accumulation
__device__ __forceinline__ void axpy4_bf16(uint32_t pw, uint2 w, float* acc) {
    asm("{\n\t.reg .b16 p, ph, v0, v1, v2, v3;\n\tmov.b32 {p, ph}, %4;\n\tmov.b32 {v0, v1}, %5;\n\t"
        "mov.b32 {v2, v3}, %6;\n\tfma.rn.f32.bf16 %0, p, v0, %0;\n\tfma.rn.f32.bf16 %1, p, v1, %1;\n\t"
        "fma.rn.f32.bf16 %2, p, v2, %2;\n\tfma.rn.f32.bf16 %3, p, v3, %3;\n\t}"
        : "+f"(acc[0]), "+f"(acc[1]), "+f"(acc[2]), "+f"(acc[3]) : "r"(pw), "r"(w.x), "r"(w.y));
}

// c + a.lo * b.lo + a.hi * b.hi for two packed f16 pairs: f16 operands, fp32 products and sum
__device__ __forceinline__ float dot2_f16(uint32_t a, uint32_t b, float c) {
    asm("{\n\t.reg .b16 al, ah, bl, bh;\n\tmov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
        "fma.rn.f32.f16 %0, al, bl, %0;\n\tfma.rn.f32.f16 %0, ah, bh, %0;\n\t}"
        : "+f"(c) : "r"(a), "r"(b));
    return c;
}
// acc[i] += p * v[i] for the 4 f16 in (w0, w1), p an f16 in the low half of pw; fp32 accumulation
__device__ __forceinline__ void axpy4_f16(uint32_t pw, uint32_t w0, uint32_t w1, float* acc) {
    asm("{\n\t.reg .b16 p, ph, v0, v1, v2, v3;\n\tmov.b32 {p, ph}, %4;\n\tmov.b32 {v0, v1}, %5;\n\t"
        "mov.b32 {v2, v3}, %6;\n\tfma.rn.f32.f16 %0, p, v0, %0;\n\tfma.rn.f32.f16 %1, p, v1, %1;\n\t"
        "fma.rn.f32.f16 %2, p, v2, %2;\n\tfma.rn.f32.f16 %3, p, v3, %3;\n\t}"
        : "+f"(acc[0]), "+f"(acc[1]), "+f"(acc[2]), "+f"(acc[3]) : "r"(pw), "r"(w0), "r"(w1));
}
struct HeadState {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};  // output columns 4 lane .. 4 lane + 3, unnormalised
    float m_run = -INFINITY;               // running max of the base-2 scores (warp-uniform)
    float l_part = 0.f;                    // this lane's share of the running sum
};

// One stage of KT slots for one head. kb / vb point at this lane's 4 channels of the stage's first
// K row and first V row of the head (8 bytes of bf16 or 4 of E4M3; rows row_bytes apart); qw is
// the lane's 4 channels of q (bf16, or f16 for the FP8 instance). FULL: all KT rows are valid.
template <bool FULL, bool FP8>
__device__ __forceinline__ void head_stage(const unsigned char* kb, const unsigned char* vb, uint2 qw,
                                           float scale_log2, int rows, int lane, HeadState& hs) {
    constexpr int RB = row_bytes<FP8>();
    // partial dots over this lane's 4 channels, one per slot
    float part[KT];
#pragma unroll
    for (int j = 0; j < KT; ++j) {
        if (FP8) {
            const uint32_t kw = *reinterpret_cast<const uint32_t*>(kb + j * RB);
            part[j] = dot2_f16(e4m3x2_to_f16x2(kw >> 16), qw.y, dot2_f16(e4m3x2_to_f16x2(kw), qw.x, 0.f));
        } else {
            const uint2 kw = *reinterpret_cast<const uint2*>(kb + j * RB);
            part[j] = dot2_bf16(kw.y, qw.y, dot2_bf16(kw.x, qw.x, 0.f));
        }
    }
    // reduce-scatter over the warp: halves of the slot set cross lane bit 4, then bit 3, then
    // bit 2; bits 1 and 0 finish the sums. Lane l ends with the score of slot (l >> 2) & 7.
    const bool b4 = (lane & 16) != 0, b3 = (lane & 8) != 0, b2 = (lane & 4) != 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float send = b4 ? part[i] : part[i + 4];
        const float keep = b4 ? part[i + 4] : part[i];
        part[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const float send = b3 ? part[i] : part[i + 2];
        const float keep = b3 ? part[i + 2] : part[i];
        part[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
    float dot;
    {
        const float send = b2 ? part[0] : part[1];
        const float keep = b2 ? part[1] : part[0];
        dot = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
    dot += __shfl_xor_sync(0xffffffffu, dot, 2);
    dot += __shfl_xor_sync(0xffffffffu, dot, 1);
    float s = dot * scale_log2;  // base-2 softmax
    if (!FULL && ((lane >> 2) & (KT - 1)) >= rows) s = -INFINITY;
    float mx = fmaxf(s, __shfl_xor_sync(0xffffffffu, s, 4));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
    if (mx > hs.m_run) {  // uniform branch
        const float alpha = ex2_approx(hs.m_run - mx);  // m_run = -inf gives 0
        hs.l_part *= alpha;
#pragma unroll
        for (int i = 0; i < 4; ++i) hs.acc[i] *= alpha;
        hs.m_run = mx;
    }
    // p in bf16 (f16 for the FP8 instance) as the weights of V; the sum takes the same rounded value
    uint32_t pw;
    if (FP8) {
        const __half ph = __float2half_rn(ex2_approx(s - hs.m_run));  // past the end: 0
        if ((lane & 3) == 0) hs.l_part += __half2float(ph);
        pw = (uint32_t)__half_as_ushort(ph);
    } else {
        const __nv_bfloat16 pb = __float2bfloat16_rn(ex2_approx(s - hs.m_run));
        if ((lane & 3) == 0) hs.l_part += __bfloat162float(pb);
        pw = (uint32_t)__bfloat16_as_ushort(pb);
    }
#pragma unroll
    for (int j = 0; j < KT; ++j) {
        const uint32_t pj = __shfl_sync(0xffffffffu, pw, 4 * j);
        if (FULL || j < rows) {  // rows past the end hold stale bytes
            if (FP8) {
                const uint32_t vw = *reinterpret_cast<const uint32_t*>(vb + j * RB);
                axpy4_f16(pj, e4m3x2_to_f16x2(vw), e4m3x2_to_f16x2(vw >> 16), hs.acc);
            } else {
                const uint2 vw = *reinterpret_cast<const uint2*>(vb + j * RB);
                axpy4_bf16(pj, vw, hs.acc);
            }
        }
    }
}

// Where the window cache lives. Contiguous: k [N][W][DH], v [N][H][W][DH], ring slot s of
// sequence n at row s. Paged (SALA blog §3.3: paged KV cache, allocated in blocks and evicted by
// window): the ring's slots are cut into pages of `page` slots; logical page i of sequence n is
// physical page table[n * pps + i] of the pools k [pages][page][DH] and v [pages][H][page][DH].
struct CacheRef {
    unsigned char* k;      // rows of row_bytes (bf16 or E4M3)
    unsigned char* v;
    const int32_t* table;  // paged only
    int page, pps;         // slots per page, pages per sequence (paged only)
    float k_scale, v_scale;  // FP8 only: value = code * scale
};
// Paged lookups read the CTA's slice of the block table, staged in shared memory at kernel start
// (pages[i] = table entry of logical page pg0 + i).
template <bool PAGED>
__device__ __forceinline__ int64_t k_row(const CacheRef& c, int64_t n, int W, int slot,
                                         const int32_t* pages, int pg0) {
    if (!PAGED) return n * W + slot;
    return (int64_t)pages[slot / c.page - pg0] * c.page + slot % c.page;
}
template <bool PAGED>
__device__ __forceinline__ int64_t v_row(const CacheRef& c, int64_t n, int H, int W, int64_t h, int slot,
                                         const int32_t* pages, int pg0) {
    if (!PAGED) return (n * H + h) * W + slot;
    return ((int64_t)pages[slot / c.page - pg0] * H + h) * c.page + slot % c.page;
}

// MULTI: several head warps per head (C > 1); the C = 1 instantiation keeps the single-ring code
template <bool PAGED, bool FP8, bool MULTI>
__global__ void __launch_bounds__(32 * (MAX_H + 1), 2)
swska_decode_warp_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k_new,
                         const __nv_bfloat16* __restrict__ v_new, CacheRef cache,
                         const int64_t* __restrict__ pos, __nv_bfloat16* __restrict__ o, int H, int HG,
                         int W, int C_arg, int D, float scale_log2) {
    const int C = MULTI ? C_arg : 1;
    extern __shared__ __align__(128) unsigned char smem[];
    cg::cluster_group cluster = cg::this_cluster();
    const int SP = (int)cluster.num_blocks();
    const int rank = (int)cluster.block_rank();
    const int64_t n = blockIdx.x / SP;
    const int hg0 = (int)blockIdx.y * HG;  // this CTA serves heads hg0 .. hg0 + HG - 1
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int RB = row_bytes<FP8>();
    const uint32_t SB = stage_bytes(HG, RB);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + MAX_STAGES;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_FLAG);
    float* s_pm = reinterpret_cast<float*>(smem + OFF_PM);
    float* s_pl = reinterpret_cast<float*>(smem + OFF_PL);
    float* s_pacc = reinterpret_cast<float*>(smem + OFF_PACC);
    unsigned char* ring = smem + ring_offset(HG);

    const int64_t P = pos[n];
    const bool bad = P < 0;
    // slot indices are below W (an int): 32-bit arithmetic keeps registers free
    const int cnt = bad ? 0 : (P + 1 < W ? (int)P + 1 : W);  // valid slots 0 .. cnt-1
    const int s_new = bad ? -1 : (int)(P % W);
    // slots per CTA, a multiple of the stage length so that no stage crosses a page
    const int per = ((cnt + SP - 1) / SP + KT - 1) / KT * KT;
    const int s_begin = rank * per < cnt ? rank * per : cnt;
    const int s_end = s_begin + per < cnt ? s_begin + per : cnt;
    const int nst = (int)((s_end - s_begin + KT - 1) / KT);

    // stage st lives in ring st mod C, buffer (st / C) mod D of it: buffer index (st mod C) D + that
    if (threadIdx.x == 0) {
        for (int s = 0; s < C * D; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], (uint32_t)HG);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == HG * C) {
        // ---------------------------------- producer warp ----------------------------------
        int32_t* pages = reinterpret_cast<int32_t*>(ring + (size_t)(C * D) * SB);
        const int pg0 = PAGED ? s_begin / cache.page : 0;
        if (PAGED) {
            const int npg = s_end > s_begin ? (s_end - 1) / cache.page - pg0 + 1 : 0;
            for (int i = lane; i < npg; i += 32) pages[i] = cache.table[n * cache.pps + pg0 + i];
            __syncwarp();
        }
        if (!MULTI) {
            // one ring, one stage per instruction (lanes 0 .. HG: the K rows and each head's V rows)
            int issued = 0;
            int buf = 0;
            uint32_t par = 0;  // parity of this use of buffer buf (uses counted from 0)
            int pi = 0, off = PAGED ? (int)(s_begin % cache.page) : 0;  // page slot of s0 (paged)
            for (int st = 0; st < nst; ++st) {
                if (st >= D) {
                    const bool ok = wait_stage(&empty[buf], par ^ 1u, abort_flag);
                    if (!__all_sync(0xffffffffu, ok)) break;
                }
                const int s0 = s_begin + st * KT;
                const int rows = s_end - s0 < KT ? s_end - s0 : KT;
                unsigned char* dst = ring + (size_t)buf * SB;
                const int r_new = (s_new >= s0 && s_new < s0 + rows) ? (int)(s_new - s0) : -1;
                if (r_new >= 0) {
                    // the evicted slot takes the new token: into the stage and into the cache (its
                    // old content lies outside the window, so it is never copied in); the shared K
                    // row goes to the cache from head group 0 only
                    for (int i = lane; i < (1 + HG) * (RB / 16); i += 32) {
                        const int row = i / (RB / 16), c16 = i % (RB / 16);
                        const int64_t hv = n * H + hg0 + (row - 1);  // (sequence, head) of a V row
                        const uint4* src = row == 0 ? reinterpret_cast<const uint4*>(k_new + n * DH)
                                                    : reinterpret_cast<const uint4*>(v_new + hv * DH);
                        // FP8: 16 codes from 16 bf16 of the row, quantized with the cache's scale
                        const uint4 val = FP8 ? quantize16(src[2 * c16], src[2 * c16 + 1], row == 0 ? cache.k_scale : cache.v_scale)
                                              : src[c16];
                        reinterpret_cast<uint4*>(dst + (size_t)row * KT * RB + (size_t)r_new * RB)[c16] = val;
                        if (row == 0) {
                            if (blockIdx.y == 0)
                                reinterpret_cast<uint4*>(cache.k + k_row<PAGED>(cache, n, W, s_new, pages, pg0) * RB)[c16] = val;
                        } else {
                            reinterpret_cast<uint4*>(cache.v + v_row<PAGED>(cache, n, H, W, hg0 + row - 1, s_new, pages, pg0) * RB)[c16] = val;
                        }
                    }
                    // the generic stores precede later bulk copies into the same bytes
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                }
                __syncwarp();
                const int copied = rows - (r_new >= 0 ? 1 : 0);
                if (lane == 0) mbar_arrive_expect_tx(&full[buf], (uint32_t)(copied * RB * (1 + HG)));
                __syncwarp();
                if (lane <= HG) {  // lane 0: the K rows; lane 1 + h: head hg0 + h's V rows
                    unsigned char* d = dst + (size_t)lane * KT * RB;
                    // rows s0 .. s0 + rows - 1 are contiguous (one page holds a whole stage)
                    int64_t row0;
                    if (PAGED) {
                        const int64_t t = pages[pi];
                        row0 = lane == 0 ? t * cache.page + off : (t * H + hg0 + lane - 1) * cache.page + off;
                    } else {
                        row0 = lane == 0 ? n * W + s0 : (n * H + hg0 + lane - 1) * W + s0;
                    }
                    const unsigned char* src = (lane == 0 ? cache.k : cache.v) + row0 * RB;
                    const int a0 = 0, a1 = r_new >= 0 ? r_new : rows;   // rows [a0, a1)
                    const int b0 = r_new >= 0 ? r_new + 1 : rows, b1 = rows;  // rows [b0, b1)
                    if (a1 > a0) bulk_g2s(d + (size_t)a0 * RB, src + (int64_t)a0 * RB, (uint32_t)((a1 - a0) * RB), &full[buf]);
                    if (b1 > b0) bulk_g2s(d + (size_t)b0 * RB, src + (int64_t)b0 * RB, (uint32_t)((b1 - b0) * RB), &full[buf]);
                }
                ++issued;
                if (++buf == D) { buf = 0; par ^= 1u; }
                if (PAGED && (off += KT) == cache.page) { off = 0; ++pi; }
            }
            // every copy issued has landed before the CTA's shared memory can go away (in the normal
            // course the head warps waited for these phases already)
            if (lane == 0) {
                for (int s2 = issued > D ? issued - D : 0; s2 < issued; ++s2)
                    if (!mbar_wait_bounded(&full[s2 % D], (uint32_t)((s2 / D) & 1), kWaitLimit))
                        atomicExch(&g_swska_decode_warp_timeout, 1u);
            }
            __syncwarp();
        } else {
            // Stages go out C at a time, one per ring (batch u holds stages u C .. u C + C - 1, each in
            // buffer u mod D of its ring). One instruction carries a batch's copies: lane l takes row
            // group l mod RG (0: the K rows, 1 + h: head hg0 + h's V rows) of the batch's stage l / RG.
            // (One thread's copies go out a few hundred clocks apart; different lanes' together.)
            const int RG = 1 + HG;
            const int lst = lane / RG, lrg = lane - lst * RG;  // this lane's stage in a batch, row group
            int ub = 0;                                        // u mod D
            uint32_t par = 0;                                  // parity of use u / D of the buffers
            int pi = 0, poff = 0;  // paged: page (index into pages) and slot of this lane's stage
            if (PAGED) {
                const int rel = s_begin - pg0 * cache.page + lst * KT;
                pi = rel / cache.page;
                poff = rel - pi * cache.page;
            }
            const int st_new = (s_new >= s_begin && s_new < s_end) ? (s_new - s_begin) / KT : -1;
            int issued_batches = 0;
            for (int st0 = 0; st0 < nst; st0 += C) {
                const int nb = nst - st0 < C ? nst - st0 : C;  // stages in this batch
                // the batch's buffers are free once their previous uses are released
                const bool need = lane < nb && st0 >= C * D;
                if (!__all_sync(0xffffffffu, !need || wait_stage(&empty[lane * D + ub], par ^ 1u, abort_flag))) break;
                if (st_new >= st0 && st_new < st0 + nb) {
                    // the evicted slot takes the new token: into the stage and into the cache (its
                    // old content lies outside the window, so it is never copied in); the shared K
                    // row goes to the cache from head group 0 only
                    const int r_new = s_new - (s_begin + st_new * KT);
                    unsigned char* dst = ring + (size_t)((st_new - st0) * D + ub) * SB;
                    for (int i = lane; i < RG * (RB / 16); i += 32) {
                        const int row = i / (RB / 16), c16 = i % (RB / 16);
                        const int64_t hv = n * H + hg0 + (row - 1);  // (sequence, head) of a V row
                        const uint4* src = row == 0 ? reinterpret_cast<const uint4*>(k_new + n * DH)
                                                    : reinterpret_cast<const uint4*>(v_new + hv * DH);
                        // FP8: 16 codes from 16 bf16 of the row, quantized with the cache's scale
                        const uint4 val = FP8 ? quantize16(src[2 * c16], src[2 * c16 + 1], row == 0 ? cache.k_scale : cache.v_scale)
                                              : src[c16];
                        reinterpret_cast<uint4*>(dst + (size_t)row * KT * RB + (size_t)r_new * RB)[c16] = val;
                        if (row == 0) {
                            if (blockIdx.y == 0)
                                reinterpret_cast<uint4*>(cache.k + k_row<PAGED>(cache, n, W, s_new, pages, pg0) * RB)[c16] = val;
                        } else {
                            reinterpret_cast<uint4*>(cache.v + v_row<PAGED>(cache, n, H, W, hg0 + row - 1, s_new, pages, pg0) * RB)[c16] = val;
                        }
                    }
                    // the generic stores precede later bulk copies into the same bytes
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                }
                __syncwarp();
                // each stage's full barrier expects its bytes before any of its copies can land
                if (lane < nb) {
                    const int st = st0 + lane, s0 = s_begin + st * KT;
                    const int rows = s_end - s0 < KT ? s_end - s0 : KT;
                    mbar_arrive_expect_tx(&full[lane * D + ub], (uint32_t)((rows - (st == st_new ? 1 : 0)) * RB * RG));
                }
                __syncwarp();
                if (lst < nb) {
                    const int st = st0 + lst, s0 = s_begin + st * KT;
                    const int rows = s_end - s0 < KT ? s_end - s0 : KT;
                    const int r_new = st == st_new ? s_new - s0 : -1;
                    uint64_t* fb = &full[lst * D + ub];
                    unsigned char* d = ring + (size_t)(lst * D + ub) * SB + (size_t)lrg * KT * RB;
                    // rows s0 .. s0 + rows - 1 are contiguous (one page holds a whole stage)
                    int64_t row0;
                    if (PAGED) {
                        const int64_t t = pages[pi];
                        row0 = lrg == 0 ? t * cache.page + poff : (t * H + hg0 + lrg - 1) * cache.page + poff;
                    } else {
                        row0 = lrg == 0 ? n * W + s0 : (n * H + hg0 + lrg - 1) * W + s0;
                    }
                    const unsigned char* src = (lrg == 0 ? cache.k : cache.v) + row0 * RB;
                    const int a0 = 0, a1 = r_new >= 0 ? r_new : rows;         // rows [a0, a1)
                    const int b0 = r_new >= 0 ? r_new + 1 : rows, b1 = rows;  // rows [b0, b1)
                    if (a1 > a0) bulk_g2s(d + (size_t)a0 * RB, src + (int64_t)a0 * RB, (uint32_t)((a1 - a0) * RB), fb);
                    if (b1 > b0) bulk_g2s(d + (size_t)b0 * RB, src + (int64_t)b0 * RB, (uint32_t)((b1 - b0) * RB), fb);
                }
                ++issued_batches;
                if (++ub == D) { ub = 0; par ^= 1u; }
                if (PAGED)
                    for (poff += C * KT; poff >= cache.page; poff -= cache.page) ++pi;
            }
            // every copy issued has landed before the CTA's shared memory can go away (in the normal
            // course the head warps waited for these phases already): the last D batches of each ring
            if (lane < C) {
                for (int u = issued_batches > D ? issued_batches - D : 0; u < issued_batches; ++u)
                    if (u * C + lane < nst &&
                        !mbar_wait_bounded(&full[lane * D + u % D], (uint32_t)((u / D) & 1), kWaitLimit))
                        atomicExch(&g_swska_decode_warp_timeout, 1u);
            }
            __syncwarp();
        }
    } else if (warp < HG * C) {
        // -------------------- head warp: head hg0 + h, stages c, c + C, ... --------------------
        const int h = warp / C, c = warp - h * C;
        uint2 qw = *reinterpret_cast<const uint2*>(q + (n * H + hg0 + h) * (int64_t)DH + 4 * lane);
        if (FP8) {  // q in f16 for the f16 x f16 products with the E4M3 rows
            const __half2 a = __floats2half2_rn(bf16lo(qw.x), bf16hi(qw.x));
            const __half2 b = __floats2half2_rn(bf16lo(qw.y), bf16hi(qw.y));
            qw = make_uint2(*reinterpret_cast<const uint32_t*>(&a), *reinterpret_cast<const uint32_t*>(&b));
        }
        HeadState hs;
        bool ok = true;
        int ub = 0;
        uint32_t par = 0;
        for (int st = c; st < nst; st += C) {
            const int bi = c * D + ub;
            if (!__all_sync(0xffffffffu, wait_stage(&full[bi], par, abort_flag))) {
                ok = false;
                break;
            }
            const int s0 = s_begin + st * KT;
            const int rows = s_end - s0 < KT ? s_end - s0 : KT;
            const unsigned char* kb = ring + (size_t)bi * SB + (RB / 32) * lane;
            const unsigned char* vb = kb + (size_t)(1 + h) * KT * RB;
            if (rows == KT) head_stage<true, FP8>(kb, vb, qw, scale_log2, KT, lane, hs);
            else head_stage<false, FP8>(kb, vb, qw, scale_log2, rows, lane, hs);
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[bi]);
            if (++ub == D) { ub = 0; par ^= 1u; }
        }
        float l = hs.l_part;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
        if (!MULTI) {
            if (lane == 0) { s_pm[h] = ok ? hs.m_run : NAN; s_pl[h] = l; }
            *reinterpret_cast<float4*>(s_pacc + h * DH + 4 * lane) =
                make_float4(hs.acc[0], hs.acc[1], hs.acc[2], hs.acc[3]);
        } else {
            float* part = reinterpret_cast<float*>(ring + (size_t)(C * D) * SB + 4u * kPageSlice) +
                          (size_t)warp * PART;
            if (lane == 0) { part[DH] = ok ? hs.m_run : NAN; part[DH + 1] = l; }
            *reinterpret_cast<float4*>(part + 4 * lane) = make_float4(hs.acc[0], hs.acc[1], hs.acc[2], hs.acc[3]);
        }
    }
    if (MULTI) {
        // merge each head's C partials, in ring order (deterministic), into the head's triple
        __syncthreads();
        if (warp < HG * C && warp % C == 0) {
            const int h = warp / C;
            const float* part = reinterpret_cast<const float*>(ring + (size_t)(C * D) * SB + 4u * kPageSlice) +
                                (size_t)warp * PART;
            float M = -INFINITY;
            bool nan = false;
            for (int cc = 0; cc < C; ++cc) {
                const float m = part[cc * PART + DH];
                nan |= isnan(m);
                M = fmaxf(M, m);
            }
            float L = 0.f, a[4] = {0.f, 0.f, 0.f, 0.f};
            for (int cc = 0; cc < C; ++cc) {
                const float* pc = part + cc * PART;
                if (!(pc[DH] > -INFINITY)) continue;  // a head warp without slots (or one that gave up)
                const float w = ex2_approx(pc[DH] - M);
                L = fmaf(w, pc[DH + 1], L);
                const float4 pa = *reinterpret_cast<const float4*>(pc + 4 * lane);
                a[0] = fmaf(w, pa.x, a[0]); a[1] = fmaf(w, pa.y, a[1]);
                a[2] = fmaf(w, pa.z, a[2]); a[3] = fmaf(w, pa.w, a[3]);
            }
            if (lane == 0) { s_pm[h] = nan ? NAN : M; s_pl[h] = L; }
            *reinterpret_cast<float4*>(s_pacc + h * DH + 4 * lane) = make_float4(a[0], a[1], a[2], a[3]);
        }
    }
    cluster.sync();
    // ---- combine: CTA `rank` finalises the heads h with h mod SP == rank (warp h, 4 columns a lane)
    if (warp < HG && warp % SP == rank) {
        const int h = warp;
        float out[4];
        if (bad) {
#pragma unroll
            for (int i = 0; i < 4; ++i) out[i] = NAN;
        } else {
            float M = -INFINITY;
            for (int r = 0; r < SP; ++r) M = fmaxf(M, cluster.map_shared_rank(s_pm, r)[h]);
            float L = 0.f, a[4] = {0.f, 0.f, 0.f, 0.f};
            for (int r = 0; r < SP; ++r) {
                const float mr = cluster.map_shared_rank(s_pm, r)[h];
                const float lr = cluster.map_shared_rank(s_pl, r)[h];
                if (!(lr > 0.f) && !isnan(mr)) continue;  // a CTA without slots
                const float w = ex2_approx(mr - M);
                L = fmaf(w, lr, L);
                const float4 pa = *reinterpret_cast<const float4*>(cluster.map_shared_rank(s_pacc, r) + h * DH + 4 * lane);
                a[0] = fmaf(w, pa.x, a[0]); a[1] = fmaf(w, pa.y, a[1]);
                a[2] = fmaf(w, pa.z, a[2]); a[3] = fmaf(w, pa.w, a[3]);
            }
            const float inv = (FP8 ? cache.v_scale : 1.f) / L;
#pragma unroll
            for (int i = 0; i < 4; ++i) out[i] = a[i] * inv;
        }
        store4(o + (n * H + hg0 + h) * (int64_t)DH + 4 * lane, make_float4(out[0], out[1], out[2], out[3]));
    }
    cluster.sync();  // this CTA's shared memory stays alive until every peer has read it
}


struct DecodeConfig {
    int SP;      // CTAs per cluster: the window split
    int HG;      // heads per CTA
    int stages;  // ring depth (per ring)
    int C = 1;   // head warps per head, one ring each
};

// ring depth: about 64 KB of copies in flight per CTA, at least 3 stages
int stages_for(int HG, int row = ROW) {
    int st = (int)(65536u / stage_bytes(HG, row));
    return st < 3 ? 3 : (st > MAX_STAGES ? MAX_STAGES : st);
}

template <bool PAGED, bool FP8, bool MULTI = false>
cudaError_t set_attributes(size_t smem) {
    cudaError_t e = cudaFuncSetAttribute(swska_decode_warp_kernel<PAGED, FP8, MULTI>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(swska_decode_warp_kernel<PAGED, FP8, MULTI>,
                                 cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    return e;
}

// Clusters of the given shape that the GPU holds at once (queried once per device, shape and
// cache format; 0 if the shape cannot be launched).
int clusters_that_fit(int HG, int sp, bool fp8) {
    static std::mutex mu;
    static int cache[64][MAX_H + 1][5][2];
    static bool init = false;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    int si = 0;
    while ((1 << si) < sp) ++si;
    std::lock_guard<std::mutex> lock(mu);
    if (!init) {
        for (auto& a : cache)
            for (auto& b : a)
                for (auto& c : b)
                    for (int& d : c) d = -1;
        init = true;
    }
    int& slot = cache[dev][HG][si][fp8 ? 1 : 0];
    if (slot < 0) {
        const int row = fp8 ? ROW8 : ROW;
        const size_t smem = smem_total(HG, 1, stages_for(HG, row), row);
        int num = 0;
        if ((fp8 ? set_attributes<false, true>(smem) : set_attributes<false, false>(smem)) == cudaSuccess) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3((unsigned)sp, 1, 1);
            cfg.blockDim = dim3((unsigned)(32 * (HG + 1)), 1, 1);
            cfg.dynamicSmemBytes = smem;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = (unsigned)sp;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            // the paged instance has the same resources as the ring one
            const cudaError_t q = fp8 ? cudaOccupancyMaxActiveClusters(&num, swska_decode_warp_kernel<false, true, false>, &cfg)
                                      : cudaOccupancyMaxActiveClusters(&num, swska_decode_warp_kernel<false, false, false>, &cfg);
            if (q != cudaSuccess) num = 0;
        }
        cudaGetLastError();
        slot = num;
    }
    return slot;
}

// Launch shape. The work is HBM-bound: per sequence W shared-K rows (read once per head group)
// and H x W V rows. Estimated time, in bytes-at-full-bandwidth units, is the larger of
//   - the total bytes, and
//   - (waves of CTAs) x (bytes one CTA streams) x (SMs-worth of CTAs that saturate HBM),
// where one CTA streams about 1/200 of the GPU's bandwidth (measured: ~31 GB/s against
// 6.4 TB/s with 16 heads per CTA). Splitting the heads (fewer per CTA) and the window (bigger
// clusters, up to 16) multiplies the CTAs for small batches at the price of reading K once per
// head group. Among equal estimates the smaller split wins. (Rows are the unit: the FP8 rows'
// halved bytes scale both terms alike.)
constexpr double kCtasToSaturate = 200.0;

DecodeConfig pick_config(int N, int H, int W, bool fp8) {
    const int row = fp8 ? ROW8 : ROW;
    // Small batches (N H <= 64): with one head warp per head, each CTA walks its 8-slot stages one
    // after the other at about 900 clocks each, and the time follows the stages per CTA, not the
    // bytes (measured at N 1: 5 us + 3.4 us per 1024 slots for any head count). There, about 256
    // CTAs of one or two heads each, a 16-CTA cluster at most splitting a window, and each head
    // spread over C = 8 head warps (each taking every C-th stage from a ring of its own, the
    // producer sending C stages per instruction): measured at H 16, W 4096, in CUDA graphs,
    // N 1: 11.9 against 20.8 us, N 4: 20.1 against 24.5 us; at N 16 it no longer pays.
    if ((int64_t)N * H <= 64) {
        const int HG = ((int64_t)N * H * 16 <= 256 || H % 2) ? 1 : 2;
        int sp = 16;
        while (sp > 1 && (int64_t)N * sp * (H / HG) > 256) sp /= 2;
        const int stages_per_cta = ((W + sp - 1) / sp + KT - 1) / KT;
        int C = 1;
        while (2 * C <= 8 && 2 * C * (1 + HG) <= 32 && 2 * C * HG <= 16 && 8 * C <= stages_per_cta) C *= 2;
        if (C > 1 && clusters_that_fit(HG, sp, fp8) > 0) {
            const int by_bytes = (int)(65536u / ((uint32_t)C * stage_bytes(HG, row)));
            const int D = 16 / C < by_bytes ? 16 / C : by_bytes;
            return DecodeConfig{sp, HG, D < 2 ? 2 : D, C};
        }
    }
    DecodeConfig best{1, H, stages_for(H, row)};
    double best_cost = -1.0;
    for (int HG = H; HG >= 1; --HG) {
        if (H % HG) continue;
        const int groups = H / HG;
        const double bytes = (double)N * W * (double)(groups + H);
        for (int sp = 1; sp <= 16; sp *= 2) {
            const int64_t cap = (int64_t)clusters_that_fit(HG, sp, fp8) * sp;  // CTAs resident at once
            if (cap <= 0) continue;
            const int64_t ctas = (int64_t)N * sp * groups;
            const double waves = (double)((ctas + cap - 1) / cap);
            const double per_cta = (double)((W + sp - 1) / sp) * (1 + HG);
            const double t = waves * per_cta * kCtasToSaturate;
            const double cost = t > bytes ? t : bytes;
            if (best_cost < 0.0 || cost < best_cost * 0.98) {
                best_cost = cost;
                best = DecodeConfig{sp, HG, stages_for(HG, row)};
            }
        }
    }
    return best;
}

}  // namespace

bool swska_decode_warp_supported(int H, int dk, int dv) {
    return dk == DH && dv == DH && H >= 1 && H <= MAX_H;
}

namespace {

template <bool PAGED, bool FP8>
cudaError_t launch(const void* q, const void* k_new, const void* v_new, CacheRef cache, const int64_t* pos,
                   void* o, int N, int H, int window, float scale, cudaStream_t stream) {
    if (N == 0) return cudaSuccess;
    constexpr int RB = row_bytes<FP8>();
    const DecodeConfig c = pick_config(N, H, window, FP8);
    const size_t smem = smem_total(c.HG, c.C, c.stages, RB);
    cudaError_t e = c.C > 1 ? set_attributes<PAGED, FP8, true>(smem) : set_attributes<PAGED, FP8, false>(smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((int64_t)N * c.SP), (unsigned)(H / c.HG), 1);
    cfg.blockDim = dim3((unsigned)(32 * (c.HG * c.C + 1)), 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)c.SP;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // the K scale multiplies every score: folded into the base-2 score scale
    const float scale_log2 = scale * 1.4426950408889634f * (FP8 ? cache.k_scale : 1.f);
    note_launches(1);
    auto* kern = c.C > 1 ? swska_decode_warp_kernel<PAGED, FP8, true> : swska_decode_warp_kernel<PAGED, FP8, false>;
    return cudaLaunchKernelEx(&cfg, kern,
                              static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k_new),
                              static_cast<const __nv_bfloat16*>(v_new), cache, pos,
                              static_cast<__nv_bfloat16*>(o), H, c.HG, window, c.C, c.stages, scale_log2);
}

}  // namespace

cudaError_t swska_decode_warp_launch(const void* q, const void* k_new, const void* v_new,
                                     void* k_cache, void* v_cache, const int64_t* pos, void* o,
                                     int N, int H, int window, float scale, cudaStream_t stream) {
    const CacheRef c{static_cast<unsigned char*>(k_cache), static_cast<unsigned char*>(v_cache), nullptr, 0, 0,
                     1.f, 1.f};
    return launch<false, false>(q, k_new, v_new, c, pos, o, N, H, window, scale, stream);
}

cudaError_t swska_decode_paged_launch(const void* q, const void* k_new, const void* v_new, void* k_pool,
                                      void* v_pool, const int32_t* block_table, int page_size,
                                      int pages_per_seq, const int64_t* pos, void* o, int N, int H,
                                      int window, float scale, cudaStream_t stream) {
    const CacheRef c{static_cast<unsigned char*>(k_pool), static_cast<unsigned char*>(v_pool), block_table,
                     page_size, pages_per_seq, 1.f, 1.f};
    return launch<true, false>(q, k_new, v_new, c, pos, o, N, H, window, scale, stream);
}

cudaError_t swska_decode_fp8_launch(const void* q, const void* k_new, const void* v_new, void* k_cache,
                                    void* v_cache, const int64_t* pos, void* o, int N, int H, int window,
                                    float scale, float k_scale, float v_scale, cudaStream_t stream) {
    const CacheRef c{static_cast<unsigned char*>(k_cache), static_cast<unsigned char*>(v_cache), nullptr, 0, 0,
                     k_scale, v_scale};
    return launch<false, true>(q, k_new, v_new, c, pos, o, N, H, window, scale, stream);
}

unsigned swska_decode_warp_take_timeout_flag() {
    unsigned v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_swska_decode_warp_timeout, sizeof(v)) != cudaSuccess) return 0;
    cudaMemcpyToSymbol(g_swska_decode_warp_timeout, &zero, sizeof(zero));
    return v;
}

}  // namespace rod
