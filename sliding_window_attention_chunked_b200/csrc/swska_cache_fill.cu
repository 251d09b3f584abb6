// swska_cache_fill.cu -- hand-off from SW-SKA prefill to decode: the rolling window of the last
// W prefill tokens is written into the decode ring buffers.
//
// SALA blog §3.3: prefill runs over the prompt in chunks; decode then keeps the most recent W
// keys/values in a self-managed circular buffer and overwrites the oldest slot each step. With
// the ring rule slot(p) = p mod W used by decode, after a prefill of T tokens the cache must hold
// position p at slot p mod W for every p in [max(0, T - W), T): then a decode step at position
// P = T sees exactly the window the prefill row T would. CodeFuse Rodimus* article, SKA
// paragraph: one K row per position shared by all heads, one V row per head.
//
//   K[b, p mod W, :]    = k[b, p, :]         (k: [B, T, dk], K: [B, W, dk])
//   V[b, h, p mod W, :] = v[b, h, p, :]      (v: [B, H, T, dv], V: [B, H, W, dv])
//
// Pure data movement (HBM-bound, each byte read and written once): every thread moves 16-byte
// pieces of whole rows, consecutive threads consecutive pieces, in a grid-stride loop.
// FP8 rings (SALA blog §4.3): the same rows quantized to E4M3 codes of x / scale (fp8.cuh); a
// thread reads 32 bytes of bf16 and writes one 16-byte piece of codes.
#include "common.cuh"
#include "fp8.cuh"
#include "kernels.h"

namespace rod {
namespace {

__global__ void __launch_bounds__(256)
swska_cache_fill_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v, uint4* __restrict__ kc,
                        uint4* __restrict__ vc, int H, int T, int W, int p0, int n, int kvec, int vvec,
                        int64_t total) {
    // piece index -> (b, row kind, position, piece): per sequence, first n K rows of kvec pieces,
    // then H x n V rows of vvec pieces
    const int64_t per_seq = (int64_t)n * kvec + (int64_t)H * n * vvec;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t b = i / per_seq;
        int64_t r = i - b * per_seq;
        if (r < (int64_t)n * kvec) {
            const int p = p0 + (int)(r / kvec), e = (int)(r % kvec);
            kc[(b * W + p % W) * kvec + e] = k[(b * T + p) * kvec + e];
        } else {
            r -= (int64_t)n * kvec;
            const int64_t hp = r / vvec;
            const int e = (int)(r % vvec), h = (int)(hp / n), p = p0 + (int)(hp % n);
            vc[((b * H + h) * W + p % W) * vvec + e] = v[((b * H + h) * T + p) * vvec + e];
        }
    }
}

__global__ void __launch_bounds__(256)
swska_cache_fill_fp8_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v, uint4* __restrict__ kc,
                            uint4* __restrict__ vc, int H, int T, int W, int p0, int n, int kvec, int vvec,
                            int64_t total, float k_scale, float v_scale) {
    // as above, with kvec / vvec counting 16-code output pieces (each from two 16-byte inputs)
    const int64_t per_seq = (int64_t)n * kvec + (int64_t)H * n * vvec;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t b = i / per_seq;
        int64_t r = i - b * per_seq;
        if (r < (int64_t)n * kvec) {
            const int p = p0 + (int)(r / kvec), e = (int)(r % kvec);
            const uint4* src = k + ((b * T + p) * kvec + e) * 2;
            kc[(b * W + p % W) * kvec + e] = quantize16(src[0], src[1], k_scale);
        } else {
            r -= (int64_t)n * kvec;
            const int64_t hp = r / vvec;
            const int e = (int)(r % vvec), h = (int)(hp / n), p = p0 + (int)(hp % n);
            const uint4* src = v + (((b * H + h) * T + p) * vvec + e) * 2;
            vc[((b * H + h) * W + p % W) * vvec + e] = quantize16(src[0], src[1], v_scale);
        }
    }
}

int fill_blocks(int64_t total) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t blocks = (total + 255) / 256;
    if (blocks > (int64_t)sms * 8) blocks = (int64_t)sms * 8;  // 8 blocks of 256 per SM, grid-stride beyond
    return (int)blocks;
}

}  // namespace

cudaError_t swska_cache_fill_fp8_launch(const void* k, const void* v, void* k_cache, void* v_cache, int B,
                                        int H, int T, int dk, int dv, int window, float k_scale, float v_scale,
                                        cudaStream_t stream) {
    const int p0 = T > window ? T - window : 0;
    const int n = T - p0;
    if (B == 0 || n <= 0) return cudaSuccess;
    const int kvec = dk / 16, vvec = dv / 16;  // output pieces of 16 codes per row
    const int64_t total = (int64_t)B * ((int64_t)n * kvec + (int64_t)H * n * vvec);
    swska_cache_fill_fp8_kernel<<<(unsigned)fill_blocks(total), 256, 0, stream>>>(
        static_cast<const uint4*>(k), static_cast<const uint4*>(v), static_cast<uint4*>(k_cache),
        static_cast<uint4*>(v_cache), H, T, window, p0, n, kvec, vvec, total, k_scale, v_scale);
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t swska_cache_fill_launch(const void* k, const void* v, void* k_cache, void* v_cache, int B,
                                    int H, int T, int dk, int dv, int window, size_t elem_bytes,
                                    cudaStream_t stream) {
    const int p0 = T > window ? T - window : 0;
    const int n = T - p0;
    if (B == 0 || n <= 0) return cudaSuccess;
    const int kvec = (int)(dk * elem_bytes / 16), vvec = (int)(dv * elem_bytes / 16);
    const int64_t total = (int64_t)B * ((int64_t)n * kvec + (int64_t)H * n * vvec);
    swska_cache_fill_kernel<<<(unsigned)fill_blocks(total), 256, 0, stream>>>(
        static_cast<const uint4*>(k), static_cast<const uint4*>(v), static_cast<uint4*>(k_cache),
        static_cast<uint4*>(v_cache), H, T, window, p0, n, kvec, vvec, total);
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace rod
