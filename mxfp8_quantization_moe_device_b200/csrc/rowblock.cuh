// rowblock.cuh - quantization of row-contiguous blocks: fp8 1x128 and
// 128x128 blocks (ao PR 2827 "[fp8 blockwise] load 2d chunks for groupwise
// quant to enable coalesced gmem accesses") and MXFP8 1x32 blocks along the
// last dimension (the to_mx-style rowwise cast named in ao PR 3002's Summary).
//
// Design: these are pure streaming kernels (2 bytes in, 1 byte out per
// element), so every lane moves 16-byte vectors with evict-first loads and
// the grid is sized to fill all SMs; a group of lanes owns one block, so the
// block's amax is a shuffle reduction and its codes are written as one
// contiguous, coalesced run. The 2-D chunking the page describes becomes a
// warp covering several consecutive blocks per load instruction.
#pragma once

#include "common.cuh"

namespace mxq {

// ---------------------------------------------------------------------------
// fp8 1x128: one half-warp per block, 8 elements (16 B) per lane.
// The (rows, cols) matrix with cols % 128 == 0 is a flat run of nblk blocks;
// block b covers elements [128b, 128b+128) and owns inv_scales[b], which is
// the row-major (rows, cols/128) layout.
// ---------------------------------------------------------------------------
constexpr int RB_THREADS = 256;
constexpr int RB_UNROLL = 4;

__global__ void __launch_bounds__(RB_THREADS) k_fp8_1x128(const uint4 *__restrict__ in, int64_t nblk,
                                                          uint2 *__restrict__ out, float *__restrict__ inv)
{
    const int lane = threadIdx.x & 31;
    const int half = lane >> 4, l16 = lane & 15;
    const int64_t warp = ((int64_t)blockIdx.x * RB_THREADS + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * RB_THREADS) >> 5;
    // warp-uniform trip count: each warp step covers 2 blocks per unroll slot
    for (int64_t w0 = warp; w0 * 2 < nblk; w0 += nwarps * RB_UNROLL) {
        uint4 v[RB_UNROLL];
#pragma unroll
        for (int u = 0; u < RB_UNROLL; ++u) {
            const int64_t b = (w0 + u * nwarps) * 2 + half;
            v[u] = b < nblk ? ld_stream_v4(in + b * 16 + l16) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < RB_UNROLL; ++u) {
            const int64_t b = (w0 + u * nwarps) * 2 + half;
            uint32_t acc = absmax_bf16x2(absmax_bf16x2(0u, v[u].x), v[u].y);
            acc = absmax_bf16x2(absmax_bf16x2(acc, v[u].z), v[u].w);
            float amax = absmax_of_pair(acc);
#pragma unroll
            for (int o = 8; o >= 1; o >>= 1)
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
            const float s = fp8_scale(amax);
            if (b < nblk) {
                st_v2(out + b * 16 + l16, quant4(v[u].x, v[u].y, s), quant4(v[u].z, v[u].w, s));
                if (l16 == 0)
                    inv[b] = fp8_inv(s);
            }
        }
    }
}

// ---------------------------------------------------------------------------
// fp8 128x128: one CTA per block. Thread t holds column chunk t%16 (8
// elements) of rows t/16 + 16i, i < 8, in registers; the block amax is a warp
// shuffle plus a shared-memory step, then the codes are written from
// registers.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_fp8_128x128(const uint4 *__restrict__ in, int64_t cols,
                                                     uint2 *__restrict__ out, float *__restrict__ inv)
{
    __shared__ float red[8];
    const int bj = blockIdx.x;
    const int64_t bi = blockIdx.y;
    const int c = threadIdx.x & 15, r0 = threadIdx.x >> 4;
    const int64_t cols8 = cols >> 3;
    const int64_t base = bi * 128 * cols8 + (int64_t)bj * 16 + c;
    uint4 v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
        v[i] = ld_stream_v4(in + base + (int64_t)(r0 + 16 * i) * cols8);
    uint32_t acc = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        acc = absmax_bf16x2(acc, v[i].x);
        acc = absmax_bf16x2(acc, v[i].y);
        acc = absmax_bf16x2(acc, v[i].z);
        acc = absmax_bf16x2(acc, v[i].w);
    }
    float amax = absmax_of_pair(acc);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1)
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if ((threadIdx.x & 31) == 0)
        red[threadIdx.x >> 5] = amax;
    __syncthreads();
    amax = red[0];
#pragma unroll
    for (int i = 1; i < 8; ++i)
        amax = fmaxf(amax, red[i]);
    const float s = fp8_scale(amax);
#pragma unroll
    for (int i = 0; i < 8; ++i)
        st_v2(out + base + (int64_t)(r0 + 16 * i) * cols8, quant4(v[i].x, v[i].y, s), quant4(v[i].z, v[i].w, s));
    if (threadIdx.x == 0)
        inv[bi * gridDim.x + bj] = fp8_inv(s);
}

// ---------------------------------------------------------------------------
// MXFP8 1x32: one lane quad per block, 8 elements per lane, a warp covers 8
// consecutive blocks (512 B in, 256 B out, 8 scale bytes). The quad's amax
// gives the E8M0 byte; lanes 0 and 16 gather four bytes each by shuffle and
// store them as one word.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(RB_THREADS) k_mx_1x32(const uint4 *__restrict__ in, int64_t nblk,
                                                       uint2 *__restrict__ out, uint8_t *__restrict__ scales,
                                                       int scales_word_aligned, int mode)
{
    const int lane = threadIdx.x & 31;
    const int q = lane >> 2, l4 = lane & 3;
    const int64_t warp = ((int64_t)blockIdx.x * RB_THREADS + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * RB_THREADS) >> 5;
    for (int64_t w0 = warp; w0 * 8 < nblk; w0 += nwarps * RB_UNROLL) {
        uint4 v[RB_UNROLL];
#pragma unroll
        for (int u = 0; u < RB_UNROLL; ++u) {
            const int64_t b = (w0 + u * nwarps) * 8 + q;
            v[u] = b < nblk ? ld_stream_v4(in + b * 4 + l4) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < RB_UNROLL; ++u) {
            const int64_t wb = w0 + u * nwarps;
            const int64_t b = wb * 8 + q;
            uint32_t acc = absmax_bf16x2(absmax_bf16x2(0u, v[u].x), v[u].y);
            acc = absmax_bf16x2(absmax_bf16x2(acc, v[u].z), v[u].w);
            float amax = absmax_of_pair(acc);
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
            const uint32_t byte = e8m0_mode(amax, mode);
            const float f = mx_factor(byte);
            // gather the four scale bytes of blocks (lane & 16)/4 .. +3
            const int src = lane & 16;
            const uint32_t s0 = __shfl_sync(0xffffffffu, byte, src + 0);
            const uint32_t s1 = __shfl_sync(0xffffffffu, byte, src + 4);
            const uint32_t s2 = __shfl_sync(0xffffffffu, byte, src + 8);
            const uint32_t s3 = __shfl_sync(0xffffffffu, byte, src + 12);
            if (b < nblk)
                st_v2(out + b * 4 + l4, quant4(v[u].x, v[u].y, f), quant4(v[u].z, v[u].w, f));
            if ((lane & 15) == 0) {
                const int64_t b0 = wb * 8 + (lane >> 2);
                if (scales_word_aligned && b0 + 4 <= nblk) {
                    *reinterpret_cast<uint32_t *>(scales + b0) = s0 | (s1 << 8) | (s2 << 16) | (s3 << 24);
                } else {
                    const uint32_t sb[4] = {s0, s1, s2, s3};
                    for (int i = 0; i < 4; ++i)
                        if (b0 + i < nblk)
                            scales[b0 + i] = (uint8_t)sb[i];
                }
            }
        }
    }
}

} // namespace mxq
