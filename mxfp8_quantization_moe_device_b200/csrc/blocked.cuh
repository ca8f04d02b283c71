// blocked.cuh - per-group conversion of an E8M0 scale matrix to the 128x4
// blocked layout consumed by block-scaled grouped GEMMs (ao PR 3504
// "[mxfp8 moe training] add CUDA kernel for per-group conversion of scale
// factors to blocked layout"). Groups are row ranges from device-resident
// offsets; each group's rows are padded to a multiple of 128 on their own.
//
// Layout: padded matrix row R, column c (cols padded to cols4 = 4*ceil(c/4))
// -> tile (R/128)*(cols4/4) + c/4, byte (R%32)*16 + ((R%128)/32)*4 + c%4.
//
// Design: a CTA owns a column chunk of 32 tiles (128 source columns) and a
// strided set of output tile rows (128 rows each). It computes the padded
// group starts from the offsets once with a block scan (no host sync, no
// second launch), and for each of its tile rows finds the owning group by
// binary search, reads the 128 source rows as coalesced words (all loads in
// flight before any use) into shared memory with a row pitch of 33 words, so
// the transposed reads are conflict-free, and writes its tiles as one
// contiguous run of 16-byte stores. Pad rows, pad columns and tile rows past
// the last group are written as zeros.
#pragma once

#include "common.cuh"

namespace mxq {
namespace blk {

constexpr int THREADS = 256;
constexpr int TILES = 32;           // 128x4 tiles per CTA along the columns
constexpr int COLS = TILES * 4;     // 128 source columns per CTA
constexpr int PITCH = COLS / 4 + 1; // words per staged row
constexpr int MAX_G = 4096;

} // namespace blk

// padded tile-row start of every group: T[g] = sum_{h<g} ceil(size_h / 128),
// by a block scan in chunks of THREADS groups (warp shuffles plus one step
// across warps); returns false on bad offsets
MXQ_DEV bool padded_tile_starts(const int32_t *__restrict__ offs, int G, int64_t rows, int *T, int *Tend)
{
    using namespace blk;
    __shared__ int wsum[THREADS / 32];
    __shared__ int carry;
    if (!offsets_ok(offs, G, rows))
        return false;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (threadIdx.x == 0)
        carry = 0;
    __syncthreads();
    for (int g0 = 0; g0 < G; g0 += THREADS) {
        const int g = g0 + threadIdx.x;
        const int n = g < G ? (offs[g] - (g ? offs[g - 1] : 0) + 127) >> 7 : 0;
        int x = n; // inclusive warp scan
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o)
                x += y;
        }
        if (lane == 31)
            wsum[warp] = x;
        __syncthreads();
        int before = carry;
        for (int w = 0; w < warp; ++w)
            before += wsum[w];
        if (g < G)
            T[g] = before + x - n;
        __syncthreads();
        if (threadIdx.x == THREADS - 1)
            carry = before + x;
        __syncthreads();
    }
    if (threadIdx.x == 0)
        *Tend = carry;
    __syncthreads();
    return true;
}

__global__ void __launch_bounds__(blk::THREADS) k_blocked_grouped(const uint8_t *__restrict__ in, int64_t rows,
                                                                  int64_t cols, const int32_t *__restrict__ offs,
                                                                  int G, uint8_t *__restrict__ out,
                                                                  int32_t *__restrict__ starts_out, int words_ok,
                                                                  int64_t cap_tile_rows)
{
    using namespace blk;
    __shared__ int T[MAX_G];
    __shared__ int Tend;
    __shared__ uint32_t stage[128 * PITCH];
    if (!padded_tile_starts(offs, G, rows, T, &Tend))
        return;
    const int64_t cols4 = (cols + 3) / 4 * 4;
    const int64_t tiles_c = cols4 / 4;
    const int64_t tc0 = (int64_t)blockIdx.x * TILES; // first tile column
    const int ntiles = (int)min((int64_t)TILES, tiles_c - tc0);
    if (blockIdx.x == 0 && blockIdx.y == 0 && starts_out)
        for (int g = threadIdx.x; g < G; g += THREADS)
            starts_out[g] = T[g] * 128;
    if (ntiles <= 0)
        return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t c0 = tc0 * 4;
    // this CTA's output tile rows: blockIdx.y, blockIdx.y + gridDim.y, ...
    for (int64_t rt = blockIdx.y; rt < cap_tile_rows; rt += gridDim.y) {
        // group owning tile row rt: the largest g with T[g] <= rt (groups with
        // no tile rows share T with the next group, so it is non-empty);
        // tile rows past the last group are all zero
        int64_t src0 = 0, nvalid = 0;
        if (rt < Tend) {
            int a = 0, b = G - 1;
            while (a < b) {
                const int m = (a + b + 1) >> 1;
                if (T[m] <= rt) a = m; else b = m - 1;
            }
            const int64_t gs = a ? offs[a - 1] : 0, ge = offs[a];
            src0 = gs + (rt - T[a]) * 128;
            nvalid = min((int64_t)128, ge - src0);
        }
        // stage rows [src0, src0 + nvalid) x columns [c0, c0 + 4*ntiles):
        // all of this thread's loads are issued before any is used
        constexpr int PER = 128 / (THREADS / 32); // rows per warp
        uint32_t v[PER];
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int r = warp + i * (THREADS / 32);
            uint32_t x = 0;
            if (r < nvalid && lane < ntiles) {
                const int64_t c = c0 + 4 * lane;
                const uint8_t *src = in + (src0 + r) * cols + c;
                if (words_ok && c + 4 <= cols) {
                    x = __ldg(reinterpret_cast<const uint32_t *>(src));
                } else {
                    for (int j = 0; j < 4; ++j)
                        if (c + j < cols)
                            x |= (uint32_t)__ldg(src + j) << (8 * j);
                }
            }
            v[i] = x;
        }
#pragma unroll
        for (int i = 0; i < PER; ++i)
            stage[(warp + i * (THREADS / 32)) * PITCH + lane] = v[i];
        __syncthreads();
        // tile t, 16-byte row j: words of source rows j, 32+j, 64+j, 96+j
        uint8_t *dst = out + (rt * tiles_c + tc0) * 512;
        for (int q = threadIdx.x; q < ntiles * 32; q += THREADS) {
            const int t = q >> 5, j = q & 31;
            st_v4(dst + t * 512 + j * 16, stage[j * PITCH + t], stage[(32 + j) * PITCH + t],
                  stage[(64 + j) * PITCH + t], stage[(96 + j) * PITCH + t]);
        }
        __syncthreads();
    }
}

} // namespace mxq
