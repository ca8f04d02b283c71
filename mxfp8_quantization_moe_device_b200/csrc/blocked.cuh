// blocked.cuh - per-group conversion of an E8M0 scale matrix to the 128x4
// blocked layout consumed by block-scaled grouped GEMMs (ao PR 3504
// "[mxfp8 moe training] add CUDA kernel for per-group conversion of scale
// factors to blocked layout"). Groups are row ranges from device-resident
// offsets; each group's rows are padded to a multiple of 128 on their own.
//
// Layout: padded matrix row R, column c (cols padded to cols4 = 4*ceil(c/4))
// -> tile (R/128)*(cols4/4) + c/4, byte (R%32)*16 + ((R%128)/32)*4 + c%4.
//
// Design: one CTA per (output tile row of 128 rows, 32 tiles = 128 columns).
// Each CTA recomputes the padded group starts from the offsets with a block
// scan (no host sync, no second launch), finds its group by binary search,
// reads the 128 source rows as coalesced words into shared memory (row pitch
// of 33 words, so the transposed reads below are conflict-free) and writes
// its 32 tiles as one contiguous 16 KB run of 16-byte stores. Pad rows, pad
// columns and tile rows past the last group are written as zeros.
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

// padded tile-row start of every group: T[g] = sum_{h<g} ceil(size_h / 128)
// computed by a block-wide scan; returns false on bad offsets
MXQ_DEV bool padded_tile_starts(const int32_t *__restrict__ offs, int G, int64_t rows, int *T, int *Tend)
{
    using namespace blk;
    __shared__ int part[THREADS];
    if (!offsets_ok(offs, G, rows))
        return false;
    const int per = (G + THREADS - 1) / THREADS;
    const int g0 = threadIdx.x * per;
    int local = 0;
    for (int g = g0; g < min(G, g0 + per); ++g) {
        const int size = offs[g] - (g ? offs[g - 1] : 0);
        local += (size + 127) >> 7;
    }
    part[threadIdx.x] = local;
    __syncthreads();
    // inclusive scan of the THREADS partial sums (Hillis-Steele)
    for (int o = 1; o < THREADS; o <<= 1) {
        const int v = threadIdx.x >= o ? part[threadIdx.x - o] : 0;
        __syncthreads();
        part[threadIdx.x] += v;
        __syncthreads();
    }
    int run = part[threadIdx.x] - local; // exclusive prefix
    for (int g = g0; g < min(G, g0 + per); ++g) {
        T[g] = run;
        const int size = offs[g] - (g ? offs[g - 1] : 0);
        run += (size + 127) >> 7;
    }
    if (threadIdx.x == THREADS - 1)
        *Tend = part[THREADS - 1];
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
    const int64_t rt = blockIdx.y;              // output tile row
    const int64_t tc0 = (int64_t)blockIdx.x * TILES; // first tile column
    const int ntiles = (int)min((int64_t)TILES, tiles_c - tc0);
    if (blockIdx.x == 0 && blockIdx.y == 0 && starts_out)
        for (int g = threadIdx.x; g < G; g += THREADS)
            starts_out[g] = T[g] * 128;
    if (rt >= cap_tile_rows || ntiles <= 0)
        return;

    // group owning this tile row (largest g with T[g] <= rt and a non-empty
    // range there), or none past the last group
    int64_t src0 = 0, nvalid = 0;
    if (rt < Tend) {
        int a = 0, b = G - 1; // last g with T[g] <= rt
        while (a < b) {
            const int m = (a + b + 1) >> 1;
            if (T[m] <= rt) a = m; else b = m - 1;
        }
        // groups with zero tile rows share T with the next group; the
        // largest g with T[g] <= rt is the one that owns tile row rt
        const int64_t gs = a ? offs[a - 1] : 0, ge = offs[a];
        const int64_t first = gs + (rt - T[a]) * 128;
        src0 = first;
        nvalid = min((int64_t)128, ge - first);
    }

    // stage rows [src0, src0 + nvalid) x columns [4*tc0, 4*tc0 + 4*ntiles)
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t c0 = tc0 * 4;
    for (int r = warp; r < 128; r += THREADS / 32) {
        for (int wd = lane; wd < TILES; wd += 32) {
            uint32_t v = 0;
            if (r < nvalid && wd < ntiles) {
                const int64_t c = c0 + 4 * wd;
                const uint8_t *src = in + (src0 + r) * cols + c;
                if (words_ok && c + 4 <= cols) {
                    v = __ldg(reinterpret_cast<const uint32_t *>(src));
                } else {
                    for (int j = 0; j < 4; ++j)
                        if (c + j < cols)
                            v |= (uint32_t)__ldg(src + j) << (8 * j);
                }
            }
            stage[r * PITCH + wd] = v;
        }
    }
    __syncthreads();

    // tile t, 16-byte row j: words of source rows j, 32+j, 64+j, 96+j
    uint8_t *dst = out + (rt * tiles_c + tc0) * 512;
    for (int q = threadIdx.x; q < ntiles * 32; q += THREADS) {
        const int t = q >> 5, j = q & 31;
        st_v4(dst + t * 512 + j * 16, stage[j * PITCH + t], stage[(32 + j) * PITCH + t],
              stage[(64 + j) * PITCH + t], stage[(96 + j) * PITCH + t]);
    }
}

} // namespace mxq
