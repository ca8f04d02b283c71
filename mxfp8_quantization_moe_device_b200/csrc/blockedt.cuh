// blockedt.cuh - the per-group 128x4 blocked scale layouts of blocked.cuh
// (ao PR 3504 "[mxfp8 moe training] add CUDA kernel for per-group conversion
// of scale factors to blocked layout": groups along the rows, and the stacked
// "groups along K" variant) as persistent TMA-ring kernels, for scale
// matrices whose rows are a multiple of 16 bytes long.
//
// Work unit: one output tile row (128 padded rows) x one chunk of 32 output
// tile columns = 32 tiles of 512 bytes, 16 KB contiguous in the output. The
// producer warp loads the unit's source block (128 rows of the source run)
// with one TMA box into a ring slot; four consumer warps each turn a quarter
// of it into output words with 32-bit shared-memory reads and write 16-byte
// vectors straight to global memory, eight lanes covering 128 contiguous
// bytes. No CTA-wide barrier sits on the per-unit path.
//
// Output word (tile t, 16-byte row j, word i) = the 4 source bytes of tile
// column t in padded row 32 i + j of the tile row. A lane takes tile
// t = 4a + lane/8 and row j = 8b + lane%8 for the warp's (a, b) pairs, so
// that its four reads and the warp's stores are conflict-free and coalesced:
//   groups along rows: the box is 128 rows x 128 bytes in the 128-byte
//   swizzle (16-byte chunk c of row r at chunk c ^ (r % 8)); the 8 lanes of a
//   tile read 8 different chunks and the 4 tiles of a chunk 4 different words.
//   groups along K: a tile column's 4 bytes start anywhere in the source row,
//   so the box is 128 rows x 144 bytes from the 16-byte boundary at or below
//   the chunk's first source byte, unswizzled (row pitch 36 words: bank
//   4 r + w, r%8 and the 4 consecutive words of a tile quad are distinct),
//   and a word that straddles two source words is assembled with a byte
//   permute.
// Rows past a group's end in the box belong to the next group (or lie past
// the matrix, where TMA fills zeros) and are masked to zero; capacity past
// the last group is written as zeros without a load.
#pragma once

#include "blocked.cuh"

namespace mxq {
namespace blkt {

constexpr int CWARPS = 4;
constexpr int THREADS = (CWARPS + 1) * 32;
constexpr int STAGES = 4;
constexpr int ROWS = 128;                 // source rows per unit
constexpr int TILES = 32;                 // output tiles per unit
constexpr int R_BOX_X = 128;              // groups along rows: bytes per box row
constexpr int K_BOX_X = 144;              // groups along K: bytes per box row
constexpr int R_STAGE = ROWS * R_BOX_X;   // 16 KB
constexpr int K_STAGE = ROWS * K_BOX_X;   // 18 KB

template <int STAGE_BYTES> struct __align__(1024) Smem {
    uint8_t in[STAGES][STAGE_BYTES];
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    int abort_flag;
    int Tend;
};
template <int STAGE_BYTES> constexpr size_t smem_fixed() { return sizeof(Smem<STAGE_BYTES>) + 1024; }

// the group owning padded unit u (< Tend): the last g with T[g] <= u (groups
// with no unit share T with the next group)
MXQ_DEV int owner(const int *T, int G, int64_t u)
{
    int a = 0, b = G - 1;
    while (a < b) {
        const int m = (a + b + 1) >> 1;
        if (T[m] <= u) a = m; else b = m - 1;
    }
    return a;
}

MXQ_DEV uint32_t lds32(uint32_t addr)
{
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

// barrier init, padded starts into T and the offsets into so (dynamic
// shared memory after the fixed part: the per-unit group lookups then touch
// no global memory), and the group starts of CTA 0; false on bad offsets
template <int STAGE_BYTES>
MXQ_DEV bool setup(Smem<STAGE_BYTES> &sm, int *T, int *so, const int32_t *offs, int G, int64_t extent, int shift,
                   int32_t *starts_out, int start_mul)
{
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], CWARPS);
        }
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    if (!padded_starts(offs, G, extent, shift, T, &sm.Tend))
        return false;
    for (int g = threadIdx.x; g < G; g += blockDim.x)
        so[g] = offs[g];
    __syncthreads();
    if (blockIdx.x == 0 && starts_out)
        for (int g = threadIdx.x; g < G; g += blockDim.x)
            starts_out[g] = T[g] * start_mul;
    return true;
}

// the producer's wait for a free slot, and its drain before the CTA exits
MXQ_DEV bool slot_free(uint64_t *empty, int it, uint64_t wait_ns, int *abort_flag)
{
    if (it >= STAGES && !mbar_wait(&empty[it % STAGES], ((uint32_t)(it / STAGES) & 1u) ^ 1u, wait_ns)) {
        *reinterpret_cast<volatile int *>(abort_flag) = 1;
        return false;
    }
    return true;
}

MXQ_DEV void drain(uint64_t *full, int it, uint64_t wait_ns)
{
    for (int j = it - STAGES; j < it; ++j)
        if (j >= 0)
            mbar_wait(&full[j % STAGES], (uint32_t)(j / STAGES) & 1u, wait_ns);
}

} // namespace blkt

// Groups along rows (the layout of k_blocked_grouped). tm_in: the (rows,
// cols) u8 scale matrix, box 128 x 128 bytes, 128-byte swizzle.
__global__ void __launch_bounds__(blkt::THREADS) k_blocked_grouped_tma(const __grid_constant__ CUtensorMap tm_in,
                                                                     int64_t rows, int64_t cols,
                                                                     const int32_t *__restrict__ offs, int G,
                                                                     uint8_t *__restrict__ out,
                                                                     int32_t *__restrict__ starts_out,
                                                                     int64_t cap_tile_rows, uint64_t wait_ns)
{
    using namespace blkt;
    using SM = Smem<R_STAGE>;
    extern __shared__ uint8_t smem_raw[];
    SM &sm = *reinterpret_cast<SM *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    int *T = reinterpret_cast<int *>(&sm + 1), *so = T + G;
    if (!setup(sm, T, so, offs, G, rows, 7, starts_out, 128))
        return;
    const int Tend = sm.Tend;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t tiles_c = (cols + 3) / 4, nch = (tiles_c + TILES - 1) / TILES;
    const int64_t units = cap_tile_rows * nch;

    if (warp == CWARPS) {
        if (lane == 0) {
            int it = 0;
            for (int64_t u = blockIdx.x; u < units; u += gridDim.x, ++it) {
                if (!slot_free(sm.empty, it, wait_ns, &sm.abort_flag))
                    break;
                const int s = it % STAGES;
                const int64_t rt = u / nch, ch = u - rt * nch;
                if (rt < Tend) {
                    const int g = owner(T, G, rt);
                    const int64_t src0 = (g ? so[g - 1] : 0) + (rt - T[g]) * ROWS;
                    mbar_arrive_expect_tx(&sm.full[s], R_STAGE);
                    tma_load_2d(sm.in[s], &tm_in, &sm.full[s], (int)(ch * R_BOX_X), (int)src0);
                } else {
                    mbar_arrive(&sm.full[s]); // capacity past the last group: zeros, nothing to read
                }
            }
            blkt::drain(sm.full, it, wait_ns);
        }
        return;
    }

    // consumer warp: (a, b) pairs a = 2 warp + k / 4, b = k % 4, k < 8
    const int tq = lane >> 3, jr = lane & 7;
    int it = 0;
    for (int64_t u = blockIdx.x; u < units; u += gridDim.x, ++it) {
        const int s = it % STAGES;
        const int64_t rt = u / nch, ch = u - rt * nch;
        int nvalid = 0;
        if (rt < Tend) {
            const int g = owner(T, G, rt);
            const int64_t src0 = (g ? so[g - 1] : 0) + (rt - T[g]) * ROWS;
            nvalid = (int)min((int64_t)ROWS, (int64_t)so[g] - src0);
        }
        const int ntiles = (int)min((int64_t)TILES, tiles_c - ch * TILES);
        bool ok = mbar_wait(&sm.full[s], (uint32_t)(it / STAGES) & 1u, wait_ns);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok || *reinterpret_cast<volatile int *>(&sm.abort_flag)) {
            *reinterpret_cast<volatile int *>(&sm.abort_flag) = 1;
            break;
        }
        const uint32_t base = smem_u32(sm.in[s]);
        uint32_t w[8][4];
        uint32_t dep = 0;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int a = 2 * warp + (k >> 2), j = 8 * (k & 3) + jr;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = 32 * i + j;
                w[k][i] = r < nvalid ? lds32(base + r * R_BOX_X + ((a ^ jr) << 4) + (tq << 2)) : 0u;
                dep ^= w[k][i];
            }
        }
        release_slot_after(&sm.empty[s], dep);
        uint8_t *dst = out + (rt * tiles_c + ch * TILES) * 512;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int t = 4 * (2 * warp + (k >> 2)) + tq, j = 8 * (k & 3) + jr;
            if (t < ntiles)
                st_v4(dst + t * 512 + j * 16, w[k][0], w[k][1], w[k][2], w[k][3]);
        }
    }
}

// Groups along K (the layout of k_blocked_grouped_k). tm_in: the (rows,
// cols) u8 scale matrix, box 128 rows x 144 bytes, no swizzle; cap_cols the
// output columns (a multiple of 4).
__global__ void __launch_bounds__(blkt::THREADS) k_blocked_grouped_k_tma(const __grid_constant__ CUtensorMap tm_in,
                                                                       int64_t rows, int64_t cols,
                                                                       const int32_t *__restrict__ offs, int G,
                                                                       uint8_t *__restrict__ out,
                                                                       int32_t *__restrict__ starts_out,
                                                                       int64_t cap_cols, uint64_t wait_ns)
{
    using namespace blkt;
    using SM = Smem<K_STAGE>;
    extern __shared__ uint8_t smem_raw[];
    SM &sm = *reinterpret_cast<SM *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    int *T = reinterpret_cast<int *>(&sm + 1), *so = T + G;
    if (!setup(sm, T, so, offs, G, cols, 2, starts_out, 4))
        return;
    const int Tend = sm.Tend;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t tiles_c = cap_cols / 4, nch = (tiles_c + TILES - 1) / TILES;
    const int64_t tile_rows = (rows + ROWS - 1) / ROWS;
    const int64_t units = tile_rows * nch;
    // source byte of output tile column tc (< Tend) and the bytes it holds
    auto column = [&](int64_t tc, int64_t &src, int &nv) {
        const int g = owner(T, G, tc);
        const int64_t gs = g ? so[g - 1] : 0;
        src = gs + (tc - T[g]) * 4;
        nv = (int)min((int64_t)4, (int64_t)so[g] - src);
    };

    if (warp == CWARPS) {
        if (lane == 0) {
            int it = 0;
            for (int64_t u = blockIdx.x; u < units; u += gridDim.x, ++it) {
                if (!slot_free(sm.empty, it, wait_ns, &sm.abort_flag))
                    break;
                const int s = it % STAGES;
                const int64_t rt = u / nch, ch = u - rt * nch;
                if (ch * TILES < Tend) {
                    int64_t s0;
                    int nv;
                    column(ch * TILES, s0, nv);
                    mbar_arrive_expect_tx(&sm.full[s], K_STAGE);
                    tma_load_2d(sm.in[s], &tm_in, &sm.full[s], (int)(s0 & ~int64_t(15)), (int)(rt * ROWS));
                } else {
                    mbar_arrive(&sm.full[s]); // columns past the last group: zeros
                }
            }
            blkt::drain(sm.full, it, wait_ns);
        }
        return;
    }

    const int tq = lane >> 3, jr = lane & 7;
    int it = 0;
    for (int64_t u = blockIdx.x; u < units; u += gridDim.x, ++it) {
        const int s = it % STAGES;
        const int64_t rt = u / nch, ch = u - rt * nch;
        const int ntiles = (int)min((int64_t)TILES, tiles_c - ch * TILES);
        // the lane's two tile columns t = 4 (2 warp + h) + tq, h < 2: byte
        // offset in the box row, the byte permute that picks its 4 bytes
        // from two adjacent words, and the mask of the bytes it holds
        int wi[2];
        uint32_t sel[2], mask[2];
        int64_t x0 = 0;
        if (ch * TILES < Tend) {
            int64_t s0;
            int nv0;
            column(ch * TILES, s0, nv0);
            x0 = s0 & ~int64_t(15);
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int64_t tc = ch * TILES + 4 * (2 * warp + h) + tq;
            int64_t src = x0;
            int nv = 0;
            if (tc < Tend)
                column(tc, src, nv);
            const int b = (int)(src - x0); // 0 .. 140
            wi[h] = b >> 2;
            sel[h] = 0x3210u + 0x1111u * (uint32_t)(b & 3);
            mask[h] = nv >= 4 ? 0xFFFFFFFFu : (nv <= 0 ? 0u : (1u << (8 * nv)) - 1u);
        }
        bool ok = mbar_wait(&sm.full[s], (uint32_t)(it / STAGES) & 1u, wait_ns);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok || *reinterpret_cast<volatile int *>(&sm.abort_flag)) {
            *reinterpret_cast<volatile int *>(&sm.abort_flag) = 1;
            break;
        }
        const uint32_t base = smem_u32(sm.in[s]);
        uint32_t w[8][4];
        uint32_t dep = 0;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int h = k >> 2, j = 8 * (k & 3) + jr;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t row = base + (32 * i + j) * K_BOX_X;
                uint32_t v = 0u;
                if (mask[h]) {
                    const uint32_t lo = lds32(row + 4 * wi[h]);
                    const uint32_t hi = wi[h] + 1 < K_BOX_X / 4 ? lds32(row + 4 * wi[h] + 4) : 0u;
                    v = __byte_perm(lo, hi, sel[h]) & mask[h];
                }
                w[k][i] = v;
                dep ^= v;
            }
        }
        release_slot_after(&sm.empty[s], dep);
        uint8_t *dst = out + (rt * tiles_c + ch * TILES) * 512;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int t = 4 * (2 * warp + (k >> 2)) + tq, j = 8 * (k & 3) + jr;
            if (t < ntiles)
                st_v4(dst + t * 512 + j * 16, w[k][0], w[k][1], w[k][2], w[k][3]);
        }
    }
}

} // namespace mxq
