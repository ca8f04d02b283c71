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

// padded start of every group in units of 2^shift: T[g] = sum_{h<g}
// ceil(size_h / 2^shift) (shift 7: tile rows of 128; shift 2: tile columns of
// 4), by a block scan in chunks of blockDim.x groups (warp shuffles plus one
// step across warps; blockDim.x a multiple of 32, at most THREADS); returns
// false on bad offsets
MXQ_DEV bool padded_starts(const int32_t *__restrict__ offs, int G, int64_t extent, int shift, int *T, int *Tend)
{
    using namespace blk;
    __shared__ int wsum[THREADS / 32];
    __shared__ int carry;
    if (!offsets_ok(offs, G, extent))
        return false;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (threadIdx.x == 0)
        carry = 0;
    __syncthreads();
    for (int g0 = 0; g0 < G; g0 += blockDim.x) {
        const int g = g0 + threadIdx.x;
        const int n = g < G ? (offs[g] - (g ? offs[g - 1] : 0) + (1 << shift) - 1) >> shift : 0;
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
        if (threadIdx.x == blockDim.x - 1)
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
    extern __shared__ int T[]; // G entries
    __shared__ int Tend;
    __shared__ uint32_t stage[128 * PITCH];
    if (!padded_starts(offs, G, rows, 7, T, &Tend))
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
    constexpr int PER = 128 / (THREADS / 32); // rows per warp
    // loads of tile row rt: rows [src0, src0 + nvalid) x columns [c0, c0 +
    // 4*ntiles) of the source, zero past the group (all issued at once)
    auto issue = [&](int64_t rt, uint32_t (&v)[PER]) {
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
    };
    // this CTA's output tile rows: blockIdx.y, blockIdx.y + gridDim.y, ...;
    // the loads of the next one are in flight while the current one is stored
    uint32_t v[PER];
    if ((int64_t)blockIdx.y < cap_tile_rows)
        issue(blockIdx.y, v);
    for (int64_t rt = blockIdx.y; rt < cap_tile_rows; rt += gridDim.y) {
#pragma unroll
        for (int i = 0; i < PER; ++i)
            stage[(warp + i * (THREADS / 32)) * PITCH + lane] = v[i];
        __syncthreads();
        if (rt + gridDim.y < cap_tile_rows)
            issue(rt + gridDim.y, v);
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

// ---------------------------------------------------------------------------
// Groups along K: group g is the scale-column range [offs[g-1], offs[g]);
// each group's columns are padded to a multiple of 4 on their own and placed
// side by side from column 4*T[g] (T in tile columns); rows are padded to a
// multiple of 128; the (128*ceil(rows/128), cap_cols) matrix is written in
// the blocked layout, zero wherever no scale lands.
//
// A CTA owns a chunk of 32 output tile columns and a strided set of tile
// rows. The chunk's tile columns map to one contiguous run of at most 128
// source columns (the map is monotone and skips only padding), so each tile
// row stages 128 source rows of that run in shared memory (row pitch 33
// words: the per-lane reads below hit 32 distinct banks), and every tile is
// written as 32 contiguous 16-byte stores. A tile column's 4 source bytes sit
// at an arbitrary byte offset in the staged row and are extracted with a
// funnel shift.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(blk::THREADS, 4) k_blocked_grouped_k(const uint8_t *__restrict__ in, int64_t rows,
                                                                    int64_t cols, const int32_t *__restrict__ offs,
                                                                    int G, uint8_t *__restrict__ out,
                                                                    int32_t *__restrict__ starts_out, int words_ok,
                                                                    int64_t cap_cols)
{
    using namespace blk;
    extern __shared__ int T[]; // G entries
    __shared__ int Tend;
    __shared__ uint32_t stage[128 * PITCH];
    __shared__ int64_t tsrc[TILES]; // source column of each tile column's first byte
    __shared__ int tval[TILES];     // source bytes it holds (0..4)
    if (!padded_starts(offs, G, cols, 2, T, &Tend))
        return;
    const int64_t tiles_c = cap_cols / 4;
    const int64_t tc0 = (int64_t)blockIdx.x * TILES;
    const int ntiles = (int)min((int64_t)TILES, tiles_c - tc0);
    if (blockIdx.x == 0 && blockIdx.y == 0 && starts_out)
        for (int g = threadIdx.x; g < G; g += THREADS)
            starts_out[g] = T[g] * 4;
    if (ntiles <= 0)
        return;
    // the owning group of each tile column (largest g with T[g] <= tc; empty
    // groups share T with the next group, so it is non-empty)
    if (threadIdx.x < TILES) {
        const int64_t tc = tc0 + threadIdx.x;
        int64_t src = 0;
        int nv = 0;
        if (threadIdx.x < ntiles && tc < Tend) {
            int a = 0, b = G - 1;
            while (a < b) {
                const int m = (a + b + 1) >> 1;
                if (T[m] <= tc) a = m; else b = m - 1;
            }
            const int64_t gs = a ? offs[a - 1] : 0, ge = offs[a];
            src = gs + (tc - T[a]) * 4;
            nv = (int)min((int64_t)4, ge - src);
        }
        tsrc[threadIdx.x] = src;
        tval[threadIdx.x] = nv;
    }
    __syncthreads();
    // contiguous source run [s0, s1) of this chunk, staged from the word
    // boundary a0 = s0 & ~3 (at most 33 words per row)
    int first = -1, last = -1;
    for (int t = 0; t < ntiles; ++t)
        if (tval[t] > 0) {
            if (first < 0)
                first = t;
            last = t;
        }
    const int64_t s0 = first >= 0 ? tsrc[first] : 0;
    const int64_t s1 = first >= 0 ? tsrc[last] + tval[last] : 0;
    const int64_t a0 = s0 & ~int64_t(3);
    const int nwords = (int)((s1 - a0 + 3) / 4);
    const int64_t rows_p = (rows + 127) / 128 * 128;
    // loads of tile row rt: source rows rt*128.. x words [a0/4, a0/4 +
    // nwords), zero past the last row, staged word idx = row * PITCH + word;
    // thread t loads words t, t + THREADS, ... (all issued at once)
    constexpr int NW = 128 * PITCH;
    constexpr int PER = (NW + THREADS - 1) / THREADS;
    auto issue = [&](int64_t rt, uint32_t (&v)[PER]) {
        const int64_t r0 = rt * 128;
        const int nrows = (int)min((int64_t)128, rows - r0);
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int idx = threadIdx.x + i * THREADS;
            const int r = idx / PITCH, w = idx - r * PITCH;
            uint32_t x = 0;
            if (idx < NW && r < nrows && w < nwords) {
                const uint8_t *row = in + (r0 + r) * cols;
                const int64_t c = a0 + 4 * (int64_t)w;
                if (words_ok && c + 4 <= cols) {
                    x = __ldg(reinterpret_cast<const uint32_t *>(row + c));
                } else {
                    for (int j = 0; j < 4; ++j)
                        if (c + j < cols)
                            x |= (uint32_t)__ldg(row + c + j) << (8 * j);
                }
            }
            v[i] = x;
        }
    };
    // the loads of the next tile row are in flight while the current one is stored
    uint32_t v[PER];
    if ((int64_t)blockIdx.y * 128 < rows_p)
        issue(blockIdx.y, v);
    for (int64_t rt = blockIdx.y; rt * 128 < rows_p; rt += gridDim.y) {
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int idx = threadIdx.x + i * THREADS;
            if (idx < NW)
                stage[idx] = v[i];
        }
        __syncthreads();
        if ((rt + gridDim.y) * 128 < rows_p)
            issue(rt + gridDim.y, v);
        // tile t, 16-byte row j: source rows j, 32+j, 64+j, 96+j, four bytes
        // each from byte offset tsrc[t] - a0 of the staged row
        uint8_t *dst = out + (rt * tiles_c + tc0) * 512;
        for (int q = threadIdx.x; q < ntiles * 32; q += THREADS) {
            const int t = q >> 5, j = q & 31;
            const int nv = tval[t];
            uint32_t w4[4] = {0u, 0u, 0u, 0u};
            if (nv > 0) {
                const int b = (int)(tsrc[t] - a0);
                const int wi = b >> 2, sh = 8 * (b & 3);
                const uint32_t mask = nv >= 4 ? 0xFFFFFFFFu : ((1u << (8 * nv)) - 1u);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint32_t *row = stage + (32 * k + j) * PITCH;
                    const uint32_t lo = row[wi], hi = wi + 1 < 33 ? row[wi + 1] : 0u;
                    w4[k] = __funnelshift_r(lo, hi, sh) & mask;
                }
            }
            st_v4(dst + t * 512 + j * 16, w4[0], w4[1], w4[2], w4[3]);
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// MXFP8 1x32 rowwise quantization whose E8M0 scales go straight into the
// per-group (row groups) blocked layout: the rowwise op followed by the
// conversion above, without the scale matrix round trip through HBM.
//
// A warp walks rows; its two half-warps take alternate 128-element pieces of
// the row (4 MX blocks, one 16-byte load per lane). The four scale bytes of a
// piece are exactly one 4-byte word of the blocked layout (one row, one tile
// column), gathered by shuffles and written by one lane at the row's padded
// position in its group; bytes of blocks past the last column are zero.
// Output rows that hold no scale (each group's padding, everything past the
// last group) are zeroed by the same launch, word by word, so no byte is
// written twice.
// ---------------------------------------------------------------------------
constexpr int MXB_UNROLL = 4;

__global__ void __launch_bounds__(256) k_mx_1x32_blocked(const uint4 *__restrict__ in, int64_t rows, int64_t cols,
                                                         const int32_t *__restrict__ offs, int G,
                                                         uint2 *__restrict__ out, uint32_t *__restrict__ sb,
                                                         int32_t *__restrict__ starts_out, int64_t cap_rows, int mode)
{
    using namespace blk;
    extern __shared__ int T[]; // G entries, then the G offsets
    __shared__ int Tend;
    int *soffs = T + G;
    if (!padded_starts(offs, G, rows, 7, T, &Tend))
        return;
    for (int g = threadIdx.x; g < G; g += blockDim.x)
        soffs[g] = offs[g];
    if (blockIdx.x == 0 && starts_out)
        for (int g = threadIdx.x; g < G; g += blockDim.x)
            starts_out[g] = T[g] * 128;
    __syncthreads();
    const int lane = threadIdx.x & 31, half = lane >> 4, l16 = lane & 15;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t tcols = (cols + 127) / 128; // tile columns = scale words per row
    const int64_t end_all = soffs[G - 1];

    for (int64_t r = warp; r < rows; r += nwarps) {
        // padded output row of r in its group, or -1 past the last group
        int64_t rb = -1;
        if (r < end_all) {
            int a = 0, b = G - 1; // first group with end > r
            while (a < b) {
                const int m = (a + b) >> 1;
                if (soffs[m] > r) b = m; else a = m + 1;
            }
            rb = (int64_t)T[a] * 128 + (r - (a ? soffs[a - 1] : 0));
        }
        const uint4 *src = in + r * (cols / 8);
        uint2 *dst = out + r * (cols / 8);
        for (int64_t tb = 0; tb < tcols; tb += 2 * MXB_UNROLL) {
            uint4 v[MXB_UNROLL];
#pragma unroll
            for (int u = 0; u < MXB_UNROLL; ++u) {
                const int64_t e0 = (tb + 2 * u + half) * 128 + 8 * l16; // first element of this lane
                v[u] = e0 < cols ? ld_stream_v4(src + e0 / 8) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < MXB_UNROLL; ++u) {
                const int64_t tc = tb + 2 * u + half;
                const int64_t e0 = tc * 128 + 8 * l16;
                uint32_t acc = absmax_bf16x2(absmax_bf16x2(0u, v[u].x), v[u].y);
                acc = absmax_bf16x2(absmax_bf16x2(acc, v[u].z), v[u].w);
                float amax = absmax_of_pair(acc);
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
                const uint32_t byte = e0 < cols ? e8m0_mode(amax, mode) : 0u;
                const float f = mx_factor(byte);
                const int base = lane & 16;
                const uint32_t s0 = __shfl_sync(0xffffffffu, byte, base + 0);
                const uint32_t s1 = __shfl_sync(0xffffffffu, byte, base + 4);
                const uint32_t s2 = __shfl_sync(0xffffffffu, byte, base + 8);
                const uint32_t s3 = __shfl_sync(0xffffffffu, byte, base + 12);
                if (e0 < cols)
                    st_v2(dst + e0 / 8, quant4(v[u].x, v[u].y, f), quant4(v[u].z, v[u].w, f));
                if (l16 == 0 && rb >= 0 && tc < tcols) {
                    const int64_t w = ((rb >> 7) * tcols + tc) * 128 + (rb & 31) * 4 + ((rb >> 5) & 3);
                    sb[w] = s0 | (s1 << 8) | (s2 << 16) | (s3 << 24);
                }
            }
        }
    }

    // zero the output rows that hold no scale
    for (int64_t rb = warp; rb < cap_rows; rb += nwarps) {
        bool pad = true;
        const int64_t trow = rb >> 7;
        if (trow < Tend) {
            int a = 0, b = G - 1; // largest g with T[g] <= trow
            while (a < b) {
                const int m = (a + b + 1) >> 1;
                if (T[m] <= trow) a = m; else b = m - 1;
            }
            const int64_t size = soffs[a] - (a ? soffs[a - 1] : 0);
            pad = rb - (int64_t)T[a] * 128 >= size;
        }
        if (pad)
            for (int64_t tc = lane; tc < tcols; tc += 32)
                sb[((trow * tcols + tc) * 128) + (rb & 31) * 4 + ((rb >> 5) & 3)] = 0u;
    }
}

} // namespace mxq

