// jagged.cuh - float8 e4m3 quantization with per-group ("jagged") scales
// (ao PR 2064 "[scaled grouped mm] add triton kernels for float8 rowwise
// quantization with per-group/jagged scales", Motivation and Summary). Group
// boundaries come from a device-resident int32 offsets tensor and are never
// copied to the host.
//
// Both public ops reduce to one problem. Call the dimension that carries a
// scale a "line" and the grouped dimension a "position":
//   rowwise on (rows, cols):  line = row,    position = column
//   colwise on (rows, cols):  line = column, position = row
// For every (group g, line l): amax over the group's positions, s = 448 /
// max(amax, 1e-12), out[l * P + p] = e4m3(x(l, p) * s), inv[g * L + l] = 1/s.
// When lines are contiguous in memory (the transposed view of grad_out for
// rowwise, a row-major input for colwise) the op reads position-major rows
// and writes their transpose.
//
// Kernels:
//   k_jagged_generic  any strides, small problems: one warp per (line, group),
//                     the group read into registers, reduced, then cast.
//   k_jagged_rows     positions contiguous (rowwise on a row-major matrix):
//                     one warp per line, 16-byte loads, two passes per group.
//   k_jagged_amax +   contiguous lines, two streaming passes. The amax pass
//   k_jagged_cast     runs warp workers, each owning 256 lines (16 bytes per
//                     lane per row) and an equal run of positions, keeping 16
//                     rows of loads in flight and merging its maxima into a
//                     global (G, L) fp32 table by atomicMax only at group ends.
//                     The cast pass has the MX 3-D kernel's structure: a TMA
//                     ring of 128 x 64 tiles, one consumer warp per 32-row
//                     block, scales from the finished table, and the
//                     transpose leaving through a 128B-swizzled staging tile
//                     and TMA stores; its tile indices are 32-bit (64-bit
//                     divisions per tile cost it a fifth of its speed). The
//                     input is read twice (5 B of HBM traffic per element
//                     instead of 3); in exchange neither kernel synchronizes
//                     across CTAs.
#pragma once

#include "common.cuh"

namespace mxq {

// Validate offsets on the device: every thread of the block takes part and
// learns the verdict. Bad offsets record MXQ_ERR_BAD_OFFSETS.
MXQ_DEV bool offsets_ok(const int32_t *__restrict__ offs, int G, int64_t extent)
{
    int bad = 0;
    for (int g = threadIdx.x; g < G; g += blockDim.x) {
        const int64_t cur = offs[g];
        const int64_t prev = g ? (int64_t)offs[g - 1] : 0;
        if (cur < prev || cur > extent || cur < 0)
            bad = 1;
    }
    bad = __syncthreads_or(bad);
    if (bad && threadIdx.x == 0)
        set_status(MXQ_ERR_BAD_OFFSETS);
    return !bad;
}

// ---------------------------------------------------------------------------
// Generic path: any strides. One warp per (line, group). A group of up to
// 32 * GB positions is read once, all loads issued together, and kept in
// registers for the cast; longer groups take two batched passes. Latency,
// not bandwidth, bounds the small problems this path serves.
// ---------------------------------------------------------------------------
constexpr int GB = 8; // positions per lane per batch

__global__ void __launch_bounds__(256) k_jagged_generic(const uint16_t *__restrict__ in, int64_t L, int64_t P,
                                                        int64_t s_line, int64_t s_pos,
                                                        const int32_t *__restrict__ offs, int G,
                                                        uint8_t *__restrict__ out, float *__restrict__ inv)
{
    if (!offsets_ok(offs, G, P))
        return;
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t tasks = L * G;
    for (int64_t task = warp; task < tasks; task += nwarps) {
        const int64_t l = task / G;
        const int g = (int)(task - l * G);
        const int64_t p0 = g ? offs[g - 1] : 0, p1 = offs[g];
        const uint16_t *src = in + l * s_line;
        uint8_t *dst = out + l * P;
        float v[GB];
        float amax = 0.0f;
        const bool one_batch = p1 - p0 <= 32 * GB;
        for (int64_t b0 = p0; b0 < p1; b0 += 32 * GB) {
#pragma unroll
            for (int i = 0; i < GB; ++i) {
                const int64_t p = b0 + lane + 32 * i;
                v[i] = p < p1 ? bf16_lo(__ldg(src + p * s_pos)) : 0.0f;
            }
#pragma unroll
            for (int i = 0; i < GB; ++i)
                amax = fmaxf(amax, fabsf(v[i]));
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1)
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const float s = fp8_scale(amax);
        if (lane == 0)
            inv[(int64_t)g * L + l] = fp8_inv(s);
        if (one_batch) {
#pragma unroll
            for (int i = 0; i < GB; ++i) {
                const int64_t p = p0 + lane + 32 * i;
                if (p < p1)
                    dst[p] = (uint8_t)e4m3x2(__fmul_rn(v[i], s), 0.0f);
            }
        } else {
            for (int64_t b0 = p0; b0 < p1; b0 += 32 * GB) {
#pragma unroll
                for (int i = 0; i < GB; ++i) {
                    const int64_t p = b0 + lane + 32 * i;
                    v[i] = p < p1 ? bf16_lo(__ldg(src + p * s_pos)) : 0.0f;
                }
#pragma unroll
                for (int i = 0; i < GB; ++i) {
                    const int64_t p = b0 + lane + 32 * i;
                    if (p < p1)
                        dst[p] = (uint8_t)e4m3x2(__fmul_rn(v[i], s), 0.0f);
                }
            }
        }
    }
}


// ---------------------------------------------------------------------------
// Positions contiguous (stride 1 along the grouped dimension, e.g. rowwise on
// a row-major matrix): one warp per line. For each group in turn the warp
// reads the group's run of the line with 16-byte loads (8 elements per lane,
// elements outside the group masked in the two boundary vectors), reduces the
// amax, then reads the run again (now in L1/L2), casts, and writes 8 bytes per
// lane; a vector that straddles a group end is written byte by byte, so each
// byte is written by exactly one group's pass. Needs 16-byte aligned lines
// (base and line stride) and an 8-byte aligned output with P % 8 == 0.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_jagged_rows(const uint16_t *__restrict__ in, int64_t L, int64_t P,
                                                     int64_t s_line, const int32_t *__restrict__ offs, int G,
                                                     uint8_t *__restrict__ out, float *__restrict__ inv)
{
    if (!offsets_ok(offs, G, P))
        return;
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t l = warp; l < L; l += nwarps) {
        const uint16_t *src = in + l * s_line;
        uint8_t *dst = out + l * P;
        int64_t s = 0;
        for (int g = 0; g < G; ++g) {
            const int64_t e = offs[g];
            // vectors of 8 covering [s, e), from the 8-aligned position at or below s
            const int64_t v0 = s & ~int64_t(7);
            uint32_t acc = 0;
#pragma unroll 4
            for (int64_t p = v0 + 8 * lane; p < e; p += 256) {
                uint4 v = *reinterpret_cast<const uint4 *>(src + p);
                if (p < s || p + 8 > e) { // boundary vector: drop elements outside [s, e)
                    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        if (p + j < s || p + j >= e)
                            w[j >> 1] &= (j & 1) ? 0x0000FFFFu : 0xFFFF0000u;
                    v = make_uint4(w[0], w[1], w[2], w[3]);
                }
                acc = absmax_bf16x2(absmax_bf16x2(acc, v.x), v.y);
                acc = absmax_bf16x2(absmax_bf16x2(acc, v.z), v.w);
            }
            float amax = absmax_of_pair(acc);
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1)
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
            const float sc = fp8_scale(amax);
            if (lane == 0)
                inv[(int64_t)g * L + l] = fp8_inv(sc);
#pragma unroll 4
            for (int64_t p = v0 + 8 * lane; p < e; p += 256) {
                const uint4 v = *reinterpret_cast<const uint4 *>(src + p);
                const uint32_t q0 = quant4(v.x, v.y, sc), q1 = quant4(v.z, v.w, sc);
                if (p >= s && p + 8 <= e) {
                    st_v2(dst + p, q0, q1);
                } else {
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        if (p + j >= s && p + j < e)
                            dst[p + j] = (uint8_t)((j < 4 ? q0 : q1) >> (8 * (j & 3)));
                }
            }
            s = e;
        }
    }
}


// ---------------------------------------------------------------------------
// Two-pass path (contiguous lines): amax pass
// ---------------------------------------------------------------------------
namespace jag {

constexpr int MAX_SEG = 64; // groups the two-pass kernels accept (host checks G)

namespace amx {
constexpr int W = 256;       // lines per chunk: 16 bytes (8 lines) per lane
constexpr int BR = 16;       // rows per batch of loads in flight per lane
constexpr int THREADS = 256;
constexpr int CTAS_PER_SM = 2;
} // namespace amx

// first group whose end is > p (p < offs[G-1])
MXQ_DEV int group_of(const int *soffs, int G, int64_t p)
{
    int a = 0, b = G - 1;
    while (a < b) {
        const int m = (a + b) >> 1;
        if (soffs[m] > p) b = m; else a = m + 1;
    }
    return a;
}

} // namespace jag

// amax[g * L + l] = max |x| over group g's positions of line l, as fp32 bits
// (the table must be zero on entry).
//
// Workers are warps. Worker (c, j) owns lines [256c, 256c + 256), a lane
// owning eight adjacent lines (one 16-byte load per row), and the j-th of
// `wpc` equal runs of positions [0, offs[G-1]). It keeps 16 rows of loads in
// flight, reduces them with packed bf16 max while the batch lies in one
// group, and merges its running maxima into the table with atomicMax on the
// fp32 bit pattern (exact and order-free for non-negative values) only when
// its run crosses a group end and when it finishes.
__global__ void __launch_bounds__(jag::amx::THREADS, jag::amx::CTAS_PER_SM)
    k_jagged_amax(const uint16_t *__restrict__ in, int64_t L, int64_t P, int64_t s_pos,
                  const int32_t *__restrict__ offs, int G, int wpc, unsigned *__restrict__ amax)
{
    using namespace jag;
    using namespace jag::amx;
    __shared__ int soffs[MAX_SEG];
    if (!offsets_ok(offs, G, P))
        return;
    for (int g = threadIdx.x; g < G; g += blockDim.x)
        soffs[g] = offs[g];
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int64_t end_all = soffs[G - 1];
    const int64_t chunks = (L + W - 1) / W;
    const int64_t wid = ((int64_t)blockIdx.x * THREADS + threadIdx.x) >> 5;
    if (wid >= chunks * wpc)
        return;
    const int64_t c = wid % chunks, j = wid / chunks;
    const int64_t run = ((end_all + wpc - 1) / wpc + BR - 1) / BR * BR;
    int64_t r = j * run;
    const int64_t rend = min(end_all, r + run);
    if (r >= rend)
        return;
    const int64_t line0 = c * W + 8 * lane;
    const int nvalid = (int)max((int64_t)0, min((int64_t)8, L - line0)); // lines of this lane
    const uint16_t *src = in + line0;

    int g = group_of(soffs, G, r);
    int64_t gend = soffs[g];
    uint32_t acc[4] = {0u, 0u, 0u, 0u};
    auto flush = [&]() {
        unsigned *dst = amax + (int64_t)g * L + line0;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            if (2 * q < nvalid && (acc[q] & 0xFFFFu))
                atomicMax(dst + 2 * q, acc[q] << 16);
            if (2 * q + 1 < nvalid && (acc[q] >> 16))
                atomicMax(dst + 2 * q + 1, acc[q] & 0xFFFF0000u);
            acc[q] = 0u;
        }
    };
    for (; r < rend; r += BR) {
        uint4 v[BR];
#pragma unroll
        for (int k = 0; k < BR; ++k) {
            const int64_t row = r + k;
            v[k] = make_uint4(0u, 0u, 0u, 0u);
            if (row < rend) {
                const uint16_t *p = src + row * s_pos;
                if (nvalid == 8) {
                    v[k] = ld_stream_v4(reinterpret_cast<const uint4 *>(p));
                } else if (nvalid > 0) {
                    uint32_t w4[4] = {0u, 0u, 0u, 0u};
                    for (int i = 0; i < nvalid; ++i)
                        w4[i >> 1] |= (uint32_t)__ldg(p + i) << (16 * (i & 1));
                    v[k] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                }
            }
        }
        if (min(r + BR, rend) <= gend) {
            // the whole batch lies in group g (rows past rend read as zero)
#pragma unroll
            for (int k = 0; k < BR; ++k) {
                acc[0] = absmax_bf16x2(acc[0], v[k].x);
                acc[1] = absmax_bf16x2(acc[1], v[k].y);
                acc[2] = absmax_bf16x2(acc[2], v[k].z);
                acc[3] = absmax_bf16x2(acc[3], v[k].w);
            }
        } else {
#pragma unroll
            for (int k = 0; k < BR; ++k) {
                const int64_t row = r + k;
                if (row < rend) {
                    if (row >= gend) {
                        flush();
                        do {
                            ++g;
                        } while (row >= soffs[g]);
                        gend = soffs[g];
                    }
                    acc[0] = absmax_bf16x2(acc[0], v[k].x);
                    acc[1] = absmax_bf16x2(acc[1], v[k].y);
                    acc[2] = absmax_bf16x2(acc[2], v[k].z);
                    acc[3] = absmax_bf16x2(acc[3], v[k].w);
                }
            }
        }
    }
    flush();
}

// ---------------------------------------------------------------------------
// Two-pass path (contiguous lines): cast pass, the MX 3-D tile structure
// ---------------------------------------------------------------------------
namespace jag {
namespace cst {
constexpr int TP = 128;                 // positions per tile (four 32-row blocks)
constexpr int TL = 64;                  // lines per tile
constexpr int STAGES = 4;
constexpr int CWARPS = 4;               // one 32-row block each
constexpr int THREADS = (CWARPS + 1) * 32;
constexpr int IN_BYTES = TP * TL * 2;   // 16 KB
constexpr int OUT_BYTES = TP * TL;      // 8 KB
constexpr int CTAS_PER_SM = 2;

struct __align__(1024) Smem {
    uint8_t in[STAGES][IN_BYTES];
    uint8_t out[2][OUT_BYTES];
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    int offs[MAX_SEG];
    int abort_flag;
};
constexpr size_t SMEM_BYTES = sizeof(Smem) + 1024;
} // namespace cst
} // namespace jag

// out[l * P + p] = e4m3(x(l, p) * s(group(p), l)), s = 448 / max(amax, 1e-12)
// from the finished amax table; inv[g * L + l] = 1 / s (written by the first
// tiles_l CTAs). Rows past offs[G-1] are not written. A consumer warp owns a
// 32-row block of each tile. `drop_load`: test hook, CTA 0 never issues its
// first tile, so the bounded waits on it expire.
__global__ void __launch_bounds__(jag::cst::THREADS, jag::cst::CTAS_PER_SM)
    k_jagged_cast(const __grid_constant__ CUtensorMap tm_in, const __grid_constant__ CUtensorMap tm_out, int64_t L,
                  int64_t P, const int32_t *__restrict__ offs, int G, const unsigned *__restrict__ amax,
                  uint8_t *__restrict__ out, float *__restrict__ inv, uint64_t wait_ns, int drop_load)
{
    using namespace jag;
    using namespace jag::cst;
    extern __shared__ uint8_t smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (!offsets_ok(offs, G, P))
        return;
    const int64_t end_all = offs[G - 1];
    // tile t = (position tile t / tiles_l, line tile t % tiles_l); the host
    // guarantees fewer than 2^31 tiles, so tile arithmetic is 32-bit
    const uint32_t tiles_p = (uint32_t)((end_all + TP - 1) / TP), tiles_l = (uint32_t)((L + TL - 1) / TL);
    const uint32_t total = tiles_p * tiles_l;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], CWARPS);
        }
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    for (int g = threadIdx.x; g < G; g += blockDim.x)
        sm.offs[g] = offs[g];
    __syncthreads();

    // inverse scales of every (group, line), empty groups included
    for (uint32_t lt = blockIdx.x; lt < tiles_l; lt += gridDim.x)
        for (int i = threadIdx.x; i < G * TL; i += blockDim.x) {
            const int g = i / TL;
            const int64_t l = (int64_t)lt * TL + (i % TL);
            if (l < L)
                inv[(int64_t)g * L + l] = fp8_inv(fp8_scale(__uint_as_float(__ldg(amax + (int64_t)g * L + l))));
        }

    if (warp == CWARPS) {
        // ------------------------------------------------ producer warp
        if (lane == 0) {
            int it = 0;
            for (uint32_t t = blockIdx.x; t < total; t += gridDim.x, ++it) {
                const int s = it % STAGES;
                if (it >= STAGES && !mbar_wait(&sm.empty[s], ((uint32_t)(it / STAGES) & 1u) ^ 1u, wait_ns))
                    break;
                if (drop_load && blockIdx.x == 0 && it == 0)
                    continue; // test hook: this tile never arrives
                const uint32_t pt = t / tiles_l, lt = t - pt * tiles_l;
                mbar_arrive_expect_tx(&sm.full[s], IN_BYTES);
                tma_load_2d(sm.in[s], &tm_in, &sm.full[s], (int)(lt * TL), (int)(pt * TP));
            }
            // drain: every issued fill lands before the CTA exits
            for (int j = it - STAGES; j < it; ++j)
                if (j >= 0 && !(drop_load && blockIdx.x == 0 && j == 0))
                    mbar_wait(&sm.full[j % STAGES], (uint32_t)(j / STAGES) & 1u, wait_ns);
        }
        return;
    }

    // ---------------------------------------------------- consumer warps
    const int w = warp; // rows 32w .. 32w+31 of the tile
    bool prev_stored = true;
    int it = 0;
    for (uint32_t t = blockIdx.x; t < total; t += gridDim.x, ++it) {
        const int s = it % STAGES;
        const int ob = it & 1;
        const uint32_t pt = t / tiles_l, lt = t - pt * tiles_l;
        const int64_t p0 = (int64_t)pt * TP + 32 * w;   // this warp's first position
        const int64_t l0 = (int64_t)lt * TL + 2 * lane; // this lane's lines l0, l0+1
        // group of the block's first row and the amax words of the lane's
        // lines, loaded before the wait so their latency overlaps it
        const int g = group_of(sm.offs, G, p0);
        const unsigned *arow = amax + (int64_t)g * L;
        const uint32_t am0 = l0 < L ? __ldg(arow + l0) : 0u;
        const uint32_t am1 = l0 + 1 < L ? __ldg(arow + l0 + 1) : 0u;
        bool ok = mbar_wait(&sm.full[s], (uint32_t)(it / STAGES) & 1u, wait_ns);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok)
            sm.abort_flag = 1;
        const uint32_t *tile = reinterpret_cast<const uint32_t *>(sm.in[s]);
        uint32_t v[32];
        uint32_t dep = 0;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            v[i] = tile[(w * 32 + i) * (TL / 2) + lane];
            dep ^= v[i];
        }
        release_slot_after(&sm.empty[s], dep);

        uint32_t q0[8], q1[8]; // lines l0, l0+1: 32 position bytes each
        if (p0 < end_all && (int64_t)sm.offs[g] >= p0 + 32) {
            // the block lies in one group
            const float s0 = fp8_scale(__uint_as_float(am0)), s1 = fp8_scale(__uint_as_float(am1));
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t *r = v + 4 * j;
                q0[j] = e4m3x2(__fmul_rn(bf16_lo(r[0]), s0), __fmul_rn(bf16_lo(r[1]), s0)) |
                        (e4m3x2(__fmul_rn(bf16_lo(r[2]), s0), __fmul_rn(bf16_lo(r[3]), s0)) << 16);
                q1[j] = e4m3x2(__fmul_rn(bf16_hi(r[0]), s1), __fmul_rn(bf16_hi(r[1]), s1)) |
                        (e4m3x2(__fmul_rn(bf16_hi(r[2]), s1), __fmul_rn(bf16_hi(r[3]), s1)) << 16);
            }
        } else {
            // the block crosses group ends (or offs[G-1]): per-row group,
            // the scales reloaded only where the group changes
            auto scale_of = [&](int grp, int64_t l) {
                return l < L ? fp8_scale(__uint_as_float(__ldg(amax + (int64_t)grp * L + l))) : 0.0f;
            };
            int gg = g;
            float s0 = fp8_scale(__uint_as_float(am0)), s1 = fp8_scale(__uint_as_float(am1));
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                uint32_t a0 = 0, a1 = 0;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int64_t row = p0 + 4 * j + k;
                    if (gg + 1 < G && (int64_t)sm.offs[gg] <= row) {
                        do {
                            ++gg;
                        } while (gg + 1 < G && (int64_t)sm.offs[gg] <= row);
                        s0 = scale_of(gg, l0);
                        s1 = scale_of(gg, l0 + 1);
                    }
                    const uint32_t x = v[4 * j + k];
                    a0 |= e4m3x2(__fmul_rn(bf16_lo(x), s0), 0.0f) << (8 * k);
                    a1 |= e4m3x2(__fmul_rn(bf16_hi(x), s1), 0.0f) << (8 * k);
                }
                q0[j] = a0;
                q1[j] = a1;
            }
        }

        // a tile wholly below offs[G-1] leaves through the staging tile and a
        // TMA store; the tile holding offs[G-1] is written directly
        const bool full_tile = (int64_t)pt * TP + TP <= end_all;
        // staging buffer ob was read by the store of tile it-2; when tile
        // it-1 issued no store, that one may be the newest group
        if (threadIdx.x == 0) {
            if (prev_stored)
                bulk_wait_read<1>();
            else
                bulk_wait_read<0>();
        }
        named_barrier(1, CWARPS * 32);
        if (full_tile) {
            // staging: 64 rows (lines) x 128 bytes (positions), 16-byte chunk c
            // of row r at chunk c ^ (r & 7) (128B swizzle); the lane's two
            // lines alternate so each 16-byte store hits 8 bank groups
            const uint32_t ob_addr = smem_u32(sm.out[ob]);
            const int bsel = (lane >> 2) & 1;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int b = bsel ^ (j & 1), h = j >> 1;
                const int row = 2 * lane + b;
                const int chunk = (2 * w + h) ^ (row & 7);
                uint4 val;
                if (b) val = make_uint4(q1[4 * h], q1[4 * h + 1], q1[4 * h + 2], q1[4 * h + 3]);
                else   val = make_uint4(q0[4 * h], q0[4 * h + 1], q0[4 * h + 2], q0[4 * h + 3]);
                sts_v4(ob_addr + row * 128 + chunk * 16, val);
            }
            fence_proxy_async_smem();
        } else {
#pragma unroll
            for (int bb = 0; bb < 2; ++bb) {
                const int64_t l = l0 + bb;
                if (l >= L)
                    continue;
                uint8_t *dst = out + l * P + p0;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const uint32_t word = bb ? q1[j >> 2] : q0[j >> 2];
                    if (p0 + j < end_all)
                        dst[j] = (uint8_t)(word >> (8 * (j & 3)));
                }
            }
        }
        if (barrier_or(1, CWARPS * 32, sm.abort_flag != 0))
            break;
        if (threadIdx.x == 0 && full_tile) {
            tma_store_2d(&tm_out, sm.out[ob], (int)(pt * TP), (int)(lt * TL));
            bulk_commit();
        }
        prev_stored = full_tile;
    }
    if (threadIdx.x == 0)
        bulk_wait<0>();
}

} // namespace mxq
