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
// Two kernels:
//   k_jagged_generic  any strides: one warp per (line, group), two passes
//                     over the group's elements (amax, then cast).
//   k_jagged_fused    contiguous lines: a single pass in one cooperative
//                     launch. Each CTA owns a fixed range of positions and
//                     walks the lines in rounds of 64. Per round it TMA-loads
//                     its (positions x 64 lines) slab into shared memory
//                     (a 3-stage ring), reduces the per-(group, line) amax of
//                     its rows and merges it into a global amax table with
//                     atomicMax on the fp32 bit pattern (exact and order-free
//                     for non-negative values), then arrives on the round's
//                     counter. One round later (so the wait overlaps the next
//                     round's loads and reduction) it waits for all CTAs,
//                     reads the final amax of its groups, casts the slab it
//                     still holds in shared memory and writes the transpose
//                     through a 64B-swizzled staging buffer with TMA stores.
//                     HBM traffic is the algorithmic 2 B read + 1 B written
//                     per element; skewed or empty groups only change how
//                     many rows of a CTA's range fall in each group.
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
// Generic path: any strides. One warp per (line, group).
// ---------------------------------------------------------------------------
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
        float amax = 0.0f;
        for (int64_t p = p0 + lane; p < p1; p += 32)
            amax = fmaxf(amax, fabsf(bf16_lo(src[p * s_pos])));
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1)
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const float s = fp8_scale(amax);
        if (lane == 0)
            inv[(int64_t)g * L + l] = fp8_inv(s);
        uint8_t *dst = out + l * P;
        for (int64_t p = p0 + lane; p < p1; p += 32)
            dst[p] = (uint8_t)e4m3x2(__fmul_rn(bf16_lo(src[p * s_pos]), s), 0.0f);
    }
}

// ---------------------------------------------------------------------------
// Single-pass cooperative path (contiguous lines).
// ---------------------------------------------------------------------------
namespace jag {

constexpr int W = 64;                 // lines per round (128 B of bf16 per position)
constexpr int CWARPS = 8;             // consumer warps
constexpr int THREADS = (CWARPS + 1) * 32;
constexpr int BOXP = 32;              // positions per TMA load box
constexpr int OBOX = 64;              // positions per TMA store box (64 B, 64B swizzle)
constexpr int MAX_SEG = 64;           // groups a CTA's range may intersect (host checks G)

struct Params {
    int64_t L, P;          // lines, positions
    int G;
    int chunk;             // positions per CTA (multiple of OBOX)
    int stages;            // TMA ring depth
    int rounds;            // ceil(L / W)
    int nseg_cap;          // segment-table capacity (>= min(G, ...))
    const int32_t *offs;
    uint8_t *out;          // out[l * P + p]
    float *inv;
    unsigned *amax;        // workspace: G * L fp32 bit patterns, zeroed
    int *counters;         // workspace: rounds ints, zeroed
    uint64_t wait_ns;
    int skip_arrival;      // test hook
};

// shared memory carve-up (byte offsets from a 1024-aligned base)
struct Layout {
    int in_off, in_stage_bytes;
    int stg_off;           // output staging: chunk/64 boxes of 64 x 64 bytes
    int stab_off;          // scale table: nseg_cap x W floats
    int red_off;           // CWARPS x 32 words
    int bar_off;           // full[stages], empty[stages]
    int misc_off;          // small ints
    int total;
};

__host__ __device__ inline Layout layout(int chunk, int stages, int nseg_cap)
{
    Layout y;
    y.in_off = 0;
    y.in_stage_bytes = chunk * W * 2;
    y.stg_off = stages * y.in_stage_bytes;               // multiple of 1024 (chunk % 64 == 0)
    y.stab_off = y.stg_off + chunk * W;
    y.red_off = y.stab_off + nseg_cap * W * 4;
    y.bar_off = y.red_off + CWARPS * 32 * 4;
    y.misc_off = y.bar_off + 2 * stages * 8;
    y.total = y.misc_off + 64;
    return y;
}

struct Misc {
    int nseg;              // non-empty group segments of this CTA's range
    int abort_flag;
    int seg_g[MAX_SEG];    // group of each segment
    int seg_lo[MAX_SEG];   // segment rows, relative to the range start
    int seg_hi[MAX_SEG];
};

} // namespace jag

__global__ void __launch_bounds__(jag::THREADS, 1)
    k_jagged_fused(const __grid_constant__ CUtensorMap tm_in, const __grid_constant__ CUtensorMap tm_out,
                   const jag::Params p)
{
    using namespace jag;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const Layout y = layout(p.chunk, p.stages, p.nseg_cap);
    uint8_t *in_s = base + y.in_off;
    uint8_t *stg = base + y.stg_off;
    float *stab = reinterpret_cast<float *>(base + y.stab_off);
    uint32_t *red = reinterpret_cast<uint32_t *>(base + y.red_off);
    uint64_t *full = reinterpret_cast<uint64_t *>(base + y.bar_off);
    uint64_t *empty = full + p.stages;
    __shared__ Misc mi;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ncta = gridDim.x;
    const int64_t lo = (int64_t)blockIdx.x * p.chunk;
    // offsets are validated by every CTA identically, so all of them return
    // together on bad offsets and no barrier is left waiting
    if (!offsets_ok(p.offs, p.G, p.P))
        return;
    const int64_t end_all = p.offs[p.G - 1];
    const int64_t hi = min(lo + (int64_t)p.chunk, end_all); // rows this CTA quantizes

    if (threadIdx.x == 0) {
        // segments: the non-empty groups intersecting [lo, hi), in order,
        // each clipped to the range; together they tile [lo, hi)
        int n = 0;
        if (hi > lo) {
            int a = 0, b = p.G - 1; // first group with end > lo
            while (a < b) {
                const int m = (a + b) >> 1;
                if (p.offs[m] > lo) b = m; else a = m + 1;
            }
            for (int g = a; g < p.G; ++g) {
                const int64_t gs = g ? p.offs[g - 1] : 0, ge = p.offs[g];
                if (gs >= hi)
                    break;
                if (ge == gs)
                    continue;
                if (n < MAX_SEG) {
                    mi.seg_g[n] = g;
                    mi.seg_lo[n] = (int)(max(gs, lo) - lo);
                    mi.seg_hi[n] = (int)(min(ge, hi) - lo);
                }
                ++n;
            }
        }
        mi.nseg = n;
        mi.abort_flag = 0;
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], CWARPS);
        }
        fence_mbar_init();
    }
    __syncthreads();
    // nseg <= G <= nseg_cap <= MAX_SEG: the host only takes this path then
    
    const int nseg = mi.nseg;
    const int R = p.rounds;
    const int nbox = p.chunk / BOXP;
    const uint32_t stage_bytes = (uint32_t)y.in_stage_bytes;

    if (warp == CWARPS) {
        // ------------------------------------------------ producer warp
        if (lane == 0) {
            int r = 0;
            for (; r < R; ++r) {
                const int s = r % p.stages;
                const uint32_t ph = (uint32_t)(r / p.stages) & 1u;
                if (r >= p.stages && !mbar_wait(&empty[s], ph ^ 1u, p.wait_ns))
                    break;
                mbar_arrive_expect_tx(&full[s], stage_bytes);
                uint8_t *dst = in_s + (size_t)s * stage_bytes;
                for (int b = 0; b < nbox; ++b)
                    tma_load_2d(dst + b * BOXP * W * 2, &tm_in, &full[s], r * W, (int)(lo + b * BOXP));
            }
            for (int j = r - p.stages; j < r; ++j)
                if (j >= 0)
                    mbar_wait(&full[j % p.stages], (uint32_t)(j / p.stages) & 1u, p.wait_ns);
        }
        return;
    }

    // ---------------------------------------------------- consumer warps
    const int ctid = threadIdx.x;              // 0 .. CWARPS*32-1
    const int NC = CWARPS * 32;
    const int64_t L = p.L;
    for (int r = 0; r <= R; ++r) {
        // ---- phase 1 of round r: per-(group, line) amax of this CTA's rows
        if (r < R) {
            const int s = r % p.stages;
            const uint32_t ph = (uint32_t)(r / p.stages) & 1u;
            bool ok = mbar_wait(&full[s], ph, p.wait_ns);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok)
                mi.abort_flag = 1;
            const uint32_t *slab = reinterpret_cast<const uint32_t *>(in_s + (size_t)s * stage_bytes);
            const int64_t l0 = (int64_t)r * W + 2 * lane; // this lane's line pair
            for (int sg = 0; sg < nseg; ++sg) {
                const int a = mi.seg_lo[sg], b = mi.seg_hi[sg];
                uint32_t acc = 0;
                int i = a + warp;
                for (; i + 3 * CWARPS < b; i += 4 * CWARPS) {
                    const uint32_t x0 = slab[(i + 0 * CWARPS) * 32 + lane];
                    const uint32_t x1 = slab[(i + 1 * CWARPS) * 32 + lane];
                    const uint32_t x2 = slab[(i + 2 * CWARPS) * 32 + lane];
                    const uint32_t x3 = slab[(i + 3 * CWARPS) * 32 + lane];
                    acc = absmax_bf16x2(absmax_bf16x2(acc, x0), x1);
                    acc = absmax_bf16x2(absmax_bf16x2(acc, x2), x3);
                }
                for (; i < b; i += CWARPS)
                    acc = absmax_bf16x2(acc, slab[i * 32 + lane]);
                red[warp * 32 + lane] = acc;
                named_barrier(1, NC);
                if (ctid < 32) {
                    uint32_t m = red[ctid];
                    for (int k = 1; k < CWARPS; ++k)
                        m = absmax_bf16x2(m, red[k * 32 + ctid]);
                    const int g = mi.seg_g[sg];
                    unsigned *dst = p.amax + (int64_t)g * L;
                    // skip lines past L; an amax of 0 never changes the table
                    const float a0 = bf16_lo(m), a1 = bf16_hi(m);
                    if (l0 < L && a0 > 0.0f)
                        atomicMax(dst + l0, __float_as_uint(a0));
                    if (l0 + 1 < L && a1 > 0.0f)
                        atomicMax(dst + l0 + 1, __float_as_uint(a1));
                }
                named_barrier(1, NC);
            }
            if (ctid == 0 && !(p.skip_arrival && blockIdx.x == 0)) {
                __threadfence();
                red_release_gpu_add(p.counters + r, 1);
            }
        }
        // ---- phase 2 of round r-1: wait for every CTA, cast, store
        if (r >= 1) {
            const int rr = r - 1;
            const int s = rr % p.stages;
            if (ctid == 0) {
                bulk_wait_read<0>(); // staging free again
                const uint64_t t0 = globaltimer();
                while (ld_acquire_gpu(p.counters + rr) < ncta) {
                    if (globaltimer() - t0 > p.wait_ns) {
                        set_status(MXQ_ERR_TIMEOUT);
                        mi.abort_flag = 1;
                        break;
                    }
                }
            }
            named_barrier(1, NC);
            if (mi.abort_flag)
                break;
            // scale table for this round's lines
            for (int t = ctid; t < nseg * W; t += NC) {
                const int sg = t / W, li = t % W;
                const int64_t l = (int64_t)rr * W + li;
                float s = 0.0f;
                if (l < L)
                    s = fp8_scale(__uint_as_float(__ldcg(p.amax + (int64_t)mi.seg_g[sg] * L + l)));
                stab[sg * W + li] = s;
            }
            // inverse scales of the groups this CTA is responsible for
            for (int g = blockIdx.x; g < p.G; g += ncta) {
                for (int li = ctid; li < W; li += NC) {
                    const int64_t l = (int64_t)rr * W + li;
                    if (l < L)
                        p.inv[(int64_t)g * L + l] = fp8_inv(fp8_scale(__uint_as_float(__ldcg(p.amax + (int64_t)g * L + l))));
                }
            }
            named_barrier(1, NC);

            // cast: a task is 16 positions x this lane's 2 lines
            const uint32_t *slab = reinterpret_cast<const uint32_t *>(in_s + (size_t)s * stage_bytes);
            const int64_t rows_here = hi - lo; // may be <= 0
            const int ntask16 = rows_here > 0 ? (int)((rows_here + 15) / 16) : 0;
            const int64_t l0 = (int64_t)rr * W + 2 * lane;
            const uint32_t stg_base = smem_u32(stg);
            const int bsel = (lane >> 2) & 1;
            // boxes that end at or before end_all use TMA; the one that
            // straddles end_all is written directly
            const int full_boxes = (int)((hi - lo) / OBOX);
            for (int t16 = warp; t16 < ntask16; t16 += CWARPS) {
                const int i0 = t16 * 16;
                // group segment of each row: find the segment of row i0
                int sg = 0;
                while (sg + 1 < nseg && mi.seg_hi[sg] <= i0)
                    ++sg;
                const bool one_seg = mi.seg_hi[sg] >= min((int64_t)i0 + 16, rows_here);
                uint32_t o0[4], o1[4];
                if (one_seg) {
                    const float s0 = stab[sg * W + 2 * lane], s1 = stab[sg * W + 2 * lane + 1];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint32_t x0 = slab[(i0 + 4 * k + 0) * 32 + lane];
                        const uint32_t x1 = slab[(i0 + 4 * k + 1) * 32 + lane];
                        const uint32_t x2 = slab[(i0 + 4 * k + 2) * 32 + lane];
                        const uint32_t x3 = slab[(i0 + 4 * k + 3) * 32 + lane];
                        o0[k] = e4m3x2(__fmul_rn(bf16_lo(x0), s0), __fmul_rn(bf16_lo(x1), s0)) |
                                (e4m3x2(__fmul_rn(bf16_lo(x2), s0), __fmul_rn(bf16_lo(x3), s0)) << 16);
                        o1[k] = e4m3x2(__fmul_rn(bf16_hi(x0), s1), __fmul_rn(bf16_hi(x1), s1)) |
                                (e4m3x2(__fmul_rn(bf16_hi(x2), s1), __fmul_rn(bf16_hi(x3), s1)) << 16);
                    }
                } else {
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        uint32_t a0 = 0, a1 = 0;
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int i = i0 + 4 * k + j;
                            int sj = sg;
                            while (sj + 1 < nseg && mi.seg_hi[sj] <= i)
                                ++sj;
                            const float s0 = stab[sj * W + 2 * lane], s1 = stab[sj * W + 2 * lane + 1];
                            const uint32_t x = slab[i * 32 + lane];
                            a0 |= e4m3x2(__fmul_rn(bf16_lo(x), s0), 0.0f) << (8 * j);
                            a1 |= e4m3x2(__fmul_rn(bf16_hi(x), s1), 0.0f) << (8 * j);
                        }
                        o0[k] = a0;
                        o1[k] = a1;
                    }
                }
                const int box = i0 / OBOX;
                if (box < full_boxes) {
                    // staging box: 64 lines x 64 bytes, 16-byte chunk c of
                    // line l stored at chunk c ^ ((l >> 1) & 3) (64B swizzle)
                    const uint32_t bbase = stg_base + box * (OBOX * W);
                    const int c = (i0 % OBOX) / 16;
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const int b = bsel ^ j;
                        const int line = 2 * lane + b;
                        const int pc = c ^ ((line >> 1) & 3);
                        const uint4 val = b ? make_uint4(o1[0], o1[1], o1[2], o1[3])
                                            : make_uint4(o0[0], o0[1], o0[2], o0[3]);
                        sts_v4(bbase + line * OBOX + pc * 16, val);
                    }
                } else {
                    // the box holding end_all: direct byte stores of rows below hi
#pragma unroll
                    for (int b = 0; b < 2; ++b) {
                        const int64_t l = l0 + b;
                        if (l >= L)
                            continue;
                        uint8_t *dst = p.out + l * p.P + lo + i0;
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const uint32_t word = b ? o1[j >> 2] : o0[j >> 2];
                            if (lo + i0 + j < hi)
                                dst[j] = (uint8_t)(word >> (8 * (j & 3)));
                        }
                    }
                }
            }
            fence_proxy_async_smem();
            named_barrier(1, NC);
            // release the input stage and store the full boxes
            if (lane == 0)
                mbar_arrive(&empty[s]);
            if (ctid == 0) {
                for (int bx = 0; bx < full_boxes; ++bx)
                    tma_store_2d(&tm_out, stg + bx * (OBOX * W), (int)(lo + bx * OBOX), rr * W);
                bulk_commit();
            }
        }
    }
    if (threadIdx.x == 0)
        bulk_wait<0>();
}

} // namespace mxq
