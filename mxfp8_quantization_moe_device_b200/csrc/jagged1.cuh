// jagged1.cuh - single-read float8 e4m3 quantization with per-group
// ("jagged") scales (ao PR 2064 "[scaled grouped mm] add triton kernels for
// float8 rowwise quantization with per-group/jagged scales", Motivation and
// Summary: one kernel, group boundaries from device-resident offsets, no
// host sync).
//
// Same problem as jagged.cuh: lines are contiguous in memory, positions are
// the grouped dimension, and for every (group g, line l) the kernel computes
// amax over the group's positions, s = 448 / max(amax, 1e-12), writes
// out[l * P + p] = e4m3(x(l, p) * s) and inv[g * L + l] = 1 / s. Here every
// input element is read from HBM exactly once.
//
// Work decomposition. The input is cut into strips of 64 lines (128 bytes of
// every position row) and each strip's 128-position blocks into `ups` units
// of consecutive blocks (sizes differing by at most one block, at most
// MAX_UT blocks). When a strip has at least as many blocks as the grid has
// CTAs, ups equals the grid size, so every round of the grid works on
// exactly one strip; otherwise every block is a unit. A persistent
// cooperative grid (one CTA per SM) takes units in ticket order
// (strip-major): CTA c owns tickets c, c + grid, c + 2 grid...
// Each CTA loads a unit (TMA, 128 x 64 tiles) into its amax ring, reduces
// it and hands the slots straight back; once the amax of every group the
// unit touches is known, a second producer loads the unit again into the
// cast ring. The second load finds the tiles in L2: the units between their
// two loads are a few tens of MB across the GPU. Group maxima:
//   * a group that lies inside one unit is reduced locally;
//   * a group spanning several units of the strip: every unit stores its
//     64 partial maxima in a slot of its own (plain stores: units never
//     contend for one cache line) and adds 1 to the (group, strip) counter
//     with release semantics; each unit's merge waits (bounded, acquire)
//     until the counter reaches the number of units the group spans, then
//     takes the max over the group's slots. Slot (g, unit b) of a strip is
//     b + g: consecutive groups share at most their boundary unit, so the
//     slots of a strip's (group, unit) pairs never collide.
//   * a unit touching more than MAXG_U groups keeps the extra groups'
//     maxima in a global (G, L) table with atomicMax on the fp32 bits
//     (small groups, hence little contention).
// Because a strip's units are consecutive tickets and there are no more of
// them than CTAs, no CTA ever holds two units of one strip, and a unit's
// CTA has completed all its earlier units before it loads it; every merge
// therefore completes (no deadlock) as long as all CTAs are resident, which
// the cooperative launch guarantees.
//
// Warp roles in a CTA (512 threads):
//   warps 0-7   cast: two quads, quad q takes the cast ring's tiles of
//               parity q; one warp = 32 rows x 64 lines of a tile, a lane
//               two lines; codes leave through a 128B-swizzled staging tile
//               and a TMA store of the 64 x 128 transpose (plain stores for
//               the tile that holds offs[G-1]).
//   warps 8-9   amax: two 32-row blocks of every tile each, packed bf16 max,
//               partial maxima per group merged in a per-unit shared table.
//   warp 10     amax producer: the TMA loads of the amax ring.
//   warp 11     cast producer: a unit's TMA loads into the cast ring, once
//               its scales are ready.
//   warps 12-15 publish and merge, unit ku on warp 12 + ku % 4 (so four
//               units' exchanges overlap): store the maxima of the groups
//               the unit shares with other units in their global slots and
//               count them in; wait for those groups' counters, turn amax
//               into scales in the shared table, write inverse scales.
// Every wait is bounded by %globaltimer; on expiry the kernel records
// MXQ_ERR_TIMEOUT, stops, and drains its own copies in flight.
#pragma once

#include "common.cuh"
#include "jagged.cuh"

namespace mxq {
namespace jg1 {

constexpr int TP = 128;       // positions per tile
constexpr int TL = 64;        // lines per tile (one strip)
constexpr int RA = 7;         // amax ring (tiles)
constexpr int RC = 4;         // cast ring (tiles; even: slot parity = quad)
constexpr int MAX_UT = 4;     // tiles per unit (the host keeps units within this)
constexpr int UQ = 4;         // units between their two loads (per-unit scale tables)
constexpr int MAXG_U = 8;     // groups of a unit kept in the shared table
constexpr int CAST_WARPS = 8;
constexpr int AMAX_WARP0 = 8;   // two amax warps
constexpr int AMAX_WARPS = 2;
constexpr int PROD_WARP = 10;
constexpr int CPROD_WARP = 11;
constexpr int PM_WARP0 = 12;    // four publish-and-merge warps, unit ku to warp ku % 4
constexpr int PM_WARPS = 4;
constexpr int THREADS = 16 * 32;
constexpr int IN_BYTES = TP * TL * 2;  // 16 KB
constexpr int OUT_BYTES = TP * TL;     // 8 KB

struct __align__(1024) Smem {
    uint8_t in[RA][IN_BYTES];           // amax ring
    uint8_t cin[RC][IN_BYTES];          // cast ring
    uint8_t out[2][2][OUT_BYTES];       // [quad][buffer]
    uint32_t tab[UQ][MAXG_U][TL];       // amax bits, then fp32 scale bits
    uint32_t red[PM_WARPS][8][TL];      // merge: partial maxima of 8 slot subsets, per warp
    uint64_t full[RA];
    uint64_t empty[RA];
    uint64_t cfull[RC];
    uint64_t cempty[RC];
    uint64_t amax_computed[UQ];
    uint64_t scales_ready[UQ];
    uint64_t scales_free[UQ];
    int offs[jag::MAX_SEG];
    int abort_flag;
};
constexpr size_t SMEM_BYTES = sizeof(Smem) + 1024;

struct Unit {
    int s;       // strip
    int b;       // unit index in the strip
    int r0, r1;  // positions [r0, r1)
    int ntiles;
    int gf, gl;  // first and last group with positions in the unit
};

// unit b of a strip covers blocks [first_block(b), first_block(b + 1))
MXQ_DEV int first_block(int b, int ups, int blocks) { return (int)((int64_t)b * blocks / ups); }

// the unit holding position p (< end)
MXQ_DEV int unit_of_pos(int p, int ups, int blocks) { return (int)(((int64_t)(p / TP + 1) * ups - 1) / blocks); }

MXQ_DEV Unit unit_of(uint32_t ticket, int ups, int blocks, int end, const int *soffs, int G)
{
    Unit u;
    u.s = (int)(ticket / (uint32_t)ups);
    u.b = (int)(ticket - (uint32_t)u.s * (uint32_t)ups);
    u.r0 = first_block(u.b, ups, blocks) * TP;
    u.r1 = min(first_block(u.b + 1, ups, blocks) * TP, end);
    u.ntiles = (u.r1 - u.r0 + TP - 1) / TP;
    u.gf = jag::group_of(soffs, G, u.r0);
    u.gl = jag::group_of(soffs, G, u.r1 - 1);
    return u;
}

MXQ_DEV uint32_t ld_relaxed_gpu(const unsigned *p)
{
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

MXQ_DEV bool abort_set(const Smem &sm) { return *reinterpret_cast<const volatile int *>(&sm.abort_flag) != 0; }

MXQ_DEV void set_abort(Smem &sm) { *reinterpret_cast<volatile int *>(&sm.abort_flag) = 1; }

} // namespace jg1

// amax: zeroed (G, L) fp32-bit table; counters: zeroed (G, strips) ints;
// partials: (strips, pstride, 64) fp32 bits, pstride >= units per strip + G,
// no clearing needed. The host launches it only when ceil(P / 128) <=
// MAX_UT * gridDim.x.
__global__ void __launch_bounds__(jg1::THREADS, 1)
    k_jagged_single(const __grid_constant__ CUtensorMap tm_in, const __grid_constant__ CUtensorMap tm_out, int L,
                    int P, const int32_t *__restrict__ offs, int G, unsigned *__restrict__ amax,
                    int *__restrict__ counters, unsigned *__restrict__ partials, int pstride,
                    uint8_t *__restrict__ out, float *__restrict__ inv, uint64_t wait_ns, int drop_load)
{
    using namespace jg1;
    extern __shared__ uint8_t smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (!offsets_ok(offs, G, P))
        return;
    const int end = offs[G - 1];
    const int nstrips = (L + TL - 1) / TL;
    const int blocks = (end + TP - 1) / TP;
    const int ups = min(blocks, (int)gridDim.x); // units per strip (<= grid)
    const uint32_t total = (uint32_t)nstrips * (uint32_t)ups;
    if (threadIdx.x == 0) {
        for (int i = 0; i < RA; ++i) {
            mbar_init(&sm.full[i], 1);
            mbar_init(&sm.empty[i], AMAX_WARPS);
        }
        for (int i = 0; i < RC; ++i) {
            mbar_init(&sm.cfull[i], 1);
            mbar_init(&sm.cempty[i], 4); // the warps of one cast quad
        }
        for (int i = 0; i < UQ; ++i) {
            mbar_init(&sm.amax_computed[i], 1);
            mbar_init(&sm.scales_ready[i], 1);
            mbar_init(&sm.scales_free[i], CAST_WARPS);
        }
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    for (int g = threadIdx.x; g < G; g += blockDim.x)
        sm.offs[g] = offs[g];
    // inverse scales of empty groups (no unit covers them)
    for (int g = 0; g < G; ++g) {
        const int st = g ? offs[g - 1] : 0;
        if (offs[g] > st)
            continue;
        const float iv = fp8_inv(fp8_scale(0.0f));
        for (int l = blockIdx.x * blockDim.x + threadIdx.x; l < L; l += gridDim.x * blockDim.x)
            inv[(int64_t)g * L + l] = iv;
    }
    __syncthreads();
    const int *soffs = sm.offs;

    if (warp == PROD_WARP || warp == CPROD_WARP) {
        // ------------------------------------------------------ producers
        // amax producer: every unit's tiles, as slots free up; cast
        // producer: a unit's tiles again once its scales are ready
        const bool cast = warp == CPROD_WARP;
        const int R = cast ? RC : RA;
        uint8_t(*ring)[IN_BYTES] = cast ? sm.cin : sm.in;
        uint64_t *fullb = cast ? sm.cfull : sm.full;
        uint64_t *emptyb = cast ? sm.cempty : sm.empty;
        if (lane == 0) {
            int i = 0, ku = 0;
            bool stop = false;
            for (uint32_t t = blockIdx.x; t < total && !stop; t += gridDim.x, ++ku) {
                const Unit u = unit_of(t, ups, blocks, end, soffs, G);
                if (cast && !mbar_wait(&sm.scales_ready[ku % UQ], (uint32_t)(ku / UQ) & 1u, wait_ns)) {
                    set_abort(sm);
                    break;
                }
                for (int k = 0; k < u.ntiles; ++k, ++i) {
                    const int slot = i % R;
                    if (i >= R && !mbar_wait(&emptyb[slot], ((uint32_t)(i / R) & 1u) ^ 1u, wait_ns)) {
                        set_abort(sm);
                        stop = true;
                        break;
                    }
                    if (abort_set(sm)) {
                        stop = true;
                        break;
                    }
                    if (!cast && drop_load && blockIdx.x == 0 && i == 0)
                        continue; // test hook: this tile never arrives
                    mbar_arrive_expect_tx(&fullb[slot], IN_BYTES);
                    tma_load_2d(ring[slot], &tm_in, &fullb[slot], u.s * TL, u.r0 + k * TP);
                }
            }
            // drain: every issued fill lands before the CTA exits
            for (int j = i - R; j < i; ++j)
                if (j >= 0 && !(!cast && drop_load && blockIdx.x == 0 && j == 0))
                    mbar_wait(&fullb[j % R], (uint32_t)(j / R) & 1u, wait_ns);
        }
        return;
    }

    if (warp >= AMAX_WARP0 && warp < AMAX_WARP0 + AMAX_WARPS) {
        // ------------------------------------------------------ amax warps
        const int aw = warp - AMAX_WARP0;
        int i = 0, ku = 0;
        for (uint32_t t = blockIdx.x; t < total; t += gridDim.x, ++ku) {
            const Unit u = unit_of(t, ups, blocks, end, soffs, G);
            const int uq = ku % UQ;
            const bool ok = ku < UQ || mbar_wait(&sm.scales_free[uq], (uint32_t)(ku / UQ - 1) & 1u, wait_ns);
            if (barrier_or(3, AMAX_WARPS * 32, !ok || abort_set(sm))) {
                set_abort(sm);
                break;
            }
            uint32_t *tab = &sm.tab[uq][0][0];
            for (int x = aw * 32 + lane; x < MAXG_U * TL; x += AMAX_WARPS * 32)
                tab[x] = 0u;
            named_barrier(3, AMAX_WARPS * 32);
            const int l0 = u.s * TL + 2 * lane;
            int g = u.gf;
            int gend = soffs[g];
            uint32_t acc = 0u;
            bool fail = false, spilled = false;
            auto flush = [&]() {
                const uint32_t lo = acc << 16, hi = acc & 0xFFFF0000u;
                const int slot = g - u.gf;
                if (slot < MAXG_U) {
                    if (lo) atomicMax(&sm.tab[uq][slot][2 * lane], lo);
                    if (hi) atomicMax(&sm.tab[uq][slot][2 * lane + 1], hi);
                } else {
                    unsigned *row = amax + (int64_t)g * L;
                    if (lo && l0 < L) atomicMax(row + l0, lo);
                    if (hi && l0 + 1 < L) atomicMax(row + l0 + 1, hi);
                    spilled = true;
                }
                acc = 0u;
            };
            for (int kt = 0; kt < u.ntiles; ++kt, ++i) {
                const int slot = i % RA;
                if (fail || !__all_sync(0xffffffffu, mbar_wait(&sm.full[slot], (uint32_t)(i / RA) & 1u, wait_ns))) {
                    fail = true; // stop at the end-of-unit barrier, together
                    continue;
                }
                uint32_t dep = 0u;
#pragma unroll 1
                for (int bb = 0; bb < 4 / AMAX_WARPS; ++bb) {
                    const int blk = (4 / AMAX_WARPS) * aw + bb; // 32-row block of the tile
                    const int row0 = u.r0 + kt * TP + 32 * blk;
                    const uint32_t *tile = reinterpret_cast<const uint32_t *>(sm.in[slot]) + (32 * blk) * (TL / 2) + lane;
                    if (row0 >= u.r1)
                        break;
                    const int nrows = min(32, u.r1 - row0);
                    if (row0 + nrows <= gend) {
                        if (nrows == 32) {
#pragma unroll
                            for (int r = 0; r < 32; ++r)
                                acc = absmax_bf16x2(acc, tile[r * (TL / 2)]);
                        } else {
                            for (int r = 0; r < nrows; ++r)
                                acc = absmax_bf16x2(acc, tile[r * (TL / 2)]);
                        }
                    } else {
                        // the block crosses group ends: one segment per
                        // group, each a fully unrolled, predicated pass
                        for (int r = 0; r < nrows;) {
                            if (row0 + r >= gend) {
                                flush();
                                do {
                                    ++g;
                                } while (row0 + r >= soffs[g]);
                                gend = soffs[g];
                            }
                            const int re = min(nrows, gend - row0);
#pragma unroll
                            for (int ii = 0; ii < 32; ++ii)
                                if (ii >= r && ii < re)
                                    acc = absmax_bf16x2(acc, tile[ii * (TL / 2)]);
                            r = re;
                        }
                    }
                    dep ^= acc;
                }
                // these reads end before the slot's next TMA fill
                release_slot_after(&sm.empty[slot], dep);
            }
            if (!fail)
                flush();
            if (__any_sync(0xffffffffu, spilled))
                __threadfence(); // global atomics of spilled groups before the counters
            if (barrier_or(3, AMAX_WARPS * 32, fail)) {
                set_abort(sm);
                break;
            }
            if (aw == 0) {
                if (lane == 0)
                    mbar_arrive(&sm.amax_computed[uq]);
                __syncwarp();
            }
        }
        return;
    }

    if (warp >= PM_WARP0) {
        // ---------------------------------------- publish and merge warps
        const int pm = warp - PM_WARP0;
        int ku = 0;
        for (uint32_t t = blockIdx.x; t < total; t += gridDim.x, ++ku) {
            if (ku % PM_WARPS != pm)
                continue;
            const Unit u = unit_of(t, ups, blocks, end, soffs, G);
            const int uq = ku % UQ;
            const bool ok = mbar_wait(&sm.amax_computed[uq], (uint32_t)(ku / UQ) & 1u, wait_ns);
            if (!__all_sync(0xffffffffu, ok) || abort_set(sm)) {
                set_abort(sm);
                break;
            }
            // every partial slot first, one fence, then the counters
            bool shared = false;
            for (int gg = u.gf; gg <= u.gl; ++gg) {
                const int st = gg ? soffs[gg - 1] : 0, en = soffs[gg];
                if (en <= st || unit_of_pos(st, ups, blocks) == unit_of_pos(en - 1, ups, blocks))
                    continue; // empty, or wholly inside this unit
                shared = true;
                const int slot = gg - u.gf;
                // a spilled group's maximum is in the table; its slot holds 0
                const uint32_t v0 = slot < MAXG_U ? sm.tab[uq][slot][2 * lane] : 0u;
                const uint32_t v1 = slot < MAXG_U ? sm.tab[uq][slot][2 * lane + 1] : 0u;
                unsigned *dst = partials + ((int64_t)u.s * pstride + u.b + gg) * TL + 2 * lane;
                *reinterpret_cast<uint2 *>(dst) = make_uint2(v0, v1);
            }
            if (shared) {
                __threadfence();
                __syncwarp();
                if (lane == 0)
                    for (int gg = u.gf; gg <= u.gl; ++gg) {
                        const int st = gg ? soffs[gg - 1] : 0, en = soffs[gg];
                        if (en > st && unit_of_pos(st, ups, blocks) != unit_of_pos(en - 1, ups, blocks))
                            red_release_gpu_add(counters + (int64_t)gg * nstrips + u.s, 1);
                    }
            }
            const int l0 = u.s * TL + 2 * lane;
            bool fail = false;
            for (int gg = u.gf; gg <= u.gl && !fail; ++gg) {
                const int st = gg ? soffs[gg - 1] : 0, en = soffs[gg];
                if (en <= st)
                    continue;
                const int slot = gg - u.gf;
                const int uf = unit_of_pos(st, ups, blocks), ul = unit_of_pos(en - 1, ups, blocks);
                const bool spans = uf != ul;
                uint32_t a0 = 0u, a1 = 0u;
                if (spans) {
                    // every unit of (group, strip) has published
                    const int need = ul - uf + 1;
                    const int *cnt = counters + (int64_t)gg * nstrips + u.s;
                    // one lane polls, backing off between reads, so the
                    // grid's waiters do not flood the counter's L2 line
                    if (lane == 0 && ld_acquire_gpu(cnt) < need) {
                        const uint64_t t0 = globaltimer();
                        while (ld_acquire_gpu(cnt) < need) {
                            if (globaltimer() - t0 > wait_ns) {
                                set_status(MXQ_ERR_TIMEOUT);
                                fail = true;
                                break;
                            }
                            __nanosleep(100);
                        }
                    }
                    if (__shfl_sync(0xffffffffu, (int)fail, 0)) {
                        fail = true;
                        break;
                    }
                    // lane 0's acquire orders the other lanes' reads too:
                    // they follow it across this warp barrier
                    __syncwarp();
                }
                if (spans) {
                    // the max over every unit's slot (and the table, which
                    // holds maxima spilled by units with many groups). Lane
                    // (k, q) reads 16 lines [16 q, 16 q + 16) of slots
                    // uf + k, uf + k + 8, ..., all loads in flight together;
                    // the 8 subsets meet in shared memory.
                    const int k = lane >> 2, qq = lane & 3;
                    uint32_t m[16];
#pragma unroll
                    for (int x = 0; x < 16; ++x)
                        m[x] = 0u;
                    const unsigned *pp = partials + ((int64_t)u.s * pstride + gg) * TL + 16 * qq;
#pragma unroll 4
                    for (int b = uf + k; b <= ul; b += 8) {
                        const uint4 *src = reinterpret_cast<const uint4 *>(pp + (int64_t)b * TL);
                        uint4 x[4];
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            x[c] = __ldcg(src + c);
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            m[4 * c] = max(m[4 * c], x[c].x);
                            m[4 * c + 1] = max(m[4 * c + 1], x[c].y);
                            m[4 * c + 2] = max(m[4 * c + 2], x[c].z);
                            m[4 * c + 3] = max(m[4 * c + 3], x[c].w);
                        }
                    }
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        *reinterpret_cast<uint4 *>(&sm.red[pm][k][16 * qq + 4 * c]) =
                            make_uint4(m[4 * c], m[4 * c + 1], m[4 * c + 2], m[4 * c + 3]);
                    __syncwarp();
                    const unsigned *row = amax + (int64_t)gg * L;
                    a0 = l0 < L ? ld_relaxed_gpu(row + l0) : 0u;
                    a1 = l0 + 1 < L ? ld_relaxed_gpu(row + l0 + 1) : 0u;
#pragma unroll
                    for (int x = 0; x < 8; ++x) {
                        a0 = max(a0, sm.red[pm][x][2 * lane]);
                        a1 = max(a1, sm.red[pm][x][2 * lane + 1]);
                    }
                    __syncwarp();
                    if (slot >= MAXG_U) {
                        // the cast reads this group's maximum from the table
                        unsigned *wrow = amax + (int64_t)gg * L;
                        if (l0 < L) atomicMax(wrow + l0, a0);
                        if (l0 + 1 < L) atomicMax(wrow + l0 + 1, a1);
                        __threadfence();
                    }
                } else if (slot >= MAXG_U) {
                    const unsigned *row = amax + (int64_t)gg * L;
                    a0 = l0 < L ? ld_relaxed_gpu(row + l0) : 0u;
                    a1 = l0 + 1 < L ? ld_relaxed_gpu(row + l0 + 1) : 0u;
                } else {
                    a0 = sm.tab[uq][slot][2 * lane];
                    a1 = sm.tab[uq][slot][2 * lane + 1];
                }
                const float s0 = fp8_scale(__uint_as_float(a0)), s1 = fp8_scale(__uint_as_float(a1));
                if (slot < MAXG_U) {
                    sm.tab[uq][slot][2 * lane] = __float_as_uint(s0);
                    sm.tab[uq][slot][2 * lane + 1] = __float_as_uint(s1);
                }
                if (st >= u.r0) { // the unit holding the group's first position
                    float *irow = inv + (int64_t)gg * L;
                    if (l0 < L) irow[l0] = fp8_inv(s0);
                    if (l0 + 1 < L) irow[l0 + 1] = fp8_inv(s1);
                }
            }
            if (fail) {
                set_abort(sm);
                break;
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&sm.scales_ready[uq]);
            __syncwarp();
        }
        return;
    }

    // ---------------------------------------------------------- cast quads
    const int q = warp >> 2, w = warp & 3;
    const int qbar = 1 + q;
    const bool store_thread = threadIdx.x == 128 * q;
    bool prev_stored = true;
    int i0 = 0, ku = 0, nq = 0; // i0: cast-ring sequence number of the unit's first tile
    for (uint32_t t = blockIdx.x; t < total; t += gridDim.x, ++ku) {
        const Unit u = unit_of(t, ups, blocks, end, soffs, G);
        const int uq = ku % UQ;
        const bool ok = mbar_wait(&sm.scales_ready[uq], (uint32_t)(ku / UQ) & 1u, wait_ns);
        if (barrier_or(qbar, 4 * 32, !ok || abort_set(sm))) {
            set_abort(sm);
            break;
        }
        const int l0 = u.s * TL + 2 * lane;
        auto scales = [&](int grp, float &s0, float &s1) {
            const int slot = grp - u.gf;
            if (slot < MAXG_U) {
                s0 = __uint_as_float(sm.tab[uq][slot][2 * lane]);
                s1 = __uint_as_float(sm.tab[uq][slot][2 * lane + 1]);
            } else {
                const unsigned *row = amax + (int64_t)grp * L;
                s0 = fp8_scale(__uint_as_float(l0 < L ? ld_relaxed_gpu(row + l0) : 0u));
                s1 = fp8_scale(__uint_as_float(l0 + 1 < L ? ld_relaxed_gpu(row + l0 + 1) : 0u));
            }
        };
        bool fail = false;
        for (int kt = (q - i0) & 1; kt < u.ntiles; kt += 2) {
            const int i = i0 + kt, slot = i % RC;
            const int ob = nq & 1;
            ++nq;
            // a failed wait is carried to the barrier below, where the quad
            // stops together (the data read meanwhile is never stored)
            fail = !__all_sync(0xffffffffu, mbar_wait(&sm.cfull[slot], (uint32_t)(i / RC) & 1u, wait_ns));
            const uint32_t *tile = reinterpret_cast<const uint32_t *>(sm.cin[slot]) + (w * 32) * (TL / 2) + lane;
            uint32_t v[32];
            uint32_t dep = 0u;
#pragma unroll
            for (int r = 0; r < 32; ++r) {
                v[r] = tile[r * (TL / 2)];
                dep ^= v[r];
            }
            if (!fail) // a slot whose fill never landed is not handed back
                release_slot_after(&sm.cempty[slot], dep);
            const int tr0 = u.r0 + kt * TP; // the tile's first position
            const int p0 = tr0 + 32 * w;    // this warp's first position
            uint32_t q0[8], q1[8];          // lines l0, l0+1: 32 position bytes each
            const int g = p0 < u.r1 ? jag::group_of(soffs, G, p0) : u.gl;
            if (p0 < u.r1 && soffs[g] >= p0 + 32) {
                float s0, s1;
                scales(g, s0, s1);
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                    const uint32_t *r = v + 4 * jj;
                    q0[jj] = e4m3x2(__fmul_rn(bf16_lo(r[0]), s0), __fmul_rn(bf16_lo(r[1]), s0)) |
                             (e4m3x2(__fmul_rn(bf16_lo(r[2]), s0), __fmul_rn(bf16_lo(r[3]), s0)) << 16);
                    q1[jj] = e4m3x2(__fmul_rn(bf16_hi(r[0]), s1), __fmul_rn(bf16_hi(r[1]), s1)) |
                             (e4m3x2(__fmul_rn(bf16_hi(r[2]), s1), __fmul_rn(bf16_hi(r[3]), s1)) << 16);
                }
            } else {
                // the block crosses group ends (or the end of the unit): one
                // segment of rows per group, each a fully unrolled,
                // predicated pass with that group's scales (rows past the
                // unit's end form the last segment and are never stored)
#pragma unroll
                for (int jj = 0; jj < 8; ++jj)
                    q0[jj] = q1[jj] = 0u;
                int gg = g;
                for (int r = 0; r < 32;) {
                    const int row = p0 + r;
                    int re = 32;
                    if (row < u.r1) {
                        while (gg < u.gl && soffs[gg] <= row)
                            ++gg;
                        re = min(32, soffs[gg] - p0);
                    }
                    float s0, s1;
                    scales(gg, s0, s1);
#pragma unroll
                    for (int ii = 0; ii < 32; ++ii)
                        if (ii >= r && ii < re) {
                            const uint32_t x = v[ii];
                            q0[ii >> 2] |= e4m3x2(__fmul_rn(bf16_lo(x), s0), 0.0f) << (8 * (ii & 3));
                            q1[ii >> 2] |= e4m3x2(__fmul_rn(bf16_hi(x), s1), 0.0f) << (8 * (ii & 3));
                        }
                    r = re;
                }
            }

            const bool full_tile = tr0 + TP <= end;
            if (store_thread) {
                if (prev_stored)
                    bulk_wait_read<1>();
                else
                    bulk_wait_read<0>();
            }
            named_barrier(qbar, 4 * 32);
            if (full_tile) {
                // staging: 64 rows (lines) x 128 bytes (positions), 16-byte
                // chunk c of row r at chunk c ^ (r & 7) (128B swizzle)
                const uint32_t ob_addr = smem_u32(sm.out[q][ob]);
                const int bsel = (lane >> 2) & 1;
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const int b = bsel ^ (jj & 1), h = jj >> 1;
                    const int row = 2 * lane + b;
                    const int chunk = (2 * w + h) ^ (row & 7);
                    uint4 val;
                    if (b) val = make_uint4(q1[4 * h], q1[4 * h + 1], q1[4 * h + 2], q1[4 * h + 3]);
                    else   val = make_uint4(q0[4 * h], q0[4 * h + 1], q0[4 * h + 2], q0[4 * h + 3]);
                    sts_v4(ob_addr + row * 128 + chunk * 16, val);
                }
                fence_proxy_async_smem();
            } else if (!fail) {
#pragma unroll
                for (int bb = 0; bb < 2; ++bb) {
                    const int l = l0 + bb;
                    if (l >= L)
                        continue;
                    uint8_t *dst = out + (int64_t)l * P + p0;
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) {
                        const uint32_t word = bb ? q1[jj >> 2] : q0[jj >> 2];
                        if (p0 + jj < end)
                            dst[jj] = (uint8_t)(word >> (8 * (jj & 3)));
                    }
                }
            }
            if (barrier_or(qbar, 4 * 32, fail || abort_set(sm))) {
                fail = true;
                break;
            }
            if (store_thread && full_tile) {
                tma_store_2d(&tm_out, sm.out[q][ob], tr0, u.s * TL);
                bulk_commit();
            }
            prev_stored = full_tile;
        }
        if (fail) {
            set_abort(sm);
            break;
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&sm.scales_free[uq]);
        __syncwarp();
        i0 += u.ntiles;
    }
    if (store_thread)
        bulk_wait<0>();
}

} // namespace mxq
