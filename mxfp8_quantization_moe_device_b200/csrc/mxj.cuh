// mxj.cuh - the MXFP8 weight gradient of a grouped (MoE) matmul: MX
// quantization along each group's tokens, and the block-scaled grouped GEMM
// that contracts over them (the stack of ao PR 3504 "[mxfp8 moe training]
// add CUDA kernel for per-group conversion of scale factors to blocked
// layout": "integrate new cuda kernel for blocked layout for groups along
// K"; the weight gradient is the grouped GEMM whose contraction dimension,
// the tokens, carries the groups).
//
// Quantization (k_mx_jagged_colwise_padded). Lines are contiguous in memory
// and positions (tokens) are grouped by device offsets, as in the jagged
// float8 ops. Each group's positions are cut into 32-element MX blocks from
// the group's first position, the last block holding the remainder; a block
// gets an E8M0 scale (floor or rceil) and e4m3 codes. The output places
// group g at padded position 128 * T[g], T[g] = sum_{h<g} ceil(size_h/128),
// codes line-major (out[l * cap + pp]) with zero codes in every pad
// position, and the scales straight in the 128 x 4 blocked layout with
// groups along K (the group's scale columns start at 4 T[g]; every column
// and row not covered by a block is zero). A 128-position tile of the output
// therefore belongs to one group and is read from a contiguous run of 128
// input positions, so the kernel is the MX 3-D colwise one with a per-tile
// input origin: persistent grid, TMA ring of 128 x 64 tiles, one consumer
// warp per 32-row block, a swizzled staging tile leaving through TMA stores.
//
// GEMM (k_mx_grouped_gemm_wgrad): out[g][n][k] = sum over group g's padded
// positions p of a[n][p] 2^(sa[n][p/32]-127) * b[k][p] 2^(sb[k][p/32]-127),
// with a (N, cap) and b (K, cap) the padded codes of grad_out^T and of the
// input and sa, sb their blocked scales. Every 128-position chunk of a group
// lies in the group (pads are zero codes), so the pipeline is the forward MX
// GEMM's over (group, n-tile, k-tile) items with the group's chunks, and the
// chunk's scale tiles are tile column T[g] + j of the blocked layouts.
#pragma once

#include "blocked.cuh"
#include "gemm_mx.cuh"

namespace mxq {
namespace mxj {

constexpr int TP = 128;              // padded positions per tile (four 32-row blocks)
constexpr int TL = 64;               // lines per tile
constexpr int STAGES = 4;
constexpr int CWARPS = 4;
constexpr int THREADS = (CWARPS + 1) * 32;
constexpr int IN_BYTES = TP * TL * 2;  // 16 KB
constexpr int OUT_BYTES = TP * TL;     // 8 KB
constexpr int CTAS_PER_SM = 2;

struct __align__(1024) Smem {
    uint8_t in[STAGES][IN_BYTES];
    uint8_t out[2][OUT_BYTES];
    uint32_t sc[2][TL];     // per line: the four blocks' scale bytes
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    int abort_flag;
    int Tend;
};
constexpr size_t SMEM_FIXED = sizeof(Smem) + 1024;

// the group owning padded tile pt (< Tend): the last g with T[g] <= pt
// (empty groups own no tile, and the group after one starts at the same T)
MXQ_DEV int tile_owner(const int *T, int G, int pt)
{
    int a = 0, b = G - 1;
    while (a < b) {
        const int m = (a + b + 1) >> 1;
        if (T[m] <= pt) a = m; else b = m - 1;
    }
    return a;
}

} // namespace mxj

// cap_tiles = cap / 128; L % 64 == 0 (the host asks L % 128 == 0 so that
// the blocked scale matrix has no pad rows)
__global__ void __launch_bounds__(mxj::THREADS, mxj::CTAS_PER_SM)
    k_mx_jagged_colwise_padded(const __grid_constant__ CUtensorMap tm_in, const __grid_constant__ CUtensorMap tm_out,
                               int L, int P, const int32_t *__restrict__ offs, int G, int cap_tiles,
                               uint8_t *__restrict__ scales, int mode, uint64_t wait_ns)
{
    using namespace mxj;
    extern __shared__ uint8_t smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    int *T = reinterpret_cast<int *>(&sm + 1); // padded group starts, in tiles
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], CWARPS);
        }
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    if (!padded_starts(offs, G, P, 7, T, &sm.Tend))
        return;
    const int Tend = sm.Tend;
    const int nlt = L / TL;
    const uint32_t total = (uint32_t)cap_tiles * (uint32_t)nlt;

    if (warp == CWARPS) {
        // ------------------------------------------------ producer warp
        if (lane == 0) {
            int it = 0;
            for (uint32_t t = blockIdx.x; t < total; t += gridDim.x, ++it) {
                const int s = it % STAGES;
                if (it >= STAGES && !mbar_wait(&sm.empty[s], ((uint32_t)(it / STAGES) & 1u) ^ 1u, wait_ns)) {
                    *reinterpret_cast<volatile int *>(&sm.abort_flag) = 1;
                    break;
                }
                const int pt = (int)(t / (uint32_t)nlt), lt = (int)(t - (uint32_t)pt * (uint32_t)nlt);
                if (pt < Tend) {
                    const int g = tile_owner(T, G, pt);
                    const int y0 = (g ? offs[g - 1] : 0) + (pt - T[g]) * TP;
                    mbar_arrive_expect_tx(&sm.full[s], IN_BYTES);
                    tma_load_2d(sm.in[s], &tm_in, &sm.full[s], lt * TL, y0);
                } else {
                    mbar_arrive(&sm.full[s]); // capacity past the last group: nothing to read
                }
            }
            for (int j = it - STAGES; j < it; ++j)
                if (j >= 0)
                    mbar_wait(&sm.full[j % STAGES], (uint32_t)(j / STAGES) & 1u, wait_ns);
        }
        return;
    }

    // ---------------------------------------------------- consumer warps
    const int w = warp; // 32-row block of the tile
    int it = 0;
    for (uint32_t t = blockIdx.x; t < total; t += gridDim.x, ++it) {
        const int s = it % STAGES;
        const int ob = it & 1;
        const int pt = (int)(t / (uint32_t)nlt), lt = (int)(t - (uint32_t)pt * (uint32_t)nlt);
        // valid rows of this warp's block: the group's remaining positions
        int nv = 0;
        if (pt < Tend) {
            const int g = tile_owner(T, G, pt);
            const int y0 = (g ? offs[g - 1] : 0) + (pt - T[g]) * TP;
            nv = min(32, max(0, offs[g] - y0 - 32 * w));
        }
        bool ok = mbar_wait(&sm.full[s], (uint32_t)(it / STAGES) & 1u, wait_ns);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok)
            sm.abort_flag = 1;
        const uint32_t *tile = reinterpret_cast<const uint32_t *>(sm.in[s]) + (w * 32) * (TL / 2) + lane;
        uint32_t v[32];
        uint32_t acc = 0u;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            v[i] = i < nv ? tile[i * (TL / 2)] : 0u; // pad positions are zero
            acc = absmax_bf16x2(acc, v[i]);
        }
        release_slot_after(&sm.empty[s], acc);

        const uint32_t b0 = e8m0_mode(bf16_lo(acc), mode), b1 = e8m0_mode(bf16_hi(acc), mode);
        const float f0 = mx_factor(b0), f1 = mx_factor(b1);
        uint32_t q0[8], q1[8]; // lines 2*lane, 2*lane+1: 32 position bytes each
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t *r = v + 4 * j;
            q0[j] = e4m3x2(__fmul_rn(bf16_lo(r[0]), f0), __fmul_rn(bf16_lo(r[1]), f0)) |
                    (e4m3x2(__fmul_rn(bf16_lo(r[2]), f0), __fmul_rn(bf16_lo(r[3]), f0)) << 16);
            q1[j] = e4m3x2(__fmul_rn(bf16_hi(r[0]), f1), __fmul_rn(bf16_hi(r[1]), f1)) |
                    (e4m3x2(__fmul_rn(bf16_hi(r[2]), f1), __fmul_rn(bf16_hi(r[3]), f1)) << 16);
        }

        // staging buffer `ob` was last read by the TMA store of tile it-2
        if (threadIdx.x == 0)
            bulk_wait_read<1>();
        named_barrier(1, CWARPS * 32);
        // out staging: 64 rows (lines) x 128 bytes (positions), 16-byte
        // chunk c of row r at chunk c ^ (r & 7) (the TMA 128-byte swizzle)
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
        reinterpret_cast<uint8_t *>(&sm.sc[ob][2 * lane])[w] = (uint8_t)b0;
        reinterpret_cast<uint8_t *>(&sm.sc[ob][2 * lane + 1])[w] = (uint8_t)b1;
        fence_proxy_async_smem();
        if (barrier_or(1, CWARPS * 32, sm.abort_flag != 0))
            break;
        if (threadIdx.x == 0) {
            tma_store_2d(&tm_out, sm.out[ob], pt * TP, lt * TL);
            bulk_commit();
        }
        if (threadIdx.x < TL) {
            // line l's four block bytes of tile column pt: one word of the
            // 128 x 4 tile (row tile l / 128, column tile pt)
            const int l = lt * TL + threadIdx.x;
            uint8_t *dst = scales + ((int64_t)(l >> 7) * cap_tiles + pt) * 512 + (l & 31) * 16 + ((l & 127) >> 5) * 4;
            *reinterpret_cast<uint32_t *>(dst) = sm.sc[ob][threadIdx.x];
        }
    }
    if (threadIdx.x == 0)
        bulk_wait<0>();
}

// ---------------------------------------------------------------------------
// MXFP8 weight-gradient grouped GEMM
// ---------------------------------------------------------------------------
template <int BN>
__global__ void __launch_bounds__(gmx::THREADS, 1)
    k_mx_grouped_gemm_wgrad(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                            const uint8_t *__restrict__ sfa, const uint8_t *__restrict__ sfb, int64_t N, int64_t K,
                            int64_t M, int cap_tiles, const int32_t *__restrict__ offs, int G,
                            uint16_t *__restrict__ out, uint64_t wait_ns)
{
    using namespace gmx;
    constexpr int ACC = Cfg<BN>::ACC, B_BYTES = Cfg<BN>::B_BYTES;
    constexpr int SF_COL = Cfg<BN>::SF_COL, SF_STAGE_COLS = Cfg<BN>::SF_STAGE_COLS;
    constexpr uint32_t IDESC = idesc<BN>();
    extern __shared__ uint8_t smem_raw[];
    Smem<BN> &sm = *reinterpret_cast<Smem<BN> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    int *T = reinterpret_cast<int *>(&sm + 1); // padded group starts, in 128-position chunks
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        for (int i = 0; i < ACC; ++i) {
            mbar_init(&sm.acc_full[i], 1);
            mbar_init(&sm.acc_empty[i], EPI_WARPS);
        }
        mbar_init(&sm.mma_done, 1);
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    if (!padded_starts(offs, G, M, 7, T, &sm.Tend))
        return;
    if (warp == 5) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem_base)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    gm::tc_fence_before();
    __syncthreads();
    gm::tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    const int64_t ntn = N / BM, ktn = K / BN;
    const int64_t per_g = ntn * ktn, total = per_g * G;
    // item it -> (group, n-tile, k-tile); the group's chunks T[g] .. T[g] + nch
    struct Item {
        int g;
        int64_t nt, kt;
        int c0, nch;
    };
    auto item = [&](int64_t it) {
        Item q;
        q.g = (int)(it / per_g);
        const int64_t rem = it - (int64_t)q.g * per_g;
        q.nt = rem / ktn;
        q.kt = rem - q.nt * ktn;
        q.c0 = T[q.g];
        const int size = offs[q.g] - (q.g ? offs[q.g - 1] : 0);
        q.nch = (size + BK - 1) / BK;
        return q;
    };

    if (warp == 4) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int seq = 0;
            for (int64_t it = blockIdx.x; it < total && !gm::aborted(&sm.abort_flag); it += gridDim.x) {
                const Item q = item(it);
                const uint8_t *sa = sfa + (q.nt * cap_tiles + q.c0) * SF_BYTES;
                const uint8_t *sb = sfb + (q.kt * (BN / 128) * cap_tiles + q.c0) * SF_BYTES;
                for (int j = 0; j < q.nch; ++j, ++seq) {
                    const int s = seq % STAGES;
                    if (seq >= STAGES && !mbar_wait(&sm.empty[s], ((uint32_t)(seq / STAGES) & 1u) ^ 1u, wait_ns)) {
                        *reinterpret_cast<volatile int *>(&sm.abort_flag) = 1;
                        break;
                    }
                    const int x = (q.c0 + j) * BK;
                    mbar_arrive_expect_tx(&sm.full[s], A_BYTES + B_BYTES + SF_BYTES * (1 + BN / 128));
                    tma_load_2d(sm.a[s], &tm_a, &sm.full[s], x, (int)(q.nt * BM));
                    tma_load_2d(sm.b[s], &tm_b, &sm.full[s], x, (int)(q.kt * BN));
                    bulk_load(sm.sfa[s], sa + (int64_t)j * SF_BYTES, SF_BYTES, &sm.full[s]);
#pragma unroll
                    for (int h = 0; h < BN / 128; ++h) // B row tiles kt*BN/128 + h: cap_tiles tiles apart
                        bulk_load(sm.sfb[s] + h * SF_BYTES, sb + ((int64_t)h * cap_tiles + j) * SF_BYTES, SF_BYTES,
                                  &sm.full[s]);
                }
            }
            for (int j = seq - STAGES; j < seq; ++j)
                if (j >= 0)
                    mbar_wait(&sm.full[j % STAGES], (uint32_t)(j / STAGES) & 1u, wait_ns);
        }
    } else if (warp == 5) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            int seq = 0, t = 0;
            bool issued = false;
            for (int64_t it = blockIdx.x; it < total && !gm::aborted(&sm.abort_flag); it += gridDim.x) {
                const Item q = item(it);
                if (q.nch == 0)
                    continue;
                const int acc = t % ACC;
                if (t >= ACC && !mbar_wait(&sm.acc_empty[acc], ((uint32_t)(t / ACC) & 1u) ^ 1u, wait_ns)) {
                    *reinterpret_cast<volatile int *>(&sm.abort_flag) = 1;
                    break;
                }
                gm::tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(acc * BN);
                // scales of stage `sq` into its slot's TMEM columns once it has
                // landed; the next stage's go ahead of this stage's MMAs
                auto land_scales = [&](int sq) {
                    const int ss = sq % STAGES;
                    if (!mbar_wait(&sm.full[ss], (uint32_t)(sq / STAGES) & 1u, wait_ns))
                        return false;
                    gm::tc_fence_after();
                    const uint32_t sft = tmem + (uint32_t)(SF_COL + ss * SF_STAGE_COLS);
                    tc_cp_sf(sft, sf_desc(smem_u32(sm.sfa[ss])));
#pragma unroll
                    for (int h = 0; h < BN / 128; ++h)
                        tc_cp_sf(sft + 4 + 4 * h, sf_desc(smem_u32(sm.sfb[ss] + h * SF_BYTES)));
                    return true;
                };
                bool ok = land_scales(seq);
                for (int j = 0; ok && j < q.nch; ++j, ++seq) {
                    const int s = seq % STAGES;
                    if (j + 1 < q.nch && !land_scales(seq + 1)) {
                        ok = false;
                        break;
                    }
                    const uint32_t sft = tmem + (uint32_t)(SF_COL + s * SF_STAGE_COLS);
                    const uint64_t ad = gm::smem_desc_k128(smem_u32(sm.a[s]));
                    const uint64_t bd = gm::smem_desc_k128(smem_u32(sm.b[s]));
#pragma unroll
                    for (int k = 0; k < BK / 32; ++k) {
                        const uint32_t id = IDESC | ((uint32_t)k << 29) | ((uint32_t)k << 4);
                        tc_mma_mx(d, ad + 2 * k, bd + 2 * k, id, sft | ((uint32_t)k << 30),
                                  (sft + 4) | ((uint32_t)k << 30), (j > 0 || k > 0) ? 1u : 0u);
                    }
                    issued = true;
                    gm::tc_commit(&sm.empty[s]);
                }
                if (!ok) {
                    *reinterpret_cast<volatile int *>(&sm.abort_flag) = 1;
                    break;
                }
                gm::tc_commit(&sm.acc_full[acc]);
                ++t;
            }
            if (issued) {
                gm::tc_commit(&sm.mma_done);
                mbar_wait(&sm.mma_done, 0u, wait_ns);
            }
        }
    } else {
        // ------------------------------------------------ epilogue (warps 0-3 and 6-9)
        const int quad = warp & 3, c_begin = warp < 4 ? 0 : BN / 64; // TMEM lanes 32 quad.., 32-column chunks
        int t = 0;
        for (int64_t it = blockIdx.x; it < total; it += gridDim.x) {
            const Item q = item(it);
            const int64_t n = q.nt * BM + 32 * quad + lane; // this thread's output row
            uint16_t *dst = out + ((int64_t)q.g * N + n) * K + q.kt * BN;
            if (q.nch == 0) { // empty group: the sum is zero
                for (int c = 32 * c_begin; c < 32 * c_begin + BN / 2; c += 8)
                    st_v4(dst + c, 0u, 0u, 0u, 0u);
                continue;
            }
            const int acc = t % ACC;
            bool ok = mbar_wait(&sm.acc_full[acc], (uint32_t)(t / ACC) & 1u, wait_ns);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok || gm::aborted(&sm.abort_flag)) {
                *reinterpret_cast<volatile int *>(&sm.abort_flag) = 1;
                break;
            }
            gm::tc_fence_after();
            // the warp's half row into registers, the accumulator released,
            // then the rounding and the stores (as in the forward MX GEMM)
            uint32_t r[BN / 2];
#pragma unroll
            for (int c = 0; c < BN / 64; ++c)
                gm::tc_ld32_nowait(tmem + (uint32_t)(acc * BN + (c_begin + c) * 32) + ((uint32_t)(32 * quad) << 16),
                                   r + 32 * c);
            gm::tc_wait_ld();
            gm::tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&sm.acc_empty[acc]);
            uint16_t *d0 = dst + 32 * c_begin;
#pragma unroll
            for (int j = 0; j < BN / 16; ++j)
                st_v4(d0 + 8 * j, gm::pack_bf16x2(__uint_as_float(r[8 * j]), __uint_as_float(r[8 * j + 1])),
                      gm::pack_bf16x2(__uint_as_float(r[8 * j + 2]), __uint_as_float(r[8 * j + 3])),
                      gm::pack_bf16x2(__uint_as_float(r[8 * j + 4]), __uint_as_float(r[8 * j + 5])),
                      gm::pack_bf16x2(__uint_as_float(r[8 * j + 6]), __uint_as_float(r[8 * j + 7])));
            ++t;
        }
    }

    gm::tc_fence_before();
    __syncthreads();
    gm::tc_fence_after();
    if (warp == 5)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
}

} // namespace mxq
