// gemm_mx.cuh - MXFP8 block-scaled grouped GEMM on the 5th-generation tensor
// cores, the consumer of the MX rowwise quantization and of the per-group
// 128x4 blocked scale layout (ao PR 3504 "[mxfp8 moe training] add CUDA
// kernel for per-group conversion of scale factors to blocked layout", title:
// per-group blocked scales for MXFP8 MoE training; taken here to feed the MoE
// layer's grouped GEMM, whose product is the OCP MX definition: an element is
// its e4m3 value times 2^(e-127) of its block's E8M0 byte e, blocks being 32
// consecutive elements along K).
//
//   out[m][n] = bf16( sum_k a[m][k] 2^(sa[m][k/32]-127) * w[g][n][k] 2^(sw[g][n][k/32]-127) )
//
// for every row m of group g (rows offs[g-1] .. offs[g]-1); a, w e4m3 K-major;
// sa are A's E8M0 scales in the grouped blocked layout (each group's rows
// padded to a multiple of 128, the (rows, K/32) matrix stored as 128 x 4
// tiles of 512 bytes, tile (row tile, K/128 block) at (rt * K/128 + kb) * 512,
// byte (r % 32) * 16 + (r % 128 / 32) * 4 + k % 4 inside it); sw are W's,
// viewed as one (E*N, K/32) matrix in the same layout (N % 128 == 0, so no
// padding between experts). Rows past offs[G-1] are not written.
//
// The pipeline is the FP8 grouped GEMM's (128 x BN tiles, BN = 256 when N
// allows, with one accumulator then: two would fill TMEM); what changes:
//   - each stage also carries the 512-byte scale tile of A (the m-tile's index
//     is its row tile in the blocked layout, since both pad every group to
//     128 rows) and the BN/128 tiles of W, fetched with bulk copies on the
//     stage's barrier;
//   - the MMA thread copies both into TMEM with tcgen05.cp 32x128b.warpx4
//     (lane r % 32, column r / 32, byte = the K/32 block within the stage:
//     exactly the blocked tile's order) and issues tcgen05.mma
//     kind::mxf8f6f4.block_scale, K 32 per instruction, the scale byte chosen
//     by the descriptor's scale-factor ids;
//   - the epilogue only rounds to bf16: the scales were applied in the MMA.
#pragma once

#include "gemm.cuh"

namespace mxq {
namespace gmx {

constexpr int BM = gm::BM, BK = gm::BK;
constexpr int STAGES = gm::STAGES;
// warps 0-3 and 6-9 drain the accumulator (warp w reads TMEM lanes
// 32 (w % 4) ..; warps 0-3 take the tile's first BN/2 columns, 6-9 the
// rest), warp 4 loads, warp 5 issues: with one accumulator at BN 256 the
// next tile's MMAs wait for the whole drain, which two warps per lane
// quadrant halve
constexpr int EPI_WARPS = 8;
constexpr int THREADS = (EPI_WARPS + 2) * 32;
constexpr int A_BYTES = BM * BK;
constexpr int SF_BYTES = 512;           // one 128 x 4 blocked scale tile
constexpr int TMEM_COLS = 512;
// per tile width: accumulators, TMEM column of the scales (after the
// accumulators), scale columns per stage (4 for A, 4 per 128 rows of W)
template <int BN> struct Cfg {
    static constexpr int ACC = BN == 256 ? 1 : 2;
    static constexpr int B_BYTES = BN * BK;
    static constexpr int SF_COL = ACC * BN;
    static constexpr int SF_STAGE_COLS = 4 + 4 * (BN / 128);
    static_assert(SF_COL + STAGES * SF_STAGE_COLS <= TMEM_COLS, "scales fit after the accumulators");
};

template <int BN> struct __align__(1024) Smem {
    uint8_t a[STAGES][A_BYTES];
    uint8_t b[STAGES][BN * BK];
    uint8_t sfa[STAGES][SF_BYTES];
    uint8_t sfb[STAGES][SF_BYTES * (BN / 128)];
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t acc_full[2];   // [0, Cfg<BN>::ACC) initialized and used
    uint64_t acc_empty[2];
    uint64_t mma_done;
    uint32_t tmem_base;
    int abort_flag;
    int Tend;
};
template <int BN> constexpr size_t smem_fixed() { return sizeof(Smem<BN>) + 1024; }

// instruction descriptor of kind::mxf8f6f4.block_scale: A and B e4m3
// (format 0), both K-major, N, E8M0 scale factors (bit 23), M; the scale
// bytes are picked per instruction by the ids in bits 4-5 (B) and 29-30 (A)
template <int BN>
constexpr uint32_t idesc() { return ((uint32_t)(BN >> 3) << 17) | (1u << 23) | ((uint32_t)(BM >> 4) << 24); }

// shared-memory descriptor of a scale tile as tcgen05.cp reads it: 32 rows
// of 16 bytes, no swizzle, 8-row core matrices 128 bytes apart; version 1
MXQ_DEV uint64_t sf_desc(uint32_t addr)
{
    return (uint64_t)((addr >> 4) & 0x3FFFu) | (uint64_t(128 >> 4) << 16) | (uint64_t(128 >> 4) << 32) |
           (uint64_t(1) << 46);
}

// untiled bulk copy of `bytes` from global to shared memory, counted on
// `bar` (both addresses 16-byte aligned, bytes a multiple of 16)
MXQ_DEV void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

// 32 rows x 16 bytes of shared memory into TMEM lanes 0-31, columns
// taddr .. taddr+3, repeated in the other three lane quadrants
MXQ_DEV void tc_cp_sf(uint32_t taddr, uint64_t sdesc)
{
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

MXQ_DEV void tc_mma_mx(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t sfa_tmem,
                       uint32_t sfb_tmem, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

} // namespace gmx

template <int BN>
__global__ void __launch_bounds__(gmx::THREADS, 1)
    k_mx_grouped_gemm(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_w,
                      const uint8_t *__restrict__ sfa, const uint8_t *__restrict__ sfw, int64_t M, int64_t N,
                      int64_t K, const int32_t *__restrict__ offs, int G, uint16_t *__restrict__ out,
                      uint64_t wait_ns)
{
    using namespace gmx;
    constexpr int ACC = Cfg<BN>::ACC, B_BYTES = Cfg<BN>::B_BYTES;
    constexpr int SF_COL = Cfg<BN>::SF_COL, SF_STAGE_COLS = Cfg<BN>::SF_STAGE_COLS;
    constexpr uint32_t IDESC = idesc<BN>();
    extern __shared__ uint8_t smem_raw[];
    Smem<BN> &sm = *reinterpret_cast<Smem<BN> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    int *T = reinterpret_cast<int *>(&sm + 1); // G group m-tile starts, after the fixed part
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
    // m-tile start of every group; also the group's first row tile in the
    // blocked scale layout of A (both pad each group to 128 rows)
    const bool ok_offs = padded_starts(offs, G, M, 7, T, &sm.Tend);
    if (!ok_offs)
        return;
    const int Tend_local = sm.Tend;
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

    const int64_t ntn = N / BN, nkb = K / BK;
    const int64_t total = (int64_t)Tend_local * ntn;
    auto tile_group = [&](int64_t mt) {
        int a = 0, b = G - 1;
        while (a < b) {
            const int m = (a + b + 1) >> 1;
            if (T[m] <= mt) a = m; else b = m - 1;
        }
        return a;
    };

    if (warp == 4) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int seq = 0;
            for (int64_t it = blockIdx.x; it < total && !gm::aborted(&sm.abort_flag); it += gridDim.x) {
                const int64_t mt = it / ntn, nt = it - mt * ntn;
                const int g = tile_group(mt);
                const int64_t m0 = (g ? offs[g - 1] : 0) + (mt - T[g]) * BM;
                const int64_t wrow = (int64_t)g * N + nt * BN; // W row; its row tile is wrow / 128
                const uint8_t *sa = sfa + mt * nkb * SF_BYTES;
                const uint8_t *sw = sfw + (wrow / 128) * nkb * SF_BYTES;
                for (int64_t kb = 0; kb < nkb; ++kb, ++seq) {
                    const int s = seq % STAGES;
                    if (seq >= STAGES && !mbar_wait(&sm.empty[s], ((uint32_t)(seq / STAGES) & 1u) ^ 1u, wait_ns)) {
                        *reinterpret_cast<volatile int *>(&sm.abort_flag) = 1;
                        break;
                    }
                    mbar_arrive_expect_tx(&sm.full[s], A_BYTES + B_BYTES + SF_BYTES * (1 + BN / 128));
                    tma_load_2d(sm.a[s], &tm_a, &sm.full[s], (int)(kb * BK), (int)m0);
                    tma_load_2d(sm.b[s], &tm_w, &sm.full[s], (int)(kb * BK), (int)wrow);
                    bulk_load(sm.sfa[s], sa + kb * SF_BYTES, SF_BYTES, &sm.full[s]);
#pragma unroll
                    for (int h = 0; h < BN / 128; ++h) // W row tiles wrow/128 + h: nkb tiles apart
                        bulk_load(sm.sfb[s] + h * SF_BYTES, sw + (h * nkb + kb) * SF_BYTES, SF_BYTES, &sm.full[s]);
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
            for (int64_t it = blockIdx.x; it < total && !gm::aborted(&sm.abort_flag); it += gridDim.x, ++t) {
                const int acc = t % ACC; // one accumulator at BN 256: every tile waits for the last epilogue
                if (t >= ACC && !mbar_wait(&sm.acc_empty[acc], ((uint32_t)(t / ACC) & 1u) ^ 1u, wait_ns)) {
                    *reinterpret_cast<volatile int *>(&sm.abort_flag) = 1;
                    break;
                }
                gm::tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(acc * BN);
                // the scales of stage `seq` into its slot's own TMEM columns,
                // once the stage has landed (its slot's previous MMAs have
                // then completed: the producer refilled the slot after them)
                auto land_scales = [&](int sq) {
                    const int ss = sq % STAGES;
                    if (!mbar_wait(&sm.full[ss], (uint32_t)(sq / STAGES) & 1u, wait_ns))
                        return false;
                    gm::tc_fence_after();
                    const uint32_t sft = tmem + (uint32_t)(SF_COL + ss * SF_STAGE_COLS);
                    tc_cp_sf(sft, sf_desc(smem_u32(sm.sfa[ss])));
#pragma unroll
                    for (int h = 0; h < BN / 128; ++h) // W rows 128h.. of the tile: 4 columns each
                        tc_cp_sf(sft + 4 + 4 * h, sf_desc(smem_u32(sm.sfb[ss] + h * SF_BYTES)));
                    return true;
                };
                bool ok = land_scales(seq);
                for (int64_t kb = 0; ok && kb < nkb; ++kb, ++seq) {
                    const int s = seq % STAGES;
                    // the next stage's scale copies go ahead of this stage's
                    // MMAs, so that they are done before the MMAs that read them
                    if (kb + 1 < nkb && !land_scales(seq + 1)) {
                        ok = false;
                        break;
                    }
                    const uint32_t sft = tmem + (uint32_t)(SF_COL + s * SF_STAGE_COLS);
                    const uint64_t ad = gm::smem_desc_k128(smem_u32(sm.a[s]));
                    const uint64_t bd = gm::smem_desc_k128(smem_u32(sm.b[s]));
#pragma unroll
                    for (int k = 0; k < BK / 32; ++k) {
                        // K 32 per instruction (+32 bytes = +2 in the address
                        // field); scale byte k of the stage's four
                        const uint32_t id = IDESC | ((uint32_t)k << 29) | ((uint32_t)k << 4);
                        tc_mma_mx(d, ad + 2 * k, bd + 2 * k, id, sft | ((uint32_t)k << 30),
                                  (sft + 4) | ((uint32_t)k << 30), (kb > 0 || k > 0) ? 1u : 0u);
                    }
                    issued = true;
                    gm::tc_commit(&sm.empty[s]);
                }
                if (!ok) {
                    *reinterpret_cast<volatile int *>(&sm.abort_flag) = 1;
                    break;
                }
                gm::tc_commit(&sm.acc_full[acc]);
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
        for (int64_t it = blockIdx.x; it < total; it += gridDim.x, ++t) {
            const int acc = t % ACC;
            bool ok = mbar_wait(&sm.acc_full[acc], (uint32_t)(t / ACC) & 1u, wait_ns);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok || gm::aborted(&sm.abort_flag)) {
                *reinterpret_cast<volatile int *>(&sm.abort_flag) = 1;
                break;
            }
            gm::tc_fence_after();
            const int64_t mt = it / ntn, nt = it - mt * ntn;
            const int g = tile_group(mt);
            const int64_t gs = g ? offs[g - 1] : 0, ge = offs[g];
            const int64_t m = gs + (mt - T[g]) * BM + 32 * quad + lane;
            const bool row_ok = m < ge;
            uint16_t *dst = out + m * N + nt * BN + 32 * c_begin;
            // the warp's half row into registers at once, the accumulator
            // released, and only then the rounding and the stores: the next
            // tile's MMAs wait for the TMEM reads alone
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
            if (row_ok) {
#pragma unroll
                for (int j = 0; j < BN / 16; ++j)
                    st_v4(dst + 8 * j, gm::pack_bf16x2(__uint_as_float(r[8 * j]), __uint_as_float(r[8 * j + 1])),
                          gm::pack_bf16x2(__uint_as_float(r[8 * j + 2]), __uint_as_float(r[8 * j + 3])),
                          gm::pack_bf16x2(__uint_as_float(r[8 * j + 4]), __uint_as_float(r[8 * j + 5])),
                          gm::pack_bf16x2(__uint_as_float(r[8 * j + 6]), __uint_as_float(r[8 * j + 7])));
            }
        }
    }

    gm::tc_fence_before();
    __syncthreads();
    gm::tc_fence_after();
    if (warp == 5)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
}

} // namespace mxq
