// gemm.cuh - FP8 rowwise-scaled grouped GEMM on the 5th-generation tensor
// cores (tcgen05), the consumer the quantization feeds (ao PR 2064
// "[scaled grouped mm] add triton kernels for float8 rowwise quantization
// with per-group/jagged scales", Motivation; PR 2077 "[scaled grouped mm]
// integrate triton kernels into differentiable scaled grouped mm", Summary).
//
//   out[m][n] = bf16( (sum_k a[m][k] * w[g][n][k]) * inv_a[m] * inv_w[g][n] )
//
// for every row m of group g (rows offs[g-1] .. offs[g]-1 of A); a and w are
// e4m3, both K-major (row-major A (M, K), row-major W (E, N, K)); inv_a and
// inv_w are the fp32 inverse scales of the rowwise quantization. Rows past
// offs[G-1] are not written.
//
// Design: a persistent grid, one CTA per SM, walks (m-tile, n-tile) work items
// with n fastest; a group's m-tiles start at its first row, so a tile never
// mixes experts (rows past the group's end are computed and dropped).
//   warp 4       TMA producer: 128 x 128-byte tiles of A and BN x 128-byte
//                tiles of W (128B swizzle) into a 4-stage ring; BN = 256 when
//                N allows, else 128;
//   warp 5       allocates 2 * BN TMEM columns (two 128 x BN fp32
//                accumulators) and, from one thread, issues tcgen05.mma
//                kind::f8f6f4 (M 128, N BN, K 32) four times per stage,
//                releasing each stage with tcgen05.commit and handing a
//                finished accumulator to the epilogue the same way;
//   warps 0-3    epilogue: tcgen05.ld of their 32 TMEM lanes (rows), scale,
//                round to bf16, store; the accumulator is then released, so
//                the next tile's MMAs overlap this tile's epilogue.
// Every wait is bounded; on expiry the kernel records MXQ_ERR_TIMEOUT, every
// role stops, the MMA thread waits for its issued MMAs, and TMEM is freed.
#pragma once

#include "common.cuh"
#include "blocked.cuh"

namespace mxq {
namespace gm {

constexpr int BM = 128, BK = 128; // BK in bytes = e4m3 elements
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK;  // 16 KB
constexpr int THREADS = 6 * 32;
constexpr int ACC = 2;            // accumulators in TMEM

// tile width BN (128 or 256): a stage holds the A tile and a BN x 128-byte W
// tile; two BM x BN fp32 accumulators take 2 * BN TMEM columns
template <int BN> struct __align__(1024) Smem {
    uint8_t a[STAGES][A_BYTES];
    uint8_t b[STAGES][BN * BK];
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t acc_full[ACC];
    uint64_t acc_empty[ACC];
    uint64_t mma_done;
    uint32_t tmem_base;
    int abort_flag;
    int Tend;
};
template <int BN> constexpr size_t smem_fixed() { return sizeof(Smem<BN>) + 1024; }

// shared-memory matrix descriptor of a K-major tile of 128-byte rows stored
// with the 128-byte swizzle (8-row groups 1024 bytes apart): start address,
// leading offset 1 (unused for this layout), stride offset 1024 B, version 1,
// layout type 2 (128-byte swizzle)
MXQ_DEV uint64_t smem_desc_k128(uint32_t addr)
{
    return (uint64_t)((addr >> 4) & 0x3FFFu) | (uint64_t(1) << 16) | (uint64_t(1024 >> 4) << 32) |
           (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

// instruction descriptor: fp32 accumulator, e4m3 x e4m3, both K-major, N, M
template <int BN>
constexpr uint32_t idesc() { return (1u << 4) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24); }

MXQ_DEV int aborted(const int *flag) { return *reinterpret_cast<const volatile int *>(flag); }

MXQ_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
MXQ_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

MXQ_DEV void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// arrive on `bar` once every MMA this thread issued before has completed
MXQ_DEV void tc_commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// 32 lanes x 32 columns of fp32 from TMEM: thread i gets lane (base lane + i)
MXQ_DEV void tc_ld32(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 "
                 "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
                 "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                   "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
                   "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
                   "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
                   "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// the same load without the wait: several may be in flight before one
// tc_wait_ld (r must resolve to registers: index it with constants only)
MXQ_DEV void tc_ld32_nowait(uint32_t taddr, uint32_t *r)
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 "
                 "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
                 "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                   "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
                   "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
                   "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
                   "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
                 : "r"(taddr));
}

MXQ_DEV void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

MXQ_DEV uint32_t pack_bf16x2(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

} // namespace gm

template <int BN>
__global__ void __launch_bounds__(gm::THREADS, 1)
    k_fp8_grouped_gemm(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_w,
                       const float *__restrict__ inv_a, const float *__restrict__ inv_w, int64_t M, int64_t N,
                       int64_t K, const int32_t *__restrict__ offs, int G, uint16_t *__restrict__ out,
                       uint64_t wait_ns, int w_group_inner)
{
    using namespace gm;
    constexpr int B_BYTES = BN * BK;
    constexpr int TMEM_COLS = ACC * BN;
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
            mbar_init(&sm.acc_empty[i], 4);
        }
        mbar_init(&sm.mma_done, 1);
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    // m-tile start of every group (ceil(size / 128) tiles each); returns false
    // (status recorded) on bad offsets, identically in every CTA
    int Tend_local = 0;
    const bool ok_offs = padded_starts(offs, G, M, 7, T, &sm.Tend);
    if (!ok_offs)
        return;
    Tend_local = sm.Tend;
    if (warp == 5) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem_base)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    const int64_t ntn = N / BN, nkb = K / BK;
    const int64_t total = (int64_t)Tend_local * ntn;
    // group of m-tile mt: the largest g with T[g] <= mt (non-empty, see padded_starts)
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
            for (int64_t it = blockIdx.x; it < total && !aborted(&sm.abort_flag); it += gridDim.x) {
                const int64_t mt = it / ntn, nt = it - mt * ntn;
                const int g = tile_group(mt);
                const int64_t m0 = (g ? offs[g - 1] : 0) + (mt - T[g]) * BM;
                for (int64_t kb = 0; kb < nkb; ++kb, ++seq) {
                    const int s = seq % STAGES;
                    if (seq >= STAGES && !mbar_wait(&sm.empty[s], ((uint32_t)(seq / STAGES) & 1u) ^ 1u, wait_ns)) {
                        *reinterpret_cast<volatile int *>(&sm.abort_flag) = 1;
                        break;
                    }
                    mbar_arrive_expect_tx(&sm.full[s], A_BYTES + B_BYTES);
                    tma_load_2d(sm.a[s], &tm_a, &sm.full[s], (int)(kb * BK), (int)m0);
                    // W's map is (k, n, group), or (k, group, n) when the
                    // group stride is the smaller one
                    if (w_group_inner)
                        tma_load_3d(sm.b[s], &tm_w, &sm.full[s], (int)(kb * BK), g, (int)(nt * BN));
                    else
                        tma_load_3d(sm.b[s], &tm_w, &sm.full[s], (int)(kb * BK), (int)(nt * BN), g);
                }
            }
            // drain: every issued fill lands before the CTA exits
            for (int j = seq - STAGES; j < seq; ++j)
                if (j >= 0)
                    mbar_wait(&sm.full[j % STAGES], (uint32_t)(j / STAGES) & 1u, wait_ns);
        }
    } else if (warp == 5) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            int seq = 0, t = 0;
            bool issued = false;
            for (int64_t it = blockIdx.x; it < total && !aborted(&sm.abort_flag); it += gridDim.x, ++t) {
                const int acc = t & 1;
                // the epilogue has drained this accumulator (tile t-2)
                if (t >= ACC && !mbar_wait(&sm.acc_empty[acc], ((uint32_t)(t / ACC) & 1u) ^ 1u, wait_ns)) {
                    *reinterpret_cast<volatile int *>(&sm.abort_flag) = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(acc * BN);
                bool ok = true;
                for (int64_t kb = 0; kb < nkb; ++kb, ++seq) {
                    const int s = seq % STAGES;
                    if (!mbar_wait(&sm.full[s], (uint32_t)(seq / STAGES) & 1u, wait_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = smem_desc_k128(smem_u32(sm.a[s]));
                    const uint64_t bd = smem_desc_k128(smem_u32(sm.b[s]));
#pragma unroll
                    for (int k = 0; k < BK / 32; ++k) // K 32 per instruction: +32 bytes = +2 in the address field
                        tc_mma(d, ad + 2 * k, bd + 2 * k, IDESC, (kb > 0 || k > 0) ? 1u : 0u);
                    issued = true;
                    tc_commit(&sm.empty[s]); // the stage is free once these MMAs are done
                }
                if (!ok) {
                    *reinterpret_cast<volatile int *>(&sm.abort_flag) = 1;
                    break;
                }
                tc_commit(&sm.acc_full[acc]); // accumulator complete
            }
            if (issued) { // every issued MMA completes before TMEM is freed
                tc_commit(&sm.mma_done);
                mbar_wait(&sm.mma_done, 0u, wait_ns);
            }
        }
    } else {
        // ------------------------------------------------ epilogue (warps 0-3, TMEM lanes 32w..32w+31)
        int t = 0;
        for (int64_t it = blockIdx.x; it < total; it += gridDim.x, ++t) {
            const int acc = t & 1;
            bool ok = mbar_wait(&sm.acc_full[acc], (uint32_t)(t / ACC) & 1u, wait_ns);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok || aborted(&sm.abort_flag)) {
                *reinterpret_cast<volatile int *>(&sm.abort_flag) = 1;
                break;
            }
            tc_fence_after();
            const int64_t mt = it / ntn, nt = it - mt * ntn;
            const int g = tile_group(mt);
            const int64_t gs = g ? offs[g - 1] : 0, ge = offs[g];
            const int64_t m = gs + (mt - T[g]) * BM + 32 * warp + lane; // this thread's row
            const bool row_ok = m < ge;
            const float sa = row_ok ? __ldg(inv_a + m) : 0.0f;
            const float *sw = inv_w + (int64_t)g * N + nt * BN;
            uint16_t *dst = out + m * N + nt * BN;
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t r[32];
                tc_ld32(tmem + (uint32_t)(acc * BN + c * 32) + ((uint32_t)(32 * warp) << 16), r);
                if (row_ok) {
                    uint32_t pk[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float v0 = __fmul_rn(__fmul_rn(__uint_as_float(r[2 * j]), sa), __ldg(sw + c * 32 + 2 * j));
                        const float v1 =
                            __fmul_rn(__fmul_rn(__uint_as_float(r[2 * j + 1]), sa), __ldg(sw + c * 32 + 2 * j + 1));
                        pk[j] = gm::pack_bf16x2(v0, v1);
                    }
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        st_v4(dst + c * 32 + 8 * j, pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&sm.acc_empty[acc]);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 5)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
}

// ---------------------------------------------------------------------------
// Weight-gradient grouped GEMM, the backward consumer of the jagged ops:
//
//   out[g][n][k] = bf16( (sum_{m in group g} a[n][m] * b[k][m])
//                        * inv_a[g][n] * inv_b[g][k] )
//
// a (N, M) is grad_out^T quantized rowwise with per-(row, group) scales, b
// (K, M) the input quantized colwise with per-(column, group) scales; both
// keep the grouped dimension M contiguous, so both are K-major operands of
// the MMA and the contraction of group g runs over its own positions.
//
// Same roles as above, on (group, n-tile, k-tile) items. The producer streams
// 128-position chunks of the group starting at the 128-aligned position at
// or below its first one (so that every 128-byte row of a box is one L2
// line: unaligned boxes read two lines per row and made the kernel L2
// bound); where a chunk reaches outside the group, the MMA warp issues only
// the K-32 slices that hold group positions, zeroes the bytes outside the
// group within the two edge slices of both tiles in shared memory (the
// bytes past the last group are not data), fences the async proxy, and
// only then issues the MMAs. Items of empty groups write zeros.
// ---------------------------------------------------------------------------
namespace gm {

// zero byte columns [b0, b1) (b1 - b0 <= 32) of a `rows` x 128-byte tile
// stored with the 128-byte swizzle (byte c of row r at r*128 + ((c/16) ^
// (r%8))*16 + c%16); lane l of the warp takes rows l, l+32, ... and every
// 16-byte chunk the range touches: a whole chunk is stored as zeros, a
// partial one is read, masked bytewise and written back
MXQ_DEV void zero_cols(uint8_t *tile, int rows, int b0, int b1)
{
    if (b1 <= b0)
        return;
    const int lane = threadIdx.x & 31;
    const int c0 = b0 >> 4, c1 = (b1 - 1) >> 4; // the range's chunks (at most 3)
#pragma unroll 1
    for (int c = c0; c <= c1; ++c) {
        const int z0 = max(b0 - 16 * c, 0), z1 = min(b1 - 16 * c, 16); // bytes [z0, z1) of the chunk
        uint32_t keep[4];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const int a = min(max(z0 - 4 * w, 0), 4), b = min(max(z1 - 4 * w, 0), 4);
            const uint32_t lo_m = a >= 4 ? 0xffffffffu : (1u << (8 * a)) - 1u; // bytes below a
            const uint32_t hi_m = b >= 4 ? 0u : ~((1u << (8 * b)) - 1u);       // bytes from b on
            keep[w] = lo_m | hi_m;
        }
        const bool whole = z0 == 0 && z1 == 16;
#pragma unroll 1
        for (int r = lane; r < rows; r += 32) {
            uint4 *chunk = reinterpret_cast<uint4 *>(tile + r * 128 + ((c ^ (r & 7)) << 4));
            if (whole) {
                *chunk = make_uint4(0u, 0u, 0u, 0u);
            } else {
                uint4 v = *chunk;
                v.x &= keep[0];
                v.y &= keep[1];
                v.z &= keep[2];
                v.w &= keep[3];
                *chunk = v;
            }
        }
    }
}

} // namespace gm

template <int BN>
__global__ void __launch_bounds__(gm::THREADS, 1)
    k_fp8_grouped_gemm_wgrad(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                             const float *__restrict__ inv_a, const float *__restrict__ inv_b, int64_t N, int64_t K,
                             int64_t M, const int32_t *__restrict__ offs, int G, uint16_t *__restrict__ out,
                             uint64_t wait_ns)
{
    using namespace gm;
    constexpr int B_BYTES = BN * BK;
    constexpr int TMEM_COLS = ACC * BN;
    constexpr uint32_t IDESC = idesc<BN>();
    extern __shared__ uint8_t smem_raw[];
    Smem<BN> &sm = *reinterpret_cast<Smem<BN> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        for (int i = 0; i < ACC; ++i) {
            mbar_init(&sm.acc_full[i], 1);
            mbar_init(&sm.acc_empty[i], 4);
        }
        mbar_init(&sm.mma_done, 1);
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    if (!offsets_ok(offs, G, M))
        return;
    if (warp == 5) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem_base)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    const int64_t ntn = N / BM, ktn = K / BN;
    const int64_t per_g = ntn * ktn, total = per_g * G;
    // item it -> group, tiles, the group's positions [s, e), first chunk x0
    struct Item {
        int g;
        int64_t nt, kt, s, e, x0, nch;
    };
    auto item = [&](int64_t it) {
        Item q;
        q.g = (int)(it / per_g);
        const int64_t rem = it - (int64_t)q.g * per_g;
        q.nt = rem / ktn;
        q.kt = rem - q.nt * ktn;
        q.s = q.g ? offs[q.g - 1] : 0;
        q.e = offs[q.g];
        q.x0 = q.s & ~int64_t(BK - 1); // 128-byte aligned chunks: a box row is one L2 line
        q.nch = q.e > q.s ? (q.e - q.x0 + BK - 1) / BK : 0;
        return q;
    };

    if (warp == 4) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int seq = 0;
            for (int64_t it = blockIdx.x; it < total && !aborted(&sm.abort_flag); it += gridDim.x) {
                const Item q = item(it);
                for (int64_t j = 0; j < q.nch; ++j, ++seq) {
                    const int s = seq % STAGES;
                    if (seq >= STAGES && !mbar_wait(&sm.empty[s], ((uint32_t)(seq / STAGES) & 1u) ^ 1u, wait_ns)) {
                        *reinterpret_cast<volatile int *>(&sm.abort_flag) = 1;
                        break;
                    }
                    mbar_arrive_expect_tx(&sm.full[s], A_BYTES + B_BYTES);
                    tma_load_2d(sm.a[s], &tm_a, &sm.full[s], (int)(q.x0 + j * BK), (int)(q.nt * BM));
                    tma_load_2d(sm.b[s], &tm_b, &sm.full[s], (int)(q.x0 + j * BK), (int)(q.kt * BN));
                }
            }
            for (int j = seq - STAGES; j < seq; ++j)
                if (j >= 0)
                    mbar_wait(&sm.full[j % STAGES], (uint32_t)(j / STAGES) & 1u, wait_ns);
        }
    } else if (warp == 5) {
        // ------------------------------------------------ MMA issuer (the whole warp fixes tiles up)
        int seq = 0, t = 0;
        bool issued = false;
        for (int64_t it = blockIdx.x; it < total && !aborted(&sm.abort_flag); it += gridDim.x) {
            const Item q = item(it);
            if (q.nch == 0)
                continue;
            const int acc = t & 1;
            bool ok = t < ACC || mbar_wait(&sm.acc_empty[acc], ((uint32_t)(t / ACC) & 1u) ^ 1u, wait_ns);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) {
                *reinterpret_cast<volatile int *>(&sm.abort_flag) = 1;
                break;
            }
            tc_fence_after();
            const uint32_t d = tmem + (uint32_t)(acc * BN);
            for (int64_t j = 0; j < q.nch; ++j, ++seq) {
                const int s = seq % STAGES;
                ok = mbar_wait(&sm.full[s], (uint32_t)(seq / STAGES) & 1u, wait_ns);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok)
                    break;
                const int64_t c0 = q.x0 + j * BK;
                const int lo = (int)max((int64_t)0, q.s - c0), hi = (int)min((int64_t)BK, q.e - c0);
                // the K-32 slices holding some of the group's positions
                // [lo, hi) of this chunk (never empty: the chunks span the
                // group); slices wholly outside are not issued, and the
                // bytes outside the group in the two edge slices are zeroed
                // in both tiles: positions past offs[G-1] were never written
                // by the quantization and may hold any byte, NaN codes
                // included, and 0 * NaN is NaN
                const int k_lo = lo >> 5, k_hi = (hi + 31) >> 5;
                if ((lo & 31) || (hi & 31)) {
                    zero_cols(sm.a[s], BM, 32 * k_lo, lo);
                    zero_cols(sm.a[s], BM, hi, 32 * k_hi);
                    zero_cols(sm.b[s], BN, 32 * k_lo, lo);
                    zero_cols(sm.b[s], BN, hi, 32 * k_hi);
                    fence_proxy_async_smem();
                }
                __syncwarp();
                if (lane == 0) {
                    tc_fence_after();
                    const uint64_t ad = smem_desc_k128(smem_u32(sm.a[s]));
                    const uint64_t bd = smem_desc_k128(smem_u32(sm.b[s]));
#pragma unroll
                    for (int k = 0; k < BK / 32; ++k)
                        if (k >= k_lo && k < k_hi)
                            tc_mma(d, ad + 2 * k, bd + 2 * k, IDESC, (j > 0 || k > k_lo) ? 1u : 0u);
                    tc_commit(&sm.empty[s]);
                }
                issued = true;
                __syncwarp();
            }
            if (!ok) {
                *reinterpret_cast<volatile int *>(&sm.abort_flag) = 1;
                break;
            }
            if (lane == 0)
                tc_commit(&sm.acc_full[acc]);
            ++t;
        }
        if (issued && lane == 0) { // every issued MMA completes before TMEM is freed
            tc_commit(&sm.mma_done);
            mbar_wait(&sm.mma_done, 0u, wait_ns);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue (warps 0-3, TMEM lanes 32w..32w+31)
        int t = 0;
        for (int64_t it = blockIdx.x; it < total; it += gridDim.x) {
            const Item q = item(it);
            const int64_t n = q.nt * BM + 32 * warp + lane; // this thread's output row
            uint16_t *dst = out + ((int64_t)q.g * N + n) * K + q.kt * BN;
            if (q.nch == 0) { // empty group: the sum is zero
                for (int c = 0; c < BN; c += 8)
                    st_v4(dst + c, 0u, 0u, 0u, 0u);
                continue;
            }
            const int acc = t & 1;
            bool ok = mbar_wait(&sm.acc_full[acc], (uint32_t)(t / ACC) & 1u, wait_ns);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok || aborted(&sm.abort_flag)) {
                *reinterpret_cast<volatile int *>(&sm.abort_flag) = 1;
                break;
            }
            tc_fence_after();
            const float sa = __ldg(inv_a + (int64_t)q.g * N + n);
            // the tile's column scales, one per lane and 32-column chunk
            // (one coalesced load per chunk), handed to the row-owning
            // lanes by shuffles: per-element loads of a scale every lane
            // shares would queue in the load/store unit
            const float *sb = inv_b + (int64_t)q.g * K + q.kt * BN;
            float sbl[BN / 32];
#pragma unroll
            for (int c = 0; c < BN / 32; ++c)
                sbl[c] = __ldg(sb + c * 32 + lane);
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t r[32];
                tc_ld32(tmem + (uint32_t)(acc * BN + c * 32) + ((uint32_t)(32 * warp) << 16), r);
                float cs = sbl[0];
#pragma unroll
                for (int cc = 1; cc < BN / 32; ++cc)
                    cs = c == cc ? sbl[cc] : cs;
                uint32_t pk[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float v0 =
                        __fmul_rn(__fmul_rn(__uint_as_float(r[2 * j]), sa), __shfl_sync(0xffffffffu, cs, 2 * j));
                    const float v1 =
                        __fmul_rn(__fmul_rn(__uint_as_float(r[2 * j + 1]), sa), __shfl_sync(0xffffffffu, cs, 2 * j + 1));
                    pk[j] = pack_bf16x2(v0, v1);
                }
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    st_v4(dst + c * 32 + 8 * j, pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&sm.acc_empty[acc]);
            ++t;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 5)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
}

} // namespace mxq

