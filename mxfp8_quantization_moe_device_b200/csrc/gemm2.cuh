// gemm2.cuh - the FP8 weight-gradient grouped GEMM of gemm.cuh on CTA pairs:
// tcgen05.mma.cta_group::2, one 256 x 256 output tile per pair of SMs.
//
//   out[g][n][k] = bf16( (sum_{m in group g} a[n][m] * b[k][m])
//                        * inv_a[g][n] * inv_b[g][k] )
//
// Why pairs: a one-SM 128 x 256 tile streams 48 KB of operands per
// 128-position chunk, four stages fill shared memory, and the operand feed
// (TMA latency over four 48 KB stages) rather than the tensor pipe bounds
// the kernel. In a pair each SM holds half of the 256 rows of a (its
// accumulator rows) and half of the 256 rows of b, and the pair's MMA gives
// each SM all 256 columns: 32 KB per SM per chunk for the same work per SM,
// six stages in flight.
//
// Roles (a cluster of two CTAs, rank 0 the leader; warps 0-3 epilogue,
// warp 4 TMA producer, warp 5 TMEM owner and, on the leader, MMA issuer,
// warp 6 fix-up):
//   producer (both)  loads its own 128-row halves of the a and b chunks into
//                    its own ring slot, counted on its own full barrier;
//   fix-up (both)    waits for its slot, zeroes the bytes outside the group
//                    in the chunk's edge K slices (as the one-SM kernel's
//                    MMA warp does), fences the async proxy and arrives on
//                    the leader's ready barrier (count 2, one per CTA);
//   leader lane 0    waits on the ready barrier alone (no warp-wide step
//                    between chunks: the gap between one chunk's last MMA
//                    and the next one's first is the tensor pipe's idle
//                    time), issues the pair's MMAs (M 256, N 256, K 32) for
//   of warp 5        the K slices that hold group positions, and commits to
//                    both CTAs' empty barriers and, per tile, both
//                    accumulator barriers (tcgen05.commit multicast, mask
//                    0b11);
//   epilogue (both)  drains its own 128 TMEM lanes x 256 columns, scales,
//                    rounds, stores, and arrives on the leader's
//                    accumulator-empty barrier (count 8).
// Every TMA load fills the loading CTA's own shared memory. Every wait is
// bounded; a CTA that gives up records MXQ_ERR_TIMEOUT and stops its roles,
// and both meet at the closing cluster barrier before TMEM is freed.
#pragma once

#include "gemm.cuh"

namespace mxq {
namespace g2 {

constexpr int HALF = 128;              // rows of a and of b per CTA
constexpr int BM = 2 * HALF;           // a rows per pair tile
constexpr int BN = 2 * HALF;           // b rows per pair tile
constexpr int BK = gm::BK;             // positions per chunk
constexpr int STAGES = 6;
constexpr int A_BYTES = HALF * BK;     // 16 KB
constexpr int B_BYTES = HALF * BK;     // 16 KB
constexpr int EPI_WARPS = 4;
constexpr int THREADS = 7 * 32;
constexpr int ACC = 2;
constexpr int TMEM_COLS = ACC * BN;    // 512

struct __align__(1024) Smem {
    uint8_t a[STAGES][A_BYTES];
    uint8_t b[STAGES][B_BYTES];
    uint64_t full[STAGES];
    uint64_t ready[STAGES];
    uint64_t empty[STAGES];
    uint64_t acc_full[ACC];
    uint64_t acc_empty[ACC];
    uint64_t mma_done;
    uint32_t tmem_base;
    int abort_flag;
};
constexpr size_t SMEM_BYTES = sizeof(Smem) + 1024;

// M 256 (the pair), N 256, fp32 accumulator, e4m3 x e4m3, both K-major
constexpr uint32_t IDESC = (1u << 4) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

MXQ_DEV uint32_t cta_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

MXQ_DEV void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// shared::cluster address of the same shared variable in CTA `rank`
MXQ_DEV uint32_t peer_addr(const void *p, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
    return r;
}

// arrive on a barrier of another CTA of the cluster (the default
// semantics: release at CTA scope, no cluster-wide fence)
MXQ_DEV void arrive_remote(uint32_t cluster_addr)
{
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// the same, releasing this thread's prior writes at cluster scope (a fence
// that costs about half a microsecond: only after shared-memory writes the
// other CTA's MMAs will read)
MXQ_DEV void arrive_remote_release(uint32_t cluster_addr)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

MXQ_DEV void mma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %3, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %4, p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(accumulate), "r"(IDESC)
        : "memory");
}

// arrive on `bar` (same offset) in every CTA of `mask` once the pair MMAs
// this thread issued before have completed
MXQ_DEV void commit_pair(uint64_t *bar, uint16_t mask)
{
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
                 ::"r"(smem_u32(bar)), "h"(mask)
                 : "memory");
}

} // namespace g2

// a (N, lda) and b (K, ldb) K-major e4m3 through tm_a, tm_b (boxes of 128
// positions x 128 rows, 128-byte swizzle); N % 256 == 0, K % 256 == 0; grid
// = an even number of CTAs in clusters of two
__global__ void __launch_bounds__(g2::THREADS, 1)
    k_fp8_grouped_gemm_wgrad_2sm(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                                 const float *__restrict__ inv_a, const float *__restrict__ inv_b, int64_t N,
                                 int64_t K, int64_t M, const int32_t *__restrict__ offs, int G,
                                 uint16_t *__restrict__ out, uint64_t wait_ns)
{
    using namespace g2;
    extern __shared__ uint8_t smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cta_rank();
    const bool leader = rank == 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.ready[s], 2);
            mbar_init(&sm.empty[s], 1);
        }
        for (int i = 0; i < ACC; ++i) {
            mbar_init(&sm.acc_full[i], 1);
            mbar_init(&sm.acc_empty[i], 2 * EPI_WARPS);
        }
        mbar_init(&sm.mma_done, 1);
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    // both CTAs see the same offsets and take the same exit
    if (!offsets_ok(offs, G, M))
        return;
    if (warp == 5) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem_base)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    gm::tc_fence_before();
    cluster_sync(); // barriers initialised and TMEM allocated in both CTAs
    gm::tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    const int64_t pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int64_t ntn = N / BM, ktn = K / BN;
    const int64_t per_g = ntn * ktn, total = per_g * G;
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
        q.x0 = q.s & ~int64_t(BK - 1);
        q.nch = q.e > q.s ? (q.e - q.x0 + BK - 1) / BK : 0;
        return q;
    };
    // this chunk's group positions [lo, hi) and the K-32 slices holding them;
    // zero this CTA's bytes outside the group in the two edge slices
    // (returns whether it wrote)
    auto fixup = [&](const Item &q, int64_t j, int s, int &k_lo, int &k_hi) {
        const int64_t c0 = q.x0 + j * BK;
        const int lo = (int)max((int64_t)0, q.s - c0), hi = (int)min((int64_t)BK, q.e - c0);
        k_lo = lo >> 5;
        k_hi = (hi + 31) >> 5;
        if ((lo & 31) || (hi & 31)) {
            gm::zero_cols(sm.a[s], HALF, 32 * k_lo, lo);
            gm::zero_cols(sm.a[s], HALF, hi, 32 * k_hi);
            gm::zero_cols(sm.b[s], HALF, 32 * k_lo, lo);
            gm::zero_cols(sm.b[s], HALF, hi, 32 * k_hi);
            fence_proxy_async_smem();
            return true;
        }
        return false;
    };

    if (warp == 4) {
        // ------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            int seq = 0;
            for (int64_t it = pair; it < total && !gm::aborted(&sm.abort_flag); it += npairs) {
                const Item q = item(it);
                for (int64_t j = 0; j < q.nch; ++j, ++seq) {
                    const int s = seq % STAGES;
                    if (seq >= STAGES && !mbar_wait(&sm.empty[s], ((uint32_t)(seq / STAGES) & 1u) ^ 1u, wait_ns)) {
                        *reinterpret_cast<volatile int *>(&sm.abort_flag) = 1;
                        break;
                    }
                    mbar_arrive_expect_tx(&sm.full[s], A_BYTES + B_BYTES);
                    const int x = (int)(q.x0 + j * BK);
                    tma_load_2d(sm.a[s], &tm_a, &sm.full[s], x, (int)(q.nt * BM + rank * HALF));
                    tma_load_2d(sm.b[s], &tm_b, &sm.full[s], x, (int)(q.kt * BN + rank * HALF));
                }
            }
            // drain: every issued fill has landed before the CTA leaves
            for (int j = seq - STAGES; j < seq; ++j)
                if (j >= 0)
                    mbar_wait(&sm.full[j % STAGES], (uint32_t)(j / STAGES) & 1u, wait_ns);
        }
    } else if (warp == 6) {
        // ------------------------------------------------ fix-up and hand-off (both CTAs)
        const uint32_t leader_ready0 = peer_addr(&sm.ready[0], 0);
        int seq = 0;
        for (int64_t it = pair; it < total && !gm::aborted(&sm.abort_flag); it += npairs) {
            const Item q = item(it);
            bool ok = true;
            for (int64_t j = 0; j < q.nch; ++j, ++seq) {
                const int s = seq % STAGES;
                ok = __all_sync(0xffffffffu, mbar_wait(&sm.full[s], (uint32_t)(seq / STAGES) & 1u, wait_ns));
                if (!ok)
                    break;
                int k_lo, k_hi;
                const bool wrote = fixup(q, j, s, k_lo, k_hi);
                __syncwarp();
                if (lane == 0) {
                    // the slot's bytes came by TMA, which this warp's wait
                    // observed; only zeroed bytes need the cluster release
                    const uint32_t bar = leader_ready0 + (uint32_t)(s * sizeof(uint64_t));
                    if (wrote)
                        arrive_remote_release(bar);
                    else
                        arrive_remote(bar);
                }
                __syncwarp();
            }
            if (!ok) {
                *reinterpret_cast<volatile int *>(&sm.abort_flag) = 1;
                break;
            }
        }
    } else if (warp == 5) {
        // ------------------------------------------------ leader: the pair's MMAs (one thread)
        if (leader && lane == 0) {
            int t = 0, s = 0;
            uint32_t ph = 0; // phase parity of slot s
            bool issued = false;
            for (int64_t it = pair; it < total && !gm::aborted(&sm.abort_flag); it += npairs) {
                const Item q = item(it);
                if (q.nch == 0)
                    continue;
                const int acc = t & 1;
                if (t >= ACC && !mbar_wait(&sm.acc_empty[acc], ((uint32_t)(t / ACC) & 1u) ^ 1u, wait_ns)) {
                    *reinterpret_cast<volatile int *>(&sm.abort_flag) = 1;
                    break;
                }
                gm::tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(acc * BN);
                // the next chunk's ready barrier is waited on between this
                // chunk's last two MMAs, so that the wait (and the loop
                // around it) overlaps MMAs already queued in the tensor pipe
                bool ok = mbar_wait(&sm.ready[s], ph, wait_ns);
                int64_t c0 = q.x0;
                for (int64_t j = 0; ok && j < q.nch; ++j, c0 += BK) {
                    gm::tc_fence_after();
                    const int lo = (int)max((int64_t)0, q.s - c0), hi = (int)min((int64_t)BK, q.e - c0);
                    const int k_lo = lo >> 5, k_last = ((hi + 31) >> 5) - 1;
                    const uint64_t ad = gm::smem_desc_k128(smem_u32(sm.a[s]));
                    const uint64_t bd = gm::smem_desc_k128(smem_u32(sm.b[s]));
#pragma unroll
                    for (int k = 0; k < BK / 32; ++k)
                        if (k >= k_lo && k < k_last)
                            mma_pair(d, ad + 2 * k, bd + 2 * k, (j > 0 || k > k_lo) ? 1u : 0u);
                    const int s_next = s + 1 == STAGES ? 0 : s + 1;
                    const uint32_t ph_next = s + 1 == STAGES ? ph ^ 1u : ph;
                    if (j + 1 < q.nch)
                        ok = mbar_wait(&sm.ready[s_next], ph_next, wait_ns);
                    mma_pair(d, ad + 2 * k_last, bd + 2 * k_last, (j > 0 || k_last > k_lo) ? 1u : 0u);
                    commit_pair(&sm.empty[s], 0x3);
                    issued = true;
                    s = s_next;
                    ph = ph_next;
                }
                if (!ok) {
                    *reinterpret_cast<volatile int *>(&sm.abort_flag) = 1;
                    break;
                }
                commit_pair(&sm.acc_full[acc], 0x3);
                ++t;
            }
            if (issued) { // every issued MMA completes before TMEM is freed
                commit_pair(&sm.mma_done, 0x1);
                mbar_wait(&sm.mma_done, 0u, wait_ns);
            }
        }
        __syncwarp();
    } else if (warp < EPI_WARPS) {
        // ------------------------------------------------ epilogue (both CTAs)
        const uint32_t leader_acc_empty0 = peer_addr(&sm.acc_empty[0], 0);
        int t = 0;
        for (int64_t it = pair; it < total; it += npairs) {
            const Item q = item(it);
            const int64_t n = q.nt * BM + rank * HALF + 32 * warp + lane; // this thread's output row
            uint16_t *dst = out + ((int64_t)q.g * N + n) * K + q.kt * BN;
            if (q.nch == 0) { // empty group: the sum is zero
                for (int c = 0; c < BN; c += 8)
                    st_v4(dst + c, 0u, 0u, 0u, 0u);
                continue;
            }
            const int acc = t & 1;
            bool ok = mbar_wait(&sm.acc_full[acc], (uint32_t)(t / ACC) & 1u, wait_ns);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok || gm::aborted(&sm.abort_flag)) {
                *reinterpret_cast<volatile int *>(&sm.abort_flag) = 1;
                break;
            }
            gm::tc_fence_after();
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
                gm::tc_ld32(tmem + (uint32_t)(acc * BN + c * 32) + ((uint32_t)(32 * warp) << 16), r);
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
                    pk[j] = gm::pack_bf16x2(v0, v1);
                }
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    st_v4(dst + c * 32 + 8 * j, pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
            }
            gm::tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (leader)
                    mbar_arrive(&sm.acc_empty[acc]);
                else
                    arrive_remote(leader_acc_empty0 + (uint32_t)(acc * sizeof(uint64_t)));
            }
            ++t;
        }
    }

    __syncwarp(); // the cluster barrier below is warp-aligned
    gm::tc_fence_before();
    cluster_sync(); // the pair's MMAs and both epilogues are done
    gm::tc_fence_after();
    if (warp == 5)
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
}

} // namespace mxq
