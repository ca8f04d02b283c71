// mx3d.cuh - MXFP8 quantization of 3-D expert weights (E, N, K) along N in
// 32x1 blocks, written straight into each expert's column-major layout
// (ao PR 3002 "[mxfp8 moe training] add CUDA kernel to quantize 3d tensor
// colwise", Summary), E8M0 scales in floor or rceil mode (same page,
// comments).
//
// Design (differs from the page's one-descriptor-pair-per-expert scheme):
//   * one rank-3 TMA map covers all experts for loads (K, N, E) and one for
//     stores (N, K, E), so host work is O(1) in E;
//   * a persistent grid (2 CTAs per SM) walks (expert, n-tile, k-tile) work
//     items with k fastest, so E = 1 fills the GPU as well as E = 64;
//   * per CTA: one producer warp drives a 4-stage TMA ring of 128 x 64 bf16
//     tiles (16 KB); four consumer warps each own one 32-row MX block of a
//     tile, a lane owning two adjacent columns. Each lane keeps its 32 x 2
//     values in registers, takes the block amax with packed bf16 max,
//     converts to E8M0 and e4m3, and writes its two 32-byte column runs into
//     a 128B-swizzled staging tile that a TMA store writes out as 64 rows of
//     128 contiguous bytes (the transpose happens in shared memory);
//   * the staging writes alternate the lane's two columns so that every
//     16-byte shared store instruction hits eight distinct bank groups.
#pragma once

#include "common.cuh"

namespace mxq {
namespace mx3d {

constexpr int TN = 128;              // n rows per tile (four 32-row MX blocks)
constexpr int TK = 64;               // k columns per tile
constexpr int STAGES = 4;
constexpr int CWARPS = 4;            // consumer warps (one per MX block)
constexpr int THREADS = (CWARPS + 1) * 32;
constexpr int IN_BYTES = TN * TK * 2;  // 16384
constexpr int OUT_BYTES = TN * TK;     // 8192
constexpr int CTAS_PER_SM = 2;

struct __align__(1024) Smem {
    uint8_t in[STAGES][IN_BYTES];
    uint8_t out[2][OUT_BYTES];
    uint8_t sc[2][TK][4]; // scale bytes: [k][n-block]
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    int abort_flag;
};

constexpr size_t SMEM_BYTES = sizeof(Smem) + 1024; // + manual 1 KB alignment

__global__ void __launch_bounds__(THREADS, CTAS_PER_SM)
    k_mx_3d_colwise(const __grid_constant__ CUtensorMap tm_in, const __grid_constant__ CUtensorMap tm_out,
                    uint8_t *__restrict__ scales, int E, int N, int K, int tiles_n, int tiles_k, int mode,
                    uint64_t wait_ns)
{
    extern __shared__ uint8_t smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t per_e = (int64_t)tiles_n * tiles_k;
    const int64_t total = per_e * E;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], CWARPS);
        }
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == CWARPS) {
        // ------------------------------------------------ producer warp
        if (lane == 0) {
            int it = 0;
            for (int64_t t = blockIdx.x; t < total; t += gridDim.x, ++it) {
                const int s = it % STAGES;
                const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
                if (it >= STAGES && !mbar_wait(&sm.empty[s], ph ^ 1u, wait_ns))
                    break;
                const int e = (int)(t / per_e);
                const int64_t rem = t - (int64_t)e * per_e;
                const int nt = (int)(rem / tiles_k), kt = (int)(rem % tiles_k);
                mbar_arrive_expect_tx(&sm.full[s], IN_BYTES);
                tma_load_3d(sm.in[s], &tm_in, &sm.full[s], kt * TK, nt * TN, e);
            }
            // drain: every stage's latest fill must land before the CTA exits
            const int issued = it;
            for (int j = issued - STAGES; j < issued; ++j) {
                if (j < 0)
                    continue;
                mbar_wait(&sm.full[j % STAGES], (uint32_t)(j / STAGES) & 1u, wait_ns);
            }
        }
        return;
    }

    // ---------------------------------------------------- consumer warps
    const int w = warp; // MX block within the tile: rows 32w .. 32w+31
    const int nblk_n = N / 32;
    int it = 0;
    for (int64_t t = blockIdx.x; t < total; t += gridDim.x, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
        const int ob = it & 1;
        const int e = (int)(t / per_e);
        const int64_t rem = t - (int64_t)e * per_e;
        const int nt = (int)(rem / tiles_k), kt = (int)(rem % tiles_k);

        bool ok = mbar_wait(&sm.full[s], ph, wait_ns);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok)
            sm.abort_flag = 1;

        // 32 rows x 2 columns of this lane, and their packed |max|
        const uint32_t *tile = reinterpret_cast<const uint32_t *>(sm.in[s]);
        uint32_t v[32];
        uint32_t acc = 0;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            v[i] = tile[(w * 32 + i) * (TK / 2) + lane];
            acc = absmax_bf16x2(acc, v[i]);
        }
        // release the input stage once every loaded word has been consumed
        // (acc depends on all 32 of them)
        release_slot_after(&sm.empty[s], acc);

        const float a0 = bf16_lo(acc), a1 = bf16_hi(acc);
        const uint32_t b0 = e8m0_mode(a0, mode), b1 = e8m0_mode(a1, mode);
        const float f0 = mx_factor(b0), f1 = mx_factor(b1);
        uint32_t q0[8], q1[8]; // column 2*lane and 2*lane+1, 32 bytes each
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

        // out staging: 64 rows (k) x 128 bytes (n), 16-byte chunk c of row
        // r stored at chunk c ^ (r & 7) (the TMA 128-byte swizzle)
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
        sm.sc[ob][2 * lane][w] = (uint8_t)b0;
        sm.sc[ob][2 * lane + 1][w] = (uint8_t)b1;
        fence_proxy_async_smem();
        if (barrier_or(1, CWARPS * 32, sm.abort_flag != 0))
            break;

        if (threadIdx.x == 0) {
            tma_store_3d(&tm_out, sm.out[ob], nt * TN, kt * TK, e);
            bulk_commit();
        }
        // scale bytes: row k gets blocks 4nt .. 4nt+3 of (E, K, N/32)
        if (threadIdx.x < TK) {
            const int k = kt * TK + threadIdx.x;
            const int nb0 = nt * 4;
            if (k < K) {
                uint8_t *dst = scales + ((int64_t)e * K + k) * nblk_n + nb0;
                const uint8_t *src = sm.sc[ob][threadIdx.x];
                if (nb0 + 4 <= nblk_n && (nblk_n & 3) == 0) {
                    *reinterpret_cast<uint32_t *>(dst) = *reinterpret_cast<const uint32_t *>(src);
                } else {
                    for (int i = 0; i < 4; ++i)
                        if (nb0 + i < nblk_n)
                            dst[i] = src[i];
                }
            }
        }
    }
    if (threadIdx.x == 0)
        bulk_wait<0>();
}

} // namespace mx3d
} // namespace mxq
