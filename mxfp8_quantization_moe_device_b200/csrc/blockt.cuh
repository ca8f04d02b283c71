// blockt.cuh - fp8 blockwise quantization with transposed output (ao PR 2827
// "[fp8 blockwise] load 2d chunks for groupwise quant to enable coalesced
// gmem accesses", description: the (blocksize x 1) tiles of the blockwise
// linear, whose right-hand operands are consumed column-major).
//
// A row-major (rows, cols) bf16 matrix is quantized in 128 x bc blocks,
// bc = 1 (one scale per 128 rows of a column: the activations as the right
// operand of the weight-gradient GEMM) or bc = 128 (the weight, transposed
// for the input-gradient GEMM), and written transposed: out[c * rows + r];
// the inverse scales form the (cols / bc, rows / 128) row-major matrix of the
// transpose.
//
// Design (the MX 3-D kernel's structure): a persistent grid, 2 CTAs per SM,
// walks 128 x 128 work items, column tiles fastest. A producer warp streams
// each item as two 128-row x 64-column TMA boxes through a 4-stage ring; four
// consumer warps own 32 rows each, a lane two adjacent columns of each half.
// The block amax is a packed bf16 max over the lane's 32 rows, then a
// shared-memory step across the four warps (per column for bc = 1, over the
// whole item for bc = 128). The e4m3 bytes leave through 128B-swizzled
// staging tiles (64 columns x 128 rows each) and TMA stores of the transpose.
#pragma once

#include "common.cuh"

namespace mxq {
namespace bt {

constexpr int TR = 128;              // rows per item (one block height)
constexpr int TH = 64;               // columns per half (one TMA box)
constexpr int STAGES = 4;            // two items in flight
constexpr int CWARPS = 4;
constexpr int THREADS = (CWARPS + 1) * 32;
constexpr int IN_BYTES = TR * TH * 2;  // 16 KB per half
constexpr int OUT_BYTES = TH * TR;     // 8 KB per staged half
constexpr int CTAS_PER_SM = 2;

struct __align__(1024) Smem {
    uint8_t in[STAGES][IN_BYTES];
    uint8_t out[2][2][OUT_BYTES]; // [buffer][half]
    float red[CWARPS][2 * TH];    // per-warp partial amax of each column
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    int abort_flag;
};

constexpr size_t SMEM_BYTES = sizeof(Smem) + 1024;

} // namespace bt

__global__ void __launch_bounds__(bt::THREADS, bt::CTAS_PER_SM)
    k_fp8_blockwise_t(const __grid_constant__ CUtensorMap tm_in, const __grid_constant__ CUtensorMap tm_out,
                      float *__restrict__ inv, int64_t rows, int64_t cols, int bc, uint64_t wait_ns)
{
    using namespace bt;
    extern __shared__ uint8_t smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // item t = (row tile t / tiles_c, column tile t % tiles_c); the host
    // guarantees fewer than 2^31 items
    const uint32_t tiles_r = (uint32_t)(rows / TR), tiles_c = (uint32_t)(cols / (2 * TH));
    const uint32_t total = tiles_r * tiles_c;

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
            int seq = 0;
            bool stop = false;
            for (uint32_t t = blockIdx.x; t < total && !stop; t += gridDim.x) {
                const uint32_t rt = t / tiles_c, ct = t - rt * tiles_c;
                for (int h = 0; h < 2; ++h, ++seq) {
                    const int s = seq % STAGES;
                    if (seq >= STAGES && !mbar_wait(&sm.empty[s], ((uint32_t)(seq / STAGES) & 1u) ^ 1u, wait_ns)) {
                        stop = true;
                        break;
                    }
                    mbar_arrive_expect_tx(&sm.full[s], IN_BYTES);
                    tma_load_2d(sm.in[s], &tm_in, &sm.full[s], (int)(ct * 2 * TH + h * TH), (int)(rt * TR));
                }
            }
            // drain: every issued fill lands before the CTA exits
            for (int j = seq - STAGES; j < seq; ++j)
                if (j >= 0)
                    mbar_wait(&sm.full[j % STAGES], (uint32_t)(j / STAGES) & 1u, wait_ns);
        }
        return;
    }

    // ---------------------------------------------------- consumer warps
    const int w = warp; // rows 32w .. 32w+31 of the item
    const int64_t rblocks = rows / TR;
    int it = 0;
    for (uint32_t t = blockIdx.x; t < total; t += gridDim.x, ++it) {
        const uint32_t rt = t / tiles_c, ct = t - rt * tiles_c;
        const int ob = it & 1;
        // both halves: 32 rows x 2 columns each, and their packed |max|
        uint32_t v[2][32];
        uint32_t acc[2] = {0u, 0u};
        bool ok = true;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int seq = 2 * it + h, s = seq % STAGES;
            ok = mbar_wait(&sm.full[s], (uint32_t)(seq / STAGES) & 1u, wait_ns) && ok;
            const uint32_t *tile = reinterpret_cast<const uint32_t *>(sm.in[s]);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                v[h][i] = tile[(w * 32 + i) * (TH / 2) + lane];
                acc[h] = absmax_bf16x2(acc[h], v[h][i]);
            }
            // the stage is free once every word read from it has been used
            release_slot_after(&sm.empty[s], acc[h]);
        }
        ok = __all_sync(0xffffffffu, ok);
        if (!ok)
            sm.abort_flag = 1;

        // block amax: per column (bc = 1) or over the whole item (bc = 128)
        float sc[4]; // scales of columns 2*lane, 2*lane+1 of half 0, then half 1
        if (bc == 1) {
            sm.red[w][2 * lane] = bf16_lo(acc[0]);
            sm.red[w][2 * lane + 1] = bf16_hi(acc[0]);
            sm.red[w][TH + 2 * lane] = bf16_lo(acc[1]);
            sm.red[w][TH + 2 * lane + 1] = bf16_hi(acc[1]);
            named_barrier(1, CWARPS * 32);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int c = (k >> 1) * TH + 2 * lane + (k & 1);
                float a = sm.red[0][c];
#pragma unroll
                for (int q = 1; q < CWARPS; ++q)
                    a = fmaxf(a, sm.red[q][c]);
                sc[k] = fp8_scale(a);
            }
            if (w == 0) {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int64_t c = (int64_t)ct * 2 * TH + (k >> 1) * TH + 2 * lane + (k & 1);
                    inv[c * rblocks + rt] = fp8_inv(sc[k]);
                }
            }
        } else {
            float a = fmaxf(fmaxf(bf16_lo(acc[0]), bf16_hi(acc[0])), fmaxf(bf16_lo(acc[1]), bf16_hi(acc[1])));
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1)
                a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
            if (lane == 0)
                sm.red[w][0] = a;
            named_barrier(1, CWARPS * 32);
            a = fmaxf(fmaxf(sm.red[0][0], sm.red[1][0]), fmaxf(sm.red[2][0], sm.red[3][0]));
            const float s = fp8_scale(a);
            sc[0] = sc[1] = sc[2] = sc[3] = s;
            if (threadIdx.x == 0)
                inv[(int64_t)ct * rblocks + rt] = fp8_inv(s);
        }

        // staging buffer ob was last read by the TMA stores of item it-2
        if (threadIdx.x == 0)
            bulk_wait_read<1>();
        named_barrier(1, CWARPS * 32);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float s0 = sc[2 * h], s1 = sc[2 * h + 1];
            uint32_t q0[8], q1[8]; // column 2*lane and 2*lane+1: 32 row bytes each
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t *r = v[h] + 4 * j;
                q0[j] = e4m3x2(__fmul_rn(bf16_lo(r[0]), s0), __fmul_rn(bf16_lo(r[1]), s0)) |
                        (e4m3x2(__fmul_rn(bf16_lo(r[2]), s0), __fmul_rn(bf16_lo(r[3]), s0)) << 16);
                q1[j] = e4m3x2(__fmul_rn(bf16_hi(r[0]), s1), __fmul_rn(bf16_hi(r[1]), s1)) |
                        (e4m3x2(__fmul_rn(bf16_hi(r[2]), s1), __fmul_rn(bf16_hi(r[3]), s1)) << 16);
            }
            // staging: 64 rows (columns of the input) x 128 bytes (its rows),
            // 16-byte chunk c of row r at chunk c ^ (r & 7) (128B swizzle); the
            // lane's two columns alternate so each store hits 8 bank groups
            const uint32_t ob_addr = smem_u32(sm.out[ob][h]);
            const int bsel = (lane >> 2) & 1;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int b = bsel ^ (j & 1), hh = j >> 1;
                const int row = 2 * lane + b;
                const int chunk = (2 * w + hh) ^ (row & 7);
                uint4 val;
                if (b) val = make_uint4(q1[4 * hh], q1[4 * hh + 1], q1[4 * hh + 2], q1[4 * hh + 3]);
                else   val = make_uint4(q0[4 * hh], q0[4 * hh + 1], q0[4 * hh + 2], q0[4 * hh + 3]);
                sts_v4(ob_addr + row * 128 + chunk * 16, val);
            }
        }
        fence_proxy_async_smem();
        if (barrier_or(1, CWARPS * 32, sm.abort_flag != 0))
            break;
        if (threadIdx.x == 0) {
            tma_store_2d(&tm_out, sm.out[ob][0], (int)(rt * TR), (int)(ct * 2 * TH));
            tma_store_2d(&tm_out, sm.out[ob][1], (int)(rt * TR), (int)(ct * 2 * TH + TH));
            bulk_commit();
        }
    }
    if (threadIdx.x == 0)
        bulk_wait<0>();
}

} // namespace mxq
