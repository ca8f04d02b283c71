/*
 * mxq.h - C ABI of libmxq, the sm_100a (B200) library for the dynamic
 * low-precision quantization path that feeds scaled grouped GEMMs in
 * mixture-of-experts training.
 *
 * Sources, pytorch/ao pull-request pages:
 *   #2064 "[scaled grouped mm] add triton kernels for float8 rowwise
 *          quantization with per-group/jagged scales" (Motivation, Summary)
 *   #2827 "[fp8 blockwise] load 2d chunks for groupwise quant to enable
 *          coalesced gmem accesses" (description, Kernel performance)
 *   #3002 "[mxfp8 moe training] add CUDA kernel to quantize 3d tensor
 *          colwise" (Summary, comments)
 *   #3504 "[mxfp8 moe training] add CUDA kernel for per-group conversion of
 *          scale factors to blocked layout" (title, Benchmarks)
 *
 * Conventions shared by every entry point
 *   - Pointers are DEVICE pointers, owned by the caller; the library never
 *     frees or retains them. bf16 inputs are raw 16-bit words; float8 e4m3
 *     and E8M0 outputs are raw bytes; scales written as fp32 are the
 *     INVERSE scales (multiply the e4m3 value by them to dequantize).
 *   - Work is enqueued on `stream`; nothing synchronizes the host, and the
 *     group offsets are never read on the host.
 *   - Calls return MXQ_OK after a successful enqueue. A call with no
 *     elements to process returns MXQ_OK without launching, and its data
 *     pointers may then be NULL. Problems visible on
 *     the host (null pointer, bad shape, misalignment, small workspace) are
 *     returned at once and nothing is launched. Problems only visible on the
 *     device (malformed offsets, an expired wait) are recorded in a device
 *     status word that mxq_device_status() reads and clears; in that case the
 *     kernel writes none of its outputs (offsets) or stops early (timeout).
 *   - Entry points are reentrant and may be called from several host
 *     threads; calls on different streams run concurrently.
 *   - Offsets: int32, `num_groups` cumulative group ENDS along the grouped
 *     dimension: group g covers [offs[g-1], offs[g]) with offs[-1] = 0.
 *     They must be non-decreasing and lie in [0, extent]. Empty groups are
 *     allowed; elements past offs[num_groups-1] are not written.
 *
 * Numerics (bit-exact, no tolerance; every rule is computed in fp32):
 *   e4m3 unit scale  s = 448 / max(amax, 1e-12f), stored inverse = 1 / s,
 *                    element = e4m3(clamp(x * s)), round to nearest even.
 *   MX (E8M0)        floor: 2^(floor(log2 amax) - 8);
 *                    rceil: 2^ceil(log2(amax / 448)); both clamped to
 *                    [2^-127, 2^127]; element = e4m3(x / scale).
 */
#ifndef MXQ_H
#define MXQ_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum mxq_status {
    MXQ_OK = 0,
    MXQ_ERR_NULL = 1,        /* a required pointer is NULL                      */
    MXQ_ERR_SHAPE = 2,       /* negative / non-divisible sizes                  */
    MXQ_ERR_ALIGN = 3,       /* pointer or stride misaligned for the op         */
    MXQ_ERR_UNSUPPORTED = 4, /* parameter combination not implemented           */
    MXQ_ERR_LAUNCH = 5,      /* the CUDA launch failed                          */
    MXQ_ERR_BAD_OFFSETS = 6, /* device: offsets decreasing, negative or > extent */
    MXQ_ERR_TIMEOUT = 7,     /* device: a bounded wait expired                  */
    MXQ_ERR_WORKSPACE = 8,   /* workspace missing or smaller than required      */
    MXQ_ERR_CUDA = 9         /* another CUDA runtime error                      */
} mxq_status;

typedef enum mxq_scale_mode {
    MXQ_E8M0_FLOOR = 0,
    MXQ_E8M0_RCEIL = 1
} mxq_scale_mode;

/* ------------------------------------------------------------------------ *
 * (a1) fp8_quant_jagged_rowwise - #2064 Summary, first kernel: float8 e4m3
 * quantization with one scale per (row, group), the groups being column
 * ranges given by `offs`, output row-major. Used on the left operand of the
 * grad_weight grouped GEMM (grad_out^T).
 *   in          logical (rows, cols) bf16; element (r, c) at
 *               in[r * stride_row + c * stride_col] (strides in elements).
 *               The transposed view of a row-major (M, N) tensor has
 *               stride_row = 1, stride_col = N and takes the fast path.
 *   offs        num_groups int32 ends along cols (device).
 *   out         rows x cols e4m3 bytes, row-major: out[r * cols + c].
 *   inv_scales  fp32 (num_groups, rows): inv_scales[g * rows + r].
 *   workspace   device scratch of at least
 *               fp8_quant_jagged_workspace_bytes(rows, cols, stride_row,
 *               stride_col, num_groups) bytes (may be NULL when that is 0);
 *               it is cleared and used by the call, so concurrent calls need
 *               distinct workspaces.
 * ------------------------------------------------------------------------ */
int fp8_quant_jagged_rowwise(const void *in, int64_t rows, int64_t cols,
                             int64_t stride_row, int64_t stride_col,
                             const int32_t *offs, int32_t num_groups,
                             void *out, float *inv_scales,
                             void *workspace, size_t workspace_bytes,
                             cudaStream_t stream);

/* ------------------------------------------------------------------------ *
 * (a2) fp8_quant_jagged_colwise - #2064 Summary, second kernel: one scale per
 * (column, group), the groups being row ranges, output column-major. Used on
 * the right operand of the grad_weight grouped GEMM (input).
 *   in          logical (rows, cols) bf16 with element strides; row-major
 *               (stride_row = cols, stride_col = 1) takes the fast path.
 *   offs        num_groups int32 ends along rows (device).
 *   out         column-major e4m3: out[c * rows + r].
 *   inv_scales  fp32 (num_groups, cols): inv_scales[g * cols + c].
 *   workspace   as for the rowwise op.
 * Rowwise on the transposed view of A and colwise on A give byte-identical
 * buffers and scales.
 * ------------------------------------------------------------------------ */
int fp8_quant_jagged_colwise(const void *in, int64_t rows, int64_t cols,
                             int64_t stride_row, int64_t stride_col,
                             const int32_t *offs, int32_t num_groups,
                             void *out, float *inv_scales,
                             void *workspace, size_t workspace_bytes,
                             cudaStream_t stream);

/* Workspace size for the jagged ops with these arguments (rowwise: pass the
 * rowwise shape and strides; colwise: the colwise ones, with is_colwise = 1).
 * Returns 0 when the call needs none. Depends only on the layout, so it may
 * be larger than a particular call uses (small problems run a kernel that
 * needs no workspace). */
size_t fp8_quant_jagged_workspace_bytes(int64_t rows, int64_t cols,
                                        int64_t stride_row, int64_t stride_col,
                                        int32_t num_groups, int32_t is_colwise);

/* ------------------------------------------------------------------------ *
 * (a3) fp8_quant_blockwise - #2827: one e4m3 scale per block of a row-major
 * (rows, cols) bf16 matrix; block 1 x 128 (activations) or 128 x 128
 * (weights).
 *   block_rows  1 or 128; block_cols 128. rows % block_rows == 0,
 *               cols % 128 == 0, else MXQ_ERR_SHAPE / MXQ_ERR_UNSUPPORTED.
 *   in, out     16-byte aligned; out row-major e4m3 (rows, cols).
 *   inv_scales  fp32 row-major (rows / block_rows, cols / 128).
 * ------------------------------------------------------------------------ */
int fp8_quant_blockwise(const void *in, int64_t rows, int64_t cols,
                        int32_t block_rows, int32_t block_cols,
                        void *out, float *inv_scales, cudaStream_t stream);

/* ------------------------------------------------------------------------ *
 * fp8_quant_blockwise_transposed - #2827 description (the blocksize x 1
 * tiles of the blockwise linear): e4m3 with one scale per 128 x block_cols
 * block of a row-major (rows, cols) bf16 matrix, written TRANSPOSED.
 *   block_rows  128; block_cols 1 (activations as the column-major right
 *               operand) or 128 (the transposed weight); else
 *               MXQ_ERR_UNSUPPORTED. rows % 128 == 0 and cols % 128 == 0,
 *               else MXQ_ERR_SHAPE.
 *   in, out     16-byte aligned; out[c * rows + r], i.e. (cols, rows)
 *               row-major.
 *   inv_scales  fp32 (cols / block_cols, rows / 128) row-major: the scale
 *               matrix of the transpose. The result equals
 *               fp8_quant_blockwise on the contiguous transpose with blocks
 *               block_cols x 128.
 * ------------------------------------------------------------------------ */
int fp8_quant_blockwise_transposed(const void *in, int64_t rows, int64_t cols,
                                   int32_t block_rows, int32_t block_cols,
                                   void *out, float *inv_scales, cudaStream_t stream);

/* ------------------------------------------------------------------------ *
 * fp8_grouped_gemm_rowwise - the consumer of these buffers (#2064
 * Motivation, #2077 Summary: the scaled grouped mm the quantization feeds):
 * a grouped GEMM on the tensor cores (tcgen05, fp32 accumulation in TMEM)
 *   out[m][n] = bf16((sum_k a[m][k] * w[g][n][k]) * inv_a[m] * inv_w[g][n])
 * for each row m of group g = [offs[g-1], offs[g]).
 *   a       e4m3 (M, K) row-major (K contiguous), 16-byte aligned.
 *   inv_a   fp32 (M): per-row inverse scales (fp8_quant_jagged_rowwise of A
 *           with one group spanning K).
 *   w       e4m3 (num_groups, N, K) row-major, 16-byte aligned.
 *   inv_w   fp32 (num_groups, N): per-(expert, row) inverse scales.
 *   offs    num_groups int32 ends along M (device).
 *   out     bf16 (M, N) row-major, 16-byte aligned; rows past
 *           offs[num_groups-1] are not written.
 *   N % 128 == 0 and K % 128 == 0 (K > 0), else MXQ_ERR_SHAPE;
 *   num_groups <= 4096, else MXQ_ERR_UNSUPPORTED.
 * ------------------------------------------------------------------------ */
int fp8_grouped_gemm_rowwise(const void *a, const float *inv_a, const void *w, const float *inv_w,
                             int64_t M, int64_t N, int64_t K,
                             const int32_t *offs, int32_t num_groups, void *out,
                             cudaStream_t stream);

/* fp8_grouped_gemm_rowwise with W at any row and group strides (bytes):
 * w[g][n][k] at w + g * w_group_stride + n * w_row_stride + k. Both strides
 * multiples of 16, w_row_stride >= K (MXQ_ERR_ALIGN otherwise). The plain
 * call is w_row_stride = K, w_group_stride = N * K. A row-major (K', G * N')
 * matrix holding every expert's W_e^T side by side (the column-major output
 * of fp8_quant_jagged_colwise on W viewed as (G * N', K') with one group per
 * expert) is read with N = K', K = N', w_row_stride = G * N',
 * w_group_stride = N'. */
int fp8_grouped_gemm_rowwise_strided(const void *a, const float *inv_a, const void *w, const float *inv_w,
                                     int64_t M, int64_t N, int64_t K,
                                     int64_t w_row_stride, int64_t w_group_stride,
                                     const int32_t *offs, int32_t num_groups, void *out,
                                     cudaStream_t stream);

/* ------------------------------------------------------------------------ *
 * mx_grouped_gemm - the MXFP8 consumer of the MX rowwise quantization and of
 * the per-group 128x4 blocked scale layout (#3504 title: per-group blocked
 * scales for MXFP8 MoE training, read here as the operands of the MoE
 * layer's grouped GEMM; one E8M0 scale per 32 elements along K as the MX
 * format defines), on the tensor cores
 * (tcgen05.mma kind::mxf8f6f4.block_scale, fp32 accumulation in TMEM):
 *   out[m][n] = bf16(sum_k a[m][k] 2^(sa[m][k/32]-127)
 *                          * w[g][n][k] 2^(sw[g][n][k/32]-127))
 * for each row m of group g = [offs[g-1], offs[g]).
 *   a       e4m3 (M, K) row-major, 16-byte aligned.
 *   sfa     A's E8M0 scales in the grouped blocked layout of
 *           mx_scales_to_blocked_grouped (groups along rows, each group's
 *           rows padded to 128): mx_blocked_grouped_rows_bound(M, G) * K/32
 *           bytes, as mx_quant_rowwise_blocked_grouped writes them; 16-byte
 *           aligned.
 *   w       e4m3 (num_groups, N, K) row-major, 16-byte aligned.
 *   sfw     W's E8M0 scales, the (num_groups * N, K/32) matrix in the same
 *           blocked layout with one group (N % 128 == 0, so experts need no
 *           padding); 16-byte aligned.
 *   offs    num_groups int32 ends along M (device).
 *   out     bf16 (M, N) row-major, 16-byte aligned; rows past
 *           offs[num_groups-1] are not written.
 *   N % 128 == 0 and K % 128 == 0 (K > 0), else MXQ_ERR_SHAPE;
 *   num_groups <= 4096, else MXQ_ERR_UNSUPPORTED.
 * ------------------------------------------------------------------------ */
int mx_grouped_gemm(const void *a, const void *sfa, const void *w, const void *sfw,
                    int64_t M, int64_t N, int64_t K,
                    const int32_t *offs, int32_t num_groups, void *out,
                    cudaStream_t stream);

/* ------------------------------------------------------------------------ *
 * fp8_grouped_gemm_wgrad - the backward consumer of the jagged ops (#2064
 * Summary: the per-group scaled operands of the grad_weight grouped GEMM),
 * on the tensor cores:
 *   out[g][n][k] = bf16((sum_{m in group g} a[n][m] * b[k][m])
 *                       * inv_a[g][n] * inv_b[g][k])
 *   a       e4m3 (N, M) row-major (M contiguous): fp8_quant_jagged_rowwise
 *           of grad_out^T; inv_a fp32 (num_groups, N), its inverse scales.
 *   b       e4m3 (K, M) row-major: the buffer of fp8_quant_jagged_colwise of
 *           the input; inv_b fp32 (num_groups, K).
 *   offs    num_groups int32 ends along M (device).
 *   out     bf16 (num_groups, N, K); empty groups give zeros.
 *   N % 128 == 0, K % 128 == 0, M % 16 == 0, else MXQ_ERR_SHAPE; a, b, out
 *   16-byte aligned.
 * ------------------------------------------------------------------------ */
int fp8_grouped_gemm_wgrad(const void *a, const float *inv_a, const void *b, const float *inv_b,
                           int64_t N, int64_t K, int64_t M,
                           const int32_t *offs, int32_t num_groups, void *out,
                           cudaStream_t stream);

/* fp8_grouped_gemm_wgrad with the operands' row strides given (bytes): a
 * row n at a + n * lda, b row k at b + k * ldb; lda, ldb >= M and multiples
 * of 16 (MXQ_ERR_ALIGN otherwise), so that row-strided views (a slice of
 * wider buffers, for example) are consumed in place. */
int fp8_grouped_gemm_wgrad_ld(const void *a, const float *inv_a, const void *b, const float *inv_b,
                              int64_t N, int64_t K, int64_t M, int64_t lda, int64_t ldb,
                              const int32_t *offs, int32_t num_groups, void *out,
                              cudaStream_t stream);

/* ------------------------------------------------------------------------ *
 * (a4) mx_quant_3d_colwise - #3002 Summary: MXFP8 quantization of expert
 * weights (E, N, K) along N in 32 x 1 blocks, written straight into each
 * expert's column-major layout.
 *   in          contiguous (E, N, K) bf16; K % 8 == 0; 16-byte aligned.
 *   mode        MXQ_E8M0_FLOOR or MXQ_E8M0_RCEIL.
 *   out         e4m3 with strides (N*K, 1, N): out[e*N*K + k*N + n];
 *               16-byte aligned.
 *   scales      E8M0 bytes (E, K, N/32) row-major.
 *   N % 32 == 0, else MXQ_ERR_SHAPE.
 * ------------------------------------------------------------------------ */
int mx_quant_3d_colwise(const void *in, int64_t E, int64_t N, int64_t K,
                        int32_t mode, void *out, uint8_t *scales,
                        cudaStream_t stream);

/* ------------------------------------------------------------------------ *
 * (a5) mx_quant_rowwise - MXFP8 1 x 32 quantization along the last dimension
 * of a row-major (rows, cols) bf16 matrix (the last-dim scaling #3002's
 * Summary describes for to_mx), used on MoE activations.
 *   cols % 32 == 0; in and out 16-byte aligned.
 *   out         e4m3 row-major (rows, cols).
 *   scales      E8M0 bytes (rows, cols / 32) row-major.
 * ------------------------------------------------------------------------ */
int mx_quant_rowwise(const void *in, int64_t rows, int64_t cols, int32_t mode,
                     void *out, uint8_t *scales, cudaStream_t stream);

/* ------------------------------------------------------------------------ *
 * (a6) mx_scales_to_blocked_grouped - #3504 title: per-group conversion of an
 * E8M0 scale matrix (rows, cols) to the 128 x 4 blocked layout, the groups
 * being row ranges from `offs`, each padded to a multiple of 128 rows on its
 * own.
 *   Layout: group g's rows start at padded row P_g = sum_{h<g}
 *   128*ceil(size_h/128); columns are padded to cols4 = 4*ceil(cols/4);
 *   byte (R, c) of the padded matrix lives at
 *   ((R/128)*(cols4/4) + c/4)*512 + (R%32)*16 + ((R%128)/32)*4 + c%4.
 *   Every byte of out is written: pad bytes and all rows past the last group
 *   are 0.
 *   out_rows_capacity  a multiple of 128 and at least
 *               mx_blocked_grouped_rows_bound(rows, num_groups); out holds
 *               out_rows_capacity * cols4 bytes and is 16-byte aligned.
 *   out_group_row_starts  optional (NULL allowed): P_g for each group, int32.
 * ------------------------------------------------------------------------ */
int mx_scales_to_blocked_grouped(const uint8_t *scales, int64_t rows, int64_t cols,
                                 const int32_t *offs, int32_t num_groups,
                                 uint8_t *out, int64_t out_rows_capacity,
                                 int32_t *out_group_row_starts,
                                 cudaStream_t stream);

/* Smallest capacity valid for any offsets: 128 * floor((rows + 127*G) / 128). */
int64_t mx_blocked_grouped_rows_bound(int64_t rows, int32_t num_groups);

/* ------------------------------------------------------------------------ *
 * mx_scales_to_blocked_grouped_k - #3504's stack, #3505 "integrate new cuda
 * kernel for blocked layout for groups along K": the same 128x4 blocked
 * layout with the groups along the COLUMNS of the scale matrix (the K
 * dimension of the quantized operand, in 32-element block units).
 *   scales      u8 (rows, cols) row-major (device).
 *   offs        num_groups int32 ends along cols (device).
 *   out         128*ceil(rows/128) x out_cols_capacity bytes, the whole
 *               padded matrix in the blocked layout: group g's columns are
 *               padded to a multiple of 4 on their own and start at output
 *               column out_group_col_starts[g] = 4 * sum_{h<g} ceil(size_h/4);
 *               pad rows, pad columns and columns past the last group are 0.
 *               16-byte aligned.
 *   out_cols_capacity  multiple of 4, at least
 *               mx_blocked_grouped_k_cols_bound(cols, num_groups), else
 *               MXQ_ERR_SHAPE. num_groups <= 4096, else MXQ_ERR_UNSUPPORTED.
 *   out_group_col_starts  optional int32 (num_groups), may be NULL.
 * Reading where the pages are silent: the output is one matrix (their byte
 * count, R*C read and R*(C + 4G) written, fits it), so group g's scales form
 * a column slice of a blocked matrix with a row-tile stride of
 * out_cols_capacity/4 tiles.
 * ------------------------------------------------------------------------ */
int mx_scales_to_blocked_grouped_k(const uint8_t *scales, int64_t rows, int64_t cols,
                                   const int32_t *offs, int32_t num_groups,
                                   uint8_t *out, int64_t out_cols_capacity,
                                   int32_t *out_group_col_starts,
                                   cudaStream_t stream);

/* Smallest capacity valid for any offsets: 4 * floor((cols + 3*G) / 4). */
int64_t mx_blocked_grouped_k_cols_bound(int64_t cols, int32_t num_groups);

/* ------------------------------------------------------------------------ *
 * mx_quant_rowwise_blocked_grouped - (a5) followed by (a6) in one launch:
 * MXFP8 1x32 rowwise quantization of a row-major (rows, cols) bf16 matrix
 * whose E8M0 scales are written straight into the per-group blocked layout
 * of mx_scales_to_blocked_grouped (groups = row ranges), never as a plain
 * (rows, cols/32) matrix.
 *   cols % 32 == 0; in, out 16-byte aligned; scales_blocked 4-byte aligned.
 *   out         e4m3 (rows, cols) row-major, every row (as mx_quant_rowwise).
 *   scales_blocked  out_rows_capacity x 4*ceil(cols/128) bytes, exactly the
 *               bytes mx_scales_to_blocked_grouped writes for the scales of
 *               mx_quant_rowwise; rows past offs[num_groups-1] get no scale.
 *   out_rows_capacity, out_group_row_starts, num_groups as for
 *   mx_scales_to_blocked_grouped.
 * ------------------------------------------------------------------------ */
int mx_quant_rowwise_blocked_grouped(const void *in, int64_t rows, int64_t cols,
                                     int32_t mode, const int32_t *offs, int32_t num_groups,
                                     void *out, uint8_t *scales_blocked,
                                     int64_t out_rows_capacity, int32_t *out_group_row_starts,
                                     cudaStream_t stream);

/* ------------------------------------------------------------------------ *
 * mx_quant_jagged_colwise_padded / mx_quant_jagged_rowwise_padded - the
 * left and right operands of the MXFP8 weight-gradient grouped GEMM
 * (#3504's stack: "integrate new cuda kernel for blocked layout for groups
 * along K"): MX quantization along the grouped dimension (the tokens).
 *   colwise     groups are row ranges of (rows, cols); one line per column.
 *   rowwise     groups are column ranges of (rows, cols); one line per row.
 *   in          bf16 with element strides; lines must be contiguous
 *               (colwise: stride_col == 1, a row-major input; rowwise:
 *               stride_row == 1, the transposed view of a row-major
 *               tensor), the other stride a multiple of 8 and >= the line
 *               count, else MXQ_ERR_UNSUPPORTED. The line count must be a
 *               multiple of 128 (MXQ_ERR_SHAPE).
 *   mode        MXQ_E8M0_FLOOR or MXQ_E8M0_RCEIL.
 *   Each group's positions are cut into 32-element blocks from the group's
 *   first position (the last block holds the remainder); every block gets
 *   an E8M0 scale over its own elements and e4m3 codes.
 *   out         e4m3, line-major (lines, out_cols_capacity): group g's
 *               positions start at padded position 128 * T[g], T[g] =
 *               sum_{h<g} ceil(size_h / 128); pad positions and the capacity
 *               past the last group are zero codes.
 *               out_cols_capacity is a multiple of 128 and >=
 *               mx_blocked_grouped_rows_bound(positions, num_groups).
 *   scales_blocked  E8M0 bytes of the (lines, out_cols_capacity / 32) scale
 *               matrix in the 128x4 blocked layout (16-byte aligned,
 *               lines * out_cols_capacity / 32 bytes): group g's scale
 *               columns start at 4 * T[g] (the groups-along-K layout of
 *               mx_scales_to_blocked_grouped_k); every byte not covered by
 *               a block is 0.
 * ------------------------------------------------------------------------ */
int mx_quant_jagged_colwise_padded(const void *in, int64_t rows, int64_t cols,
                                   int64_t stride_row, int64_t stride_col,
                                   const int32_t *offs, int32_t num_groups, int32_t mode,
                                   void *out, int64_t out_cols_capacity, uint8_t *scales_blocked,
                                   cudaStream_t stream);
int mx_quant_jagged_rowwise_padded(const void *in, int64_t rows, int64_t cols,
                                   int64_t stride_row, int64_t stride_col,
                                   const int32_t *offs, int32_t num_groups, int32_t mode,
                                   void *out, int64_t out_cols_capacity, uint8_t *scales_blocked,
                                   cudaStream_t stream);

/* ------------------------------------------------------------------------ *
 * mx_grouped_gemm_wgrad - the MXFP8 weight gradient of a grouped matmul on
 * the tensor cores: for every group g (token range [offs[g-1], offs[g])),
 *   out[g][n][k] = sum over the group's padded positions p of
 *                  a[n][p] 2^(sa[n][p/32] - 127) * b[k][p] 2^(sb[k][p/32] - 127)
 * with a (N, capacity) and b (K, capacity) the padded codes and sfa, sfb the
 * blocked scales written by mx_quant_jagged_*_padded (a from grad_out^T,
 * rowwise; b from the input, colwise) with the same offsets and capacity.
 * M is the token count the offsets index. N % 128 == 0, K % 128 == 0,
 * capacity % 128 == 0 and >= mx_blocked_grouped_rows_bound(M, num_groups).
 * out: bf16 (num_groups, N, K); empty groups give zeros.
 * ------------------------------------------------------------------------ */
int mx_grouped_gemm_wgrad(const void *a, const uint8_t *sfa, const void *b, const uint8_t *sfb,
                          int64_t N, int64_t K, int64_t M, int64_t capacity,
                          const int32_t *offs, int32_t num_groups, void *out, cudaStream_t stream);

/* ------------------------------------------------------------------------ *
 * fp8_quant_jagged_colwise_noalloc - the source pages have no counterpart to
 * this entry point; it exists for callers that cannot allocate device memory
 * (a plugin inside a framework that owns all device memory and passes no
 * workspace, or a path where cudaMalloc's device-wide synchronization is not
 * acceptable). Same arguments, layout and results as
 * fp8_quant_jagged_colwise, without the workspace: the scratch is a fixed
 * array of fp8_quant_jagged_colwise_noalloc_max_scratch_bytes() bytes
 * (1 MiB) inside the library, held by every GPU that loads it until exit.
 *   - The scratch this call needs is decided by the kernels it picks for
 *     these very arguments: the kernels that keep a per-(group, column)
 *     amax table use G * cols * 4 bytes of it (rounded up to 256), the
 *     single-kernel path of small or strided problems none. A call that
 *     would need more than the array holds returns MXQ_ERR_WORKSPACE and
 *     launches nothing.
 *   - `stream` must belong to the current device (MXQ_ERR_UNSUPPORTED
 *     otherwise). The first call on a device that needs scratch looks up
 *     the array's device address with that device current; make it before
 *     any stream capture.
 *   - The call allocates nothing. All calls on a device share the array
 *     (each clears what it uses first), so calls that overlap on the GPU
 *     race; serialize them.
 * ------------------------------------------------------------------------ */
int fp8_quant_jagged_colwise_noalloc(const void *in, int64_t rows, int64_t cols,
                                     int64_t stride_row, int64_t stride_col,
                                     const int32_t *offs, int32_t num_groups,
                                     void *out, float *inv_scales,
                                     cudaStream_t stream);

/* Size in bytes of the fixed scratch array of the allocation-free entry point. */
size_t fp8_quant_jagged_colwise_noalloc_max_scratch_bytes(void);

/* ------------------------------------------------------------------------ *
 * Status and housekeeping
 * ------------------------------------------------------------------------ */

/* Synchronizes `stream`, stores the first device-side error recorded since
 * the last call (MXQ_OK if none) in *host_status and clears it. */
int mxq_device_status(cudaStream_t stream, int32_t *host_status);

/* Static text for a status code. */
const char *mxq_status_string(int status);

/* Library version, major * 10000 + minor * 100 + patch. */
int mxq_version(void);

/* Test hooks (host-side settings read at launch time):
 *   MXQ_TESTING_WAIT_LIMIT_NS  bound of every device-side wait, nanoseconds
 *                              (default 1e9; 0 restores the default).
 *   MXQ_TESTING_SKIP_ARRIVAL   when 1, CTA 0 of the jagged cast pass (or
 *                              of the single-read kernel) never issues its
 *                              first TMA load, so the transaction
 *                              arrival on that ring slot never comes, the
 *                              bounded waits on it expire and report
 *                              MXQ_ERR_TIMEOUT; 0 turns it off.
 *   MXQ_TESTING_FORCE_PATH     jagged ops: 0 automatic, 1 two-pass TMA
 *                              kernels (amax, then cast), 2 generic kernel,
 *                              3 single-read kernel (cooperative launch).
 *   MXQ_TESTING_GEMM_TILE_N    mx_grouped_gemm (and mx_grouped_gemm_wgrad)
 *                              tile width: 0 automatic (256
 *                              when N % 256 == 0, else 128), 128 forced.
 *   MXQ_TESTING_BLOCKED_PATH   mx_scales_to_blocked_grouped(_k): 0
 *                              automatic (the TMA ring kernels when the
 *                              scale rows are a multiple of 16 bytes and
 *                              at least one box wide, 128 bytes along rows
 *                              and 144 along K), 1 the word-load kernels.
 *   MXQ_TESTING_GEMM_ONE_SM    fp8_grouped_gemm_wgrad(_ld): 0 automatic
 *                              (CTA pairs with 256 x 256 tiles when N and
 *                              K are multiples of 256), 1 the one-SM
 *                              kernel. */
#define MXQ_TESTING_WAIT_LIMIT_NS 1
#define MXQ_TESTING_SKIP_ARRIVAL 2
#define MXQ_TESTING_FORCE_PATH 3
#define MXQ_TESTING_GEMM_TILE_N 4
#define MXQ_TESTING_BLOCKED_PATH 5
#define MXQ_TESTING_GEMM_ONE_SM 6
int mxq_testing_set(int32_t what, int64_t value);

#ifdef __cplusplus
}
#endif

#endif /* MXQ_H */
