// mxq.cu - host side of libmxq: argument checks, TMA descriptor encoding,
// launch configuration and the C ABI declared in include/mxq.h. All kernels
// are compiled into this one translation unit for sm_100a.
#include <atomic>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "rowblock.cuh"
#include "blockt.cuh"
#include "mx3d.cuh"
#include "jagged.cuh"
#include "jagged1.cuh"
#include "blocked.cuh"
#include "blockedt.cuh"
#include "gemm.cuh"
#include "gemm_mx.cuh"
#include "gemm2.cuh"
#include "mxj.cuh"

using namespace mxq;

namespace {

std::atomic<int64_t> g_wait_ns{1000000000LL};
std::atomic<int> g_drop_load{0};
std::atomic<int> g_force_path{0};
std::atomic<int> g_mx_bn{0}; // MX grouped GEMM tile width: 0 automatic, 128 forced
std::atomic<int> g_blocked_words{0}; // blocked layouts: 1 forces the word-load kernels
std::atomic<int> g_gemm_one_sm{0};   // weight-gradient GEMM: 1 forces the one-SM kernel

uint64_t wait_ns() { return (uint64_t)g_wait_ns.load(); }

// ------------------------------------------------------------ driver entry
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// rank-N tiled map; dims/box innermost first, strides in bytes for dims 1..N-1
int make_map(CUtensorMap *m, CUtensorMapDataType dt, int rank, const void *ptr, const uint64_t *dims,
             const uint64_t *strides, const uint32_t *box, CUtensorMapSwizzle swz)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return MXQ_ERR_CUDA;
    cuuint64_t d[5], s[5];
    cuuint32_t b[5], e[5];
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        b[i] = box[i];
        e[i] = 1;
        if (i + 1 < rank)
            s[i] = strides[i];
    }
    const CUresult r = fn(m, dt, (cuuint32_t)rank, const_cast<void *>(ptr), d, s, b, e,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MXQ_OK : MXQ_ERR_ALIGN;
}

// ------------------------------------------------------------ device info
struct DevInfo {
    bool ready = false;
    int sms = 0;
    int smem_optin = 0;
    int coop = 0;
    int amx_per_sm = 0;   // resident CTAs of the jagged amax pass
    int cst_per_sm = 0;   // resident CTAs of the jagged cast pass
    int sg_per_sm = 0;    // resident CTAs of the single-read jagged kernel
    int rb_per_sm = 0;    // resident CTAs of the 1x128 kernel
    int wg2_pairs = 0;    // co-resident CTA pairs of the pair weight-gradient GEMM
    int mx32_per_sm = 0;  // resident CTAs of the 1x32 kernel
    int mxb_per_sm = 0;   // resident CTAs of the 1x32 kernel with blocked scales
    int mxj_per_sm = 0;   // resident CTAs of the padded MX jagged kernel (at MAX_G groups)
};

DevInfo g_dev[128];
std::mutex g_dev_mu;

// co-resident clusters of two for a kernel with `smem` dynamic bytes
template <typename... K>
int max_pairs(void (*kernel)(K...), dim3 block, size_t smem, int *pairs)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2);
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(pairs, (void *)kernel, &cfg) != cudaSuccess) {
        (void)cudaGetLastError();
        return MXQ_ERR_CUDA;
    }
    return MXQ_OK;
}

int device_info(const DevInfo **out)
{
    int d = 0;
    if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= 128)
        return MXQ_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DevInfo &di = g_dev[d];
    if (!di.ready) {
        if (cudaDeviceGetAttribute(&di.sms, cudaDevAttrMultiProcessorCount, d) != cudaSuccess ||
            cudaDeviceGetAttribute(&di.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, d) != cudaSuccess ||
            cudaDeviceGetAttribute(&di.coop, cudaDevAttrCooperativeLaunch, d) != cudaSuccess)
            return MXQ_ERR_CUDA;
        if (cudaFuncSetAttribute(mx3d::k_mx_3d_colwise, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)mx3d::SMEM_BYTES) != cudaSuccess ||
            cudaFuncSetAttribute(k_fp8_blockwise_t, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)bt::SMEM_BYTES) != cudaSuccess ||
            cudaFuncSetAttribute(k_fp8_grouped_gemm<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)(gm::smem_fixed<128>() + blk::MAX_G * sizeof(int))) != cudaSuccess ||
            cudaFuncSetAttribute(k_fp8_grouped_gemm<256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)(gm::smem_fixed<256>() + blk::MAX_G * sizeof(int))) != cudaSuccess ||
            cudaFuncSetAttribute(k_mx_grouped_gemm<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)(gmx::smem_fixed<128>() + blk::MAX_G * sizeof(int))) != cudaSuccess ||
            cudaFuncSetAttribute(k_mx_grouped_gemm<256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)(gmx::smem_fixed<256>() + blk::MAX_G * sizeof(int))) != cudaSuccess ||
            cudaFuncSetAttribute(k_fp8_grouped_gemm_wgrad<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)gm::smem_fixed<128>()) != cudaSuccess ||
            cudaFuncSetAttribute(k_fp8_grouped_gemm_wgrad<256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)gm::smem_fixed<256>()) != cudaSuccess ||
            cudaFuncSetAttribute(k_jagged_cast, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)jag::cst::SMEM_BYTES) != cudaSuccess ||
            cudaFuncSetAttribute(k_jagged_single, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)jg1::SMEM_BYTES) != cudaSuccess ||
            cudaFuncSetAttribute(k_mx_jagged_colwise_padded, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)(mxj::SMEM_FIXED + blk::MAX_G * sizeof(int))) != cudaSuccess ||
            cudaFuncSetAttribute(k_mx_grouped_gemm_wgrad<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)(gmx::smem_fixed<128>() + blk::MAX_G * sizeof(int))) != cudaSuccess ||
            cudaFuncSetAttribute(k_mx_grouped_gemm_wgrad<256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)(gmx::smem_fixed<256>() + blk::MAX_G * sizeof(int))) != cudaSuccess ||
            cudaFuncSetAttribute(k_blocked_grouped_tma, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)(blkt::smem_fixed<blkt::R_STAGE>() + 2 * blk::MAX_G * sizeof(int))) != cudaSuccess ||
            cudaFuncSetAttribute(k_blocked_grouped_k_tma, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)(blkt::smem_fixed<blkt::K_STAGE>() + 2 * blk::MAX_G * sizeof(int))) != cudaSuccess ||
            cudaFuncSetAttribute(k_fp8_grouped_gemm_wgrad_2sm, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)g2::SMEM_BYTES) != cudaSuccess)
            return MXQ_ERR_CUDA;
        if (max_pairs(k_fp8_grouped_gemm_wgrad_2sm, dim3(g2::THREADS), g2::SMEM_BYTES, &di.wg2_pairs) != MXQ_OK)
            return MXQ_ERR_CUDA;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&di.amx_per_sm, k_jagged_amax, jag::amx::THREADS, 0) !=
                cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&di.cst_per_sm, k_jagged_cast, jag::cst::THREADS,
                                                          jag::cst::SMEM_BYTES) != cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&di.sg_per_sm, k_jagged_single, jg1::THREADS,
                                                          jg1::SMEM_BYTES) != cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&di.rb_per_sm, k_fp8_1x128, RB_THREADS, 0) != cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&di.mx32_per_sm, k_mx_1x32, RB_THREADS, 0) != cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&di.mxb_per_sm, k_mx_1x32_blocked, 256, 0) != cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&di.mxj_per_sm, k_mx_jagged_colwise_padded, mxj::THREADS,
                                                          mxj::SMEM_FIXED + blk::MAX_G * sizeof(int)) != cudaSuccess)
            return MXQ_ERR_CUDA;
        di.ready = true;
    }
    *out = &di;
    return MXQ_OK;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }


template <typename... K, typename... A>
int launch(void (*kernel)(K...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream, bool coop, A &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    if (coop) {
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<A>(args)...);
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return MXQ_ERR_LAUNCH;
    }
    return MXQ_OK;
}

// launch in clusters of two CTAs along x (grid.x even)
template <typename... K, typename... A>
int launch_pairs(void (*kernel)(K...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream, A &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<A>(args)...);
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return MXQ_ERR_LAUNCH;
    }
    return MXQ_OK;
}


// ------------------------------------------------------------ jagged plan
struct JaggedPlan {
    bool twopass = false;     // k_jagged_amax + k_jagged_cast
    bool single = false;      // k_jagged_single
    int wpc = 0;              // amax pass: warps per 256-line chunk
    int grid_a = 0, grid_c = 0;
    int grid_s = 0;           // single-read kernel: grid (all resident)
    size_t ws = 0;
};

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// host-checkable conditions of the two-pass kernels (no device queries):
// lines contiguous, 16-byte aligned rows for the vector loads and the TMA
// maps of input and output, at most jag::MAX_SEG groups
bool twopass_layout_ok(const void *in, int64_t L, int64_t P, int64_t s_line, int64_t s_pos, int G, const void *out)
{
    return s_line == 1 && s_pos % 8 == 0 && s_pos >= L && L > 0 && P > 0 && P % 16 == 0 && G >= 1 &&
           G <= jag::MAX_SEG && (in == nullptr || aligned(in, 16)) && (out == nullptr || aligned(out, 16)) &&
           P < (int64_t(1) << 31) && L < (int64_t(1) << 31);
}

// scratch of the table kernels: the (G, L) fp32 amax table, then the
// (G, strips of 64 lines) merge counters of the single-read kernel
size_t table_bytes(int64_t L, int G) { return round_up((size_t)G * (size_t)L * 4, 256); }
size_t counter_bytes(int64_t L, int G) { return round_up((size_t)G * (size_t)((L + 63) / 64) * 4, 256); }
size_t twopass_workspace(int64_t L, int G) { return table_bytes(L, G) + counter_bytes(L, G); }

// partial-maximum slots of the single-read kernel: (strips, units + G, 64) fp32
int64_t single_units(int64_t P, int64_t grid) { return std::min<int64_t>((P + 127) / 128, grid); }
size_t partial_bytes(int64_t L, int64_t P, int G, int64_t grid)
{
    return round_up((size_t)((L + 63) / 64) * (size_t)(single_units(P, grid) + G) * 64 * 4, 256);
}

int plan_jagged(const void *in, int64_t L, int64_t P, int64_t s_line, int64_t s_pos, int G, const void *out,
                JaggedPlan *pl)
{
    *pl = JaggedPlan();
    const int force = g_force_path.load();
    if (force == 2 || !twopass_layout_ok(in, L, P, s_line, s_pos, G, out))
        return MXQ_OK;
    // small problems are launch- and latency-bound: the generic kernel (one
    // launch, no workspace clear) is faster
    if (force == 0 && L * P <= (int64_t(1) << 21))
        return MXQ_OK;
    const DevInfo *di = nullptr;
    int rc = device_info(&di);
    if (rc != MXQ_OK)
        return rc;
    // the single-read kernel runs only when asked for: on B200 it is still
    // slower than the two passes (its cross-CTA merges serialize)
    if (force == 3 && di->coop && di->sg_per_sm >= 1) {
        // single read: a strip's 128-position blocks fall into at most
        // `grid` units (the grid is all resident) of at most MAX_UT blocks
        const int64_t grid = (int64_t)di->sms * di->sg_per_sm;
        const int64_t blocks = (P + jg1::TP - 1) / jg1::TP;
        if (blocks <= grid * jg1::MAX_UT) {
            pl->single = true;
            pl->grid_s = (int)grid;
            pl->ws = twopass_workspace(L, G) + partial_bytes(L, P, G, grid);
            return MXQ_OK;
        }
    }
    if (force == 3)
        return MXQ_OK; // not eligible: the caller reports MXQ_ERR_UNSUPPORTED
    if (di->amx_per_sm < 1 || di->cst_per_sm < 1)
        return MXQ_OK;
    pl->twopass = true;
    // amax pass: every resident warp is a worker; the warps of a 256-line
    // chunk split the positions into equal runs of at least 64 rows
    const int64_t chunks = (L + jag::amx::W - 1) / jag::amx::W;
    const int64_t warps = (int64_t)di->sms * di->amx_per_sm * (jag::amx::THREADS / 32);
    const int64_t wpc = std::max<int64_t>(1, std::min<int64_t>(warps / chunks, (P + 63) / 64));
    pl->wpc = (int)wpc;
    pl->grid_a = (int)((chunks * wpc * 32 + jag::amx::THREADS - 1) / jag::amx::THREADS);
    const int64_t tiles = (P + jag::cst::TP - 1) / jag::cst::TP * ((L + jag::cst::TL - 1) / jag::cst::TL);
    if (tiles >= (int64_t(1) << 31))
        return MXQ_OK; // the cast pass indexes tiles with 32 bits
    pl->grid_c = (int)std::min<int64_t>(tiles, (int64_t)di->sms * di->cst_per_sm);
    pl->ws = twopass_workspace(L, G);
    return MXQ_OK;
}

int jagged(const void *in, int64_t L, int64_t P, int64_t s_line, int64_t s_pos, const int32_t *offs, int G,
           void *out, float *inv, void *ws, size_t ws_bytes, cudaStream_t stream)
{
    if (L < 0 || P < 0 || G < 1)
        return MXQ_ERR_SHAPE;
    if (L == 0)
        return MXQ_OK;
    if (!offs || !inv || (P > 0 && (!in || !out)))
        return MXQ_ERR_NULL;
    JaggedPlan pl;
    int rc = plan_jagged(in, L, P, s_line, s_pos, G, out, &pl);
    if (rc != MXQ_OK)
        return rc;
    if ((g_force_path.load() == 1 && !pl.twopass) || (g_force_path.load() == 3 && !pl.single))
        return MXQ_ERR_UNSUPPORTED;
    if (pl.single) {
        if (!ws || ws_bytes < pl.ws)
            return MXQ_ERR_WORKSPACE;
        if (!aligned(ws, 256))
            return MXQ_ERR_ALIGN;
        CUtensorMap tc, to;
        const uint64_t din[2] = {(uint64_t)L, (uint64_t)P};
        const uint64_t sin[1] = {(uint64_t)s_pos * 2};
        const uint32_t bc[2] = {jg1::TL, jg1::TP};
        rc = make_map(&tc, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, in, din, sin, bc, CU_TENSOR_MAP_SWIZZLE_NONE);
        if (rc != MXQ_OK)
            return rc;
        const uint64_t dout[2] = {(uint64_t)P, (uint64_t)L};
        const uint64_t sout[1] = {(uint64_t)P};
        const uint32_t bo[2] = {jg1::TP, jg1::TL};
        rc = make_map(&to, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, out, dout, sout, bo, CU_TENSOR_MAP_SWIZZLE_128B);
        if (rc != MXQ_OK)
            return rc;
        unsigned *amax = static_cast<unsigned *>(ws);
        int *counters = reinterpret_cast<int *>(static_cast<uint8_t *>(ws) + table_bytes(L, G));
        unsigned *partials = reinterpret_cast<unsigned *>(static_cast<uint8_t *>(ws) + twopass_workspace(L, G));
        // the table and the counters start at zero; the partial slots are
        // always written before they are read
        if (cudaMemsetAsync(ws, 0, twopass_workspace(L, G), stream) != cudaSuccess)
            return MXQ_ERR_CUDA;
        const int pstride = (int)(single_units(P, pl.grid_s) + G);
        return launch(k_jagged_single, dim3(pl.grid_s), dim3(jg1::THREADS), jg1::SMEM_BYTES, stream, true,
                      tc, to, (int)L, (int)P, offs, G, amax, counters, partials, pstride, static_cast<uint8_t *>(out), inv,
                      wait_ns(), g_drop_load.load());
    }
    if (pl.twopass) {
        if (!ws || ws_bytes < pl.ws)
            return MXQ_ERR_WORKSPACE;
        if (!aligned(ws, 256))
            return MXQ_ERR_ALIGN;
        // cast pass: 128 positions x 64 lines in, the 64 x 128 transpose out
        CUtensorMap tc, to;
        const uint64_t din[2] = {(uint64_t)L, (uint64_t)P};
        const uint64_t sin[1] = {(uint64_t)s_pos * 2};
        const uint32_t bc[2] = {jag::cst::TL, jag::cst::TP};
        rc = make_map(&tc, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, in, din, sin, bc, CU_TENSOR_MAP_SWIZZLE_NONE);
        if (rc != MXQ_OK)
            return rc;
        const uint64_t dout[2] = {(uint64_t)P, (uint64_t)L};
        const uint64_t sout[1] = {(uint64_t)P};
        const uint32_t bo[2] = {jag::cst::TP, jag::cst::TL};
        rc = make_map(&to, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, out, dout, sout, bo, CU_TENSOR_MAP_SWIZZLE_128B);
        if (rc != MXQ_OK)
            return rc;
        unsigned *amax = static_cast<unsigned *>(ws);
        if (cudaMemsetAsync(ws, 0, (size_t)G * (size_t)L * 4, stream) != cudaSuccess)
            return MXQ_ERR_CUDA;
        rc = launch(k_jagged_amax, dim3(pl.grid_a), dim3(jag::amx::THREADS), 0, stream, false,
                    static_cast<const uint16_t *>(in), L, P, s_pos, offs, G, pl.wpc, amax);
        if (rc != MXQ_OK)
            return rc;
        return launch(k_jagged_cast, dim3(pl.grid_c), dim3(jag::cst::THREADS), jag::cst::SMEM_BYTES, stream, false,
                      tc, to, L, P, offs, G, static_cast<const unsigned *>(amax), static_cast<uint8_t *>(out), inv,
                      wait_ns(), g_drop_load.load());
    }
    const DevInfo *di = nullptr;
    rc = device_info(&di);
    if (rc != MXQ_OK)
        return rc;
    if (g_force_path.load() != 2 && s_pos == 1 && s_line % 8 == 0 && s_line >= P && P % 8 == 0 && aligned(in, 16) &&
        aligned(out, 16)) {
        // positions contiguous: one warp per line, vector loads
        const int64_t grid = std::max<int64_t>(1, std::min<int64_t>((L + 7) / 8, (int64_t)di->sms * 16));
        return launch(k_jagged_rows, dim3((unsigned)grid), dim3(256), 0, stream, false,
                      static_cast<const uint16_t *>(in), L, P, s_line, offs, G, static_cast<uint8_t *>(out), inv);
    }
    const int64_t warps = L * G;
    const int64_t grid = std::min<int64_t>((warps + 7) / 8, (int64_t)di->sms * 16);
    return launch(k_jagged_generic, dim3((unsigned)std::max<int64_t>(grid, 1)), dim3(256), 0, stream, false,
                  static_cast<const uint16_t *>(in), L, P, s_line, s_pos, offs, G, static_cast<uint8_t *>(out), inv);
}

} // namespace

// ======================================================================= ABI
extern "C" {

int fp8_quant_jagged_rowwise(const void *in, int64_t rows, int64_t cols, int64_t stride_row, int64_t stride_col,
                             const int32_t *offs, int32_t num_groups, void *out, float *inv_scales,
                             void *workspace, size_t workspace_bytes, cudaStream_t stream)
{
    // line = row, position = column
    return jagged(in, rows, cols, stride_row, stride_col, offs, num_groups, out, inv_scales, workspace,
                  workspace_bytes, stream);
}

int fp8_quant_jagged_colwise(const void *in, int64_t rows, int64_t cols, int64_t stride_row, int64_t stride_col,
                             const int32_t *offs, int32_t num_groups, void *out, float *inv_scales,
                             void *workspace, size_t workspace_bytes, cudaStream_t stream)
{
    // line = column, position = row
    return jagged(in, cols, rows, stride_col, stride_row, offs, num_groups, out, inv_scales, workspace,
                  workspace_bytes, stream);
}

size_t fp8_quant_jagged_workspace_bytes(int64_t rows, int64_t cols, int64_t stride_row, int64_t stride_col,
                                        int32_t num_groups, int32_t is_colwise)
{
    const int64_t L = is_colwise ? cols : rows, P = is_colwise ? rows : cols;
    const int64_t sl = is_colwise ? stride_col : stride_row, sp = is_colwise ? stride_row : stride_col;
    if (!twopass_layout_ok(nullptr, L, P, sl, sp, num_groups, nullptr))
        return 0;
    // the single-read kernel's partial slots depend on the current device's
    // resident grid; without device information, size for 1024 CTAs
    const DevInfo *di = nullptr;
    const int64_t grid = device_info(&di) == MXQ_OK ? (int64_t)di->sms * std::max(di->sg_per_sm, 1) : 1024;
    return twopass_workspace(L, num_groups) + partial_bytes(L, P, num_groups, grid);
}

int fp8_quant_blockwise(const void *in, int64_t rows, int64_t cols, int32_t block_rows, int32_t block_cols,
                        void *out, float *inv_scales, cudaStream_t stream)
{
    if (rows < 0 || cols < 0)
        return MXQ_ERR_SHAPE;
    if (block_cols != 128 || (block_rows != 1 && block_rows != 128))
        return MXQ_ERR_UNSUPPORTED;
    if (cols % 128 || rows % block_rows)
        return MXQ_ERR_SHAPE;
    if (rows == 0 || cols == 0)
        return MXQ_OK;
    if (!in || !out || !inv_scales)
        return MXQ_ERR_NULL;
    if (!aligned(in, 16) || !aligned(out, 16) || !aligned(inv_scales, 4))
        return MXQ_ERR_ALIGN;
    const DevInfo *di = nullptr;
    int rc = device_info(&di);
    if (rc != MXQ_OK)
        return rc;
    if (block_rows == 1) {
        const int64_t nblk = rows * (cols / 128);
        const int64_t per_cta = (RB_THREADS / 32) * 2 * RB_UNROLL;
        const int64_t grid = std::min<int64_t>((nblk + per_cta - 1) / per_cta, (int64_t)std::max(di->rb_per_sm, 1) * di->sms);
        return launch(k_fp8_1x128, dim3((unsigned)grid), dim3(RB_THREADS), 0, stream, false,
                      static_cast<const uint4 *>(in), nblk, static_cast<uint2 *>(out), inv_scales);
    }
    if (rows / 128 > 65535)
        return MXQ_ERR_UNSUPPORTED;
    return launch(k_fp8_128x128, dim3((unsigned)(cols / 128), (unsigned)(rows / 128)), dim3(256), 0, stream, false,
                  static_cast<const uint4 *>(in), cols, static_cast<uint2 *>(out), inv_scales);
}

int fp8_quant_blockwise_transposed(const void *in, int64_t rows, int64_t cols, int32_t block_rows,
                                   int32_t block_cols, void *out, float *inv_scales, cudaStream_t stream)
{
    if (rows < 0 || cols < 0)
        return MXQ_ERR_SHAPE;
    if (block_rows != 128 || (block_cols != 1 && block_cols != 128))
        return MXQ_ERR_UNSUPPORTED;
    if (rows % 128 || cols % 128)
        return MXQ_ERR_SHAPE;
    if (rows == 0 || cols == 0)
        return MXQ_OK;
    if (!in || !out || !inv_scales)
        return MXQ_ERR_NULL;
    if (!aligned(in, 16) || !aligned(out, 16) || !aligned(inv_scales, 4))
        return MXQ_ERR_ALIGN;
    if ((rows / 128) * (cols / 128) >= (int64_t(1) << 31) || rows >= (int64_t(1) << 31) ||
        cols >= (int64_t(1) << 31))
        return MXQ_ERR_UNSUPPORTED;
    const DevInfo *di = nullptr;
    int rc = device_info(&di);
    if (rc != MXQ_OK)
        return rc;
    CUtensorMap tin, tout;
    const uint64_t din[2] = {(uint64_t)cols, (uint64_t)rows};
    const uint64_t sin[1] = {(uint64_t)cols * 2};
    const uint32_t bin[2] = {bt::TH, bt::TR};
    rc = make_map(&tin, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, in, din, sin, bin, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (rc != MXQ_OK)
        return rc;
    const uint64_t dout[2] = {(uint64_t)rows, (uint64_t)cols};
    const uint64_t sout[1] = {(uint64_t)rows};
    const uint32_t bout[2] = {bt::TR, bt::TH};
    rc = make_map(&tout, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, out, dout, sout, bout, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc != MXQ_OK)
        return rc;
    const int64_t items = (rows / 128) * (cols / 128);
    const int64_t grid = std::min<int64_t>(items, (int64_t)di->sms * bt::CTAS_PER_SM);
    return launch(k_fp8_blockwise_t, dim3((unsigned)grid), dim3(bt::THREADS), bt::SMEM_BYTES, stream, false, tin,
                  tout, inv_scales, rows, cols, (int)block_cols, wait_ns());
}

int fp8_grouped_gemm_rowwise_strided(const void *a, const float *inv_a, const void *w, const float *inv_w, int64_t M,
                                     int64_t N, int64_t K, int64_t w_row_stride, int64_t w_group_stride,
                                     const int32_t *offs, int32_t num_groups, void *out, cudaStream_t stream)
{
    if (M < 0 || N < 0 || K < 0 || num_groups < 1 || N % 128 || K % gm::BK)
        return MXQ_ERR_SHAPE;
    if (num_groups > blk::MAX_G)
        return MXQ_ERR_UNSUPPORTED;
    if (M == 0 || N == 0)
        return MXQ_OK;
    if (K == 0)
        return MXQ_ERR_SHAPE;
    if (!a || !inv_a || !w || !inv_w || !offs || !out)
        return MXQ_ERR_NULL;
    if (!aligned(a, 16) || !aligned(w, 16) || !aligned(out, 16) || !aligned(inv_a, 4) || !aligned(inv_w, 4))
        return MXQ_ERR_ALIGN;
    // W rows must not overlap and start on 16-byte boundaries (TMA strides)
    if (w_row_stride < K || w_row_stride % 16 || w_group_stride < 0 || w_group_stride % 16 ||
        (num_groups > 1 && w_group_stride == 0))
        return MXQ_ERR_ALIGN;
    if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31) ||
        num_groups >= (int64_t(1) << 31))
        return MXQ_ERR_UNSUPPORTED;
    const DevInfo *di = nullptr;
    int rc = device_info(&di);
    if (rc != MXQ_OK)
        return rc;
    CUtensorMap ta, tw;
    const uint64_t da[2] = {(uint64_t)K, (uint64_t)M};
    const uint64_t sa[1] = {(uint64_t)K};
    const uint32_t box[2] = {gm::BK, gm::BM};
    rc = make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, a, da, sa, box, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc != MXQ_OK)
        return rc;
    // tiles 128 x 256 when N allows, else 128 x 128; W through a rank-3 map
    // with its dimensions in increasing stride order: (k, n, group), or
    // (k, group, n) when the groups sit side by side within a row
    const int bn = N % 256 == 0 ? 256 : 128;
    const int group_inner = num_groups > 1 && w_group_stride < w_row_stride ? 1 : 0;
    const uint64_t gs = (uint64_t)std::max<int64_t>(w_group_stride, 16);
    const uint64_t dw[3] = {(uint64_t)K, group_inner ? (uint64_t)num_groups : (uint64_t)N,
                            group_inner ? (uint64_t)N : (uint64_t)num_groups};
    const uint64_t sw[2] = {group_inner ? gs : (uint64_t)w_row_stride, group_inner ? (uint64_t)w_row_stride : gs};
    const uint32_t boxw[3] = {gm::BK, group_inner ? 1u : (uint32_t)bn, group_inner ? (uint32_t)bn : 1u};
    rc = make_map(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, w, dw, sw, boxw, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc != MXQ_OK)
        return rc;
    // work items: at most (M / 128 + G) m-tiles times N / bn n-tiles
    const int64_t items = (M / gm::BM + num_groups) * (N / bn);
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(items, di->sms));
    if (bn == 256)
        return launch(k_fp8_grouped_gemm<256>, dim3((unsigned)grid), dim3(gm::THREADS),
                      gm::smem_fixed<256>() + (size_t)num_groups * sizeof(int), stream, false, ta, tw, inv_a, inv_w, M,
                      N, K, offs, (int)num_groups, static_cast<uint16_t *>(out), wait_ns(), group_inner);
    return launch(k_fp8_grouped_gemm<128>, dim3((unsigned)grid), dim3(gm::THREADS),
                  gm::smem_fixed<128>() + (size_t)num_groups * sizeof(int), stream, false, ta, tw, inv_a, inv_w, M, N,
                  K, offs, (int)num_groups, static_cast<uint16_t *>(out), wait_ns(), group_inner);
}

int fp8_grouped_gemm_rowwise(const void *a, const float *inv_a, const void *w, const float *inv_w, int64_t M,
                             int64_t N, int64_t K, const int32_t *offs, int32_t num_groups, void *out,
                             cudaStream_t stream)
{
    // W (num_groups, N, K) row-major
    return fp8_grouped_gemm_rowwise_strided(a, inv_a, w, inv_w, M, N, K, K, N * K, offs, num_groups, out, stream);
}

int mx_grouped_gemm(const void *a, const void *sfa, const void *w, const void *sfw, int64_t M, int64_t N, int64_t K,
                    const int32_t *offs, int32_t num_groups, void *out, cudaStream_t stream)
{
    if (M < 0 || N < 0 || K < 0 || num_groups < 1 || N % 128 || K % gmx::BK)
        return MXQ_ERR_SHAPE;
    if (num_groups > blk::MAX_G)
        return MXQ_ERR_UNSUPPORTED;
    if (M == 0 || N == 0)
        return MXQ_OK;
    if (K == 0)
        return MXQ_ERR_SHAPE;
    if (!a || !sfa || !w || !sfw || !offs || !out)
        return MXQ_ERR_NULL;
    if (!aligned(a, 16) || !aligned(w, 16) || !aligned(out, 16) || !aligned(sfa, 16) || !aligned(sfw, 16))
        return MXQ_ERR_ALIGN;
    if (M >= (int64_t(1) << 31) || (int64_t)num_groups * N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31))
        return MXQ_ERR_UNSUPPORTED;
    const DevInfo *di = nullptr;
    int rc = device_info(&di);
    if (rc != MXQ_OK)
        return rc;
    CUtensorMap ta, tw;
    const uint64_t da[2] = {(uint64_t)K, (uint64_t)M};
    const uint64_t sa[1] = {(uint64_t)K};
    const uint32_t box[2] = {gmx::BK, gmx::BM};
    rc = make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, a, da, sa, box, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc != MXQ_OK)
        return rc;
    // tiles 128 x 256 when N allows (one accumulator), else 128 x 128 (two)
    const int bn = N % 256 == 0 && g_mx_bn.load() != 128 ? 256 : 128;
    const uint64_t dw[2] = {(uint64_t)K, (uint64_t)(num_groups * N)};
    const uint32_t boxw[2] = {gmx::BK, (uint32_t)bn};
    rc = make_map(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, w, dw, sa, boxw, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc != MXQ_OK)
        return rc;
    const int64_t items = (M / gmx::BM + num_groups) * (N / bn);
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(items, di->sms));
    const size_t smem_g = (size_t)num_groups * sizeof(int);
    if (bn == 256)
        return launch(k_mx_grouped_gemm<256>, dim3((unsigned)grid), dim3(gmx::THREADS), gmx::smem_fixed<256>() + smem_g,
                      stream, false, ta, tw, static_cast<const uint8_t *>(sfa), static_cast<const uint8_t *>(sfw), M, N,
                      K, offs, (int)num_groups, static_cast<uint16_t *>(out), wait_ns());
    return launch(k_mx_grouped_gemm<128>, dim3((unsigned)grid), dim3(gmx::THREADS), gmx::smem_fixed<128>() + smem_g,
                  stream, false, ta, tw, static_cast<const uint8_t *>(sfa), static_cast<const uint8_t *>(sfw), M, N, K,
                  offs, (int)num_groups, static_cast<uint16_t *>(out), wait_ns());
}

int fp8_grouped_gemm_wgrad_ld(const void *a, const float *inv_a, const void *b, const float *inv_b, int64_t N,
                              int64_t K, int64_t M, int64_t lda, int64_t ldb, const int32_t *offs, int32_t num_groups,
                              void *out, cudaStream_t stream)
{
    if (M < 0 || N < 0 || K < 0 || num_groups < 1 || N % gm::BM || K % 128 || M % 16)
        return MXQ_ERR_SHAPE;
    if (N == 0 || K == 0)
        return MXQ_OK;
    if (!a || !inv_a || !b || !inv_b || !offs || !out)
        return MXQ_ERR_NULL;
    if (!aligned(a, 16) || !aligned(b, 16) || !aligned(out, 16) || !aligned(inv_a, 4) || !aligned(inv_b, 4))
        return MXQ_ERR_ALIGN;
    if (lda < M || ldb < M || lda % 16 || ldb % 16)
        return MXQ_ERR_ALIGN;
    if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31))
        return MXQ_ERR_UNSUPPORTED;
    const DevInfo *di = nullptr;
    int rc = device_info(&di);
    if (rc != MXQ_OK)
        return rc;
    const int bn = K % 256 == 0 ? 256 : 128;
    CUtensorMap ta, tb;
    const uint64_t mm = (uint64_t)std::max<int64_t>(M, 16); // a map needs a non-zero extent
    if (N % g2::BM == 0 && K % g2::BN == 0 && di->wg2_pairs > 0 && g_gemm_one_sm.load() == 0) {
        // CTA pairs: 256 x 256 tiles, each CTA loading 128 rows of a and of b
        const uint64_t da[2] = {mm, (uint64_t)N};
        const uint64_t sa[1] = {(uint64_t)std::max<int64_t>(lda, 16)};
        const uint32_t box[2] = {g2::BK, g2::HALF};
        rc = make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, a, da, sa, box, CU_TENSOR_MAP_SWIZZLE_128B);
        if (rc != MXQ_OK)
            return rc;
        const uint64_t db[2] = {mm, (uint64_t)K};
        const uint64_t sb[1] = {(uint64_t)std::max<int64_t>(ldb, 16)};
        rc = make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, b, db, sb, box, CU_TENSOR_MAP_SWIZZLE_128B);
        if (rc != MXQ_OK)
            return rc;
        const int64_t items = (int64_t)num_groups * (N / g2::BM) * (K / g2::BN);
        const int64_t pairs = std::max<int64_t>(1, std::min<int64_t>(items, di->wg2_pairs));
        return launch_pairs(k_fp8_grouped_gemm_wgrad_2sm, dim3((unsigned)(2 * pairs)), dim3(g2::THREADS),
                            g2::SMEM_BYTES, stream, ta, tb, inv_a, inv_b, N, K, M, offs, (int)num_groups,
                            static_cast<uint16_t *>(out), wait_ns());
    }
    const uint64_t da[2] = {mm, (uint64_t)N};
    const uint64_t sa[1] = {(uint64_t)std::max<int64_t>(lda, 16)};
    const uint32_t boxa[2] = {gm::BK, gm::BM};
    rc = make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, a, da, sa, boxa, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc != MXQ_OK)
        return rc;
    const uint64_t db[2] = {mm, (uint64_t)K};
    const uint64_t sb[1] = {(uint64_t)std::max<int64_t>(ldb, 16)};
    const uint32_t boxb[2] = {gm::BK, (uint32_t)bn};
    rc = make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, b, db, sb, boxb, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc != MXQ_OK)
        return rc;
    const int64_t items = (int64_t)num_groups * (N / gm::BM) * (K / bn);
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(items, di->sms));
    if (bn == 256)
        return launch(k_fp8_grouped_gemm_wgrad<256>, dim3((unsigned)grid), dim3(gm::THREADS), gm::smem_fixed<256>(),
                      stream, false, ta, tb, inv_a, inv_b, N, K, M, offs, (int)num_groups,
                      static_cast<uint16_t *>(out), wait_ns());
    return launch(k_fp8_grouped_gemm_wgrad<128>, dim3((unsigned)grid), dim3(gm::THREADS), gm::smem_fixed<128>(),
                  stream, false, ta, tb, inv_a, inv_b, N, K, M, offs, (int)num_groups, static_cast<uint16_t *>(out),
                  wait_ns());
}

int fp8_grouped_gemm_wgrad(const void *a, const float *inv_a, const void *b, const float *inv_b, int64_t N,
                           int64_t K, int64_t M, const int32_t *offs, int32_t num_groups, void *out,
                           cudaStream_t stream)
{
    return fp8_grouped_gemm_wgrad_ld(a, inv_a, b, inv_b, N, K, M, M, M, offs, num_groups, out, stream);
}

int mx_quant_3d_colwise(const void *in, int64_t E, int64_t N, int64_t K, int32_t mode, void *out, uint8_t *scales,
                        cudaStream_t stream)
{
    if (E < 0 || N < 0 || K < 0 || N % 32)
        return MXQ_ERR_SHAPE;
    if (mode != MXQ_E8M0_FLOOR && mode != MXQ_E8M0_RCEIL)
        return MXQ_ERR_UNSUPPORTED;
    if (E == 0 || N == 0 || K == 0)
        return MXQ_OK;
    if (!in || !out || !scales)
        return MXQ_ERR_NULL;
    if (K % 8 || !aligned(in, 16) || !aligned(out, 16))
        return MXQ_ERR_ALIGN;
    if (E >= (int64_t(1) << 31) || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31))
        return MXQ_ERR_UNSUPPORTED;
    const DevInfo *di = nullptr;
    int rc = device_info(&di);
    if (rc != MXQ_OK)
        return rc;
    CUtensorMap tin, tout;
    const uint64_t din[3] = {(uint64_t)K, (uint64_t)N, (uint64_t)E};
    const uint64_t sin[2] = {(uint64_t)K * 2, (uint64_t)N * K * 2};
    const uint32_t bin[3] = {mx3d::TK, mx3d::TN, 1};
    rc = make_map(&tin, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, in, din, sin, bin, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (rc != MXQ_OK)
        return rc;
    const uint64_t dout[3] = {(uint64_t)N, (uint64_t)K, (uint64_t)E};
    const uint64_t sout[2] = {(uint64_t)N, (uint64_t)N * K};
    const uint32_t bout[3] = {mx3d::TN, mx3d::TK, 1};
    rc = make_map(&tout, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, out, dout, sout, bout, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc != MXQ_OK)
        return rc;
    const int tiles_n = (int)((N + mx3d::TN - 1) / mx3d::TN), tiles_k = (int)((K + mx3d::TK - 1) / mx3d::TK);
    const int64_t total = E * tiles_n * tiles_k;
    const int64_t grid = std::min<int64_t>(total, (int64_t)di->sms * mx3d::CTAS_PER_SM);
    return launch(mx3d::k_mx_3d_colwise, dim3((unsigned)grid), dim3(mx3d::THREADS), mx3d::SMEM_BYTES, stream, false,
                  tin, tout, scales, (int)E, (int)N, (int)K, tiles_n, tiles_k, (int)mode, wait_ns());
}

int mx_quant_rowwise(const void *in, int64_t rows, int64_t cols, int32_t mode, void *out, uint8_t *scales,
                     cudaStream_t stream)
{
    if (rows < 0 || cols < 0 || cols % 32)
        return MXQ_ERR_SHAPE;
    if (mode != MXQ_E8M0_FLOOR && mode != MXQ_E8M0_RCEIL)
        return MXQ_ERR_UNSUPPORTED;
    if (rows == 0 || cols == 0)
        return MXQ_OK;
    if (!in || !out || !scales)
        return MXQ_ERR_NULL;
    if (!aligned(in, 16) || !aligned(out, 16))
        return MXQ_ERR_ALIGN;
    const DevInfo *di = nullptr;
    int rc = device_info(&di);
    if (rc != MXQ_OK)
        return rc;
    const int64_t nblk = rows * (cols / 32);
    const int64_t per_cta = (RB_THREADS / 32) * 8 * RB_UNROLL;
    const int64_t grid = std::min<int64_t>((nblk + per_cta - 1) / per_cta, (int64_t)std::max(di->mx32_per_sm, 1) * di->sms);
    const int wa = aligned(scales, 4) ? 1 : 0;
    return launch(k_mx_1x32, dim3((unsigned)grid), dim3(RB_THREADS), 0, stream, false, static_cast<const uint4 *>(in),
                  nblk, static_cast<uint2 *>(out), scales, wa, (int)mode);
}

int64_t mx_blocked_grouped_rows_bound(int64_t rows, int32_t num_groups)
{
    if (rows < 0 || num_groups < 0)
        return -1;
    return 128 * ((rows + 127 * (int64_t)num_groups) / 128);
}

int mx_scales_to_blocked_grouped(const uint8_t *scales, int64_t rows, int64_t cols, const int32_t *offs,
                                 int32_t num_groups, uint8_t *out, int64_t out_rows_capacity,
                                 int32_t *out_group_row_starts, cudaStream_t stream)
{
    if (rows < 0 || cols < 0 || num_groups < 1 || out_rows_capacity < 0 || out_rows_capacity % 128)
        return MXQ_ERR_SHAPE;
    if (!offs || (rows * cols > 0 && !scales) || (out_rows_capacity * cols > 0 && !out))
        return MXQ_ERR_NULL;
    if (out_rows_capacity < mx_blocked_grouped_rows_bound(rows, num_groups))
        return MXQ_ERR_SHAPE;
    if (num_groups > blk::MAX_G)
        return MXQ_ERR_UNSUPPORTED;
    if (out && !aligned(out, 16))
        return MXQ_ERR_ALIGN;
    const int64_t cols4 = (cols + 3) / 4 * 4;
    if ((cols4 == 0 || out_rows_capacity == 0) && !out_group_row_starts)
        return MXQ_OK;
    const int64_t tiles_c = cols4 / 4;
    const DevInfo *di = nullptr;
    int rc = device_info(&di);
    if (rc != MXQ_OK)
        return rc;
    if (rows > 0 && cols >= blkt::R_BOX_X && cols % 16 == 0 && aligned(scales, 16) && rows < (int64_t(1) << 31) &&
        g_blocked_words.load() == 0) {
        // TMA ring: rows of 16-byte multiples, at least one full box wide
        CUtensorMap tm;
        const uint64_t dims[2] = {(uint64_t)cols, (uint64_t)rows};
        const uint64_t strides[1] = {(uint64_t)cols};
        const uint32_t box[2] = {blkt::R_BOX_X, blkt::ROWS};
        rc = make_map(&tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, scales, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
        if (rc != MXQ_OK)
            return rc;
        const size_t smem = blkt::smem_fixed<blkt::R_STAGE>() + 2 * (size_t)num_groups * sizeof(int);
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_blocked_grouped_tma, blkt::THREADS, smem) !=
            cudaSuccess)
            return MXQ_ERR_CUDA;
        const int64_t units = out_rows_capacity / 128 * ((tiles_c + blkt::TILES - 1) / blkt::TILES);
        const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(units, (int64_t)di->sms * std::max(per_sm, 1)));
        return launch(k_blocked_grouped_tma, dim3((unsigned)grid), dim3(blkt::THREADS), smem, stream, false, tm, rows,
                      cols, offs, (int)num_groups, out, out_group_row_starts, out_rows_capacity / 128, wait_ns());
    }
    const int64_t gx = std::max<int64_t>((tiles_c + blk::TILES - 1) / blk::TILES, 1);
    // enough CTAs to fill the GPU; each walks tile rows with stride gy
    const int64_t tile_rows = std::max<int64_t>(out_rows_capacity / 128, 1);
    const int64_t want = std::max<int64_t>((int64_t)di->sms * 8 / gx, 1);
    const int64_t gy = std::min<int64_t>(tile_rows, std::min<int64_t>(want, 65535));
    const int words_ok = (aligned(scales, 4) && cols % 4 == 0) ? 1 : 0;
    return launch(k_blocked_grouped, dim3((unsigned)gx, (unsigned)gy), dim3(blk::THREADS),
                  (size_t)num_groups * sizeof(int), stream, false, scales,
                  rows, cols, offs, (int)num_groups, out, out_group_row_starts, words_ok,
                  out_rows_capacity / 128);
}

int64_t mx_blocked_grouped_k_cols_bound(int64_t cols, int32_t num_groups)
{
    if (cols < 0 || num_groups < 0)
        return -1;
    return 4 * ((cols + 3 * (int64_t)num_groups) / 4);
}

int mx_scales_to_blocked_grouped_k(const uint8_t *scales, int64_t rows, int64_t cols, const int32_t *offs,
                                   int32_t num_groups, uint8_t *out, int64_t out_cols_capacity,
                                   int32_t *out_group_col_starts, cudaStream_t stream)
{
    if (rows < 0 || cols < 0 || num_groups < 1 || out_cols_capacity < 0 || out_cols_capacity % 4)
        return MXQ_ERR_SHAPE;
    const int64_t rows_p = (rows + 127) / 128 * 128;
    if (!offs || (rows * cols > 0 && !scales) || (rows_p * out_cols_capacity > 0 && !out))
        return MXQ_ERR_NULL;
    if (out_cols_capacity < mx_blocked_grouped_k_cols_bound(cols, num_groups))
        return MXQ_ERR_SHAPE;
    if (num_groups > blk::MAX_G)
        return MXQ_ERR_UNSUPPORTED;
    if (out && !aligned(out, 16))
        return MXQ_ERR_ALIGN;
    if ((rows_p == 0 || out_cols_capacity == 0) && !out_group_col_starts)
        return MXQ_OK;
    const DevInfo *di = nullptr;
    int rc = device_info(&di);
    if (rc != MXQ_OK)
        return rc;
    const int64_t tiles_c = out_cols_capacity / 4;
    if (rows > 0 && cols >= blkt::K_BOX_X && cols % 16 == 0 && aligned(scales, 16) && cols < (int64_t(1) << 31) &&
        g_blocked_words.load() == 0) {
        // TMA ring: rows of 16-byte multiples, at least one box wide
        CUtensorMap tm;
        const uint64_t dims[2] = {(uint64_t)cols, (uint64_t)rows};
        const uint64_t strides[1] = {(uint64_t)cols};
        const uint32_t box[2] = {blkt::K_BOX_X, blkt::ROWS};
        rc = make_map(&tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, scales, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE);
        if (rc != MXQ_OK)
            return rc;
        const size_t smem = blkt::smem_fixed<blkt::K_STAGE>() + 2 * (size_t)num_groups * sizeof(int);
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_blocked_grouped_k_tma, blkt::THREADS, smem) !=
            cudaSuccess)
            return MXQ_ERR_CUDA;
        const int64_t units = rows_p / 128 * ((tiles_c + blkt::TILES - 1) / blkt::TILES);
        const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(units, (int64_t)di->sms * std::max(per_sm, 1)));
        return launch(k_blocked_grouped_k_tma, dim3((unsigned)grid), dim3(blkt::THREADS), smem, stream, false, tm,
                      rows, cols, offs, (int)num_groups, out, out_group_col_starts, out_cols_capacity, wait_ns());
    }
    const int64_t gx = std::max<int64_t>((tiles_c + blk::TILES - 1) / blk::TILES, 1);
    const int64_t tile_rows = std::max<int64_t>(rows_p / 128, 1);
    const int64_t want = std::max<int64_t>((int64_t)di->sms * 8 / gx, 1);
    const int64_t gy = std::min<int64_t>(tile_rows, std::min<int64_t>(want, 65535));
    if (gx > 0x7fffffff)
        return MXQ_ERR_UNSUPPORTED;
    const int words_ok = (aligned(scales, 4) && cols % 4 == 0) ? 1 : 0;
    return launch(k_blocked_grouped_k, dim3((unsigned)gx, (unsigned)gy), dim3(blk::THREADS),
                  (size_t)num_groups * sizeof(int), stream, false, scales,
                  rows, cols, offs, (int)num_groups, out, out_group_col_starts, words_ok, out_cols_capacity);
}

int mx_quant_rowwise_blocked_grouped(const void *in, int64_t rows, int64_t cols, int32_t mode, const int32_t *offs,
                                     int32_t num_groups, void *out, uint8_t *scales_blocked,
                                     int64_t out_rows_capacity, int32_t *out_group_row_starts, cudaStream_t stream)
{
    if (rows < 0 || cols < 0 || cols % 32 || num_groups < 1 || out_rows_capacity < 0 || out_rows_capacity % 128)
        return MXQ_ERR_SHAPE;
    if (mode != MXQ_E8M0_FLOOR && mode != MXQ_E8M0_RCEIL)
        return MXQ_ERR_UNSUPPORTED;
    const int64_t tcols = (cols + 127) / 128;
    if (!offs || (rows * cols > 0 && (!in || !out)) || (out_rows_capacity * tcols > 0 && !scales_blocked))
        return MXQ_ERR_NULL;
    if (out_rows_capacity < mx_blocked_grouped_rows_bound(rows, num_groups))
        return MXQ_ERR_SHAPE;
    if (num_groups > blk::MAX_G)
        return MXQ_ERR_UNSUPPORTED;
    if ((in && !aligned(in, 16)) || (out && !aligned(out, 16)) || (scales_blocked && !aligned(scales_blocked, 4)))
        return MXQ_ERR_ALIGN;
    if (rows * cols == 0 && out_rows_capacity * tcols == 0 && !out_group_row_starts)
        return MXQ_OK;
    const DevInfo *di = nullptr;
    int rc = device_info(&di);
    if (rc != MXQ_OK)
        return rc;
    const int64_t warps = std::max<int64_t>(rows, out_rows_capacity);
    const int64_t grid = std::max<int64_t>(std::min<int64_t>((warps + 7) / 8, (int64_t)di->sms * di->mxb_per_sm), 1);
    return launch(k_mx_1x32_blocked, dim3((unsigned)grid), dim3(256), (size_t)num_groups * 2 * sizeof(int), stream,
                  false,
                  static_cast<const uint4 *>(in), rows, cols, offs, (int)num_groups, static_cast<uint2 *>(out),
                  reinterpret_cast<uint32_t *>(scales_blocked), out_group_row_starts, out_rows_capacity, (int)mode);
}

} // extern "C"

namespace {

// MX quantization along grouped positions, groups padded to 128 positions:
// lines contiguous (s_line == 1), L a multiple of 128
int mx_jagged_padded(const void *in, int64_t L, int64_t P, int64_t s_line, int64_t s_pos, const int32_t *offs, int G,
                     int mode, void *out, int64_t cap, uint8_t *scales, cudaStream_t stream)
{
    if (L < 0 || P < 0 || G < 1 || cap < 0 || cap % 128)
        return MXQ_ERR_SHAPE;
    if (mode != MXQ_E8M0_FLOOR && mode != MXQ_E8M0_RCEIL)
        return MXQ_ERR_UNSUPPORTED;
    if (cap < mx_blocked_grouped_rows_bound(P, G))
        return MXQ_ERR_SHAPE;
    if (G > blk::MAX_G)
        return MXQ_ERR_UNSUPPORTED;
    if (L == 0 || cap == 0)
        return MXQ_OK;
    if (!offs || !out || !scales || (P > 0 && !in))
        return MXQ_ERR_NULL;
    if (L % 128)
        return MXQ_ERR_SHAPE;
    // the TMA path: lines contiguous, 16-byte aligned rows of positions
    if (s_line != 1 || s_pos % 8 || s_pos < L)
        return MXQ_ERR_UNSUPPORTED;
    if ((in && !aligned(in, 16)) || !aligned(out, 16) || !aligned(scales, 16))
        return MXQ_ERR_ALIGN;
    if (P >= (int64_t(1) << 31) || L >= (int64_t(1) << 31) || cap >= (int64_t(1) << 31) ||
        (cap / 128) * (L / 64) >= (int64_t(1) << 31))
        return MXQ_ERR_UNSUPPORTED;
    const DevInfo *di = nullptr;
    int rc = device_info(&di);
    if (rc != MXQ_OK)
        return rc;
    CUtensorMap tin, tout;
    // a map needs a non-zero extent: with P == 0 every tile is padding and
    // the map is never read
    const uint64_t din[2] = {(uint64_t)L, (uint64_t)std::max<int64_t>(P, 1)};
    const uint64_t sin[1] = {(uint64_t)s_pos * 2};
    const uint32_t bin[2] = {mxj::TL, mxj::TP};
    rc = make_map(&tin, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, P > 0 ? in : out, din, sin, bin,
                  CU_TENSOR_MAP_SWIZZLE_NONE);
    if (rc != MXQ_OK)
        return rc;
    const uint64_t dout[2] = {(uint64_t)cap, (uint64_t)L};
    const uint64_t sout[1] = {(uint64_t)cap};
    const uint32_t bout[2] = {mxj::TP, mxj::TL};
    rc = make_map(&tout, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, out, dout, sout, bout, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc != MXQ_OK)
        return rc;
    const int64_t items = (cap / 128) * (L / 64);
    const int64_t grid = std::min<int64_t>(items, (int64_t)di->sms * std::max(di->mxj_per_sm, 1));
    return launch(k_mx_jagged_colwise_padded, dim3((unsigned)grid), dim3(mxj::THREADS),
                  mxj::SMEM_FIXED + (size_t)G * sizeof(int), stream, false, tin, tout, (int)L, (int)P, offs, G,
                  (int)(cap / 128), scales, mode, wait_ns());
}

} // namespace

extern "C" {

int mx_quant_jagged_colwise_padded(const void *in, int64_t rows, int64_t cols, int64_t stride_row,
                                   int64_t stride_col, const int32_t *offs, int32_t num_groups, int32_t mode,
                                   void *out, int64_t out_cols_capacity, uint8_t *scales_blocked, cudaStream_t stream)
{
    // line = column, position = row
    return mx_jagged_padded(in, cols, rows, stride_col, stride_row, offs, num_groups, mode, out, out_cols_capacity,
                            scales_blocked, stream);
}

int mx_quant_jagged_rowwise_padded(const void *in, int64_t rows, int64_t cols, int64_t stride_row,
                                   int64_t stride_col, const int32_t *offs, int32_t num_groups, int32_t mode,
                                   void *out, int64_t out_cols_capacity, uint8_t *scales_blocked, cudaStream_t stream)
{
    // line = row, position = column
    return mx_jagged_padded(in, rows, cols, stride_row, stride_col, offs, num_groups, mode, out, out_cols_capacity,
                            scales_blocked, stream);
}

int mx_grouped_gemm_wgrad(const void *a, const uint8_t *sfa, const void *b, const uint8_t *sfb, int64_t N, int64_t K,
                          int64_t M, int64_t capacity, const int32_t *offs, int32_t num_groups, void *out,
                          cudaStream_t stream)
{
    if (M < 0 || N < 0 || K < 0 || capacity < 0 || num_groups < 1 || N % gmx::BM || K % 128 || capacity % 128)
        return MXQ_ERR_SHAPE;
    if (capacity < mx_blocked_grouped_rows_bound(M, num_groups))
        return MXQ_ERR_SHAPE;
    if (num_groups > blk::MAX_G)
        return MXQ_ERR_UNSUPPORTED;
    if (N == 0 || K == 0)
        return MXQ_OK;
    if (!a || !sfa || !b || !sfb || !offs || !out)
        return MXQ_ERR_NULL;
    if (!aligned(a, 16) || !aligned(b, 16) || !aligned(out, 16) || !aligned(sfa, 16) || !aligned(sfb, 16))
        return MXQ_ERR_ALIGN;
    if (capacity >= (int64_t(1) << 31) || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31) ||
        M >= (int64_t(1) << 31))
        return MXQ_ERR_UNSUPPORTED;
    const DevInfo *di = nullptr;
    int rc = device_info(&di);
    if (rc != MXQ_OK)
        return rc;
    const int bn = K % 256 == 0 && g_mx_bn.load() != 128 ? 256 : 128;
    CUtensorMap ta, tb;
    const uint64_t cc = (uint64_t)std::max<int64_t>(capacity, 128); // a map needs a non-zero extent
    const uint64_t da[2] = {cc, (uint64_t)N};
    const uint64_t sa[1] = {cc};
    const uint32_t boxa[2] = {gmx::BK, gmx::BM};
    rc = make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, a, da, sa, boxa, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc != MXQ_OK)
        return rc;
    const uint64_t db[2] = {cc, (uint64_t)K};
    const uint32_t boxb[2] = {gmx::BK, (uint32_t)bn};
    rc = make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, b, db, sa, boxb, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc != MXQ_OK)
        return rc;
    const int64_t items = (int64_t)num_groups * (N / gmx::BM) * (K / bn);
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(items, di->sms));
    const size_t smem_g = (size_t)num_groups * sizeof(int);
    if (bn == 256)
        return launch(k_mx_grouped_gemm_wgrad<256>, dim3((unsigned)grid), dim3(gmx::THREADS),
                      gmx::smem_fixed<256>() + smem_g, stream, false, ta, tb, sfa, sfb, N, K, M,
                      (int)(capacity / 128), offs, (int)num_groups, static_cast<uint16_t *>(out), wait_ns());
    return launch(k_mx_grouped_gemm_wgrad<128>, dim3((unsigned)grid), dim3(gmx::THREADS),
                  gmx::smem_fixed<128>() + smem_g, stream, false, ta, tb, sfa, sfb, N, K, M, (int)(capacity / 128),
                  offs, (int)num_groups, static_cast<uint16_t *>(out), wait_ns());
}

} // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free variant of fp8_quant_jagged_colwise.
//
// Some callers cannot call cudaMalloc: a plugin running inside a framework
// that owns all of the device memory and hands it no workspace argument, or
// a latency-critical path where cudaMalloc's implicit device-wide
// synchronization is not acceptable. This entry point needs no workspace from
// them: its scratch (the per-(group, column) amax table) lives in the
// fixed-size array below, which every GPU that loads this library keeps for
// the life of the process.
//
// The array's host-side name is only a stand-in for the device symbol, so its
// device address is looked up once per device with cudaGetSymbolAddress, with
// that device current, on the first call made on that device. Make that first
// call before any stream capture. All calls on a device share the one array
// and each call clears the part it uses before its kernel runs; calls that
// overlap on the GPU (on different streams, or from several host threads)
// race on it and must be serialized by the caller.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(1) << 20; // 1 MiB per device

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

void *g_noalloc_ptr[128];
std::mutex g_noalloc_mu;

int noalloc_scratch(cudaStream_t stream, void **out)
{
    // the array of the stream's device; the kernels launch on the current
    // device, so the two must agree
    int d = 0, sd = 0;
    if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= 128 || cudaStreamGetDevice(stream, &sd) != cudaSuccess)
        return MXQ_ERR_CUDA;
    if (sd != d)
        return MXQ_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[d]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p)
            return MXQ_ERR_CUDA;
        g_noalloc_ptr[d] = p;
    }
    *out = g_noalloc_ptr[d];
    return MXQ_OK;
}

} // namespace

extern "C" int fp8_quant_jagged_colwise_noalloc(const void *in, int64_t rows, int64_t cols, int64_t stride_row,
                                                int64_t stride_col, const int32_t *offs, int32_t num_groups,
                                                void *out, float *inv_scales, cudaStream_t stream)
{
    if (rows < 0 || cols < 0 || num_groups < 1)
        return MXQ_ERR_SHAPE;
    // the plan of this very call (real pointers): only the kernels that keep
    // a table need scratch, and only they are limited by the array's size
    JaggedPlan pl;
    int rc = plan_jagged(in, cols, rows, stride_col, stride_row, num_groups, out, &pl);
    if (rc != MXQ_OK)
        return rc;
    void *scratch = nullptr;
    if (pl.ws > 0) {
        if (pl.ws > kNoAllocScratchBytes)
            return MXQ_ERR_WORKSPACE;
        rc = noalloc_scratch(stream, &scratch);
        if (rc != MXQ_OK)
            return rc;
    }
    return fp8_quant_jagged_colwise(in, rows, cols, stride_row, stride_col, offs, num_groups, out, inv_scales,
                                    scratch, scratch ? kNoAllocScratchBytes : 0, stream);
}

extern "C" size_t fp8_quant_jagged_colwise_noalloc_max_scratch_bytes(void) { return kNoAllocScratchBytes; }

extern "C" {

int mxq_device_status(cudaStream_t stream, int32_t *host_status)
{
    if (!host_status)
        return MXQ_ERR_NULL;
    int v = 0;
    const int zero = 0;
    if (cudaMemcpyFromSymbolAsync(&v, g_status, sizeof(int), 0, cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
        cudaMemcpyToSymbolAsync(g_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, stream) != cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess)
        return MXQ_ERR_CUDA;
    *host_status = v;
    return MXQ_OK;
}

const char *mxq_status_string(int status)
{
    switch (status) {
    case MXQ_OK: return "ok";
    case MXQ_ERR_NULL: return "null pointer";
    case MXQ_ERR_SHAPE: return "invalid shape";
    case MXQ_ERR_ALIGN: return "misaligned pointer or stride";
    case MXQ_ERR_UNSUPPORTED: return "unsupported parameters";
    case MXQ_ERR_LAUNCH: return "kernel launch failed";
    case MXQ_ERR_BAD_OFFSETS: return "malformed group offsets";
    case MXQ_ERR_TIMEOUT: return "device wait timed out";
    case MXQ_ERR_WORKSPACE: return "workspace missing or too small";
    case MXQ_ERR_CUDA: return "CUDA runtime error";
    default: return "unknown status";
    }
}

int mxq_version(void) { return 10000; }

int mxq_testing_set(int32_t what, int64_t value)
{
    switch (what) {
    case MXQ_TESTING_WAIT_LIMIT_NS: g_wait_ns.store(value > 0 ? value : 1000000000LL); return MXQ_OK;
    case MXQ_TESTING_SKIP_ARRIVAL: g_drop_load.store(value ? 1 : 0); return MXQ_OK;
    case MXQ_TESTING_FORCE_PATH:
        if (value < 0 || value > 3)
            return MXQ_ERR_UNSUPPORTED;
        g_force_path.store((int)value);
        return MXQ_OK;
    case MXQ_TESTING_GEMM_TILE_N:
        if (value != 0 && value != 128)
            return MXQ_ERR_UNSUPPORTED;
        g_mx_bn.store((int)value);
        return MXQ_OK;
    case MXQ_TESTING_BLOCKED_PATH:
        if (value != 0 && value != 1)
            return MXQ_ERR_UNSUPPORTED;
        g_blocked_words.store((int)value);
        return MXQ_OK;
    case MXQ_TESTING_GEMM_ONE_SM:
        if (value != 0 && value != 1)
            return MXQ_ERR_UNSUPPORTED;
        g_gemm_one_sm.store((int)value);
        return MXQ_OK;
    default: return MXQ_ERR_UNSUPPORTED;
    }
}

} // extern "C"
