// common.cuh - device helpers shared by the libmxq kernels (sm_100a).
//
// PTX wrappers for mbarriers, TMA (cp.async.bulk.tensor) and bulk groups,
// the device status word, and the scalar conversions of the quantization
// path written against PTX instructions (cvt ... e4m3x2) and IEEE fp32
// operations; no approximate math is used anywhere.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "mxq.h"

#define MXQ_DEV __device__ __forceinline__

namespace mxq {

// First error recorded by any kernel since the host last read it.
__device__ int g_status;

MXQ_DEV void set_status(int code) { atomicCAS(&g_status, 0, code); }

MXQ_DEV uint64_t globaltimer()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

MXQ_DEV uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

// ---------------------------------------------------------------- mbarrier
MXQ_DEV void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

MXQ_DEV void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

MXQ_DEV void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

MXQ_DEV void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Release a TMA ring slot this warp has read with ordinary loads: every lane
// orders its reads (generic proxy) before the next fill of the slot (a TMA
// write, async proxy) with a proxy fence, issued once `dep` - a value
// computed from every word the lane loaded - is available, so no load is
// still in flight; then lane 0 arrives on the slot's empty barrier. Without
// the fence the refill can overwrite words the loads have not read.
MXQ_DEV void release_slot_after(uint64_t *empty, uint32_t dep)
{
    asm volatile("fence.proxy.async.shared::cta;" ::"r"(dep) : "memory");
    __syncwarp();
    if ((threadIdx.x & 31) == 0)
        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(empty)) : "memory");
    __syncwarp();
}

MXQ_DEV bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait until the phase with the given parity has completed, for at most
// limit_ns; on expiry record MXQ_ERR_TIMEOUT and return false.
MXQ_DEV bool mbar_wait(uint64_t *bar, uint32_t parity, uint64_t limit_ns)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = globaltimer();
    for (;;) {
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait(bar, parity))
                return true;
        if (globaltimer() - t0 > limit_ns) {
            set_status(MXQ_ERR_TIMEOUT);
            return false;
        }
    }
}

// ---------------------------------------------------------------- TMA
MXQ_DEV void tma_load_2d(void *dst, const CUtensorMap *map, uint64_t *bar, int x, int y)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

MXQ_DEV void tma_load_3d(void *dst, const CUtensorMap *map, uint64_t *bar, int x, int y, int z)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
        "l"(map), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}

MXQ_DEV void tma_store_2d(const CUtensorMap *map, const void *src, int x, int y)
{
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(map),
                 "r"(smem_u32(src)), "r"(x), "r"(y)
                 : "memory");
}

MXQ_DEV void tma_store_3d(const CUtensorMap *map, const void *src, int x, int y, int z)
{
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(map),
                 "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
                 : "memory");
}

MXQ_DEV void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

template <int N> MXQ_DEV void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory"); }

template <int N> MXQ_DEV void bulk_wait() { asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory"); }

// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (TMA stores that read them).
MXQ_DEV void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

MXQ_DEV void named_barrier(int id, int nthreads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Named barrier over `n` threads that also ORs `pred` across them: every
// participant gets the same answer, so a stop decision taken at it is
// uniform and no thread is left waiting at a later barrier.
MXQ_DEV bool barrier_or(int id, int n, bool pred)
{
    uint32_t r;
    asm volatile("{\n\t.reg .pred p, q;\n\t"
                 "setp.ne.u32 p, %1, 0;\n\t"
                 "bar.red.or.pred q, %2, %3, p;\n\t"
                 "selp.u32 %0, 1, 0, q;\n\t}"
                 : "=r"(r)
                 : "r"((uint32_t)pred), "r"(id), "r"(n)
                 : "memory");
    return r != 0;
}

// ---------------------------------------------------------------- memory
MXQ_DEV uint4 ld_stream_v4(const void *p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

MXQ_DEV void st_v2(void *p, uint32_t a, uint32_t b)
{
    asm volatile("st.global.v2.u32 [%0], {%1, %2};" ::"l"(p), "r"(a), "r"(b) : "memory");
}

MXQ_DEV void st_v4(void *p, uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

MXQ_DEV void sts_v4(uint32_t addr, uint4 v)
{
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

MXQ_DEV int ld_acquire_gpu(const int *p)
{
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

MXQ_DEV void red_release_gpu_add(int *p, int v)
{
    asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// ---------------------------------------------------------------- numerics
// bf16 is the upper half of an fp32 word: widening is exact bit placement.
MXQ_DEV float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
MXQ_DEV float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Running max of |x| over packed bf16 pairs (exact: a max of bf16 values).
MXQ_DEV uint32_t absmax_bf16x2(uint32_t acc, uint32_t w)
{
    uint32_t d;
    const uint32_t a = w & 0x7FFF7FFFu;
    asm("max.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(acc), "r"(a));
    return d;
}

MXQ_DEV float absmax_of_pair(uint32_t acc) { return fmaxf(bf16_lo(acc), bf16_hi(acc)); }

// Two fp32 values -> two e4m3 bytes (lo in the low byte), round to nearest
// even, saturating to +-448 (cvt ... satfinite).
MXQ_DEV uint32_t e4m3x2(float lo, float hi)
{
    uint16_t d;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
    return (uint32_t)d;
}

// Four e4m3 bytes from the packed bf16 pairs w0 = (x0, x1), w1 = (x2, x3),
// each multiplied by s in fp32 first.
MXQ_DEV uint32_t quant4(uint32_t w0, uint32_t w1, float s)
{
    const uint32_t a = e4m3x2(__fmul_rn(bf16_lo(w0), s), __fmul_rn(bf16_hi(w0), s));
    const uint32_t b = e4m3x2(__fmul_rn(bf16_lo(w1), s), __fmul_rn(bf16_hi(w1), s));
    return a | (b << 16);
}

// float8 e4m3 unit scale: s = 448 / max(amax, 1e-12), IEEE fp32 division.
MXQ_DEV float fp8_scale(float amax) { return __fdiv_rn(448.0f, fmaxf(amax, 1e-12f)); }
MXQ_DEV float fp8_inv(float s) { return __fdiv_rn(1.0f, s); }

// E8M0 scale byte, floor mode: floor(log2 amax) - 8, clamped to [-127, 127],
// biased by 127. Read from the fp32 exponent field; zero and subnormal amax
// give the smallest scale.
MXQ_DEV uint32_t e8m0_floor(float amax)
{
    const int e = (int)(__float_as_uint(amax) >> 23); // amax >= 0
    int k = e - 127 - 8;
    k = k < -127 ? -127 : (k > 127 ? 127 : k);
    return (uint32_t)(k + 127);
}

// E8M0 scale byte, rceil mode: ceil(log2(amax / 448)), clamped to
// [-127, 127], biased by 127. For a normal amax = M * 2^E with M in [1, 2),
// amax / 448 = (M / 1.75) * 2^(E - 8) and log2(M / 1.75) lies in (-1, 0] for
// M <= 1.75 and in (0, 1) above, so the exponent is E - 8 plus one exactly
// when the mantissa exceeds 1.75 (fraction bits > 0x600000). Zero and
// subnormal amax lie below 448 * 2^-127 and give the smallest scale.
MXQ_DEV uint32_t e8m0_rceil(float amax)
{
    const uint32_t bits = __float_as_uint(amax); // amax >= 0
    const int e = (int)(bits >> 23);
    if (e == 0)
        return 0u;
    int k = e - 127 - 8 + ((bits & 0x7FFFFFu) > 0x600000u ? 1 : 0);
    k = k < -127 ? -127 : (k > 127 ? 127 : k);
    return (uint32_t)(k + 127);
}

MXQ_DEV uint32_t e8m0_mode(float amax, int mode) { return mode == MXQ_E8M0_RCEIL ? e8m0_rceil(amax) : e8m0_floor(amax); }

// 2^(127 - byte) as an exact fp32 power of two (byte <= 253).
MXQ_DEV float mx_factor(uint32_t byte) { return __uint_as_float((254u - byte) << 23); }

} // namespace mxq
