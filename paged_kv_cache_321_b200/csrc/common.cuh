// Shared internals of libkvpaged: the pool handle, error reporting, and the
// sm_100a device primitives (mbarrier, 1-D bulk async copy, 16-bit
// conversion) used by the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/kvpaged.h"

struct kvp_pool {
    kvp_cache_config cfg;
    uint16_t *k_base;
    uint16_t *v_base;
    size_t layer_words;  // num_blocks * Hkv * block_size * D
    int *status;         // device: [0] first error code, [1] detail
};

namespace kvp {

// ------------------------------------------------------------------ host side
int set_error(int code, const char *fmt, ...);
int check_cuda(cudaError_t e, const char *what);
int check_pool(const kvp_pool *pool, int layer);
// Resolves num_kv_heads == 0 and checks the attention config against the pool.
int resolve_attn(const kvp_pool *pool, const kvp_attn_config *attn, int *Hq, int *Hkv, int *G);

inline bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

// Tensor map over one layer's K or V pool viewed as [blocks*Hkv][bs][D] 16-bit
// words, with a box of 64 columns x box_rows rows x 1 (block, head) tile and
// the 128-byte swizzle (the canonical layout of a 128-byte-row operand).
int make_pool_tmap(CUtensorMap *map, const uint16_t *base, const kvp_pool *pool, int box_rows);

// --------------------------------------------------------------- device side
constexpr int kWaitLimitNs = 1000 * 1000 * 1000;  // 1 s bound on any wait

__device__ __forceinline__ void report(int *status, int code, int detail)
{
    if (atomicCAS(status, 0, code) == 0) status[1] = detail;
}

__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// Makes the initialised barriers visible to the async (bulk copy) proxy.
__device__ __forceinline__ void mbar_init_fence()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred P;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, P;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Waits for phase `parity` of the barrier to complete, giving up after
// kWaitLimitNs. Returns false on timeout.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if (global_ns() - t0 > (uint64_t)kWaitLimitNs) return false;
    }
}

// Orders this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy (bulk copy) writes to the same memory.
__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 1-D bulk copy global -> shared (no multicast), completing on `bar`.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// L2 policy for data read exactly once (streamed K/V): its lines are the
// first to go, so small reused data (block tables, queries, partials) stays.
__device__ __forceinline__ uint64_t l2_evict_first_policy()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// bulk_g2s with an L2 cache policy.
__device__ __forceinline__ void bulk_g2s_hint(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar,
                                              uint64_t pol)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar), "l"(pol)
        : "memory");
}

__device__ __forceinline__ void prefetch_l2(const void *p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }
__device__ __forceinline__ void prefetch_l1(const void *p) { asm volatile("prefetch.global.L1 [%0];" ::"l"(p)); }

// Programmatic dependent launch: wait until the grid launched before this one
// on the stream has completed and its writes are visible (a no-op without a
// programmatic dependency), and let the next grid start launching.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Launches `kern` on `s` with the programmatic stream serialization
// attribute, so its launch and prologue may overlap the previous grid.
template <typename... Args>
inline cudaError_t launch_pdl(void (*kern)(Args...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

// ------------------------------------------------------------- conversions
// Nearest 16-bit value, ties to the even fraction, overflow to infinity,
// subnormals kept (the hardware cvt.rn forms are IEEE round-to-nearest-even
// without flush-to-zero); a NaN keeps its sign and top payload bits and gets
// the quiet bit, which the hardware forms would replace by a canonical NaN.
__device__ __forceinline__ uint16_t nan_to_f16(uint32_t b)
{
    return static_cast<uint16_t>(((b >> 16) & 0x8000u) | 0x7E00u | ((b & 0x7FFFFFu) >> 13));
}
__device__ __forceinline__ uint16_t nan_to_bf16(uint32_t b)
{
    return static_cast<uint16_t>((b >> 16) | 0x0040u);
}
__device__ __forceinline__ bool is_nan_bits(uint32_t b) { return (b & 0x7FFFFFFFu) > 0x7F800000u; }

template <bool BF16>
__device__ __forceinline__ uint32_t cvt_pair(float lo, float hi)
{
    uint32_t r;
    if (BF16) {
        __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
        r = *reinterpret_cast<uint32_t *>(&h);
    } else {
        __half2 h = __floats2half2_rn(lo, hi);
        r = *reinterpret_cast<uint32_t *>(&h);
    }
    const uint32_t bl = __float_as_uint(lo), bh = __float_as_uint(hi);
    if (is_nan_bits(bl)) r = (r & 0xFFFF0000u) | (BF16 ? nan_to_bf16(bl) : nan_to_f16(bl));
    if (is_nan_bits(bh)) r = (r & 0x0000FFFFu) | (uint32_t(BF16 ? nan_to_bf16(bh) : nan_to_f16(bh)) << 16);
    return r;
}

// Two packed 16-bit values -> float2 (exact).
template <bool BF16>
__device__ __forceinline__ float2 unpack2(uint32_t w)
{
    if (BF16) return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
    __half2 h = *reinterpret_cast<__half2 *>(&w);
    return __half22float2(h);
}

}  // namespace kvp
