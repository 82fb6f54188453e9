// Pool handle, error reporting, RoPE table set-up and the exported
// conversion kernels of libkvpaged.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <vector>

#include <mutex>

#include "common.cuh"

namespace kvp {

static thread_local char g_msg[512] = "";

int set_error(int code, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
    va_end(ap);
    return code;
}

int check_cuda(cudaError_t e, const char *what)
{
    if (e == cudaSuccess) return KVP_OK;
    return set_error(KVP_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

int check_pool(const kvp_pool *pool, int layer)
{
    if (!pool) return set_error(KVP_EINVAL, "pool is NULL");
    if (layer < 0 || layer >= pool->cfg.num_layers)
        return set_error(KVP_EINVAL, "invalid layer %d (pool has %d)", layer, pool->cfg.num_layers);
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != pool->cfg.device)
        return set_error(KVP_EINVAL, "current device %d is not the pool's device %d", dev, pool->cfg.device);
    return KVP_OK;
}

int resolve_attn(const kvp_pool *pool, const kvp_attn_config *attn, int *Hq, int *Hkv, int *G)
{
    if (!attn) return set_error(KVP_EINVAL, "attention config is NULL");
    const int hq = attn->num_heads;
    const int hkv = attn->num_kv_heads == 0 ? attn->num_heads : attn->num_kv_heads;
    if (hq <= 0 || hkv <= 0 || hq % hkv)
        return set_error(KVP_EINVAL, "num_heads %d must be a positive multiple of num_kv_heads %d", hq, hkv);
    if (attn->head_dim != pool->cfg.head_dim)
        return set_error(KVP_EINVAL, "head_dim %d differs from the pool's %d", attn->head_dim, pool->cfg.head_dim);
    if (hkv != pool->cfg.num_kv_heads)
        return set_error(KVP_EINVAL, "num_kv_heads %d differs from the pool's %d", hkv, pool->cfg.num_kv_heads);
    if (attn->rope_dim < 0 || attn->rope_dim > attn->head_dim || (attn->rope_dim & 1))
        return set_error(KVP_EINVAL, "rope_dim %d must be 0 or even and <= head_dim", attn->rope_dim);
    if (attn->rope_style != KVP_ROPE_HALF && attn->rope_style != KVP_ROPE_INTERLEAVED)
        return set_error(KVP_EINVAL, "rope_style %d is neither KVP_ROPE_HALF nor KVP_ROPE_INTERLEAVED",
                         attn->rope_style);
    if (attn->window < 0) return set_error(KVP_EINVAL, "window %d must be >= 0", attn->window);
    *Hq = hq;
    *Hkv = hkv;
    *G = hq / hkv;
    return KVP_OK;
}

// ------------------------------------------------------------ conversions
template <bool BF16>
__global__ void convert_kernel(const float *__restrict__ x, uint16_t *__restrict__ out, int64_t n)
{
    const int64_t i = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 2;
    if (i + 1 < n) {
        const float2 v = *reinterpret_cast<const float2 *>(x + i);
        *reinterpret_cast<uint32_t *>(out + i) = cvt_pair<BF16>(v.x, v.y);
    } else if (i < n) {
        out[i] = static_cast<uint16_t>(cvt_pair<BF16>(x[i], 0.0f) & 0xFFFFu);
    }
}

template <bool BF16>
__global__ void convert_bits_kernel(uint64_t start, uint16_t *__restrict__ out, int64_t count)
{
    const int64_t i = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 2;
    if (i + 1 < count) {
        const float lo = __uint_as_float(static_cast<uint32_t>(start + i));
        const float hi = __uint_as_float(static_cast<uint32_t>(start + i + 1));
        *reinterpret_cast<uint32_t *>(out + i) = cvt_pair<BF16>(lo, hi);
    } else if (i < count) {
        out[i] = static_cast<uint16_t>(cvt_pair<BF16>(__uint_as_float(static_cast<uint32_t>(start + i)), 0.0f) &
                                       0xFFFFu);
    }
}

}  // namespace kvp

using namespace kvp;

extern "C" {

const char *kvp_last_error(void) { return g_msg; }

int kvp_version(void) { return 100; }

int kv_pool_create(const kvp_cache_config *cfg, void *k_base, void *v_base, kvp_pool **out)
{
    if (!cfg || !out) return set_error(KVP_EINVAL, "config or output handle is NULL");
    *out = nullptr;
    if (!k_base || !v_base) return set_error(KVP_EINVAL, "pool memory is NULL");
    if (cfg->num_layers <= 0 || cfg->num_kv_heads <= 0 || cfg->num_blocks <= 0 || cfg->max_seq_len <= 0)
        return set_error(KVP_EINVAL, "num_layers, num_kv_heads, num_blocks and max_seq_len must be positive");
    if (cfg->head_dim != 64 && cfg->head_dim != 128 && cfg->head_dim != 256)
        return set_error(KVP_EUNSUPPORTED, "head_dim %d not built (64, 128, 256)", cfg->head_dim);
    if (!is_pow2(cfg->block_size) || cfg->block_size > 256)
        return set_error(KVP_EUNSUPPORTED, "block_size %d must be a power of two <= 256", cfg->block_size);
    if (cfg->kv_dtype != KVP_F16 && cfg->kv_dtype != KVP_BF16)
        return set_error(KVP_EINVAL, "kv_dtype %d is neither KVP_F16 nor KVP_BF16", cfg->kv_dtype);
    if ((reinterpret_cast<uintptr_t>(k_base) | reinterpret_cast<uintptr_t>(v_base)) & 255)
        return set_error(KVP_EINVAL, "pool memory must be 256-byte aligned");
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != cfg->device)
        return set_error(KVP_EINVAL, "current device %d is not the pool's device %d", dev, cfg->device);
    kvp_pool *p = static_cast<kvp_pool *>(calloc(1, sizeof(kvp_pool)));
    if (!p) return set_error(KVP_EINVAL, "out of host memory");
    p->cfg = *cfg;
    p->k_base = static_cast<uint16_t *>(k_base);
    p->v_base = static_cast<uint16_t *>(v_base);
    p->layer_words = static_cast<size_t>(cfg->num_blocks) * cfg->num_kv_heads * cfg->block_size * cfg->head_dim;
    int rc = check_cuda(cudaMalloc(&p->status, 2 * sizeof(int)), "cudaMalloc(status)");
    if (rc == KVP_OK) rc = check_cuda(cudaMemset(p->status, 0, 2 * sizeof(int)), "cudaMemset(status)");
    if (rc != KVP_OK) {
        if (p->status) cudaFree(p->status);
        free(p);
        return rc;
    }
    *out = p;
    return KVP_OK;
}

int kv_pool_destroy(kvp_pool *pool)
{
    if (!pool) return KVP_OK;
    const int rc = check_cuda(cudaFree(pool->status), "cudaFree(status)");
    free(pool);
    return rc;
}

int kv_pool_layer_ptrs(const kvp_pool *pool, int layer, void **k, void **v)
{
    if (!pool || layer < 0 || layer >= pool->cfg.num_layers)
        return set_error(KVP_EINVAL, "invalid pool or layer %d", layer);
    if (k) *k = pool->k_base + pool->layer_words * layer;
    if (v) *v = pool->v_base + pool->layer_words * layer;
    return KVP_OK;
}

int kv_pool_sync_status(kvp_pool *pool, void *stream, int *device_code)
{
    if (!pool) return set_error(KVP_EINVAL, "pool is NULL");
    if (device_code) *device_code = KVP_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int rc = check_cuda(cudaStreamSynchronize(s), "cudaStreamSynchronize");
    if (rc != KVP_OK) return rc;
    int st[2] = {0, 0};
    rc = check_cuda(cudaMemcpy(st, pool->status, sizeof(st), cudaMemcpyDeviceToHost), "read status");
    if (rc != KVP_OK) return rc;
    if (st[0] == 0) return KVP_OK;
    rc = check_cuda(cudaMemset(pool->status, 0, sizeof(st)), "clear status");
    if (rc != KVP_OK) return rc;
    if (device_code) *device_code = st[0];
    const char *what = st[0] == KVP_ERANGE      ? "block id, block index or context length out of range"
                       : st[0] == KVP_EOVERFLOW ? "KV cache overflow: position past max_seq_len or the rope table"
                       : st[0] == KVP_EINVAL    ? "token refers to an unknown sequence"
                       : st[0] == KVP_ETIMEOUT  ? "a bounded wait inside a kernel ran out"
                                                : "unknown device error";
    return set_error(KVP_EDEVICE, "device error %d (%s), detail %d", st[0], what, st[1]);
}

// Rotary width of a config: rope_dim, or head_dim when 0 (-1 if invalid).
static int rotary_width(const kvp_attn_config *attn)
{
    const int D = attn->head_dim, R = attn->rope_dim == 0 ? D : attn->rope_dim;
    return (D <= 0 || (D & 1) || R <= 0 || R > D || (R & 1)) ? -1 : R;
}

size_t kvp_rope_table_bytes(const kvp_attn_config *attn, int max_pos)
{
    if (!attn || rotary_width(attn) < 0 || max_pos <= 0) return 0;
    return static_cast<size_t>(max_pos) * rotary_width(attn) * sizeof(float);
}

int kvp_rope_table_fill(const kvp_attn_config *attn, int max_pos, float *table)
{
    if (!attn || !table) return set_error(KVP_EINVAL, "config or table is NULL");
    const int D = attn->head_dim;
    if (D <= 0 || D > 256 || (D & 1))
        return set_error(KVP_EUNSUPPORTED, "rope needs an even head_dim <= 256 (got %d)", D);
    const int R = rotary_width(attn);
    if (R < 0) return set_error(KVP_EINVAL, "rope_dim %d must be 0 or even and <= head_dim", attn->rope_dim);
    if (!(attn->rope_theta > 0.0f)) return set_error(KVP_EINVAL, "rope_theta must be > 0");
    if (max_pos <= 0) return set_error(KVP_EINVAL, "max_pos must be > 0");
    const int half = R / 2;
    const double theta = static_cast<double>(attn->rope_theta);
    std::vector<double> inv_freq(half);
    for (int i = 0; i < half; ++i) inv_freq[i] = ::pow(theta, -(2.0 * static_cast<double>(i)) / static_cast<double>(R));
    std::vector<float> host(static_cast<size_t>(max_pos) * R);
    for (int p = 0; p < max_pos; ++p) {
        float *row = host.data() + static_cast<size_t>(p) * R;
        for (int i = 0; i < half; ++i) {
            const double ang = static_cast<double>(p) * inv_freq[i];
            row[2 * i] = static_cast<float>(::cos(ang));
            row[2 * i + 1] = static_cast<float>(::sin(ang));
        }
    }
    return check_cuda(cudaMemcpy(table, host.data(), host.size() * sizeof(float), cudaMemcpyHostToDevice),
                      "copy rope table");
}

int kvp_convert_f32(const float *x, uint16_t *out, int64_t n, int kv_dtype, void *stream)
{
    if (n < 0 || (n > 0 && (!x || !out))) return set_error(KVP_EINVAL, "bad convert arguments");
    if (kv_dtype != KVP_F16 && kv_dtype != KVP_BF16) return set_error(KVP_EINVAL, "bad kv_dtype %d", kv_dtype);
    if ((reinterpret_cast<uintptr_t>(x) & 7) || (reinterpret_cast<uintptr_t>(out) & 3))
        return set_error(KVP_EINVAL, "x must be 8-byte and out 4-byte aligned");
    if (n == 0) return KVP_OK;
    const int threads = 256;
    const int64_t blocks = (n + 2 * threads - 1) / (2 * threads);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (kv_dtype == KVP_BF16)
        convert_kernel<true><<<static_cast<unsigned>(blocks), threads, 0, s>>>(x, out, n);
    else
        convert_kernel<false><<<static_cast<unsigned>(blocks), threads, 0, s>>>(x, out, n);
    return check_cuda(cudaGetLastError(), "convert launch");
}

int kvp_convert_bits(uint64_t start, int64_t count, int kv_dtype, uint16_t *out, void *stream)
{
    if (count < 0 || (count > 0 && !out)) return set_error(KVP_EINVAL, "bad convert arguments");
    if (kv_dtype != KVP_F16 && kv_dtype != KVP_BF16) return set_error(KVP_EINVAL, "bad kv_dtype %d", kv_dtype);
    if (reinterpret_cast<uintptr_t>(out) & 3) return set_error(KVP_EINVAL, "out must be 4-byte aligned");
    if (count > (int64_t(1) << 32)) return set_error(KVP_EINVAL, "count above 2^32");
    if (count == 0) return KVP_OK;
    const int threads = 256;
    const int64_t blocks = (count + 2 * threads - 1) / (2 * threads);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (kv_dtype == KVP_BF16)
        convert_bits_kernel<true><<<static_cast<unsigned>(blocks), threads, 0, s>>>(start, out, count);
    else
        convert_bits_kernel<false><<<static_cast<unsigned>(blocks), threads, 0, s>>>(start, out, count);
    return check_cuda(cudaGetLastError(), "convert launch");
}

}  // extern "C"

// ------------------------------------------------------------ tensor maps
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

}  // namespace

int kvp::make_pool_tmap(CUtensorMap *map, const uint16_t *base, const kvp_pool *pool, int box_rows)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return set_error(KVP_ECUDA, "cuTensorMapEncodeTiled is unavailable");
    const kvp_cache_config &c = pool->cfg;
    if (box_rows < 1 || box_rows > c.block_size || box_rows > 256)
        return set_error(KVP_EUNSUPPORTED, "tensor map box of %d rows over blocks of %d", box_rows, c.block_size);
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(c.head_dim), static_cast<cuuint64_t>(c.block_size),
                          static_cast<cuuint64_t>(c.num_blocks) * c.num_kv_heads};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(c.head_dim) * 2,
                             static_cast<cuuint64_t>(c.head_dim) * c.block_size * 2};
    cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = fn(map, c.kv_dtype == KVP_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                          3, const_cast<uint16_t *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return set_error(KVP_ECUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    return KVP_OK;
}
