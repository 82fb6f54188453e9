// kv_append: per-head q/k RMSNorm -> RoPE -> fp32 -> fp16/bf16 (nearest,
// ties to even) -> scatter into the token's block slot.
//
// The step of makarna/pkg/model/arch/hybrid_decoder.go (runHybridAttentionBlock:
// QNorm/KNorm, RoPE, cache.Append) fused into one launch, with the slot rule
// and conversion of makarna/pkg/kvcache/paged_cache.go (Append / AppendKV,
// GetBlockForPosition, GetBlockOffset, float32ToFloat16Bits,
// float32ToBFloat16Bits). The RMS form follows forward_layer in
// soft3/glia/run/arch/decoder/forward.rs.
//
// Mapping: one warp per (token, row), rows = Hq query heads, Hkv key heads,
// Hkv value heads. Lane l owns the D/32 consecutive elements starting at
// l*D/32, so for full rotate-half RoPE the partner of every element sits in
// lane l^16; partial or interleaved RoPE (the per-layer rope_dim of
// forward_layer in soft3/glia/run/arch/decoder/forward.rs) reads the partner
// from the row staged in shared memory.
// The sum of squares is taken in order d = 0..D-1 from shared memory (every
// lane reads the same addresses, a broadcast), each product and sum a
// separate IEEE operation; RoPE uses separately rounded products and sums.
// Launch-bound for decode batches (T rows of ~1 KB): the kernel's job is to
// issue all rows at once, so each warp handles exactly one row.
#include "common.cuh"

namespace kvp {

struct AppendParams {
    const float *q, *k, *v;
    const float *qn, *kn;
    const float2 *rope;  // [rope_max_pos][D/2] (cos, sin) or nullptr
    const int32_t *tok_req, *positions, *bt;
    uint16_t *pk, *pv;  // this layer's pools
    float *q_out;
    int *status;
    int T, S, Hq, Hkv, bs, mbps, num_blocks, max_seq_len, rope_max_pos;
    int R, style, window;  // rotary width, pairing, sliding window (> 0: ring rows)
    float eps;
};

constexpr int kAppendWarps = 8;

template <int D>
struct RowVec {
    static constexpr int E = D / 32;  // elements per lane: 2, 4 or 8
    float x[E];
    __device__ __forceinline__ void load(const float *src)
    {
        if constexpr (E == 2) {
            const float2 a = *reinterpret_cast<const float2 *>(src);
            x[0] = a.x, x[1] = a.y;
        } else {
#pragma unroll
            for (int i = 0; i < E; i += 4) {
                const float4 a = *reinterpret_cast<const float4 *>(src + i);
                x[i] = a.x, x[i + 1] = a.y, x[i + 2] = a.z, x[i + 3] = a.w;
            }
        }
    }
    __device__ __forceinline__ void store(float *dst) const
    {
        if constexpr (E == 2) {
            *reinterpret_cast<float2 *>(dst) = make_float2(x[0], x[1]);
        } else {
#pragma unroll
            for (int i = 0; i < E; i += 4)
                *reinterpret_cast<float4 *>(dst + i) = make_float4(x[i], x[i + 1], x[i + 2], x[i + 3]);
        }
    }
    template <bool BF16>
    __device__ __forceinline__ void store16(uint16_t *dst) const
    {
        uint32_t w[E / 2];
#pragma unroll
        for (int i = 0; i < E / 2; ++i) w[i] = cvt_pair<BF16>(x[2 * i], x[2 * i + 1]);
        if constexpr (E == 2)
            *reinterpret_cast<uint32_t *>(dst) = w[0];
        else if constexpr (E == 4)
            *reinterpret_cast<uint2 *>(dst) = make_uint2(w[0], w[1]);
        else
            *reinterpret_cast<uint4 *>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
    }
};

template <int D, bool BF16>
__global__ void __launch_bounds__(kAppendWarps * 32) kv_append_kernel(const AppendParams p)
{
    constexpr int E = D / 32;
    __shared__ __align__(16) float rowbuf[kAppendWarps][D];
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    const int R = p.Hq + 2 * p.Hkv;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * kAppendWarps + wib;
    // launched with a programmatic dependency: wait for the previous grid's
    // results, then let the next grid launch (it waits for this one in turn)
    grid_dependency_wait();
    grid_launch_dependents();
    if (row >= static_cast<int64_t>(p.T) * R) return;
    const int t = static_cast<int>(row / R), rr = static_cast<int>(row % R);
    const int kind = rr < p.Hq ? 0 : (rr < p.Hq + p.Hkv ? 1 : 2);  // q, k, v
    const int head = kind == 0 ? rr : (kind == 1 ? rr - p.Hq : rr - p.Hq - p.Hkv);

    const int r = p.tok_req[t], pos = p.positions[t];
    const bool seq_ok = r >= 0 && r < p.S;
    const bool pos_ok = pos >= 0 && pos < p.max_seq_len && (p.rope == nullptr || pos < p.rope_max_pos);
    if (!seq_ok || !pos_ok) {
        if (rr == 0 && lane == 0) report(p.status, seq_ok ? KVP_EOVERFLOW : KVP_EINVAL, t);
        if (kind == 0) {
            RowVec<D> z;
#pragma unroll
            for (int e = 0; e < E; ++e) z.x[e] = 0.0f;
            z.store(p.q_out + (static_cast<int64_t>(t) * p.Hq + head) * D + lane * E);
        }
        return;
    }

    const float *src = kind == 0 ? p.q + (static_cast<int64_t>(t) * p.Hq + head) * D
                                 : (kind == 1 ? p.k : p.v) + (static_cast<int64_t>(t) * p.Hkv + head) * D;
    RowVec<D> x;
    x.load(src + lane * E);

    if (kind != 2) {
        const float *w = kind == 0 ? p.qn : p.kn;
        if (w != nullptr) {
            x.store(&rowbuf[wib][lane * E]);
            __syncwarp();
            float ss = 0.0f;
#pragma unroll 8
            for (int d = 0; d < D; d += 4) {
                const float4 a = *reinterpret_cast<const float4 *>(&rowbuf[wib][d]);
                ss = __fadd_rn(ss, __fmul_rn(a.x, a.x));
                ss = __fadd_rn(ss, __fmul_rn(a.y, a.y));
                ss = __fadd_rn(ss, __fmul_rn(a.z, a.z));
                ss = __fadd_rn(ss, __fmul_rn(a.w, a.w));
            }
            const float ms = __fmul_rn(ss, __fdiv_rn(1.0f, static_cast<float>(D)));
            const float inv = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, p.eps)));
            RowVec<D> wv;
            wv.load(w + lane * E);
#pragma unroll
            for (int e = 0; e < E; ++e) x.x[e] = __fmul_rn(__fmul_rn(x.x[e], inv), wv.x[e]);
        }
        if (p.rope != nullptr && p.R == D && p.style == KVP_ROPE_HALF) {
            // lanes 0..15 hold dims [0, D/2), lanes 16..31 the partners [D/2, D)
            const float2 *cs = p.rope + static_cast<int64_t>(pos) * (D / 2) + (lane & 15) * E;
            const bool lower = lane < 16;
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const float other = __shfl_xor_sync(0xffffffffu, x.x[e], 16);
                const float2 c = cs[e];
                x.x[e] = lower ? __fsub_rn(__fmul_rn(x.x[e], c.x), __fmul_rn(other, c.y))
                               : __fadd_rn(__fmul_rn(x.x[e], c.x), __fmul_rn(other, c.y));
            }
        } else if (p.rope != nullptr) {
            // pair i turns (a, b) = (i, i + R/2) or (2i, 2i + 1) of the first
            // R dims: y_a = x_a c - x_b s, y_b = x_b c + x_a s
            __syncwarp();  // every lane is done reading the norm's staging
            x.store(&rowbuf[wib][lane * E]);
            __syncwarp();
            const float2 *cs = p.rope + static_cast<int64_t>(pos) * (p.R / 2);
            const int hr = p.R / 2;
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const int d = lane * E + e;
                if (d >= p.R) continue;
                const bool inter = p.style == KVP_ROPE_INTERLEAVED;
                const bool lower = inter ? (d & 1) == 0 : d < hr;
                const int i = inter ? d >> 1 : (lower ? d : d - hr);
                const int partner = inter ? d ^ 1 : (lower ? d + hr : d - hr);
                const float other = rowbuf[wib][partner];
                const float2 c = cs[i];
                x.x[e] = lower ? __fsub_rn(__fmul_rn(x.x[e], c.x), __fmul_rn(other, c.y))
                               : __fadd_rn(__fmul_rn(x.x[e], c.x), __fmul_rn(other, c.y));
            }
        }
        if (kind == 0) {
            x.store(p.q_out + (static_cast<int64_t>(t) * p.Hq + head) * D + lane * E);
            return;
        }
    }

    // K or V row: resolve the slot (GetBlockForPosition / GetBlockOffset);
    // with a sliding window the row is a ring of mbps entries
    const int j = p.window > 0 ? (pos / p.bs) % p.mbps : pos / p.bs, slot = pos % p.bs;
    if (j >= p.mbps) {
        if (lane == 0) report(p.status, KVP_ERANGE, t);
        return;
    }
    const int blk = p.bt[static_cast<int64_t>(r) * p.mbps + j];
    if (blk < 0 || blk >= p.num_blocks) {
        if (lane == 0) report(p.status, KVP_ERANGE, t);
        return;
    }
    uint16_t *dst = (kind == 1 ? p.pk : p.pv) +
                    ((static_cast<int64_t>(blk) * p.Hkv + head) * p.bs + slot) * D + lane * E;
    x.template store16<BF16>(dst);
}

template <int D>
static cudaError_t launch_append(const AppendParams &p, bool bf16, cudaStream_t s)
{
    const int64_t rows = static_cast<int64_t>(p.T) * (p.Hq + 2 * p.Hkv);
    const unsigned blocks = static_cast<unsigned>((rows + kAppendWarps - 1) / kAppendWarps);
    return launch_pdl(bf16 ? kv_append_kernel<D, true> : kv_append_kernel<D, false>, dim3(blocks),
                      dim3(kAppendWarps * 32), 0, s, p);
}

}  // namespace kvp

using namespace kvp;

extern "C" int kv_append(kvp_pool *pool, int layer, const kvp_attn_config *attn, int T, const float *q,
                         const float *k, const float *v, const float *q_norm_w, const float *k_norm_w,
                         const float *rope_table, int rope_max_pos, const int32_t *tok_req, const int32_t *positions,
                         int num_seqs, const int32_t *block_tables, int max_blocks_per_seq, float *q_out,
                         void *stream)
{
    int rc = check_pool(pool, layer);
    if (rc) return rc;
    int Hq, Hkv, G;
    if ((rc = resolve_attn(pool, attn, &Hq, &Hkv, &G))) return rc;
    if (T < 0 || num_seqs < 0 || max_blocks_per_seq <= 0)
        return set_error(KVP_EINVAL, "T, num_seqs must be >= 0 and max_blocks_per_seq > 0");
    if (T == 0) return KVP_OK;
    if (!q || !k || !v || !tok_req || !positions || !block_tables || !q_out)
        return set_error(KVP_EINVAL, "kv_append: a required pointer is NULL");
    if (rope_table && rope_max_pos <= 0) return set_error(KVP_EINVAL, "rope_max_pos must be > 0");
    const int D = pool->cfg.head_dim;
    if (attn->window > 0 && static_cast<int64_t>(max_blocks_per_seq) * pool->cfg.block_size < attn->window)
        return set_error(KVP_EINVAL, "a ring of %d blocks of %d cannot hold the window of %d", max_blocks_per_seq,
                         pool->cfg.block_size, attn->window);
    const uintptr_t align = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                            reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(q_out) |
                            reinterpret_cast<uintptr_t>(q_norm_w) | reinterpret_cast<uintptr_t>(k_norm_w) |
                            reinterpret_cast<uintptr_t>(rope_table);
    if (align & 15) return set_error(KVP_EINVAL, "kv_append: float buffers must be 16-byte aligned");
    AppendParams p;
    p.q = q, p.k = k, p.v = v, p.qn = q_norm_w, p.kn = k_norm_w;
    p.rope = reinterpret_cast<const float2 *>(rope_table);
    p.tok_req = tok_req, p.positions = positions, p.bt = block_tables;
    p.pk = pool->k_base + pool->layer_words * layer;
    p.pv = pool->v_base + pool->layer_words * layer;
    p.q_out = q_out, p.status = pool->status;
    p.T = T, p.S = num_seqs, p.Hq = Hq, p.Hkv = Hkv, p.bs = pool->cfg.block_size, p.mbps = max_blocks_per_seq;
    p.num_blocks = pool->cfg.num_blocks, p.max_seq_len = pool->cfg.max_seq_len;
    p.rope_max_pos = rope_table ? rope_max_pos : 0;
    p.R = attn->rope_dim == 0 ? D : attn->rope_dim, p.style = attn->rope_style, p.window = attn->window;
    p.eps = attn->rms_eps;
    const bool bf16 = pool->cfg.kv_dtype == KVP_BF16;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    switch (D) {
    case 64: return check_cuda(launch_append<64>(p, bf16, s), "kv_append launch");
    case 128: return check_cuda(launch_append<128>(p, bf16, s), "kv_append launch");
    case 256: return check_cuda(launch_append<256>(p, bf16, s), "kv_append launch");
    default: return set_error(KVP_EUNSUPPORTED, "head_dim %d", D);
    }
}
