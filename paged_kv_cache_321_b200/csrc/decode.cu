// paged_decode_attention: one query token per sequence, GQA attention over a
// block-pooled KV cache, with split-K over the context.
//
// Method: the batch kernel of runHybridAttentionBlockBatch in
// makarna/pkg/model/arch/hybrid_decoder.go (one query per request, per-request
// block tables and kvLens, scale = float32(1/sqrt(float64(HeadDim)))), whose
// arithmetic is the textbook attention of forward_layer in
// soft3/glia/run/arch/decoder/forward.rs (kv head = h / (Hq/Hkv), max-subtracted
// softmax, sum of p * v), computed as an online softmax over 16-token tiles.
//
// B200 design (HBM-bound: every K/V byte is read once, ~4-8 flop per byte):
//  * grid (split, kv head, sequence); one CTA streams one split of one
//    (sequence, kv head) and serves all G query heads of that kv head from a
//    single read of K and V;
//  * 4 warps per CTA, each with a private 2-stage ring of 16-token tiles. A
//    tile of K (and of V) for one head is one contiguous run of the
//    head-major pool, fetched by ONE 1-D bulk async copy (cp.async.bulk, TMA
//    engine, no multicast) that completes on the stage's mbarrier, so no
//    registers are spent on loads in flight;
//  * each token is handled by LPT lanes; lane j of a token owns DPL dims
//    (16-byte shared-memory chunks j, j+LPT, ..., conflict-free) and keeps
//    q (pre-scaled by scale*log2(e)) and the output accumulators for all G
//    heads in registers; products use packed f32x2 FMAs;
//  * the G partial dot products of a token are summed across its LPT lanes
//    by a transposed butterfly (each step halves the values per lane), which
//    leaves lane j holding the full score of head j >> HSHIFT;
//  * per tile: one max, one rescale of the accumulators (skipped when no
//    head's max moved), exp2 of the scores, P broadcast through shared
//    memory, P.V;
//  * the CTA's 4 warps are merged in shared memory; a CTA whose split is not
//    the only one writes (max, sum, unnormalised output) to the workspace and
//    bumps the (sequence, head) counter; the last split to finish combines
//    all partials by log-sum-exp and resets the counter (no second launch).
#include <math.h>

#include "common.cuh"

namespace kvp {
namespace dec {

constexpr int NW = 4;   // warps per CTA
constexpr int TT = 16;  // tokens per tile (stage)
constexpr int NST = 2;  // stages per warp
constexpr int kMaxSplits = 128;

constexpr int ilog2(int x) { return x <= 1 ? 0 : 1 + ilog2(x / 2); }

template <int D, int G>
struct Shape {
    static constexpr int DPL = (G <= 4 && D >= 128) ? 16 : 8;  // dims per lane
    static constexpr int LPT = D / DPL;                          // lanes per token
    static constexpr int TPW = 32 / LPT;                         // tokens per warp pass
    static constexpr int CH = DPL / 8;                           // 16-byte chunks per lane per row
    static constexpr int ITERS = TT / TPW;                       // passes per tile
    static constexpr int HSHIFT = ilog2(LPT) - ilog2(G);         // lane j -> head j >> HSHIFT
    static constexpr int TILE_WORDS = TT * D;                    // 16-bit words of K (or V) per tile
    static constexpr int STAGE_WORDS = 2 * TILE_WORDS;
    static constexpr int STAGE_BYTES_ALL = NW * NST * STAGE_WORDS * 2;
    static_assert(LPT >= 8 && LPT <= 32, "lanes per token");
    static_assert(HSHIFT >= 0, "group larger than lanes per token");
    static_assert(NW * TPW * G * D * 4 <= STAGE_BYTES_ALL, "combine area");
};

struct Params {
    const uint16_t *kp, *vp;  // this layer's pools
    const float *q;           // [B][Hq][D]
    const int32_t *bt;        // [B][mbps]
    const int32_t *ctx;       // [B]
    float *out;               // [B][Hq][D]
    float *ws_ml;             // [B][Hkv][max_splits][G][2]
    float *ws_o;              // [B][Hkv][max_splits][G][D]
    int *counters;            // [B][Hkv]
    int *status;
    int Hq, Hkv, mbps, bs, num_blocks, max_ctx, max_seq_len, split, max_splits, chunk_blocks;
    float qscale;  // softmax scale * log2(e)
};

__host__ __device__ constexpr size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

template <int D, int G>
struct Smem {
    using S = Shape<D, G>;
    static constexpr size_t stages = 0;
    static constexpr size_t bars = S::STAGE_BYTES_ALL;
    static constexpr size_t masks = bars + NW * NST * 8;
    static constexpr size_t pbuf = align_up(masks + NW * NST * 4, 16);
    static constexpr size_t cm = pbuf + NW * TT * G * 4;  // per-warp (max, sum), aliased later
    static constexpr size_t flag = align_up(cm + 2 * NW * G * 4, 16);
    static constexpr size_t bids = flag + 16;
    static size_t total(int chunk_blocks) { return align_up(bids + 4 * static_cast<size_t>(chunk_blocks), 128); }
};

template <bool BF16>
__device__ __forceinline__ void unpack8(const uint4 w, float2 (&f)[4])
{
    f[0] = unpack2<BF16>(w.x);
    f[1] = unpack2<BF16>(w.y);
    f[2] = unpack2<BF16>(w.z);
    f[3] = unpack2<BF16>(w.w);
}

// Sums v[0..G) over the LPT lanes of a token group; afterwards v[0] of lane j
// holds the total of head j >> HSHIFT.
template <int G, int LPT>
__device__ __forceinline__ void transposed_reduce(float (&v)[G], int j)
{
    int n = G;
#pragma unroll
    for (int off = LPT / 2; off >= 1; off >>= 1) {
        if (n > 1) {
            const bool up = (j & off) != 0;
            const int half = n / 2;
#pragma unroll
            for (int k = 0; k < G / 2; ++k) {
                if (k < half) {
                    const float send = up ? v[k] : v[k + half];
                    const float keep = up ? v[k + half] : v[k];
                    v[k] = keep + __shfl_xor_sync(0xffffffffu, send, off);
                }
            }
            n = half;
        } else {
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], off);
        }
    }
}

template <int D, int G, bool BF16>
__global__ void __launch_bounds__(NW * 32, 3) decode_kernel(const Params p)
{
    using S = Shape<D, G>;
    using M = Smem<D, G>;
    constexpr int DPL = S::DPL, LPT = S::LPT, TPW = S::TPW, CH = S::CH, ITERS = S::ITERS;
    extern __shared__ __align__(128) unsigned char smem[];
    uint16_t *stages = reinterpret_cast<uint16_t *>(smem + M::stages);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + M::bars);
    uint32_t *masks = reinterpret_cast<uint32_t *>(smem + M::masks);
    float *pbuf = reinterpret_cast<float *>(smem + M::pbuf);
    float *cm_m = reinterpret_cast<float *>(smem + M::cm);
    float *cm_l = cm_m + NW * G;
    int *sflag = reinterpret_cast<int *>(smem + M::flag);
    int *bids = reinterpret_cast<int *>(smem + M::bids);

    const int split = blockIdx.x, h = blockIdx.y, r = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ctx = p.ctx[r];
    float *out_rh = p.out + (static_cast<size_t>(r) * p.Hq + static_cast<size_t>(h) * G) * D;

    const bool bad = ctx < 0 || ctx > p.max_ctx || ctx > p.mbps * p.bs || ctx > p.max_seq_len;
    if (bad || ctx == 0) {
        if (split == 0) {
            if (bad && tid == 0) report(p.status, KVP_ERANGE, r);
            for (int i = tid; i < G * D; i += NW * 32) out_rh[i] = 0.0f;
        }
        return;
    }
    const int nsplit = (ctx + p.split - 1) / p.split;
    if (split >= nsplit) return;
    const int tok0 = split * p.split;
    const int tok1 = min(ctx, tok0 + p.split);
    const int ntiles = (tok1 - tok0 + TT - 1) / TT;
    const int blk0 = tok0 / p.bs;
    const int nblk = (tok1 - 1) / p.bs - blk0 + 1;
    const int32_t *bt_row = p.bt + static_cast<size_t>(r) * p.mbps;
    for (int i = tid; i < nblk; i += NW * 32) bids[i] = bt_row[blk0 + i];
    if (tid < NW * NST) mbar_init(smem_addr(&bars[tid]), 1);
    mbar_init_fence();
    __syncthreads();

    // ---- per-lane state
    const int grp = lane / LPT, j = lane % LPT;
    const int hl = j >> S::HSHIFT;  // head whose score this lane ends up holding
    float2 q2[G][DPL / 2];
    {
        const float *qb = p.q + (static_cast<size_t>(r) * p.Hq + static_cast<size_t>(h) * G) * D;
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int c = 0; c < CH; ++c) {
                const float4 *src = reinterpret_cast<const float4 *>(qb + g * D + (j + c * LPT) * 8);
                const float4 a = src[0], b = src[1];
                q2[g][c * 4 + 0] = make_float2(a.x * p.qscale, a.y * p.qscale);
                q2[g][c * 4 + 1] = make_float2(a.z * p.qscale, a.w * p.qscale);
                q2[g][c * 4 + 2] = make_float2(b.x * p.qscale, b.y * p.qscale);
                q2[g][c * 4 + 3] = make_float2(b.z * p.qscale, b.w * p.qscale);
            }
    }
    float2 o2[G][DPL / 2];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int k = 0; k < DPL / 2; ++k) o2[g][k] = make_float2(0.0f, 0.0f);
    float m_run[G];
#pragma unroll
    for (int g = 0; g < G; ++g) m_run[g] = -INFINITY;
    float l_run = 0.0f;

    // ---- this warp's tiles: warp, warp + NW, ...
    const int nt_w = ntiles > warp ? (ntiles - warp + NW - 1) / NW : 0;
    uint16_t *wst = stages + static_cast<size_t>(warp) * NST * S::STAGE_WORDS;
    const uint32_t bar0 = smem_addr(&bars[warp * NST]);
    const size_t head_off = static_cast<size_t>(h) * p.bs * D;
    const size_t blk_stride = static_cast<size_t>(p.Hkv) * p.bs * D;

    // Issues the copies of this warp's i-th tile into stage i % NST (lane 0).
    auto issue = [&](int i) {
        const int st = i % NST;
        const int tb = tok0 + (warp + i * NW) * TT;
        const uint32_t bar = bar0 + st * 8;
        uint16_t *dk = wst + st * S::STAGE_WORDS;
        uint16_t *dv = dk + S::TILE_WORDS;
        uint32_t mask = 0;
        if (p.bs >= TT) {
            const int blk = bids[tb / p.bs - blk0];
            const int nvalid = min(TT, tok1 - tb);
            if (blk >= 0 && blk < p.num_blocks) {
                mask = (1u << nvalid) - 1u;
                const size_t off = blk * blk_stride + head_off + static_cast<size_t>(tb % p.bs) * D;
                mbar_arrive_expect_tx(bar, 2 * S::TILE_WORDS * 2);
                bulk_g2s(smem_addr(dk), p.kp + off, S::TILE_WORDS * 2, bar);
                bulk_g2s(smem_addr(dv), p.vp + off, S::TILE_WORDS * 2, bar);
            } else {
                report(p.status, KVP_ERANGE, r);
                mbar_arrive(bar);
            }
        } else {
            uint32_t bytes = 0;
            for (int t = 0; t < TT && tb + t < tok1; t += p.bs) {
                const int blk = bids[(tb + t) / p.bs - blk0];
                if (blk >= 0 && blk < p.num_blocks) {
                    bytes += 2 * p.bs * D * 2;
                    const int nv = min(p.bs, tok1 - tb - t);
                    mask |= ((1u << nv) - 1u) << t;
                } else {
                    report(p.status, KVP_ERANGE, r);
                }
            }
            if (bytes) {
                mbar_arrive_expect_tx(bar, bytes);
                for (int t = 0; t < TT && tb + t < tok1; t += p.bs) {
                    const int blk = bids[(tb + t) / p.bs - blk0];
                    if (blk >= 0 && blk < p.num_blocks) {
                        const size_t off = blk * blk_stride + head_off;
                        bulk_g2s(smem_addr(dk + t * D), p.kp + off, p.bs * D * 2, bar);
                        bulk_g2s(smem_addr(dv + t * D), p.vp + off, p.bs * D * 2, bar);
                    }
                }
            } else {
                mbar_arrive(bar);
            }
        }
        masks[warp * NST + st] = mask;
    };

    if (lane == 0)
        for (int i = 0; i < NST && i < nt_w; ++i) issue(i);
    __syncwarp();

    float *pw = pbuf + warp * TT * G;
    for (int i = 0; i < nt_w; ++i) {
        const int st = i % NST;
        const bool done = mbar_wait_bounded(bar0 + st * 8, (i / NST) & 1);
        if (!__all_sync(0xffffffffu, done)) {
            if (lane == 0) report(p.status, KVP_ETIMEOUT, r);
            break;
        }
        const uint32_t mask = masks[warp * NST + st];
        const uint16_t *sk = wst + st * S::STAGE_WORDS;
        const uint16_t *sv = sk + S::TILE_WORDS;
        if (mask) {
            // ---- scores: lane holds head hl's score for tokens it*TPW + grp
            float sc[ITERS];
#pragma unroll
            for (int it = 0; it < ITERS; ++it) {
                const int tok = it * TPW + grp;
                const uint16_t *krow = sk + tok * D;
                float2 acc[G];
#pragma unroll
                for (int g = 0; g < G; ++g) acc[g] = make_float2(0.0f, 0.0f);
#pragma unroll
                for (int c = 0; c < CH; ++c) {
                    const uint4 w = *reinterpret_cast<const uint4 *>(krow + (j + c * LPT) * 8);
                    float2 kf[4];
                    unpack8<BF16>(w, kf);
#pragma unroll
                    for (int g = 0; g < G; ++g)
#pragma unroll
                        for (int e = 0; e < 4; ++e) acc[g] = __ffma2_rn(q2[g][c * 4 + e], kf[e], acc[g]);
                }
                float v[G];
#pragma unroll
                for (int g = 0; g < G; ++g) v[g] = acc[g].x + acc[g].y;
                transposed_reduce<G, LPT>(v, j);
                sc[it] = ((mask >> tok) & 1u) ? v[0] : -INFINITY;
            }
            // ---- tile max per head, new running max, rescale factors
            float mt = sc[0];
#pragma unroll
            for (int it = 1; it < ITERS; ++it) mt = fmaxf(mt, sc[it]);
#pragma unroll
            for (int off = LPT; off < 32; off <<= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
            float alpha[G];
            bool moved = false;
            float m_me = 0.0f, a_me = 1.0f;
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float mg = __shfl_sync(0xffffffffu, mt, g << S::HSHIFT);
                const float mn = fmaxf(m_run[g], mg);
                alpha[g] = (mn == m_run[g]) ? 1.0f : exp2f(m_run[g] - mn);
                moved |= (mn != m_run[g]);
                m_run[g] = mn;
                if (g == hl) m_me = mn, a_me = alpha[g];
            }
            float psum = 0.0f;
#pragma unroll
            for (int it = 0; it < ITERS; ++it) {
                const float pv = (sc[it] == -INFINITY) ? 0.0f : exp2f(sc[it] - m_me);
                sc[it] = pv;
                psum += pv;
            }
            l_run = l_run * a_me + psum;
            if (moved) {
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float2 a2 = make_float2(alpha[g], alpha[g]);
#pragma unroll
                    for (int k = 0; k < DPL / 2; ++k) o2[g][k] = __fmul2_rn(o2[g][k], a2);
                }
            }
            if ((j & ((1 << S::HSHIFT) - 1)) == 0) {
#pragma unroll
                for (int it = 0; it < ITERS; ++it) pw[(it * TPW + grp) * G + hl] = sc[it];
            }
            __syncwarp();
            // ---- P.V
#pragma unroll
            for (int it = 0; it < ITERS; ++it) {
                const int tok = it * TPW + grp;
                if (!((mask >> tok) & 1u)) continue;
                float pg[G];
#pragma unroll
                for (int g = 0; g < G; g += 2) {
                    if (g + 1 < G) {
                        const float2 t2 = *reinterpret_cast<const float2 *>(pw + tok * G + g);
                        pg[g] = t2.x, pg[g + 1] = t2.y;
                    } else {
                        pg[g] = pw[tok * G + g];
                    }
                }
                const uint16_t *vrow = sv + tok * D;
#pragma unroll
                for (int c = 0; c < CH; ++c) {
                    const uint4 w = *reinterpret_cast<const uint4 *>(vrow + (j + c * LPT) * 8);
                    float2 vf[4];
                    unpack8<BF16>(w, vf);
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        const float2 pp = make_float2(pg[g], pg[g]);
#pragma unroll
                        for (int e = 0; e < 4; ++e) o2[g][c * 4 + e] = __ffma2_rn(pp, vf[e], o2[g][c * 4 + e]);
                    }
                }
            }
        }
        __syncwarp();
        if (i + NST < nt_w && lane == 0) {
            fence_proxy_async_smem();
            issue(i + NST);
        }
        __syncwarp();
    }

    // ---- merge the token groups' sums, then the warps, in shared memory
#pragma unroll
    for (int off = LPT; off < 32; off <<= 1) l_run += __shfl_xor_sync(0xffffffffu, l_run, off);
    __syncthreads();  // every warp is done with its stages
    float *cm_o = reinterpret_cast<float *>(smem);  // [NW][TPW][G][D], aliases the stages
    if (lane == 0)
#pragma unroll
        for (int g = 0; g < G; ++g) cm_m[warp * G + g] = m_run[g];
    if (grp == 0 && (j & ((1 << S::HSHIFT) - 1)) == 0) cm_l[warp * G + hl] = l_run;
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int c = 0; c < CH; ++c) {
            float *dst = cm_o + ((warp * TPW + grp) * G + g) * D + (j + c * LPT) * 8;
            reinterpret_cast<float4 *>(dst)[0] =
                make_float4(o2[g][c * 4].x, o2[g][c * 4].y, o2[g][c * 4 + 1].x, o2[g][c * 4 + 1].y);
            reinterpret_cast<float4 *>(dst)[1] =
                make_float4(o2[g][c * 4 + 2].x, o2[g][c * 4 + 2].y, o2[g][c * 4 + 3].x, o2[g][c * 4 + 3].y);
        }
    __syncthreads();

    const size_t rh = static_cast<size_t>(r) * p.Hkv + h;
    for (int idx = tid; idx < G * D; idx += NW * 32) {
        const int g = idx / D, d = idx % D;
        float Mx = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; ++w) Mx = fmaxf(Mx, cm_m[w * G + g]);
        float L = 0.0f, O = 0.0f;
        if (Mx != -INFINITY) {
#pragma unroll
            for (int w = 0; w < NW; ++w) {
                const float mw = cm_m[w * G + g];
                if (mw == -INFINITY) continue;
                const float f = exp2f(mw - Mx);
                L += cm_l[w * G + g] * f;
                float ow = 0.0f;
#pragma unroll
                for (int t = 0; t < TPW; ++t) ow += cm_o[((w * TPW + t) * G + g) * D + d];
                O += ow * f;
            }
        }
        if (nsplit == 1) {
            out_rh[idx] = L > 0.0f ? O / L : 0.0f;
        } else {
            p.ws_o[((rh * p.max_splits + split) * G + g) * D + d] = O;
            if (d == 0) {
                p.ws_ml[((rh * p.max_splits + split) * G + g) * 2 + 0] = Mx;
                p.ws_ml[((rh * p.max_splits + split) * G + g) * 2 + 1] = L;
            }
        }
    }
    if (nsplit == 1) return;

    // ---- split-K: the last split of (r, h) to finish combines all partials
    __threadfence();
    __syncthreads();
    if (tid == 0) *sflag = atomicAdd(&p.counters[rh], 1) == nsplit - 1;
    __syncthreads();
    if (!*sflag) return;
    __threadfence();
    float *wts = reinterpret_cast<float *>(smem);  // [nsplit][G] weights, then [G] total
    float *tot = wts + kMaxSplits * G;
    const float *ml = p.ws_ml + rh * p.max_splits * G * 2;
    if (tid < G) {
        float Mx = -INFINITY;
        for (int s2 = 0; s2 < nsplit; ++s2) Mx = fmaxf(Mx, __ldcg(ml + (s2 * G + tid) * 2));
        float L = 0.0f;
        for (int s2 = 0; s2 < nsplit; ++s2) {
            const float ms = __ldcg(ml + (s2 * G + tid) * 2);
            const float f = (ms == -INFINITY) ? 0.0f : exp2f(ms - Mx);
            wts[s2 * G + tid] = f;
            L += __ldcg(ml + (s2 * G + tid) * 2 + 1) * f;
        }
        tot[tid] = L > 0.0f ? 1.0f / L : 0.0f;
    }
    __syncthreads();
    const float *po = p.ws_o + rh * p.max_splits * G * D;
    for (int idx = tid; idx < G * D; idx += NW * 32) {
        const int g = idx / D;
        float O = 0.0f;
        for (int s2 = 0; s2 < nsplit; ++s2) O += __ldcg(po + static_cast<size_t>(s2) * G * D + idx) * wts[s2 * G + g];
        out_rh[idx] = O * tot[g];
    }
    if (tid == 0) p.counters[rh] = 0;
}

template <int D, int G>
static int launch(const Params &p, bool bf16, int B, cudaStream_t s)
{
    const size_t smem = Smem<D, G>::total(p.chunk_blocks);
    if (smem > 227 * 1024) return set_error(KVP_EUNSUPPORTED, "decode: %zu bytes of shared memory", smem);
    auto kern = bf16 ? decode_kernel<D, G, true> : decode_kernel<D, G, false>;
    int rc = check_cuda(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)),
                        "decode smem attribute");
    if (rc) return rc;
    dim3 grid(p.max_splits, p.Hkv, B);
    kern<<<grid, NW * 32, smem, s>>>(p);
    return check_cuda(cudaGetLastError(), "decode launch");
}

template <int D>
static int launch_g(const Params &p, bool bf16, int B, int G, cudaStream_t s)
{
    switch (G) {
    case 1: return launch<D, 1>(p, bf16, B, s);
    case 2: return launch<D, 2>(p, bf16, B, s);
    case 4: return launch<D, 4>(p, bf16, B, s);
    case 8: return launch<D, 8>(p, bf16, B, s);
    default: return set_error(KVP_EUNSUPPORTED, "decode: GQA group %d not built (1, 2, 4, 8)", G);
    }
}

// Split size: multiples of max(16, block_size); ~256 keys, smaller when the
// batch is too small to fill 4 CTAs per SM, larger when a context would need
// more than kMaxSplits splits.
static int choose_split(int bs, int B, int Hkv, int max_ctx, int requested)
{
    const int unit = bs > TT ? bs : TT;
    if (requested > 0) return requested;
    if (max_ctx <= 0) return unit;
    auto up = [&](long long x) { return static_cast<int>((x + unit - 1) / unit * unit); };
    int split = up(256);
    const long long units = static_cast<long long>(B) * Hkv;
    const long long target = 4LL * 148;
    if (units * ((max_ctx + split - 1) / split) < target) {
        split = up((static_cast<long long>(max_ctx) * units + target - 1) / target);
        if (split < unit) split = unit;
    }
    if ((max_ctx + split - 1) / split > kMaxSplits) split = up((max_ctx + kMaxSplits - 1) / kMaxSplits);
    return split;
}

struct Layout {
    int split, max_splits;
    size_t counters, ml, o, total;
};

static int plan(const kvp_pool *pool, int G, int Hkv, int B, int max_ctx, int split_req, Layout *L)
{
    const int bs = pool->cfg.block_size;
    const int unit = bs > TT ? bs : TT;
    if (split_req < 0 || (split_req > 0 && split_req % unit))
        return set_error(KVP_EINVAL, "split_tokens %d must be 0 or a multiple of %d", split_req, unit);
    if (B < 0 || max_ctx < 0) return set_error(KVP_EINVAL, "B and max_ctx_len must be >= 0");
    L->split = choose_split(bs, B, Hkv, max_ctx, split_req);
    L->max_splits = max_ctx > 0 ? (max_ctx + L->split - 1) / L->split : 1;
    if (L->max_splits > kMaxSplits)
        return set_error(KVP_EINVAL, "split_tokens %d gives %d splits (max %d)", L->split, L->max_splits, kMaxSplits);
    const size_t rh = static_cast<size_t>(B) * Hkv;
    L->counters = 0;
    L->ml = align_up(rh * 4, 256);
    L->o = align_up(L->ml + rh * L->max_splits * G * 2 * 4, 256);
    L->total = align_up(L->o + rh * L->max_splits * G * pool->cfg.head_dim * 4, 256);
    return KVP_OK;
}

}  // namespace dec
}  // namespace kvp

using namespace kvp;

extern "C" size_t paged_decode_workspace_size(const kvp_pool *pool, const kvp_attn_config *attn, int B,
                                              int max_ctx_len, int split_tokens)
{
    if (!pool) return 0;
    int Hq, Hkv, G;
    if (resolve_attn(pool, attn, &Hq, &Hkv, &G)) return 0;
    dec::Layout L;
    if (dec::plan(pool, G, Hkv, B, max_ctx_len, split_tokens, &L)) return 0;
    return L.total;
}

extern "C" int paged_decode_attention(kvp_pool *pool, int layer, const kvp_attn_config *attn, int B,
                                      const float *q, const int32_t *block_tables, int max_blocks_per_seq,
                                      const int32_t *ctx_lens, int max_ctx_len, int split_tokens, float *out,
                                      void *workspace, size_t ws_bytes, void *stream)
{
    int rc = check_pool(pool, layer);
    if (rc) return rc;
    int Hq, Hkv, G;
    if ((rc = resolve_attn(pool, attn, &Hq, &Hkv, &G))) return rc;
    if (B == 0) return KVP_OK;
    if (B < 0 || B > 65535) return set_error(KVP_EINVAL, "B %d outside [0, 65535]", B);
    if (max_blocks_per_seq <= 0) return set_error(KVP_EINVAL, "max_blocks_per_seq must be > 0");
    if (!q || !block_tables || !ctx_lens || !out || !workspace)
        return set_error(KVP_EINVAL, "paged_decode_attention: a required pointer is NULL");
    if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(out)) & 15)
        return set_error(KVP_EINVAL, "q and out must be 16-byte aligned");
    if (reinterpret_cast<uintptr_t>(workspace) & 255) return set_error(KVP_EINVAL, "workspace must be 256-byte aligned");
    dec::Layout L;
    if ((rc = dec::plan(pool, G, Hkv, B, max_ctx_len, split_tokens, &L))) return rc;
    if (ws_bytes < L.total)
        return set_error(KVP_EINVAL, "workspace of %zu bytes, %zu needed", ws_bytes, L.total);
    dec::Params p;
    p.kp = pool->k_base + pool->layer_words * layer;
    p.vp = pool->v_base + pool->layer_words * layer;
    p.q = q, p.bt = block_tables, p.ctx = ctx_lens, p.out = out;
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    p.counters = reinterpret_cast<int *>(ws + L.counters);
    p.ws_ml = reinterpret_cast<float *>(ws + L.ml);
    p.ws_o = reinterpret_cast<float *>(ws + L.o);
    p.status = pool->status;
    p.Hq = Hq, p.Hkv = Hkv, p.mbps = max_blocks_per_seq, p.bs = pool->cfg.block_size;
    p.num_blocks = pool->cfg.num_blocks, p.max_ctx = max_ctx_len, p.max_seq_len = pool->cfg.max_seq_len;
    p.split = L.split, p.max_splits = L.max_splits;
    p.chunk_blocks = L.split / p.bs + 1;
    const double scale = static_cast<double>(static_cast<float>(1.0 / sqrt(static_cast<double>(pool->cfg.head_dim))));
    p.qscale = static_cast<float>(scale * 1.4426950408889634);  // log2(e): softmax via exp2
    const bool bf16 = pool->cfg.kv_dtype == KVP_BF16;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    switch (pool->cfg.head_dim) {
    case 64: return dec::launch_g<64>(p, bf16, B, G, s);
    case 128: return dec::launch_g<128>(p, bf16, B, G, s);
    case 256: return dec::launch_g<256>(p, bf16, B, G, s);
    default: return set_error(KVP_EUNSUPPORTED, "head_dim %d", pool->cfg.head_dim);
    }
}
