// paged_decode_attention: one query token per sequence, GQA attention over a
// block-pooled KV cache, split over the context with a log-sum-exp combine.
// Two kernels share the work distribution below: decode_kernel computes on
// CUDA cores (any group size and block size), decode_tc_kernel on tensor
// cores (groups of 4 and 8 with blocks of at least 16 tokens; see its own
// description further down).
//
// Method: the batch kernel of runHybridAttentionBlockBatch in
// makarna/pkg/model/arch/hybrid_decoder.go (one query per request, per-request
// block tables and kvLens, scale = float32(1/sqrt(float64(HeadDim)))), whose
// arithmetic is the textbook attention of forward_layer in
// soft3/glia/run/arch/decoder/forward.rs (kv head = h / (Hq/Hkv), max-subtracted
// softmax, sum of p * v), computed as an online softmax over 16-token tiles.
//
// B200 design. The step is HBM-bound (every K/V byte is read once, ~4-8 flop
// per byte on CUDA cores), so the kernel is built to keep bytes in flight and
// the issue slots busy:
//  * persistent: one CTA per SM, NW independent warps. The tiles of all
//    (sequence, kv head) contexts, taken in order, form one global sequence
//    that is cut into equal contiguous ranges, one per warp (stream-K), so the
//    load is balanced to one tile whatever the context lengths;
//  * each warp streams its range through a private ring of NST stages; a
//    stage holds one 16-token tile of K and of V for one head, each fetched by
//    ONE 1-D bulk async copy (cp.async.bulk on the TMA engine, no multicast)
//    completing on the stage's mbarrier. The ring runs on across context
//    boundaries, so the next context's tiles are in flight while the current
//    one is finished;
//  * LPT lanes per token, each owning DPL dims (16-byte chunks j, j+LPT, ...:
//    conflict-free shared-memory reads); q (pre-scaled by scale*log2 e) and
//    the output accumulators for all G heads of the kv head stay in
//    registers; products are packed f32x2 FMAs;
//  * the partial dot products of a pass (ITERS tokens x G heads) are summed
//    over the LPT lanes by one batched transposed butterfly that halves the
//    values at every step, leaving each lane with distinct (token, head)
//    scores; one exp2 per score, P goes to the PV pass through shared memory;
//  * a context split over several warps leaves (max, sum, unnormalised
//    output) partials in the workspace and counts them in after a release
//    fence (the count's reply is looked at only at the end of the range, so
//    the stream does not wait for it); the warp that brings a count to the
//    number of segments merges them by log-sum-exp and resets the counter,
//    so no second launch (and no grid-wide drain before the merge) is
//    needed. With 8 query heads per kv head (no registers to spare) a second
//    grid, one warp per (context, head), does the merge instead. A context
//    inside one warp's range is normalised and written by that warp;
//  * the first tile of each segment also brings the segment's queries into
//    L1 (prefetch), and the K/V copies carry an L2 evict-first policy.
#include <math.h>

#include <type_traits>

#include "common.cuh"

namespace kvp {
namespace dec {

constexpr int TT = 16;             // tokens per tile (stage)
constexpr int NST = 2;             // stages per warp
constexpr int kMaxBatch = 2048;    // sequences per call (per-CTA prefix in shared memory)
constexpr int kAutoMinTiles = 2;   // default minimum tiles per warp
constexpr int kStageBudget = 200 * 1024;
constexpr float kLazy = 8.0f;   // log2 headroom before the reference max must move

constexpr int ilog2(int x) { return x <= 1 ? 0 : 1 + ilog2(x / 2); }
constexpr int cmin(int a, int b) { return a < b ? a : b; }
constexpr int cmax(int a, int b) { return a > b ? a : b; }

template <int D, int G>
struct Shape {
    static constexpr int DPL = 8;                                // dims per lane (one 16-byte chunk)
    static constexpr int LPT = D / DPL;                          // lanes per token
    static constexpr int TPW = 32 / LPT;                         // tokens per warp pass
    static constexpr int ITERS = TT / TPW;                       // passes per tile
    static constexpr int RB = cmin(ITERS, cmax(1, 32 / G));      // passes reduced together
    static constexpr int NB = ITERS / RB;                        // reduction batches per tile
    static constexpr int NV = RB * G;                            // partial sums per lane per batch
    static constexpr int LEVELS = ilog2(LPT);                    // butterfly steps over a token's lanes
    static constexpr int HALV = cmin(LEVELS, ilog2(RB));         // steps that halve the passes kept
    static constexpr int PPL = RB >> HALV;                       // passes a lane keeps per batch
    static constexpr int REP = 1 << (LEVELS - HALV);             // lanes holding copies of a score
    static constexpr int TILE_WORDS = TT * D;                    // 16-bit words of K (or V) per tile
    static constexpr int STAGE_BYTES = 2 * TILE_WORDS * 2;
    static constexpr int NO = G * DPL / 2;                       // float2 output accumulators per lane
    static constexpr int OLEV = ilog2(TPW);
    static constexpr int OVPL = NO >> OLEV;                      // float2 outputs a lane owns
    // warps per CTA (one CTA per SM): within the register budget and the
    // shared-memory budget of the stage rings
    static constexpr int NW = cmin(G >= 8 ? 8 : 12, kStageBudget / (NST * STAGE_BYTES));
    static_assert(LPT >= 8 && LPT <= 32, "lanes per token");
    static_assert(ITERS % RB == 0, "reduction batches");
    static_assert(ilog2(NO) >= OLEV, "token-group reduction must halve at every step");
};

struct Params {
    const uint16_t *kp, *vp;  // this layer's pools
    const float *q;           // [B][Hq][D]
    const int32_t *bt;        // [B][mbps]
    const int32_t *ctx;       // [B]
    float *out;               // [B][Hq][D]
    float *part;              // [W + B*Hkv] slots of slot_floats(G, D): outputs, then (max, sum) per head
    int *counters;            // [B*Hkv] segments finished per split context
    int *status;
    int B, Hq, Hkv, mbps, bs, num_blocks, max_ctx, max_seq_len, warps_total, min_tiles;
    int window;    // sliding window in keys (0: none); > 0 makes block-table rows rings
    float qscale;  // softmax scale * log2(e)
};

__host__ __device__ constexpr size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

template <int D, int G>
struct Smem {
    using S = Shape<D, G>;
    static constexpr size_t stages = 0;
    static constexpr size_t bars = static_cast<size_t>(S::NW) * NST * S::STAGE_BYTES;
    static constexpr size_t masks = bars + S::NW * NST * 2 * 8;
    static constexpr size_t pbuf = align_up(masks + S::NW * NST * 4, 16);
    static constexpr size_t tiles = pbuf + S::NW * TT * G * 8;  // [B] context lengths
    __host__ __device__ static size_t pref(int B) { return align_up(tiles + 4 * static_cast<size_t>(B), 16); }  // [B + 1]
    __host__ __device__ static size_t cpref(int B) { return align_up(pref(B) + 4 * static_cast<size_t>(B + 1), 16); }  // [B + 1]
    __host__ __device__ static size_t total(int B) { return align_up(cpref(B) + 4 * static_cast<size_t>(B + 1), 128); }
};

__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float shfl_xor(float x, int off) { return __shfl_xor_sync(0xffffffffu, x, off); }
__device__ __forceinline__ float2 shfl_xor(float2 x, int off)
{
    return make_float2(__shfl_xor_sync(0xffffffffu, x.x, off), __shfl_xor_sync(0xffffffffu, x.y, off));
}

template <bool BF16>
__device__ __forceinline__ void unpack8(const uint4 w, float2 (&f)[4])
{
    f[0] = unpack2<BF16>(w.x);
    f[1] = unpack2<BF16>(w.y);
    f[2] = unpack2<BF16>(w.z);
    f[3] = unpack2<BF16>(w.w);
}

// First value index a lane keeps after HALV halving steps over the lane bits
// lo_off, 2*lo_off, ... starting from N values.
template <int N, int HALV>
__device__ __forceinline__ int halving_base(int lane, int lo_off)
{
    int base = 0, n = N, off = lo_off;
#pragma unroll
    for (int s = 0; s < HALV; ++s) {
        n >>= 1;
        if (lane & off) base += n;
        off <<= 1;
    }
    return base;
}

// Reduces v[0..N) with `op` over the lanes that differ in bits lo_off,
// 2*lo_off, ... below lim_off. The first HALV steps halve the values a lane
// keeps (the half chosen by its lane bit, the other half is sent to the
// partner); later steps combine the single remaining value. Afterwards
// v[0 .. N >> HALV) hold the complete results for value indices
// halving_base<N, HALV>(lane, lo_off) + 0, 1, ...
template <int N, int HALV, typename T, typename Op>
__device__ __forceinline__ void transposed_reduce(T (&v)[N], int lane, int lo_off, int lim_off, Op op)
{
    int n = N;
    int off = lo_off;
#pragma unroll
    for (int step = 0; step < 5; ++step) {
        if (off >= lim_off) break;
        if (step < HALV) {
            const bool up = (lane & off) != 0;
            const int half = n / 2;
#pragma unroll
            for (int k = 0; k < N / 2; ++k) {
                if (k < half) {
                    const T send = up ? v[k] : v[k + half];
                    const T keep = up ? v[k + half] : v[k];
                    v[k] = op(keep, shfl_xor(send, off));
                }
            }
            n = half;
        } else {
            v[0] = op(v[0], shfl_xor(v[0], off));
        }
        off <<= 1;
    }
}

// Position of a warp's cursor in the global tile sequence.
struct Cursor {
    int t;   // global tile index
    int r;   // sequence
    int h;   // kv head
    int ti;  // tile index inside the (r, h) context
    int nt;  // tiles of sequence r
};

// A context length the kernels accept (else the row is zero and an error is
// reported by the decode kernel).
__device__ __forceinline__ bool ctx_ok(const Params &p, int c)
{
    return c >= 0 && c <= p.max_ctx && c <= p.max_seq_len && (p.window > 0 || c <= p.mbps * p.bs);
}

// Cost of starting a context on a warp, in tiles: a warp whose range crosses
// a context boundary pays for a second segment end (reductions, partial
// write, fence) and a cold first tile, about one tile's time. The warps'
// ranges are cut evenly in cost space, where every context is preceded by
// kCtxCost empty units, so such a warp gets about one tile less.
constexpr int kCtxCost = 1;

// The kernels keep each sequence's context length in shared memory (-1 for
// one the kernel refuses), and derive its tiles from it: the keys of a
// context are 0 .. ctx-1, or with a sliding window ctx-window .. ctx-1,
// covered by the 16-key tiles first_tile .. (ctx-1)/16 of the position axis.
__device__ __forceinline__ int first_tile(int ctx, int window)
{
    return window > 0 && ctx > window ? (ctx - window) / TT : 0;
}
__device__ __forceinline__ int tiles_of(int ctx, int window)
{
    return ctx > 0 ? (ctx + TT - 1) / TT - first_tile(ctx, window) : 0;
}
// Block-table entry of position `pos` (a ring of mbps entries with a window).
__device__ __forceinline__ int entry_of(const Params &p, int window, int pos)
{
    return window > 0 ? (pos / p.bs) % p.mbps : pos / p.bs;
}
// Valid rows of the 16-key tile starting at position tb: below the context
// end and (with a window) at or after its first key.
__device__ __forceinline__ uint32_t tile_rows(int ctx, int window, int tb)
{
    const int nv = min(TT, ctx - tb);
    const int f = window > 0 ? max(0, ctx - window - tb) : 0;
    return ((1u << nv) - 1u) & ~((1u << f) - 1u);
}

// Exclusive prefixes over the B sequences, by one warp: s_pref[i] of the
// tiles (tiles_of(s_ctx) * Hkv), s_cpref[i] of the cost units (Hkv * (tiles +
// kCtxCost) for a sequence with tiles). s_pref[B] is the number of tiles,
// s_cpref[B] the length of the cost space.
__device__ __forceinline__ void tile_prefix(const int *s_ctx, int *s_pref, int *s_cpref, int B, int Hkv, int lane,
                                            int window)
{
    int run = 0, crun = 0;
    for (int base = 0; base < B; base += 32) {
        const int i = base + lane;
        const int nt = i < B ? tiles_of(s_ctx[i], window) : 0;
        const int v = nt * Hkv, cv = nt > 0 ? (nt + kCtxCost) * Hkv : 0;
        int x = v, cx = cv;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, off);
            const int cy = __shfl_up_sync(0xffffffffu, cx, off);
            if (lane >= off) x += y, cx += cy;
        }
        if (i < B) s_pref[i] = run + x - v, s_cpref[i] = crun + cx - cv;
        run += __shfl_sync(0xffffffffu, x, 31);
        crun += __shfl_sync(0xffffffffu, cx, 31);
    }
    if (lane == 0) s_pref[B] = run, s_cpref[B] = crun;
}

// Number of warps the global tile sequence of `total` tiles is cut over.
__device__ __forceinline__ int active_warps(const Params &p, int total)
{
    return max(1, min(p.warps_total, (total + p.min_tiles - 1) / p.min_tiles));
}

// Warp w owns the cost units [floor(w*TC/W), floor((w+1)*TC/W)). The first
// tile whose cost position is at least U (the tiles of context (r, h) sit at
// cost positions s_cpref[r] + h*(nt + kCtxCost) + kCtxCost + i).
__device__ __forceinline__ int cost_to_tile(int64_t U, const int *s_ctx, const int *s_pref, const int *s_cpref,
                                            int B, int window)
{
    if (U >= s_cpref[B]) return s_pref[B];
    int lo = 0, hi = B;  // s_cpref[lo] <= U < s_cpref[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s_cpref[mid] <= U) lo = mid;
        else hi = mid;
    }
    const int nt = tiles_of(s_ctx[lo], window), span = nt + kCtxCost;
    const int local = static_cast<int>(U - s_cpref[lo]);
    const int h = local / span, off = local - h * span;
    return s_pref[lo] + h * nt + max(0, off - kCtxCost);
}

// First and last warp whose cost range holds a tile of the context whose
// first tile sits at cost position P (nt tiles); TC is the cost-space length.
__device__ __forceinline__ void context_warps(int P, int nt, int W, int TC, int &w_first, int &w_last)
{
    w_first = static_cast<int>(((static_cast<int64_t>(P) + 1) * W - 1) / TC);
    w_last = static_cast<int>(((static_cast<int64_t>(P) + nt) * W - 1) / TC);
}

// Floats in one partial-result slot: G output rows of D, then G (max, sum)
// pairs padded to 16 bytes, so every slot and row starts 16-byte aligned.
__host__ __device__ constexpr int slot_floats(int G, int D) { return G * D + ((2 * G + 3) & ~3); }

// Partial-result slot of the segment of context rh computed by warp w: the
// slots of one context's segments are consecutive (w_first + rh ...), and a
// warp's two split segments (its first and its last) never collide with
// another warp's, because contexts advance with the warp index.
template <int D, int G>
__device__ __forceinline__ float *part_slot(const Params &p, int w, int rh)
{
    return p.part + static_cast<size_t>(w + rh) * slot_floats(G, D);
}

// Log-sum-exp merge of the partials of context rh (query heads h*G ..
// h*G+G-1), written by warps w_first .. w_last into consecutive slots; run by
// one warp, the one that finished the context last, so its latency is the
// tail of the kernel. One load round trip brings every segment's (max, sum)
// pairs (lane = segment); the weights come from warp reductions; then the
// (segment, head) output rows stream in chunks of CI rows per lane, each
// chunk's loads all issued (predicated, no remainder loop) before the first
// is used. Loads bypass L1: the partials were written on other SMs. Kept
// out of line with a small chunk: its registers must not cost the streaming
// loop any (a larger chunk made that loop spill).
template <int D, int G>
__device__ __noinline__ void combine(const Params &p, int rh, int w_first, int w_last, int lane, float *out_rh)
{
    constexpr int SL = slot_floats(G, D);
    constexpr int DL = D / 32;                    // output dims per lane: 2, 4 or 8
    constexpr int CI = cmax(G, 32 / DL);          // (segment, head) rows per chunk: 32 floats per lane
    constexpr int CS = CI / G;                    // segments per chunk
    using V = typename std::conditional<DL == 2, float2, float4>::type;
    constexpr int NV = DL * 4 / static_cast<int>(sizeof(V));  // vectors per row and lane
    const int nseg = w_last - w_first + 1;
    const float *base = part_slot<D, G>(p, w_first, rh);
    if (nseg <= 32) {
        float m[G], l[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            m[g] = -INFINITY;
            l[g] = 0.0f;
        }
        if (lane < nseg) {
            const float2 *ml = reinterpret_cast<const float2 *>(base + static_cast<size_t>(lane) * SL + G * D);
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float2 v = __ldcg(ml + g);
                m[g] = v.x;
                l[g] = v.y;
            }
        }
        float w[G], L[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            float M = m[g];
#pragma unroll
            for (int off = 16; off; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
            w[g] = (m[g] == -INFINITY) ? 0.0f : ex2(m[g] - M);
            L[g] = l[g] * w[g];
#pragma unroll
            for (int off = 16; off; off >>= 1) L[g] += __shfl_xor_sync(0xffffffffu, L[g], off);
        }
        float acc[G][DL];
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int d = 0; d < DL; ++d) acc[g][d] = 0.0f;
        const float *row0 = base + lane * DL;
#pragma unroll 1
        for (int s0 = 0; s0 < nseg; s0 += CS) {
            V buf[CS][G][NV];
#pragma unroll
            for (int k = 0; k < CS; ++k) {
                const bool live = s0 + k < nseg;
                const float *srow = row0 + static_cast<size_t>(s0 + k) * SL;
#pragma unroll
                for (int g = 0; g < G; ++g)
#pragma unroll
                    for (int v = 0; v < NV; ++v) {
                        if (live) buf[k][g][v] = __ldcg(reinterpret_cast<const V *>(srow + g * D) + v);
                        else buf[k][g][v] = V{};
                    }
            }
#pragma unroll
            for (int k = 0; k < CS; ++k) {
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float ws = __shfl_sync(0xffffffffu, w[g], min(s0 + k, 31));  // 0 past nseg
                    const float *f = reinterpret_cast<const float *>(buf[k][g]);
#pragma unroll
                    for (int d = 0; d < DL; ++d) acc[g][d] = fmaf(f[d], ws, acc[g][d]);
                }
            }
        }
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float inv = L[g] > 0.0f ? 1.0f / L[g] : 0.0f;
#pragma unroll
            for (int d = 0; d < DL; d += 2)
                *reinterpret_cast<float2 *>(out_rh + g * D + lane * DL + d) =
                    make_float2(acc[g][d] * inv, acc[g][d + 1] * inv);
        }
        return;
    }
    // more than 32 segments: per head, max, sum, then the outputs
#pragma unroll 1
    for (int g = 0; g < G; ++g) {
        float M = -INFINITY;
        for (int s = lane; s < nseg; s += 32) M = fmaxf(M, __ldcg(base + static_cast<size_t>(s) * SL + G * D + 2 * g));
#pragma unroll
        for (int off = 16; off; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
        float L = 0.0f;
        for (int s = lane; s < nseg; s += 32) {
            const float2 v = __ldcg(reinterpret_cast<const float2 *>(base + static_cast<size_t>(s) * SL + G * D) + g);
            L += (v.x == -INFINITY) ? 0.0f : v.y * ex2(v.x - M);
        }
#pragma unroll
        for (int off = 16; off; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
        const float inv = L > 0.0f ? 1.0f / L : 0.0f;
        float acc[DL];
#pragma unroll
        for (int d = 0; d < DL; ++d) acc[d] = 0.0f;
#pragma unroll 8
        for (int s = 0; s < nseg; ++s) {
            const float *sl = base + static_cast<size_t>(s) * SL;
            const float m = __ldcg(sl + G * D + 2 * g);
            const float wgt = (m == -INFINITY) ? 0.0f : ex2(m - M);
            const float *src = sl + g * D + lane * DL;
#pragma unroll
            for (int d = 0; d < DL; d += 2) {
                const float2 v = __ldcg(reinterpret_cast<const float2 *>(src + d));
                acc[d] += v.x * wgt;
                acc[d + 1] += v.y * wgt;
            }
        }
#pragma unroll
        for (int d = 0; d < DL; d += 2)
            *reinterpret_cast<float2 *>(out_rh + g * D + lane * DL + d) = make_float2(acc[d] * inv, acc[d + 1] * inv);
    }
}

// With 8 query heads per kv head the streaming loop already needs every
// register a thread can have; any merge code inside it costs spills there.
// Those contexts are merged by a separate grid instead (combine_kernel),
// one warp per (context, head), so a context's merge is also spread over
// G warps rather than run by one.
template <int G>
struct GridCombine {
    static constexpr bool value = G >= 8;
};

// GPU-scope fence with acquire-release semantics. Before a count: this
// warp's partials (ordered before it by __syncwarp) are visible before the
// count moves. After the final count: every earlier contributor's partial is
// visible to the warp that merges.
__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }

__device__ __forceinline__ int atomic_add_relaxed(int *addr, int v)
{
    int old;
    asm volatile("atom.relaxed.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(addr), "r"(v) : "memory");
    return old;
}

template <int D, int G, bool BF16, bool WIN>
__global__ void __launch_bounds__(Shape<D, G>::NW * 32, 1) decode_kernel(const Params p)
{
    const int win = WIN ? p.window : 0;  // a compile-time 0 in the instance without a window
    using S = Shape<D, G>;
    using M = Smem<D, G>;
    constexpr int NW = S::NW;
    constexpr int LPT = S::LPT, TPW = S::TPW, ITERS = S::ITERS;
    constexpr int RB = S::RB, NB = S::NB, NV = S::NV, HALV = S::HALV, PPL = S::PPL;
    extern __shared__ __align__(128) unsigned char smem[];
    uint16_t *stages = reinterpret_cast<uint16_t *>(smem + M::stages);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + M::bars);
    uint32_t *masks = reinterpret_cast<uint32_t *>(smem + M::masks);
    float2 *pbuf = reinterpret_cast<float2 *>(smem + M::pbuf);
    int *s_ctx = reinterpret_cast<int *>(smem + M::tiles);  // context lengths
    int *s_pref = reinterpret_cast<int *>(smem + M::pref(p.B));
    int *s_cpref = reinterpret_cast<int *>(smem + M::cpref(p.B));

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int B = p.B, Hkv = p.Hkv;

    // Nothing global is touched before the previous grid on the stream has
    // completed: with a programmatic launch only the launch itself overlaps.
    grid_dependency_wait();

    // ---- start the block table on its way to L2 (this CTA's share of it)
    // while the context lengths are read; the copy descriptors read it next
    {
        const int64_t lines = (static_cast<int64_t>(B) * p.mbps * 4 + 127) / 128;
        const int64_t lo = lines * blockIdx.x / gridDim.x, hi = lines * (blockIdx.x + 1) / gridDim.x;
        const char *bt_bytes = reinterpret_cast<const char *>(p.bt);
        for (int64_t l = lo + tid; l < hi && l < lo + 4 * NW * 32; l += NW * 32) prefetch_l2(bt_bytes + l * 128);
    }

    // ---- tiles per sequence; invalid or empty sequences get none and a zero row
    for (int i = tid; i < B; i += NW * 32) {
        const int c = p.ctx[i];
        const bool ok = ctx_ok(p, c);
        s_ctx[i] = ok ? c : -1;
        if (blockIdx.x == 0 && (!ok || c == 0)) {
            if (!ok) report(p.status, KVP_ERANGE, i);
            float4 *o = reinterpret_cast<float4 *>(p.out + static_cast<size_t>(i) * p.Hq * D);
            for (int k = 0; k < p.Hq * D / 4; ++k) o[k] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    __syncthreads();
    if (warp == 0) tile_prefix(s_ctx, s_pref, s_cpref, B, Hkv, lane, win);
    __syncthreads();

    grid_launch_dependents();  // the next grid may be placed (it waits for this one)

    // ---- this warp's share of the global tile sequence (cut in cost space)
    const int total = s_pref[B], TC = s_cpref[B];
    const int W = active_warps(p, total);
    const int w = blockIdx.x * NW + warp;
    if (w >= W) return;
    const int t_begin = cost_to_tile(static_cast<int64_t>(w) * TC / W, s_ctx, s_pref, s_cpref, B, win);
    const int t_end = cost_to_tile(static_cast<int64_t>(w + 1) * TC / W, s_ctx, s_pref, s_cpref, B, win);
    if (t_begin >= t_end) return;  // no CTA-wide barrier follows

    // barriers: [warp][stage][K, V] "tile half landed"
    const uint32_t kbar0 = smem_addr(&bars[warp * NST * 2]);
    if (lane < 2 * NST) mbar_init(kbar0 + lane * 8, 1);
    mbar_init_fence();
    __syncwarp();

    auto locate = [&](int t, Cursor &c) {
        int lo = 0, hi = B;  // s_pref[lo] <= t < s_pref[hi]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (s_pref[mid] <= t) lo = mid;
            else hi = mid;
        }
        c.t = t;
        c.r = lo;
        c.nt = tiles_of(s_ctx[lo], win);
        const int local = t - s_pref[lo];
        c.h = local / c.nt;
        c.ti = local - c.h * c.nt;
    };
    auto advance = [&](Cursor &c) {
        ++c.t;
        if (++c.ti == c.nt) {
            c.ti = 0;
            if (++c.h == Hkv) {
                c.h = 0;
                do {
                    ++c.r;
                } while (c.r < B && tiles_of(s_ctx[c.r], win) == 0);
                if (c.r < B) c.nt = tiles_of(s_ctx[c.r], win);
            }
        }
    };

    uint16_t *wst = stages + static_cast<size_t>(warp) * NST * (S::STAGE_BYTES / 2);
    int *nvalid = reinterpret_cast<int *>(masks) + warp * NST;
    float2 *pw = pbuf + warp * TT * G;  // (p, p) pairs per (token, head)
    const size_t blk_stride = static_cast<size_t>(Hkv) * p.bs * D;
    const bool big_blocks = p.bs >= TT;  // a tile lies inside one block
    const int ntile = t_end - t_begin;
    const uint64_t l2pol = l2_evict_first_policy();

    // Copy descriptors of 32 consecutive tiles, one per lane: the element
    // offset of the tile's K (and V) run in the layer pool and its mask of
    // valid rows (0: block id outside the pool).
    int64_t d_off = 0;
    int d_nv = 0, dbase = 0, d_q = -1;
    auto load_desc = [&](int base) {
        dbase = base;
        d_off = 0;
        d_nv = 0;
        d_q = -1;
        const int i = base + lane;
        if (big_blocks && i < ntile) {
            Cursor c;
            locate(t_begin + i, c);
            // a segment starts here: its queries are wanted when this tile is
            if (c.ti == 0 || i == 0) d_q = c.r * p.Hq + c.h * G;
            const int ctx = s_ctx[c.r];
            const int tb = (first_tile(ctx, win) + c.ti) * TT;  // position of the tile's first key
            const int blk = p.bt[static_cast<size_t>(c.r) * p.mbps + entry_of(p, win, tb)];
            if (blk >= 0 && blk < p.num_blocks) {
                d_off = static_cast<int64_t>(blk) * blk_stride + static_cast<int64_t>(c.h) * p.bs * D +
                        static_cast<int64_t>(tb % p.bs) * D;
                d_nv = static_cast<int>(tile_rows(ctx, win, tb));
            } else {
                report(p.status, KVP_ERANGE, c.r);
            }
        }
    };
    // Small blocks (a tile spans several): the issuing lane walks the blocks.
    auto issue_small = [&](int i, int half, int st) {
        Cursor c;
        locate(t_begin + i, c);
        const int ctx = s_ctx[c.r];
        const int tb = (first_tile(ctx, win) + c.ti) * TT;
        const int32_t *btr = p.bt + static_cast<size_t>(c.r) * p.mbps;
        const uint32_t bar = kbar0 + (st * 2 + half) * 8;
        uint16_t *dst = wst + st * (S::STAGE_BYTES / 2) + half * S::TILE_WORDS;
        const uint16_t *src = half ? p.vp : p.kp;
        uint32_t bytes = 0;
        int nv = 0;
        for (int t = 0; t < TT && tb + t < ctx; t += p.bs) {
            const int b = btr[entry_of(p, win, tb + t)];
            if (b >= 0 && b < p.num_blocks) {
                bytes += p.bs * D * 2;
                nv = t + min(p.bs, ctx - tb - t);
            } else {
                report(p.status, KVP_ERANGE, c.r);
                break;  // tokens up to the bad block only
            }
        }
        if (bytes) {
            mbar_arrive_expect_tx(bar, bytes);
            for (int t = 0; t < nv; t += p.bs) {
                const int b = btr[entry_of(p, win, tb + t)];
                bulk_g2s_hint(smem_addr(dst + t * D), src + b * blk_stride + static_cast<size_t>(c.h) * p.bs * D,
                              p.bs * D * 2, bar, l2pol);
            }
        } else {
            mbar_arrive(bar);
        }
        if (half == 0) nvalid[st] = nv > 0 ? static_cast<int>(tile_rows(ctx, win, tb) & ((1u << nv) - 1u)) : 0;
    };
    // Issues half (0: K, 1: V) of tile i (warp-relative) into stage st.
    auto issue = [&](int i, int half, int st) {
        if (big_blocks) {
            if (i - dbase >= 32) load_desc(i);
            const int64_t off = __shfl_sync(0xffffffffu, d_off, i - dbase);
            const int nv = __shfl_sync(0xffffffffu, d_nv, i - dbase);
            if (half == 0) {
                // the first tile of a segment: bring its G query rows into L1
                // now, so the segment does not start with an L2 round trip
                const int qrow = __shfl_sync(0xffffffffu, d_q, i - dbase);
                if (qrow >= 0)
                    for (int l = lane; l < G * D / 32; l += 32) prefetch_l1(p.q + static_cast<size_t>(qrow) * D + l * 32);
            }
            if (lane == 0) {
                fence_proxy_async_smem();
                const uint32_t bar = kbar0 + (st * 2 + half) * 8;
                if (nv > 0) {
                    mbar_arrive_expect_tx(bar, S::TILE_WORDS * 2);
                    bulk_g2s_hint(smem_addr(wst + st * (S::STAGE_BYTES / 2) + half * S::TILE_WORDS),
                                  (half ? p.vp : p.kp) + off, S::TILE_WORDS * 2, bar, l2pol);
                } else {
                    mbar_arrive(bar);
                }
                if (half == 0) nvalid[st] = nv;
            }
        } else if (lane == 0) {
            fence_proxy_async_smem();
            issue_small(i, half, st);
        }
    };

    load_desc(0);
    for (int i = 0; i < NST && i < ntile; ++i) {
        issue(i, 0, i);
        issue(i, 1, i);
    }
    __syncwarp();

    Cursor cons;
    locate(t_begin, cons);

    // ---- per-lane state
    const int grp = lane / LPT, j = lane % LPT;
    // The passes of a batch are split over the token's lanes: lane j keeps
    // passes ppass .. ppass + PPL - 1 after the butterfly, and computes the
    // pass in slot sp as pass sp ^ ppass so that every butterfly step sends
    // the upper half of its slots (no per-lane selects).
    int ppass = 0;
#pragma unroll
    for (int l = 0; l < HALV; ++l)
        if (j & (1 << l)) ppass |= RB >> (l + 1);
    const bool primary = ((j >> HALV) & (S::REP - 1)) == 0;  // one of the REP copies
    float2 q2[G][4];
    float2 o2[G][4];
    float m_run[G], l_run[G];
    // Split segments to count in: (context, first warp, last warp) of the
    // range's first (0) and last (1) one. The first is counted in when it
    // ends, but the count's old value (lane 0) is looked at only at the end
    // of the range, so the stream does not wait for the atomic's reply; the
    // last is counted in at the end of the range.
    int npub = 0, rh0 = 0, wf0 = 0, wl0 = 0, rh1 = 0, wf1 = 0, wl1 = 0, old0 = -1;

    for (int seq = 0; seq < ntile; ++seq) {
        if (seq == 0 || cons.ti == 0) {  // a new context segment starts
            const float *qb = p.q + (static_cast<size_t>(cons.r) * p.Hq + static_cast<size_t>(cons.h) * G) * D + j * 8;
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float4 *src = reinterpret_cast<const float4 *>(qb + g * D);
                const float4 a = __ldg(src), b = __ldg(src + 1);
                q2[g][0] = make_float2(a.x * p.qscale, a.y * p.qscale);
                q2[g][1] = make_float2(a.z * p.qscale, a.w * p.qscale);
                q2[g][2] = make_float2(b.x * p.qscale, b.y * p.qscale);
                q2[g][3] = make_float2(b.z * p.qscale, b.w * p.qscale);
                m_run[g] = -INFINITY;
                l_run[g] = 0.0f;
#pragma unroll
                for (int k = 0; k < 4; ++k) o2[g][k] = make_float2(0.0f, 0.0f);
            }
        }

        const int st = seq % NST;
        const uint32_t par = (seq / NST) & 1;
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(kbar0 + st * 16, par))) {
            if (lane == 0) report(p.status, KVP_ETIMEOUT, cons.r);
            return;
        }
        const uint32_t mask = static_cast<uint32_t>(nvalid[st]);  // valid rows of the tile
        const uint16_t *sk = wst + st * (S::STAGE_BYTES / 2) + j * 8;
        const uint16_t *sv = sk + S::TILE_WORDS;

        auto tile_qk = [&](auto full_tag) {
            constexpr bool FULL = decltype(full_tag)::value;
            // ---- scores: per batch, lane computes slot sp = pass sp ^ ppass
            float sc[NB][PPL][G];
#pragma unroll
            for (int bi = 0; bi < NB; ++bi) {
                float v[NV];
#pragma unroll
                for (int sp = 0; sp < RB; ++sp) {
                    const int tok = (bi * RB + (sp ^ ppass)) * TPW + grp;
                    const uint4 wv = *reinterpret_cast<const uint4 *>(sk + tok * D);
                    float2 kf[4];
                    unpack8<BF16>(wv, kf);
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        float2 acc = __fmul2_rn(q2[g][0], kf[0]);
                        acc = __ffma2_rn(q2[g][1], kf[1], acc);
                        acc = __ffma2_rn(q2[g][2], kf[2], acc);
                        acc = __ffma2_rn(q2[g][3], kf[3], acc);
                        v[sp * G + g] = acc.x + acc.y;
                    }
                }
                // sum over the token's lanes; halving steps keep the lower slots
#pragma unroll
                for (int l = 0; l < S::LEVELS; ++l) {
                    if (l < HALV) {
                        const int half = (RB >> (l + 1)) * G;
#pragma unroll
                        for (int k = 0; k < NV / 2; ++k)
                            if (k < half) v[k] += __shfl_xor_sync(0xffffffffu, v[k + half], 1 << l);
                    } else {
#pragma unroll
                        for (int k = 0; k < PPL * G; ++k) v[k] += __shfl_xor_sync(0xffffffffu, v[k], 1 << l);
                    }
                }
#pragma unroll
                for (int sp = 0; sp < PPL; ++sp) {
                    const int tok = (bi * RB + ppass + sp) * TPW + grp;
                    const bool valid = FULL || ((mask >> tok) & 1u);
#pragma unroll
                    for (int g = 0; g < G; ++g) sc[bi][sp][g] = valid ? v[sp * G + g] : -INFINITY;
                }
            }
            // ---- reference max per head. Scores are exponentiated against a
            // per-head reference m_run that only moves when some score exceeds
            // it by more than kLazy (log2 units), so p stays below 2^kLazy and
            // most tiles need no warp-wide max and no rescale.
            bool above = false;
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int bi = 0; bi < NB; ++bi)
#pragma unroll
                    for (int sp = 0; sp < PPL; ++sp) above |= sc[bi][sp][g] > m_run[g] + kLazy;
            float alpha[G];
#pragma unroll
            for (int g = 0; g < G; ++g) alpha[g] = 1.0f;
            if (__any_sync(0xffffffffu, above)) {
                float mt[G];
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    mt[g] = sc[0][0][g];
#pragma unroll
                    for (int bi = 0; bi < NB; ++bi)
#pragma unroll
                        for (int sp = 0; sp < PPL; ++sp) mt[g] = fmaxf(mt[g], sc[bi][sp][g]);
                }
#pragma unroll
                for (int l = 0; l < 5; ++l) {
                    if (l >= HALV && l < S::LEVELS) continue;  // copies hold equal values
#pragma unroll
                    for (int g = 0; g < G; ++g) mt[g] = fmaxf(mt[g], __shfl_xor_sync(0xffffffffu, mt[g], 1 << l));
                }
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float mn = fmaxf(m_run[g], mt[g]);
                    alpha[g] = (mn == m_run[g]) ? 1.0f : ex2(m_run[g] - mn);
                    m_run[g] = mn;
                }
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float2 a2 = make_float2(alpha[g], alpha[g]);
#pragma unroll
                    for (int k = 0; k < 4; ++k) o2[g][k] = __fmul2_rn(o2[g][k], a2);
                }
            }
            // ---- probabilities: one exp2 per score; publish (p, p) pairs
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float ps = 0.0f;
#pragma unroll
                for (int bi = 0; bi < NB; ++bi)
#pragma unroll
                    for (int sp = 0; sp < PPL; ++sp) {
                        const float x = sc[bi][sp][g];
                        const float pv = (!FULL && x == -INFINITY) ? 0.0f : ex2(x - m_run[g]);
                        sc[bi][sp][g] = pv;
                        ps += pv;
                    }
                l_run[g] = l_run[g] * alpha[g] + ps;
            }
            if (primary) {
#pragma unroll
                for (int bi = 0; bi < NB; ++bi)
#pragma unroll
                    for (int sp = 0; sp < PPL; ++sp) {
                        const int tok = (bi * RB + ppass + sp) * TPW + grp;
#pragma unroll
                        for (int g = 0; g < G; g += 2) {
                            const float a = sc[bi][sp][g];
                            const float b = (g + 1 < G) ? sc[bi][sp][g + 1] : 0.0f;
                            if (g + 1 < G)
                                *reinterpret_cast<float4 *>(pw + tok * G + g) = make_float4(a, a, b, b);
                            else
                                pw[tok * G + g] = make_float2(a, a);
                        }
                    }
            }
        };
        auto tile_pv = [&](auto full_tag) {
            constexpr bool FULL = decltype(full_tag)::value;
            // ---- P.V
#pragma unroll
            for (int it = 0; it < ITERS; ++it) {
                const int tok = it * TPW + grp;
                if (!FULL && !((mask >> tok) & 1u)) continue;
                float2 pp[G];
#pragma unroll
                for (int g = 0; g < G; g += 2) {
                    if (g + 1 < G) {
                        const float4 t4 = *reinterpret_cast<const float4 *>(pw + tok * G + g);
                        pp[g] = make_float2(t4.x, t4.y);
                        pp[g + 1] = make_float2(t4.z, t4.w);
                    } else {
                        pp[g] = pw[tok * G + g];
                    }
                }
                const uint4 wv = *reinterpret_cast<const uint4 *>(sv + tok * D);
                float2 vf[4];
                unpack8<BF16>(wv, vf);
#pragma unroll
                for (int g = 0; g < G; ++g)
#pragma unroll
                    for (int e = 0; e < 4; ++e) o2[g][e] = __ffma2_rn(pp[g], vf[e], o2[g][e]);
            }
        };
        if (mask == 0xFFFFu) tile_qk(std::true_type{});
        else if (mask != 0) tile_qk(std::false_type{});
        __syncwarp();  // K half and the previous P are free
        if (seq + NST < ntile) issue(seq + NST, 0, st);
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(kbar0 + st * 16 + 8, par))) {
            if (lane == 0) report(p.status, KVP_ETIMEOUT, cons.r);
            return;
        }
        if (mask == 0xFFFFu) tile_pv(std::true_type{});
        else if (mask != 0) tile_pv(std::false_type{});
        __syncwarp();  // V half and P buffer are free
        if (seq + NST < ntile) issue(seq + NST, 1, st);

        // ---- end of this warp's segment of the (r, h) context
        if (cons.ti == cons.nt - 1 || seq == ntile - 1) {
            const int r = cons.r, h = cons.h, nt = cons.nt;
            // softmax sums per head over the distinct lanes
            float lh[G];
#pragma unroll
            for (int g = 0; g < G; ++g) lh[g] = l_run[g];
#pragma unroll
            for (int l = 0; l < 5; ++l) {
                if (l >= HALV && l < S::LEVELS) continue;
#pragma unroll
                for (int g = 0; g < G; ++g) lh[g] += __shfl_xor_sync(0xffffffffu, lh[g], 1 << l);
            }
            // outputs: sum over the TPW token groups (lane bits LPT, 2 LPT, ...)
            float2 ov[S::NO];
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int k = 0; k < 4; ++k) ov[g * 4 + k] = o2[g][k];
            transposed_reduce<S::NO, S::OLEV>(ov, lane, LPT, 32,
                                              [](float2 a, float2 b) { return make_float2(a.x + b.x, a.y + b.y); });
            const int obase = halving_base<S::NO, S::OLEV>(lane, LPT);
            // the warps covering this context's global tiles [A, A + nt)
            int w_first, w_last;
            context_warps(s_cpref[r] + h * (nt + kCtxCost) + kCtxCost, nt, W, TC, w_first, w_last);
            float *out_rh = p.out + (static_cast<size_t>(r) * p.Hq + static_cast<size_t>(h) * G) * D;
            const bool whole = (w_first == w_last);
            float *slot = part_slot<D, G>(p, w, r * Hkv + h);
#pragma unroll
            for (int x = 0; x < S::OVPL; ++x) {
                const int k = obase + x;
                const int g = k / 4, dim = j * 8 + (k % 4) * 2;
                float lg = 0.0f;
#pragma unroll
                for (int gg = 0; gg < G; ++gg)
                    if (gg == g) lg = lh[gg];
                if (whole) {
                    const float inv = lg > 0.0f ? 1.0f / lg : 0.0f;
                    *reinterpret_cast<float2 *>(out_rh + g * D + dim) = make_float2(ov[x].x * inv, ov[x].y * inv);
                } else {
                    *reinterpret_cast<float2 *>(slot + g * D + dim) = ov[x];
                }
            }
            if (!whole) {
                if (lane < G) {
                    float mg = 0.0f, lg = 0.0f;
#pragma unroll
                    for (int gg = 0; gg < G; ++gg)
                        if (gg == lane) mg = m_run[gg], lg = lh[gg];
                    slot[G * D + lane * 2 + 0] = mg;
                    slot[G * D + lane * 2 + 1] = lg;
                }
                if constexpr (!GridCombine<G>::value) {
                    // counted in at the end of the range (below), together
                    // with the range's other split segment, so the stream
                    // never waits on the count here
                    if (npub++ == 0) {
                        rh0 = r * Hkv + h, wf0 = w_first, wl0 = w_last;
                        if (seq != ntile - 1) {
                            __syncwarp();
                            if (lane == 0) {
                                fence_acq_rel_gpu();
                                old0 = atomic_add_relaxed(&p.counters[rh0], 1);
                            }
                        }
                    } else {
                        rh1 = r * Hkv + h, wf1 = w_first, wl1 = w_last;
                    }
                }
            }
        }
        advance(cons);
    }

    if constexpr (!GridCombine<G>::value) {
        // Publish this warp's split segments (at most two: the range's first
        // and last): one release fence for all partials written above, then
        // the counts. The warp that completes a context merges it.
        if (npub > 0) {
            __syncwarp();
            int last0 = 0, last1 = 0;
            if (lane == 0) {
                fence_acq_rel_gpu();
                if (old0 < 0) old0 = atomic_add_relaxed(&p.counters[rh0], 1);  // not counted in yet
                const int old1 = npub > 1 ? atomic_add_relaxed(&p.counters[rh1], 1) : -1;
                last0 = old0 == wl0 - wf0;
                last1 = npub > 1 && old1 == wl1 - wf1;
                if (last0 || last1) fence_acq_rel_gpu();  // the other contributors' partials
            }
            last0 = __shfl_sync(0xffffffffu, last0, 0);
            last1 = __shfl_sync(0xffffffffu, last1, 0);
            __syncwarp();  // lane 0's acquire orders the other lanes' loads too
            if (last0) {
                combine<D, G>(p, rh0, wf0, wl0, lane, p.out + static_cast<size_t>(rh0) * G * D);
                if (lane == 0) p.counters[rh0] = 0;  // ready for the next call
            }
            if (last1) {
                combine<D, G>(p, rh1, wf1, wl1, lane, p.out + static_cast<size_t>(rh1) * G * D);
                if (lane == 0) p.counters[rh1] = 0;
            }
        }
    }
}


// ------------------------------------- groups of 4 and 8 heads: tensor cores
// With 4 or 8 query heads per kv head the per-tile arithmetic (2 x 16 tokens
// x D x G multiply-adds, plus unpacking and lane reductions) costs the
// CUDA-core kernel about as many issue slots as the memory system needs to
// deliver the tile (8 heads: twice as many), so this variant does both
// contractions of a tile with warp-level mma.sync (m16n8k16, 16-bit inputs,
// fp32 accumulation); the rest of the design is unchanged (persistent,
// stream-K in cost space, per-warp rings, split partials merged by the last
// warp of a context for groups of 4 and by the merge grid for groups of 8):
//  * S = Q K^T: A = the group's query heads (rows past the group and rows
//    8..15 zero), B = the K tile as loaded; q is split into a 16-bit high
//    part and the 16-bit rounding of the remainder, both multiplied, so the
//    scores keep about 16 bits more than a 16-bit q would (K is exact);
//  * the accumulator of S holds (head g, tokens 2q, 2q+1, 2q+8, 2q+9) in lane
//    4g+q, which is exactly the B operand of O^T += V^T P^T: the online
//    softmax runs in registers (quad shuffles for the row max and sum) and P
//    feeds the PV product directly, again as high + low 16-bit parts whose
//    sum is also what the row sum adds;
//  * A of the PV product is V^T, read with ldmatrix.trans; K and V tiles come
//    in as 64-column boxes of a tensor map with the 128-byte swizzle (three
//    ring stages per warp), so all ldmatrix reads are free of bank conflicts;
//  * O^T (D x 8 heads) stays in registers; the segment end writes the rows
//    (or the partial) straight from the accumulator layout.
template <int D>
struct TcShape {
    static constexpr int KC = D / 16;           // 16-wide chunks of the head dim
    static constexpr int NH = D / 64;           // 64-column (128-byte) boxes per tile
    static constexpr int BOX_BYTES = TT * 128;  // one box: 16 rows x 128 bytes
    static constexpr int HALF_BYTES = NH * BOX_BYTES;  // K (or V) of one tile
    static constexpr int STAGE_BYTES = 2 * HALF_BYTES;
    static constexpr int NS = 3;                              // ring stages per warp
    // the rings fill 192 KB of shared memory: deeper rings beat more warps
    // (12 x 2 stages) except where many requests share blocks in L2
    static constexpr int NW = (D <= 128 ? 12 : 6) * 2 / NS;
    static_assert(D % 64 == 0, "head dim");
};

template <int D>
struct TcSmem {
    using S = TcShape<D>;
    static constexpr size_t bars = static_cast<size_t>(S::NW) * S::NS * S::STAGE_BYTES;  // stages first (1024-aligned)
    static constexpr size_t masks = bars + S::NW * S::NS * 2 * 8;
    static constexpr size_t tiles = align_up(masks + S::NW * S::NS * 4, 16);
    __host__ __device__ static size_t pref(int B) { return align_up(tiles + 4 * static_cast<size_t>(B), 16); }
    __host__ __device__ static size_t cpref(int B) { return align_up(pref(B) + 4 * static_cast<size_t>(B + 1), 16); }
    __host__ __device__ static size_t total(int B) { return align_up(cpref(B) + 4 * static_cast<size_t>(B + 1), 128); }
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4])
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4])
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

// d += A (16x16, row) * B (16x8, col); A rows 8..15 of the QK product are zero.
template <bool BF16>
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1)
{
    if (BF16)
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    else
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// (hi, lo) 16-bit pairs of (x, y): hi = nearest 16-bit value, lo = nearest
// 16-bit value of the remainder (computed exactly in fp32).
template <bool BF16>
__device__ __forceinline__ void split2(float x, float y, uint32_t &hi, uint32_t &lo)
{
    hi = cvt_pair<BF16>(x, y);
    const float2 h = unpack2<BF16>(hi);
    lo = cvt_pair<BF16>(x - h.x, y - h.y);
}

// Address of the 16-byte chunk (row, 8-element chunk c8 of the D columns) in
// a K or V tile stored as NH swizzled 64-column boxes.
template <int D>
__device__ __forceinline__ uint32_t tc_addr(uint32_t tile, int row, int c8)
{
    return tile + (c8 >> 3) * TcShape<D>::BOX_BYTES + row * 128 + (((c8 & 7) ^ (row & 7)) << 4);
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, int c0, int c1, int c2, uint32_t bar,
                                            uint64_t pol)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar), "l"(pol)
        : "memory");
}

template <int D, int G, bool BF16, bool WIN>
__global__ void __launch_bounds__(TcShape<D>::NW * 32, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                     const Params p)
{
    const int win = WIN ? p.window : 0;  // a compile-time 0 in the instance without a window
    static_assert(G == 4 || G == 8, "the MMA rows hold 8 heads: groups of 4 use half of them");
    using S = TcShape<D>;
    using M = TcSmem<D>;
    constexpr int NW = S::NW, KC = S::KC, NH = S::NH, NST = S::NS;
    extern __shared__ __align__(1024) unsigned char tc_smem[];
    unsigned char *smem = tc_smem;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + M::bars);
    int *nvalid_all = reinterpret_cast<int *>(smem + M::masks);
    int *s_ctx = reinterpret_cast<int *>(smem + M::tiles);  // context lengths
    int *s_pref = reinterpret_cast<int *>(smem + M::pref(p.B));
    int *s_cpref = reinterpret_cast<int *>(smem + M::cpref(p.B));

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int B = p.B, Hkv = p.Hkv;
    if (smem_addr(smem) & 1023) {  // the swizzled boxes need a 1024-aligned region
        if (tid == 0) report(p.status, KVP_EUNSUPPORTED, -1);
        return;  // uniform for the CTA, before any barrier
    }

    grid_dependency_wait();
    {
        const int64_t lines = (static_cast<int64_t>(B) * p.mbps * 4 + 127) / 128;
        const int64_t lo = lines * blockIdx.x / gridDim.x, hi = lines * (blockIdx.x + 1) / gridDim.x;
        const char *bt_bytes = reinterpret_cast<const char *>(p.bt);
        for (int64_t l = lo + tid; l < hi && l < lo + 4 * NW * 32; l += NW * 32) prefetch_l2(bt_bytes + l * 128);
    }
    for (int i = tid; i < B; i += NW * 32) {
        const int c = p.ctx[i];
        const bool ok = ctx_ok(p, c);
        s_ctx[i] = ok ? c : -1;
        if (blockIdx.x == 0 && (!ok || c == 0)) {
            if (!ok) report(p.status, KVP_ERANGE, i);
            float4 *o = reinterpret_cast<float4 *>(p.out + static_cast<size_t>(i) * p.Hq * D);
            for (int k = 0; k < p.Hq * D / 4; ++k) o[k] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    __syncthreads();
    if (warp == 0) tile_prefix(s_ctx, s_pref, s_cpref, B, Hkv, lane, win);
    __syncthreads();
    grid_launch_dependents();

    const int total = s_pref[B], TC = s_cpref[B];
    const int W = active_warps(p, total);
    const int w = blockIdx.x * NW + warp;
    if (w >= W) return;
    const int t_begin = cost_to_tile(static_cast<int64_t>(w) * TC / W, s_ctx, s_pref, s_cpref, B, win);
    const int t_end = cost_to_tile(static_cast<int64_t>(w + 1) * TC / W, s_ctx, s_pref, s_cpref, B, win);
    if (t_begin >= t_end) return;  // no CTA-wide barrier follows

    const uint32_t kbar0 = smem_addr(&bars[warp * NST * 2]);
    if (lane < 2 * NST) mbar_init(kbar0 + lane * 8, 1);
    mbar_init_fence();
    __syncwarp();

    auto locate = [&](int t, Cursor &c) {
        int lo = 0, hi = B;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (s_pref[mid] <= t) lo = mid;
            else hi = mid;
        }
        c.t = t;
        c.r = lo;
        c.nt = tiles_of(s_ctx[lo], win);
        const int local = t - s_pref[lo];
        c.h = local / c.nt;
        c.ti = local - c.h * c.nt;
    };
    auto advance = [&](Cursor &c) {
        ++c.t;
        if (++c.ti == c.nt) {
            c.ti = 0;
            if (++c.h == Hkv) {
                c.h = 0;
                do {
                    ++c.r;
                } while (c.r < B && tiles_of(s_ctx[c.r], win) == 0);
                if (c.r < B) c.nt = tiles_of(s_ctx[c.r], win);
            }
        }
    };

    const uint32_t ring = smem_addr(smem) + warp * NST * S::STAGE_BYTES;
    int *nvalid = nvalid_all + warp * NST;
    const int ntile = t_end - t_begin;
    const uint64_t l2pol = l2_evict_first_policy();

    // copy descriptors of 32 consecutive tiles, one per lane: tensor
    // coordinates (block * Hkv + head, first row in the block), valid rows
    // [f, nv) packed as nv | f << 8 (0: block id outside the pool) and the
    // segment's query row
    int d_tile = 0, d_row = 0, d_nv = 0, d_q = -1, dbase = 0;
    auto load_desc = [&](int base) {
        dbase = base;
        d_tile = d_row = d_nv = 0;
        d_q = -1;
        const int i = base + lane;
        if (i < ntile) {
            Cursor c;
            locate(t_begin + i, c);
            if (c.ti == 0 || i == 0) d_q = c.r * p.Hq + c.h * G;
            const int ctx = s_ctx[c.r];
            const int tb = (first_tile(ctx, win) + c.ti) * TT;  // position of the tile's first key
            const int blk = p.bt[static_cast<size_t>(c.r) * p.mbps + entry_of(p, win, tb)];
            if (blk >= 0 && blk < p.num_blocks) {
                d_tile = blk * Hkv + c.h;
                d_row = tb % p.bs;
                d_nv = min(TT, ctx - tb) | (win > 0 ? max(0, ctx - win - tb) : 0) << 8;
            } else {
                report(p.status, KVP_ERANGE, c.r);
            }
        }
    };
    auto issue = [&](int i, int half, int st) {
        if (i - dbase >= 32) load_desc(i);
        const int tile = __shfl_sync(0xffffffffu, d_tile, i - dbase);
        const int row = __shfl_sync(0xffffffffu, d_row, i - dbase);
        const int nv = __shfl_sync(0xffffffffu, d_nv, i - dbase);
        if (half == 0) {
            const int qrow = __shfl_sync(0xffffffffu, d_q, i - dbase);
            if (qrow >= 0)
                for (int l = lane; l < G * D / 32; l += 32) prefetch_l1(p.q + static_cast<size_t>(qrow) * D + l * 32);
        }
        if (lane == 0) {
            fence_proxy_async_smem();
            const uint32_t bar = kbar0 + (st * 2 + half) * 8;
            if (nv > 0) {
                mbar_arrive_expect_tx(bar, S::HALF_BYTES);
                const uint32_t dst = ring + st * S::STAGE_BYTES + half * S::HALF_BYTES;
                for (int hh = 0; hh < NH; ++hh)
                    tma_load_3d(dst + hh * S::BOX_BYTES, half ? &tmap_v : &tmap_k, hh * 64, row, tile, bar, l2pol);
            } else {
                mbar_arrive(bar);
            }
            if (half == 0) nvalid[st] = nv;
        }
    };

    load_desc(0);
    for (int i = 0; i < NST && i < ntile; ++i) {
        issue(i, 0, i);
        issue(i, 1, i);
    }
    __syncwarp();

    Cursor cons;
    locate(t_begin, cons);

    const int g = lane >> 2, q4 = lane & 3;  // head g; token / column pair q4
    uint32_t qh[KC][2], ql[KC][2];            // A fragments of q (high, low): (head g, dims 2q4.., 2q4+8..)
    float o[KC][4];                           // O^T: (dim 16i + g (+8), heads 2q4, 2q4 + 1)
    float m_run = -INFINITY, l_run = 0.0f;    // head g (replicated over the quad)
    // split segments to count in (groups merged in the kernel, as in decode_kernel)
    int npub = 0, rh0 = 0, wf0 = 0, wl0 = 0, rh1 = 0, wf1 = 0, wl1 = 0, old0 = -1;

    for (int seq = 0; seq < ntile; ++seq) {
        if (seq == 0 || cons.ti == 0) {  // a new context segment starts
            const float *qb = p.q + (static_cast<size_t>(cons.r) * p.Hq + static_cast<size_t>(cons.h) * G + g) * D;
#pragma unroll
            for (int c = 0; c < KC; ++c) {
                float2 x0 = make_float2(0.0f, 0.0f), x1 = x0;  // rows of heads past the group stay zero
                if (g < G) {
                    x0 = __ldg(reinterpret_cast<const float2 *>(qb + 16 * c + 2 * q4));
                    x1 = __ldg(reinterpret_cast<const float2 *>(qb + 16 * c + 8 + 2 * q4));
                }
                split2<BF16>(x0.x * p.qscale, x0.y * p.qscale, qh[c][0], ql[c][0]);
                split2<BF16>(x1.x * p.qscale, x1.y * p.qscale, qh[c][1], ql[c][1]);
#pragma unroll
                for (int e = 0; e < 4; ++e) o[c][e] = 0.0f;
            }
            m_run = -INFINITY;
            l_run = 0.0f;
        }

        const int st = seq % NST;
        const uint32_t par = (seq / NST) & 1;
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(kbar0 + st * 16, par))) {
            if (lane == 0) report(p.status, KVP_ETIMEOUT, cons.r);
            return;
        }
        const int nv = nvalid[st] & 0xFF, f0 = WIN ? nvalid[st] >> 8 : 0;  // valid rows [f0, nv)
        const uint32_t kt = ring + st * S::STAGE_BYTES, vt = kt + S::HALF_BYTES;
        // ldmatrix row of this lane: matrix lane/8 covers tokens 8*(lane/16) ..
        // and the 8-column chunk (lane/8) % 2 of each 16-column step
        const int lrow = (lane & 7) + ((lane >> 4) << 3), lsub = (lane >> 3) & 1;
        float sc[2][4];  // tokens 0-7 and 8-15
        if (nv > 0) {
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2)
#pragma unroll
                for (int e = 0; e < 4; ++e) sc[h2][e] = 0.0f;
#pragma unroll
            for (int c = 0; c < KC; ++c) {
                uint32_t b[4];
                ldsm_x4(tc_addr<D>(kt, lrow, 2 * c + lsub), b);
                // b: (tokens 0-7: dims lo, hi), (tokens 8-15: dims lo, hi)
                mma16816<BF16>(sc[0], qh[c][0], 0u, qh[c][1], 0u, b[0], b[1]);
                mma16816<BF16>(sc[0], ql[c][0], 0u, ql[c][1], 0u, b[0], b[1]);
                mma16816<BF16>(sc[1], qh[c][0], 0u, qh[c][1], 0u, b[2], b[3]);
                mma16816<BF16>(sc[1], ql[c][0], 0u, ql[c][1], 0u, b[2], b[3]);
            }
        }
        __syncwarp();  // K half is free
        if (seq + NST < ntile) issue(seq + NST, 0, st);

        if (!__all_sync(0xffffffffu, mbar_wait_bounded(kbar0 + st * 16 + 8, par))) {
            if (lane == 0) report(p.status, KVP_ETIMEOUT, cons.r);
            return;
        }
        if (nv > 0) {
            // scores of head g at tokens 2q4, 2q4+1, 8+2q4, 9+2q4 (masked by select)
            float x[4] = {sc[0][0], sc[0][1], sc[1][0], sc[1][1]};
            const int t0 = 2 * q4;
            if (t0 >= nv) x[0] = -INFINITY;
            if (t0 + 1 >= nv) x[1] = -INFINITY;
            if (t0 + 8 >= nv) x[2] = -INFINITY;
            if (t0 + 9 >= nv) x[3] = -INFINITY;
            if (f0 > 0) {  // a window's first tile: rows before its first key (uniform branch)
                if (t0 < f0) x[0] = -INFINITY;
                if (t0 + 1 < f0) x[1] = -INFINITY;
                if (t0 + 8 < f0) x[2] = -INFINITY;
                if (t0 + 9 < f0) x[3] = -INFINITY;
            }
            float mt = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
            mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 1));
            mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
            // lazy reference max (as in the CUDA-core kernel): it moves only
            // when some score exceeds it by more than kLazy
            if (__any_sync(0xffffffffu, mt > m_run + kLazy)) {
                const float mn = fmaxf(m_run, mt);
                const float alpha = (mn == m_run) ? 1.0f : ex2(m_run - mn);
                m_run = mn;
                l_run *= alpha;
                const float aA = __shfl_sync(0xffffffffu, alpha, 8 * q4);      // head 2q4
                const float aB = __shfl_sync(0xffffffffu, alpha, 8 * q4 + 4);  // head 2q4 + 1
#pragma unroll
                for (int c = 0; c < KC; ++c) {
                    o[c][0] *= aA;
                    o[c][1] *= aB;
                    o[c][2] *= aA;
                    o[c][3] *= aB;
                }
            }
            float pr[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) pr[e] = ex2(x[e] - m_run);  // masked: exp2(-inf) = 0
            uint32_t ph0, pl0, ph1, pl1;  // B fragments of P^T (tokens 2q4.., 8+2q4..; head g)
            split2<BF16>(pr[0], pr[1], ph0, pl0);
            split2<BF16>(pr[2], pr[3], ph1, pl1);
            {
                // the row sum adds exactly the weights the product uses (hi + lo)
                const float2 h0 = unpack2<BF16>(ph0), l0 = unpack2<BF16>(pl0);
                const float2 h1 = unpack2<BF16>(ph1), l1 = unpack2<BF16>(pl1);
                l_run += ((h0.x + l0.x) + (h0.y + l0.y)) + ((h1.x + l1.x) + (h1.y + l1.y));
            }
            if (nv < TT || f0 > 0) {
                // V rows past the context may hold anything (never-written
                // slots), and so may rows before a window: zero them so
                // 0 * V stays 0 in the product
                const uint4 z = make_uint4(0u, 0u, 0u, 0u);
                for (int k = lane; k < (TT - nv) * (D / 8); k += 32) {
                    const int row = nv + k / (D / 8), c8 = k % (D / 8);
                    *reinterpret_cast<uint4 *>(smem + (tc_addr<D>(vt, row, c8) - smem_addr(smem))) = z;
                }
                for (int k = lane; k < f0 * (D / 8); k += 32) {
                    const int row = k / (D / 8), c8 = k % (D / 8);
                    *reinterpret_cast<uint4 *>(smem + (tc_addr<D>(vt, row, c8) - smem_addr(smem))) = z;
                }
                __syncwarp();
            }
#pragma unroll
            for (int c = 0; c < KC; ++c) {
                uint32_t a[4];
                // V^T rows (dims 16c ..), columns (tokens): transposed 8x8 loads
                ldsm_x4_trans(tc_addr<D>(vt, (lane & 7) + ((lane >> 4) << 3), 2 * c + ((lane >> 3) & 1)), a);
                mma16816<BF16>(o[c], a[0], a[1], a[2], a[3], ph0, ph1);
                mma16816<BF16>(o[c], a[0], a[1], a[2], a[3], pl0, pl1);
            }
        }
        __syncwarp();  // V half is free
        if (seq + NST < ntile) issue(seq + NST, 1, st);

        // ---- end of this warp's segment of the (r, h) context
        if (cons.ti == cons.nt - 1 || seq == ntile - 1) {
            const int r = cons.r, h = cons.h, nt = cons.nt;
            float lh = l_run;
            lh += __shfl_xor_sync(0xffffffffu, lh, 1);
            lh += __shfl_xor_sync(0xffffffffu, lh, 2);
            int w_first, w_last;
            context_warps(s_cpref[r] + h * (nt + kCtxCost) + kCtxCost, nt, W, TC, w_first, w_last);
            const bool whole = (w_first == w_last);
            const float lA = __shfl_sync(0xffffffffu, lh, 8 * q4), lB = __shfl_sync(0xffffffffu, lh, 8 * q4 + 4);
            float *dst;
            float sA = 1.0f, sB = 1.0f;
            if (whole) {
                dst = p.out + (static_cast<size_t>(r) * p.Hq + static_cast<size_t>(h) * G) * D;
                sA = lA > 0.0f ? 1.0f / lA : 0.0f;
                sB = lB > 0.0f ? 1.0f / lB : 0.0f;
            } else {
                dst = part_slot<D, G>(p, w, r * Hkv + h);
                if (q4 == 0 && g < G) {
                    dst[G * D + 2 * g] = m_run;
                    dst[G * D + 2 * g + 1] = lh;
                }
            }
            if (2 * q4 < G) {  // this lane's heads 2q4, 2q4 + 1 are in the group
#pragma unroll
                for (int c = 0; c < KC; ++c) {
                    const int d0 = 16 * c + g;
                    dst[(2 * q4) * D + d0] = o[c][0] * sA;
                    dst[(2 * q4 + 1) * D + d0] = o[c][1] * sB;
                    dst[(2 * q4) * D + d0 + 8] = o[c][2] * sA;
                    dst[(2 * q4 + 1) * D + d0 + 8] = o[c][3] * sB;
                }
            }
            if constexpr (!GridCombine<G>::value) {
                if (!whole) {
                    if (npub++ == 0) {
                        rh0 = r * Hkv + h, wf0 = w_first, wl0 = w_last;
                        if (seq != ntile - 1) {  // counted in now, the reply looked at later
                            __syncwarp();
                            if (lane == 0) {
                                fence_acq_rel_gpu();
                                old0 = atomic_add_relaxed(&p.counters[rh0], 1);
                            }
                        }
                    } else {
                        rh1 = r * Hkv + h, wf1 = w_first, wl1 = w_last;
                    }
                }
            }
        }
        advance(cons);
    }

    if constexpr (!GridCombine<G>::value) {
        // count the range's split segments in; the warp that completes a
        // count merges that context and resets its counter
        if (npub > 0) {
            __syncwarp();
            int last0 = 0, last1 = 0;
            if (lane == 0) {
                fence_acq_rel_gpu();
                if (old0 < 0) old0 = atomic_add_relaxed(&p.counters[rh0], 1);
                const int old1 = npub > 1 ? atomic_add_relaxed(&p.counters[rh1], 1) : -1;
                last0 = old0 == wl0 - wf0;
                last1 = npub > 1 && old1 == wl1 - wf1;
                if (last0 || last1) fence_acq_rel_gpu();
            }
            last0 = __shfl_sync(0xffffffffu, last0, 0);
            last1 = __shfl_sync(0xffffffffu, last1, 0);
            __syncwarp();
            if (last0) {
                combine<D, G>(p, rh0, wf0, wl0, lane, p.out + static_cast<size_t>(rh0) * G * D);
                if (lane == 0) p.counters[rh0] = 0;
            }
            if (last1) {
                combine<D, G>(p, rh1, wf1, wl1, lane, p.out + static_cast<size_t>(rh1) * G * D);
                if (lane == 0) p.counters[rh1] = 0;
            }
        }
    }
}

// ------------------------------------------------------------ combine grid
// Log-sum-exp merge for GridCombine group sizes: one warp per (context,
// query head of the group). All segments' (max, sum) pairs come in one load
// (lane = segment), then all segments' output rows in one batch of loads.
// Launched right after the decode grid with a programmatic dependency, so
// its launch and the prefix over the context lengths overlap the decode
// grid's tail.
constexpr int kCombineWarps = 8;

template <int D, int G>
__global__ void __launch_bounds__(kCombineWarps * 32) combine_kernel(const Params p)
{
    constexpr int SL = slot_floats(G, D);
    constexpr int DL = D / 32;  // output dims per lane: 2, 4 or 8
    extern __shared__ __align__(16) int csm[];
    int *s_ctx = csm;
    int *s_pref = csm + p.B;
    int *s_cpref = s_pref + p.B + 1;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int B = p.B, Hkv = p.Hkv;

    // The context lengths were final before the decode grid started (it
    // waited for its predecessor), so they may be read before it finishes.
    for (int i = tid; i < B; i += kCombineWarps * 32) {
        const int c = p.ctx[i];
        s_ctx[i] = ctx_ok(p, c) ? c : -1;
    }
    __syncthreads();
    if (warp == 0) tile_prefix(s_ctx, s_pref, s_cpref, B, Hkv, lane, p.window);
    __syncthreads();
    const int total = s_pref[B], TC = s_cpref[B];
    const int W = active_warps(p, total);

    grid_dependency_wait();  // the partials are complete and visible
    grid_launch_dependents();

    const int ntask = B * Hkv * G;
    for (int task = blockIdx.x * kCombineWarps + warp; task < ntask; task += gridDim.x * kCombineWarps) {
        const int g = task % G, rh = task / G;
        const int r = rh / Hkv, h = rh - r * Hkv;
        const int nt = tiles_of(s_ctx[r], p.window);
        if (nt == 0) continue;
        int w_first, w_last;
        context_warps(s_cpref[r] + h * (nt + kCtxCost) + kCtxCost, nt, W, TC, w_first, w_last);
        if (w_first == w_last) continue;  // written by the decode grid itself
        const int nseg = w_last - w_first + 1;
        const float *base = part_slot<D, G>(p, w_first, rh);

        // (max, sum) of the segments; lane s keeps segment s
        float m0 = -INFINITY, l0 = 0.0f;
        if (lane < nseg) {
            const float2 v = __ldcg(reinterpret_cast<const float2 *>(base + static_cast<size_t>(lane) * SL + G * D) + g);
            m0 = v.x;
            l0 = v.y;
        }
        float M = m0;
        for (int s = lane + 32; s < nseg; s += 32) M = fmaxf(M, __ldcg(base + static_cast<size_t>(s) * SL + G * D + 2 * g));
#pragma unroll
        for (int off = 16; off; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
        const float w0 = (m0 == -INFINITY) ? 0.0f : ex2(m0 - M);
        float L = l0 * w0;
        for (int s = lane + 32; s < nseg; s += 32) {
            const float2 v = __ldcg(reinterpret_cast<const float2 *>(base + static_cast<size_t>(s) * SL + G * D) + g);
            L += (v.x == -INFINITY) ? 0.0f : v.y * ex2(v.x - M);
        }
#pragma unroll
        for (int off = 16; off; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);

        // weighted sum of the segments' rows of head g; lane owns DL dims
        float acc[DL];
#pragma unroll
        for (int d = 0; d < DL; ++d) acc[d] = 0.0f;
        const float *row = base + g * D + lane * DL;
        constexpr int CS = 8;  // segments per batch of loads
#pragma unroll 1
        for (int s0 = 0; s0 < nseg; s0 += CS) {
            float buf[CS][DL];
#pragma unroll
            for (int k = 0; k < CS; ++k) {
                const float *src = row + static_cast<size_t>(s0 + k) * SL;
#pragma unroll
                for (int d = 0; d < DL; d += 2) {
                    float2 v = make_float2(0.0f, 0.0f);
                    if (s0 + k < nseg) v = __ldcg(reinterpret_cast<const float2 *>(src + d));
                    buf[k][d] = v.x;
                    buf[k][d + 1] = v.y;
                }
            }
#pragma unroll
            for (int k = 0; k < CS; ++k) {
                const int s = s0 + k;
                float ws;
                if (s < 32) {
                    ws = __shfl_sync(0xffffffffu, w0, s & 31);  // 0 past nseg
                } else {
                    const float m = s < nseg ? __ldcg(base + static_cast<size_t>(s) * SL + G * D + 2 * g) : -INFINITY;
                    ws = (m == -INFINITY) ? 0.0f : ex2(m - M);
                }
#pragma unroll
                for (int d = 0; d < DL; ++d) acc[d] = fmaf(buf[k][d], ws, acc[d]);
            }
        }
        const float inv = L > 0.0f ? 1.0f / L : 0.0f;
        float *dst = p.out + (static_cast<size_t>(r) * p.Hq + static_cast<size_t>(h) * G + g) * D + lane * DL;
#pragma unroll
        for (int d = 0; d < DL; d += 2)
            *reinterpret_cast<float2 *>(dst + d) = make_float2(acc[d] * inv, acc[d + 1] * inv);
    }
}

// ------------------------------------------------------------------- host
static int sm_count(int dev)
{
    static int cache[64] = {0};
    if (dev < 0 || dev >= 64) return 0;
    if (!cache[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        cache[dev] = n;
    }
    return cache[dev];
}

template <int D, int G>
static int warps_per_cta() { return Shape<D, G>::NW; }

// The tensor-core kernel serves groups of 4 and 8 query heads when a
// 16-token tile lies inside one block (block size >= 16); the CUDA-core
// kernel serves the rest (groups of 1 and 2, smaller blocks).
static bool use_tc(const kvp_pool *pool, int G)
{
    return (G == 4 || G == 8) && pool->cfg.block_size >= TT && pool->cfg.head_dim % 64 == 0;
}

static int nw_for(int D, int G, bool tc)
{
    if (tc) return D <= 128 ? TcShape<128>::NW : TcShape<256>::NW;
#define KVP_NW(d, g) \
    if (D == d && G == g) return warps_per_cta<d, g>();
    KVP_NW(64, 1) KVP_NW(64, 2) KVP_NW(64, 4) KVP_NW(64, 8)
    KVP_NW(128, 1) KVP_NW(128, 2) KVP_NW(128, 4) KVP_NW(128, 8)
    KVP_NW(256, 1) KVP_NW(256, 2) KVP_NW(256, 4) KVP_NW(256, 8)
#undef KVP_NW
    return 0;
}

struct Layout {
    int warps_total, min_tiles;
    size_t counters, part, total;
};

static int plan(const kvp_pool *pool, int G, int Hkv, int B, int max_ctx, int split_req, Layout *L)
{
    const bool tc = use_tc(pool, G);
    if (split_req < 0 || split_req % TT)
        return set_error(KVP_EINVAL, "split_tokens %d must be 0 or a positive multiple of %d", split_req, TT);
    if (B < 0 || B > kMaxBatch) return set_error(KVP_EUNSUPPORTED, "B %d outside [0, %d]", B, kMaxBatch);
    if (max_ctx < 0) return set_error(KVP_EINVAL, "max_ctx_len must be >= 0");
    const int nw = nw_for(pool->cfg.head_dim, G, tc);
    if (!nw) return set_error(KVP_EUNSUPPORTED, "decode: head_dim %d with GQA group %d not built", pool->cfg.head_dim, G);
    const int sms = sm_count(pool->cfg.device);
    if (!sms) return set_error(KVP_ECUDA, "cannot query the SM count of device %d", pool->cfg.device);
    L->warps_total = sms * nw;
    L->min_tiles = split_req > 0 ? split_req / TT : kAutoMinTiles;
    const size_t rh = static_cast<size_t>(B) * Hkv;
    const size_t slot = static_cast<size_t>(slot_floats(G, pool->cfg.head_dim)) * 4;
    L->counters = 0;
    L->part = align_up(rh * 4, 256);
    L->total = align_up(L->part + (L->warps_total + rh) * slot, 256);
    return KVP_OK;
}

template <int D, int G>
static int launch(const Params &p, bool bf16, int blocks, cudaStream_t s)
{
    const size_t smem = Smem<D, G>::total(p.B);
    if (smem > 227 * 1024) return set_error(KVP_EUNSUPPORTED, "decode: %zu bytes of shared memory", smem);
    const bool win = p.window > 0;
    auto kern = bf16 ? (win ? decode_kernel<D, G, true, true> : decode_kernel<D, G, true, false>)
                     : (win ? decode_kernel<D, G, false, true> : decode_kernel<D, G, false, false>);
    int rc = check_cuda(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)),
                        "decode smem attribute");
    if (rc) return rc;
    if ((rc = check_cuda(launch_pdl(kern, dim3(blocks), dim3(Shape<D, G>::NW * 32), smem, s, p), "decode launch")))
        return rc;
    if constexpr (GridCombine<G>::value) {
        const int tasks = p.B * p.Hkv * G;
        const int cblocks = max(1, min((tasks + kCombineWarps - 1) / kCombineWarps, 4 * blocks));
        const size_t csmem = align_up(sizeof(int) * (3 * static_cast<size_t>(p.B) + 2), 16);
        rc = check_cuda(launch_pdl(combine_kernel<D, G>, dim3(cblocks), dim3(kCombineWarps * 32), csmem, s, p),
                        "decode combine launch");
    }
    return rc;
}

// 8-head groups on the tensor-core kernel (block size >= 16: a tile is one
// 16-row box inside one block), then the merge grid.
template <int D, int G>
static int launch_tc(const Params &p, const kvp_pool *pool, int layer, bool bf16, cudaStream_t s)
{
    const size_t smem = TcSmem<D>::total(p.B);
    if (smem > 227 * 1024) return set_error(KVP_EUNSUPPORTED, "decode: %zu bytes of shared memory", smem);
    CUtensorMap mk, mv;
    int rc;
    if ((rc = make_pool_tmap(&mk, pool->k_base + pool->layer_words * layer, pool, TT)) ||
        (rc = make_pool_tmap(&mv, pool->v_base + pool->layer_words * layer, pool, TT)))
        return rc;
    const bool win = p.window > 0;
    auto kern = bf16 ? (win ? decode_tc_kernel<D, G, true, true> : decode_tc_kernel<D, G, true, false>)
                     : (win ? decode_tc_kernel<D, G, false, true> : decode_tc_kernel<D, G, false, false>);
    if ((rc = check_cuda(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)),
                         "decode smem attribute")))
        return rc;
    const int blocks = p.warps_total / TcShape<D>::NW;
    if ((rc = check_cuda(launch_pdl(kern, dim3(blocks), dim3(TcShape<D>::NW * 32), smem, s, mk, mv, p), "decode launch")))
        return rc;
    if constexpr (!GridCombine<G>::value) return KVP_OK;  // merged inside the kernel
    const int tasks = p.B * p.Hkv * G;
    const int cblocks = max(1, min((tasks + kCombineWarps - 1) / kCombineWarps, 4 * blocks));
    const size_t csmem = align_up(sizeof(int) * (3 * static_cast<size_t>(p.B) + 2), 16);
    return check_cuda(launch_pdl(combine_kernel<D, G>, dim3(cblocks), dim3(kCombineWarps * 32), csmem, s, p),
                      "decode combine launch");
}

template <int D>
static int launch_g(const Params &p, bool bf16, int blocks, int G, cudaStream_t s)
{
    switch (G) {
    case 1: return launch<D, 1>(p, bf16, blocks, s);
    case 2: return launch<D, 2>(p, bf16, blocks, s);
    case 4: return launch<D, 4>(p, bf16, blocks, s);
    case 8: return launch<D, 8>(p, bf16, blocks, s);
    default: return set_error(KVP_EUNSUPPORTED, "decode: GQA group %d not built (1, 2, 4, 8)", G);
    }
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
    if (max_blocks_per_seq <= 0) return set_error(KVP_EINVAL, "max_blocks_per_seq must be > 0");
    if (attn->window > 0 && static_cast<int64_t>(max_blocks_per_seq) * pool->cfg.block_size < attn->window)
        return set_error(KVP_EINVAL, "a ring of %d blocks of %d cannot hold the window of %d", max_blocks_per_seq,
                         pool->cfg.block_size, attn->window);
    if (!q || !block_tables || !ctx_lens || !out || !workspace)
        return set_error(KVP_EINVAL, "paged_decode_attention: a required pointer is NULL");
    if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(out)) & 15)
        return set_error(KVP_EINVAL, "q and out must be 16-byte aligned");
    if (reinterpret_cast<uintptr_t>(workspace) & 255) return set_error(KVP_EINVAL, "workspace must be 256-byte aligned");
    dec::Layout L;
    if ((rc = dec::plan(pool, G, Hkv, B, max_ctx_len, split_tokens, &L))) return rc;
    if (ws_bytes < L.total) return set_error(KVP_EINVAL, "workspace of %zu bytes, %zu needed", ws_bytes, L.total);
    dec::Params p;
    p.kp = pool->k_base + pool->layer_words * layer;
    p.vp = pool->v_base + pool->layer_words * layer;
    p.q = q, p.bt = block_tables, p.ctx = ctx_lens, p.out = out;
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    p.counters = reinterpret_cast<int *>(ws + L.counters);
    p.part = reinterpret_cast<float *>(ws + L.part);
    p.status = pool->status;
    p.B = B, p.Hq = Hq, p.Hkv = Hkv, p.mbps = max_blocks_per_seq, p.bs = pool->cfg.block_size;
    p.num_blocks = pool->cfg.num_blocks, p.max_ctx = max_ctx_len, p.max_seq_len = pool->cfg.max_seq_len;
    p.warps_total = L.warps_total, p.min_tiles = L.min_tiles;
    p.window = attn->window;
    const double scale = static_cast<double>(static_cast<float>(1.0 / sqrt(static_cast<double>(pool->cfg.head_dim))));
    p.qscale = static_cast<float>(scale * 1.4426950408889634);  // log2(e): softmax via exp2
    const bool bf16 = pool->cfg.kv_dtype == KVP_BF16;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dec::use_tc(pool, G)) {
        const int D = pool->cfg.head_dim;
        if (G == 8) {
            if (D == 64) return dec::launch_tc<64, 8>(p, pool, layer, bf16, s);
            if (D == 128) return dec::launch_tc<128, 8>(p, pool, layer, bf16, s);
            if (D == 256) return dec::launch_tc<256, 8>(p, pool, layer, bf16, s);
        } else {
            if (D == 64) return dec::launch_tc<64, 4>(p, pool, layer, bf16, s);
            if (D == 128) return dec::launch_tc<128, 4>(p, pool, layer, bf16, s);
            if (D == 256) return dec::launch_tc<256, 4>(p, pool, layer, bf16, s);
        }
        return set_error(KVP_EUNSUPPORTED, "head_dim %d", D);
    }
    const int blocks = L.warps_total / dec::nw_for(pool->cfg.head_dim, G, false);
    switch (pool->cfg.head_dim) {
    case 64: return dec::launch_g<64>(p, bf16, blocks, G, s);
    case 128: return dec::launch_g<128>(p, bf16, blocks, G, s);
    case 256: return dec::launch_g<256>(p, bf16, blocks, G, s);
    default: return set_error(KVP_EUNSUPPORTED, "head_dim %d", pool->cfg.head_dim);
    }
}
