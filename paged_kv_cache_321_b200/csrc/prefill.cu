// paged_prefill_attention: chunked-prefill attention over the paged cache on
// the tcgen05 tensor cores.
//
// Method: the single-request paged kernel of runHybridAttentionBlock in
// makarna/pkg/model/arch/hybrid_decoder.go for seqLen > 1 (kvLen = startPos +
// seqLen, query i at position startPos + i sees keys 0..startPos + i), with
// the textbook attention of forward_layer in
// soft3/glia/run/arch/decoder/forward.rs.
//
// B200 design. Prefill is a dense contraction (S = Q K^T and O = P V over
// 128-key tiles), so it runs on the 5th-generation tensor cores:
//  * one CTA per (sequence, kv head, 128/G query tokens), launched longest
//    first (a counting sort of the work items in every CTA's prologue): its
//    128 rows are
//    (query token, query head of the GQA group) pairs sharing the kv head's
//    K and V, so one M=128 MMA serves the whole group;
//  * warps 9 and 10 stream K and V tiles of 128 keys with tiled TMA
//    copies (cp.async.bulk.tensor, no multicast) straight out of the block
//    pool through a tensor map over [blocks*Hkv][block_size][D]; the block
//    table supplies the third coordinate, the 128-byte swizzle produces the
//    canonical UMMA operand layout;
//  * warp 8 (one thread) issues tcgen05.mma kind::f16 (fp16 operands, fp32
//    accumulation in TMEM): S(j) into one of two TMEM buffers while the
//    softmax warps work on S(j-1), then O += P(j-1) V(j-1) into a TMEM
//    accumulator;
//  * warps 0-7 own half a row each (two warps per 32-row TMEM quarter, one
//    per 64-column half; row max and sum exchanged through shared memory):
//    tcgen05.ld of the S row half, causal mask,
//    online softmax with a lazily moved reference max (O in TMEM is rescaled
//    only when a row max grows by more than 2^8), P rounded to fp16 and
//    written swizzled to shared memory as the A operand of the PV MMA. P is
//    double-buffered, so the softmax of tile j runs while the tensor core
//    does PV(j-1) and QK(j+1); it waits for PV(j-1) only to rescale O;
//  * the epilogue reads O from TMEM, divides by the row sum and writes fp32.
#include <cuda.h>

#include <climits>
#include <math.h>

#include "common.cuh"

namespace kvp {
namespace pre {

constexpr int D = 128;       // head dim of this kernel
constexpr int BM = 128;      // rows per CTA: (query token, group head) pairs
constexpr int BN = 128;      // keys per KV tile
constexpr int NSTAGE = 2;    // K/V stages
constexpr int NSMX = 8;                       // softmax warps: two per 32-row quarter (one per 64-column half)
constexpr int MMA_WARP = NSMX, K_WARP = NSMX + 1, V_WARP = NSMX + 2;  // MMA issuer, K and V producers
constexpr int NTHREADS = (NSMX + 3) * 32;
constexpr float kLazy = 8.0f;

// shared-memory layout (bytes from a 1024-aligned base)
constexpr int HALF_BYTES = 128 * 128;            // [128 rows][64 fp16] with 128B swizzle
constexpr int TILE_BYTES = 2 * HALF_BYTES;       // 128 rows x 128 fp16
constexpr int Q_OFF = 0;
constexpr int K_OFF = Q_OFF + TILE_BYTES;
constexpr int V_OFF = K_OFF + NSTAGE * TILE_BYTES;
constexpr int P_OFF = V_OFF + NSTAGE * TILE_BYTES;  // [2] P buffers: tile j uses P_OFF + (j & 1) * TILE_BYTES
constexpr int BAR_OFF = P_OFF + 2 * TILE_BYTES;
// barriers
enum {
    B_KFULL = 0,             // [NSTAGE] K tile landed (TMA tx)
    B_VFULL = B_KFULL + 2,   // [NSTAGE] V tile landed
    B_KEMPTY = B_VFULL + 2,  // [NSTAGE] K stage free (QK of the tile done)
    B_VEMPTY = B_KEMPTY + 2, // [NSTAGE] V stage free (PV of the tile done)
    B_SFULL = B_VEMPTY + 2,  // [2] S buffer computed
    B_SFREE = B_SFULL + 2,   // [2] S buffer read by the softmax warps
    B_PFULL = B_SFREE + 2,   // [2] P buffer written by the softmax warps
    B_ODONE = B_PFULL + 2,   // [2] PV of tile j done (j & 1): O holds it, P buffer j & 1 is free
    B_QFULL = B_ODONE + 2,   // Q written by the softmax warps
    B_XCH = B_QFULL + 1,     // [4 quarters][2] row max (last: row sum) of both halves of a row published
    NBARS = B_XCH + 8
};
constexpr int TMEM_PTR_OFF = BAR_OFF + NBARS * 8;
constexpr int XCH_OFF = TMEM_PTR_OFF + 16;          // float [2 parities][2 halves][128 rows]
constexpr int SMEM_BYTES = XCH_OFF + 2 * 2 * BM * 4;  // the dynamic region is 1024-aligned
static_assert(SMEM_BYTES <= 227 * 1024, "prefill shared memory");
constexpr uint32_t TMEM_COLS = 512;                    // S0, S1, O (128 columns each)

struct Params {
    const float *q;         // [total_q][Hq][D]
    float *out;             // [total_q][Hq][D]
    const int32_t *cu_q;    // [S + 1]
    const int32_t *ctx;     // [S]
    const int32_t *bt;      // [S][mbps]
    int *status;
    int S, Hq, Hkv, G, mbps, bs, num_blocks, max_seq_len, ntq;  // ntq: query tiles per sequence (grid)
    int nbins;              // cost bins: KV tiles an item can read, 0 .. max_seq_len / BN + 1
    int window;             // sliding window in keys (0: none); > 0 makes block-table rows rings
    float qscale;           // softmax scale * log2(e), folded into Q
};

// A sequence the kernel refuses: an empty or over-long chunk, a context past
// the table (without a window) or max_seq_len, or (with a ring) a chunk whose
// own later keys have overwritten a ring slot one of its queries still needs
// (the smallest key needed, max(0, first query position - window + 1), must
// be newer than ctx - 1 - mbps * bs).
__device__ __forceinline__ bool seq_refused(const Params &p, int q_len, int ctx)
{
    if (q_len <= 0 || ctx < q_len || ctx > p.max_seq_len) return true;
    if (p.window == 0) return ctx > p.mbps * p.bs;
    const int need = max(0, ctx - q_len - p.window + 1);
    return static_cast<int64_t>(need) + static_cast<int64_t>(p.mbps) * p.bs <= ctx - 1;
}

// First KV tile (of BN keys) the query at position `pos` needs.
__device__ __forceinline__ int first_kv_tile(const Params &p, int pos)
{
    return p.window > 0 ? max(0, pos - p.window + 1) / BN : 0;
}

// ---------------------------------------------------------------- PTX
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, int c0, int c1, int c2, uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, bool acc)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc ? 1u : 0u));
}

__device__ __forceinline__ void mma_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 consecutive fp32 columns of this thread's TMEM lane
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32])
{
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
        "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
        "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15])),
        "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])), "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])),
        "r"(__float_as_uint(v[20])), "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
        "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])), "r"(__float_as_uint(v[27])),
        "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])), "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
        : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// UMMA shared-memory descriptor, 128-byte swizzle, version 1 (sm100).
// K-major: LBO unused (1), SBO = 1024 B between 8-row groups.
// MN-major: LBO = bytes between 64-element MN groups, SBO = 1024 B.
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo_bytes, uint32_t sbo_bytes)
{
    uint64_t d = 0;
    d |= static_cast<uint64_t>((addr >> 4) & 0x3FFF);
    d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFF) << 16;
    d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFF) << 32;
    d |= static_cast<uint64_t>(1) << 46;  // version
    d |= static_cast<uint64_t>(2) << 61;  // SWIZZLE_128B
    return d;
}

// Instruction descriptor of kind::f16 with fp32 accumulation.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, bool bf16, bool b_mn_major)
{
    return (1u << 4)                                  // D format f32
           | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10)  // A, B format
           | (0u << 15)                               // A K-major
           | ((b_mn_major ? 1u : 0u) << 16)           // B major
           | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// Byte offset of 16-byte chunk c (0..7) of row r inside a [rows][128 B]
// region with the 128-byte swizzle (chunk index XOR row % 8).
__device__ __forceinline__ uint32_t swz(int r, int c) { return r * 128 + ((c ^ (r & 7)) << 4); }

template <bool BF16>
__device__ __forceinline__ uint32_t pack2(float a, float b)
{
    uint32_t r;
    if (BF16) {
        __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
        r = *reinterpret_cast<uint32_t *>(&h);
    } else {
        __half2 h = __floats2half2_rn(a, b);
        r = *reinterpret_cast<uint32_t *>(&h);
    }
    return r;
}

template <bool BF16>
__device__ __forceinline__ float2 unpack(uint32_t w)
{
    if (BF16) return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
    __half2 h = *reinterpret_cast<__half2 *>(&w);
    return __half22float2(h);
}

template <int G, bool BF16>
__global__ void __launch_bounds__(NTHREADS, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v, const Params p)
{
    constexpr int TQ = BM / G;  // query tokens per CTA
    extern __shared__ __align__(1024) unsigned char smem[];
    const uint32_t sbase = smem_addr(smem);
    auto bar = [&](int i) { return sbase + BAR_OFF + i * 8; };
    uint32_t *tmem_ptr = reinterpret_cast<uint32_t *>(smem + TMEM_PTR_OFF);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // launched with a programmatic dependency: nothing global is read before
    // the previous grid has completed
    grid_dependency_wait();
    grid_launch_dependents();
    // ---- longest-first work order. Items are (sequence, query tile); an
    // item's cost is the number of KV tiles it reads (0 for query tiles past
    // its sequence's chunk and for sequences in error). The CTA launched
    // L-th takes the unit of rank L in descending cost (ties by item index,
    // kv heads innermost), so the longest items start first and the short
    // ones fill the tail. Every CTA computes the same order: a counting sort
    // of the item costs in shared memory (the P buffers are not in use yet).
    int s, h, qt;
    {
        int *hist = reinterpret_cast<int *>(smem + P_OFF);
        int *pick = reinterpret_cast<int *>(smem + XCH_OFF);
        const int nitems = p.S * p.ntq;
        auto cost = [&](int i) -> int {
            const int si = i / p.ntq, t0i = (i - si * p.ntq) * TQ;
            const int ql = p.cu_q[si + 1] - p.cu_q[si], c = p.ctx[si];
            if (t0i >= ql || seq_refused(p, ql, c)) return 0;
            return (c - ql + min(ql, t0i + TQ) - 1) / BN + 1 - first_kv_tile(p, c - ql + t0i);
        };
        for (int i = tid; i < p.nbins; i += NTHREADS) hist[i] = 0;
        __syncthreads();
        for (int i = tid; i < nitems; i += NTHREADS) atomicAdd(&hist[cost(i)], 1);
        __syncthreads();
        if (warp == 0) {
            const int R = blockIdx.x / p.Hkv;  // rank of this CTA's item
            // the cost bin holding rank R, scanning bins from the most costly
            int above = 0, bin = 0;
            for (int top = p.nbins - 1; top >= 0; top -= 32) {
                const int v = top - lane;
                const int n = v >= 0 ? hist[v] : 0;
                int x = n;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, x, off);
                    if (lane >= off) x += y;
                }
                const unsigned hit = __ballot_sync(0xffffffffu, n > 0 && above + x - n <= R && R < above + x);
                if (hit) {
                    const int src = __ffs(hit) - 1;
                    bin = top - src;
                    above += __shfl_sync(0xffffffffu, x - n, src);
                    break;
                }
                above += __shfl_sync(0xffffffffu, x, 31);
            }
            // the (R - above)-th item of that cost, in index order
            int k = R - above, item = 0;
            for (int base = 0; base < nitems; base += 32) {
                const int i = base + lane;
                const unsigned m = __ballot_sync(0xffffffffu, i < nitems && cost(i) == bin);
                const int c = __popc(m);
                if (k < c) {
                    unsigned mm = m;
                    for (int q = 0; q < k; ++q) mm &= mm - 1;  // drop the k lowest matches
                    item = base + __ffs(mm) - 1;
                    break;
                }
                k -= c;
            }
            if (lane == 0) pick[0] = item;
        }
        __syncthreads();
        const int item = pick[0];
        s = item / p.ntq;
        qt = item - s * p.ntq;
        h = blockIdx.x - (blockIdx.x / p.Hkv) * p.Hkv;
        __syncthreads();  // pick and hist are reused below
    }
    const int q0 = p.cu_q[s], q_len = p.cu_q[s + 1] - q0;
    const int ctx = p.ctx[s];
    const int t0 = qt * TQ;  // first query token of this tile (within the sequence)
    if (t0 >= q_len) return;
    if (seq_refused(p, q_len, ctx)) {
        if (qt == 0 && h == 0 && tid == 0) report(p.status, KVP_ERANGE, s);
        return;  // uniform for the CTA: nothing allocated yet
    }
    if (sbase & 1023) {  // the 128-byte swizzle atoms need a 1024-aligned region
        if (tid == 0) report(p.status, KVP_EUNSUPPORTED, -1);
        return;  // uniform for the CTA: nothing allocated yet
    }
    const int first_pos = ctx - q_len;                   // position of query 0
    const int last_pos = first_pos + min(q_len, t0 + TQ) - 1;
    const int j0 = first_kv_tile(p, first_pos + t0);     // KV tiles j0 .. j0 + nkv - 1 of the position axis
    const int nkv = last_pos / BN + 1 - j0;              // KV tiles this CTA reads

    if (tid == 0) {
        for (int i = 0; i < NBARS; ++i) {
            const bool by_softmax_warps =
                i == B_SFREE || i == B_SFREE + 1 || i == B_PFULL || i == B_PFULL + 1 || i == B_QFULL;
            mbar_init(bar(i), by_softmax_warps ? NSMX : (i >= B_XCH ? 2 : 1));
        }
        mbar_init_fence();
    }
    if (warp == MMA_WARP) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_ptr)),
                     "r"(TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_ptr;
    bool timed_out = false;

    if (warp == K_WARP || warp == V_WARP) {
        // ------------------------------------------------- TMA producers (K, V)
        // One warp streams K tiles, another V tiles, each gated only by its
        // own stage-free barrier: K of stage st is free once QK of tile
        // j - NSTAGE is done, V once its PV is, so K runs ahead of the
        // softmax and QK(j + 1) overlaps the softmax of tile j. Lane b handles
        // block b of each 128-key tile (at most 8 blocks: the block size is at
        // least 16): the block ids of a tile come in one batch of loads (the
        // next tile's while this one's copies fly), and each lane issues its
        // own block's copies.
        const int kv = warp == V_WARP;
        const int32_t *btr = p.bt + static_cast<size_t>(s) * p.mbps;
        const uint32_t half_rows_bytes = p.bs * 128;  // one block's rows of one 64-column half
        auto block_of = [&](int j) {  // j: tile of the position axis
            const int first = (j * BN) / p.bs;
            const int nblk = (min(BN, ctx - j * BN) + p.bs - 1) / p.bs;
            const int e = p.window > 0 ? (first + lane) % p.mbps : first + lane;  // the ring
            return lane < nblk ? btr[e] : -1;
        };
        int blk = block_of(j0);
        for (int j = 0; j < nkv && !timed_out; ++j) {
            const int st = j % NSTAGE;
            const int nblk = (min(BN, ctx - (j0 + j) * BN) + p.bs - 1) / p.bs;
            const bool mine = lane < nblk;
            const bool valid = mine && blk >= 0 && blk < p.num_blocks;
            if (mine && !valid && !kv) report(p.status, KVP_ERANGE, s);
            const int loaded = __popc(__ballot_sync(0xffffffffu, valid));
            const uint32_t bytes = static_cast<uint32_t>(loaded) * 2 * half_rows_bytes;
            if (j >= NSTAGE) {
                bool ok = true;
                if (lane == 0) ok = mbar_wait_bounded(bar((kv ? B_VEMPTY : B_KEMPTY) + st), ((j / NSTAGE) - 1) & 1);
                if (!__shfl_sync(0xffffffffu, ok, 0)) {
                    timed_out = true;
                    break;
                }
            }
            const uint32_t full = bar((kv ? B_VFULL : B_KFULL) + st);
            if (lane == 0) {
                if (bytes) mbar_arrive_expect_tx(full, bytes);
                else mbar_arrive(full);
            }
            __syncwarp();
            if (valid) {
                const int tile = blk * p.Hkv + h;
                const uint32_t dst0 = sbase + (kv ? V_OFF : K_OFF) + st * TILE_BYTES + lane * half_rows_bytes;
                for (int hf = 0; hf < 2; ++hf)
                    tma_load_3d(dst0 + hf * HALF_BYTES, kv ? &tmap_v : &tmap_k, hf * 64, 0, tile, full);
            }
            if (j + 1 < nkv) blk = block_of(j0 + j + 1);
        }
    } else if (warp == MMA_WARP) {
        // ------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t IDS = idesc_f16(BM, BN, BF16, false);  // S = Q K^T
            constexpr uint32_t IDO = idesc_f16(BM, D, BF16, true);    // O += P V (V MN-major)
            auto qk = [&](int j) -> bool {
                const int st = j % NSTAGE, b = j & 1;
                if (!mbar_wait_bounded(bar(B_KFULL + st), (j / NSTAGE) & 1)) return false;
                if (j >= 2 && !mbar_wait_bounded(bar(B_SFREE + b), ((j >> 1) - 1) & 1)) return false;
                tc_fence_after();
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t koff = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
                    mma_f16(tmem + b * 128, sdesc(sbase + Q_OFF + koff, 16, 1024),
                            sdesc(sbase + K_OFF + st * TILE_BYTES + koff, 16, 1024), IDS, kk > 0);
                }
                mma_commit(bar(B_SFULL + b));
                mma_commit(bar(B_KEMPTY + st));
                return true;
            };
            auto pv = [&](int j) -> bool {
                const int st = j % NSTAGE, pb = j & 1;
                if (!mbar_wait_bounded(bar(B_PFULL + pb), (j >> 1) & 1)) return false;
                if (!mbar_wait_bounded(bar(B_VFULL + st), (j / NSTAGE) & 1)) return false;
                tc_fence_after();
                for (int kk = 0; kk < BN / 16; ++kk) {
                    const uint32_t aoff = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;  // P: keys are K
                    const uint32_t boff = kk * 16 * 128;                              // V: 16 key rows
                    mma_f16(tmem + 256, sdesc(sbase + P_OFF + pb * TILE_BYTES + aoff, 16, 1024),
                            sdesc(sbase + V_OFF + st * TILE_BYTES + boff, HALF_BYTES, 1024), IDO, j > 0 || kk > 0);
                }
                mma_commit(bar(B_ODONE + pb));
                mma_commit(bar(B_VEMPTY + st));
                return true;
            };
            bool ok = mbar_wait_bounded(bar(B_QFULL), 0);
            for (int j = 0; ok && j < nkv; ++j) {
                ok = qk(j);
                if (ok && j >= 1) ok = pv(j - 1);
            }
            if (ok) ok = pv(nkv - 1);
            if (!ok) timed_out = true;
        }
    } else {
        // ------------------------------------------------------ softmax warps
        // Warp w owns rows r = 32*(w%4) + lane (its TMEM lanes) and columns
        // 64*(w/4) .. +63 of them; the two warps of a row exchange the row
        // max (and at the end the row sum) through shared memory, ordered by
        // a 2-arrival mbarrier per quarter and tile parity.
        const int qw = warp & 3, hf = warp >> 2;
        const int r = qw * 32 + lane;  // row = g * TQ + t
        const int g = r / TQ, t = r % TQ;
        const int qi = t0 + t;  // query index in the sequence
        const bool row_ok = qi < q_len;
        const int pos = row_ok ? first_pos + qi : -1;  // sees keys 0..pos (or lo_key..pos)
        const int lo_key = p.window > 0 ? pos - p.window + 1 : INT_MIN;
        const size_t qrow = (static_cast<size_t>(q0 + qi) * p.Hq + static_cast<size_t>(h) * G + g) * D;
        float *xch = reinterpret_cast<float *>(smem + XCH_OFF);  // [parity][half][row]
        // publishes v for this row and returns the partner half's value for
        // exchange round k (k = tile index; the final sums use k = nkv)
        auto exchange = [&](int k, float v, float &other) -> bool {
            xch[((k & 1) * 2 + hf) * BM + r] = v;
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_XCH + qw * 2 + (k & 1)));
            if (!__all_sync(0xffffffffu, mbar_wait_bounded(bar(B_XCH + qw * 2 + (k & 1)), (k >> 1) & 1))) return false;
            other = xch[((k & 1) * 2 + (hf ^ 1)) * BM + r];
            return true;
        };
        // Q row half: scale, round to 16 bits, store swizzled
        {
            const float4 *src = reinterpret_cast<const float4 *>(p.q + qrow) + hf * 16;
#pragma unroll
            for (int c = 0; c < 8; ++c) {  // 8 chunks of 8 values
                float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b4 = a;
                if (row_ok) {
                    a = src[2 * c];
                    b4 = src[2 * c + 1];
                }
                const float sc = p.qscale;
                const uint4 w = make_uint4(pack2<BF16>(a.x * sc, a.y * sc), pack2<BF16>(a.z * sc, a.w * sc),
                                           pack2<BF16>(b4.x * sc, b4.y * sc), pack2<BF16>(b4.z * sc, b4.w * sc));
                *reinterpret_cast<uint4 *>(smem + Q_OFF + hf * HALF_BYTES + swz(r, c)) = w;
            }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_QFULL));

        const uint32_t lane_base = static_cast<uint32_t>(qw * 32) << 16;
        const uint32_t col0 = hf * 64;  // this warp's first column of S and O
        float m_ref = -INFINITY, l = 0.0f;
        for (int j = 0; j < nkv && !timed_out; ++j) {
            const int b = j & 1;
            if (!__all_sync(0xffffffffu, mbar_wait_bounded(bar(B_SFULL + b), (j >> 1) & 1))) {
                timed_out = true;
                break;
            }
            tc_fence_after();
            float sv[64];
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                float tmp[32];
                tmem_ld32(tmem + lane_base + b * 128 + col0 + c * 32, tmp);
#pragma unroll
                for (int i = 0; i < 32; ++i) sv[c * 32 + i] = tmp[i];
            }
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_SFREE + b));
            // causal (and window) mask, skipped when all 64 keys are visible
            // to every row of the warp, as for all but the diagonal tiles
            // (and the window's edge), and row max
            const int key0 = (j0 + j) * BN + col0;
            float mx = -INFINITY;
            if (__all_sync(0xffffffffu, key0 + 63 <= pos && key0 >= lo_key)) {
#pragma unroll
                for (int i = 0; i < 64; ++i) mx = fmaxf(mx, sv[i]);
            } else {
#pragma unroll
                for (int i = 0; i < 64; ++i) {
                    if (key0 + i > pos || key0 + i < lo_key) sv[i] = -INFINITY;
                    mx = fmaxf(mx, sv[i]);
                }
            }
            float mo;
            if (!exchange(j, mx, mo)) {
                timed_out = true;
                break;
            }
            mx = fmaxf(mx, mo);
            // O may be rescaled only once the PV of the previous tile is in it
            // (rare: the reference max moves lazily); P buffer j & 1 is free
            // once the PV of tile j - 2 is done. Otherwise this tile's
            // softmax overlaps the tensor core's PV(j - 1) and QK(j + 1).
            const bool move = mx > m_ref + kLazy;  // the same in both halves of a row
            const bool rescale = __any_sync(0xffffffffu, move) && j > 0;
            if (rescale && !__all_sync(0xffffffffu, mbar_wait_bounded(bar(B_ODONE + ((j - 1) & 1)), ((j - 1) >> 1) & 1))) {
                timed_out = true;
                break;
            }
            if (j >= 2 && !__all_sync(0xffffffffu, mbar_wait_bounded(bar(B_ODONE + (j & 1)), ((j - 2) >> 1) & 1))) {
                timed_out = true;
                break;
            }
            tc_fence_after();
            if (rescale) {
                const float alpha = move ? ex2(m_ref - mx) : 1.0f;
#pragma unroll 1
                for (int c = 0; c < 2; ++c) {
                    float o[32];
                    tmem_ld32(tmem + lane_base + 256 + col0 + c * 32, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] *= alpha;
                    tmem_st32(tmem + lane_base + 256 + col0 + c * 32, o);
                }
                tmem_wait_st();
                l *= alpha;
            }
            if (move) m_ref = mx;
            // With a window a row may see no key of a tile (m_ref still -inf):
            // its scores are all -inf, and a finite reference keeps P at 0
            const float mr = (p.window > 0 && m_ref == -INFINITY) ? 0.0f : m_ref;
            // P = exp2(s - m_ref) rounded to 16 bits; l sums the rounded values
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float x0 = sv[c * 8 + 2 * e], x1 = sv[c * 8 + 2 * e + 1];
                    // a masked score gives exp2(-inf) = 0: without a window m_ref
                    // is finite from the first tile on in every row that has a
                    // query (key 0 is visible to all), with one mr is; rows past
                    // the chunk are never stored
                    const float p0 = ex2(x0 - mr);
                    const float p1 = ex2(x1 - mr);
                    w[e] = pack2<BF16>(p0, p1);
                    const float2 back = unpack<BF16>(w[e]);
                    l += back.x + back.y;
                }
                *reinterpret_cast<uint4 *>(smem + P_OFF + (j & 1) * TILE_BYTES + hf * HALF_BYTES + swz(r, c)) =
                    make_uint4(w[0], w[1], w[2], w[3]);
            }
            // keys of this tile past the context: their V rows may hold
            // anything (or were not loaded); zero them so 0 * V stays 0
            const int nkeys = min(BN, ctx - (j0 + j) * BN);
            if (nkeys < BN) {
                const int st = j % NSTAGE;
                if (!__all_sync(0xffffffffu, mbar_wait_bounded(bar(B_VFULL + st), (j / NSTAGE) & 1))) {
                    timed_out = true;
                    break;
                }
                unsigned char *vt = smem + V_OFF + st * TILE_BYTES;
                for (int idx = r + hf * BM; idx < (BN - nkeys) * 16; idx += 2 * BM) {
                    const int row = nkeys + idx / 16, chunk = idx % 16;
                    *reinterpret_cast<uint4 *>(vt + (chunk >> 3) * HALF_BYTES + row * 128 + ((chunk & 7) << 4)) =
                        make_uint4(0u, 0u, 0u, 0u);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_PFULL + (j & 1)));
        }
        // epilogue: O / (sum of both halves' l)
        float lo = 0.0f;
        if (!timed_out && exchange(nkv, l, lo) &&
            __all_sync(0xffffffffu, mbar_wait_bounded(bar(B_ODONE + ((nkv - 1) & 1)), ((nkv - 1) >> 1) & 1))) {
            tc_fence_after();
            const float lt = l + lo;
            const float inv = lt > 0.0f ? 1.0f / lt : 0.0f;
            float4 *dst = reinterpret_cast<float4 *>(p.out + qrow) + hf * 16;
#pragma unroll 1
            for (int c = 0; c < 2; ++c) {
                float o[32];
                tmem_ld32(tmem + lane_base + 256 + col0 + c * 32, o);
                tmem_wait_ld();
                if (row_ok) {
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        dst[c * 8 + i] = make_float4(o[4 * i] * inv, o[4 * i + 1] * inv, o[4 * i + 2] * inv, o[4 * i + 3] * inv);
                }
            }
        } else {
            timed_out = true;
        }
    }
    if (timed_out && (lane == 0)) report(p.status, KVP_ETIMEOUT, s);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == MMA_WARP)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS));
}

// ------------------------------------------------------------------- host
template <int G, bool BF16>
static int launch(const CUtensorMap &mk, const CUtensorMap &mv, const Params &p, cudaStream_t s)
{
    auto kern = prefill_kernel<G, BF16>;
    int rc = check_cuda(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES),
                        "prefill smem attribute");
    if (rc) return rc;
    const int64_t units = static_cast<int64_t>(p.ntq) * p.Hkv * p.S;
    if (units > 0x7FFFFFFF) return set_error(KVP_EINVAL, "prefill: too many query tiles");
    if (static_cast<int64_t>(p.nbins) * 4 > TILE_BYTES * 2) return set_error(KVP_EUNSUPPORTED, "prefill: max_seq_len too large");
    return check_cuda(launch_pdl(kern, dim3(static_cast<unsigned>(units)), dim3(NTHREADS), SMEM_BYTES, s, mk, mv, p),
                      "prefill launch");
}

}  // namespace pre
}  // namespace kvp

using namespace kvp;

extern "C" size_t paged_prefill_workspace_size(const kvp_pool *pool, const kvp_attn_config *attn, int S,
                                               int total_q, int max_q_len)
{
    (void)pool, (void)attn, (void)S, (void)total_q, (void)max_q_len;
    return 0;  // the prefill kernel keeps everything on chip
}

extern "C" int paged_prefill_attention(kvp_pool *pool, int layer, const kvp_attn_config *attn, int S,
                                       const float *q, const int32_t *cu_q, const int32_t *ctx_lens,
                                       const int32_t *block_tables, int max_blocks_per_seq, int total_q,
                                       int max_q_len, float *out, void *workspace, size_t ws_bytes, void *stream)
{
    (void)workspace, (void)ws_bytes;
    int rc = check_pool(pool, layer);
    if (rc) return rc;
    int Hq, Hkv, G;
    if ((rc = resolve_attn(pool, attn, &Hq, &Hkv, &G))) return rc;
    if (S == 0 || total_q == 0) return KVP_OK;
    if (S < 0 || S > 65535 || total_q < 0 || max_q_len <= 0 || max_blocks_per_seq <= 0)
        return set_error(KVP_EINVAL, "bad prefill sizes (S %d, total_q %d, max_q_len %d)", S, total_q, max_q_len);
    if (!q || !cu_q || !ctx_lens || !block_tables || !out)
        return set_error(KVP_EINVAL, "paged_prefill_attention: a required pointer is NULL");
    if (pool->cfg.head_dim != pre::D)
        return set_error(KVP_EUNSUPPORTED, "prefill is built for head_dim %d (got %d)", pre::D, pool->cfg.head_dim);
    const int bs = pool->cfg.block_size;
    if (bs < 16 || bs > pre::BN) return set_error(KVP_EUNSUPPORTED, "prefill needs 16 <= block_size <= %d", pre::BN);
    if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(out)) & 15)
        return set_error(KVP_EINVAL, "q and out must be 16-byte aligned");
    CUtensorMap mk, mv;
    const uint16_t *kp = pool->k_base + pool->layer_words * layer;
    const uint16_t *vp = pool->v_base + pool->layer_words * layer;
    if ((rc = make_pool_tmap(&mk, kp, pool, bs)) || (rc = make_pool_tmap(&mv, vp, pool, bs))) return rc;
    pre::Params p;
    p.q = q, p.out = out, p.cu_q = cu_q, p.ctx = ctx_lens, p.bt = block_tables, p.status = pool->status;
    p.S = S, p.Hq = Hq, p.Hkv = Hkv, p.G = G, p.mbps = max_blocks_per_seq, p.bs = bs;
    p.num_blocks = pool->cfg.num_blocks, p.max_seq_len = pool->cfg.max_seq_len;
    p.nbins = pool->cfg.max_seq_len / pre::BN + 2;
    p.window = attn->window;
    if (attn->window > 0 && static_cast<int64_t>(max_blocks_per_seq) * bs < attn->window)
        return set_error(KVP_EINVAL, "a ring of %d blocks of %d cannot hold the window of %d", max_blocks_per_seq, bs,
                         attn->window);
    const double scale = static_cast<double>(static_cast<float>(1.0 / sqrt(static_cast<double>(pre::D))));
    p.qscale = static_cast<float>(scale * 1.4426950408889634);
    const bool bf16 = pool->cfg.kv_dtype == KVP_BF16;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    auto go = [&](auto g_tag) -> int {
        constexpr int GG = decltype(g_tag)::value;
        p.ntq = (max_q_len + pre::BM / GG - 1) / (pre::BM / GG);
        return bf16 ? pre::launch<GG, true>(mk, mv, p, s) : pre::launch<GG, false>(mk, mv, p, s);
    };
    switch (G) {
    case 1: return go(std::integral_constant<int, 1>{});
    case 2: return go(std::integral_constant<int, 2>{});
    case 4: return go(std::integral_constant<int, 4>{});
    case 8: return go(std::integral_constant<int, 8>{});
    default: return set_error(KVP_EUNSUPPORTED, "prefill: GQA group %d not built (1, 2, 4, 8)", G);
    }
}
