/*
 * oracle.c -- plain, slow CPU reference for the paged KV cache hot path.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product (the CUDA library and its
 * Python binding) includes, links or calls this file. Only the test suite,
 * the smoke check and the benchmark's CPU-baseline leg load it.
 *
 * Built with: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fno-builtin-{sin,cos,pow}
 *             -fopenmp -shared -fPIC ... -lm
 * so every float operation below is one IEEE-754 operation rounded to
 * nearest-even, in the order written (no contraction into FMA, no
 * reassociation, no flush-to-zero).
 *
 * Sources (cited by page title and function):
 *   makarna/pkg/kvcache/paged_cache.go
 *     - float32ToFloat16Bits / float32ToBFloat16Bits : fp32 -> 16-bit RNE
 *     - GetBlockForPosition / GetBlockOffset, Append : position -> (block, slot)
 *     - viewsLockedAt : last block holds (computed - start) valid slots
 *     - writePackedBlockU32 : head-major [head][slot][dim] block layout
 *     - Append / AppendKV : "KV cache overflow" past MaxSeqLen,
 *       "block index out of range"
 *   makarna/pkg/model/arch/hybrid_decoder.go
 *     - runHybridAttentionBlock : QNorm/KNorm, then RoPE, then append, then
 *       paged attention over kvLen = startPos + seqLen keys with
 *       scale = float32(1/sqrt(float64(HeadDim)))
 *     - normalizeHybridDecoderConfig : NumKVHeads 0 means NumHeads
 *   soft3/glia/run/arch/decoder/forward.rs (forward_layer)
 *     - per-head RMS normalisation: sumsq, (sumsq * 1/D + eps).sqrt(), 1/rms
 *     - textbook attention: kv head = h / (Hq/Hkv); scores * scale; subtract
 *       the max; exp; normalise; sum of p * v
 *
 * Readings where the pages are silent: NaN conversion keeps the payload's top bits and sets the quiet bit;
 * RMSNorm sums squares sequentially in fp32 and applies the weight after the
 * normalisation; RoPE rotates the first rope_dim dims (all by default) as
 * rotate-half pairs (i, i + rope_dim/2) or interleaved pairs (2i, 2i+1), with
 * angle p * theta^(-2i/rope_dim), cos/sin evaluated in fp64 and rounded to
 * fp32; a query at position p sees keys 0..p, or the last `window` of them
 * read through a ring of block-table entries; attention accumulates in fp64
 * from the exact values of the stored 16-bit keys and values.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_F16 = 1, ORC_BF16 = 2, ORC_F32 = 3 };
enum {
    ORC_OK = 0,
    ORC_EINVAL = -1,
    ORC_ERANGE = -2,
    ORC_EOVERFLOW = -3,
    ORC_EUNSUPPORTED = -4
};

/* ------------------------------------------------------------------------ */
/* 16-bit formats, from their definitions                                    */
/* ------------------------------------------------------------------------ */

static float bits_to_f32(uint32_t b) { float f; memcpy(&f, &b, 4); return f; }

/* Exact value of a binary16 pattern: sign, 5-bit exponent (bias 15), 10-bit
 * fraction; exponent 0 is subnormal (fraction * 2^-24). */
double orc_f16_value(uint16_t h)
{
    int sign = h >> 15, e = (h >> 10) & 0x1F, f = h & 0x3FF;
    double mag;
    if (e == 0x1F)
        mag = f ? NAN : INFINITY;
    else if (e == 0)
        mag = ldexp((double)f, -24);
    else
        mag = ldexp((double)(1024 + f), e - 25);
    return sign ? -mag : mag;
}

/* bfloat16 is the upper half of a binary32 word. */
double orc_bf16_value(uint16_t h) { return (double)bits_to_f32((uint32_t)h << 16); }

double orc_value16(uint16_t h, int dtype) { return dtype == ORC_F16 ? orc_f16_value(h) : orc_bf16_value(h); }

/* Nearest binary16 to the float32 x, ties to the even fraction
 * (makarna/pkg/kvcache/paged_cache.go, float32ToFloat16Bits). Written as the definition:
 * find the spacing of binary16 values at |x|, round |x|/spacing to the
 * nearest integer with ties to even, and encode the result. Magnitudes that
 * round to 2^16 or beyond become infinity. */
uint16_t orc_f32_to_f16(uint32_t xb)
{
    uint16_t sign = (uint16_t)((xb >> 16) & 0x8000);
    float x = bits_to_f32(xb);
    if (isnan(x))  /* reading: quiet NaN, top 10 payload bits kept */
        return sign | 0x7E00 | (uint16_t)((xb & 0x7FFFFF) >> 13);
    double a = fabs((double)x);
    if (isinf(a))
        return sign | 0x7C00;
    int e;                     /* a = m * 2^e with m in [0.5, 1) */
    if (a == 0.0)
        return sign;
    frexp(a, &e);
    int ulp_exp = (e - 1) - 10;  /* spacing 2^(floor(log2 a) - 10) ... */
    if (ulp_exp < -24)
        ulp_exp = -24;           /* ... but never below the subnormal step */
    double n = rint(ldexp(a, -ulp_exp));  /* exact scaling; rint = ties-to-even */
    double r = ldexp(n, ulp_exp);
    if (r >= 65536.0)
        return sign | 0x7C00;
    if (r < ldexp(1.0, -14))     /* subnormal (or zero): fraction = r / 2^-24 */
        return sign | (uint16_t)ldexp(r, 24);
    int re;
    frexp(r, &re);
    int E = re - 1;              /* r in [2^E, 2^(E+1)) */
    uint16_t frac = (uint16_t)(ldexp(r, 10 - E) - 1024.0);
    return sign | (uint16_t)((E + 15) << 10) | frac;
}

/* Nearest bfloat16 to the float32 x, ties to even
 * (makarna/pkg/kvcache/paged_cache.go, float32ToBFloat16Bits). bfloat16 keeps binary32's
 * exponent range with 8 significant bits, so the spacing at |x| is
 * 2^(floor(log2|x|) - 7), never below 2^-133. */
uint16_t orc_f32_to_bf16(uint32_t xb)
{
    float x = bits_to_f32(xb);
    if (isnan(x))  /* reading: quiet NaN, top payload bits kept */
        return (uint16_t)(xb >> 16) | 0x0040;
    uint16_t sign = (uint16_t)((xb >> 16) & 0x8000);
    double a = fabs((double)x);
    if (isinf(a))
        return sign | 0x7F80;
    if (a == 0.0)
        return sign;
    int e;
    frexp(a, &e);
    int ulp_exp = (e - 1) - 7;
    if (ulp_exp < -133)
        ulp_exp = -133;
    double r = ldexp(rint(ldexp(a, -ulp_exp)), ulp_exp);
    if (r >= ldexp(1.0, 128))
        return sign | 0x7F80;
    float rf = (float)r;         /* exact: r lies on the bfloat16 grid */
    uint32_t rb;
    memcpy(&rb, &rf, 4);
    return sign | (uint16_t)(rb >> 16);
}

uint16_t orc_convert(uint32_t xb, int dtype) { return dtype == ORC_F16 ? orc_f32_to_f16(xb) : orc_f32_to_bf16(xb); }

/* Pool elements. A 16-bit pool (fp16, bf16) holds the conversion of each
 * float32; an fp32 pool (the float32 K/V blocks the pages' paged attention
 * also reads, runHybridAttentionBlock's f32 path) holds the float32 itself. */
static double pool_value(const void *pool, int64_t i, int dtype)
{
    if (dtype == ORC_F32) return (double)bits_to_f32(((const uint32_t *)pool)[i]);
    return orc_value16(((const uint16_t *)pool)[i], dtype);
}

static void pool_store(void *pool, int64_t i, uint32_t xb, int dtype)
{
    if (dtype == ORC_F32) ((uint32_t *)pool)[i] = xb;
    else ((uint16_t *)pool)[i] = orc_convert(xb, dtype);
}

/* Converts the bit patterns start .. start+count-1 (exhaustive checks). */
void orc_convert_range(uint64_t start, uint64_t count, int dtype, uint16_t *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)count; ++i)
        out[i] = orc_convert((uint32_t)(start + (uint64_t)i), dtype);
}

void orc_convert_array(const float *x, int64_t n, int dtype, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i) {
        uint32_t b;
        memcpy(&b, &x[i], 4);
        out[i] = orc_convert(b, dtype);
    }
}

/* ------------------------------------------------------------------------ */
/* Per-head RMSNorm (soft3/glia/run/arch/decoder/forward.rs, forward_layer's per-head RMS form, plus the weight)     */
/* ------------------------------------------------------------------------ */

void orc_rmsnorm_row(const float *x, const float *w, int D, float eps, float *y)
{
    float ss = 0.0f;
    for (int d = 0; d < D; ++d) {
        float sq = x[d] * x[d];
        ss = ss + sq;
    }
    float inv_d = 1.0f / (float)D;
    float ms = ss * inv_d;
    float rms = sqrtf(ms + eps);
    float inv = 1.0f / rms;
    for (int d = 0; d < D; ++d) {
        float t = x[d] * inv;
        y[d] = w ? t * w[d] : t;
    }
}

/* ------------------------------------------------------------------------ */
/* RoPE (reading: pairs of the first rope_dim dims, angle p * theta^(-2i/rope_dim)) */
/* ------------------------------------------------------------------------ */

/* table[p][i] = (cos, sin) of p * theta^(-2i/R), i < R/2, fp64 rounded to fp32,
 * for a rotary width R (R = head_dim for full rotary; the rope_dim of a
 * partial-rotary layer, Op::Rope's rope_dim in the per-layer RoPE step of
 * forward_layer in soft3/glia/run/arch/decoder/forward.rs). */
void orc_rope_table(double theta, int R, int max_pos, float *table)
{
    int half = R / 2;
    for (int p = 0; p < max_pos; ++p) {
        for (int i = 0; i < half; ++i) {
            double inv_freq = pow(theta, -(2.0 * (double)i) / (double)R);
            double ang = (double)p * inv_freq;
            table[((int64_t)p * half + i) * 2 + 0] = (float)cos(ang);
            table[((int64_t)p * half + i) * 2 + 1] = (float)sin(ang);
        }
    }
}

/* Rotates one head row of D dims by the (cos, sin) pairs cs[i] of one
 * position. Only the first R dims rotate (partial rotary); the rest are
 * copied. Pair i is (i, i + R/2) for style 0 (rotate-half) and (2i, 2i + 1)
 * for style 1 (interleaved); either way
 *   y[a] = x[a]*c - x[b]*s,  y[b] = x[b]*c + x[a]*s,
 * every product and sum rounded to fp32 separately. */
void orc_rope_row_ex(const float *x, int D, int R, int style, const float *cs, float *y)
{
    int half = R / 2;
    for (int d = R; d < D; ++d) y[d] = x[d];
    for (int i = 0; i < half; ++i) {
        int a = style ? 2 * i : i, b = style ? 2 * i + 1 : i + half;
        float c = cs[2 * i], s = cs[2 * i + 1];
        float xa = x[a], xb = x[b];
        float ac = xa * c, bs = xb * s, bc = xb * c, as = xa * s;
        y[a] = ac - bs;
        y[b] = bc + as;
    }
}

/* Full rotary, rotate-half. */
void orc_rope_row(const float *x, int D, const float *cs, float *y) { orc_rope_row_ex(x, D, D, 0, cs, y); }

/* ------------------------------------------------------------------------ */
/* kv_append                                                                 */
/* ------------------------------------------------------------------------ */

/* Pool of ONE layer: [num_blocks][Hkv][bs][D] 16-bit words (head-major block,
 * as the packed CPU blocks of makarna/pkg/kvcache/paged_cache.go, writePackedBlockU32). */
static int64_t slot_index(int blk, int h, int slot, int d, int Hkv, int bs, int D)
{
    return (((int64_t)blk * Hkv + h) * bs + slot) * D + d;
}

/* Block-table entry holding position p. With a sliding window (window > 0)
 * a row is a ring of mbps blocks, the paged form of the window-sized ring
 * cache of a sliding layer (kv_slot = past_seq_len % cache_seq in
 * forward_layer, soft3/glia/run/arch/decoder/forward.rs): position p lives in
 * entry (p / bs) mod mbps, slot p % bs. Without a window the entry is p / bs. */
static int entry_of(int p, int bs, int mbps, int window)
{
    return window > 0 ? (p / bs) % mbps : p / bs;
}

/*
 * For each new token t of sequence r = tok_req[t] at position p = positions[t]:
 *   q' = rope(norm_q(q)), k' = rope(norm_k(k)), v' = v   (norm/rope optional;
 *        rope over the first rope_dim dims, pairing by rope_style)
 *   K/V slot = (block_tables[r][entry_of(p)], p % bs); store convert(k'), convert(v')
 *   q_out[t] = q'
 * Rejected tokens (first error code returned):
 *   window > 0 with mbps * bs < window -> ORC_EINVAL for the call, nothing done
 *   r outside [0, S)                   -> ORC_EINVAL, q_out row zeroed
 *   p outside [0, max_seq_len) or past the rope table
 *                                      -> ORC_EOVERFLOW, q_out row zeroed
 *   entry >= max_blocks_per_seq, or a block id outside [0, num_blocks)
 *                                      -> ORC_ERANGE, q_out written, no store
 */
int orc_kv_append(int T, int S, int Hq, int Hkv, int D, int bs, int num_blocks, int max_seq_len, int dtype,
                  const float *q, const float *k, const float *v, const float *q_norm_w, const float *k_norm_w,
                  float eps, const float *rope, int rope_max_pos, int rope_dim, int rope_style, int window,
                  const int32_t *tok_req, const int32_t *positions, const int32_t *block_tables, int mbps,
                  void *pool_k, void *pool_v, float *q_out)
{
    int status = ORC_OK;
    if (rope_dim == 0) rope_dim = D;
    if (window > 0 && (int64_t)mbps * bs < window) return ORC_EINVAL;
    float *t0 = malloc(sizeof(float) * D), *t1 = malloc(sizeof(float) * D);
#define ORC_FAIL(code) do { if (status == ORC_OK) status = (code); } while (0)
    for (int t = 0; t < T; ++t) {
        int r = tok_req[t], p = positions[t];
        float *qo = q_out + (int64_t)t * Hq * D;
        if (r < 0 || r >= S) {
            ORC_FAIL(ORC_EINVAL);
            memset(qo, 0, sizeof(float) * Hq * D);
            continue;
        }
        if (p < 0 || p >= max_seq_len || (rope && p >= rope_max_pos)) {
            ORC_FAIL(ORC_EOVERFLOW);
            memset(qo, 0, sizeof(float) * Hq * D);
            continue;
        }
        const float *cs = rope ? rope + (int64_t)p * rope_dim : NULL; /* rope_dim/2 pairs */
        for (int g = 0; g < Hq; ++g) {
            const float *x = q + ((int64_t)t * Hq + g) * D;
            memcpy(t0, x, sizeof(float) * D);
            if (q_norm_w) { orc_rmsnorm_row(t0, q_norm_w, D, eps, t1); memcpy(t0, t1, sizeof(float) * D); }
            if (cs) { orc_rope_row_ex(t0, D, rope_dim, rope_style, cs, t1); memcpy(t0, t1, sizeof(float) * D); }
            memcpy(qo + (int64_t)g * D, t0, sizeof(float) * D);
        }
        int j = entry_of(p, bs, mbps, window), slot = p % bs;
        if (j >= mbps) { ORC_FAIL(ORC_ERANGE); continue; }
        int blk = block_tables[(int64_t)r * mbps + j];
        if (blk < 0 || blk >= num_blocks) { ORC_FAIL(ORC_ERANGE); continue; }
        for (int h = 0; h < Hkv; ++h) {
            const float *x = k + ((int64_t)t * Hkv + h) * D;
            memcpy(t0, x, sizeof(float) * D);
            if (k_norm_w) { orc_rmsnorm_row(t0, k_norm_w, D, eps, t1); memcpy(t0, t1, sizeof(float) * D); }
            if (cs) { orc_rope_row_ex(t0, D, rope_dim, rope_style, cs, t1); memcpy(t0, t1, sizeof(float) * D); }
            const float *vx = v + ((int64_t)t * Hkv + h) * D;
            for (int d = 0; d < D; ++d) {
                uint32_t kb, vb;
                memcpy(&kb, &t0[d], 4);
                memcpy(&vb, &vx[d], 4);
                pool_store(pool_k, slot_index(blk, h, slot, d, Hkv, bs, D), kb, dtype);
                pool_store(pool_v, slot_index(blk, h, slot, d, Hkv, bs, D), vb, dtype);
            }
        }
    }
#undef ORC_FAIL
    free(t0);
    free(t1);
    return status;
}

/* ------------------------------------------------------------------------ */
/* Attention over the paged cache                                            */
/* ------------------------------------------------------------------------ */

/* One query head against nk keys whose exact values are given by callbacks
 * of the storage (paged or contiguous). s_j = (q . k_j) * scale;
 * w_j = exp(s_j - max) / sum; out = sum_j w_j v_j; all fp64. */
typedef struct {
    const void *k, *v;
    const int32_t *bt; /* paged: this sequence's block table row */
    int paged, Hkv, bs, D, h, dtype;
    int mbps, window;  /* paged: entry_of's ring when window > 0 */
} kv_src;

/* Element index of key (or value) row j. */
static int64_t key_row(const kv_src *s, int j)
{
    if (s->paged)
        return slot_index(s->bt[entry_of(j, s->bs, s->mbps, s->window)], s->h, j % s->bs, 0, s->Hkv, s->bs, s->D);
    return ((int64_t)j * s->Hkv + s->h) * s->D; /* contiguous [nk][Hkv][D] */
}

/* One query head over keys j0 .. nk-1 (sbuf holds nk doubles; w_out, if
 * given, receives weight j at index j and 0 below j0). */
static void attend_one(const float *qrow, int j0, int nk, const kv_src *src, double scale, double *sbuf, float *out,
                       double *w_out)
{
    int D = src->D;
    if (nk <= j0) {
        for (int d = 0; d < D; ++d) out[d] = 0.0f;
        return;
    }
    for (int j = 0; j < j0; ++j) sbuf[j] = 0.0;
    double m = -INFINITY;
    for (int j = j0; j < nk; ++j) {
        const int64_t kr = key_row(src, j);
        double acc = 0.0;
        for (int d = 0; d < D; ++d)
            acc += (double)qrow[d] * pool_value(src->k, kr + d, src->dtype);
        sbuf[j] = acc * scale;
        if (sbuf[j] > m) m = sbuf[j];
    }
    double l = 0.0;
    for (int j = j0; j < nk; ++j) {
        sbuf[j] = exp(sbuf[j] - m);
        l += sbuf[j];
    }
    for (int j = j0; j < nk; ++j) sbuf[j] /= l;
    if (w_out) memcpy(w_out, sbuf, sizeof(double) * nk);
    double *acc = calloc(D, sizeof(double));
    for (int j = j0; j < nk; ++j) {
        const int64_t vr = key_row(src, j);
        for (int d = 0; d < D; ++d) acc[d] += sbuf[j] * pool_value(src->v, vr + d, src->dtype);
    }
    for (int d = 0; d < D; ++d) out[d] = (float)acc[d];
    free(acc);
}

/* The softmax scale of makarna/pkg/model/arch/hybrid_decoder.go, runHybridAttentionBlock: float32(1/sqrt(float64(D))). */
double orc_softmax_scale(int D) { return (double)(float)(1.0 / sqrt((double)D)); }

/*
 * Paged attention for NQ queries. Query i belongs to sequence q_seq[i], sits at
 * position p = q_pos[i] and sees keys 0..p of that sequence (q_pos = -1: no
 * keys, output zeros); with a sliding window (window > 0) only keys
 * max(0, p - window + 1)..p, read through entry_of's ring (the window of
 * forward_layer in soft3/glia/run/arch/decoder/forward.rs: the last cache_seq
 * positions, read_start = total_seq - cache_seq). q and out are [NQ][Hq][D]
 * float32. Query head g reads kv head g / (Hq / Hkv). weights (optional)
 * receives the softmax weights, [NQ][Hq][max_keys], indexed by key position.
 * A block id outside [0, num_blocks) or a block index past mbps zeroes that
 * query's output and returns ORC_ERANGE; window > 0 with mbps * bs < window
 * returns ORC_EINVAL before any work.
 */
int orc_paged_attention(int NQ, int Hq, int Hkv, int D, int bs, int num_blocks, int dtype, const float *q,
                        const int32_t *q_seq, const int32_t *q_pos, const int32_t *block_tables, int mbps,
                        const void *pool_k, const void *pool_v, float *out, double *weights, int max_keys,
                        int window, int threads)
{
    if (Hkv <= 0 || Hq % Hkv) return ORC_EUNSUPPORTED;
    if (window > 0 && (int64_t)mbps * bs < window) return ORC_EINVAL;
    int group = Hq / Hkv, status = ORC_OK;
    double scale = orc_softmax_scale(D);
#ifdef _OPENMP
    if (threads > 0) omp_set_num_threads(threads);
#endif
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < NQ; ++i) {
        int r = q_seq[i], nk = q_pos[i] + 1;
        int j0 = window > 0 && nk > window ? nk - window : 0;
        const int32_t *bt = block_tables + (int64_t)r * mbps;
        int bad = window == 0 && nk > mbps * bs;
        for (int j = j0; !bad && j < nk; ++j) {
            int e = entry_of(j, bs, mbps, window);
            bad = bt[e] < 0 || bt[e] >= num_blocks;
        }
        if (bad) {
            memset(out + (int64_t)i * Hq * D, 0, sizeof(float) * Hq * D);
#pragma omp critical
            status = ORC_ERANGE;
            continue;
        }
        double *sbuf = malloc(sizeof(double) * (nk > 0 ? nk : 1));
        for (int g = 0; g < Hq; ++g) {
            kv_src src = {pool_k, pool_v, bt, 1, Hkv, bs, D, g / group, dtype, mbps, window};
            double *w = weights ? weights + ((int64_t)i * Hq + g) * max_keys : NULL;
            attend_one(q + ((int64_t)i * Hq + g) * D, j0, nk, &src, scale, sbuf, out + ((int64_t)i * Hq + g) * D,
                       w);
        }
        free(sbuf);
    }
    return status;
}

/* Contiguous, unpaged copy of one sequence's first nk tokens: [nk][Hkv][D],
 * built token by token through the block table (the idea of gatherKV in
 * makarna/pkg/model/arch/hybrid_decoder.go). */
int orc_gather_contiguous(int nk, int Hkv, int D, int bs, int num_blocks, const int32_t *bt_row, int mbps,
                          const void *pool, void *dst, int dtype)
{
    const size_t es = dtype == ORC_F32 ? 4 : 2; /* bytes per element */
    for (int t = 0; t < nk; ++t) {
        int j = t / bs;
        if (j >= mbps || bt_row[j] < 0 || bt_row[j] >= num_blocks) return ORC_ERANGE;
        for (int h = 0; h < Hkv; ++h)
            memcpy((char *)dst + (((int64_t)t * Hkv + h) * D) * es,
                   (const char *)pool + slot_index(bt_row[j], h, t % bs, 0, Hkv, bs, D) * es, es * D);
    }
    return ORC_OK;
}

/* Dense attention of Hq query heads over a contiguous [nk][Hkv][D] copy. */
int orc_dense_attention(int Hq, int Hkv, int D, int dtype, const float *q, int nk, const void *ck,
                        const void *cv, float *out)
{
    if (Hkv <= 0 || Hq % Hkv) return ORC_EUNSUPPORTED;
    double *sbuf = malloc(sizeof(double) * (nk > 0 ? nk : 1));
    double scale = orc_softmax_scale(D);
    for (int g = 0; g < Hq; ++g) {
        kv_src src = {ck, cv, NULL, 0, Hkv, 0, D, g / (Hq / Hkv), dtype, 0, 0};
        attend_one(q + (int64_t)g * D, 0, nk, &src, scale, sbuf, out + (int64_t)g * D, NULL);
    }
    free(sbuf);
    return ORC_OK;
}
