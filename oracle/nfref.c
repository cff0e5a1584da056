/*
 * nfref.c -- plain, slow CPU oracle for K8/V4 quantised-KV decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  It shares
 * no source, header, table or helper with the CUDA library under
 * long_context_quantized_b200/csrc, and neither side includes the other.
 *
 * What it computes, and where that comes from:
 *
 *  - The KV dtype is "rk8v4 (K8/V4)": int8 keys, 4-bit values
 *    (page "3090 单卡跑 Qwen3.8-27B：NInfer 上机实测（180K 上下文 / C2 并发 /
 *    4bit KV）", section 一.3 启动, flag --kv-dtype rk8v4).  The pages do not
 *    give the bit format; the format implemented here is the one this project
 *    fixes:
 *      K: symmetric int8, one fp16 scale absmax/127 per (token, kv-head),
 *         codes in [-127, 127];
 *      V: symmetric int4, one fp16 scale absmax/7 per (token, kv-head, group of
 *         32 channels), codes in [-7, 7], two's-complement nibbles, the even
 *         channel in the low nibble;
 *      scale = fp16_rne_saturating(fp32(absmax / 127 or 7));
 *      code  = clamp(round_half_even(fp32(x / float(scale)))), 0 if scale == 0.
 *  - The same section lists the --kv-dtype options int8 and fp8, by name only.
 *    Read here as: int8 -- K and V both by the K rule above; fp8 -- K and V as
 *    OCP E4M3FN codes of x / scale with scale = absmax / 448 per (token,
 *    kv-head), rounded half to even and saturated at +-448 (formats 2 and 3
 *    of the pool below).
 *  - Page "影片筆記：NInfer + 千问3.8 27b = 1.5倍速@256K上下文(单张4090 24GB)",
 *    section 三, names "RK4V4-E8" as the KV quantisation that fits a 256K
 *    context into 24 GB (its own transcription-doubts section questions the
 *    name; no page gives its bits).  Read here as format 4: K and V both
 *    symmetric 4-bit codes in [-7, 7] (nibbles packed as the K8/V4 values
 *    are), every group of 32 channels of a (token, kv-head) with one shared
 *    power-of-two scale 2^e stored as an 8-bit exponent byte e + 127 ("E8");
 *    e is the smallest integer with 2^e >= fp32(absmax / 7), clamped to
 *    [-126, 127]; code = clamp(round_half_even(fp32(x / 2^e)), -7, 7).  The
 *    "R" is left unread, as for rk8v4: no rotation.
 *  - The cache is segmented (page "標籤: vLLM", section 2 "C++/CUDA 層的 kernel
 *    fusion 與 KV cache 策略": KV managed as segments rather than one buffer);
 *    here a segment is a 256-token block found through a per-sequence block
 *    table, in a pool of fixed capacity (--kv-capacity 184320, page "3090 单卡跑
 *    Qwen3.8-27B", section 一.3).
 *  - Attention is textbook softmax attention, computed in fp64 over the exactly
 *    dequantised keys and values: k_hat = code * scale is exact in fp32 and
 *    fp64 (at most 7 + 11 significant bits).  Query j of an n_q-token step
 *    (MTP verification, --spec mtp --draft-tokens 3, same section) sits at
 *    position L - n_q + j and, when causal, sees keys 0 .. L - n_q + j.
 *  - Query head h uses kv-head h / (H_q / H_kv) (grouped-query attention).
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fopenmp -shared -fPIC
 * (no contraction into FMA, IEEE division, round-to-nearest-even mode).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define NFREF_BLOCK 256

/* ------------------------------------------------------------------ */
/* IEEE binary16 / bfloat16 conversions written from the definitions. */
/* ------------------------------------------------------------------ */

/* Round a finite, non-negative double a to the grid of a binary format with
 * `p` significand bits (including the hidden bit) and minimum normal exponent
 * `emin` (subnormal spacing 2^(emin - p + 1)).  Round half to even.  The
 * division by a power of two and the product are exact. */
static double round_to_grid(double a, int p, int emin)
{
    if (a == 0.0)
        return 0.0;
    int e;
    frexp(a, &e);            /* a in [2^(e-1), 2^e) */
    int E = e - 1;
    if (E < emin)
        E = emin;            /* subnormal range: fixed spacing */
    double ulp = ldexp(1.0, E - (p - 1));
    return nearbyint(a / ulp) * ulp;  /* default rounding mode: nearest-even */
}

/* fp32 -> fp16, round half to even, saturating at +-65504. */
uint16_t nfref_f32_to_f16(float xf)
{
    double x = (double)xf;
    uint16_t sign = signbit(xf) ? 0x8000u : 0u;
    double r = round_to_grid(fabs(x), 11, -14);
    if (r > 65504.0)
        r = 65504.0;
    if (r == 0.0)
        return sign;
    if (r < ldexp(1.0, -14))  /* subnormal: r = m * 2^-24 */
        return (uint16_t)(sign | (uint16_t)(r / ldexp(1.0, -24)));
    int e;
    frexp(r, &e);
    int E = e - 1;
    uint16_t mant = (uint16_t)(r / ldexp(1.0, E - 10) - 1024.0);
    return (uint16_t)(sign | (uint16_t)((E + 15) << 10) | mant);
}

float nfref_f16_to_f32(uint16_t h)
{
    int s = h >> 15, E = (h >> 10) & 31, m = h & 1023;
    double v;
    if (E == 0)
        v = ldexp((double)m, -24);
    else if (E == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), E - 25);
    return (float)(s ? -v : v);
}

/* fp32 -> bfloat16 (8 significand bits, fp32 exponent range), round half to
 * even.  Finite inputs whose rounding overflows are out of contract. */
uint16_t nfref_f32_to_bf16(float xf)
{
    uint16_t sign = signbit(xf) ? 0x8000u : 0u;
    double r = round_to_grid(fabs((double)xf), 8, -126);
    if (r == 0.0)
        return sign;
    if (r < ldexp(1.0, -126))
        return (uint16_t)(sign | (uint16_t)(r / ldexp(1.0, -133)));
    int e;
    frexp(r, &e);
    int E = e - 1;
    uint16_t mant = (uint16_t)(r / ldexp(1.0, E - 7) - 128.0);
    return (uint16_t)(sign | (uint16_t)((E + 127) << 7) | mant);
}

float nfref_bf16_to_f32(uint16_t h)
{
    int s = h >> 15, E = (h >> 7) & 255, m = h & 127;
    double v;
    if (E == 0)
        v = ldexp((double)m, -133);
    else if (E == 255)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(128 + m), E - 134);
    return (float)(s ? -v : v);
}

/* Array forms of the four conversions (for the tests). */
void nfref_f32_to_f16_n(const float *x, uint16_t *y, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        y[i] = nfref_f32_to_f16(x[i]);
}
void nfref_f16_to_f32_n(const uint16_t *x, float *y, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        y[i] = nfref_f16_to_f32(x[i]);
}
void nfref_f32_to_bf16_n(const float *x, uint16_t *y, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        y[i] = nfref_f32_to_bf16(x[i]);
}
void nfref_bf16_to_f32_n(const uint16_t *x, float *y, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        y[i] = nfref_bf16_to_f32(x[i]);
}

/* ------------------------------------------------------------------ */
/* K8 / V4 quantisation of one vector.                                 */
/* ------------------------------------------------------------------ */

/* Symmetric quantisation of n values with one scale absmax/qmax.  Returns the
 * fp16 scale bits and writes integer codes in [-qmax, qmax]. */
static uint16_t quant_symmetric(const float *x, int n, float qmax, int *codes)
{
    float a = 0.0f;
    for (int c = 0; c < n; ++c) {
        float v = fabsf(x[c]);
        if (v > a)
            a = v;
    }
    float s32 = a / qmax;                 /* fp32 division, round-to-nearest */
    uint16_t s16 = nfref_f32_to_f16(s32); /* fp16 round-half-even, saturating */
    float sigma = nfref_f16_to_f32(s16);  /* the stored scale, as a float */
    for (int c = 0; c < n; ++c) {
        if (sigma == 0.0f) {
            codes[c] = 0;
            continue;
        }
        float t = x[c] / sigma;           /* fp32 division by the stored scale */
        float r = nearbyintf(t);          /* round half to even */
        if (r > qmax)
            r = qmax;
        if (r < -qmax)
            r = -qmax;
        codes[c] = (int)r;
    }
    return s16;
}

/* ------------------------------------------------------------------ */
/* fp8 e4m3 (OCP "E4M3FN": 1 sign, 4 exponent bits with bias 7, 3      */
/* mantissa bits; subnormals m * 2^-9; no infinities; 0x7F / 0xFF NaN; */
/* largest finite 448), written from that definition.                 */
/* ------------------------------------------------------------------ */

/* fp32 -> e4m3, round half to even, saturating at +-448 (values beyond the
 * largest finite one become it), the sign kept for zero results. */
uint8_t nfref_e4m3_encode(float t)
{
    uint8_t sign = signbit(t) ? 0x80 : 0x00;
    double a = fabs((double)t);
    if (a > 448.0)
        a = 448.0;
    double v = round_to_grid(a, 4, -6);  /* 4 significant bits, emin = -6 */
    if (v == 0.0)
        return sign;
    int e;
    frexp(v, &e);
    int E = e - 1;                        /* v in [2^E, 2^(E+1)) */
    if (E < -6)
        return (uint8_t)(sign | (uint8_t)(v / ldexp(1.0, -9)));
    return (uint8_t)(sign | (uint8_t)(((E + 7) << 3) | (int)(v / ldexp(1.0, E - 3) - 8.0)));
}

double nfref_e4m3_decode(uint8_t b)
{
    if ((b & 0x7F) == 0x7F)
        return NAN;
    int E = (b >> 3) & 15, m = b & 7;
    double v = E == 0 ? ldexp((double)m, -9) : ldexp((double)(8 + m), E - 10);
    return (b & 0x80) ? -v : v;
}

void nfref_e4m3_encode_n(const float *x, uint8_t *y, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        y[i] = nfref_e4m3_encode(x[i]);
}
void nfref_e4m3_decode_n(const uint8_t *x, double *y, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        y[i] = nfref_e4m3_decode(x[i]);
}

/* fp8 KV: d values -> one fp16 scale absmax/448 and d e4m3 codes of
 * x / scale (fp32 division by the stored scale); all codes 0 when the scale
 * is 0. */
void nfref_quant_f8(const float *x, int d, uint16_t *scale, uint8_t *codes)
{
    float a = 0.0f;
    for (int c = 0; c < d; ++c) {
        float v = fabsf(x[c]);
        if (v > a)
            a = v;
    }
    float s32 = a / 448.0f;
    uint16_t s16 = nfref_f32_to_f16(s32);
    float sigma = nfref_f16_to_f32(s16);
    for (int c = 0; c < d; ++c)
        codes[c] = sigma == 0.0f ? 0 : nfref_e4m3_encode(x[c] / sigma);
    *scale = s16;
}

/* K: d values -> one fp16 scale and d int8 codes. */
void nfref_quant_k(const float *x, int d, uint16_t *scale, int8_t *codes)
{
    int *tmp = (int *)malloc(sizeof(int) * (size_t)d);
    *scale = quant_symmetric(x, d, 127.0f, tmp);
    for (int c = 0; c < d; ++c)
        codes[c] = (int8_t)tmp[c];
    free(tmp);
}

/* V: d values -> d/group fp16 scales and d/2 bytes of packed nibbles.
 * Byte j holds channel 2j in bits 0..3 and channel 2j+1 in bits 4..7. */
void nfref_quant_v(const float *x, int d, int group, uint16_t *scales, uint8_t *packed)
{
    int *codes = (int *)malloc(sizeof(int) * (size_t)d);
    for (int g = 0; g < d / group; ++g)
        scales[g] = quant_symmetric(x + g * group, group, 7.0f, codes + g * group);
    for (int j = 0; j < d / 2; ++j)
        packed[j] = (uint8_t)((codes[2 * j] & 0xF) | ((codes[2 * j + 1] & 0xF) << 4));
    free(codes);
}

/* ------------------------------------------------------------------ */
/* Format 4 ("RK4V4-E8"): 4-bit codes, power-of-two scale per 32 ch.  */
/* ------------------------------------------------------------------ */

/* The exponent e of the group scale 2^e: the smallest integer with
 * 2^e >= s, clamped to [-126, 127].  frexp writes s = m * 2^E with
 * 0.5 <= m < 1, so 2^(E - 1) <= s < 2^E, and s is itself a power of two
 * exactly when m == 0.5. */
int nfref_e8_exponent(float s)
{
    if (!(s > 0.0f))
        return -126;
    int E;
    double m = frexp((double)s, &E);
    int e = (m == 0.5) ? E - 1 : E;
    if (e < -126)
        e = -126;
    if (e > 127)
        e = 127;
    return e;
}

/* d values -> d/32 scale bytes (e + 127) and d/2 bytes of packed nibbles
 * (channel 2j in bits 0..3 of byte j, channel 2j+1 in bits 4..7). */
void nfref_quant_e8(const float *x, int d, uint8_t *scales, uint8_t *packed)
{
    int *codes = (int *)malloc(sizeof(int) * (size_t)d);
    for (int g = 0; g < d / 32; ++g) {
        const float *xg = x + g * 32;
        float a = 0.0f;
        for (int c = 0; c < 32; ++c) {
            float v = fabsf(xg[c]);
            if (v > a)
                a = v;
        }
        float s = a / 7.0f;                      /* fp32 division, round-to-nearest */
        int e = nfref_e8_exponent(s);
        float scale = ldexpf(1.0f, e);           /* 2^e, a normal fp32 number */
        for (int c = 0; c < 32; ++c) {
            float r = nearbyintf(xg[c] / scale); /* exact division, round half to even */
            if (r > 7.0f)
                r = 7.0f;
            if (r < -7.0f)
                r = -7.0f;
            codes[g * 32 + c] = (int)r;
        }
        scales[g] = (uint8_t)(e + 127);
    }
    for (int j = 0; j < d / 2; ++j)
        packed[j] = (uint8_t)((codes[2 * j] & 0xF) | ((codes[2 * j + 1] & 0xF) << 4));
    free(codes);
}

/* ------------------------------------------------------------------ */
/* Pool layout.                                                        */
/* ------------------------------------------------------------------ */
/*
 * One layer's pool, fmt 0 (K8V4), with H kv-heads and d = 128 channels:
 *   k_plane  int8   [num_blocks][H][256][d]
 *   k_scale  fp16   [num_blocks][H][256]
 *   v_plane  uint8  [num_blocks][H][256][d/2]
 *   v_scale  fp16   [num_blocks][H][256][d/32]
 * fmt 1 (BF16 cache): k_plane, v_plane bf16 [num_blocks][H][256][d]; no scales.
 * fmt 2 (K8V8, int8 KV): k_plane, v_plane int8 [num_blocks][H][256][d]; k_scale,
 *   v_scale fp16 [num_blocks][H][256]; V quantised by the K rule (absmax/127
 *   per token and kv-head).
 * fmt 3 (fp8 KV): k_plane, v_plane e4m3 bytes [num_blocks][H][256][d]; k_scale,
 *   v_scale fp16 [num_blocks][H][256] (absmax/448 per token and kv-head).
 * fmt 4 ("RK4V4-E8"): k_plane, v_plane uint8 nibbles [num_blocks][H][256][d/2];
 *   k_scale, v_scale uint8 exponent bytes [num_blocks][H][256][d/32] (the
 *   scale arguments point at bytes for this format).
 * Token position p of sequence b lives in block block_table[b][p / 256],
 * slot p % 256.
 */

static size_t slot_index(int32_t blk, int H, int h, int slot)
{
    return ((size_t)blk * (size_t)H + (size_t)h) * NFREF_BLOCK + (size_t)slot;
}

/* Dequantised key / value channel c of the token at pool slot `si`. */
/* Channel c of the packed nibbles of the token at slot si, as an integer. */
static int nibble_code(const void *plane, size_t si, int d, int c)
{
    uint8_t byte = ((const uint8_t *)plane)[si * (size_t)(d / 2) + (size_t)(c / 2)];
    int nib = (c & 1) ? (byte >> 4) : (byte & 0xF);
    return nib >= 8 ? nib - 16 : nib;
}

/* Format 4: code * 2^(byte - 127) for channel c. */
static double e8_hat(const void *plane, const uint16_t *scale, size_t si, int d, int c)
{
    uint8_t byte = ((const uint8_t *)scale)[si * (size_t)(d / 32) + (size_t)(c / 32)];
    return ldexp((double)nibble_code(plane, si, d, c), (int)byte - 127);
}

static double k_hat(int fmt, const void *k_plane, const uint16_t *k_scale, size_t si, int d, int c)
{
    if (fmt == 4)
        return e8_hat(k_plane, k_scale, si, d, c);
    if (fmt == 1)
        return (double)nfref_bf16_to_f32(((const uint16_t *)k_plane)[si * d + c]);
    if (fmt == 3)
        return nfref_e4m3_decode(((const uint8_t *)k_plane)[si * d + c]) * (double)nfref_f16_to_f32(k_scale[si]);
    double code = (double)((const int8_t *)k_plane)[si * d + c];
    return code * (double)nfref_f16_to_f32(k_scale[si]);
}

static double v_hat(int fmt, const void *v_plane, const uint16_t *v_scale, size_t si, int d, int c)
{
    if (fmt == 4)
        return e8_hat(v_plane, v_scale, si, d, c);
    if (fmt == 1)
        return (double)nfref_bf16_to_f32(((const uint16_t *)v_plane)[si * d + c]);
    if (fmt == 2)
        return (double)((const int8_t *)v_plane)[si * d + c] * (double)nfref_f16_to_f32(v_scale[si]);
    if (fmt == 3)
        return nfref_e4m3_decode(((const uint8_t *)v_plane)[si * d + c]) * (double)nfref_f16_to_f32(v_scale[si]);
    uint8_t byte = ((const uint8_t *)v_plane)[si * (size_t)(d / 2) + (size_t)(c / 2)];
    int nib = (c & 1) ? (byte >> 4) : (byte & 0xF);
    int code = nib >= 8 ? nib - 16 : nib;
    return (double)code * (double)nfref_f16_to_f32(v_scale[si * (size_t)(d / 32) + (size_t)(c / 32)]);
}

/* ------------------------------------------------------------------ */
/* Append: quantise new tokens and place them in the pool.             */
/* ------------------------------------------------------------------ */
/*
 * k_new, v_new: fp32 values [batch][n_new][H][d] (a bf16 input is passed here
 * already widened to fp32, which is exact).  Token i of sequence b goes to
 * position seqlens_before[b] + i.  Returns 0, or -1 if a position falls
 * outside the block table or a block id outside the pool (nothing is written
 * for that token).
 */
int nfref_append(int fmt, int num_blocks, int H, int d,
                 void *k_plane, uint16_t *k_scale, void *v_plane, uint16_t *v_scale,
                 const float *k_new, const float *v_new, int batch, int n_new,
                 const int32_t *block_table, int max_blocks, const int32_t *seqlens_before)
{
    int status = 0;
    /* Tokens of one (sequence, kv-head) pair are taken in order; different
     * pairs write disjoint slots (unless two sequences' tables name the same
     * block, which is outside the contract), so the pairs may run in parallel
     * without changing any byte of the result. */
#pragma omp parallel for collapse(2) schedule(dynamic, 1) reduction(min : status) if ((int64_t)batch * n_new * H > 65536)
    for (int b = 0; b < batch; ++b)
        for (int h = 0; h < H; ++h)
            for (int i = 0; i < n_new; ++i) {
                int pos = seqlens_before[b] + i;
                int bi = pos / NFREF_BLOCK;
                if (pos < 0 || bi >= max_blocks) {
                    status = -1;
                    continue;
                }
                int32_t blk = block_table[(size_t)b * max_blocks + bi];
                if (blk < 0 || blk >= num_blocks) {
                    status = -1;
                    continue;
                }
                size_t si = slot_index(blk, H, h, pos % NFREF_BLOCK);
                const float *kx = k_new + (((size_t)b * n_new + i) * H + h) * d;
                const float *vx = v_new + (((size_t)b * n_new + i) * H + h) * d;
                if (fmt == 1) {
                    for (int c = 0; c < d; ++c) {
                        ((uint16_t *)k_plane)[si * d + c] = nfref_f32_to_bf16(kx[c]);
                        ((uint16_t *)v_plane)[si * d + c] = nfref_f32_to_bf16(vx[c]);
                    }
                } else if (fmt == 2) {
                    nfref_quant_k(kx, d, &k_scale[si], (int8_t *)k_plane + si * d);
                    nfref_quant_k(vx, d, &v_scale[si], (int8_t *)v_plane + si * d);
                } else if (fmt == 3) {
                    nfref_quant_f8(kx, d, &k_scale[si], (uint8_t *)k_plane + si * d);
                    nfref_quant_f8(vx, d, &v_scale[si], (uint8_t *)v_plane + si * d);
                } else if (fmt == 4) {
                    nfref_quant_e8(kx, d, (uint8_t *)k_scale + si * (size_t)(d / 32),
                                   (uint8_t *)k_plane + si * (size_t)(d / 2));
                    nfref_quant_e8(vx, d, (uint8_t *)v_scale + si * (size_t)(d / 32),
                                   (uint8_t *)v_plane + si * (size_t)(d / 2));
                } else {
                    nfref_quant_k(kx, d, &k_scale[si], (int8_t *)k_plane + si * d);
                    nfref_quant_v(vx, d, 32, &v_scale[si * (size_t)(d / 32)],
                                  (uint8_t *)v_plane + si * (size_t)(d / 2));
                }
            }
    return status;
}

/* ------------------------------------------------------------------ */
/* Attention.                                                          */
/* ------------------------------------------------------------------ */

/* One query row against keys [k_begin, k_end) of one sequence and kv-head.
 * o = sum_t w_t v_t / sum_t w_t, w_t = exp(s_t - max s), s_t = scale * q . k_t,
 * lse = max s + log(sum_t w_t).  An empty range gives o = 0, lse = -inf. */
void nfref_attn_row(int fmt, int H, int d,
                    const void *k_plane, const uint16_t *k_scale,
                    const void *v_plane, const uint16_t *v_scale,
                    const int32_t *bt_row, int k_begin, int k_end,
                    const double *q, int kvh, double scale, double *o, double *lse)
{
    for (int c = 0; c < d; ++c)
        o[c] = 0.0;
    if (k_end <= k_begin) {
        *lse = -INFINITY;
        return;
    }
    int n = k_end - k_begin;
    double *s = (double *)malloc(sizeof(double) * (size_t)n);
    double m = -INFINITY;
    for (int t = 0; t < n; ++t) {
        int p = k_begin + t;
        size_t si = slot_index(bt_row[p / NFREF_BLOCK], H, kvh, p % NFREF_BLOCK);
        double dot = 0.0;
        for (int c = 0; c < d; ++c)
            dot += q[c] * k_hat(fmt, k_plane, k_scale, si, d, c);
        s[t] = scale * dot;
        if (s[t] > m)
            m = s[t];
    }
    double l = 0.0;
    for (int t = 0; t < n; ++t) {
        int p = k_begin + t;
        size_t si = slot_index(bt_row[p / NFREF_BLOCK], H, kvh, p % NFREF_BLOCK);
        double w = exp(s[t] - m);
        l += w;
        for (int c = 0; c < d; ++c)
            o[c] += w * v_hat(fmt, v_plane, v_scale, si, d, c);
    }
    for (int c = 0; c < d; ++c)
        o[c] /= l;
    *lse = m + log(l);
    free(s);
}

/* Decode attention for every (sequence b, query j, query head h) row, or for
 * the listed rows only (row id = (b * n_q + j) * H_q + h; rows == NULL means
 * all).  q: fp64 [batch][n_q][H_q][d]; out: [n_rows][d]; out_lse: [n_rows].
 * The softmax scale is the fp32 value given, used exactly.
 * Returns 0, or -1 if some L_b < n_q (no position for the queries). */
int nfref_decode_attn(int fmt, int H_kv, int d,
                      const void *k_plane, const uint16_t *k_scale,
                      const void *v_plane, const uint16_t *v_scale,
                      const double *q, int batch, int n_q, int H_q,
                      const int32_t *block_table, int max_blocks, const int32_t *seqlens,
                      float softmax_scale, int causal,
                      const int64_t *rows, int64_t n_rows,
                      double *out, double *out_lse, int nthreads)
{
    int G = H_q / H_kv;
    int64_t total = rows ? n_rows : (int64_t)batch * n_q * H_q;
    int status = 0;
    for (int b = 0; b < batch; ++b)
        if (seqlens[b] < n_q)
            status = -1;
    if (status)
        return status;
    if (nthreads < 1)
        nthreads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (int64_t k = 0; k < total; ++k) {
        int64_t rid = rows ? rows[k] : k;
        int h = (int)(rid % H_q);
        int j = (int)((rid / H_q) % n_q);
        int b = (int)(rid / ((int64_t)H_q * n_q));
        int L = seqlens[b];
        int k_end = causal ? (L - n_q + j + 1) : L;
        nfref_attn_row(fmt, H_kv, d, k_plane, k_scale, v_plane, v_scale,
                       block_table + (size_t)b * max_blocks, 0, k_end,
                       q + (size_t)rid * d, h / G, (double)softmax_scale,
                       out + (size_t)k * d, out_lse + k);
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Log-sum-exp merge of split results.                                 */
/* ------------------------------------------------------------------ */
/* part_o [n_splits][rows][d], part_lse [n_splits][rows].  A split whose lse is
 * -inf (it saw no key) is skipped; a row with no finite split gives o = 0,
 * lse = -inf.  lse = log sum_j exp(lse_j), o = sum_j exp(lse_j - lse) o_j. */
void nfref_combine(const double *part_o, const double *part_lse, int n_splits, int rows, int d,
                   double *out, double *out_lse)
{
    for (int r = 0; r < rows; ++r) {
        double m = -INFINITY;
        for (int j = 0; j < n_splits; ++j) {
            double v = part_lse[(size_t)j * rows + r];
            if (v > m)
                m = v;
        }
        for (int c = 0; c < d; ++c)
            out[(size_t)r * d + c] = 0.0;
        if (m == -INFINITY) {
            out_lse[r] = -INFINITY;
            continue;
        }
        double l = 0.0;
        for (int j = 0; j < n_splits; ++j) {
            double v = part_lse[(size_t)j * rows + r];
            if (v != -INFINITY)
                l += exp(v - m);
        }
        double lse = m + log(l);
        out_lse[r] = lse;
        for (int j = 0; j < n_splits; ++j) {
            double v = part_lse[(size_t)j * rows + r];
            if (v == -INFINITY)
                continue;
            double w = exp(v - lse);
            for (int c = 0; c < d; ++c)
                out[(size_t)r * d + c] += w * part_o[((size_t)j * rows + r) * d + c];
        }
    }
}
