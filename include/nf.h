/*
 * nf.h -- C ABI of the B200 (sm_100a) library for single-request, long-context
 * decode attention over a K8/V4-quantised, segmented KV cache.
 *
 * Sources of the operations (pages of the NInfer write-ups; no page gives
 * code or a kernel interface, so the interface below is this library's own):
 *  - KV dtype "rk8v4 (K8/V4)": int8 keys, 4-bit values.  Page "3090 单卡跑
 *    Qwen3.8-27B：NInfer 上机实测（180K 上下文 / C2 并发 / 4bit KV）", section
 *    一.3 启动 (--kv-dtype rk8v4; int8 KV reaches 160K where rk8v4 reaches 180K
 *    at equal speed).  The pages do not define the bits; this header does (see
 *    nf_kv_layer).  The int8 and fp8 KV dtypes of the same section
 *    (--kv-dtype int8 / fp8) are NF_KV_K8V8 and NF_KV_F8.
 *  - A segmented KV cache in a pool of fixed capacity, one segment streamed
 *    at a time, decode tuned for one long request.  Page "標籤: vLLM", section
 *    2 "C++/CUDA 層的 kernel fusion 與 KV cache 策略"; page "3090 单卡跑
 *    Qwen3.8-27B", section 一.3 (--kv-capacity 184320, --max-concurrency 2).
 *  - MTP draft verification (1 + 3 query tokens with a causal mask among
 *    them).  Page "3090 单卡跑 Qwen3.8-27B", section 一.3 (--spec mtp
 *    --draft-tokens 3).
 *  - Decode is HBM-bandwidth bound and KV bytes per token drive long-context
 *    decode.  Page "3090 单卡跑 Qwen3.8-27B", section 二 测评 and the replies.
 *  - Refuse rather than overrun a memory budget.  Same page, section 一.3
 *    (the engine refuses to start over budget); here: every call validates its
 *    arguments on the host and returns a status before launching anything.
 *
 * Conventions for every call:
 *  - The caller owns every buffer (pool planes, block tables, lengths, q, out,
 *    workspace).  The library never allocates, frees or synchronises; all work
 *    is enqueued on `stream` (NULL = the legacy default stream) of the current
 *    CUDA device, and all pointers except `kv` itself are device pointers.
 *  - Arguments are validated on the host first; on any error nothing is
 *    launched and the status says why (nf_last_error() gives a message).
 *  - A launch failure or an earlier asynchronous CUDA error is returned as
 *    NF_ERR_CUDA.
 *  - Data-dependent problems that only the device sees (a block id outside the
 *    pool, a length outside [n_q, max_seqlen]) never trap: the kernel skips the
 *    offending work and records a code that nf_get_device_error() returns.
 *  - Calls keep no state between them and are safe to call from several host
 *    threads on different streams.
 */
#ifndef NF_H_
#define NF_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* The same type as cudaStream_t. */
typedef struct CUstream_st *nf_stream_t;

typedef int32_t nf_status;
#define NF_OK 0
#define NF_ERR_INVALID_ARG 1  /* null pointer, negative size, inconsistent shape */
#define NF_ERR_UNSUPPORTED 2  /* head_dim != 128, block_size != 256, v_group != 32, dtype */
#define NF_ERR_WORKSPACE 3    /* workspace smaller than nf_decode_attn_workspace_size() */
#define NF_ERR_CUDA 4         /* a CUDA launch or earlier asynchronous error */
#define NF_ERR_DEVICE_CHECK 5 /* returned by nf_get_device_error() when a code is set */

/* Device error codes recorded by the kernels (nf_get_device_error). */
#define NF_DEVERR_NONE 0
#define NF_DEVERR_BLOCK_ID 1  /* a block-table entry outside [0, num_blocks) */
#define NF_DEVERR_TABLE 2     /* a position whose block index is >= max_blocks */
#define NF_DEVERR_SEQLEN 3    /* seqlens[b] < n_q or > max_seqlen */
#define NF_DEVERR_TIMEOUT 4   /* a bounded wait inside a kernel gave up (the kernel returned) */
#define NF_DEVERR_INTERNAL 5  /* a launch-time invariant of the kernel failed (e.g. shared-memory
                                 alignment); the call did no work */
#define NF_DEVERR_RANGE 6     /* nf_prefill_attn: a K or V scale whose dequantised codes leave the
                                 fp16 range the kernel computes in (the results are not finite) */

/* Element types. */
#define NF_F32 0
#define NF_BF16 1
#define NF_F16 2

/* KV cache formats. */
#define NF_KV_K8V4 0 /* the rk8v4 format defined below */
#define NF_KV_BF16 1 /* unquantised bf16 K and V (for byte-count comparison) */
#define NF_KV_K8V8 2 /* the int8 KV dtype defined below (K and V both int8) */
#define NF_KV_F8 3   /* the fp8 KV dtype defined below (K and V both e4m3) */
#define NF_KV_K4V4 4 /* the RK4V4-E8 reading defined below (K and V both 4-bit) */

/*
 * One layer's view of the caller-owned KV pool.
 *
 * The pool holds `num_blocks` segments of `block_size` = 256 token slots for
 * each of `num_kv_heads` heads; head_dim is 128.  Token position p of
 * sequence b lives in block block_table[b * max_blocks + p / 256], slot p % 256.
 *
 * fmt NF_KV_K8V4 ("rk8v4"; 202 bytes per token per kv-head):
 *   k_codes  int8    [num_blocks][num_kv_heads][256][128]  K codes in [-127, 127]
 *   k_scales fp16    [num_blocks][num_kv_heads][256]       one K scale per token
 *   v_codes  uint8   [num_blocks][num_kv_heads][256][64]   V codes in [-7, 7] as
 *            two's-complement nibbles; byte j holds channel 2j in bits 0..3 and
 *            channel 2j+1 in bits 4..7
 *   v_scales fp16    [num_blocks][num_kv_heads][256][4]    one V scale per 32
 *            channels (v_group = 32)
 *   Quantisation of a vector x (128 K channels, or one 32-channel V group):
 *     scale = fp16(fp32(max|x| / Q)) rounded half to even, saturated at 65504,
 *             Q = 127 for K and 7 for V;
 *     code  = clamp(round_half_even(fp32(x / float(scale))), -Q, Q), or 0 when
 *             scale is 0.
 *   Dequantised value = code * scale (exact in fp32).
 * fmt NF_KV_K8V8 (the pages' int8 KV dtype; 260 bytes per token per kv-head):
 *   k_codes  int8    [num_blocks][num_kv_heads][256][128]  K codes in [-127, 127]
 *   k_scales fp16    [num_blocks][num_kv_heads][256]       one K scale per token
 *   v_codes  int8    [num_blocks][num_kv_heads][256][128]  V codes in [-127, 127]
 *   v_scales fp16    [num_blocks][num_kv_heads][256]       one V scale per token
 *   K and V are both quantised by the K rule above (Q = 127, one scale per
 *   token and kv-head); v_group is ignored.
 * fmt NF_KV_F8 (the pages' fp8 KV dtype; 260 bytes per token per kv-head):
 *   k_codes, v_codes uint8 [num_blocks][num_kv_heads][256][128]  fp8 e4m3
 *            codes (OCP E4M3FN: bias 7, 3 mantissa bits, largest finite 448)
 *   k_scales, v_scales fp16 [num_blocks][num_kv_heads][256]  one scale per token
 *   scale = fp16(fp32(max|x| / 448)) as above; code = e4m3(fp32(x / float(scale)))
 *   rounded half to even and saturated at +-448 (a zero result keeps the sign
 *   of x), or 0x00 when scale is 0.  Dequantised value = e4m3 value * scale.
 * fmt NF_KV_K4V4 (the "RK4V4-E8" KV quantisation of page "影片筆記：NInfer +
 *   千问3.8 27b = 1.5倍速@256K上下文(单张4090 24GB)", section 三, which gives no bit
 *   format; this is the reading defined here; 136 bytes per token per kv-head):
 *   k_codes  uint8 [num_blocks][num_kv_heads][256][64]  K codes in [-7, 7] as
 *            nibbles, packed as the K8/V4 V codes
 *   k_scales uint8 [num_blocks][num_kv_heads][256][4]   one scale byte per 32 channels
 *   v_codes, v_scales: the same for V
 *   Quantisation of one 32-channel group x (K or V):
 *     e = the smallest integer with 2^e >= fp32(max|x| / 7), clamped to
 *         [-126, 127]; stored as the byte e + 127 (an 8-bit exponent);
 *     code = clamp(round_half_even(fp32(x / 2^e)), -7, 7).
 *   Dequantised value = code * 2^e (exact).  The decoder reads scale bytes 1 ..
 *   254 (the quantiser writes no other); within one sequence the V scales
 *   should span fewer than 2^100 (their exponents are folded into fp32 sums).
 * fmt NF_KV_BF16 (512 bytes per token per kv-head):
 *   k_codes  bf16 [num_blocks][num_kv_heads][256][128]  (keys)
 *   v_codes  bf16 [num_blocks][num_kv_heads][256][128]  (values)
 *   k_scales, v_scales unused (may be NULL); v_group ignored.
 * Every plane must be 16-byte aligned.
 */
typedef struct {
    int32_t fmt;          /* NF_KV_K8V4, NF_KV_K8V8, NF_KV_F8, NF_KV_K4V4 or NF_KV_BF16 */
    int32_t num_blocks;   /* pool capacity in blocks (>= 1) */
    int32_t block_size;   /* must be 256 */
    int32_t num_kv_heads; /* >= 1 */
    int32_t head_dim;     /* must be 128 */
    int32_t v_group;      /* must be 32 for NF_KV_K8V4 */
    void *k_codes;
    void *k_scales;
    void *v_codes;
    void *v_scales;
} nf_kv_layer;

/*
 * nf_kv_append_quant -- quantise new K/V tokens and write them into the pool.
 *
 * k_new, v_new: [batch][n_new][num_kv_heads][128] of in_dtype (NF_F32 or
 *   NF_BF16), contiguous.  Token i of sequence b is written at position
 *   seqlens_before[b] + i (seqlens_before: int32 [batch], device), through
 *   block_table (int32 [batch][max_blocks], device).  Slots not written keep
 *   their bytes.  The call does not advance any length: the caller does that
 *   once per step.  For NF_KV_BF16 pools the values are rounded to bf16
 *   (half to even) and stored.
 * A token whose block index is >= max_blocks or whose block id is outside the
 * pool is skipped and NF_DEVERR_TABLE / NF_DEVERR_BLOCK_ID is recorded.
 * batch * n_new == 0 launches nothing and returns NF_OK.
 */
nf_status nf_kv_append_quant(const nf_kv_layer *kv, const void *k_new, const void *v_new,
                             int32_t in_dtype, int32_t batch, int32_t n_new,
                             const int32_t *block_table, int32_t max_blocks,
                             const int32_t *seqlens_before, nf_stream_t stream);

/*
 * nf_decode_attn_workspace_size -- bytes of device workspace nf_decode_attn
 * needs for this shape on a device with `num_sms` streaming multiprocessors
 * (pass the device's count; nf_decode_attn uses the current device's).  The
 * workspace holds ticket counters (per (sequence, kv-head) and per split) and
 * the (o, lse) partials of the context splits.  Zero-fill it once before its first use
 * (e.g. cudaMemsetAsync); every call leaves it zero-filled where it must be
 * when its kernel completes, so it can be reused call after call on one
 * stream.  Returns 0 for an invalid or unsupported shape.
 */
size_t nf_decode_attn_workspace_size(int32_t batch, int32_t n_q, int32_t num_q_heads,
                                     int32_t num_kv_heads, int32_t max_seqlen, int32_t num_sms);

/*
 * nf_decode_attn -- split-K decode attention over the pool.
 *
 * For every sequence b < batch, query token j < n_q and query head h <
 * num_q_heads, with G = num_q_heads / num_kv_heads and L = seqlens[b] (keys in
 * the cache, including tokens appended for this step):
 *   query j sits at position P = L - n_q + j and sees keys t in [0, P] when
 *   causal != 0, else all t in [0, L);
 *   s_t = softmax_scale * (q[b][j][h] . k_hat_t) with k_hat of kv-head h / G;
 *   out[b][j][h] = sum_t exp(s_t - m) v_hat_t / sum_t exp(s_t - m);
 *   out_lse[b][j][h] = m + ln sum_t exp(s_t - m)   (natural log; m = max s_t).
 * q: [batch][n_q][num_q_heads][128] of q_dtype (NF_F32 or NF_BF16), device.
 * out: fp32 [batch][n_q][num_q_heads][128]; out_lse: fp32 [batch][n_q]
 *   [num_q_heads] or NULL.
 * seqlens: int32 [batch], device; each must lie in [n_q, max_seqlen], the host
 *   bound used to size the split plan (violations: NF_DEVERR_SEQLEN, and that
 *   sequence's rows come out as o = 0, lse = -inf).
 * block_table: int32 [batch][max_blocks], device; max_blocks >= ceil(max_seqlen
 *   / 256).  Only entries for positions < L are read.
 * workspace: device scratch of at least nf_decode_attn_workspace_size(...)
 *   bytes, 256-byte aligned, zero-filled before its first use (see above).
 *   Calls that share a workspace must not overlap on the GPU.
 * Supported: batch <= 256, (num_q_heads / num_kv_heads) * n_q <= 64; other
 *   shapes return NF_ERR_UNSUPPORTED.
 * Numerics (K8/V4): the K codes enter the integer tensor cores exactly and each
 *   query row as two int8 digits, q ~= s (d1 + d2 / 254) with s = max|q| / 127
 *   (error below 2^-16 max|q| per element); the V codes are exact in fp16 and
 *   each softmax weight times its V scale is rounded to fp16 before the
 *   tensor-core P.V product; scores, softmax statistics and accumulators are
 *   fp32.  (K8V8: the same, the int8 V codes exact in fp16 likewise.  fp8:
 *   the e4m3 codes are exact in fp16; S = Q . K^T uses fp16 products with each
 *   query row split as q = s (hi + lo), s = max|q|, hi and lo fp16.  bf16
 *   cache: bf16 products, the fp32 query and the weights split into bf16 high
 *   and low parts.)  With 9 to 32 query rows per kv-head, K8/V4, K8V8 and fp8
 *   run on the tcgen05 tensor cores instead: the same two-digit Q . K for
 *   int8 K; for e4m3 K, the query row scaled to max|q| = 1 in three e4m3 parts
 *   (q ~= s (p1 + p2 / 16 + p3 / 256), each part the rounding of what the
 *   earlier ones leave, times 16) against the exact codes, in fp32; and P . V as
 *   V' = code x scale x 2^(15 - E) times P' = weight x 2^(E - 15), each rounded
 *   to fp16 once (E: the largest exponent field of the key's V scales).
 * Launch: the kernel is launched with programmatic dependent launch, so it may
 *   start while the previous kernel on `stream` finishes; it waits for that
 *   kernel before reading any argument (see nf_decode_attn_ex for a weaker
 *   wait).
 */
nf_status nf_decode_attn(const nf_kv_layer *kv, const void *q, int32_t q_dtype, int32_t batch,
                         int32_t n_q, int32_t num_q_heads, const int32_t *block_table,
                         int32_t max_blocks, const int32_t *seqlens, int32_t max_seqlen,
                         float softmax_scale, int32_t causal, float *out, float *out_lse,
                         void *workspace, size_t workspace_bytes, nf_stream_t stream);

/*
 * nf_decode_attn_ex -- nf_decode_attn with flags.
 *
 * NF_DECODE_EARLY_KV: start streaming the cache before the previous kernel on
 *   `stream` has finished.  The caller guarantees that the kernels still
 *   running when this call's kernel starts write neither seqlens, nor
 *   block_table, nor any pool row at a position < seqlens[b] - n_q (they may
 *   write the rows of the n_q newest positions, as nf_kv_append_quant does for
 *   the tokens of a decode or verification step).  The kernel then reads the
 *   lengths, the tables and the older rows at once, and waits for the previous
 *   kernel before it reads q or the newest rows and before it writes out,
 *   out_lse or the workspace.  This hides the start-up of each call behind the
 *   end of the previous one in a sequence of layers.  Without the guarantee
 *   the results are undefined; nf_decode_attn is this call with flags = 0.
 * Other bits must be zero (NF_ERR_INVALID_ARG).
 */
#define NF_DECODE_EARLY_KV 1u
nf_status nf_decode_attn_ex(const nf_kv_layer *kv, const void *q, int32_t q_dtype, int32_t batch,
                            int32_t n_q, int32_t num_q_heads, const int32_t *block_table,
                            int32_t max_blocks, const int32_t *seqlens, int32_t max_seqlen,
                            float softmax_scale, int32_t causal, uint32_t flags, float *out,
                            float *out_lse, void *workspace, size_t workspace_bytes, nf_stream_t stream);

/*
 * nf_decode_attn_noalloc -- nf_decode_attn for callers that cannot allocate
 * device memory when they call: for example a host engine that reserves its
 * whole memory budget at start-up and gives plug-in kernels no allocator, or
 * a latency-critical loop where cudaMalloc's implicit device synchronisation
 * is not acceptable.  The pages have no counterpart of this call; it exists
 * for such callers only.
 *
 * Same arguments and results as nf_decode_attn, minus the workspace.  The
 * split partials go to a scratch array of NF_NOALLOC_SCRATCH_BYTES that lives
 * in the library's device image: every GPU that loads libnf holds it until the
 * process exits.  The call allocates nothing (no cudaMalloc, no allocating
 * library routine).
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current) and caches it; make that
 *    first call before any stream capture on the device.  The cached address
 *    belongs to the device's primary context: do not reset the device
 *    (cudaDeviceReset) in a process that keeps calling this entry point.
 *  - Shapes whose nf_decode_attn_workspace_size() exceeds
 *    NF_NOALLOC_SCRATCH_BYTES are refused with NF_ERR_WORKSPACE.
 *  - All calls on a device share the one array and it keeps the last call's
 *    contents; each call first clears (cudaMemsetAsync on `stream`) the
 *    counters that must start at zero.  Calls that overlap on the GPU
 *    (concurrent streams, or other host threads) race on it: order them on
 *    one stream.
 */
#define NF_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)
nf_status nf_decode_attn_noalloc(const nf_kv_layer *kv, const void *q, int32_t q_dtype, int32_t batch,
                                 int32_t n_q, int32_t num_q_heads, const int32_t *block_table,
                                 int32_t max_blocks, const int32_t *seqlens, int32_t max_seqlen,
                                 float softmax_scale, int32_t causal, float *out, float *out_lse,
                                 nf_stream_t stream);

/*
 * nf_attn_combine -- log-sum-exp merge of split attention results (the
 * flash-decoding reduction; the pages do not describe it).
 *
 * part_o: fp32 [n_splits][rows][head_dim]; part_lse: fp32 [n_splits][rows]
 * (natural log).  For each row: lse = ln sum_j exp(part_lse[j]) and
 * out = sum_j exp(part_lse[j] - lse) part_o[j], skipping splits whose lse is
 * -inf (they saw no key); a row with no finite split gets out = 0, lse = -inf.
 * out: fp32 [rows][head_dim]; out_lse: fp32 [rows] or NULL.  head_dim must be a
 * multiple of 4 in [4, 1024].  rows == 0 launches nothing.
 */
nf_status nf_attn_combine(const float *part_o, const float *part_lse, int32_t n_splits,
                          int32_t rows, int32_t head_dim, float *out, float *out_lse,
                          nf_stream_t stream);

/*
 * nf_attn_combine_packed -- nf_attn_combine of splits stored packed, one slot
 * per split: parts is fp32 [n_splits][slot], slot = nf_attn_packed_slot_floats(
 * rows, head_dim) = rows * (head_dim + 1) rounded up to a multiple of 4, each
 * slot holding o [rows][head_dim] followed by lse [rows] (the layout the decode
 * kernel gives its own split partials).  A context-sharded decode writes each
 * rank's partial into one such slot (out = the slot, out_lse = slot + rows *
 * head_dim), exchanges the slots in one all-gather and merges them with this
 * call.  parts and out 16-byte aligned; other arguments and results as for
 * nf_attn_combine.
 */
size_t nf_attn_packed_slot_floats(int32_t rows, int32_t head_dim);
nf_status nf_attn_combine_packed(const float *parts, int32_t n_splits, int32_t rows, int32_t head_dim,
                                 float *out, float *out_lse, nf_stream_t stream);

/*
 * nf_prefill_attn -- chunked-prefill attention over a K8/V4 pool (page "3090
 * 单卡跑 Qwen3.8-27B：NInfer 上机实测", section 一.3: prompts are prefilled in
 * chunks of --prefill-chunk 1024 tokens; section 二: prefill runs on a
 * dequantise -> fp16 tensor-core path).
 *
 * The operation is nf_decode_attn's for a large n_q: query j of sequence b
 * sits at position L_b - n_q + j (the chunk's K/V already appended with
 * nf_kv_append_quant) and, with causal != 0, sees keys 0 .. L_b - n_q + j;
 * otherwise all L_b keys.  Arguments, layouts and outputs as for
 * nf_decode_attn, with these differences:
 *   kv->fmt must be NF_KV_K8V4 and q_dtype NF_BF16 (else NF_ERR_UNSUPPORTED);
 *   any n_q >= 1 and any GQA group; no workspace (nothing is split across
 *   CTAs); batch <= 65535, num_kv_heads <= 65535.
 *   The dequantised K and V values (code x scale) must lie inside the fp16
 *   range the kernel holds them in: K scales <= 515.5 (127 x 515.5 < 65504)
 *   and V scales <= 9352 (7 x 9352 < 65504), that is K and V inputs of
 *   magnitude below about 65500.  A larger scale of a key the call reads is
 *   recorded as NF_DEVERR_RANGE (and the affected outputs are not finite);
 *   nf_decode_attn has no such limit.
 * Numerics: each query row is scaled to max |q| = 1 and rounded to fp16 once;
 *   K and V are dequantised to fp16 (code x scale, one rounding each); the
 *   softmax weights are rounded to fp16; products accumulate in fp32 on the
 *   5th-generation tensor cores (tcgen05.mma kind::f16, M = 128).
 * Device errors: NF_DEVERR_SEQLEN (the sequence's rows come out o = 0,
 *   lse = -inf), NF_DEVERR_BLOCK_ID (that tile's keys read as zeros),
 *   NF_DEVERR_RANGE (see above).
 * Launch: programmatic dependent launch, as nf_decode_attn; the kernel waits
 *   for the previous kernel on `stream` before reading any argument.
 */
nf_status nf_prefill_attn(const nf_kv_layer *kv, const void *q, int32_t q_dtype, int32_t batch,
                          int32_t n_q, int32_t num_q_heads, const int32_t *block_table,
                          int32_t max_blocks, const int32_t *seqlens, int32_t max_seqlen,
                          float softmax_scale, int32_t causal, float *out, float *out_lse,
                          nf_stream_t stream);

/*
 * nf_get_device_error -- read and clear the device error code of the current
 * device (NF_DEVERR_*).  Synchronises with the device.  Returns NF_OK when no
 * code was set, NF_ERR_DEVICE_CHECK when one was (written to *code), or
 * NF_ERR_CUDA.
 */
nf_status nf_get_device_error(int32_t *code);

/* Static text for a status code. */
/*
 * nf_selftest_bounded_wait -- diagnostics: launch one thread that waits on an
 * mbarrier nothing ever arrives on, for at most limit_us microseconds (1 ..
 * 1000000), through the same bounded wait every wait of the decode kernel uses.
 * The wait gives up, records NF_DEVERR_TIMEOUT in the device error word and
 * the kernel returns; the context stays usable.  Read the word with
 * nf_get_device_error.  The pages have no counterpart: this checks the
 * library's stall detection without faulting or hanging the GPU.
 */
nf_status nf_selftest_bounded_wait(uint32_t limit_us, nf_stream_t stream);

const char *nf_status_string(nf_status status);

/* Message describing the last failing call on this host thread ("" if none). */
const char *nf_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* NF_H_ */
