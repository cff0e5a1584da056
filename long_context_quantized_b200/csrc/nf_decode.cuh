// nf_decode.cuh -- persistent split-K decode attention over the segmented
// K8/V4 (or int8, fp8 or bf16) KV pool, with the log-sum-exp combine fused in.
//
// The pages' engine streams the KV cache one segment at a time through the SM
// and tunes decode for a single long request (page "標籤: vLLM", section 2
// "C++/CUDA 層的 kernel fusion 與 KV cache 策略"); decode is HBM-bound and
// KV bytes per token drive it (page "3090 单卡跑 Qwen3.8-27B：NInfer 上机实测",
// section 二 and its replies).  The B200 form of that idea:
//
// Work: every (sequence b, kv-head h) is a segment of ceil(L_b / 32) chunks of
//   32 keys; the segments, each counted kSegPad chunks longer (the cost of a
//   piece's set-up and merge), form one list that the persistent grid (one
//   CTA per SM) cuts into equal contiguous ranges, read from the device-side
//   lengths -- ragged batches balance by keys, with no host read of the
//   lengths.  A CTA's range covers pieces of one or more segments; all G * n_q
//   query rows of a kv-head (GQA group x MTP queries) are served by the CTA
//   that streams the keys, so each byte is fetched from HBM once.
// Pipeline: a producer warp cuts each piece into stages of up to 256 keys
//   (128 for the int8 cache, 64 for bf16) inside one 256-key block and moves each stage's K
//   codes, V nibbles, K scales and V scales into a ring of shared-memory
//   buffers on the TMA engine (1-D bulk copies; the V nibbles as 2-D tiles
//   through a tensor map with the 64-byte swizzle, so that eight keys' rows
//   of one 16-byte column sit in eight different bank groups), completing on
//   an mbarrier.  Stages are large because a ring buffer turns over at a
//   roughly fixed rate per SM (about 2.7 stages per microsecond measured on
//   B200): bandwidth is stage bytes x that rate, so 32-52 KB stages keep it
//   above the HBM rate.  All consumer warps work on every stage -- each takes
//   units of 32 keys (16 for bf16) -- and release it on an "empty" mbarrier,
//   so stages retire in order.
// Math per 16-key m-tile, 8 query rows per warp (a second tile for 16 rows):
//   S = Q . K^T on the integer tensor cores (mma.sync m16n8k32 s8 x s8 -> s32)
//   straight from the int8 codes in shared memory.  Each query row is written
//   as two int8 digits, q ~= s (d1 + d2 / 254) with s = max|q| / 127 (error
//   below 2^-16 max|q| per element); A-fragment rows 0-7 hold the rows' high
//   digits and rows 8-15 their low digits, so one product gives both, and the
//   lane's K words land in B-fragment pairs as loaded.  The two int32 sums
//   are recombined in fp32 and scaled by the key's K scale.  (The bf16 cache
//   uses bf16 mma.sync the same way, the rows 8-15 holding the low half of an
//   fp32 query; the fp8 cache converts its e4m3 codes to fp16 with the
//   hardware conversion and uses fp16 mma.sync, the query row scaled to
//   max |q| = 1 and split into fp16 high and low parts.  The int8 and fp8 V
//   codes become fp16 pairs the same way, one V scale per key.)
//   O^T += V_codes^T . (P^T x sigma_V) (mma.sync m16n8k16 fp16, fp32
//   accumulate): the score fragment of S is already the B-fragment layout of
//   P^T; ldmatrix.trans hands each lane the nibbles of one channel for two
//   consecutive keys, a lop3 and one fp16 op turn a pair into exact fp16
//   codes -- already in A-fragment layout, with no transpose -- and, since
//   every 16-channel m-tile lies in one 32-channel scale group, the V scale of
//   (key, group) multiplies the weights (the B operand) instead of the values.
//   The running max of a row is only raised (and O rescaled) when a tile's
//   max exceeds it by more than 2^4, and the weights are taken relative to
//   max + 4, so they never exceed 1 and weight x scale stays inside fp16; the
//   cross-lane max is only reduced when some lane asks for that.
// Merge: at the end of each piece the consumer warps merge through shared
//   memory.  A segment owned by one CTA is written straight to out; otherwise
//   each piece writes an (o, lse) partial and takes a ticket of the segment's
//   counter (acquire-release); the CTA with the last ticket merges the
//   partials into out straight from L2 -- the weights of every (row, piece)
//   first, then each output item in piece order -- and resets the counter
//   (no CTA ever waits for another).  The CTAs take the ranges of the cut in
//   reverse order, so the CTA placed last (on the SM the previous kernel's
//   merging CTA leaves last) gets range 0, whose segment padding means fewer
//   keys.
// Every mbarrier wait is bounded (2 s); a timeout records NF_DEVERR_TIMEOUT
// and the kernel runs to its end without further waits.
#pragma once

#include <cuda.h>  // CUtensorMap (a plain struct; no driver call is made here)

#include "nf_common.cuh"

namespace nf {

constexpr int kChunk = 32;  // keys per unit of work balance
constexpr int kConsumerWarps = 8;
constexpr int kDecodeThreads = (kConsumerWarps + 1) * 32;
constexpr int kMaxBatch = 256;
constexpr int kMaxRows = 64;  // G * n_q per kv-head
constexpr int kMaxCtas = 160;  // grid size cap: a segment has at most this many pieces
// The running max of a row is raised when a tile's max exceeds it by more than
// kLazy (log2 units); weights are 2^(x - max - kLazy) <= 1.
constexpr float kLazy = 4.0f;
// A CTA whose range crosses into a new segment pays an extra piece set-up and
// merge (about 3.5-4.5 us measured: the piece's merge, its ticket and the
// stall of the stream meanwhile); each segment is counted kSegPad chunks (of about 0.15 us of
// streaming each) longer when the work is cut, so such CTAs get that many
// fewer keys.
constexpr int kSegPad = 32;

template <int FMT, int NT>
struct Stage;
template <int NT>
struct Stage<NF_KV_K8V4, NT> {
    static constexpr int kTok = 256;                  // keys per stage: one block
    static constexpr int kK = 0;                      // int8  [kTok][128]
    static constexpr int kV = kTok * 128;             // uint8 [kTok][64]
    static constexpr int kKs = kV + kTok * 64;        // fp16  [kTok]
    static constexpr int kVs = kKs + kTok * 2;        // fp16  [kTok][4]
    static constexpr int kBytesPerTok = 202;
    // 51712 bytes of data; buffers start on 1024-byte boundaries, which the
    // swizzled V tile (a 512-byte pattern) needs
    static constexpr int kStride = (kTok * kBytesPerTok + 1023) / 1024 * 1024;
    static constexpr int kStages = 3;
    static constexpr int kUnitTiles = NT == 1 ? 2 : 1;  // 16-key m-tiles per consumer work unit
};
// int8 KV (K8V8): 260 bytes per key; 128-key stages, so that four fit beside
// the merge buffer.  The V rows are 128 bytes, copied with the 128-byte swizzle.
template <int NT>
struct Stage<NF_KV_K8V8, NT> {
    static constexpr int kTok = 128;
    static constexpr int kK = 0;                      // int8 [kTok][128]
    static constexpr int kV = kTok * 128;             // int8 [kTok][128] (swizzled)
    static constexpr int kKs = kV + kTok * 128;       // fp16 [kTok]
    static constexpr int kVs = kKs + kTok * 2;        // fp16 [kTok]
    static constexpr int kBytesPerTok = 260;
    static constexpr int kStride = (kTok * kBytesPerTok + 1023) / 1024 * 1024;
    static constexpr int kStages = 4;
    static constexpr int kUnitTiles = 1;  // 8 units of 16 keys per stage: one per consumer warp
};
// RK4V4-E8: 136 bytes per key; K and V nibble rows of 64 bytes (both through
// tensor maps with the 64-byte swizzle), one exponent byte per 32 channels.
template <int NT>
struct Stage<NF_KV_K4V4, NT> {
    static constexpr int kTok = 256;
    static constexpr int kK = 0;                      // uint8 [kTok][64] (swizzled)
    static constexpr int kV = kTok * 64;              // uint8 [kTok][64] (swizzled)
    static constexpr int kKs = kV + kTok * 64;        // uint8 [kTok][4]
    static constexpr int kVs = kKs + kTok * 4;        // uint8 [kTok][4]
    static constexpr int kBytesPerTok = 136;
    static constexpr int kStride = (kTok * kBytesPerTok + 1023) / 1024 * 1024;
    static constexpr int kStages = 4;
    static constexpr int kUnitTiles = NT == 1 ? 2 : 1;
};
// fp8 KV: the same bytes per key and layout as K8V8 (e4m3 codes for int8 ones).
template <int NT>
struct Stage<NF_KV_F8, NT> : Stage<NF_KV_K8V8, NT> {};
template <int NT>
struct Stage<NF_KV_BF16, NT> {
    static constexpr int kTok = 64;
    static constexpr int kK = 0;                      // bf16 [kTok][128]
    static constexpr int kV = kTok * 256;             // bf16 [kTok][128]
    static constexpr int kKs = 0, kVs = 0;
    static constexpr int kBytesPerTok = 512;
    static constexpr int kStride = kTok * kBytesPerTok;
    static constexpr int kStages = 4;
    static constexpr int kUnitTiles = 1;
};

struct DecodeParams {
    CUtensorMap vmap;  // v_codes as [num_blocks * H_kv * 256 rows][64 (K8/V4) or 128 (K8V8) bytes],
                       // 32-row boxes, swizzle as wide as a row (unused for bf16)
    CUtensorMap kmap;  // k_codes as [num_blocks * H_kv * 256 rows][128 bytes], 32-row boxes,
                       // 128-byte swizzle (the tensor-core decode of many rows only)
    CUtensorMap vmap_full, kmap_full;  // the same planes with boxes of a whole stage (decode_kernel:
                                       // a full stage's rows in one copy each)
    const void *k_codes;
    const __half *k_scales;
    const void *v_codes;
    const __half *v_scales;
    int num_blocks, num_kv_heads;
    const void *q;
    int batch, n_q, num_q_heads, group, rows;  // rows = group * n_q per kv-head
    int n_rg;                                  // row groups (of 8 * NT rows)
    const int32_t *block_table;
    int max_blocks;
    const int32_t *seqlens;
    int max_seqlen;
    float scale_log2;  // softmax_scale * log2(e)
    int causal;
    int early_kv;      // read lengths, tables and older pool rows before the dependency wait
    float *out;      // [batch][n_q][H_q][128]
    float *out_lse;  // [batch][n_q][H_q] or null
    int32_t *tickets;  // [batch * H_kv] ticket counters, zero between calls
    int32_t *done;     // [batch * H_kv] done counters of the final merges, zero between calls
    int32_t *claims;   // [gridDim.x + batch * H_kv] share flags, indexed like the slots; zero between calls
    float *partials;   // [gridDim.x + batch * H_kv] slots of slot_floats
    int slot_floats;   // rows * 128 (o) + rows (lse), rounded up to 4 floats
};

template <int NT, int FMT>
struct DecodeSmem {
    static constexpr int NR = NT * 8;
    using ST = Stage<FMT, NT>;
    static constexpr int kStagesBytes = ST::kStages * ST::kStride;
    static constexpr int kMergeO = kStagesBytes;                               // float [warp][NR][132]
    static constexpr int kMergeM = kMergeO + kConsumerWarps * NR * 132 * 4;    // float [warp][NR]
    static constexpr int kMergeL = kMergeM + kConsumerWarps * NR * 4;          // float [warp][NR]
    static constexpr int kBars = kMergeL + kConsumerWarps * NR * 4;            // u64 [2][stages] + 1
    static constexpr int kStageOk = kBars + (2 * ST::kStages + 1) * 8;         // int [stages]
    static constexpr int kSeqC = kStageOk + ST::kStages * 4;                   // int [kMaxBatch]
    static constexpr int kSeqL = kSeqC + kMaxBatch * 4;                        // int [kMaxBatch]
    static constexpr int kSeqBase = (kSeqL + kMaxBatch * 4 + 7) / 8 * 8;       // i64 [kMaxBatch + 1]
    static constexpr int kMisc = kSeqBase + (kMaxBatch + 1) * 8;              // int [4]
    static constexpr int kBytes = kMisc + 16;
    static_assert(kBytes <= 232448, "shared memory per CTA");
    // final merge: (row, 4 channels) items of at most 8 rows (NT = 1) or kMaxRows
    // the final merge's weights (rows x pieces) in the merge buffer
    static constexpr int kMergeFloats = (kMergeM - kMergeO) / 4;
    static_assert(kMergeFloats >= kMaxCtas, "a row of final-merge weights in the merge buffer");
    static_assert(ST::kStride % 128 == 0, "stage alignment");
};

// Output channel of row `rho` (0..15) of PV m-tile `m` (K8/V4): m-tile m = 2cg
// + ip covers scale group cg; row rho < 8 is channel 32cg + 4rho + 2ip (the
// nibble 2ip of b16 column rho of the group's 16-byte column), row rho + 8 the
// channel after it.
__device__ __forceinline__ int v_channel_k8v4(int m, int rho) {
    const int cg = m >> 1, ip = m & 1;
    return 32 * cg + 4 * (rho & 7) + 2 * ip + (rho >> 3);
}
// K8V8 and fp8: m-tile m is the 16-byte column m (channels 16m..16m+15); row rho < 8
// is channel 16m + 2rho (the low byte of b16 column rho), row rho + 8 the
// channel after it.
__device__ __forceinline__ int v_channel_k8v8(int m, int rho) { return 16 * m + 2 * (rho & 7) + (rho >> 3); }
// bf16 cache: lane t's u-th 16-byte load holds channels 32u + 8t .. 32u + 8t + 7.
__device__ __forceinline__ int v_channel_bf16(int m, int rho) {
    const int p = 2 * m + (rho >> 3), jj = rho & 7;
    return 32 * (p >> 2) + 8 * (jj >> 1) + 2 * (p & 3) + (jj & 1);
}
// Walks a CTA's chunk range piece by piece (a piece = the part of one segment
// that falls in the range).  Positions are in "cut" units: segment s spans
// `pad` padding units and then its C_b chunks; base[b] is the position of
// sequence b's first segment.  Producer and consumers walk it identically.
struct PieceWalker {
    const int *C;              // chunks per sequence
    const long long *base;     // position of sequence b's first segment
    int H, batch, pad;
    long long x, end;          // next position, end of the CTA range
    int b = 0;
    // current piece
    int pb, ph;                // sequence, kv-head
    long long s0, xs, xe;      // position of the segment's first chunk, piece [xs, xe)
    __device__ bool next() {
        while (x < end) {
            while (b + 1 <= batch && base[b + 1] <= x) ++b;
            const long long span = pad + (long long)C[b];
            pb = b;
            ph = (int)((x - base[b]) / span);
            s0 = base[b] + (long long)ph * span + pad;
            xs = x > s0 ? x : s0;
            xe = min(s0 + C[b], end);
            if (xs < xe) {
                x = xe;
                return true;
            }
            x = s0 + C[b];  // the range holds only padding of this segment
        }
        return false;
    }
};

// End (exclusive, in chunks of the segment) of the stage that starts at chunk
// cx: at most kTok keys, never crossing a 256-key block.
template <int FMT, int NT>
__device__ __forceinline__ int stage_end(int cx, int cx_end) {
    constexpr int per_blk = kBlock / kChunk, per_stage = Stage<FMT, NT>::kTok / kChunk;
    return min(cx_end, min((cx / per_blk + 1) * per_blk, cx + per_stage));
}

__device__ __forceinline__ int owner_cta(long long x, long long W, int P) {
    return (int)(((x + 1) * P - 1) / W);
}

// Brings the query rows of (sequence b, kv-head h) into L2 -- thread t < rows
// x lines per row takes one 128-byte line -- so that the piece that reads
// them later finds them there.  No value is read into the thread.
template <bool QF32>
__device__ __forceinline__ void prefetch_q_rows(const DecodeParams &p, int b, int h, int t) {
    constexpr int rb = kHeadDim * (QF32 ? 4 : 2) / 128;  // 128-byte lines per row
    if (t < p.rows * rb) {
        const int r = t / rb, j = r / p.group, gq = r % p.group;
        const size_t row = ((size_t)b * p.n_q + j) * p.num_q_heads + (size_t)h * p.group + gq;
        prefetch_l2(static_cast<const char *>(p.q) + row * kHeadDim * (QF32 ? 4 : 2) + (t % rb) * 128);
    }
}

// Per-warp consumer state: the query fragments of the current (sequence,
// kv-head) and the running softmax of the warp's rows.  In the S = Q . K^T
// product the query rows are the M dimension: rows 0-7 of an A fragment are
// the 8 query rows of tile nt (lane row g = query row 8nt + g), rows 8-15 a
// second operand of the same rows -- the low int8 digit (int8 K) or the low
// bf16 half of an fp32 query (bf16 cache; zero for a bf16 query) -- so one
// product yields both parts.
template <int NT, bool QF32, int FMT>
struct WarpState {
    static constexpr bool K8 = FMT == NF_KV_K8V4 || FMT == NF_KV_K8V8 || FMT == NF_KV_K4V4;  // int8 products
    uint32_t qa[NT][K8 ? 4 : 8][4];  // A fragments per k-step (32 channels int8 K, 16 channels fp16 / bf16)
    float qw[NT];                    // int8 K: s / 254, fp8 K: s, bf16: 1; times softmax scale x log2(e)
    float m_run[NT], l_run[NT];      // running max (log2 units) and weight sum of row g (lane's keys)
    float acc[8][NT][4];             // O^T fragments: channel rows, query columns 2t, 2t + 1
    int lim[NT];                     // last key position row g sees (-1: padding row)
};

// Byte offsets of a lane's data inside a stage buffer, relative to the first
// key of an m-tile.
struct LaneOffsets {
    uint32_t k, ks, v, vs;
};

// One work unit of a consumer warp: MT m-tiles of 16 keys starting at key ub
// of the stage buffer st (key tok0 + ub of the segment).  FAST: every row sees
// every key of the unit, so no mask is applied.
template <int NT, int MT, bool QF32, int FMT, bool FAST>
__device__ __forceinline__ void decode_unit(WarpState<NT, QF32, FMT> &ws, const unsigned char *st, int ub,
                                            int tok0, int L, int lane, const LaneOffsets &lo) {
    using ST = Stage<FMT, NT>;
    constexpr bool K8 = FMT == NF_KV_K8V4 || FMT == NF_KV_K8V8;  // int8 K codes
    constexpr bool K4 = FMT == NF_KV_K4V4;                         // 4-bit K and V, exponent-byte scales
    constexpr bool F8 = FMT == NF_KV_F8;                           // e4m3 K and V codes
    constexpr bool PF16 = FMT != NF_KV_BF16;                       // fp16 weights and V codes
    const int g = lane >> 2, t = lane & 3;

    // ---- S = Q . K^T: per m-tile two n-tiles j of 8 keys; the lane's results are
    // row g x keys tb + 8j + 2t + e (e = 0, 1) -> x[mt][nt][2j + e]
    float xv[MT][NT][4];
    float rl[MT][4];  // K4: 2^-E of the lane's keys 2t, 2t+1, 2t+8, 2t+9 (E: the key's largest V exponent)
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        const int tb = ub + 16 * mt;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            // K^T B fragments: the lane's column is key tb + 8j + g
            if (K4) {
                // word t of 16-byte column i (group i: channels 32i + 8t .. + 7) of key
                // tb + 8j + g; its even nibbles shifted up and its odd nibbles masked
                // are 16 x the codes as int8, in the B pairs of k-step i (the query
                // digits were laid out for that channel order)
                uint32_t w[4];
                ldsm_x4(smem_addr(st + ST::kK + (tb + 8 * j) * 64) + lo.k, w[0], w[1], w[2], w[3]);
                // exponent bytes of the lane's two result keys 2t, 2t + 1
                const uint2 ke = *reinterpret_cast<const uint2 *>(st + ST::kKs + (tb + 8 * j + 2 * t) * 4);
                // ... and of their V scales: the largest (E) shifts the key's score by E
                const uint2 ve = *reinterpret_cast<const uint2 *>(st + ST::kVs + (tb + 8 * j + 2 * t) * 4);
                const uint32_t m0 = __vmaxu4(ve.x, ve.x >> 16), m1 = __vmaxu4(ve.y, ve.y >> 16);
                const int E0 = (int)(__vmaxu4(m0, m0 >> 8) & 0xFFu), E1 = (int)(__vmaxu4(m1, m1 >> 8) & 0xFFu);
                rl[mt][2 * j] = E0 == 254 ? 5.877471754e-39f : __int_as_float((254 - E0) << 23);
                rl[mt][2 * j + 1] = E1 == 254 ? 5.877471754e-39f : __int_as_float((254 - E1) << 23);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    float x0 = 0.f, x1 = 0.f;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        int d[4] = {0, 0, 0, 0};
                        mma_s8(d, ws.qa[nt][i][0], ws.qa[nt][i][1], ws.qa[nt][i][2], ws.qa[nt][i][3],
                               (w[i] << 4) & 0xF0F0F0F0u, w[i] & 0xF0F0F0F0u);
                        // group i's sum times its 2^e (exponent byte e + 127 -> fp32 bits)
                        x0 = fmaf((float)(d[0] * 254 + d[2]), __int_as_float(((ke.x >> (8 * i)) & 0xFFu) << 23), x0);
                        x1 = fmaf((float)(d[1] * 254 + d[3]), __int_as_float(((ke.y >> (8 * i)) & 0xFFu) << 23), x1);
                    }
                    xv[mt][nt][2 * j] = fmaf(x0, ws.qw[nt], (float)(E0 - 127));
                    xv[mt][nt][2 * j + 1] = fmaf(x1, ws.qw[nt], (float)(E1 - 127));
                }
            } else if (F8) {
                // e4m3 bytes 32t..32t+31 of the key -> fp16 pairs; k-step ks takes
                // channels 32t + 4ks + 0, 1 (b0) and + 2, 3 (b1), the order the
                // query fragments were written in
                const unsigned char *k0 = st + ST::kK + (tb + 8 * j) * 128 + lo.k;
                const uint4 w0 = lds128(k0), w1 = lds128(k0 + 16);
                const uint32_t kw[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
                uint32_t kb[8][2];
#pragma unroll
                for (int u = 0; u < 8; ++u) e4m3x4_to_f16(kw[u], kb[u][0], kb[u][1]);
                const float2 sk = __half22float2(
                    *reinterpret_cast<const __half2 *>(st + ST::kKs + (tb + 8 * j + 2 * t) * 2));
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        mma_f16(d, ws.qa[nt][ks][0], ws.qa[nt][ks][1], ws.qa[nt][ks][2], ws.qa[nt][ks][3], kb[ks][0],
                                kb[ks][1]);
                    // d0, d1: the high fp16 part of the row . keys 2t, 2t+1; d2, d3: the low part
                    xv[mt][nt][2 * j] = (d[0] + d[2]) * (ws.qw[nt] * sk.x);
                    xv[mt][nt][2 * j + 1] = (d[1] + d[3]) * (ws.qw[nt] * sk.y);
                }
            } else if (K8) {
                const unsigned char *k0 = st + ST::kK + (tb + 8 * j) * 128 + lo.k;  // bytes 32t..32t+31
                const uint4 w0 = lds128(k0), w1 = lds128(k0 + 16);
                const uint32_t kb[4][2] = {{w0.x, w0.y}, {w0.z, w0.w}, {w1.x, w1.y}, {w1.z, w1.w}};
                // K scales of the lane's two result keys
                const float2 sk = __half22float2(
                    *reinterpret_cast<const __half2 *>(st + ST::kKs + (tb + 8 * j + 2 * t) * 2));
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    int d[4] = {0, 0, 0, 0};
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_s8(d, ws.qa[nt][ks][0], ws.qa[nt][ks][1], ws.qa[nt][ks][2], ws.qa[nt][ks][3], kb[ks][0],
                               kb[ks][1]);
                    // d0, d1: high digit . keys 2t, 2t+1; d2, d3: low digit.  |.| < 2^30,
                    // the conversion rounds once (relative 2^-24)
                    xv[mt][nt][2 * j] = (float)(d[0] * 254 + d[2]) * (ws.qw[nt] * sk.x);
                    xv[mt][nt][2 * j + 1] = (float)(d[1] * 254 + d[3]) * (ws.qw[nt] * sk.y);
                }
            } else {
                const unsigned char *k0 = st + ST::kK + (tb + 8 * j) * 256 + lo.k;  // bytes 64u + 16t .. + 15
                uint32_t kb[8][2];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const uint4 w = lds128(k0 + 64 * u);
                    kb[2 * u][0] = w.x; kb[2 * u][1] = w.y;
                    kb[2 * u + 1][0] = w.z; kb[2 * u + 1][1] = w.w;
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        mma_bf16(d, ws.qa[nt][ks][0], ws.qa[nt][ks][1], ws.qa[nt][ks][2], ws.qa[nt][ks][3], kb[ks][0],
                                 kb[ks][1]);
                    xv[mt][nt][2 * j] = (QF32 ? d[0] + d[2] : d[0]) * ws.qw[nt];
                    xv[mt][nt][2 * j + 1] = (QF32 ? d[1] + d[3] : d[1]) * ws.qw[nt];
                }
            }
        }
        if (!FAST) {
            // keys past the end hold stale bytes; causal rows see keys <= lim
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int pos = tok0 + tb + 8 * (i >> 1) + 2 * t + (i & 1);
                    if (!(pos < L && pos <= ws.lim[nt])) xv[mt][nt][i] = -INFINITY;
                }
            if (K4) {
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    if (!(tok0 + tb + 8 * (i >> 1) + 2 * t + (i & 1) < L)) rl[mt][i] = 0.f;
            }
        }
    }

    // ---- lazy running max of row g (the 4 lanes of a row agree on it)
    bool raise = false;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        float mx = fmaxf(fmaxf(xv[0][nt][0], xv[0][nt][1]), fmaxf(xv[0][nt][2], xv[0][nt][3]));
#pragma unroll
        for (int mt = 1; mt < MT; ++mt)
            mx = fmaxf(mx, fmaxf(fmaxf(xv[mt][nt][0], xv[mt][nt][1]), fmaxf(xv[mt][nt][2], xv[mt][nt][3])));
        raise |= mx > ws.m_run[nt] + kLazy;  // true when m_run is -inf and mx finite
    }
    if (__any_sync(0xffffffffu, raise)) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            float mx = fmaxf(fmaxf(xv[0][nt][0], xv[0][nt][1]), fmaxf(xv[0][nt][2], xv[0][nt][3]));
#pragma unroll
            for (int mt = 1; mt < MT; ++mt)
                mx = fmaxf(mx, fmaxf(fmaxf(xv[mt][nt][0], xv[mt][nt][1]), fmaxf(xv[mt][nt][2], xv[mt][nt][3])));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            const float m_new = fmaxf(ws.m_run[nt], mx);
            const float alpha = m_new == -INFINITY ? 1.f : ex2(ws.m_run[nt] - m_new);
            ws.m_run[nt] = m_new;
            ws.l_run[nt] *= alpha;
            // the accumulators hold query rows 2t and 2t + 1: take their factors
            const float a0 = __shfl_sync(0xffffffffu, alpha, 8 * t);
            const float a1 = __shfl_sync(0xffffffffu, alpha, 8 * t + 4);
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                ws.acc[m][nt][0] *= a0;
                ws.acc[m][nt][1] *= a1;
                ws.acc[m][nt][2] *= a0;
                ws.acc[m][nt][3] *= a1;
            }
        }
    }
    // ---- weights 2^(x - m - kLazy) <= 1, already in the B-fragment layout of
    // the PV product: b0 = keys 2t, 2t+1 of row g, b1 = keys 8 + 2t, 9 + 2t
    uint32_t pb[MT][NT][2], pbl[MT][NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const float mu = (ws.m_run[nt] == -INFINITY ? 0.f : ws.m_run[nt]) + kLazy;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            const float p0 = ex2(xv[mt][nt][0] - mu), p1 = ex2(xv[mt][nt][1] - mu);
            const float p2 = ex2(xv[mt][nt][2] - mu), p3 = ex2(xv[mt][nt][3] - mu);
            if (K4)  // the weights carry each key's 2^E: the row sum takes it out again
                ws.l_run[nt] += fmaf(p0, rl[mt][0], p1 * rl[mt][1]) + fmaf(p2, rl[mt][2], p3 * rl[mt][3]);
            else
                ws.l_run[nt] += (p0 + p1) + (p2 + p3);
            if (PF16) {
                pb[mt][nt][0] = pack_f16(p0, p1);
                pb[mt][nt][1] = pack_f16(p2, p3);
            } else {
                // bf16 weights split into hi + lo so they keep ~16 bits
                const uint32_t h0 = pack_bf16(p0, p1), h1 = pack_bf16(p2, p3);
                pb[mt][nt][0] = h0;
                pb[mt][nt][1] = h1;
                pbl[mt][nt][0] = pack_bf16(p0 - __uint_as_float(h0 << 16), p1 - __uint_as_float(h0 & 0xFFFF0000u));
                pbl[mt][nt][1] = pack_bf16(p2 - __uint_as_float(h1 << 16), p3 - __uint_as_float(h1 & 0xFFFF0000u));
            }
        }
    }

    // ---- O^T += V^T . P^T over 8 channel m-tiles, one 16-key k-tile per m-tile of the unit
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        const int tb = ub + 16 * mt;
        if (FMT == NF_KV_K8V8 || F8) {
            // V scales of keys (2t, 2t+1) and (2t+8, 2t+9) as fp16 pairs: one
            // scale per key serves all channels, so each B fragment takes it once
            uint32_t sp0 = *reinterpret_cast<const uint32_t *>(st + ST::kVs + (tb + 2 * t) * 2);
            uint32_t sp1 = *reinterpret_cast<const uint32_t *>(st + ST::kVs + (tb + 8 + 2 * t) * 2);
            // keys past the end hold stale bytes: zero their scales (and, for
            // e4m3, whose stale bytes may be NaN, their codes: the lane's code
            // word holds key 2t in bytes 0-1 and key 2t+1 in bytes 2-3, the
            // layout of a scale pair)
            uint32_t keep0 = 0xFFFFFFFFu, keep1 = 0xFFFFFFFFu;
            if (!FAST) {
                const int pa = tok0 + tb + 2 * t;
                keep0 = (pa < L ? 0x0000FFFFu : 0u) | (pa + 1 < L ? 0xFFFF0000u : 0u);
                keep1 = (pa + 8 < L ? 0x0000FFFFu : 0u) | (pa + 9 < L ? 0xFFFF0000u : 0u);
                sp0 &= keep0;
                sp1 &= keep1;
            }
            uint32_t b0[NT], b1[NT];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                b0[nt] = h2_u32(__hmul2(u32_h2(pb[mt][nt][0]), u32_h2(sp0)));
                b1[nt] = h2_u32(__hmul2(u32_h2(pb[mt][nt][1]), u32_h2(sp1)));
            }
            // codes: matrix i of a load (lanes 8i..8i+7 address its rows) = keys
            // tb + 8 (i & 1) + 0..7 of the 16-byte column 2cp + (i >> 1), which
            // the swizzled copy stores at column position column ^ (key & 7); the
            // lane receives channels 16 column + 2g, + 1 of keys 2t, 2t + 1
            const uint32_t va = smem_addr(st + ST::kV + tb * 128) + lo.v;
#pragma unroll
            for (int cp = 0; cp < 4; ++cp) {
                uint32_t R[4];
                ldsm_x4_t(va ^ (32u * cp), R[0], R[1], R[2], R[3]);
#pragma unroll
                for (int jc = 0; jc < 2; ++jc) {
                    uint32_t a[4];
                    if (F8) {
                        // bytes (0, 2) and (1, 3) -> fp16 pairs: rows g and g + 8
                        const uint32_t r0 = prmt(FAST ? R[2 * jc] : R[2 * jc] & keep0, 0u, 0x3120);
                        const uint32_t r1 = prmt(FAST ? R[2 * jc + 1] : R[2 * jc + 1] & keep1, 0u, 0x3120);
                        e4m3x4_to_f16(r0, a[0], a[1]);
                        e4m3x4_to_f16(r1, a[2], a[3]);
                    } else {
                        i8x4_to_f16_eo(R[2 * jc], a[0], a[1]);      // keys 2t, 2t+1: rows g, g + 8
                        i8x4_to_f16_eo(R[2 * jc + 1], a[2], a[3]);  // keys 2t+8, 2t+9
                    }
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
                        mma_f16(ws.acc[2 * cp + jc][nt], a[0], a[1], a[2], a[3], b0[nt], b1[nt]);
                }
            }
        } else if (K8 || K4) {
            // nibbles: matrix cg (lanes 8cg..8cg+7 address its rows) = the 16-byte
            // column cg (channels 32cg..32cg+31) of 8 keys, stored at column
            // position cg ^ (row address bits 7-8) by the swizzled copy
            uint32_t R[2][4];
            const uint32_t va = smem_addr(st + ST::kV + tb * 64) + lo.v;
            ldsm_x4_t(va, R[0][0], R[0][1], R[0][2], R[0][3]);            // keys tb + 0..7
            ldsm_x4_t(va + 8 * 64, R[1][0], R[1][1], R[1][2], R[1][3]);   // keys tb + 8..15
            // V scales of keys (2t, 2t+1) and (2t+8, 2t+9) per group, as fp16 pairs
            // (K4: the factors 2^(e_g - E) <= 1 of the group exponents relative to
            // the key's largest, whose 2^E the weights already carry; factors below
            // 2^-14 flush to zero)
            uint32_t sp[2][4];
#pragma unroll
            for (int kh = 0; kh < 2; ++kh) {
                if (K4) {
                    const uint2 ve = *reinterpret_cast<const uint2 *>(st + ST::kVs + (tb + 8 * kh + 2 * t) * 4);
                    uint32_t dd[2];
                    const uint32_t vv[2] = {ve.x, ve.y};
#pragma unroll
                    for (int k2 = 0; k2 < 2; ++k2) {
                        const uint32_t m = __vmaxu4(vv[k2], vv[k2] >> 16);
                        const uint32_t E = (__vmaxu4(m, m >> 8) & 0xFFu) * 0x01010101u;
                        // 15 - (E - e_g) per byte, at least 0: the fp16 exponent field of 2^(e_g - E)
                        dd[k2] = __vsubus4(0x0F0F0F0Fu, __vsubus4(E, vv[k2]));
                    }
#pragma unroll
                    for (int cg = 0; cg < 4; ++cg)  // byte cg of key 2t -> half 0, of key 2t + 1 -> half 1
                        sp[kh][cg] = prmt_sx(dd[0], dd[1], 0x8080u | (uint32_t)cg | ((uint32_t)(cg + 4) << 8)) << 10;
                } else {
                    const uint4 sv = lds128(st + ST::kVs + (tb + 8 * kh) * 8 + lo.vs);
                    sp[kh][0] = prmt(sv.x, sv.z, 0x5410);
                    sp[kh][1] = prmt(sv.x, sv.z, 0x7632);
                    sp[kh][2] = prmt(sv.y, sv.w, 0x5410);
                    sp[kh][3] = prmt(sv.y, sv.w, 0x7632);
                }
                if (!FAST) {
                    // keys past the end hold stale bytes: zero their scales
                    const int pa = tok0 + tb + 8 * kh + 2 * t;
                    const uint32_t keep = (pa < L ? 0x0000FFFFu : 0u) | (pa + 1 < L ? 0xFFFF0000u : 0u);
#pragma unroll
                    for (int cg = 0; cg < 4; ++cg) sp[kh][cg] &= keep;
                }
            }
#pragma unroll
            for (int cg = 0; cg < 4; ++cg) {
                // exact fp16 codes of channel 32cg + 4g + i for the key pairs
                const uint32_t lo0 = R[0][cg], hi0 = R[0][cg] >> 8;
                const uint32_t lo1 = R[1][cg], hi1 = R[1][cg] >> 8;
                const uint32_t a[2][4] = {
                    {h2_u32(nib_even(lo0)), h2_u32(nib_odd(lo0)), h2_u32(nib_even(lo1)), h2_u32(nib_odd(lo1))},
                    {h2_u32(nib_even(hi0)), h2_u32(nib_odd(hi0)), h2_u32(nib_even(hi1)), h2_u32(nib_odd(hi1))}};
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const uint32_t b0 = h2_u32(__hmul2(u32_h2(pb[mt][nt][0]), u32_h2(sp[0][cg])));
                    const uint32_t b1 = h2_u32(__hmul2(u32_h2(pb[mt][nt][1]), u32_h2(sp[1][cg])));
#pragma unroll
                    for (int ip = 0; ip < 2; ++ip)
                        mma_f16(ws.acc[2 * cg + ip][nt], a[ip][0], a[ip][1], a[ip][2], a[ip][3], b0, b1);
                }
            }
        } else {
            const unsigned char *v0p = st + ST::kV + tb * 256 + lo.v;
            const bool ok0 = FAST || tok0 + tb + g < L, ok1 = FAST || tok0 + tb + g + 8 < L;
            uint32_t w0[16], w1[16];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                uint4 va = lds128(v0p + 64 * u), vb = lds128(v0p + 8 * 256 + 64 * u);
                if (!ok0) va = make_uint4(0, 0, 0, 0);  // stale bytes past the end
                if (!ok1) vb = make_uint4(0, 0, 0, 0);
                w0[4 * u] = va.x; w0[4 * u + 1] = va.y; w0[4 * u + 2] = va.z; w0[4 * u + 3] = va.w;
                w1[4 * u] = vb.x; w1[4 * u + 1] = vb.y; w1[4 * u + 2] = vb.z; w1[4 * u + 3] = vb.w;
            }
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const uint32_t a0 = movmatrix_t(w0[2 * m]), a1 = movmatrix_t(w0[2 * m + 1]);
                const uint32_t a2 = movmatrix_t(w1[2 * m]), a3 = movmatrix_t(w1[2 * m + 1]);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    mma_bf16(ws.acc[m][nt], a0, a1, a2, a3, pb[mt][nt][0], pb[mt][nt][1]);
                    mma_bf16(ws.acc[m][nt], a0, a1, a2, a3, pbl[mt][nt][0], pbl[mt][nt][1]);
                }
            }
        }
    }
}

// How long a CTA whose piece shares the final merge of its segment waits for
// the segment's last piece before it leaves its share to the CTA that draws
// the last ticket.  Far above the spread of the pieces' end times (a few
// microseconds); it only comes into play when some CTA of the grid could not
// be placed on an SM while the others wait.
constexpr uint64_t kCoopWaitNs = 50000ull;

// Share j of m of a segment's final merge: output items [j I / m, (j + 1) I /
// m) of the I = rows x 32 items (row, 4 channels), each the sum over the n
// pieces of w_k o_k, w_k = e^(lse_k - M) / sum_i e^(lse_i - M) with M the
// row's largest lse.  slots: piece k's slot at slots + k * p.slot_floats (its
// normalised o rows, then their lse), read from L2.  Threads 0 .. NTHR - 1,
// named barrier BAR; sm: scratch of (NTHR / 32 + 2) kMaxCtas + 4 NTHR floats.
// The items go in chunks of up to NTHR; in a chunk of c items thread t takes
// item t % c and the pieces t / c, t / c + Q, ... (Q = NTHR / c), and the Q
// partial sums are then added in order, so the arithmetic depends only on (n,
// m, j, rows), not on which CTA merges the share.  A row no piece saw a key
// of (every lse -inf) comes out as o = 0, lse = -inf.
template <int NTHR, uint32_t BAR>
__device__ __forceinline__ void merge_share(const DecodeParams &p, const float *slots, int n, int rows, int j, int m,
                                            float *sm, int b, int h) {
    constexpr float kLog2e = 1.4426950408889634f;
    constexpr int NW = NTHR / 32, NJ = kMaxCtas / 32, KB = 4;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const size_t sf = p.slot_floats;
    const int lse_off = rows * kHeadDim;
    const int I = rows * (kHeadDim / 4);
    const int i0 = (int)((long long)I * j / m), i1 = (int)((long long)I * (j + 1) / m);
    float *wsm = sm;                                                       // [rows of the chunk][n]
    float4 *red = reinterpret_cast<float4 *>(sm + (NW + 2) * kMaxCtas);  // [Q][c]
    for (int c0 = i0; c0 < i1; c0 += NTHR) {
        const int c = min(NTHR, i1 - c0), Q = NTHR / c;
        const int r_lo = c0 / 32, nrr = (c0 + c - 1) / 32 - r_lo + 1;
        const bool act = tid < Q * c;
        const int it = c0 + (act ? tid % c : 0), q = act ? tid / c : 0;
        const int r = it / 32, c4 = it % 32;
        const float *src = slots + (size_t)r * kHeadDim + 4 * c4;
        // the first pieces' o, in flight while the weights are worked out
        float4 o[KB];
#pragma unroll
        for (int u = 0; u < KB; ++u) {
            const int k = q + Q * u;
            o[u] = act && k < n ? __ldcg(reinterpret_cast<const float4 *>(src + k * sf)) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        // the weights of the chunk's rows: one warp per row, lane l holds pieces l + 32 i
        for (int rr = warp; rr < nrr; rr += NW) {
            const int rw = r_lo + rr;
            float lv[NJ], w[NJ];
            float mx = -INFINITY, s = 0.f;
#pragma unroll
            for (int i = 0; i < NJ; ++i) {
                const int k = lane + 32 * i;
                lv[i] = k < n ? __ldcg(slots + k * sf + lse_off + rw) : -INFINITY;
                mx = fmaxf(mx, lv[i]);
            }
#pragma unroll
            for (int d = 16; d > 0; d >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, d));
#pragma unroll
            for (int i = 0; i < NJ; ++i) {
                w[i] = lv[i] == -INFINITY ? 0.f : ex2((lv[i] - mx) * kLog2e);
                s += w[i];
            }
#pragma unroll
            for (int d = 16; d > 0; d >>= 1) s += __shfl_xor_sync(0xffffffffu, s, d);
            const float inv = mx == -INFINITY ? 0.f : 1.0f / s;
#pragma unroll
            for (int i = 0; i < NJ; ++i)
                if (lane + 32 * i < n) wsm[rr * n + lane + 32 * i] = w[i] * inv;
            // the row's lse goes with the share that holds the row's first item
            if (lane == 0 && p.out_lse && rw * 32 >= c0 && rw * 32 < c0 + c) {
                const int jq = rw / p.group, gq = rw % p.group;
                const size_t row = ((size_t)b * p.n_q + jq) * p.num_q_heads + (size_t)h * p.group + gq;
                p.out_lse[row] = mx == -INFINITY ? -INFINITY : mx + logf(s);
            }
        }
        named_sync(BAR, NTHR);
        // this thread's pieces, KB loads at a time
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        const float *wr = wsm + (r - r_lo) * n;
        for (int u0 = 0;; u0 += KB) {
#pragma unroll
            for (int u = 0; u < KB; ++u) {
                const int k = q + Q * (u0 + u);
                const float wk = act && k < n ? wr[k] : 0.f;
                acc.x = fmaf(wk, o[u].x, acc.x);
                acc.y = fmaf(wk, o[u].y, acc.y);
                acc.z = fmaf(wk, o[u].z, acc.z);
                acc.w = fmaf(wk, o[u].w, acc.w);
            }
            if (!act || q + Q * (u0 + KB) >= n) break;
#pragma unroll
            for (int u = 0; u < KB; ++u) {
                const int k = q + Q * (u0 + KB + u);
                o[u] = k < n ? __ldcg(reinterpret_cast<const float4 *>(src + k * sf)) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
        if (act) red[q * c + tid % c] = acc;
        named_sync(BAR, NTHR);
        if (tid < c) {
            float4 sum = red[tid];
            for (int qq = 1; qq < Q; ++qq) {
                const float4 v = red[qq * c + tid];
                sum.x += v.x; sum.y += v.y; sum.z += v.z; sum.w += v.w;
            }
            const int ri = (c0 + tid) / 32, ci = (c0 + tid) % 32;
            const int jq = ri / p.group, gq = ri % p.group;
            const size_t row = ((size_t)b * p.n_q + jq) * p.num_q_heads + (size_t)h * p.group + gq;
            reinterpret_cast<float4 *>(p.out + row * kHeadDim)[ci] = sum;
        }
        named_sync(BAR, NTHR);  // the scratch is free again
    }
}

// The final merge of a segment's n partial slots -- slot k at src + k * sf
// floats: its normalised o rows [rows][128], then their lse [rows] -- into the
// output rows (row r of the kv-head's group at out + orow(r) * 128, its lse at
// out_lse + orow(r)), in two steps run by threads 0 .. NTHR - 1 (named barrier
// BAR):
//  merge_weights  per row r in [r0, r0 + nr), one warp per row: w_k = e^(lse_k
//                 - M) / sum_i e^(lse_i - M) (M the row's largest lse) into
//                 wsm[(r - r0) n + k], and the row's lse = M + ln sum; the lse
//                 values come from L2 (the last ticket's acquire made them
//                 visible);
//  merge_items    every (row, 4 channels) item of those rows: sum_k w_k o_k in
//                 piece order, o read from shared memory (SMEM, the slots
//                 copied into this CTA) or from L2 -- the same arithmetic
//                 either way.
// A row no piece saw a key of comes out as o = 0, lse = -inf.
struct OutRows {
    float *out, *out_lse;
    size_t base;  // row index of (b, query 0, first q-head of the group)
    int group, n_q, num_q_heads;
    __device__ size_t operator()(int r) const {
        return base + (size_t)(r / group) * num_q_heads + r % group;
    }
};

template <int NTHR>
__device__ __noinline__ void merge_weights(const float *src, size_t sf, int n, int rows, int r0, int nr, float *wsm,
                                           const OutRows orow) {
    constexpr float kLog2e = 1.4426950408889634f;
    constexpr int NW = NTHR / 32, NJ = kMaxCtas / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int lse_off = rows * kHeadDim;
    for (int rr = warp; rr < nr; rr += NW) {
        const int r = r0 + rr;
        float lv[NJ], w[NJ];
        float mx = -INFINITY, s = 0.f;
#pragma unroll
        for (int i = 0; i < NJ; ++i) {
            const int k = lane + 32 * i;
            lv[i] = k < n ? __ldcg(src + k * sf + lse_off + r) : -INFINITY;
            mx = fmaxf(mx, lv[i]);
        }
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, d));
#pragma unroll
        for (int i = 0; i < NJ; ++i) {
            w[i] = lv[i] == -INFINITY ? 0.f : ex2((lv[i] - mx) * kLog2e);
            s += w[i];
        }
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) s += __shfl_xor_sync(0xffffffffu, s, d);
        const float inv = mx == -INFINITY ? 0.f : 1.0f / s;
#pragma unroll
        for (int i = 0; i < NJ; ++i)
            if (lane + 32 * i < n) wsm[rr * n + lane + 32 * i] = w[i] * inv;
        if (lane == 0 && orow.out_lse) orow.out_lse[orow(r)] = mx == -INFINITY ? -INFINITY : mx + logf(s);
    }
}

template <int NTHR, bool SMEM>
__device__ __noinline__ void merge_items(const float *src, size_t sf, int n, int r0, int nr, const float *wsm,
                                         const OutRows orow) {
    constexpr int KB = 16;
    const size_t s4 = sf / 4;
    for (int it = threadIdx.x; it < nr * (kHeadDim / 4); it += NTHR) {
        const int rr = it / (kHeadDim / 4), c4 = it % (kHeadDim / 4), r = r0 + rr;
        const float *wr = wsm + rr * n;
        const float4 *op = reinterpret_cast<const float4 *>(src + (size_t)r * kHeadDim) + c4;
        const uint32_t sop = SMEM ? smem_addr(op) : 0u;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int k0 = 0; k0 < n; k0 += KB) {
            float4 o[KB];
#pragma unroll
            for (int j = 0; j < KB; ++j)
                o[j] = k0 + j >= n ? make_float4(0.f, 0.f, 0.f, 0.f)
                       : SMEM      ? lds_f4(sop + (uint32_t)((k0 + j) * s4 * 16))
                                   : __ldcg(op + (k0 + j) * s4);
#pragma unroll
            for (int j = 0; j < KB; ++j) {
                const float wk = k0 + j < n ? wr[k0 + j] : 0.f;
                acc.x = fmaf(wk, o[j].x, acc.x);
                acc.y = fmaf(wk, o[j].y, acc.y);
                acc.z = fmaf(wk, o[j].z, acc.z);
                acc.w = fmaf(wk, o[j].w, acc.w);
            }
        }
        reinterpret_cast<float4 *>(orow.out + orow(r) * kHeadDim)[c4] = acc;
    }
}

// The end of a piece of a segment split over n > 1 CTAs, its partial already
// in its slot, run by threads 0 .. NTHR - 1 after a barrier that orders the
// slot writes before thread 0; no CTA waits for another.  The piece draws a
// ticket of the segment's counter (acquire-release: it publishes the slot
// and, for the last ticket, makes every other slot visible); the CTA with the
// last ticket merges the segment's partials into out and resets the counter.
// When this was the CTA's last piece (ring_idle: every stage consumed, no copy
// in flight) and the n slots fit the ring and every row's weights fit wsm
// (wcap floats), one bulk copy brings the slots into the ring while the
// weights are worked out from L2, and the items read shared memory; else the
// merge reads L2, in passes of as many rows as wsm holds.
template <int NTHR, uint32_t BAR>
__device__ __forceinline__ void finish_piece_single(const DecodeParams &p, int s_id, int first, int n, int rows,
                                                    int b, int h, bool ring_idle, unsigned char *ring,
                                                    uint32_t ring_bytes, uint64_t *fin_bar, uint32_t &fin_phase,
                                                    float *wsm, int wcap, volatile int *misc) {
    if (n < 2) return;
    const float *slots = p.partials + (size_t)(s_id + first) * p.slot_floats;
    const size_t sf = p.slot_floats;
    const uint32_t bytes = (uint32_t)n * (uint32_t)sf * 4u;
    const bool in_ring = ring_idle && bytes <= ring_bytes && rows * n <= wcap;
    if (threadIdx.x == 0) {
        const bool last = atomic_add_acq_rel(&p.tickets[s_id], 1) == n - 1;
        misc[1] = last;
        if (last && in_ring && !misc[0]) {
            // the ring's last reads (generic proxy) and the other CTAs' slot
            // writes (visible through the ticket's acquire) precede the copy
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            asm volatile("fence.proxy.async.global;" ::: "memory");
            mbar_arrive_expect_tx(fin_bar, bytes);
            bulk_g2s(ring, slots, bytes, fin_bar);
        }
    }
    named_sync(BAR, NTHR);
    if (!misc[1]) return;
    const OutRows orow{p.out, p.out_lse, (size_t)b * p.n_q * p.num_q_heads + (size_t)h * p.group, p.group, p.n_q,
                       p.num_q_heads};
    if (in_ring) {
        merge_weights<NTHR>(slots, sf, n, rows, 0, rows, wsm, orow);  // while the copy is in flight
        if (!misc[0] && !mbar_wait(fin_bar, fin_phase)) {
            report(NF_DEVERR_TIMEOUT);
            misc[0] = 1;
        }
        fin_phase ^= 1u;
        named_sync(BAR, NTHR);
        if (!misc[0])
            merge_items<NTHR, true>(reinterpret_cast<const float *>(ring), sf, n, 0, rows, wsm, orow);
        else  // after a timeout the slots are read from L2 instead
            merge_items<NTHR, false>(slots, sf, n, 0, rows, wsm, orow);
    } else {
        const int rpp = min(rows, max(1, wcap / n));
        for (int r0 = 0; r0 < rows; r0 += rpp) {
            const int nr = min(rpp, rows - r0);
            merge_weights<NTHR>(slots, sf, n, rows, r0, nr, wsm, orow);
            named_sync(BAR, NTHR);
            merge_items<NTHR, false>(slots, sf, n, r0, nr, wsm, orow);
            named_sync(BAR, NTHR);  // wsm is free again
        }
    }
    if (threadIdx.x == 0) p.tickets[s_id] = 0;
}

// The end of a piece of a segment split over n > 1 CTAs, with the final merge
// shared among the segment's CTAs (decode_tc_kernel, whose 32-row partials
// are too large for one CTA to read quickly).  The partial (o, lse) is
// already in its slot -- slot s_id + first + k, k the piece's index in the
// segment -- and threads 0 .. NTHR - 1 run this after a barrier that orders the
// slot writes before thread 0.  Each piece draws a ticket of the segment's counter
// (acquire-release: it publishes the slot and, for the last ticket, makes
// every other slot visible).  The final merge is cut into m shares, one per
// participating piece: pieces 0 .. m - 1, whose CTAs have no further work (m
// = n, or n - 1 when the last piece's CTA goes on into the next segment).
//  - A participant waits, at most kCoopWaitNs, until all n pieces hold
//    tickets, then claims its share (compare-and-swap on the share's flag) and
//    merges it; one that times out leaves its share unclaimed.
//  - The CTA with the last ticket, after its own share, claims and merges
//    every share still unclaimed, so each share is merged exactly once
//    whatever the timing.
//  - Every piece then counts itself done; the last one returns the ticket,
//    the done count and the share flags to zero for the next call.
// No wait is unbounded, and a CTA that stops waiting loses nothing: its share
// is swept by the last ticket's CTA.
template <int NTHR, uint32_t BAR>
__device__ __forceinline__ void finish_piece_coop(const DecodeParams &p, int s_id, int first, int k, int n, int m,
                                                     float *sm, volatile int *misc, int rows, int b, int h) {
    constexpr int NW = NTHR / 32;
    if (n < 2) return;
    const float *slots = p.partials + (size_t)(s_id + first) * p.slot_floats;
    int *flag = p.claims + s_id + first;  // flag j: share j claimed
    if (threadIdx.x == 0) {
        const bool last = atomic_add_acq_rel(&p.tickets[s_id], 1) == n - 1;
        bool ready = last;
        if (!last && k < m) {
            const uint64_t t0 = global_ns();
            while (!(ready = ld_acquire(&p.tickets[s_id]) == n) && global_ns() - t0 < kCoopWaitNs) __nanosleep(100);
        }
        misc[1] = last;
        misc[2] = ready && k < m && atomicCAS(&flag[k], 0, 1) == 0;
    }
    named_sync(BAR, NTHR);
    if (misc[2]) merge_share<NTHR, BAR>(p, slots, n, rows, k, m, sm, b, h);
    if (misc[1]) {
        // the sweep: the shares nobody has claimed
        int *won = reinterpret_cast<int *>(sm + (NW + 2) * kMaxCtas + 4 * NTHR);
        if ((int)threadIdx.x < m) won[threadIdx.x] = atomicCAS(&flag[threadIdx.x], 0, 1) == 0;
        named_sync(BAR, NTHR);
        for (int j = 0; j < m; ++j)
            if (won[j]) merge_share<NTHR, BAR>(p, slots, n, rows, j, m, sm, b, h);
    }
    named_sync(BAR, NTHR);  // this CTA's merge reads and writes precede its done count
    if (threadIdx.x == 0 && atomic_add_acq_rel(&p.done[s_id], 1) == n - 1) {
        p.tickets[s_id] = 0;
        p.done[s_id] = 0;
        for (int j = 0; j < m; ++j) flag[j] = 0;
    }
}

template <int NT, bool QF32, int FMT>
__global__ void __launch_bounds__(kDecodeThreads, 1) decode_kernel(const __grid_constant__ DecodeParams p) {
    using ST = Stage<FMT, NT>;
    using SM = DecodeSmem<NT, FMT>;
    constexpr int MT = ST::kUnitTiles;
    constexpr bool K8 = (FMT != NF_KV_BF16);  // scaled codes through the bulk/tensor-map copies
    constexpr bool V8 = (FMT == NF_KV_K8V8 || FMT == NF_KV_F8);  // 128-byte V rows, one V scale per key
    constexpr bool F8 = (FMT == NF_KV_F8);
    constexpr bool K4 = (FMT == NF_KV_K4V4);  // nibble K rows (tensor map), exponent-byte scales
    static_assert(SM::kMergeM - SM::kMergeO >= (kMaxRows * 128 + (NT == 1 ? 8 : kMaxRows)) * 4,
                  "fp8 query fragments and factors in the merge buffer");
    constexpr int NS = ST::kStages;
    constexpr int NR = SM::NR;
    extern __shared__ __align__(1024) unsigned char smem[];
    float *sm_o = reinterpret_cast<float *>(smem + SM::kMergeO);
    float *sm_m = reinterpret_cast<float *>(smem + SM::kMergeM);
    float *sm_l = reinterpret_cast<float *>(smem + SM::kMergeL);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + SM::kBars);
    uint64_t *empty = full + NS;
    uint64_t *fin_bar = full + 2 * NS;  // the final merge's bulk copy
    volatile int *stage_ok = reinterpret_cast<volatile int *>(smem + SM::kStageOk);
    int *seqC = reinterpret_cast<int *>(smem + SM::kSeqC);
    int *seqL = reinterpret_cast<int *>(smem + SM::kSeqL);
    long long *seqBase = reinterpret_cast<long long *>(smem + SM::kSeqBase);
    volatile int *misc = reinterpret_cast<volatile int *>(smem + SM::kMisc);  // [0] abort, [1] last-ticket

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int H = p.num_kv_heads;

    // ---- set-up: barriers and the chunk list (every CTA computes the same)
    if (threadIdx.x == 0) {
        for (int i = 0; i < NS; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kConsumerWarps);
            stage_ok[i] = 0;
        }
        mbar_init(fin_bar, 1);
        misc[0] = 0;
        misc[1] = 0;
        // the stage buffers must start on 1024-byte boundaries (swizzled V
        // tiles); if the shared window ever were not so aligned, do no work
        if (smem_addr(smem) & 1023u) {
            if (blockIdx.x == 0) report(NF_DEVERR_INTERNAL);
            misc[0] = 1;
        }
        fence_mbar_init();
    }
    // everything above touched shared memory only; the lengths, tables, query,
    // pool and workspace may come from the kernels before this one.  With
    // early_kv the caller guarantees that the kernels still running write
    // neither the lengths, the block tables nor the pool rows older than the
    // newest n_q positions of each sequence: those are read at once, and the
    // wait is taken before the query, the newest rows, the outputs and the
    // workspace are touched.
    if (!p.early_kv) pdl_wait();
    pdl_trigger();
    if (warp == 0) {
        for (int b = lane; b < p.batch; b += 32) {
            const int L = p.seqlens[b];
            const bool ok = L >= p.n_q && L <= p.max_seqlen;
            if (!ok && blockIdx.x == 0) report(NF_DEVERR_SEQLEN);
            seqC[b] = ok ? (L + kChunk - 1) / kChunk : 0;
            seqL[b] = ok ? L : 0;
        }
        __syncwarp();
        if (lane == 0) {
            long long acc = 0;
            for (int b = 0; b < p.batch; ++b) {
                seqBase[b] = acc;
                acc += seqC[b] ? (long long)(seqC[b] + kSegPad) * H : 0;
            }
            seqBase[p.batch] = acc;
        }
    }
    __syncthreads();
    const long long W = seqBase[p.batch];
    // CTAs taking part: never more than there are chunks, so that every CTA
    // between a segment's first and last owner holds a piece of it
    const int P = (int)(W < (long long)gridDim.x ? W : (long long)gridDim.x);
    // The CTAs take the ranges in reverse order: the highest-numbered CTA is
    // the last one placed when the previous kernel's CTAs leave the SMs, so it
    // starts last; range 0 opens a segment with its padding (fewer keys).
    const int vb = (int)blockIdx.x < P ? P - 1 - (int)blockIdx.x : (int)blockIdx.x;
    const long long c_begin = vb < P ? W * vb / P : 0;
    const long long c_end = vb < P ? W * (vb + 1) / P : 0;

    PieceWalker walk{seqC, seqBase, H, p.batch, kSegPad, c_begin, c_end};

    // =================================================================== producer
    // The whole warp walks the stages; its lanes hold a window of 32 block-table
    // entries (one global load per 32 blocks), lane 0 waits for free buffers
    // and issues the bulk copies.
    if (warp == kConsumerWarps) {
        uint32_t kst = 0;  // CTA-wide stage counter
        bool stop = false;
        bool waited = !p.early_kv;
        while (!stop && walk.next()) {
            const int32_t *bt = p.block_table + (size_t)walk.pb * p.max_blocks;
            const int nblk = (seqC[walk.pb] * kChunk + kBlock - 1) / kBlock;
            int win = -1000000, my_blk = 0;
            const int cx1 = (int)(walk.xe - walk.s0);
            for (int cx = (int)(walk.xs - walk.s0); cx < cx1; ++kst) {
                const int ce = stage_end<FMT, NT>(cx, cx1);
                const int tok0 = cx * kChunk, ntok = (ce - cx) * kChunk;
                cx = ce;
                if (!waited && tok0 + ntok > seqL[walk.pb] - p.n_q) {
                    pdl_wait();  // the newest rows may come from the kernels before this one
                    waited = true;
                }
                const int bi = tok0 >> 8;
                if (bi >= win + 32) {  // warp-uniform refill of the window
                    win = bi;
                    my_blk = win + lane < nblk ? bt[win + lane] : -1;
                }
                const int blk = __shfl_sync(0xffffffffu, my_blk, bi - win);
                if (lane == 0) {
                    const int stage = (int)(kst % NS);
                    const uint32_t round = kst / NS;
                    if (!misc[0] && !mbar_wait(&empty[stage], (round & 1) ^ 1)) {
                        report(NF_DEVERR_TIMEOUT);
                        misc[0] = 1;
                    }
                    if (!misc[0]) {
                        unsigned char *st = smem + stage * ST::kStride;
                        if (blk < 0 || blk >= p.num_blocks) {
                            report(NF_DEVERR_BLOCK_ID);
                            stage_ok[stage] = 0;
                            mbar_arrive(&full[stage]);
                        } else {
                            stage_ok[stage] = 1;
                            const size_t si = ((size_t)blk * H + walk.ph) * kBlock + (tok0 & (kBlock - 1));
                            mbar_arrive_expect_tx(&full[stage], (uint32_t)(ntok * ST::kBytesPerTok));
                            if (K4) {
                                if (ntok == ST::kTok) {  // a whole stage: one box each
                                    tma_load_2d(st + ST::kK, &p.kmap_full, 0, (int)si, &full[stage]);
                                    tma_load_2d(st + ST::kV, &p.vmap_full, 0, (int)si, &full[stage]);
                                } else {
                                    for (int c = 0; c < ntok; c += kChunk) {
                                        tma_load_2d(st + ST::kK + c * 64, &p.kmap, 0, (int)si + c, &full[stage]);
                                        tma_load_2d(st + ST::kV + c * 64, &p.vmap, 0, (int)si + c, &full[stage]);
                                    }
                                }
                                bulk_g2s(st + ST::kKs, reinterpret_cast<const uint8_t *>(p.k_scales) + si * 4, ntok * 4,
                                         &full[stage]);
                                bulk_g2s(st + ST::kVs, reinterpret_cast<const uint8_t *>(p.v_scales) + si * 4, ntok * 4,
                                         &full[stage]);
                            } else if (K8) {
                                constexpr int vrow = V8 ? 128 : 64, vsc = V8 ? 1 : 4;  // V bytes, V scales per key
                                bulk_g2s(st + ST::kK, static_cast<const int8_t *>(p.k_codes) + si * 128, ntok * 128, &full[stage]);
                                if (ntok == ST::kTok)  // a whole stage: one box
                                    tma_load_2d(st + ST::kV, &p.vmap_full, 0, (int)si, &full[stage]);
                                else
                                    for (int c = 0; c < ntok; c += kChunk)
                                        tma_load_2d(st + ST::kV + c * vrow, &p.vmap, 0, (int)si + c, &full[stage]);
                                bulk_g2s(st + ST::kKs, p.k_scales + si, ntok * 2, &full[stage]);
                                bulk_g2s(st + ST::kVs, p.v_scales + si * vsc, ntok * 2 * vsc, &full[stage]);
                            } else {
                                bulk_g2s(st + ST::kK, static_cast<const __nv_bfloat16 *>(p.k_codes) + si * 128, ntok * 256, &full[stage]);
                                bulk_g2s(st + ST::kV, static_cast<const __nv_bfloat16 *>(p.v_codes) + si * 128, ntok * 256, &full[stage]);
                            }
                        }
                    }
                }
                if (__shfl_sync(0xffffffffu, misc[0], 0)) {
                    stop = true;
                    break;
                }
            }
        }
        if (lane == 0) {
            // before leaving, make sure no copy into this CTA's shared memory is
            // still in flight: wait for the buffers of the last round issued
            const uint32_t issued = kst;
            for (uint32_t kk = issued > (uint32_t)NS ? issued - NS : 0; kk < issued && !misc[0]; ++kk)
                if (!mbar_wait(&full[kk % NS], (kk / NS) & 1)) {
                    report(NF_DEVERR_TIMEOUT);
                    misc[0] = 1;
                }
        }
        return;  // the merge barriers below are among the consumer warps only
    }

    // =================================================================== consumers
    if (p.early_kv) {
        // the first piece's query rows into L2 while the kernels before this
        // one finish (no value is read before the wait)
        PieceWalker w0 = walk;
        if (w0.next()) prefetch_q_rows<QF32>(p, w0.pb, w0.ph, threadIdx.x);
        pdl_wait();
    }
    // segments of sequences with no valid key: o = 0, lse = -inf
    for (int s = blockIdx.x; s < p.batch * H; s += gridDim.x) {
        const int b = s / H, h = s % H;
        if (seqC[b] != 0) continue;
        for (int idx = threadIdx.x; idx < p.rows * kHeadDim; idx += kConsumerWarps * 32) {
            const int r = idx / kHeadDim, ch = idx % kHeadDim;
            const int j = r / p.group, gq = r % p.group;
            const size_t row = ((size_t)b * p.n_q + j) * p.num_q_heads + (size_t)h * p.group + gq;
            p.out[row * kHeadDim + ch] = 0.f;
            if (ch == 0 && p.out_lse) p.out_lse[row] = -INFINITY;
        }
    }

    const int CW = kConsumerWarps / p.n_rg;  // warps per row group
    const int rg = warp / CW, slot = warp % CW;
    const int g = lane >> 2, t = lane & 3;
    const int row0 = rg * NR;

    WarpState<NT, QF32, FMT> ws;
    LaneOffsets lo;
    if (V8) {
        lo.k = g * 128 + 32 * t;
        lo.ks = lo.vs = 0;
        // ldmatrix row address of lane l: key 8 ((l >> 3) & 1) + (l & 7) of the
        // m-tile, 16-byte column (l >> 4) stored at position (l >> 4) ^ (l & 7)
        // (128-byte swizzle; m-tiles start on 2048-byte boundaries)
        lo.v = (8 * (((uint32_t)lane >> 3) & 1u) + ((uint32_t)lane & 7u)) * 128 +
               ((((uint32_t)lane >> 4) ^ ((uint32_t)lane & 7u)) * 16);
    } else if (K4) {
        // ldmatrix row address of lane l: key l & 7 of an n-tile, 16-byte column
        // l >> 3 (a scale group) at position (l >> 3) ^ ((l & 7) >> 1) (64-byte
        // swizzle); the V nibbles likewise
        lo.k = (lane & 7) * 64 + ((((uint32_t)lane >> 3) ^ (((uint32_t)lane & 7) >> 1)) & 3u) * 16;
        lo.v = lo.k;
        lo.ks = lo.vs = 0;
    } else if (K8) {
        lo.k = g * 128 + 32 * t;
        lo.ks = 0;
        // the swizzled copy puts column c of key row r at position c ^ ((r >> 1) & 3)
        // (stage buffers and m-tiles start on 1024-byte boundaries of the V plane)
        lo.v = (lane & 7) * 64 + ((((uint32_t)lane >> 3) ^ (((uint32_t)lane & 7) >> 1)) & 3u) * 16;
        lo.vs = 16 * t;
    } else {
        lo.k = g * 256 + 16 * t;
        lo.v = lo.k;
        lo.ks = lo.vs = 0;
    }

    int stage = 0;
    uint32_t phase = 0;      // parity of the ring's current round
    uint32_t fin_phase = 0;  // parity of the final merge's copy barrier
    while (walk.next()) {
        const int b = walk.pb, h = walk.ph;
        const int L = seqL[b];  // (read once at the start; 0 for a sequence with no valid key)
        // query fragments of this (sequence, kv-head): lane (g, t) holds row g of
        // tile nt, channels 32t..32t+31 (int8 K: k-step ks takes channels 32t + 8ks
        // + 0..3 and + 4..7; fp8 K: 32t + 4ks + 0..3) or 32u + 8t + 4h + 0..3
        // (bf16 cache: k-step 2u + h)
        if (K8) {
            // The fragments are computed once per CTA into the (idle) merge buffer:
            // warp w encodes rows w, w + 8, ...; lane l takes channels 4l..4l+3.
            // int8 K: 4l..4l+3 = 32t + 8ks + 4hh + e (t = l / 8, ks = l / 2 % 4,
            // hh = l % 2); layout [row][t][ks][d1 word hh=0, d2 word hh=0, d1 word
            // hh=1, d2 word hh=1].  fp8 K: 4l..4l+3 = 32t + 4ks + e (t = l / 8,
            // ks = l % 8); layout [row][t][ks][hi e=0,1; lo e=0,1; hi e=2,3; lo
            // e=2,3] (an f16 A fragment: rows g hold hi, rows g + 8 lo).
            uint32_t *qsm = reinterpret_cast<uint32_t *>(sm_o);
            float *qwsm = reinterpret_cast<float *>(sm_o) + kMaxRows * (F8 ? 128 : 64);
            for (int r = warp; r < p.rows; r += kConsumerWarps) {
                const int j = r / p.group, gq = r % p.group;
                const size_t qoff =
                    (((size_t)b * p.n_q + j) * p.num_q_heads + (size_t)h * p.group + gq) * kHeadDim + 4 * lane;
                float x[4];
                if (QF32) {
                    const float4 v = *reinterpret_cast<const float4 *>(static_cast<const float *>(p.q) + qoff);
                    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
                } else {
                    const uint2 v = *reinterpret_cast<const uint2 *>(static_cast<const __nv_bfloat16 *>(p.q) + qoff);
                    x[0] = __uint_as_float(v.x << 16);
                    x[1] = __uint_as_float(v.x & 0xFFFF0000u);
                    x[2] = __uint_as_float(v.y << 16);
                    x[3] = __uint_as_float(v.y & 0xFFFF0000u);
                }
                float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
                if (F8) {
                    // q = s (hi + lo), s = max|q|: |q / s| <= 1 stays inside fp16,
                    // hi = fp16(q / s), lo = fp16(q / s - hi)
                    const float inv = amax > 0.f ? 1.0f / amax : 0.f;
                    float y[4], hi[4], lo[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        y[e] = x[e] * inv;
                        hi[e] = __half2float(__float2half_rn(y[e]));
                        lo[e] = y[e] - hi[e];
                    }
                    const uint4 frag = make_uint4(pack_f16(hi[0], hi[1]), pack_f16(lo[0], lo[1]), pack_f16(hi[2], hi[3]),
                                                  pack_f16(lo[2], lo[3]));
                    *reinterpret_cast<uint4 *>(qsm + (r * 4 + (lane >> 3)) * 32 + (lane & 7) * 4) = frag;
                    if (lane == 0) qwsm[r] = amax * p.scale_log2;
                    continue;
                }
                // q ~= s (d1 + d2 / 254), s = max|q| / 127, digits in [-127, 127]
                const float s1 = amax / 127.0f;
                const float inv = amax > 0.f ? 127.0f / amax : 0.f;
                uint32_t d1w = 0, d2w = 0;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float d1 = fminf(fmaxf(rintf(x[e] * inv), -127.f), 127.f);
                    const float r1 = fmaf(-d1, s1, x[e]);
                    const float d2 = fminf(fmaxf(rintf(r1 * inv * 254.0f), -127.f), 127.f);
                    d1w |= ((uint32_t)(int)d1 & 0xFFu) << (8 * e);
                    d2w |= ((uint32_t)(int)d2 & 0xFFu) << (8 * e);
                }
                if (K4) {
                    // channels 8m .. 8m + 7 (m = lane / 2 = 4i + t) form k-step i of
                    // lane t: its even channels in the first word of each digit pair,
                    // its odd ones in the second (the order of the expanded K nibbles)
                    const uint32_t p1 = __shfl_xor_sync(0xffffffffu, d1w, 1), p2 = __shfl_xor_sync(0xffffffffu, d2w, 1);
                    const bool odd = lane & 1;
                    const uint32_t w1 = odd ? prmt(p1, d1w, 0x7531) : prmt(d1w, p1, 0x6420);
                    const uint32_t w2 = odd ? prmt(p2, d2w, 0x7531) : prmt(d2w, p2, 0x6420);
                    const int m = lane >> 1;
                    uint32_t *dst = qsm + (r * 4 + (m & 3)) * 16 + (m >> 2) * 4 + (odd ? 2 : 0);
                    dst[0] = w1;
                    dst[1] = w2;
                    // the expanded K codes are 16 x code
                    if (lane == 0) qwsm[r] = s1 / 254.0f * p.scale_log2 * 0.0625f;
                    continue;
                }
                uint32_t *dst = qsm + (r * 4 + (lane >> 3)) * 16 + ((lane >> 1) & 3) * 4 + 2 * (lane & 1);
                dst[0] = d1w;
                dst[1] = d2w;
                if (lane == 0) qwsm[r] = s1 / 254.0f * p.scale_log2;
            }
            named_sync(1, kConsumerWarps * 32);
            {
                // the next piece's query rows into L2, ahead of its start
                PieceWalker nx = walk;
                if (nx.next()) prefetch_q_rows<QF32>(p, nx.pb, nx.ph, threadIdx.x);
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int r = row0 + nt * 8 + g;
                const bool rv = r < p.rows;
                constexpr int KS = F8 ? 8 : 4;
#pragma unroll
                for (int ks = 0; ks < KS; ++ks) {
                    const uint4 v = rv ? lds128(qsm + (r * 4 + t) * (4 * KS) + ks * 4) : make_uint4(0, 0, 0, 0);
                    ws.qa[nt][ks][0] = v.x; ws.qa[nt][ks][1] = v.y; ws.qa[nt][ks][2] = v.z; ws.qa[nt][ks][3] = v.w;
                }
                ws.qw[nt] = rv ? qwsm[r] : 0.f;
            }
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int r = row0 + nt * 8 + g;
            const bool rv = r < p.rows;
            if (!K8) {
                const int j = rv ? r / p.group : 0, gq = rv ? r % p.group : 0;
                const size_t qoff = (((size_t)b * p.n_q + j) * p.num_q_heads + (size_t)h * p.group + gq) * kHeadDim;
                float x[32];
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const size_t ch = qoff + 32 * (c >> 3) + 8 * t + (c & 7);
                    x[c] = !rv ? 0.f
                                : QF32 ? static_cast<const float *>(p.q)[ch]
                                       : __bfloat162float(static_cast<const __nv_bfloat16 *>(p.q)[ch]);
                }
#pragma unroll
                for (int w = 0; w < 16; ++w) {
                    // word w = 2 (2u + hh) + e2 holds channels 32u + 8t + 4hh + 2e2 + 0..1
                    const uint32_t hi = pack_bf16(x[2 * w], x[2 * w + 1]);
                    const uint32_t lo_ = QF32 ? pack_bf16(x[2 * w] - __uint_as_float(hi << 16),
                                                          x[2 * w + 1] - __uint_as_float(hi & 0xFFFF0000u))
                                              : 0u;
                    ws.qa[nt][w >> 1][2 * (w & 1)] = hi;
                    ws.qa[nt][w >> 1][2 * (w & 1) + 1] = lo_;
                }
                ws.qw[nt] = p.scale_log2;
            }
            ws.lim[nt] = !rv ? -1 : (p.causal ? L - p.n_q + r / p.group : L - 1);
            ws.m_run[nt] = -INFINITY;
            ws.l_run[nt] = 0.f;
#pragma unroll
            for (int m = 0; m < 8; ++m) ws.acc[m][nt][0] = ws.acc[m][nt][1] = ws.acc[m][nt][2] = ws.acc[m][nt][3] = 0.f;
        }
        // keys every row of the group sees, for the no-mask fast path
        const int all_see = p.causal ? L - p.n_q + 1 : L;

        const int cx1 = (int)(walk.xe - walk.s0);
        for (int cx = (int)(walk.xs - walk.s0); cx < cx1;) {
            const int ce = stage_end<FMT, NT>(cx, cx1);
            const int tok0 = cx * kChunk, n_units = (ce - cx) * (kChunk / (16 * MT));
            cx = ce;
            if (!misc[0] && !mbar_wait(&full[stage], phase)) {
                report(NF_DEVERR_TIMEOUT);
                misc[0] = 1;
            }
            if (!misc[0] && stage_ok[stage]) {
                const unsigned char *st = smem + stage * ST::kStride;
                for (int un = slot; un < n_units; un += CW) {
                    const int ub = 16 * MT * un;  // first key of the unit in the stage
                    if (tok0 + ub + 16 * MT <= all_see)
                        decode_unit<NT, MT, QF32, FMT, true>(ws, st, ub, tok0, L, lane, lo);
                    else
                        decode_unit<NT, MT, QF32, FMT, false>(ws, st, ub, tok0, L, lane, lo);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
            if (++stage == NS) {
                stage = 0;
                phase ^= 1u;
            }
        }

        // ---- merge the consumer warps of each row group (shared memory)
        const int s_id = b * H + h;
        const int first = owner_cta(walk.s0, W, P);
        const int last = owner_cta(walk.s0 + seqC[b] - 1, W, P);
        const int n_pieces = last - first + 1;
        const int rows_here = p.rows;
        // every warp's raw accumulators, and its rows' (m, l), into shared memory
        {
            float *buf = sm_o + warp * NR * 132;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                float l = ws.l_run[nt];
                l += __shfl_xor_sync(0xffffffffu, l, 1);
                l += __shfl_xor_sync(0xffffffffu, l, 2);
                if (t == 0) {
                    sm_m[warp * NR + nt * 8 + g] = ws.m_run[nt];
                    sm_l[warp * NR + nt * 8 + g] = l;
                }
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int rr = nt * 8 + 2 * t + e;
#pragma unroll
                    for (int m = 0; m < 8; ++m) {
                        const int c0 = V8 ? v_channel_k8v8(m, g) : K8 ? v_channel_k8v4(m, g) : v_channel_bf16(m, g);
                        const int c1 = V8 ? v_channel_k8v8(m, g + 8)
                                          : K8 ? v_channel_k8v4(m, g + 8) : v_channel_bf16(m, g + 8);
                        buf[rr * 132 + c0] = ws.acc[m][nt][e];
                        buf[rr * 132 + c1] = ws.acc[m][nt][2 + e];
                    }
                }
            }
        }
        named_sync(1, kConsumerWarps * 32);
        {
            // per (row, 4 channels): o = sum_w 2^(m_w - M) acc_w / sum_w 2^(m_w - M) l_w
            // over the row group's warps (M = max_w m_w; the weights were taken
            // relative to m + kLazy, so lse = (M + kLazy + log2 of the sum) ln 2)
            const int tid = slot * 32 + lane, nthr = CW * 32;
            float *slotp = p.partials + (size_t)(s_id + vb) * p.slot_floats;
            for (int idx = tid; idx < NR * (kHeadDim / 4); idx += nthr) {
                const int rr = idx / (kHeadDim / 4), c4 = idx % (kHeadDim / 4);
                const int r = row0 + rr;
                if (r >= rows_here) continue;
                float M = -INFINITY;
                for (int w = 0; w < CW; ++w) M = fmaxf(M, sm_m[(rg * CW + w) * NR + rr]);
                float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
                float lse = -INFINITY;
                if (M != -INFINITY) {
                    float den = 0.f;
                    for (int w = 0; w < CW; ++w) {
                        const float f = ex2(sm_m[(rg * CW + w) * NR + rr] - M);
                        den = fmaf(f, sm_l[(rg * CW + w) * NR + rr], den);
                        const float4 x = *reinterpret_cast<const float4 *>(sm_o + ((rg * CW + w) * NR + rr) * 132 + 4 * c4);
                        o.x = fmaf(f, x.x, o.x); o.y = fmaf(f, x.y, o.y); o.z = fmaf(f, x.z, o.z); o.w = fmaf(f, x.w, o.w);
                    }
                    const float inv = __frcp_rn(den);
                    o.x *= inv; o.y *= inv; o.z *= inv; o.w *= inv;
                    if (c4 == 0) lse = (M + kLazy + log2f(den)) * 0.69314718055994531f;
                }
                if (n_pieces == 1) {
                    const int j = r / p.group, gq = r % p.group;
                    const size_t row = ((size_t)b * p.n_q + j) * p.num_q_heads + (size_t)h * p.group + gq;
                    reinterpret_cast<float4 *>(p.out + row * kHeadDim)[c4] = o;
                    if (c4 == 0 && p.out_lse) p.out_lse[row] = lse;
                } else {
                    reinterpret_cast<float4 *>(slotp + r * kHeadDim)[c4] = o;
                    if (c4 == 0) slotp[rows_here * kHeadDim + r] = lse;
                }
            }
        }
        named_sync(1, kConsumerWarps * 32);
        PieceWalker rest = walk;
        const bool more = rest.next();  // another piece follows: its stages may be in the ring
        finish_piece_single<kConsumerWarps * 32, 1>(p, s_id, first, n_pieces, rows_here, b, h, !more, smem,
                                                    NS * ST::kStride, fin_bar, fin_phase, sm_o, SM::kMergeFloats,
                                                    misc);
    }
}

}  // namespace nf
