// nf_decode_tc.cuh -- split-K decode attention over the K8/V4 (or the int8
// K8V8, or the fp8) pool for many query rows per kv-head, on the 5th-generation
// tensor cores (tcgen05).  K8V8 differs only in the V side: 128-byte rows of
// int8 codes with one fp16 scale per key, dequantised in channel order, and
// three ring stages instead of four.  fp8 has the K8V8 layout with e4m3 codes;
// its S = K . Q^T runs on kind::f8f6f4 against the query row in three e4m3
// parts, q ~= s (p1 + p2 / 16 + p3 / 256) with s = max|q|, each part the e4m3
// rounding of what the earlier parts leave (times 16), into three fp32
// columns per row (2^-12 of max|q| per element and better).
//
// MTP draft verification is the engine's normal decode step: 1 + 3 query
// tokens per step (page "3090 单卡跑 Qwen3.8-27B：NInfer 上机实测", section
// 一.3, --spec mtp --draft-tokens 3), each with the G query heads of a GQA
// group, so a kv-head serves G * n_q = 32 rows (G = 8).  The work per key then
// grows with the rows (two products of 128 channels per row and key), and on
// the per-warp mma.sync path it outgrows the HBM time.  Here the products run
// as whole-tile tcgen05 MMAs, each stream issued by one thread of its own
// warp, with the accumulators in tensor memory, and the CUDA cores only do
// the softmax and the V dequantisation.  The work cut, the split partials and the last-ticket merge
// are those of decode_kernel (nf_decode.cuh); results and workspace layout are
// the same.
//
// Per tile of up to 128 keys (never crossing a 256-key block):
//   S^T = K . Q^T       kind::i8, M = 128 keys, N = 2 RP (the query rows'
//                       high int8 digits, then their low digits), K = 128
//                       channels; A = the int8 K codes as the TMA brought them
//                       (128-byte swizzle), B = the query digits.
//   softmax             one thread per key (its tensor-memory lane): x_r =
//                       (d1_r * 254 + d2_r) * qw_r * kscale for each row r;
//                       lazy running max per row (raised, and O rescaled, only
//                       when a tile exceeds it by 2^4); weights p = 2^(x - m - 4)
//                       <= 1, times the key's power-of-two V factor f_k, as
//                       fp16 P' [key][row].
//   V dequantisation    one thread per key: code x (V scale / f_k) as fp16 V'
//                       [key][channel]; f_k = 2^(E - 15) with E the largest
//                       exponent of the key's V scales (four, or K8V8's one),
//                       so V' < 14 (K8V8: < 254) and P' <= 2^15 both stay
//                       inside fp16 for any fp16 scale, and P' x V' = p x code
//                       x scale.
//   O^T += V'^T . P'    kind::f16, M = 128 channels, N = 64 (rows, padded),
//                       K = 128 keys; A = V' and B = P', both MN-major
//                       (128-byte swizzle); O^T lives in tensor memory.
// Roles (20 warps): warps 0-15 are alike -- warp (q, h) = (w % 4, w / 4)
// takes the keys (and O^T channel lanes) of tensor-memory quadrant q,
// dequantises their V' channels of scale group h and runs the softmax of a
// quarter of the rows; it reads its slice of a stage and releases the stage at
// once.  Four such warps share each SM sub-partition, so one's latency hides
// behind the others' work.  Warp 16 is the TMA producer; warp 17 holds the
// tensor memory and issues the S MMAs; warps 18 and 19 issue the P.V MMAs of
// the even and the odd tiles, each issuer on one thread.  The issue streams
// sit one on each sub-partition: issuing an MMA takes issue cycles from the
// consumer warps beside it, and the row-group barrier waits for the slowest
// of its four warps, one per sub-partition.  Warps 0-15 also encode the query
// digits at each piece's start and run the segment's final merge.  Every
// mbarrier wait is bounded (2 s); a timeout records NF_DEVERR_TIMEOUT and
// every role runs to its end without further waits.
#pragma once

#include <cfloat>

#include "nf_decode.cuh"
#include "nf_tc.cuh"

namespace nf {

constexpr int kDtConsumers = 16;                   // consumer warps
constexpr int kDtRowGroups = kDtConsumers / 4;     // warps of one tensor-memory quadrant: row groups
constexpr int kDtVG = 4 / kDtRowGroups;            // V scale groups (32 channels) per consumer warp
constexpr int kDtThreads = (kDtConsumers + 4) * 32;  // + producer, S-issue and two P.V-issue warps
// one extra warp on each sub-partition (warp w runs on w % 4); the P.V
// issuers take the even and the odd tiles
constexpr int kDtProducer = kDtConsumers, kDtMma = kDtConsumers + 1, kDtPv = kDtConsumers + 2;
constexpr int kDtStages = 4;
constexpr int kDtTileKeys = 128;  // keys of a full tile: one TMA box of K and one of V rows
constexpr int kDtPvN = 64;       // N of the P.V product: the rows, padded
constexpr int kDtMaxRows = 32;   // rows per kv-head this kernel serves
constexpr int kDtChunkTiles = kBlock / kChunk;
// Segment padding of the work cut (see kSegPad): a piece's set-up and merge
// cost about 4 us here, 12 chunks of this kernel's streaming.
constexpr int kDtSegPad = 12;
// named barriers: 2..5 the four warps of one row quarter, 6 all consumer
// warps (also the final merge's)
constexpr uint32_t kDtBarAll = 6;

// Shared-memory layout for the pool format FMT: NF_KV_K8V4, NF_KV_K8V8 or NF_KV_F8.
template <int FMT>
struct DtSmem {
    // one ring stage: K codes [128 keys][128 B] (128-byte swizzle); V codes
    // [128 keys][64 B nibbles] (64-byte swizzle, K8/V4) or [128 keys][128 B]
    // (128-byte swizzle, K8V8); K scales fp16 [128]; V scales fp16 [128][4]
    // (K8/V4) or [128] (K8V8).  Three K8V8 stages fit beside the other buffers.
    static constexpr bool kF8 = FMT == NF_KV_F8;                // e4m3 K and V codes
    static constexpr bool kV8 = FMT == NF_KV_K8V8 || kF8;       // 128-byte V rows, one V scale per key
    static constexpr int kQBuf = kF8 ? 12288 : 8192;            // query operand rows (2 or 3 per row) x 128 B
    static constexpr int kVRow = kV8 ? 128 : 64, kVScales = kV8 ? 1 : 4;
    static constexpr int kStages = kV8 ? 3 : kDtStages;
    static constexpr int kStK = 0, kStV = 16384, kStKs = kStV + 128 * kVRow, kStVs = kStKs + 256;
    static constexpr int kStride = (kStVs + 128 * 2 * kVScales + 1023) / 1024 * 1024;
    static constexpr int kBytesPerTok = 128 + kVRow + 2 + 2 * kVScales;
    static constexpr int kRingBytes = kStages * kStride;
    static constexpr int kVh = kRingBytes;        // fp16 V' [2 buffers][2 blocks of 64 channels][128 keys][128 B]
    static constexpr int kP = kVh + 2 * 32768;    // fp16 P' [2 buffers][128 keys][64 rows x 2 B]
    static constexpr int kQ = kP + 2 * 16384;     // query operand [2 buffers][64 int8 digit rows or 96 e4m3 part rows][128 B]
    static constexpr int kQw = kQ + 2 * kQBuf;    // float [2][kDtMaxRows]: row factors
    static constexpr int kRed = kQw + 2 * kDtMaxRows * 4;   // float [4 quadrants][kDtMaxRows]: row maxima
    static constexpr int kRed2 = kRed + 4 * kDtMaxRows * 4; // float [4 quadrants][kDtMaxRows]: row sums
    static constexpr int kBars = kRed2 + 4 * kDtMaxRows * 4;
    static constexpr int kNumBars = 2 * kStages + 10 + 1;
    static constexpr int kStageOk = kBars + kNumBars * 8;   // int [stages]
    static constexpr int kTmem = kStageOk + kStages * 4;    // u32
    static constexpr int kSeqC = (kTmem + 4 + 15) / 16 * 16;  // int [kMaxBatch]
    static constexpr int kSeqL = kSeqC + kMaxBatch * 4;       // int [kMaxBatch]
    static constexpr int kSeqBase = kSeqL + kMaxBatch * 4;    // i64 [kMaxBatch + 1]
    static constexpr int kMisc = kSeqBase + (kMaxBatch + 1) * 8;  // int [4]
    static constexpr int kPiece = kMisc + 16;                     // DtPiece: the consumers' current piece
    static constexpr int kWalk = kPiece + 32;                     // DtWalk: the consumers' walker
    static constexpr int kBytes = kWalk + 144;
    static_assert(kBytes <= 232448, "shared memory per CTA");
    static_assert(kStride % 1024 == 0 && kVh % 1024 == 0 && kP % 1024 == 0 && kQ % 1024 == 0, "swizzle atoms");
    // the final merge's scratch in the idle V' buffers
    static_assert(2 * 32768 / 4 >= (kDtConsumers + 3) * kMaxCtas + 4 * kDtConsumers * 32, "final-merge scratch");
};

// A piece as the consumer warps see it: read from shared memory at its start,
// so that the walker over the CTA's range holds no registers in the tile loop.
struct DtPiece {
    int valid, b, h, cx0, cx1;  // sequence, kv-head, chunks [cx0, cx1) of the segment
    int first, n, m;            // the segment's first CTA, its pieces, the final merge's shares
};
// The consumers' walker over the CTA's range and the work cut it follows (W
// chunks, padding included, over P CTAs), in shared memory.
struct DtWalk {
    PieceWalker w;
    long long W;
    int P;
};
static_assert(sizeof(DtWalk) <= 144, "walker slot");

// Advances the consumers' walker (one thread, in shared memory) to the next
// piece and describes it: n pieces of the segment from CTA `first`, m of them
// on CTAs with no further work (see finish_piece_coop).
__device__ __forceinline__ void dt_next_piece(DtWalk *dw, DtPiece *pd) {
    PieceWalker *wk = &dw->w;
    const long long W = dw->W;
    const int P = dw->P;
    if (!wk->next()) {
        pd->valid = 0;
        return;
    }
    const long long s0 = wk->s0;
    const int C = wk->C[wk->pb];
    const int first = owner_cta(s0, W, P), last = owner_cta(s0 + C - 1, W, P);
    // the last piece's CTA goes on into the next segment (see decode_kernel)
    const bool cont = W * (last + 1) / P > s0 + C + kDtSegPad;
    pd->b = wk->pb;
    pd->h = wk->ph;
    pd->cx0 = (int)(wk->xs - s0);
    pd->cx1 = (int)(wk->xe - s0);
    pd->first = first;
    pd->n = last - first + 1;
    pd->m = last - first + 1 - (cont ? 1 : 0);
    pd->valid = 1;
}

// End (exclusive, in chunks) of the tile that starts at chunk cx: at most 128
// keys, never crossing a 256-key block.
__device__ __forceinline__ int dt_tile_end(int cx, int cx_end) {
    return min(cx_end, min((cx / kDtChunkTiles + 1) * kDtChunkTiles, cx + 128 / kChunk));
}

// The largest exponent field E (at least 1) of a key's four fp16 V scales:
// V' = code x scale x 2^(15 - E) and f = 2^(E - 15) (both sides must agree).
__device__ __forceinline__ int dt_v_exponent(uint2 vs) {
    const uint32_t a = max(vs.x & 0x7FFFu, (vs.x >> 16) & 0x7FFFu);
    const uint32_t c = max(vs.y & 0x7FFFu, (vs.y >> 16) & 0x7FFFu);
    return max((int)(max(a, c) >> 10), 1);
}

// Barrier with an OR reduction over `count` threads (named barrier `id`).
__device__ __forceinline__ bool bar_red_or(uint32_t id, uint32_t count, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}\n"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(count)
        : "memory");
    return r != 0;
}

// Output channel of tensor-memory lane m of O^T: each 8-channel chunk of V'
// holds the nibble-unpacking order (0, 4, 1, 5, 2, 6, 3, 7).
__device__ __forceinline__ int dt_channel(int m) {
    const int q = m & 7;
    return (m & ~7) | ((q >> 1) + 4 * (q & 1));
}

// bounded waits shared by all roles: skipped once the kernel has aborted
__device__ __forceinline__ void dt_wait(uint64_t *bar, uint32_t parity, volatile int *misc) {
    if (mbar_try_wait(bar, parity)) return;
    if (!misc[0] && !mbar_wait_spin(bar, parity)) {
        report(NF_DEVERR_TIMEOUT);
        misc[0] = 1;
    }
}

// HR consecutive tensor-memory columns of the warp's lanes (HR = 4 or 8)
template <int HR>
__device__ __forceinline__ void dt_ld(uint32_t taddr, uint32_t (&r)[HR]) {
    if constexpr (HR == 16) tmem_ld16(taddr, r); else if constexpr (HR == 8) tmem_ld8(taddr, r); else tmem_ld4(taddr, r);
}
template <int HR>
__device__ __forceinline__ void dt_st(uint32_t taddr, const uint32_t (&r)[HR]) {
    if constexpr (HR == 16) tmem_st16(taddr, r); else if constexpr (HR == 8) tmem_st8(taddr, r); else tmem_st4(taddr, r);
}

// One consumer warp's softmax of one tile for its HR rows: scores from the S
// columns, the lazy running max (a collective step of the four warps of the
// rows when some score exceeds it by kLazy), the weights times f into P'.
// Each row keeps nthr = -max(m + kLazy, -FLT_MAX), FLT_MAX while the row has
// no max yet, so one FMA per score gives the exponent y = x - m - kLazy (a
// score's x = v c with v its integer dot product and c the row's and key's
// factors) and y > 0 flags a score above the threshold.
// FAST: every row sees every key of the tile (no mask).
// When the max rises and O^T holds earlier tiles of the piece (has_o), the
// rows' columns of O^T (taddr) are scaled once the last P.V is done (pv_bar).
// The raw product of a row and key from the S words: int8 digits S1 * 254 +
// S2, or e4m3 parts S1 + S2 / 16 + S3 / 256 (fp32 accumulators).
template <bool F8>
__device__ __forceinline__ float dt_product(uint32_t w1, uint32_t w2, uint32_t w3) {
    if constexpr (F8)
        return fmaf(__uint_as_float(w3), 0.00390625f, fmaf(__uint_as_float(w2), 0.0625f, __uint_as_float(w1)));
    else
        return (float)((int)w1 * 254 + (int)w2);
}

template <int HR, bool FAST, bool F8>
__device__ __forceinline__ void dt_softmax(const uint32_t (&d1)[HR], const uint32_t (&d2)[HR], const uint32_t (&d3)[HR],
                                           const float *qwr,
                                           float ksv, int rmin, int R, int r0, float (&nthr)[HR], float (&l_part)[HR],
                                           float *red, int qd, int lane, uint32_t gbar, float f,
                                           uint32_t (&pk)[HR / 2], bool has_o, uint32_t taddr, uint64_t *pv_bar,
                                           uint32_t pv_parity, volatile int *misc) {
    float c[HR], y[HR];
    bool raise = false;
#pragma unroll
    for (int e = 0; e < HR; e += 4) {
        const float4 w = *reinterpret_cast<const float4 *>(qwr + e);  // (rows >= R: never used unmasked)
        c[e] = w.x * ksv;
        c[e + 1] = w.y * ksv;
        c[e + 2] = w.z * ksv;
        c[e + 3] = w.w * ksv;
    }
#pragma unroll
    for (int e = 0; e < HR; ++e) {
        const float v = dt_product<F8>(d1[e], d2[e], d3[e]);
        y[e] = (FAST || (r0 + e >= rmin && r0 + e < R)) ? fmaf(v, c[e], nthr[e]) : -INFINITY;
        raise |= y[e] > 0.f;  // true when no max yet and the score finite
    }
    raise = bar_red_or(gbar, 128, raise);
    if (raise) {
        // the scores themselves (y loses them while a row has no max)
        float x[HR];
#pragma unroll
        for (int e = 0; e < HR; ++e)
            x[e] = (FAST || (r0 + e >= rmin && r0 + e < R)) ? dt_product<F8>(d1[e], d2[e], d3[e]) * c[e] : -INFINITY;
        // row maxima of the tile over its 128 keys: the four warps of these rows
#pragma unroll
        for (int e = 0; e < HR; ++e) {
            float mx = x[e];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            if (lane == 0) red[qd * kDtMaxRows + r0 + e] = mx;
        }
        named_sync(gbar, 128);
        // every thread of the four warps derives the same new maxima
        float alpha[HR];
        bool rescale = false;
#pragma unroll
        for (int e = 0; e < HR; ++e) {
            const int r = r0 + e;
            const float tm = fmaxf(fmaxf(red[r], red[kDtMaxRows + r]), fmaxf(red[2 * kDtMaxRows + r], red[3 * kDtMaxRows + r]));
            const float m_old = nthr[e] == FLT_MAX ? -INFINITY : -nthr[e] - kLazy;
            const float m_new = fmaxf(m_old, tm);
            alpha[e] = m_old == -INFINITY ? 0.f : ex2(m_old - m_new);
            rescale |= m_new > m_old && m_old != -INFINITY;
            l_part[e] *= alpha[e];
            nthr[e] = -fmaxf(m_new + kLazy, -FLT_MAX);
            y[e] = x[e] + nthr[e];
        }
        if (rescale && has_o) {  // the same decision in the four warps of the rows
            dt_wait(pv_bar, pv_parity, misc);
            tc_fence_after();
            uint32_t o[HR];
            dt_ld<HR>(taddr, o);
            tmem_wait_ld_tied<HR>(o);
#pragma unroll
            for (int e = 0; e < HR; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha[e]);
            dt_st<HR>(taddr, o);
            tmem_wait_st();
        }
    }
    // weights 2^y <= 1 (the row sum), times f into P'; a row with no max yet
    // has only -inf scores, and y = -inf gives 0
#pragma unroll
    for (int e = 0; e < HR; e += 2) {
        const float p0 = ex2(y[e]), p1 = ex2(y[e + 1]);
        l_part[e] += p0;
        l_part[e + 1] += p1;
        pk[e / 2] = pack_f16(p0 * f, p1 * f);
    }
}

template <int RP, bool QF32, int FMT>
__global__ void __launch_bounds__(kDtThreads, 1) decode_tc_kernel(const __grid_constant__ DecodeParams p) {
    static_assert(RP == 16 || RP == 32, "rows padded to 16 or 32");
    static_assert(FMT == NF_KV_K8V4 || FMT == NF_KV_K8V8 || FMT == NF_KV_F8, "int8 or e4m3 K codes");
    using SM = DtSmem<FMT>;
    constexpr bool V8 = SM::kV8;  // int8 or e4m3 V codes, one V scale per key
    constexpr bool F8 = SM::kF8;  // e4m3 K: S = K . Q^T on kind::f8f6f4 with the query in three e4m3 parts
    constexpr int NS = SM::kStages;
    constexpr int HR = RP / kDtRowGroups;                         // rows per consumer warp
    constexpr int NSC = (F8 ? 3 : 2) * RP;                        // S columns per buffer
    constexpr uint32_t kIdescS = F8 ? umma_idesc_e4m3(128, NSC) : umma_idesc_s8(128, NSC);
    constexpr uint32_t kIdescO = umma_idesc_f16(128, kDtPvN, true, true);
    constexpr uint32_t kSCol = (F8 && RP == 32) ? 96 : 64;        // S buffer b at columns kSCol b
    constexpr uint32_t kOCol = 2 * kSCol;                         // O^T: 64 columns from kOCol (<= 256)
    extern __shared__ __align__(1024) unsigned char smem[];
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + SM::kBars);
    uint64_t *full = bars, *empty = bars + NS;
    uint64_t *sfull = bars + 2 * NS, *sfree = sfull + 2, *pfull = sfree + 2;
    uint64_t *pvdone = pfull + 2, *qfull = pvdone + 2, *drain = qfull + 2;
    volatile int *stage_ok = reinterpret_cast<volatile int *>(smem + SM::kStageOk);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + SM::kTmem);
    int *seqC = reinterpret_cast<int *>(smem + SM::kSeqC);
    int *seqL = reinterpret_cast<int *>(smem + SM::kSeqL);
    long long *seqBase = reinterpret_cast<long long *>(smem + SM::kSeqBase);
    volatile int *misc = reinterpret_cast<volatile int *>(smem + SM::kMisc);  // [0] abort, [1] last ticket
    float *qw_sm = reinterpret_cast<float *>(smem + SM::kQw);
    float *red = reinterpret_cast<float *>(smem + SM::kRed);
    float *red2 = reinterpret_cast<float *>(smem + SM::kRed2);

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int H = p.num_kv_heads;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NS; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1 + kDtConsumers * 32);  // the S MMA's commit and every consumer thread
            stage_ok[i] = 0;
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sfull[i], 1);
            // every consumer thread arrives on its own (its accesses are ordered
            // before its arrival): no warp convergence or elected lane per tile
            mbar_init(&sfree[i], kDtConsumers * 32);
            mbar_init(&pfull[i], kDtConsumers * 32);  // V' and P' of a tile written
            mbar_init(&pvdone[i], 1);
            mbar_init(&qfull[i], 1);
        }
        mbar_init(drain, 3);  // the S and the two P.V issuers' last commits
        misc[0] = 0;
        misc[1] = 0;
        // the swizzled operands need 1024-byte alignment of the shared window
        if (smem_addr(smem) & 1023u) {
            if (blockIdx.x == 0) report(NF_DEVERR_INTERNAL);
            misc[0] = 1;
        }
        fence_mbar_init();
    }
    // the query-digit buffers' padding rows stay zero
    for (int i = threadIdx.x; i < 2 * SM::kQBuf / 16; i += kDtThreads)
        reinterpret_cast<uint4 *>(smem + SM::kQ)[i] = make_uint4(0, 0, 0, 0);
    fence_async_smem();
    if (warp == kDtMma) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
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
                acc += seqC[b] ? (long long)(seqC[b] + kDtSegPad) * H : 0;
            }
            seqBase[p.batch] = acc;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const long long W = seqBase[p.batch];
    const int P = (int)(W < (long long)gridDim.x ? W : (long long)gridDim.x);
    // ranges in reverse order of the CTAs (see decode_kernel)
    const int vb = (int)blockIdx.x < P ? P - 1 - (int)blockIdx.x : (int)blockIdx.x;
    const long long c_begin = vb < P ? W * vb / P : 0;
    const long long c_end = vb < P ? W * (vb + 1) / P : 0;
    PieceWalker walk{seqC, seqBase, H, p.batch, kDtSegPad, c_begin, c_end};

    if (warp == kDtProducer) {
        // =============================================================== producer
        uint32_t kst = 0;
        bool stop = false;
        bool waited = !p.early_kv;
        while (!stop && walk.next()) {
            const int32_t *bt = p.block_table + (size_t)walk.pb * p.max_blocks;
            const int nblk = (seqC[walk.pb] * kChunk + kBlock - 1) / kBlock;
            int win = -1000000, my_blk = 0;
            const int cx1 = (int)(walk.xe - walk.s0);
            for (int cx = (int)(walk.xs - walk.s0); cx < cx1; ++kst) {
                const int ce = dt_tile_end(cx, cx1);
                const int tok0 = cx * kChunk, ntok = (ce - cx) * kChunk;
                cx = ce;
                if (!waited && tok0 + ntok > seqL[walk.pb] - p.n_q) {
                    pdl_wait();  // the newest rows may come from the kernels before this one
                    waited = true;
                }
                const int bi = tok0 >> 8;
                if (bi >= win + 32) {
                    win = bi;
                    my_blk = win + lane < nblk ? bt[win + lane] : -1;
                }
                const int blk = __shfl_sync(0xffffffffu, my_blk, bi - win);
                if (lane == 0) {
                    const int stage = (int)(kst % NS);
                    dt_wait(&empty[stage], ((kst / NS) & 1) ^ 1, misc);
                    if (!misc[0]) {
                        unsigned char *st = smem + stage * SM::kStride;
                        if (blk < 0 || blk >= p.num_blocks) {
                            report(NF_DEVERR_BLOCK_ID);
                            stage_ok[stage] = 0;
                            mbar_arrive(&full[stage]);
                        } else {
                            stage_ok[stage] = 1;
                            const size_t si = ((size_t)blk * H + walk.ph) * kBlock + (tok0 & (kBlock - 1));
                            // one box of 128 K rows and one of 128 V rows, whatever ntok: a
                            // shorter tile's extra rows (the next rows of the plane, or the
                            // fill past its end) are never used unmasked
                            mbar_arrive_expect_tx(&full[stage], (uint32_t)(kDtTileKeys * (128 + SM::kVRow) +
                                                                           ntok * (2 + 2 * SM::kVScales)));
                            tma_load_2d(st + SM::kStK, &p.kmap, 0, (int)si, &full[stage]);
                            tma_load_2d(st + SM::kStV, &p.vmap, 0, (int)si, &full[stage]);
                            bulk_g2s(st + SM::kStKs, p.k_scales + si, ntok * 2, &full[stage]);
                            bulk_g2s(st + SM::kStVs, p.v_scales + si * SM::kVScales, ntok * 2 * SM::kVScales,
                                     &full[stage]);
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
            // no copy into this CTA's shared memory may be in flight at exit
            for (uint32_t kk = kst > (uint32_t)NS ? kst - NS : 0; kk < kst && !misc[0]; ++kk)
                dt_wait(&full[kk % NS], (kk / NS) & 1, misc);
        }
    } else if (warp == kDtMma) {
        // =============================================================== S issue
        // S of tile kt once its stage is full, its S buffer free and, at a
        // piece's first tile, the piece's query digits written.  The two
        // streams of MMAs (S here, P.V on warp kDtPv) are issued from different
        // sub-partitions, as is the producer's TMA work.
        if (lane == 0) {
            const uint32_t sRing = smem_addr(smem), sQ = smem_addr(smem + SM::kQ);
            uint32_t kt = 0, pc = 0;
            while (!misc[0] && walk.next()) {
                dt_wait(&qfull[pc & 1], (pc >> 1) & 1, misc);
                const uint32_t qaddr = sQ + (pc & 1) * (uint32_t)SM::kQBuf;
                const int cx1 = (int)(walk.xe - walk.s0);
                for (int cx = (int)(walk.xs - walk.s0); cx < cx1 && !misc[0]; ++kt) {
                    cx = dt_tile_end(cx, cx1);
                    const uint32_t stage = kt % NS, sb = kt & 1;
                    dt_wait(&full[stage], (kt / NS) & 1, misc);
                    dt_wait(&sfree[sb], ((kt >> 1) & 1) ^ 1, misc);
                    if (misc[0]) break;
                    tc_fence_after();
                    const uint32_t kaddr = sRing + stage * SM::kStride + SM::kStK;
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                        if constexpr (F8)
                            umma_e4m3(tmem + sb * kSCol, umma_desc_sw128(kaddr + 32 * ks, 16, 1024),
                                      umma_desc_sw128(qaddr + 32 * ks, 16, 1024), kIdescS, ks > 0 ? 1u : 0u);
                        else
                            umma_s8(tmem + sb * kSCol, umma_desc_sw128(kaddr + 32 * ks, 16, 1024),
                                    umma_desc_sw128(qaddr + 32 * ks, 16, 1024), kIdescS, ks > 0 ? 1u : 0u);
                    }
                    umma_commit(&sfull[sb]);
                    umma_commit(&empty[stage]);  // the stage's K codes are consumed
                }
                ++pc;
            }
            umma_commit(drain);  // arrives once every MMA this thread issued has completed
        }
    } else if (warp == kDtPv || warp == kDtPv + 1) {
        // =============================================================== P.V issue
        // P.V of tile j once V' and P' of j are written, tile j on warp
        // kDtPv + (j & 1) -- so that buffer b = j & 1 and its pvdone[b] belong
        // to one issuer -- and only after P.V of tile j - 1 has completed, so
        // that O^T accumulates in tile order; a piece's first tile overwrites O^T.
        if (lane == 0) {
            const uint32_t mine = (uint32_t)(warp - kDtPv);
            const uint32_t sVh = smem_addr(smem + SM::kVh), sP = smem_addr(smem + SM::kP);
            uint32_t pj = 0;
            while (!misc[0] && walk.next()) {
                const int cx1 = (int)(walk.xe - walk.s0);
                bool ovw = true;
                for (int cx = (int)(walk.xs - walk.s0); cx < cx1 && !misc[0]; ++pj) {
                    cx = dt_tile_end(cx, cx1);
                    const uint32_t b = pj & 1;
                    if (b == mine) {
                        dt_wait(&pfull[b], (pj >> 1) & 1, misc);
                        if (pj > 0) dt_wait(&pvdone[b ^ 1], ((pj - 1) >> 1) & 1, misc);
                        if (misc[0]) break;
                        tc_fence_after();
                        const uint64_t ad = umma_desc_sw128(sVh + b * 32768u, 16384, 1024);
                        const uint64_t bd = umma_desc_sw128(sP + b * 16384u, 16384, 1024);
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)  // + 2048 bytes along K: + 128 in the address field
                            umma_f16(tmem + kOCol, ad + 128u * kk, bd + 128u * kk, kIdescO, (ovw && kk == 0) ? 0u : 1u);
                        umma_commit(&pvdone[b]);
                    }
                    ovw = false;
                }
            }
            umma_commit(drain);
        }
    } else {
        // =============================================================== warps 0-15
        // Warp (q, h) = (warp % 4, warp / 4): tensor-memory lane quadrant q, so
        // key 32 q + lane of each tile (the lane of S) and channel lane 32 q +
        // lane of O^T; rows h HR .. h HR + HR - 1 of the softmax, P' and O^T; and
        // the kDtVG V scale groups h kDtVG .. of 32 channels in the dequantisation.
        DtPiece *pd = reinterpret_cast<DtPiece *>(smem + SM::kPiece);
        DtWalk *wk = reinterpret_cast<DtWalk *>(smem + SM::kWalk);
        if (threadIdx.x == 0) {
            wk->w = walk;
            wk->W = W;
            wk->P = P;
            dt_next_piece(wk, pd);
        }
        named_sync(kDtBarAll, kDtConsumers * 32);
        if (p.early_kv) {
            // the first piece's query rows into L2 while the kernels before
            // this one finish (no value is read before the wait)
            if (pd->valid) prefetch_q_rows<QF32>(p, pd->b, pd->h, threadIdx.x);
            pdl_wait();
        }
        // segments of sequences with no valid key: o = 0, lse = -inf
        for (int s = blockIdx.x; s < p.batch * H; s += gridDim.x) {
            const int b = s / H, h = s % H;
            if (seqC[b] != 0) continue;
            for (int idx = threadIdx.x; idx < p.rows * kHeadDim; idx += kDtConsumers * 32) {
                const int r = idx / kHeadDim, ch = idx % kHeadDim;
                const int j = r / p.group, gq = r % p.group;
                const size_t row = ((size_t)b * p.n_q + j) * p.num_q_heads + (size_t)h * p.group + gq;
                p.out[row * kHeadDim + ch] = 0.f;
                if (ch == 0 && p.out_lse) p.out_lse[row] = -INFINITY;
            }
        }
        const int qd = warp & 3, hq = warp >> 2;
        const int i = 32 * qd + lane;  // key of the tile (lane of S, channel lane of O^T)
        const uint32_t lane_base = (uint32_t)(32 * qd) << 16;
        const int r0 = hq * HR;        // first row of this warp
        const uint32_t gbar = 2 + hq;  // named barrier of the 4 warps with these rows
        const int R = p.rows;
        uint32_t kt = 0, pc = 0;
        float l_part[HR], nthr[HR];
        while (true) {
            const DtPiece pce = *pd;
            if (!pce.valid) break;
            const int b = pce.b, h = pce.h;
            const int L = seqL[b];
            // ---- query digits of (b, h): q ~= s (d1 + d2 / 254), s = max|q| / 127;
            // digit row r (d1) and RP + r (d2) of the K-major B operand of S
            {
                unsigned char *qb = smem + SM::kQ + (pc & 1) * SM::kQBuf;
                for (int r = warp; r < R; r += kDtConsumers) {
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
                    // channels 4 lane .. + 3 of operand row rr: 16-byte chunk lane / 4, swizzled
                    auto put = [&](int rr, uint32_t w) {
                        *reinterpret_cast<uint32_t *>(qb + rr * 128 + ((((uint32_t)lane >> 2) ^ ((uint32_t)rr & 7u)) << 4) +
                                                      4u * (lane & 3)) = w;
                    };
                    if constexpr (F8) {
                        // q ~= s (p1 + p2 / 16 + p3 / 256), s = max|q|: each part the
                        // e4m3 rounding of what the earlier parts leave (times 16)
                        const float inv = amax > 0.f ? 1.0f / amax : 0.f;
                        float y[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) y[e] = x[e] * inv;
#pragma unroll
                        for (int part = 0; part < 3; ++part) {
                            const uint32_t w = f32x4_to_e4m3(y[0], y[1], y[2], y[3]);
                            put(part * RP + r, w);
                            if (part < 2) {
                                uint32_t lo, hi;
                                e4m3x4_to_f16(w, lo, hi);
                                const float2 a = __half22float2(u32_h2(lo)), c2 = __half22float2(u32_h2(hi));
                                y[0] = (y[0] - a.x) * 16.f;
                                y[1] = (y[1] - a.y) * 16.f;
                                y[2] = (y[2] - c2.x) * 16.f;
                                y[3] = (y[3] - c2.y) * 16.f;
                            }
                        }
                        if (lane == 0) qw_sm[(pc & 1) * kDtMaxRows + r] = amax * p.scale_log2;
                    } else {
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
                        put(r, d1w);
                        put(RP + r, d2w);
                        if (lane == 0) qw_sm[(pc & 1) * kDtMaxRows + r] = s1 / 254.0f * p.scale_log2;
                    }
                }
                fence_async_smem();
                named_sync(kDtBarAll, kDtConsumers * 32);
                if (threadIdx.x == 0) mbar_arrive(&qfull[pc & 1]);
                if (warp == 0) {
                    // the next piece into the slot (every consumer warp has read
                    // this one), and its query rows into L2 ahead of its start
                    if (lane == 0) dt_next_piece(wk, pd);
                    __syncwarp();
                    if (pd->valid)
                        for (int t = lane; t < R * 4; t += 32) prefetch_q_rows<QF32>(p, pd->b, pd->h, t);
                }
            }
            // this warp's rows: empty running maxima and sums (the rows' factors
            // are read from qw_sm at each tile)
#pragma unroll
            for (int e = 0; e < HR; ++e) {
                nthr[e] = FLT_MAX;
                l_part[e] = 0.f;
            }
            const float *qwr = qw_sm + (pc & 1) * kDtMaxRows + r0;
            // causal: key position pos is seen by rows r >= (pos - (L - n_q)) * G
            const int causal_base = p.causal ? L - p.n_q : 0x7fffffff;
            const int all_see = p.causal ? L - p.n_q + 1 : L;  // keys every row sees
            const uint32_t kfirst = kt;
            const int cx1 = pce.cx1;
            for (int cx = pce.cx0; cx < cx1; ++kt) {
                const int ce = dt_tile_end(cx, cx1);
                const int tok0 = cx * kChunk, ntok = (ce - cx) * kChunk;
                cx = ce;
                const uint32_t stage = kt % NS, sb = kt & 1;
                const unsigned char *st = smem + stage * SM::kStride;
                // ---- the stage: this key's V nibbles of group hq, its scales;
                // then the stage is released
                dt_wait(&full[stage], (kt / NS) & 1, misc);
                const int pos = tok0 + i;
                const bool sok = stage_ok[stage] != 0;  // (garbage after an abort is never used)
                const bool kv_ok = sok && i < ntok && pos < L;
                const bool fast = sok && ntok == 128 && tok0 + 128 <= all_see && R == RP;
                // K8/V4: the group's 16 bytes of nibbles; K8V8: its 32 bytes of codes
                constexpr int VW = V8 ? 2 : 1;
                uint4 nib[kDtVG][VW];
                uint2 vsr = make_uint2(0, 0);
                float ksv = 0.f;
#pragma unroll
                for (int gg = 0; gg < kDtVG; ++gg)
#pragma unroll
                    for (int u = 0; u < VW; ++u) nib[gg][u] = make_uint4(0, 0, 0, 0);
                if (kv_ok) {
#pragma unroll
                    for (int gg = 0; gg < kDtVG; ++gg) {
                        const uint32_t g = (uint32_t)(hq * kDtVG + gg);
                        if constexpr (V8) {
#pragma unroll
                            for (int u = 0; u < 2; ++u)
                                nib[gg][u] = *reinterpret_cast<const uint4 *>(
                                    st + SM::kStV + i * 128 + (((2 * g + u) ^ ((uint32_t)i & 7u)) << 4));
                        } else {
                            nib[gg][0] = *reinterpret_cast<const uint4 *>(st + SM::kStV + i * 64 +
                                                                           ((g ^ (((uint32_t)i >> 1) & 3u)) << 4));
                        }
                    }
                    if constexpr (V8)
                        vsr.x = *reinterpret_cast<const unsigned short *>(st + SM::kStVs + i * 2);
                    else
                        vsr = *reinterpret_cast<const uint2 *>(st + SM::kStVs + i * 8);
                    ksv = __half2float(*reinterpret_cast<const __half *>(st + SM::kStKs + i * 2));
                }
                mbar_arrive(&empty[stage]);
                const int ev = dt_v_exponent(vsr);  // (K8V8: the one scale's exponent; the other words are 0)
                // ---- V' and P' buffers sb are free once the P.V of tile kt - 2 is done
                if (kt >= 2) dt_wait(&pvdone[sb], ((kt >> 1) - 1) & 1, misc);
#pragma unroll
                for (int gg = 0; gg < kDtVG; ++gg) {
                    // V' = code x scale / f: group vg of the key's row (block vg / 2,
                    // 16-byte chunks 4 (vg % 2) .. + 3)
                    const int vg = hq * kDtVG + gg;
                    unsigned char *vd = smem + SM::kVh + sb * 32768 + (vg >> 1) * 16384 + i * 128;
                    const uint32_t sw = (uint32_t)i & 7u;
                    const uint32_t sbits = V8 ? vsr.x : (vg < 2 ? vsr.x : vsr.y) >> (16 * (vg & 1));
                    const float sg = __half2float(__ushort_as_half((unsigned short)(sbits & 0xFFFFu))) *
                                     __int_as_float((127 + 15 - ev) << 23);
                    const __half2 sv = __float2half2_rn(sg);
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        uint4 o;
                        if constexpr (V8) {
                            // channels 8w .. 8w + 7 of the group in order: codes of words 2w, 2w + 1
                            const uint4 q = nib[gg][w >> 1];
                            const uint32_t w0 = (w & 1) ? q.z : q.x, w1 = (w & 1) ? q.w : q.y;
                            uint32_t lo0, hi0, lo1, hi1;
                            if constexpr (F8) {
                                e4m3x4_to_f16(w0, lo0, hi0);
                                e4m3x4_to_f16(w1, lo1, hi1);
                            } else {
                                i8x4_to_f16(w0, lo0, hi0);
                                i8x4_to_f16(w1, lo1, hi1);
                            }
                            o.x = h2_u32(__hmul2(u32_h2(lo0), sv));
                            o.y = h2_u32(__hmul2(u32_h2(hi0), sv));
                            o.z = h2_u32(__hmul2(u32_h2(lo1), sv));
                            o.w = h2_u32(__hmul2(u32_h2(hi1), sv));
                        } else {
                            const uint32_t wd[4] = {nib[gg][0].x, nib[gg][0].y, nib[gg][0].z, nib[gg][0].w};
                            o.x = h2_u32(__hmul2(nib_even(wd[w]), sv));
                            o.y = h2_u32(__hmul2(nib_odd(wd[w]), sv));
                            o.z = h2_u32(__hmul2(nib_even(wd[w] >> 8), sv));
                            o.w = h2_u32(__hmul2(nib_odd(wd[w] >> 8), sv));
                        }
                        const uint32_t cc = (uint32_t)(4 * (vg & 1) + w);
                        *reinterpret_cast<uint4 *>(vd + ((cc ^ sw) << 4)) = o;
                    }
                }
                // ---- softmax of rows r0 .. r0 + HR - 1 for this key
                dt_wait(&sfull[sb], (kt >> 1) & 1, misc);
                tc_fence_after();
                // the S words of the rows (int8 digits: two per row; e4m3 parts: three)
                uint32_t d1[HR], d2[HR], d3[HR];
                {
                    const uint32_t ta = tmem + lane_base + sb * kSCol + r0;
                    dt_ld<HR>(ta, d1);
                    dt_ld<HR>(ta + RP, d2);
                    if constexpr (F8) {
                        dt_ld<HR>(ta + 2 * RP, d3);
                        tmem_wait_ld_tied<HR>(d3);
#pragma unroll
                        for (int k = 0; k < HR; ++k) asm volatile("" : "+r"(d1[k]), "+r"(d2[k]));
                    } else {
#pragma unroll
                        for (int k = 0; k < HR; ++k) d3[k] = 0u;
                        tmem_wait_ld_tied<HR>(d1);
#pragma unroll
                        for (int k = 0; k < HR; ++k) asm volatile("" : "+r"(d2[k]));
                    }
                }
                tc_fence_before();
                mbar_arrive(&sfree[sb]);
                const int dpos = pos - causal_base;
                const int rmin = kv_ok ? (dpos > 0 ? dpos * p.group : 0) : 0x7fffffff;  // rows rmin .. R - 1 see it
                const float f = __int_as_float((127 + ev - 15) << 23);
                uint32_t pk[HR / 2];
                const uint32_t ota = tmem + lane_base + kOCol + r0;
                if (fast)
                    dt_softmax<HR, true, F8>(d1, d2, d3, qwr, ksv, rmin, R, r0, nthr, l_part, red, qd, lane, gbar, f, pk,
                                         kt > kfirst, ota, &pvdone[(kt - 1) & 1], ((kt - 1) >> 1) & 1, misc);
                else
                    dt_softmax<HR, false, F8>(d1, d2, d3, qwr, ksv, rmin, R, r0, nthr, l_part, red, qd, lane, gbar, f, pk,
                                          kt > kfirst, ota, &pvdone[(kt - 1) & 1], ((kt - 1) >> 1) & 1, misc);
                // P' row of this key, rows r0 .. r0 + HR - 1 (half of one, one or two
                // 16-byte chunks)
                {
                    unsigned char *pr = smem + SM::kP + sb * 16384 + i * 128;
                    if constexpr (HR >= 8) {
#pragma unroll
                        for (int c = 0; c < HR / 8; ++c)
                            *reinterpret_cast<uint4 *>(pr + (((((uint32_t)r0 >> 3) + c) ^ ((uint32_t)i & 7u)) << 4)) =
                                make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
                    } else {
                        *reinterpret_cast<uint2 *>(pr + ((((uint32_t)r0 >> 3) ^ ((uint32_t)i & 7u)) << 4) +
                                                   (r0 & 7) * 2) = make_uint2(pk[0], pk[1]);
                    }
                }
                fence_async_smem();
                tc_fence_before();
                mbar_arrive(&pfull[sb]);
            }

            // ---- end of the piece: O^T / l into out (one piece) or the partial slot
            const int s_id = b * H + h;
            const int first = pce.first, n_pieces = pce.n;
            {
                // row sums: the four warps' partial sums of each row
#pragma unroll
                for (int e = 0; e < HR; ++e) {
                    float v = l_part[e];
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                    if (lane == 0) red2[qd * kDtMaxRows + r0 + e] = v;
                }
                named_sync(gbar, 128);
                if (kt > kfirst) dt_wait(&pvdone[(kt - 1) & 1], ((kt - 1) >> 1) & 1, misc);
                tc_fence_after();
                const int ch = V8 ? i : dt_channel(i);  // K8V8: channels in order
                float *slotp = p.partials + (size_t)(s_id + vb) * p.slot_floats;
                // O^T / l, four rows at a time (few live registers)
#pragma unroll
                for (int e0 = 0; e0 < HR; e0 += 4) {
                    uint32_t o[4];
                    tmem_ld4(tmem + lane_base + kOCol + r0 + e0, o);
                    tmem_wait_ld_tied<4>(o);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int r = r0 + e0 + e;
                        if (r >= R) break;
                        const float l = (red2[r] + red2[kDtMaxRows + r]) + (red2[2 * kDtMaxRows + r] + red2[3 * kDtMaxRows + r]);
                        const bool any = nthr[e0 + e] != FLT_MAX;  // nthr = -(m + kLazy): the weights were 2^(x - m - kLazy)
                        const float val = any ? __uint_as_float(o[e]) * rcp_approx(l) : 0.f;
                        const size_t row = n_pieces == 1 ? ((size_t)b * p.n_q + r / p.group) * p.num_q_heads +
                                                               (size_t)h * p.group + r % p.group
                                                         : 0;
                        if (n_pieces == 1)
                            p.out[row * kHeadDim + ch] = val;
                        else
                            slotp[r * kHeadDim + ch] = val;
                        if (i == e0 + e) {  // one lane per row: the row's lse
                            const float lse = any ? (lg2_approx(l) - nthr[e0 + e]) * 0.69314718055994531f : -INFINITY;
                            if (n_pieces > 1)
                                slotp[R * kHeadDim + r] = lse;
                            else if (p.out_lse)
                                p.out_lse[row] = lse;
                        }
                    }
                }
                tc_fence_before();
            }
            named_sync(kDtBarAll, kDtConsumers * 32);  // the piece's outputs are written
            finish_piece_coop<kDtConsumers * 32, kDtBarAll>(p, s_id, first, vb - first, n_pieces, pce.m,
                                                               reinterpret_cast<float *>(smem + SM::kVh), misc, R, b,
                                                               h);
            named_sync(kDtBarAll, kDtConsumers * 32);  // the merge is done: its buffers are free again
            ++pc;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kDtMma) {
        // every MMA of both issuers has completed before tensor memory is freed
        if (lane == 0) {
            const uint64_t t0 = global_ns();
            while (!mbar_try_wait_sleep(drain, 0, 20000u))
                if (global_ns() - t0 > kWaitLimitNs) {
                    report(NF_DEVERR_TIMEOUT);
                    break;
                }
        }
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

}  // namespace nf
