// nf_prefill.cuh -- chunked-prefill attention over the segmented K8/V4 pool,
// on the 5th-generation tensor cores (tcgen05).
//
// The pages' engine prefills a prompt in chunks of 1024 tokens (page "3090 单卡跑
// Qwen3.8-27B：NInfer 上机实测", section 一.3, --prefill-chunk 1024) on a
// dequantise -> fp16 tensor-core path (same page, section 二 and its replies on
// prefill efficiency), and prefill is where long context costs most (section
// 二, time to first token).  The n_q queries of a chunk sit at positions
// L - n_q .. L - 1, their K/V already appended, and with the causal flag each
// sees the keys up to its own position: the decode definition with a large n_q.
//
// Work: one CTA per (sequence, kv-head, tile of 128 query rows).  The rows of a
//   kv-head are its G * n_q (position, q-head) pairs in position-major order,
//   so the G heads of a position sit in one tile and share its K/V (GQA
//   packing), and a tile spans 128 / G positions, whose causal limits differ
//   by that much.  Tiles of late positions, which see the most keys, start
//   first.
#pragma once

#include "nf_common.cuh"
#include "nf_tc.cuh"

namespace nf {

struct PrefillParams {
    const int8_t *k_codes;
    const __half *k_scales;
    const uint8_t *v_codes;
    const __half *v_scales;
    int num_blocks, num_kv_heads;
    const __nv_bfloat16 *q;
    int batch, n_q, num_q_heads, group;
    int rows;       // group * n_q per (sequence, kv-head)
    int row_tiles;  // ceil(rows / 128)
    const int32_t *block_table;
    int max_blocks;
    const int32_t *seqlens;
    int max_seqlen;
    float scale_log2;  // softmax_scale * log2(e)
    int causal;
    float *out;      // [batch][n_q][H_q][128]
    float *out_lse;  // [batch][n_q][H_q] or null
};

// ============================================================================
// CTA = 256 query rows: two tiles a, b of 128 rows (each the M of its own
// MMAs) that share every K/V tile, and four roles:
//   warps 0-3, 4-7  softmax of tile a, of tile b: thread r owns row r of its
//              tile; reads its row of S from tensor memory (tcgen05.ld), runs
//              the online softmax, writes its row of P (fp16) to shared memory,
//              rescales its row of O in tensor memory when its running max
//              rises, and at the end reads O, normalises and writes the output;
//   warps 8-11 converters: they stage both tiles' query rows (scaled to
//              max |q| = 1, fp16) once; then for every 64-key tile thread t
//              loads key t's K codes (t < 64) or key t - 64's V nibbles and
//              scales (prefetched a tile ahead in registers) and writes that
//              dequantised fp16 row into a three-stage ring;
//   warps 12-15 the MMAs, each stream on one thread of its own warp: warp
//              12 (which also holds the tensor memory) S_a = Q_a . K_j^T and
//              warp 13 S_b, each into one of two S buffers of its tile once
//              the softmax has read that buffer's last S; warps 14 and 15
//              O_a += P_a . V_j and O_b += P_b . V_j.  Each group is committed
//              to an mbarrier.  One issue stream per SM sub-partition: issuing
//              an MMA takes issue cycles from the warps beside it, and each
//              softmax tile waits for the slowest of its four warps.
// The K/V ring is converted once for 256 rows, and each SM sub-partition runs
// two softmax warps, one of each tile.
// Tensor memory (512 columns x 128 lanes): S of tile x, buffer b at columns
// 128x + 64b (64 keys), O of tile x at 256 + 128x.  Shared operands use the
// 128-byte-swizzled canonical layouts (rows of 128 bytes = 64 fp16, 8-row
// groups of 1024 bytes):
//   Q_x    A of S, K-major: [2 blocks of 64 channels][128 rows][128 bytes];
//   K      B of S, K-major: [2 blocks of 64 channels][64 keys][128 bytes] (x 3 stages);
//   P_x    A of O, K-major: [128 rows][64 keys x 2 bytes];
//   V      B of O, MN-major: [2 blocks of 64 channels][64 keys][128 bytes],
//          channels inside each 8-channel chunk in the nibble-unpacking order.
// Weights are 2^(x - m) with a lazy running max m: it is raised (and O
// rescaled) only when a tile's max exceeds it by more than 8, so P <= 2^8.
// Every mbarrier wait is bounded; a timeout records NF_DEVERR_TIMEOUT and
// every role leaves its loop.
// ============================================================================
constexpr int kTcThreads = 512;
constexpr int kTcRows = 256;   // query rows per CTA (two MMA tiles of 128)
constexpr int kTcKeys = 64;    // keys per K/V tile (N of S = Q.K^T, K of O += P.V)
constexpr float kTcLazy = 8.0f;
constexpr uint32_t kTcIdescQK = umma_idesc_f16(128, 64, false);   // B = K rows, K-major
constexpr uint32_t kTcIdescPV = umma_idesc_f16(128, 128, true);   // B = V rows, MN-major

struct TcSmem {
    static constexpr int kQ = 0;                      // [2 tiles][2 blocks][128 rows][128 B]
    static constexpr int kStages = 3;                 // K/V ring depth
    static constexpr int kK = 65536;                  // [3 stages][2 blocks][64 keys][128 B]
    static constexpr int kV = kK + kStages * 16384;   // [3 stages][2 blocks][64 keys][128 B]
    static constexpr int kP = kV + kStages * 16384;   // [2 buffers][2 tiles][128 rows][128 B]
    static constexpr int kBars = kP + 65536;          // mbarriers
    static constexpr int kQf = kBars + 256;           // float [256]
    static constexpr int kMisc = kQf + 256 * 4;       // tmem base, abort flag
    static constexpr int kBytes = kMisc + 16;
    static_assert(kBytes <= 232448, "shared memory per CTA");
};
// mbarrier slots
enum { kBarQ = 0, kBarKV = 1, kBarFree = 4, kBarS = 7, kBarP = 11, kBarPV = 15, kBarO = 19, kBarDrain = 20, kNumBars = 21 };
static_assert(kNumBars * 8 <= 256, "mbarrier slots");

// byte offset of row r, 16-byte chunk c (0..15: 8 fp16 each) in a two-block
// 128-byte-swizzled operand whose blocks are `blk` bytes apart
__device__ __forceinline__ uint32_t tc_swz(int r, int c, uint32_t blk) {
    return (uint32_t)(c >> 3) * blk + (uint32_t)r * 128u + (uint32_t)(((c ^ r) & 7) * 16);
}

struct TcRawK {
    uint4 k[8];   // K codes of the key
    uint32_t ks;  // K scale (low half)
    int ok;       // key inside the sequence
};
struct TcRawV {
    uint4 v[4];   // V nibbles
    uint2 vs;     // 4 V scales
    int ok;
};

// a tile lies in one 256-key block, and its first key is < L, so the table
// entry of that block exists; a bad entry reads as zeros (and is reported)
__device__ __forceinline__ size_t tc_slot(const PrefillParams &p, const int32_t *bt, int h, int pos, bool &good) {
    const int blk = bt[pos >> 8];
    good = blk >= 0 && blk < p.num_blocks;
    if (!good) {
        report(NF_DEVERR_BLOCK_ID);
        return 0;
    }
    return ((size_t)blk * p.num_kv_heads + h) * kBlock + (pos & (kBlock - 1));
}
__device__ __forceinline__ void tc_load_k(const PrefillParams &p, const int32_t *bt, int L, int h, int tile, int key,
                                          TcRawK &r) {
    const int pos = tile * kTcKeys + key;
    bool good;
    const size_t si = tc_slot(p, bt, h, pos, good);
    r.ok = good && pos < L;
    if (!good) {
#pragma unroll
        for (int u = 0; u < 8; ++u) r.k[u] = make_uint4(0, 0, 0, 0);
        r.ks = 0;
        return;
    }
    const unsigned char *kp = reinterpret_cast<const unsigned char *>(p.k_codes) + si * kHeadDim;
#pragma unroll
    for (int u = 0; u < 8; ++u) r.k[u] = ldg16(kp + 16 * u);
    r.ks = __ldg(reinterpret_cast<const unsigned short *>(p.k_scales + si));
}
__device__ __forceinline__ void tc_load_v(const PrefillParams &p, const int32_t *bt, int L, int h, int tile, int key,
                                          TcRawV &r) {
    const int pos = tile * kTcKeys + key;
    bool good;
    const size_t si = tc_slot(p, bt, h, pos, good);
    r.ok = good && pos < L;
    if (!good) {
#pragma unroll
        for (int u = 0; u < 4; ++u) r.v[u] = make_uint4(0, 0, 0, 0);
        r.vs = make_uint2(0, 0);
        return;
    }
    const unsigned char *vp = p.v_codes + si * (kHeadDim / 2);
#pragma unroll
    for (int u = 0; u < 4; ++u) r.v[u] = ldg16(vp + 16 * u);
    r.vs = __ldg(reinterpret_cast<const uint2 *>(p.v_scales + si * (kHeadDim / kVGroup)));
}
// Largest K and V scales (fp16 bits) whose dequantised codes stay finite in
// fp16: 127 x 515.5 and 7 x 9352 round to finite values, 127 x 516 and 7 x
// 9360 to infinity.  A larger scale is reported as NF_DEVERR_RANGE.
constexpr uint32_t kTcMaxKScaleBits = 0x6007u;  // 515.5
constexpr uint32_t kTcMaxVScaleBits = 0x7091u;  // 9352
// key's dequantised fp16 K row (code x K scale)
__device__ __forceinline__ void tc_convert_k(const TcRawK &r, int key, unsigned char *kb) {
    if (r.ok && (r.ks & 0x7FFFu) > kTcMaxKScaleBits) report(NF_DEVERR_RANGE);
    const __half2 sk = u32_h2(r.ok ? (r.ks & 0xFFFFu) * 0x10001u : 0u);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        uint4 a, c;
        i8x4_to_f16(r.k[u].x, a.x, a.y);
        i8x4_to_f16(r.k[u].y, a.z, a.w);
        i8x4_to_f16(r.k[u].z, c.x, c.y);
        i8x4_to_f16(r.k[u].w, c.z, c.w);
        a.x = h2_u32(__hmul2(u32_h2(a.x), sk)); a.y = h2_u32(__hmul2(u32_h2(a.y), sk));
        a.z = h2_u32(__hmul2(u32_h2(a.z), sk)); a.w = h2_u32(__hmul2(u32_h2(a.w), sk));
        c.x = h2_u32(__hmul2(u32_h2(c.x), sk)); c.y = h2_u32(__hmul2(u32_h2(c.y), sk));
        c.z = h2_u32(__hmul2(u32_h2(c.z), sk)); c.w = h2_u32(__hmul2(u32_h2(c.w), sk));
        *reinterpret_cast<uint4 *>(kb + tc_swz(key, 2 * u, 8192u)) = a;
        *reinterpret_cast<uint4 *>(kb + tc_swz(key, 2 * u + 1, 8192u)) = c;
    }
}
// key's dequantised fp16 V row (code x V scale; 0 past the end)
__device__ __forceinline__ void tc_convert_v(const TcRawV &r, int key, unsigned char *vb) {
    const uint32_t keep = r.ok ? 0xFFFFFFFFu : 0u;
    if (r.ok) {
        const uint32_t sb[4] = {r.vs.x & 0x7FFFu, (r.vs.x >> 16) & 0x7FFFu, r.vs.y & 0x7FFFu, (r.vs.y >> 16) & 0x7FFFu};
        if (max(max(sb[0], sb[1]), max(sb[2], sb[3])) > kTcMaxVScaleBits) report(NF_DEVERR_RANGE);
    }
    const uint32_t vsg[4] = {prmt(r.vs.x, 0, 0x1010) & keep, prmt(r.vs.x, 0, 0x3232) & keep,
                             prmt(r.vs.y, 0, 0x1010) & keep, prmt(r.vs.y, 0, 0x3232) & keep};
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const uint32_t w = (i & 3) == 0 ? r.v[i >> 2].x : (i & 3) == 1 ? r.v[i >> 2].y
                         : (i & 3) == 2 ? r.v[i >> 2].z : r.v[i >> 2].w;
        const __half2 sv = u32_h2(vsg[i >> 2]);  // 32-channel scale group i / 4
        uint4 o;
        o.x = h2_u32(__hmul2(nib_even(w), sv));
        o.y = h2_u32(__hmul2(nib_odd(w), sv));
        o.z = h2_u32(__hmul2(nib_even(w >> 8), sv));
        o.w = h2_u32(__hmul2(nib_odd(w >> 8), sv));
        *reinterpret_cast<uint4 *>(vb + tc_swz(key, i, 8192u)) = o;
    }
}

// bounded wait that also gives up once another role has aborted
__device__ __forceinline__ bool tc_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait_sleep(bar, parity, 20000u)) {
        if (*abort_flag) return false;
        if (global_ns() - t0 > kWaitLimitNs) {
            report(NF_DEVERR_TIMEOUT);
            *abort_flag = 1;
            return false;
        }
    }
    return true;
}

__global__ void __launch_bounds__(kTcThreads, 1) prefill_tc_kernel(const __grid_constant__ PrefillParams p) {
    extern __shared__ __align__(1024) unsigned char smem[];
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + TcSmem::kBars);
    uint64_t *q_full = bars + kBarQ, *kv_full = bars + kBarKV, *kv_free = bars + kBarFree, *o_full = bars + kBarO,
             *drain = bars + kBarDrain;
    // [tile][buffer]
    auto s_full = [&](int x, int b) { return bars + kBarS + 2 * x + b; };
    auto p_full = [&](int x, int b) { return bars + kBarP + 2 * x + b; };
    auto pv_done = [&](int x, int b) { return bars + kBarPV + 2 * x + b; };
    float *qfs = reinterpret_cast<float *>(smem + TcSmem::kQf);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(smem + TcSmem::kMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + TcSmem::kMisc + 4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.z, h = blockIdx.y;
    const int rt = p.row_tiles - 1 - (int)blockIdx.x;  // late positions first
    const int r0 = rt * kTcRows;
    const int G = p.group;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 128);
        for (int i = 0; i < TcSmem::kStages; ++i) {
            mbar_init(&kv_full[i], 128);
            mbar_init(&kv_free[i], 4);  // the four MMA streams' commits for the stage's tile
        }
        for (int i = 0; i < 2; ++i) {
            for (int x = 0; x < 2; ++x) {
                mbar_init(s_full(x, i), 1);
                mbar_init(p_full(x, i), 128);
                mbar_init(pv_done(x, i), 1);
            }
        }
        mbar_init(o_full, 2);  // the two P.V streams' last commits
        mbar_init(drain, 4);
        *abort_flag = 0;
        // the swizzled operands need 1024-byte alignment of the window
        if (smem_addr(smem) & 1023u) {
            if (blockIdx.x == 0 && h == 0 && b == 0) report(NF_DEVERR_INTERNAL);
            *abort_flag = 1;
        }
        fence_mbar_init();
    }
    if (warp == 12) {
        tmem_alloc(tslot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;

    pdl_wait();
    pdl_trigger();
    const int L = p.seqlens[b];
    auto out_row = [&](int r) {
        const int j = r / G, gq = r % G;
        return ((size_t)b * p.n_q + j) * p.num_q_heads + (size_t)h * G + gq;
    };
    const bool bad_len = L < p.n_q || L > p.max_seqlen;
    const int last_row = min(r0 + kTcRows, p.rows) - 1;
    const int n_keys = bad_len ? 0 : (p.causal ? L - p.n_q + last_row / G + 1 : L);
    const int T = (n_keys + kTcKeys - 1) / kTcKeys;
    const int32_t *bt = p.block_table + (size_t)b * p.max_blocks;

    if (bad_len) {
        if (threadIdx.x == 0 && rt == p.row_tiles - 1 && h == 0) report(NF_DEVERR_SEQLEN);
        for (int idx = threadIdx.x; idx < kTcRows * kHeadDim; idx += kTcThreads) {
            const int r = r0 + idx / kHeadDim, ch = idx % kHeadDim;
            if (r >= p.rows) continue;
            p.out[out_row(r) * kHeadDim + ch] = 0.f;
            if (ch == 0 && p.out_lse) p.out_lse[out_row(r)] = -INFINITY;
        }
    } else if (warp >= 8 && warp < 12 && !*abort_flag) {
        // ================================================== converters
        const int t = threadIdx.x - 256;
        for (int x = 0; x < 2; ++x) {
            const int r = r0 + 128 * x + t;
            uint4 qw[16];  // the row as packed bf16
            if (r < p.rows) {
                const uint4 *qp = reinterpret_cast<const uint4 *>(p.q + out_row(r) * kHeadDim);
#pragma unroll
                for (int u = 0; u < 16; ++u) qw[u] = __ldg(qp + u);
            } else {
#pragma unroll
                for (int u = 0; u < 16; ++u) qw[u] = make_uint4(0, 0, 0, 0);
            }
            // max |q| straight from the bf16 bits (sign cleared)
            uint32_t am = 0;
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const uint32_t ww[4] = {qw[u].x, qw[u].y, qw[u].z, qw[u].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) am = max(am, max((ww[e] << 16) & 0x7FFFFFFFu, ww[e] & 0x7FFF0000u));
            }
            const float amax = __uint_as_float(am);
            const float inv = amax > 0.f ? 1.0f / amax : 0.f;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const uint32_t ww[4] = {qw[c].x, qw[c].y, qw[c].z, qw[c].w};
                uint32_t o4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    o4[e] = pack_f16(__uint_as_float(ww[e] << 16) * inv, __uint_as_float(ww[e] & 0xFFFF0000u) * inv);
                *reinterpret_cast<uint4 *>(smem + TcSmem::kQ + x * 32768 + tc_swz(t, c, 16384u)) =
                    make_uint4(o4[0], o4[1], o4[2], o4[3]);
            }
            qfs[128 * x + t] = amax * p.scale_log2;
        }
        fence_async_smem();
        mbar_arrive(q_full);
        // K/V rows: warps 8-9 the K rows of keys 0..63, warps 10-11 the V rows
        auto ring = [&](auto &ra, auto &rb, auto load, auto convert, int key, int region) {
            if (T > 0) load(0, ra);
            auto stage_tile = [&](int j, auto &cur, auto &nxt) -> bool {
                if (j + 1 < T) load(j + 1, nxt);
                const int s = j % TcSmem::kStages;
                // the stage is free once every MMA of tile j - 3 has completed
                if (j >= TcSmem::kStages &&
                    !tc_wait(&kv_free[s], (j / TcSmem::kStages - 1) & 1, abort_flag))
                    return false;
                convert(cur, key, smem + region + s * 16384);
                fence_async_smem();
                mbar_arrive(&kv_full[s]);
                return true;
            };
            for (int j = 0; j < T; j += 2) {
                if (!stage_tile(j, ra, rb)) break;
                if (j + 1 < T && !stage_tile(j + 1, rb, ra)) break;
            }
        };
        if (t < 64) {
            TcRawK ra, rb;
            ring(ra, rb, [&](int tile, TcRawK &r) { tc_load_k(p, bt, L, h, tile, t, r); },
                 [&](const TcRawK &r, int key, unsigned char *dst) { tc_convert_k(r, key, dst); }, t, TcSmem::kK);
        } else {
            TcRawV ra, rb;
            ring(ra, rb, [&](int tile, TcRawV &r) { tc_load_v(p, bt, L, h, tile, t - 64, r); },
                 [&](const TcRawV &r, int key, unsigned char *dst) { tc_convert_v(r, key, dst); }, t - 64, TcSmem::kV);
        }
    } else if (warp < 8 && !*abort_flag) {
        // ================================================== softmax (tile x)
        const int x = warp >> 2;
        const int r = threadIdx.x & 127;
        const int row = r0 + 128 * x + r;
        const int lim = row < p.rows ? (p.causal ? L - p.n_q + row / G : L - 1) : -1;
        const uint32_t t_lane = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
        const uint32_t s_col = 128u * x, o_col = 256u + 128u * x;
        float m_run = -INFINITY, l_run = 0.f;
        // every wait's outcome is made warp-uniform: the tcgen05 loads and
        // stores below are warp-collective
        bool ok = __all_sync(0xffffffffu, tc_wait(q_full, 0, abort_flag));
        const float qf = ok ? qfs[128 * x + r] : 0.f;
        for (int j = 0; ok && j < T; ++j) {
            const int sb = j & 1;
            if (!__all_sync(0xffffffffu, tc_wait(s_full(x, sb), (j >> 1) & 1, abort_flag))) { ok = false; break; }
            tc_fence_after();
            uint32_t sa[32], sbv[32];
            tmem_ld32(t_lane + s_col + 64u * sb, sa);
            tmem_ld32(t_lane + s_col + 64u * sb + 32u, sbv);
            tmem_wait_ld();
#define SV(i) ((i) < 32 ? sa[(i)] : sbv[(i) - 32])
            const int key0 = j * kTcKeys;
            const int nvis = min(kTcKeys, lim - key0 + 1);  // keys of the tile this row sees (may be <= 0)
            if (nvis < kTcKeys) {
#pragma unroll
                for (int i = 0; i < kTcKeys; ++i)
                    if (i >= nvis) SV(i) = __float_as_uint(-INFINITY);
            }
            // row max over 8 independent partial maxima (short dependency chains)
            float m8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) m8[e] = __uint_as_float(SV(e));
#pragma unroll
            for (int i = 8; i < kTcKeys; ++i) m8[i & 7] = fmaxf(m8[i & 7], __uint_as_float(SV(i)));
            const float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                                   fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
            const float tmax = mx == -INFINITY ? -INFINITY : mx * qf;
            const bool raise = tmax > m_run + kTcLazy;
            // the warp rescales its rows of O (below, once S is no longer
            // held) when any of its rows raises its max
            const bool rescale_o = __any_sync(0xffffffffu, raise) && j >= 1;
            const float alpha = raise ? ex2(m_run - tmax) : 1.f;  // 0 when m_run was -inf
            if (raise) {
                l_run *= alpha;
                m_run = tmax;
            }
            // weights 2^(x - m) <= 2^kTcLazy: inside fp16, and the flat-attention
            // bulk (a few units below the max) stays in its normal range
            const float mu = m_run == -INFINITY ? 0.f : m_run;
            // the P buffer was last read by O of tile j - 2
            if (j >= 2 && !__all_sync(0xffffffffu, tc_wait(pv_done(x, sb), ((j - 2) >> 1) & 1, abort_flag))) {
                ok = false;
                break;
            }
            unsigned char *pb = smem + TcSmem::kP + sb * 32768 + x * 16384;
            // P = 2^(s qf - m), two at a time in fp16 (masked keys hold -inf: 0)
            float lsum[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                uint32_t ph[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float x0 = fmaf(__uint_as_float(SV(8 * c + 2 * e)), qf, -mu);
                    const float x1 = fmaf(__uint_as_float(SV(8 * c + 2 * e + 1)), qf, -mu);
                    ph[e] = ex2_h2(pack_f16(x0, x1));
                }
                *reinterpret_cast<uint4 *>(pb + tc_swz(r, c, 0u)) = make_uint4(ph[0], ph[1], ph[2], ph[3]);
                // the row sum from the stored fp16 weights, in fp32
                const __half2 s01 = __hadd2(u32_h2(ph[0]), u32_h2(ph[1]));
                const __half2 s23 = __hadd2(u32_h2(ph[2]), u32_h2(ph[3]));
                const float2 f01 = __half22float2(s01), f23 = __half22float2(s23);
                lsum[c & 3] += (f01.x + f01.y) + (f23.x + f23.y);
            }
            l_run += (lsum[0] + lsum[1]) + (lsum[2] + lsum[3]);
#undef SV
            if (rescale_o) {
                // O holds the products up to tile j - 1 once that group has
                // completed; tile j's is issued only after this thread's arrival
                if (!__all_sync(0xffffffffu, tc_wait(pv_done(x, (j - 1) & 1), ((j - 1) >> 1) & 1, abort_flag))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t o[32];
                    tmem_ld32(t_lane + o_col + 32u * c, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                    tmem_st32(t_lane + o_col + 32u * c, o);
                }
                tmem_wait_st();
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(p_full(x, sb));
        }
        if (ok && __all_sync(0xffffffffu, tc_wait(o_full, 0, abort_flag))) {
            tc_fence_after();
            const float inv = l_run > 0.f ? 1.0f / l_run : 0.f;
            float *dst = row < p.rows ? p.out + out_row(row) * kHeadDim : nullptr;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t o[32];
                tmem_ld32(t_lane + o_col + 32u * c, o);
                tmem_wait_ld();
                if (dst) {
                    // column 8g + e holds channel 8g + (0, 4, 1, 5, 2, 6, 3, 7)[e]
#pragma unroll
                    for (int g8 = 0; g8 < 4; ++g8) {
                        const uint32_t *q8 = o + 8 * g8;
                        float4 lo4 = make_float4(__uint_as_float(q8[0]) * inv, __uint_as_float(q8[2]) * inv,
                                                 __uint_as_float(q8[4]) * inv, __uint_as_float(q8[6]) * inv);
                        float4 hi4 = make_float4(__uint_as_float(q8[1]) * inv, __uint_as_float(q8[3]) * inv,
                                                 __uint_as_float(q8[5]) * inv, __uint_as_float(q8[7]) * inv);
                        float4 *d4 = reinterpret_cast<float4 *>(dst + 32 * c + 8 * g8);
                        d4[0] = lo4;
                        d4[1] = hi4;
                    }
                }
            }
            if (dst && p.out_lse)
                p.out_lse[out_row(row)] = l_run > 0.f ? (m_run + log2f(l_run)) * 0.69314718055994531f : -INFINITY;
        }
    } else if (warp >= 12 && lane == 0 && !*abort_flag) {
        // ================================================== MMA issue
        const int role = warp - 12, x = role & 1;
        const uint32_t sQ = smem_addr(smem + TcSmem::kQ), sK = smem_addr(smem + TcSmem::kK);
        const uint32_t sV = smem_addr(smem + TcSmem::kV), sP = smem_addr(smem + TcSmem::kP);
        bool ok = true;
        if (role < 2) {
            // S_x of tile j once K of tile j is staged and the softmax of tile
            // x has read S of tile j - 2 (the same buffer)
            ok = tc_wait(q_full, 0, abort_flag);
            for (int j = 0; ok && j < T; ++j) {
                const int s = j & 1, st = j % TcSmem::kStages;
                if (!tc_wait(&kv_full[st], (j / TcSmem::kStages) & 1, abort_flag) ||
                    (j >= 2 && !tc_wait(p_full(x, s), ((j - 2) >> 1) & 1, abort_flag))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint64_t ad = umma_desc_sw128(sQ + x * 32768 + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
                    const uint64_t bd = umma_desc_sw128(sK + st * 16384 + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024);
                    umma_f16(tmem + 128u * x + 64u * s, ad, bd, kTcIdescQK, ks > 0 ? 1u : 0u);
                }
                umma_commit(s_full(x, s));
                umma_commit(&kv_free[st]);  // this stream's reads of stage st are done
            }
        } else {
            // O_x += P_x . V of tile j once the softmax of tile x has written P
            for (int j = 0; ok && j < T; ++j) {
                const int s = j & 1, st = j % TcSmem::kStages;
                if (!tc_wait(&kv_full[st], (j / TcSmem::kStages) & 1, abort_flag) ||
                    !tc_wait(p_full(x, s), (j >> 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t ad = umma_desc_sw128(sP + s * 32768 + x * 16384 + kk * 32, 16, 1024);
                    const uint64_t bd = umma_desc_sw128(sV + st * 16384 + kk * 2048, 8192, 1024);
                    umma_f16(tmem + 256u + 128u * x, ad, bd, kTcIdescPV, (j > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(pv_done(x, s));
                umma_commit(&kv_free[st]);
            }
            if (ok) umma_commit(o_full);
        }
        umma_commit(drain);  // arrives once every MMA this thread issued has completed
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 12) {
        // every MMA of the four streams has completed before tensor memory is freed
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
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace nf
