// nf_prefill.cuh -- chunked-prefill attention over the segmented K8/V4 pool.
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
//   so the G heads of a position sit in one tile and share its K/V reads (GQA
//   packing), and a tile spans 128 / G positions, whose causal limits differ
//   by that much.  Tiles of late positions, which see the most keys, start
//   first.
// Pipeline: each thread holds its share of the next 64-key tile's codes and
//   scales in registers (read while the warps compute on the current tile) and
//   then converts them into the other of two shared-memory buffers:
//     K codes -> exact fp16 codes [key][channel]; the K scale stays per key
//       and multiplies the scores;
//     V nibbles x V scale -> fp16 values [key][channel, permuted inside each
//       8-channel chunk as the nibble unpacking delivers them];
//   rows of 256 bytes whose 16-byte chunks are XOR-swizzled by key & 7, so
//   that the ldmatrix reads of 8 keys hit 8 different bank groups.
// Math per warp (16 query rows): S = Q . K^T on mma.sync m16n8k16 (fp16 in,
//   fp32 accumulate), each query row scaled to max |q| = 1 and rounded to fp16
//   once; the online softmax in the log2 domain with a lazy running max (the
//   max is raised and O rescaled only when a tile exceeds it by more than 4,
//   the weights 2^(x - max - 4) <= 1); O += P . V with P taken as fp16 straight
//   from the score registers (the score layout of S is the A layout of P).
#pragma once

#include "nf_common.cuh"

namespace nf {

constexpr int kPfWarps = 8;
constexpr int kPfThreads = kPfWarps * 32;
constexpr int kPfRows = 16 * kPfWarps;  // query rows per CTA
constexpr int kPfKeys = 64;             // keys per tile
constexpr float kPfLazy = 4.0f;

struct PrefillParams {
    const int8_t *k_codes;
    const __half *k_scales;
    const uint8_t *v_codes;
    const __half *v_scales;
    int num_blocks, num_kv_heads;
    const __nv_bfloat16 *q;
    int batch, n_q, num_q_heads, group;
    int rows;       // group * n_q per (sequence, kv-head)
    int row_tiles;  // ceil(rows / kPfRows)
    const int32_t *block_table;
    int max_blocks;
    const int32_t *seqlens;
    int max_seqlen;
    float scale_log2;  // softmax_scale * log2(e)
    int causal;
    float *out;      // [batch][n_q][H_q][128]
    float *out_lse;  // [batch][n_q][H_q] or null
};

struct PfSmem {
    static constexpr int kTile = kPfKeys * kHeadDim * 2;  // one fp16 [64][128] tile
    static constexpr int kK = 0;                          // K codes  [2][64][128]
    static constexpr int kV = 2 * kTile;                  // V values [2][64][128]
    static constexpr int kSk = 4 * kTile;                 // K scales float [2][64]
    static constexpr int kBytes = kSk + 2 * kPfKeys * 4;
    // at start-up the query tile [128][128] fp16 is staged in the K buffers
    static_assert(kPfRows * kHeadDim * 2 <= 2 * kTile, "query staging");
};

// Byte offset of 16-byte chunk c of row r in a [rows][256 bytes] swizzled tile.
__device__ __forceinline__ uint32_t pf_swz(int r, int c) {
    return (uint32_t)r * 256u + (uint32_t)(((c ^ r) & 7) | (c & 8)) * 16u;
}

// One thread's share of a tile: key tid / 4, quarter q = tid % 4 (channels
// 32q .. 32q + 31, one V scale group).
struct PfRaw {
    uint4 k0, k1;  // K codes
    uint4 v;       // V nibbles
    __half vs;     // the group's V scale
    __half ks;     // the key's K scale
    bool ok;       // the key lies inside the sequence
};

__device__ __forceinline__ void pf_load(const PrefillParams &p, const int32_t *bt, int L, int h, int tile,
                                        PfRaw &r) {
    const int key = threadIdx.x >> 2, qtr = threadIdx.x & 3;
    const int pos = tile * kPfKeys + key;
    // a tile lies in one 256-key block, and its first key is < L, so the table
    // entry of that block exists
    const int blk = bt[(tile * kPfKeys) >> 8];
    r.ok = pos < L;
    if (blk < 0 || blk >= p.num_blocks) {
        if (threadIdx.x == 0) report(NF_DEVERR_BLOCK_ID);
        r.k0 = r.k1 = r.v = make_uint4(0, 0, 0, 0);
        r.vs = r.ks = __float2half(0.f);
        r.ok = false;
        return;
    }
    const size_t si = ((size_t)blk * p.num_kv_heads + h) * kBlock + (pos & (kBlock - 1));
    r.k0 = ldg16(p.k_codes + si * kHeadDim + 32 * qtr);
    r.k1 = ldg16(p.k_codes + si * kHeadDim + 32 * qtr + 16);
    r.v = ldg16(p.v_codes + si * (kHeadDim / 2) + 16 * qtr);
    r.vs = p.v_scales[si * (kHeadDim / kVGroup) + qtr];
    r.ks = p.k_scales[si];
}

__device__ __forceinline__ void pf_convert(const PfRaw &r, unsigned char *kbuf, unsigned char *vbuf, float *skbuf) {
    const int key = threadIdx.x >> 2, qtr = threadIdx.x & 3;
    // K: 32 int8 codes -> 4 chunks of 8 exact fp16 codes, in channel order
    const uint32_t w[8] = {r.k0.x, r.k0.y, r.k0.z, r.k0.w, r.k1.x, r.k1.y, r.k1.z, r.k1.w};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint4 o;
        i8x4_to_f16(w[2 * c], o.x, o.y);
        i8x4_to_f16(w[2 * c + 1], o.z, o.w);
        *reinterpret_cast<uint4 *>(kbuf + pf_swz(key, 4 * qtr + c)) = o;
    }
    // V: word u holds channels 32q + 8u + 0..7 (nibble i = channel 8u + i); the
    // chunk stores them as (0, 4, 1, 5, 2, 6, 3, 7), each times the V scale.
    // Keys past the end get scale 0 (their stale scale may be anything).
    const __half2 s2 = r.ok ? __half2half2(r.vs) : __float2half2_rn(0.f);
    const uint32_t vw[4] = {r.v.x, r.v.y, r.v.z, r.v.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        uint4 o;
        o.x = h2_u32(__hmul2(nib_even(vw[u]), s2));
        o.y = h2_u32(__hmul2(nib_odd(vw[u]), s2));
        o.z = h2_u32(__hmul2(nib_even(vw[u] >> 8), s2));
        o.w = h2_u32(__hmul2(nib_odd(vw[u] >> 8), s2));
        *reinterpret_cast<uint4 *>(vbuf + pf_swz(key, 4 * qtr + u)) = o;
    }
    if (qtr == 0) skbuf[key] = r.ok ? __half2float(r.ks) : 0.f;
}

__global__ void __launch_bounds__(kPfThreads, 1) prefill_kernel(const __grid_constant__ PrefillParams p) {
    extern __shared__ __align__(128) unsigned char smem[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int b = blockIdx.z, h = blockIdx.y;
    const int rt = p.row_tiles - 1 - (int)blockIdx.x;  // late positions first
    const int r0 = rt * kPfRows;
    const int G = p.group;

    pdl_wait();
    pdl_trigger();
    const int L = p.seqlens[b];
    const int32_t *bt = p.block_table + (size_t)b * p.max_blocks;
    auto out_row = [&](int r) {
        const int j = r / G, gq = r % G;
        return ((size_t)b * p.n_q + j) * p.num_q_heads + (size_t)h * G + gq;
    };
    if (L < p.n_q || L > p.max_seqlen) {
        if (threadIdx.x == 0 && rt == p.row_tiles - 1 && h == 0) report(NF_DEVERR_SEQLEN);
        for (int idx = threadIdx.x; idx < kPfRows * kHeadDim; idx += kPfThreads) {
            const int r = r0 + idx / kHeadDim, ch = idx % kHeadDim;
            if (r >= p.rows) continue;
            p.out[out_row(r) * kHeadDim + ch] = 0.f;
            if (ch == 0 && p.out_lse) p.out_lse[out_row(r)] = -INFINITY;
        }
        return;
    }
    const int last_row = min(r0 + kPfRows, p.rows) - 1;
    const int n_keys = p.causal ? L - p.n_q + last_row / G + 1 : L;
    const int tiles = (n_keys + kPfKeys - 1) / kPfKeys;

    PfRaw raw;
    pf_load(p, bt, L, h, 0, raw);  // in flight while the query is staged

    // ---- query: warp w stages its rows 16w..16w+15 (scaled to max |q| = 1,
    // fp16) into the K buffers, then loads its A fragments
    const int rw0 = r0 + 16 * warp;
    float qf[2] = {0.f, 0.f};  // max |q| x softmax scale x log2(e) of rows g, g + 8
    {
        unsigned char *qs = smem + PfSmem::kK;
        for (int i = 0; i < 16; ++i) {
            const int r = rw0 + i;
            float x[4] = {0.f, 0.f, 0.f, 0.f};
            if (r < p.rows) {
                const uint2 v = *reinterpret_cast<const uint2 *>(p.q + out_row(r) * kHeadDim + 4 * lane);
                x[0] = __uint_as_float(v.x << 16);
                x[1] = __uint_as_float(v.x & 0xFFFF0000u);
                x[2] = __uint_as_float(v.y << 16);
                x[3] = __uint_as_float(v.y & 0xFFFF0000u);
            }
            float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
            const float inv = amax > 0.f ? 1.0f / amax : 0.f;
            uint2 hv;
            hv.x = pack_f16(x[0] * inv, x[1] * inv);
            hv.y = pack_f16(x[2] * inv, x[3] * inv);
            *reinterpret_cast<uint2 *>(qs + pf_swz(16 * warp + i, lane >> 1) + (lane & 1) * 8) = hv;
            if (i == g) qf[0] = amax * p.scale_log2;
            if (i == g + 8) qf[1] = amax * p.scale_log2;
        }
    }
    __syncwarp();
    uint32_t qa[8][4];
    {
        const uint32_t qb = smem_addr(smem + PfSmem::kK);
        const int i = lane >> 3, rr = lane & 7;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
            ldsm_x4(qb + pf_swz(16 * warp + 8 * (i & 1) + rr, 2 * ks + (i >> 1)), qa[ks][0], qa[ks][1], qa[ks][2],
                    qa[ks][3]);
    }
    __syncthreads();  // every warp holds its query before the buffers are overwritten

    // ---- per-row limits
    int lim[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const int r = rw0 + g + 8 * e;
        lim[e] = r >= p.rows ? -1 : (p.causal ? L - p.n_q + r / G : L - 1);
    }
    const bool warp_on = rw0 < p.rows;
    const int wmin = p.causal ? L - p.n_q + rw0 / G : L - 1;                        // smallest limit of the warp
    const int wmax = p.causal ? L - p.n_q + min(rw0 + 15, p.rows - 1) / G : L - 1;  // largest

    float o[16][4];
#pragma unroll
    for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};

    if (tiles > 0) pf_convert(raw, smem + PfSmem::kK, smem + PfSmem::kV, reinterpret_cast<float *>(smem + PfSmem::kSk));
    __syncthreads();

    const int li = lane >> 3, lr = lane & 7;  // ldmatrix: matrix and row of this lane's address
    for (int it = 0; it < tiles; ++it) {
        const int cur = it & 1;
        if (it + 1 < tiles) pf_load(p, bt, L, h, it + 1, raw);
        const int key0 = it * kPfKeys;
        if (warp_on && key0 <= wmax) {
            const uint32_t kb = smem_addr(smem + PfSmem::kK + cur * PfSmem::kTile);
            const uint32_t vb = smem_addr(smem + PfSmem::kV + cur * PfSmem::kTile);
            const float *sk = reinterpret_cast<const float *>(smem + PfSmem::kSk) + cur * kPfKeys;
            // ---- S = Q . K^T: n-tile n = keys 8n..8n+7; lane: rows g, g + 8 x keys 8n + 2t, +1
            float s[8][4];
#pragma unroll
            for (int n = 0; n < 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
#pragma unroll
                for (int np = 0; np < 4; ++np) {
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(kb + pf_swz(16 * np + 8 * (li >> 1) + lr, 2 * ks + (li & 1)), b0, b1, b2, b3);
                    mma_f16(s[2 * np], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b0, b1);
                    mma_f16(s[2 * np + 1], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b2, b3);
                }
            const bool fast = key0 + kPfKeys - 1 <= wmin;
#pragma unroll
            for (int n = 0; n < 8; ++n) {
                const float2 kk = *reinterpret_cast<const float2 *>(sk + 8 * n + 2 * t);
                s[n][0] *= qf[0] * kk.x;
                s[n][1] *= qf[0] * kk.y;
                s[n][2] *= qf[1] * kk.x;
                s[n][3] *= qf[1] * kk.y;
                if (!fast) {
                    const int kp = key0 + 8 * n + 2 * t;
                    if (kp > lim[0]) s[n][0] = -INFINITY;
                    if (kp + 1 > lim[0]) s[n][1] = -INFINITY;
                    if (kp > lim[1]) s[n][2] = -INFINITY;
                    if (kp + 1 > lim[1]) s[n][3] = -INFINITY;
                }
            }
            // ---- lazy running max (the 4 lanes of a row agree on it)
            float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int n = 0; n < 8; ++n) {
                mx[0] = fmaxf(mx[0], fmaxf(s[n][0], s[n][1]));
                mx[1] = fmaxf(mx[1], fmaxf(s[n][2], s[n][3]));
            }
            const bool raise = mx[0] > m_run[0] + kPfLazy || mx[1] > m_run[1] + kPfLazy;
            if (__any_sync(0xffffffffu, raise)) {
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    float m = fmaxf(mx[e], __shfl_xor_sync(0xffffffffu, mx[e], 1));
                    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
                    const float m_new = fmaxf(m_run[e], m);
                    const float alpha = m_new == -INFINITY ? 1.f : ex2(m_run[e] - m_new);
                    m_run[e] = m_new;
                    l_run[e] *= alpha;
#pragma unroll
                    for (int n = 0; n < 16; ++n) {
                        o[n][2 * e] *= alpha;
                        o[n][2 * e + 1] *= alpha;
                    }
                }
            }
            // ---- P = 2^(x - m - 4) as fp16 A fragments: k-step kk = keys 16kk..16kk+15
            const float mu0 = (m_run[0] == -INFINITY ? 0.f : m_run[0]) + kPfLazy;
            const float mu1 = (m_run[1] == -INFINITY ? 0.f : m_run[1]) + kPfLazy;
            uint32_t pa[4][4];
#pragma unroll
            for (int n = 0; n < 8; ++n) {
                const float p0 = ex2(s[n][0] - mu0), p1 = ex2(s[n][1] - mu0);
                const float p2 = ex2(s[n][2] - mu1), p3 = ex2(s[n][3] - mu1);
                l_run[0] += p0 + p1;
                l_run[1] += p2 + p3;
                pa[n >> 1][2 * (n & 1)] = pack_f16(p0, p1);
                pa[n >> 1][2 * (n & 1) + 1] = pack_f16(p2, p3);
            }
            // ---- O += P . V: n-tile n = stored channel positions 8n..8n+7
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
#pragma unroll
                for (int cp = 0; cp < 8; ++cp) {
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(vb + pf_swz(16 * kk + 8 * (li & 1) + lr, 2 * cp + (li >> 1)), b0, b1, b2, b3);
                    mma_f16(o[2 * cp], pa[kk][0], pa[kk][1], pa[kk][2], pa[kk][3], b0, b1);
                    mma_f16(o[2 * cp + 1], pa[kk][0], pa[kk][1], pa[kk][2], pa[kk][3], b2, b3);
                }
        }
        if (it + 1 < tiles)
            pf_convert(raw, smem + PfSmem::kK + (cur ^ 1) * PfSmem::kTile, smem + PfSmem::kV + (cur ^ 1) * PfSmem::kTile,
                       reinterpret_cast<float *>(smem + PfSmem::kSk) + (cur ^ 1) * kPfKeys);
        __syncthreads();
    }

    // ---- normalise and write: accumulator (n, 2t + e) is channel 8n + t + 4e
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        float l = l_run[e];
        l += __shfl_xor_sync(0xffffffffu, l, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);
        const int r = rw0 + g + 8 * e;
        if (r >= p.rows) continue;
        const float inv = l > 0.f ? 1.0f / l : 0.f;
        float *dst = p.out + out_row(r) * kHeadDim;
#pragma unroll
        for (int n = 0; n < 16; ++n) {
            dst[8 * n + t] = o[n][2 * e] * inv;
            dst[8 * n + t + 4] = o[n][2 * e + 1] * inv;
        }
        if (t == 0 && p.out_lse)
            p.out_lse[out_row(r)] =
                l > 0.f ? (m_run[e] + kPfLazy + log2f(l)) * 0.69314718055994531f : -INFINITY;
    }
}

}  // namespace nf
