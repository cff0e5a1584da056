// nf_decode.cuh -- split-K decode attention over the segmented K8/V4 (or bf16)
// pool.
//
// Work unit: one CTA per (sequence b, kv-head h, context split, row group).
// The GQA group's G * n_q query rows of kv-head h are served by the same CTA,
// so each key/value byte of the split is fetched once for all of them (page
// "標籤: vLLM", section 2: stream one KV segment at a time, decode tuned for a
// single long request).  A row group is 16 query rows; wider groups (n_q * G >
// 16, MTP verification) run one CTA per 16 rows over the same split, launched
// next to each other so the second read of the split is served by L2.
//
// Inside a CTA each warp takes 16-token tiles of the split in turn and keeps
// its own online-softmax state; the warps are merged at the end and the CTA
// writes one (o, lse) partial per row for nf_attn_combine.
//
// Tensor-core mapping (mma.sync m16n8k16, "swap AB" so that the 16-token tile
// is the M dimension and the query rows are N = 8):
//   S^T[token][row] = K_codes[token][ch] . Q^T[ch][row]   (fp16, exact codes)
//     lane (g, t) reads bytes 32t..32t+31 of tokens g and g+8, which it feeds
//     to the 8 k-steps; q is permuted the same way once per CTA.
//   O^T[ch][row] += V_hat^T[ch][token] . P^T[token][row]  (fp16, fp32 acc)
//     lane (g, t) reads the 32 channels of V group t for tokens g and g+8,
//     converts them to fp16 and scales them, and movmatrix transposes them
//     into the A fragments; P^T comes from the S^T accumulator layout through
//     movmatrix as well.
// The K scale is per token and multiplies the rows of S^T after the MMA.
#pragma once

#include "nf_common.cuh"

namespace nf {

constexpr int kDecodeWarps = 4;
constexpr int kTile = 16;
constexpr int kRowsPerCta = 16;

struct DecodeParams {
    const void *k_codes;
    const __half *k_scales;
    const void *v_codes;
    const __half *v_scales;
    int num_blocks, num_kv_heads;
    const void *q;
    int batch, n_q, num_q_heads, group, rows_per_head;  // rows_per_head = group * n_q
    const int32_t *block_table;
    int max_blocks;
    const int32_t *seqlens;
    int max_seqlen;
    float scale_log2;  // softmax_scale * log2(e)
    int causal;
    int split_len, n_splits, n_row_groups;
    float *part_o;    // [n_splits][rows_total][128]
    float *part_lse;  // [n_splits][rows_total]
    int rows_total;
};

// Output channel held by row `rho` (0..15) of PV m-tile `m`, for the K8/V4
// V layout (lane t converts channels 32t..32t+31, pairing nibbles k and k+4).
__device__ __forceinline__ int v_channel_k8v4(int m, int rho) {
    const int p = 2 * m + (rho >> 3), jj = rho & 7;
    return 32 * (jj >> 1) + 8 * (p >> 2) + (p & 3) + 4 * (jj & 1);
}
// Same for the bf16 cache (lane t holds channel pairs 32t + 2p, 32t + 2p + 1).
__device__ __forceinline__ int v_channel_bf16(int m, int rho) {
    const int p = 2 * m + (rho >> 3), jj = rho & 7;
    return 32 * (jj >> 1) + 2 * p + (jj & 1);
}

template <int NT, bool QF32, int FMT>
__global__ void __launch_bounds__(kDecodeWarps * 32) decode_split_kernel(const DecodeParams p) {
    constexpr bool K8 = (FMT == NF_KV_K8V4);
    constexpr int NR = NT * 8;  // rows held by this CTA
    __shared__ float sm_m[kDecodeWarps][NR];
    __shared__ float sm_l[kDecodeWarps][NR];
    __shared__ float sm_o[kDecodeWarps][NR][kHeadDim + 4];

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int b = blockIdx.z, h = blockIdx.y;
    const int split = blockIdx.x / p.n_row_groups, rg = blockIdx.x % p.n_row_groups;
    const int row0 = rg * kRowsPerCta;

    int L = p.seqlens[b];
    if (L < p.n_q || L > p.max_seqlen) {
        if (threadIdx.x == 0 && split == 0 && rg == 0 && h == 0) report(NF_DEVERR_SEQLEN);
        L = 0;
    }
    const int t0 = split * p.split_len;
    const int t1 = min(t0 + p.split_len, L);

    // ---- query fragments (B operand of S^T = K . Q^T), permuted like the K bytes
    uint32_t qf[NT][8][2];
    uint32_t ql[QF32 ? NT : 1][8][2];
    int lim[NT][2];  // last visible key position for rows 8nt+2t+e (-1: row unused)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int r = row0 + nt * 8 + g;
        const bool rv = r < p.rows_per_head;
        const int j = rv ? r / p.group : 0, gq = rv ? r % p.group : 0;
        const size_t qoff = (((size_t)b * p.n_q + j) * p.num_q_heads + (size_t)h * p.group + gq) * kHeadDim;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const int c = 32 * t + 4 * ks;
            float x[4] = {0.f, 0.f, 0.f, 0.f};
            if (rv) {
                if (QF32) {
                    const float4 v = *reinterpret_cast<const float4 *>(static_cast<const float *>(p.q) + qoff + c);
                    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
                } else {
                    const uint2 v = *reinterpret_cast<const uint2 *>(static_cast<const __nv_bfloat16 *>(p.q) + qoff + c);
                    x[0] = __uint_as_float(v.x << 16); x[1] = __uint_as_float(v.x & 0xFFFF0000u);
                    x[2] = __uint_as_float(v.y << 16); x[3] = __uint_as_float(v.y & 0xFFFF0000u);
                }
            }
            if (K8) {
                qf[nt][ks][0] = pack_f16(x[0], x[1]);
                qf[nt][ks][1] = pack_f16(x[2], x[3]);
                if (QF32) {
                    const float2 h0 = __half22float2(u32_h2(qf[nt][ks][0]));
                    const float2 h1 = __half22float2(u32_h2(qf[nt][ks][1]));
                    ql[nt][ks][0] = pack_f16(x[0] - h0.x, x[1] - h0.y);
                    ql[nt][ks][1] = pack_f16(x[2] - h1.x, x[3] - h1.y);
                }
            } else {
                qf[nt][ks][0] = pack_bf16(x[0], x[1]);
                qf[nt][ks][1] = pack_bf16(x[2], x[3]);
                if (QF32) {
                    const float lo0 = x[0] - __uint_as_float(qf[nt][ks][0] << 16);
                    const float lo1 = x[1] - __uint_as_float(qf[nt][ks][0] & 0xFFFF0000u);
                    const float lo2 = x[2] - __uint_as_float(qf[nt][ks][1] << 16);
                    const float lo3 = x[3] - __uint_as_float(qf[nt][ks][1] & 0xFFFF0000u);
                    ql[nt][ks][0] = pack_bf16(lo0, lo1);
                    ql[nt][ks][1] = pack_bf16(lo2, lo3);
                }
            }
        }
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int rr = row0 + nt * 8 + 2 * t + e;
            if (rr >= p.rows_per_head) lim[nt][e] = -1;
            else lim[nt][e] = p.causal ? (L - p.n_q + rr / p.group) : (L - 1);
        }
    }

    float m_run[NT][2], l_run[NT][2];
    float acc[8][NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        m_run[nt][0] = m_run[nt][1] = -INFINITY;
        l_run[nt][0] = l_run[nt][1] = 0.f;
#pragma unroll
        for (int m = 0; m < 8; ++m) acc[m][nt][0] = acc[m][nt][1] = acc[m][nt][2] = acc[m][nt][3] = 0.f;
    }

    const int ntiles = t1 > t0 ? (t1 - t0 + kTile - 1) / kTile : 0;
    const int32_t *bt = p.block_table + (size_t)b * p.max_blocks;

    for (int tile = warp; tile < ntiles; tile += kDecodeWarps) {
        const int tb = t0 + tile * kTile;
        const int blk = bt[tb >> 8];
        if (blk < 0 || blk >= p.num_blocks) {
            if (lane == 0) report(NF_DEVERR_BLOCK_ID);
            continue;
        }
        const size_t si = ((size_t)blk * p.num_kv_heads + h) * kBlock + (tb & (kBlock - 1));
        const bool vg0 = tb + g < L, vg1 = tb + g + 8 < L;

        // ---- loads for tokens g and g + 8
        uint4 kq[2][K8 ? 2 : 4];
        uint4 vq[2][K8 ? 1 : 4];
        float sk[2];
        uint32_t sv[2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const size_t s = si + g + 8 * hh;
            if (K8) {
                const int8_t *kp = static_cast<const int8_t *>(p.k_codes) + s * kHeadDim + 32 * t;
                kq[hh][0] = ldg16(kp);
                kq[hh][1] = ldg16(kp + 16);
                vq[hh][0] = ldg16(static_cast<const uint8_t *>(p.v_codes) + s * (kHeadDim / 2) + 16 * t);
                sk[hh] = __half2float(p.k_scales[s]);
                const __half vs = p.v_scales[s * (kHeadDim / kVGroup) + t];
                sv[hh] = h2_u32(__half2half2(vs));
            } else {
                const __nv_bfloat16 *kp = static_cast<const __nv_bfloat16 *>(p.k_codes) + s * kHeadDim + 32 * t;
                const __nv_bfloat16 *vp = static_cast<const __nv_bfloat16 *>(p.v_codes) + s * kHeadDim + 32 * t;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    kq[hh][u] = ldg16(kp + 8 * u);
                    vq[hh][u] = ldg16(vp + 8 * u);
                }
                sk[hh] = 1.0f;
            }
        }
        // keys past the end of the sequence: their slots hold stale bytes, so
        // their values are zeroed (not just their weights)
        if (K8) {
            if (!vg0) sv[0] = 0u;
            if (!vg1) sv[1] = 0u;
        } else {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                if (!vg0) vq[0][u] = make_uint4(0, 0, 0, 0);
                if (!vg1) vq[1][u] = make_uint4(0, 0, 0, 0);
            }
        }

        // ---- S^T = K . Q^T
        float s[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            uint32_t a0, a1, a2, a3;
            if (K8) {
                const uint32_t w0 = reinterpret_cast<const uint32_t *>(&kq[0][ks >> 2])[ks & 3];
                const uint32_t w1 = reinterpret_cast<const uint32_t *>(&kq[1][ks >> 2])[ks & 3];
                i8x4_to_f16(w0, a0, a2);
                i8x4_to_f16(w1, a1, a3);
            } else {
                // 4 bf16 channels 32t + 4ks .. +3: words 2ks, 2ks+1 of the 32-channel run
                const uint32_t *k0 = reinterpret_cast<const uint32_t *>(&kq[0][0]);
                const uint32_t *k1 = reinterpret_cast<const uint32_t *>(&kq[1][0]);
                a0 = k0[2 * ks]; a2 = k0[2 * ks + 1];
                a1 = k1[2 * ks]; a3 = k1[2 * ks + 1];
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                if (K8) {
                    mma_f16(s[nt], a0, a1, a2, a3, qf[nt][ks][0], qf[nt][ks][1]);
                    if (QF32) mma_f16(s[nt], a0, a1, a2, a3, ql[nt][ks][0], ql[nt][ks][1]);
                } else {
                    mma_bf16(s[nt], a0, a1, a2, a3, qf[nt][ks][0], qf[nt][ks][1]);
                    if (QF32) mma_bf16(s[nt], a0, a1, a2, a3, ql[nt][ks][0], ql[nt][ks][1]);
                }
            }
        }

        // ---- online softmax (log2 domain); rows 8nt + 2t + e, tokens g and g + 8
        uint32_t pb0[NT], pb1[NT], pb0l[NT], pb1l[NT];
        const float c0 = sk[0] * p.scale_log2, c1 = sk[1] * p.scale_log2;
        const int pos0 = tb + g, pos1 = tb + g + 8;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            float pr[2][2];  // [token half][e]
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const float x0 = (vg0 && pos0 <= lim[nt][e]) ? s[nt][e] * c0 : -INFINITY;
                const float x1 = (vg1 && pos1 <= lim[nt][e]) ? s[nt][2 + e] * c1 : -INFINITY;
                float mx = fmaxf(x0, x1);
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                const float m_new = fmaxf(m_run[nt][e], mx);
                const float m_use = m_new == -INFINITY ? 0.f : m_new;
                const float alpha = ex2(m_run[nt][e] - m_use);
                m_run[nt][e] = m_new;
                pr[0][e] = ex2(x0 - m_use);
                pr[1][e] = ex2(x1 - m_use);
                l_run[nt][e] = l_run[nt][e] * alpha + pr[0][e] + pr[1][e];
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    acc[m][nt][e] *= alpha;
                    acc[m][nt][2 + e] *= alpha;
                }
            }
            if (K8) {
                pb0[nt] = movmatrix_t(pack_f16(pr[0][0], pr[0][1]));
                pb1[nt] = movmatrix_t(pack_f16(pr[1][0], pr[1][1]));
            } else {
                // bf16 P split into hi + lo so the weights keep ~16 bits
                const uint32_t h0 = pack_bf16(pr[0][0], pr[0][1]);
                const uint32_t h1 = pack_bf16(pr[1][0], pr[1][1]);
                pb0[nt] = movmatrix_t(h0);
                pb1[nt] = movmatrix_t(h1);
                pb0l[nt] = movmatrix_t(pack_bf16(pr[0][0] - __uint_as_float(h0 << 16),
                                                 pr[0][1] - __uint_as_float(h0 & 0xFFFF0000u)));
                pb1l[nt] = movmatrix_t(pack_bf16(pr[1][0] - __uint_as_float(h1 << 16),
                                                 pr[1][1] - __uint_as_float(h1 & 0xFFFF0000u)));
            }
        }

        // ---- O^T += V^T . P^T over 8 m-tiles of 16 channels
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            uint32_t xa0, xb0, xa1, xb1;  // 8x8 tiles p = 2m, 2m+1 for token halves 0, 1
            if (K8) {
                const int i = m >> 1;
                const uint32_t w0 = reinterpret_cast<const uint32_t *>(&vq[0][0])[i] >> ((m & 1) * 8);
                const uint32_t w1 = reinterpret_cast<const uint32_t *>(&vq[1][0])[i] >> ((m & 1) * 8);
                const __half2 s0 = u32_h2(sv[0]), s1 = u32_h2(sv[1]);
                xa0 = h2_u32(__hmul2(nib_even(w0), s0));
                xb0 = h2_u32(__hmul2(nib_odd(w0), s0));
                xa1 = h2_u32(__hmul2(nib_even(w1), s1));
                xb1 = h2_u32(__hmul2(nib_odd(w1), s1));
            } else {
                const uint32_t *v0 = reinterpret_cast<const uint32_t *>(&vq[0][0]);
                const uint32_t *v1 = reinterpret_cast<const uint32_t *>(&vq[1][0]);
                xa0 = v0[2 * m]; xb0 = v0[2 * m + 1];
                xa1 = v1[2 * m]; xb1 = v1[2 * m + 1];
            }
            const uint32_t a0 = movmatrix_t(xa0), a1 = movmatrix_t(xb0);
            const uint32_t a2 = movmatrix_t(xa1), a3 = movmatrix_t(xb1);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                if (K8) {
                    mma_f16(acc[m][nt], a0, a1, a2, a3, pb0[nt], pb1[nt]);
                } else {
                    mma_bf16(acc[m][nt], a0, a1, a2, a3, pb0[nt], pb1[nt]);
                    mma_bf16(acc[m][nt], a0, a1, a2, a3, pb0l[nt], pb1l[nt]);
                }
            }
        }
    }

    // ---- merge the warps of the CTA
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            float l = l_run[nt][e];
            l += __shfl_xor_sync(0xffffffffu, l, 4);
            l += __shfl_xor_sync(0xffffffffu, l, 8);
            l += __shfl_xor_sync(0xffffffffu, l, 16);
            if (g == 0) {
                sm_m[warp][nt * 8 + 2 * t + e] = m_run[nt][e];
                sm_l[warp][nt * 8 + 2 * t + e] = l;
            }
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const int ch0 = K8 ? v_channel_k8v4(m, g) : v_channel_bf16(m, g);
                const int ch1 = K8 ? v_channel_k8v4(m, g + 8) : v_channel_bf16(m, g + 8);
                sm_o[warp][nt * 8 + 2 * t + e][ch0] = acc[m][nt][e];
                sm_o[warp][nt * 8 + 2 * t + e][ch1] = acc[m][nt][2 + e];
            }
        }
    __syncthreads();

    for (int idx = threadIdx.x; idx < NR * kHeadDim; idx += blockDim.x) {
        const int rr = idx / kHeadDim, ch = idx % kHeadDim;
        const int r = row0 + rr;
        if (r >= p.rows_per_head) continue;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kDecodeWarps; ++w) M = fmaxf(M, sm_m[w][rr]);
        float o = 0.f, lse = -INFINITY;
        if (M != -INFINITY) {
            float lsum = 0.f, osum = 0.f;
#pragma unroll
            for (int w = 0; w < kDecodeWarps; ++w) {
                const float f = ex2(sm_m[w][rr] - M);
                lsum += sm_l[w][rr] * f;
                osum += sm_o[w][rr][ch] * f;
            }
            o = osum / lsum;
            lse = (M + log2f(lsum)) * 0.69314718055994531f;
        }
        const int j = r / p.group, gq = r % p.group;
        const size_t grow = ((size_t)b * p.n_q + j) * p.num_q_heads + (size_t)h * p.group + gq;
        p.part_o[((size_t)split * p.rows_total + grow) * kHeadDim + ch] = o;
        if (ch == 0) p.part_lse[(size_t)split * p.rows_total + grow] = lse;
    }
}

}  // namespace nf
