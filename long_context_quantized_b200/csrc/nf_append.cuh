// nf_append.cuh -- quantise-and-append of new K/V tokens into the segmented
// pool (the rk8v4 KV dtype of page "3090 单卡跑 Qwen3.8-27B：NInfer 上机实测",
// section 一.3; bit format as defined in nf.h).
//
// One warp per (sequence, new token, kv-head); lane l owns channels 4l..4l+3.
// K: absmax over the warp -> fp16 scale absmax/127 -> int8 codes (4 bytes per
// lane, a coalesced 128-byte row).  V: absmax over each 8-lane group of 32
// channels -> fp16 scale absmax/7 -> 4 nibbles per lane packed into 2 bytes;
// for the int8 KV dtype (same section, --kv-dtype int8) V takes the K rule; the
// fp8 dtype (--kv-dtype fp8) stores e4m3 codes of x / (absmax / 448) for both;
// the RK4V4-E8 reading (page "影片筆記：NInfer + 千问3.8 27b = 1.5倍速@256K上下文",
// section 三) stores 4-bit codes of both with a power-of-two scale per 32 channels.
// Division and rounding are the IEEE fp32 ones (__fdiv_rn, round half to even),
// subnormals kept, so the codes are bit-identical to the format definition.
#pragma once

#include "nf_common.cuh"

namespace nf {

struct AppendParams {
    const void *k_new;
    const void *v_new;
    int in_f32;  // 1: fp32 inputs, 0: bf16 inputs
    int batch, n_new, num_kv_heads;
    const int32_t *block_table;
    int max_blocks;
    const int32_t *seqlens_before;
    int num_blocks;
    int fmt;
    void *k_codes;
    __half *k_scales;
    void *v_codes;
    __half *v_scales;
};

__device__ __forceinline__ void load4(const void *base, size_t elem, bool f32, float (&x)[4]) {
    if (f32) {
        const float4 v = *reinterpret_cast<const float4 *>(static_cast<const float *>(base) + elem);
        x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
    } else {
        const uint2 v =
            *reinterpret_cast<const uint2 *>(static_cast<const __nv_bfloat16 *>(base) + elem);
        x[0] = __uint_as_float(v.x << 16);
        x[1] = __uint_as_float(v.x & 0xFFFF0000u);
        x[2] = __uint_as_float(v.y << 16);
        x[3] = __uint_as_float(v.y & 0xFFFF0000u);
    }
}

// fp16 scale for absmax a and code limit q: fp32 a / q, then fp16 round half to
// even, saturated at 65504 (clamping first gives the same fp16 value).
__device__ __forceinline__ __half make_scale(float a, float q, float &sigma) {
    const float s32 = fminf(__fdiv_rn(a, q), 65504.0f);
    const __half s16 = __float2half_rn(s32);
    sigma = __half2float(s16);
    return s16;
}

__device__ __forceinline__ int make_code(float x, float sigma, int q) {
    if (sigma == 0.0f) return 0;
    const int c = __float2int_rn(__fdiv_rn(x, sigma));  // round half to even
    return min(max(c, -q), q);
}

// One 128-channel row held 4 channels per lane -> int8 codes (absmax / 127
// scale, a coalesced 128-byte row) and its fp16 scale.
__device__ __forceinline__ void quant_row8(const float (&x)[4], int lane, int8_t *codes, __half *scale) {
    float a = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    float sigma;
    const __half h = make_scale(a, 127.0f, sigma);
    uint32_t c8 = 0;
#pragma unroll
    for (int c = 0; c < 4; ++c) c8 |= (uint32_t)(make_code(x[c], sigma, 127) & 0xFF) << (8 * c);
    *reinterpret_cast<uint32_t *>(codes + 4 * lane) = c8;
    if (lane == 0) *scale = h;
}

// The same row -> e4m3 codes of x / scale (scale absmax / 448), 0 when the
// scale is 0.
__device__ __forceinline__ void quant_row_f8(const float (&x)[4], int lane, uint8_t *codes, __half *scale) {
    float a = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    float sigma;
    const __half h = make_scale(a, 448.0f, sigma);
    float t[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) t[c] = sigma == 0.0f ? 0.0f : __fdiv_rn(x[c], sigma);
    *reinterpret_cast<uint32_t *>(codes + 4 * lane) = f32x4_to_e4m3(t[0], t[1], t[2], t[3]);
    if (lane == 0) *scale = h;
}

// RK4V4-E8 (both K and V): one power-of-two scale 2^e per 32 channels = 8
// lanes, e the smallest integer with 2^e >= fp32(absmax / 7) (read from the
// bits of the quotient: an exact power of two keeps its exponent, anything
// above it takes the next one), clamped to [-126, 127] and stored as the byte
// e + 127; codes round_half_even(x / 2^e) clamped to [-7, 7], packed two per
// byte (the even channel in the low nibble).
__device__ __forceinline__ void quant_row_e8(const float (&x)[4], int lane, uint8_t *codes, uint8_t *scales) {
    float a = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    const uint32_t sb = __float_as_uint(__fdiv_rn(a, 7.0f));
    const int ef = (int)(sb >> 23);  // biased exponent; 0 for zero and subnormal quotients
    int e = ef == 0 ? -126 : ef - 127 + ((sb & 0x7FFFFFu) != 0u ? 1 : 0);
    e = min(max(e, -126), 127);
    const float scale = __int_as_float((e + 127) << 23);
    uint32_t c4 = 0;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const int q = min(max(__float2int_rn(__fdiv_rn(x[c], scale)), -7), 7);
        c4 |= (uint32_t)(q & 0xF) << (4 * c);
    }
    *reinterpret_cast<uint16_t *>(codes + 2 * lane) = (uint16_t)c4;
    if ((lane & 7) == 0) scales[lane >> 3] = (uint8_t)(e + 127);
}

__global__ void __launch_bounds__(256) append_quant_kernel(const AppendParams p) {
    // let the next kernel place its CTAs at once (it waits for this grid to
    // complete before it reads what this one writes)
    pdl_trigger();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const long long item = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const long long total = (long long)p.batch * p.n_new * p.num_kv_heads;
    if (item >= total) return;
    const int h = (int)(item % p.num_kv_heads);
    const long long bi = item / p.num_kv_heads;
    const int i = (int)(bi % p.n_new);
    const int b = (int)(bi / p.n_new);

    // the new token's values do not depend on where it goes: load them first,
    // so their latency overlaps the lengths -> block-table lookups
    const size_t src = (size_t)item * kHeadDim + 4 * lane;
    float k[4], v[4];
    load4(p.k_new, src, p.in_f32 != 0, k);
    load4(p.v_new, src, p.in_f32 != 0, v);

    const int pos = p.seqlens_before[b] + i;
    const int blk_i = pos >> 8;
    if (pos < 0 || blk_i >= p.max_blocks) {
        if (lane == 0) report(NF_DEVERR_TABLE);
        return;
    }
    const int blk = p.block_table[(size_t)b * p.max_blocks + blk_i];
    if (blk < 0 || blk >= p.num_blocks) {
        if (lane == 0) report(NF_DEVERR_BLOCK_ID);
        return;
    }
    const size_t si = ((size_t)blk * p.num_kv_heads + h) * kBlock + (pos & (kBlock - 1));

    if (p.fmt == NF_KV_BF16) {
        uint2 kb, vb;
        kb.x = pack_bf16(k[0], k[1]); kb.y = pack_bf16(k[2], k[3]);
        vb.x = pack_bf16(v[0], v[1]); vb.y = pack_bf16(v[2], v[3]);
        *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(p.k_codes) + si * kHeadDim + 4 * lane) = kb;
        *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(p.v_codes) + si * kHeadDim + 4 * lane) = vb;
        return;
    }

    if (p.fmt == NF_KV_K4V4) {
        quant_row_e8(k, lane, static_cast<uint8_t *>(p.k_codes) + si * (kHeadDim / 2),
                     reinterpret_cast<uint8_t *>(p.k_scales) + si * (kHeadDim / 32));
        quant_row_e8(v, lane, static_cast<uint8_t *>(p.v_codes) + si * (kHeadDim / 2),
                     reinterpret_cast<uint8_t *>(p.v_scales) + si * (kHeadDim / 32));
        return;
    }

    if (p.fmt == NF_KV_F8) {
        quant_row_f8(k, lane, static_cast<uint8_t *>(p.k_codes) + si * kHeadDim, p.k_scales + si);
        quant_row_f8(v, lane, static_cast<uint8_t *>(p.v_codes) + si * kHeadDim, p.v_scales + si);
        return;
    }

    // ---- K: one scale per (token, kv-head)
    quant_row8(k, lane, static_cast<int8_t *>(p.k_codes) + si * kHeadDim, p.k_scales + si);
    if (p.fmt == NF_KV_K8V8) {
        // int8 KV: V by the same rule
        quant_row8(v, lane, static_cast<int8_t *>(p.v_codes) + si * kHeadDim, p.v_scales + si);
        return;
    }

    // ---- V: one scale per 32 channels = 8 lanes
    float av = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) av = fmaxf(av, __shfl_xor_sync(0xffffffffu, av, o));
    float sv;
    const __half hv = make_scale(av, 7.0f, sv);
    uint32_t vc = 0;
#pragma unroll
    for (int c = 0; c < 4; ++c) vc |= (uint32_t)(make_code(v[c], sv, 7) & 0xF) << (4 * c);
    *reinterpret_cast<uint16_t *>(static_cast<uint8_t *>(p.v_codes) + si * (kHeadDim / 2) + 2 * lane) =
        (uint16_t)vc;
    if ((lane & 7) == 0) p.v_scales[si * (kHeadDim / kVGroup) + (lane >> 3)] = hv;
}

}  // namespace nf
