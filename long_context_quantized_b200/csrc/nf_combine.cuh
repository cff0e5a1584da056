// nf_combine.cuh -- log-sum-exp merge of split-K attention partials.
//
// The splits come either as two arrays (o [splits][rows][d], lse
// [splits][rows]) or packed, one slot per split holding its o rows and then
// its lse values (the layout of the decode kernel's split partials).
// One CTA of 8 warps per output row.  The splits are dealt round-robin to the
// warps (so the loads of different splits are in flight together instead of
// one after another); each lane owns 4 consecutive channels per 128 of the
// row (16-byte loads, coalesced across the warp).  Weights are exp(lse_j - M)
// with M the largest split lse; splits that saw no key carry lse = -inf and
// get weight 0.  The warps' sums are added in shared memory.
#pragma once

#include "nf_common.cuh"

namespace nf {

constexpr int kCombineWarps = 8;
constexpr int kCombineMaxDim = 1024;

struct CombineParams {
    const float *part_o;    // split j's row r at part_o + j * o_stride + r * head_dim
    const float *part_lse;  // split j's row r at part_lse + j * lse_stride + r
    int n_splits, rows, head_dim;
    size_t o_stride, lse_stride;  // floats between consecutive splits
    float *out;
    float *out_lse;
};

__global__ void __launch_bounds__(kCombineWarps * 32) combine_kernel(const CombineParams p) {
    __shared__ float red[kCombineWarps];
    __shared__ float4 acc_sm[kCombineWarps][kCombineMaxDim / 4];
    constexpr float kLog2e = 1.4426950408889634f;
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int row = blockIdx.x;
    const float *lse_col = p.part_lse + row;  // stride p.lse_stride

    // M = max_j lse_j
    float M = -INFINITY;
    for (int j = threadIdx.x; j < p.n_splits; j += blockDim.x) M = fmaxf(M, lse_col[(size_t)j * p.lse_stride]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    if (lane == 0) red[warp] = M;
    __syncthreads();
    M = red[0];
#pragma unroll
    for (int w = 1; w < kCombineWarps; ++w) M = fmaxf(M, red[w]);
    __syncthreads();

    if (M == -INFINITY) {  // no split saw a key
        for (int c = 4 * threadIdx.x; c < p.head_dim; c += 4 * blockDim.x)
            *reinterpret_cast<float4 *>(p.out + (size_t)row * p.head_dim + c) = make_float4(0.f, 0.f, 0.f, 0.f);
        if (threadIdx.x == 0 && p.out_lse) p.out_lse[row] = -INFINITY;
        return;
    }

    const int nchunk = p.head_dim / 4;  // float4 chunks per row
    float wsum = 0.f;
    for (int c0 = 0; c0 < nchunk; c0 += 32) {
        const int c = c0 + lane;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        float ws = 0.f;
#pragma unroll 4
        for (int j = warp; j < p.n_splits; j += kCombineWarps) {
            const float w = ex2((lse_col[(size_t)j * p.lse_stride] - M) * kLog2e);  // -inf -> 0
            ws += w;
            if (c < nchunk && w > 0.f) {
                const float4 o =
                    reinterpret_cast<const float4 *>(p.part_o + (size_t)j * p.o_stride + (size_t)row * p.head_dim)[c];
                acc.x += w * o.x; acc.y += w * o.y; acc.z += w * o.z; acc.w += w * o.w;
            }
        }
        if (c < nchunk) acc_sm[warp][c] = acc;
        if (c0 == 0) wsum = ws;
    }
    if (lane == 0) red[warp] = wsum;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < kCombineWarps; ++w) tot += red[w];
    const float inv = 1.0f / tot;
    for (int c = threadIdx.x; c < nchunk; c += blockDim.x) {
        float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w = 0; w < kCombineWarps; ++w) {
            const float4 a = acc_sm[w][c];
            s.x += a.x; s.y += a.y; s.z += a.z; s.w += a.w;
        }
        s.x *= inv; s.y *= inv; s.z *= inv; s.w *= inv;
        reinterpret_cast<float4 *>(p.out + (size_t)row * p.head_dim)[c] = s;
    }
    if (threadIdx.x == 0 && p.out_lse) p.out_lse[row] = M + logf(tot);
}

}  // namespace nf
