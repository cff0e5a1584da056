// nf_common.cuh -- device helpers shared by the kernels of libnf (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "nf.h"

namespace nf {

constexpr int kHeadDim = 128;
constexpr int kBlock = 256;   // tokens per KV segment
constexpr int kVGroup = 32;   // V channels per scale

// First device-side problem seen since the last nf_get_device_error().
__device__ int32_t g_device_error;

__device__ __forceinline__ void report(int32_t code) { atomicCAS(&g_device_error, 0, code); }

__device__ __forceinline__ uint32_t h2_u32(__half2 h) { return *reinterpret_cast<uint32_t *>(&h); }
__device__ __forceinline__ __half2 u32_h2(uint32_t u) { return *reinterpret_cast<__half2 *>(&u); }

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
    return h2_u32(__floats2half2_rn(lo, hi));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// Two 2^x at once on the MUFU unit, fp16 in and out (-inf gives +0).
__device__ __forceinline__ uint32_t ex2_h2(uint32_t x) {
    uint32_t y;
    asm("ex2.approx.f16x2 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}
// 2^x on the MUFU unit (relative error ~2^-22; -inf gives +0).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// D = A * B + D, m16n8k16, fp16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Same with bf16 inputs.
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D = A * B + D, m16n8k32, int8 inputs, int32 accumulate (exact).
__device__ __forceinline__ void mma_s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                       uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Transpose an 8x8 matrix of 16-bit elements held one row-pair per lane.
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

// ---------------------------------------------------------------- mbarrier / TMA
__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// Wait for the phase of `bar` with the given parity to complete, for at most
// kWaitLimitNs.  Returns false on timeout (the caller records the error).
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s
// try_wait that lets the thread sleep (up to `ns`) until the phase completes,
// instead of spinning and taking issue slots from the warps that do the work
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t *bar, uint32_t parity, uint32_t ns) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity), "r"(ns)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_limit(uint64_t *bar, uint32_t parity, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait_sleep(bar, parity, 100000u))
        if (global_ns() - t0 > limit_ns) return false;
    return true;
}
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity) {
    return mbar_wait_limit(bar, parity, kWaitLimitNs);
}
// Non-blocking test of the phase with the given parity.
__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// The same wait without the sleeping form: try_wait (which holds the thread for
// a short, hardware-defined time) in a loop, for waits on short pipeline steps
// where waking from a long sleep would cost more than the step.  Bounded by
// kWaitLimitNs like mbar_wait.
__device__ __forceinline__ bool mbar_wait_spin(uint64_t *bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t n = 1;; ++n) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((n & 255u) == 0 && global_ns() - t0 > kWaitLimitNs) return false;
    }
}
// 1-D bulk copy global -> shared on the TMA engine, completing on `bar`
// (16-byte aligned addresses, size a multiple of 16).  No multicast.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}
// 2-D tiled copy global -> shared on the TMA engine through a tensor map (a
// __grid_constant__ kernel parameter), completing on `bar`.  x is the inner
// (contiguous) coordinate in elements, y the row.  No multicast.
__device__ __forceinline__ void tma_load_2d(void *dst, const void *tmap, int x, int y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(smem_addr(bar))
        : "memory");
}
// Four 8x8 matrices of 16-bit elements from shared memory, transposed: lanes
// 8i..8i+7 give the row addresses of matrix i; lane (g, t) receives elements
// [2t][g] (low half) and [2t+1][g] (high half) of each matrix.
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    return __byte_perm(a, b, sel);
}
// prmt with the full 4-bit selectors: a selector nibble with its top bit set
// fills its byte with the sign of the selected byte (0x00 for bytes < 0x80).
__device__ __forceinline__ uint32_t prmt_sx(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}
// Programmatic dependent launch.  pdl_wait: block until the grids this one
// depends on have completed and their memory operations are visible (at once
// when the kernel was launched without the attribute); every kernel of libnf
// calls it before its first global-memory access.  pdl_trigger: let the next
// kernel in the stream start placing its CTAs (they block in pdl_wait).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
// atomicAdd with release semantics at GPU scope (returns the old value).
__device__ __forceinline__ int atomic_add_release(int *p, int v) {
    int old;
    asm volatile("atom.release.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}
// Ticket on a counter that both publishes this CTA's earlier writes (release)
// and, for the CTA that draws the last ticket, makes the other CTAs' writes
// visible to it (acquire).
__device__ __forceinline__ int atomic_add_acq_rel(int *p, int v) {
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}
// Reciprocal and base-2 logarithm, hardware approximations (relative error
// about 2^-23 and absolute about 2^-22), for epilogues whose results only need
// to lie well inside the output tolerance.
__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float lg2_approx(float x) {
    float y;
    asm("lg2.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// Load with acquire semantics at GPU scope (sees, and orders after, the
// writes a release by another CTA published).
__device__ __forceinline__ int ld_acquire(const int *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
// Brings a line of global memory into L2 (no value is read into the thread).
__device__ __forceinline__ void prefetch_l2(const void *p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}
// Named barrier among `count` threads (a multiple of 32).
__device__ __forceinline__ void named_sync(uint32_t id, uint32_t count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
__device__ __forceinline__ uint4 lds128(const void *p) { return *reinterpret_cast<const uint4 *>(p); }
// 16-byte shared-memory load at a shared-window address.
__device__ __forceinline__ float4 lds_f4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
    return v;
}

// Read-only 16-byte global load.
__device__ __forceinline__ uint4 ldg16(const void *p) {
    return __ldg(reinterpret_cast<const uint4 *>(p));
}

// Four int8 codes (one per byte of w) -> two fp16x2: even = (c0, c2), odd =
// (c1, c3).  Offset-binary trick: byte u = c + 128 placed under the exponent
// of 1024 gives the fp16 value 1024 + u exactly; subtracting 1152 leaves c
// exactly.
__device__ __forceinline__ void i8x4_to_f16_eo(uint32_t w, uint32_t &even, uint32_t &odd) {
    const uint32_t u = w ^ 0x80808080u;
    const __half2 bias = u32_h2(0x64806480u);  // 1152, 1152
    even = h2_u32(__hsub2(u32_h2(__byte_perm(u, 0x64646464u, 0x4240)), bias));
    odd = h2_u32(__hsub2(u32_h2(__byte_perm(u, 0x64646464u, 0x4341)), bias));
}
// The same in byte order: lo = (c0, c1), hi = (c2, c3).
__device__ __forceinline__ void i8x4_to_f16(uint32_t w, uint32_t &lo, uint32_t &hi) {
    const uint32_t u = w ^ 0x80808080u;
    const __half2 bias = u32_h2(0x64806480u);
    lo = h2_u32(__hsub2(u32_h2(__byte_perm(u, 0x64646464u, 0x4140)), bias));
    hi = h2_u32(__hsub2(u32_h2(__byte_perm(u, 0x64646464u, 0x4342)), bias));
}

// fp8 e4m3 <-> fp16 / fp32 with the hardware conversions (sm_89 and later).
// e4m3x4_to_f16: the four e4m3 bytes of w -> (b0, b1) and (b2, b3) as fp16x2,
// exact (every e4m3 value is an fp16 value).
__device__ __forceinline__ void e4m3x4_to_f16(uint32_t w, uint32_t &lo, uint32_t &hi) {
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, l;\n\tcvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(w));
}
// Four fp32 values -> four e4m3 bytes (x0 in the low byte), each rounded half
// to even and saturated at +-448.
__device__ __forceinline__ uint32_t f32x4_to_e4m3(float x0, float x1, float x2, float x3) {
    uint32_t d;
    // cvt ... d16, a, b puts a in the upper byte and b in the lower one
    asm("{\n\t.reg .b16 l, h;\n\tcvt.rn.satfinite.e4m3x2.f32 l, %2, %1;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 h, %4, %3;\n\tmov.b32 %0, {l, h};\n\t}"
        : "=r"(d)
        : "f"(x0), "f"(x1), "f"(x2), "f"(x3));
    return d;
}

// Packed two's-complement nibbles -> fp16x2 codes, exact.  For a word w with
// nibbles n0..n7 (n_k in bits 4k..4k+3):
//   nib_even(w) = (n0, n4) as fp16 values in [-8, 7]
//   nib_odd(w)  = (n1, n5)
// (apply to w >> 8 for (n2, n6) and (n3, n7)).  The sign bit is flipped to get
// u = c + 8; u sits under the exponent of 1024 (or 1024 * 16 for the odd
// nibble) and the bias is removed exactly.
// One lop3 does the sign flip, the mask and the exponent insertion: where mask
// bit b is set the result is w ^ c, elsewhere c (truth table 0x6a).
__device__ __forceinline__ uint32_t lop3_sel_xor(uint32_t w, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0x6a;" : "=r"(d) : "r"(w), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ __half2 nib_even(uint32_t w) {
    const uint32_t x = lop3_sel_xor(w, 0x000F000Fu, 0x64086408u);      // 1024 + u
    return __hsub2(u32_h2(x), u32_h2(0x64086408u));                      // - 1032
}
__device__ __forceinline__ __half2 nib_odd(uint32_t w) {
    const uint32_t x = lop3_sel_xor(w, 0x00F000F0u, 0x64806480u);      // 1024 + 16u
    return __hfma2(u32_h2(x), u32_h2(0x2C002C00u), u32_h2(0xD480D480u)); // /16 - 72
}

}  // namespace nf
