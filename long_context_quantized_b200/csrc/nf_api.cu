// nf_api.cu -- the C ABI of libnf: host-side validation, split planning and
// kernel launches.  The declarations and their contracts are in include/nf.h.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <atomic>
#include <mutex>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "nf.h"
#include "nf_append.cuh"
#include "nf_combine.cuh"
#include "nf_common.cuh"
#include "nf_decode.cuh"
#include "nf_decode_tc.cuh"
#include "nf_prefill.cuh"

namespace nf {
// Self-test of the bounded wait: one thread waits on an mbarrier that nothing
// arrives on, for at most limit_ns, and records NF_DEVERR_TIMEOUT when the
// wait gives up (the path every wait of the decode kernel takes on a stall).
__global__ void bounded_wait_selftest_kernel(uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    fence_mbar_init();
    if (!mbar_wait_limit(&bar, 0, limit_ns)) report(NF_DEVERR_TIMEOUT);
    asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(smem_addr(&bar)) : "memory");
}
}  // namespace nf

namespace {

thread_local char g_msg[512] = "";

nf_status fail(nf_status s, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
    va_end(ap);
    return s;
}

nf_status after_launch(const char *what) {
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(NF_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    g_msg[0] = '\0';
    return NF_OK;
}

nf_status check_layer(const nf_kv_layer *kv) {
    if (!kv) return fail(NF_ERR_INVALID_ARG, "kv is NULL");
    if (kv->fmt != NF_KV_K8V4 && kv->fmt != NF_KV_K8V8 && kv->fmt != NF_KV_F8 && kv->fmt != NF_KV_K4V4 &&
        kv->fmt != NF_KV_BF16)
        return fail(NF_ERR_UNSUPPORTED,
                    "kv->fmt %d is not NF_KV_K8V4, NF_KV_K8V8, NF_KV_F8, NF_KV_K4V4 or NF_KV_BF16", kv->fmt);
    const bool scaled = kv->fmt != NF_KV_BF16;
    if (kv->block_size != nf::kBlock)
        return fail(NF_ERR_UNSUPPORTED, "kv->block_size %d (only 256)", kv->block_size);
    if (kv->head_dim != nf::kHeadDim)
        return fail(NF_ERR_UNSUPPORTED, "kv->head_dim %d (only 128)", kv->head_dim);
    if (kv->fmt == NF_KV_K8V4 && kv->v_group != nf::kVGroup)
        return fail(NF_ERR_UNSUPPORTED, "kv->v_group %d (only 32)", kv->v_group);
    if (kv->num_blocks < 1 || kv->num_kv_heads < 1)
        return fail(NF_ERR_INVALID_ARG, "kv->num_blocks %d / num_kv_heads %d must be >= 1",
                    kv->num_blocks, kv->num_kv_heads);
    if (!kv->k_codes || !kv->v_codes) return fail(NF_ERR_INVALID_ARG, "kv code planes are NULL");
    if (scaled && (!kv->k_scales || !kv->v_scales))
        return fail(NF_ERR_INVALID_ARG, "kv scale planes are NULL");
    auto misaligned = [](const void *ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15) != 0; };
    if (misaligned(kv->k_codes) || misaligned(kv->v_codes) ||
        (scaled && (misaligned(kv->k_scales) || misaligned(kv->v_scales))))
        return fail(NF_ERR_INVALID_ARG, "kv planes must be 16-byte aligned");
    return NF_OK;
}

// ---------------------------------------------------------------- plan
// The decode kernel is persistent: one CTA per SM, each taking an equal share
// of all (sequence, kv-head) key chunks (computed on the device from seqlens).
// The workspace holds ticket counters -- one per (sequence, kv-head) and one
// per partial slot, zero between calls -- and one (o, lse) partial slot per
// CTA plus one per segment (a CTA's pieces and a segment's pieces both form
// contiguous runs, so slot segment + cta is unique).
struct Plan {
    int ctas = 0, nt = 0, n_rg = 0, rows = 0, segments = 0, slot_floats = 0;
    size_t ticket_bytes = 0, partial_bytes = 0;
    size_t bytes() const { return ticket_bytes + partial_bytes; }
};

bool make_plan(int batch, int n_q, int H_q, int H_kv, int max_seqlen, int num_sms, Plan &pl) {
    if (batch < 1 || n_q < 1 || H_q < 1 || H_kv < 1 || H_q % H_kv != 0 || max_seqlen < n_q ||
        num_sms < 1 || batch > nf::kMaxBatch)
        return false;
    const long long rows = (long long)(H_q / H_kv) * n_q;
    if (rows > nf::kMaxRows) return false;
    pl.rows = (int)rows;
    pl.nt = rows <= 8 ? 1 : 2;
    pl.n_rg = pl.nt == 1 ? 1 : (int)((rows + 15) / 16);
    if (pl.n_rg == 3) pl.n_rg = 4;  // 8 consumer warps split evenly over 1, 2 or 4 row groups
    pl.ctas = num_sms < nf::kMaxCtas ? num_sms : nf::kMaxCtas;
    pl.segments = batch * H_kv;
    // per segment a ticket and a done counter, then one share flag per
    // partial slot (indexed like the slots)
    pl.ticket_bytes = ((size_t)(2 * pl.segments + pl.ctas + pl.segments) * 4 + 255) / 256 * 256;
    pl.slot_floats = (pl.rows * (nf::kHeadDim + 1) + 3) / 4 * 4;
    pl.partial_bytes = ((size_t)(pl.ctas + pl.segments) * pl.slot_floats * sizeof(float) + 255) / 256 * 256;
    return true;
}

// cuTensorMapEncodeTiled, fetched once from the driver through the runtime (no
// link against libcuda).  It is a host-only function: it packs the tensor map.
PFN_cuTensorMapEncodeTiled_v12000 g_encode_tiled = nullptr;
std::once_flag g_encode_once;

// Tensor map of a quantised layer's V codes (or, k_plane, of its int8 K codes)
// for the decode kernels: the plane as [num_blocks * H_kv * 256 rows][row
// bytes], boxes of box_rows rows (32: any chunk of decode_kernel's stages; a
// whole stage, 128 or 256; 128 for decode_tc_kernel's tiles), the swizzle as
// wide as a row -- K8/V4 nibbles 64 bytes (64-byte swizzle), K8V8 and fp8 V
// codes and int8 K codes 128 bytes (128-byte swizzle).
nf_status encode_v_map(const nf_kv_layer *kv, CUtensorMap *map, bool k_plane = false,
                       unsigned box_rows = nf::kChunk) {
    std::call_once(g_encode_once, [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode_tiled = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    if (!g_encode_tiled) return fail(NF_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    const cuuint64_t rows = (cuuint64_t)kv->num_blocks * (cuuint64_t)kv->num_kv_heads * nf::kBlock;
    if (rows > 0x7fffffffull)
        return fail(NF_ERR_UNSUPPORTED, "pool of %llu token rows per plane (at most 2^31 - 1)", (unsigned long long)rows);
    // 128-byte rows: int8 K codes, int8 / e4m3 V codes; 64-byte rows: nibbles
    const bool v8 = k_plane ? kv->fmt != NF_KV_K4V4 : (kv->fmt == NF_KV_K8V8 || kv->fmt == NF_KV_F8);
    const cuuint64_t row_bytes = v8 ? 128 : 64;
    const cuuint64_t dims[2] = {row_bytes, rows};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {(cuuint32_t)row_bytes, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = g_encode_tiled(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, k_plane ? kv->k_codes : kv->v_codes,
                                      dims, strides, box, estr,
                                      CU_TENSOR_MAP_INTERLEAVE_NONE,
                                      v8 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(NF_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
    return NF_OK;
}

int current_sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return n;
}

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel in the stream finishes; it waits for it (pdl_wait)
// before touching global memory.
template <typename Kern, typename Params>
cudaError_t launch_pdl(Kern kernel, unsigned grid, unsigned block, size_t smem, cudaStream_t s, const Params &p) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, p);
}

template <int NT, bool QF32, int FMT>
cudaError_t launch_decode(const nf::DecodeParams &p, int ctas, cudaStream_t s) {
    constexpr int smem = nf::DecodeSmem<NT, FMT>::kBytes;
    // opt in to the large dynamic shared memory, once per device
    static std::atomic<uint64_t> opted{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = dev < 64 ? (1ull << dev) : 0;
    if (!bit || !(opted.load(std::memory_order_acquire) & bit)) {
        e = cudaFuncSetAttribute(nf::decode_kernel<NT, QF32, FMT>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        opted.fetch_or(bit, std::memory_order_acq_rel);
    }
    return launch_pdl(nf::decode_kernel<NT, QF32, FMT>, (unsigned)ctas, nf::kDecodeThreads, smem, s, p);
}

// The tensor-core decode of many rows (K8/V4 or K8V8, 9 to 32 query rows per
// kv-head), rows padded to RP = 16 or 32.
template <int RP, bool QF32, int FMT>
cudaError_t launch_decode_tc(const nf::DecodeParams &p, int ctas, cudaStream_t s) {
    constexpr int smem = nf::DtSmem<FMT>::kBytes;
    static std::atomic<uint64_t> opted{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = dev < 64 ? (1ull << dev) : 0;
    if (!bit || !(opted.load(std::memory_order_acquire) & bit)) {
        e = cudaFuncSetAttribute(nf::decode_tc_kernel<RP, QF32, FMT>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        opted.fetch_or(bit, std::memory_order_acq_rel);
    }
    return launch_pdl(nf::decode_tc_kernel<RP, QF32, FMT>, (unsigned)ctas, nf::kDtThreads, smem, s, p);
}
template <int FMT>
cudaError_t dispatch_decode_tc(const nf::DecodeParams &p, bool qf32, int rows, int ctas, cudaStream_t s) {
    return rows <= 16 ? (qf32 ? launch_decode_tc<16, true, FMT>(p, ctas, s) : launch_decode_tc<16, false, FMT>(p, ctas, s))
                      : (qf32 ? launch_decode_tc<32, true, FMT>(p, ctas, s) : launch_decode_tc<32, false, FMT>(p, ctas, s));
}

bool uses_decode_tc(int fmt, int rows) {
    return (fmt == NF_KV_K8V4 || fmt == NF_KV_K8V8 || fmt == NF_KV_F8) && rows > 8 && rows <= nf::kDtMaxRows;
}

template <int NT>
cudaError_t dispatch_decode(const nf::DecodeParams &p, bool qf32, int fmt, int ctas, cudaStream_t s) {
    if (fmt == NF_KV_K8V4)
        return qf32 ? launch_decode<NT, true, NF_KV_K8V4>(p, ctas, s) : launch_decode<NT, false, NF_KV_K8V4>(p, ctas, s);
    if (fmt == NF_KV_K8V8)
        return qf32 ? launch_decode<NT, true, NF_KV_K8V8>(p, ctas, s) : launch_decode<NT, false, NF_KV_K8V8>(p, ctas, s);
    if (fmt == NF_KV_F8)
        return qf32 ? launch_decode<NT, true, NF_KV_F8>(p, ctas, s) : launch_decode<NT, false, NF_KV_F8>(p, ctas, s);
    if (fmt == NF_KV_K4V4)
        return qf32 ? launch_decode<NT, true, NF_KV_K4V4>(p, ctas, s) : launch_decode<NT, false, NF_KV_K4V4>(p, ctas, s);
    return qf32 ? launch_decode<NT, true, NF_KV_BF16>(p, ctas, s) : launch_decode<NT, false, NF_KV_BF16>(p, ctas, s);
}

nf_status launch_combine(const float *part_o, const float *part_lse, int n_splits, int rows,
                         int head_dim, size_t o_stride, size_t lse_stride, float *out, float *out_lse,
                         cudaStream_t s) {
    nf::CombineParams c{part_o, part_lse, n_splits, rows, head_dim, o_stride, lse_stride, out, out_lse};
    const cudaError_t e = launch_pdl(nf::combine_kernel, (unsigned)rows, nf::kCombineWarps * 32, 0, s, c);
    if (e != cudaSuccess) return fail(NF_ERR_CUDA, "combine kernel launch: %s", cudaGetErrorString(e));
    return after_launch("combine kernel launch");
}

// Scratch of nf_decode_attn_noalloc (for callers that cannot allocate device
// memory).  It is part of the library's device image, so every GPU that loads
// libnf holds NF_NOALLOC_SCRATCH_BYTES of it until the process exits.  In host
// code the name is only a stand-in for the symbol: its device address comes
// from cudaGetSymbolAddress on each device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[NF_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device, looked up once
// per device with that device current.
nf_status noalloc_scratch(void **ptr) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(NF_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return fail(NF_ERR_UNSUPPORTED, "device %d >= %d", dev, kMaxDevices);
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p)
            return fail(NF_ERR_CUDA, "cudaGetSymbolAddress(no-alloc scratch): %s", cudaGetErrorString(e));
        g_noalloc_ptr[dev] = p;
    }
    *ptr = g_noalloc_ptr[dev];
    return NF_OK;
}

}  // namespace

extern "C" {

nf_status nf_kv_append_quant(const nf_kv_layer *kv, const void *k_new, const void *v_new,
                             int32_t in_dtype, int32_t batch, int32_t n_new,
                             const int32_t *block_table, int32_t max_blocks,
                             const int32_t *seqlens_before, nf_stream_t stream) {
    nf_status st = check_layer(kv);
    if (st != NF_OK) return st;
    if (batch < 0 || n_new < 0) return fail(NF_ERR_INVALID_ARG, "batch %d / n_new %d < 0", batch, n_new);
    if (in_dtype != NF_F32 && in_dtype != NF_BF16)
        return fail(NF_ERR_UNSUPPORTED, "in_dtype %d (NF_F32 or NF_BF16)", in_dtype);
    if ((long long)batch * n_new == 0) {
        g_msg[0] = '\0';
        return NF_OK;
    }
    if (!k_new || !v_new || !block_table || !seqlens_before)
        return fail(NF_ERR_INVALID_ARG, "a device pointer is NULL");
    if (max_blocks < 1) return fail(NF_ERR_INVALID_ARG, "max_blocks %d < 1", max_blocks);
    const size_t align = in_dtype == NF_F32 ? 16 : 8;
    if ((reinterpret_cast<uintptr_t>(k_new) | reinterpret_cast<uintptr_t>(v_new)) & (align - 1))
        return fail(NF_ERR_INVALID_ARG, "k_new / v_new must be %zu-byte aligned", align);
    nf::AppendParams p{};
    p.k_new = k_new;
    p.v_new = v_new;
    p.in_f32 = in_dtype == NF_F32;
    p.batch = batch;
    p.n_new = n_new;
    p.num_kv_heads = kv->num_kv_heads;
    p.block_table = block_table;
    p.max_blocks = max_blocks;
    p.seqlens_before = seqlens_before;
    p.num_blocks = kv->num_blocks;
    p.fmt = kv->fmt;
    p.k_codes = kv->k_codes;
    p.k_scales = static_cast<__half *>(kv->k_scales);
    p.v_codes = kv->v_codes;
    p.v_scales = static_cast<__half *>(kv->v_scales);
    const long long items = (long long)batch * n_new * kv->num_kv_heads;
    const long long blocks = (items + 7) / 8;
    if (blocks > 0x7fffffffLL) return fail(NF_ERR_INVALID_ARG, "too many tokens in one append");
    const cudaError_t e = launch_pdl(nf::append_quant_kernel, (unsigned)blocks, 256, 0,
                                     reinterpret_cast<cudaStream_t>(stream), p);
    if (e != cudaSuccess) return fail(NF_ERR_CUDA, "append kernel launch: %s", cudaGetErrorString(e));
    return after_launch("append kernel launch");
}

size_t nf_decode_attn_workspace_size(int32_t batch, int32_t n_q, int32_t num_q_heads,
                                     int32_t num_kv_heads, int32_t max_seqlen, int32_t num_sms) {
    Plan pl;
    if (!make_plan(batch, n_q, num_q_heads, num_kv_heads, max_seqlen, num_sms, pl)) return 0;
    return pl.bytes();
}

nf_status nf_decode_attn(const nf_kv_layer *kv, const void *q, int32_t q_dtype, int32_t batch,
                         int32_t n_q, int32_t num_q_heads, const int32_t *block_table,
                         int32_t max_blocks, const int32_t *seqlens, int32_t max_seqlen,
                         float softmax_scale, int32_t causal, float *out, float *out_lse,
                         void *workspace, size_t workspace_bytes, nf_stream_t stream) {
    return nf_decode_attn_ex(kv, q, q_dtype, batch, n_q, num_q_heads, block_table, max_blocks, seqlens,
                             max_seqlen, softmax_scale, causal, 0u, out, out_lse, workspace, workspace_bytes,
                             stream);
}

nf_status nf_decode_attn_ex(const nf_kv_layer *kv, const void *q, int32_t q_dtype, int32_t batch,
                            int32_t n_q, int32_t num_q_heads, const int32_t *block_table,
                            int32_t max_blocks, const int32_t *seqlens, int32_t max_seqlen,
                            float softmax_scale, int32_t causal, uint32_t flags, float *out,
                            float *out_lse, void *workspace, size_t workspace_bytes, nf_stream_t stream) {
    if (flags & ~NF_DECODE_EARLY_KV) return fail(NF_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
    nf_status st = check_layer(kv);
    if (st != NF_OK) return st;
    if (q_dtype != NF_F32 && q_dtype != NF_BF16)
        return fail(NF_ERR_UNSUPPORTED, "q_dtype %d (NF_F32 or NF_BF16)", q_dtype);
    if (batch < 1 || n_q < 1 || num_q_heads < 1)
        return fail(NF_ERR_INVALID_ARG, "batch %d, n_q %d, num_q_heads %d must be >= 1", batch, n_q,
                    num_q_heads);
    if (batch > 65535 || kv->num_kv_heads > 65535)
        return fail(NF_ERR_UNSUPPORTED, "batch %d / num_kv_heads %d above 65535", batch, kv->num_kv_heads);
    if (num_q_heads % kv->num_kv_heads != 0)
        return fail(NF_ERR_INVALID_ARG, "num_q_heads %d not a multiple of num_kv_heads %d",
                    num_q_heads, kv->num_kv_heads);
    if (max_seqlen < n_q) return fail(NF_ERR_INVALID_ARG, "max_seqlen %d < n_q %d", max_seqlen, n_q);
    if ((long long)max_blocks * nf::kBlock < max_seqlen)
        return fail(NF_ERR_INVALID_ARG, "max_blocks %d cannot hold max_seqlen %d", max_blocks, max_seqlen);
    if (!q || !block_table || !seqlens || !out) return fail(NF_ERR_INVALID_ARG, "a device pointer is NULL");
    if (!std::isfinite(softmax_scale)) return fail(NF_ERR_INVALID_ARG, "softmax_scale is not finite");
    const uintptr_t qa = reinterpret_cast<uintptr_t>(q);
    if ((q_dtype == NF_F32 && (qa & 15)) || (q_dtype == NF_BF16 && (qa & 7)) ||
        (reinterpret_cast<uintptr_t>(out) & 15))
        return fail(NF_ERR_INVALID_ARG, "q / out misaligned");
    const int sms = current_sm_count();
    if (sms < 1) return fail(NF_ERR_CUDA, "cannot query the current device");
    Plan pl;
    if (!make_plan(batch, n_q, num_q_heads, kv->num_kv_heads, max_seqlen, sms, pl))
        return fail(NF_ERR_UNSUPPORTED, "unsupported shape (batch <= %d and group * n_q <= %d)", nf::kMaxBatch,
                    nf::kMaxRows);
    if (workspace_bytes < pl.bytes() || !workspace)
        return fail(NF_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", workspace_bytes, pl.bytes());
    if (reinterpret_cast<uintptr_t>(workspace) & 255)
        return fail(NF_ERR_INVALID_ARG, "workspace must be 256-byte aligned");

    nf::DecodeParams p{};
    const bool tc = uses_decode_tc(kv->fmt, pl.rows);
    // decode_tc_kernel loads a tile's K and V rows with one box each
    const unsigned box_rows = tc ? (unsigned)nf::kDtTileKeys : (unsigned)nf::kChunk;
    if (kv->fmt != NF_KV_BF16) {
        st = encode_v_map(kv, &p.vmap, false, box_rows);
        if (st != NF_OK) return st;
    }
    if (tc || kv->fmt == NF_KV_K4V4) {
        st = encode_v_map(kv, &p.kmap, true, box_rows);
        if (st != NF_OK) return st;
    }
    if (!tc && kv->fmt != NF_KV_BF16) {
        // decode_kernel: a whole stage's V (and RK4V4 K) rows in one box
        const unsigned stage_rows = (kv->fmt == NF_KV_K8V8 || kv->fmt == NF_KV_F8) ? 128u : 256u;
        st = encode_v_map(kv, &p.vmap_full, false, stage_rows);
        if (st != NF_OK) return st;
        if (kv->fmt == NF_KV_K4V4) {
            st = encode_v_map(kv, &p.kmap_full, true, stage_rows);
            if (st != NF_OK) return st;
        }
    }
    p.k_codes = kv->k_codes;
    p.k_scales = static_cast<const __half *>(kv->k_scales);
    p.v_codes = kv->v_codes;
    p.v_scales = static_cast<const __half *>(kv->v_scales);
    p.num_blocks = kv->num_blocks;
    p.num_kv_heads = kv->num_kv_heads;
    p.q = q;
    p.batch = batch;
    p.n_q = n_q;
    p.num_q_heads = num_q_heads;
    p.group = num_q_heads / kv->num_kv_heads;
    p.rows = pl.rows;
    p.n_rg = pl.n_rg;
    p.block_table = block_table;
    p.max_blocks = max_blocks;
    p.seqlens = seqlens;
    p.max_seqlen = max_seqlen;
    p.scale_log2 = softmax_scale * 1.4426950408889634f;
    p.causal = causal != 0;
    p.early_kv = (flags & NF_DECODE_EARLY_KV) != 0;
    p.out = out;
    p.out_lse = out_lse;
    p.tickets = static_cast<int32_t *>(workspace);
    p.done = p.tickets + pl.segments;
    p.claims = p.done + pl.segments;
    p.partials = reinterpret_cast<float *>(static_cast<char *>(workspace) + pl.ticket_bytes);
    p.slot_floats = pl.slot_floats;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const bool qf32 = q_dtype == NF_F32;
    const cudaError_t e =
        tc ? (kv->fmt == NF_KV_K8V8 ? dispatch_decode_tc<NF_KV_K8V8>(p, qf32, pl.rows, pl.ctas, s)
              : kv->fmt == NF_KV_F8 ? dispatch_decode_tc<NF_KV_F8>(p, qf32, pl.rows, pl.ctas, s)
                                    : dispatch_decode_tc<NF_KV_K8V4>(p, qf32, pl.rows, pl.ctas, s))
        : pl.nt == 1 ? dispatch_decode<1>(p, qf32, kv->fmt, pl.ctas, s)
                     : dispatch_decode<2>(p, qf32, kv->fmt, pl.ctas, s);
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return fail(NF_ERR_CUDA, "decode kernel set-up: %s", cudaGetErrorString(e));
    }
    return after_launch("decode kernel launch");
}

nf_status nf_decode_attn_noalloc(const nf_kv_layer *kv, const void *q, int32_t q_dtype, int32_t batch,
                                 int32_t n_q, int32_t num_q_heads, const int32_t *block_table,
                                 int32_t max_blocks, const int32_t *seqlens, int32_t max_seqlen,
                                 float softmax_scale, int32_t causal, float *out, float *out_lse,
                                 nf_stream_t stream) {
    size_t tickets = 0;
    if (kv && kv->num_kv_heads > 0) {
        const int sms = current_sm_count();
        Plan pl;
        if (sms > 0 && make_plan(batch, n_q, num_q_heads, kv->num_kv_heads, max_seqlen, sms, pl)) {
            if (pl.bytes() > NF_NOALLOC_SCRATCH_BYTES)
                return fail(NF_ERR_WORKSPACE, "shape needs %zu bytes of scratch, above the %zu-byte no-alloc maximum",
                            pl.bytes(), (size_t)NF_NOALLOC_SCRATCH_BYTES);
            tickets = pl.ticket_bytes;
        }
    }
    void *scratch = nullptr;
    const nf_status st = noalloc_scratch(&scratch);
    if (st != NF_OK) return st;
    // the ticket counters must start at zero; the array keeps the last call's bytes
    if (tickets) {
        const cudaError_t e = cudaMemsetAsync(scratch, 0, tickets, reinterpret_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) return fail(NF_ERR_CUDA, "clearing the no-alloc tickets: %s", cudaGetErrorString(e));
    }
    return nf_decode_attn(kv, q, q_dtype, batch, n_q, num_q_heads, block_table, max_blocks, seqlens,
                          max_seqlen, softmax_scale, causal, out, out_lse, scratch,
                          NF_NOALLOC_SCRATCH_BYTES, stream);
}

nf_status nf_attn_combine(const float *part_o, const float *part_lse, int32_t n_splits,
                          int32_t rows, int32_t head_dim, float *out, float *out_lse,
                          nf_stream_t stream) {
    if (n_splits < 1 || rows < 0) return fail(NF_ERR_INVALID_ARG, "n_splits %d / rows %d", n_splits, rows);
    if (head_dim < 4 || head_dim > 1024 || head_dim % 4 != 0)
        return fail(NF_ERR_UNSUPPORTED, "head_dim %d (multiple of 4 in [4, 1024])", head_dim);
    if (rows == 0) {
        g_msg[0] = '\0';
        return NF_OK;
    }
    if (!part_o || !part_lse || !out) return fail(NF_ERR_INVALID_ARG, "a device pointer is NULL");
    if ((reinterpret_cast<uintptr_t>(part_o) | reinterpret_cast<uintptr_t>(out)) & 15)
        return fail(NF_ERR_INVALID_ARG, "part_o / out must be 16-byte aligned");
    return launch_combine(part_o, part_lse, n_splits, rows, head_dim, (size_t)rows * head_dim, (size_t)rows, out,
                          out_lse, reinterpret_cast<cudaStream_t>(stream));
}

size_t nf_attn_packed_slot_floats(int32_t rows, int32_t head_dim) {
    if (rows < 1 || head_dim < 1) return 0;
    return ((size_t)rows * (size_t)(head_dim + 1) + 3) / 4 * 4;
}

nf_status nf_attn_combine_packed(const float *parts, int32_t n_splits, int32_t rows, int32_t head_dim, float *out,
                                 float *out_lse, nf_stream_t stream) {
    if (n_splits < 1 || rows < 0) return fail(NF_ERR_INVALID_ARG, "n_splits %d / rows %d", n_splits, rows);
    if (head_dim < 4 || head_dim > 1024 || head_dim % 4 != 0)
        return fail(NF_ERR_UNSUPPORTED, "head_dim %d (multiple of 4 in [4, 1024])", head_dim);
    if (rows == 0) {
        g_msg[0] = '\0';
        return NF_OK;
    }
    if (!parts || !out) return fail(NF_ERR_INVALID_ARG, "a device pointer is NULL");
    if ((reinterpret_cast<uintptr_t>(parts) | reinterpret_cast<uintptr_t>(out)) & 15)
        return fail(NF_ERR_INVALID_ARG, "parts / out must be 16-byte aligned");
    const size_t slot = nf_attn_packed_slot_floats(rows, head_dim);
    return launch_combine(parts, parts + (size_t)rows * head_dim, n_splits, rows, head_dim, slot, slot, out, out_lse,
                          reinterpret_cast<cudaStream_t>(stream));
}

nf_status nf_get_device_error(int32_t *code) {
    if (!code) return fail(NF_ERR_INVALID_ARG, "code is NULL");
    int32_t v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, nf::g_device_error, sizeof(v));
    if (e == cudaSuccess) {
        const int32_t zero = 0;
        e = cudaMemcpyToSymbol(nf::g_device_error, &zero, sizeof(zero));
    }
    if (e != cudaSuccess) return fail(NF_ERR_CUDA, "reading the device error word: %s", cudaGetErrorString(e));
    *code = v;
    return v ? NF_ERR_DEVICE_CHECK : NF_OK;
}

nf_status nf_selftest_bounded_wait(uint32_t limit_us, nf_stream_t stream) {
    if (limit_us == 0 || limit_us > 1000000u)
        return fail(NF_ERR_INVALID_ARG, "limit_us %u (1 .. 1000000)", limit_us);
    nf::bounded_wait_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        (uint64_t)limit_us * 1000u);
    return after_launch("bounded-wait self-test launch");
}

const char *nf_status_string(nf_status status) {
    switch (status) {
        case NF_OK: return "ok";
        case NF_ERR_INVALID_ARG: return "invalid argument";
        case NF_ERR_UNSUPPORTED: return "unsupported shape or dtype";
        case NF_ERR_WORKSPACE: return "workspace too small";
        case NF_ERR_CUDA: return "CUDA error";
        case NF_ERR_DEVICE_CHECK: return "device-side check failed";
        default: return "unknown status";
    }
}

const char *nf_last_error(void) { return g_msg; }

}  // extern "C"

// ---------------------------------------------------------------- prefill
extern "C" nf_status nf_prefill_attn(const nf_kv_layer *kv, const void *q, int32_t q_dtype, int32_t batch,
                                     int32_t n_q, int32_t num_q_heads, const int32_t *block_table,
                                     int32_t max_blocks, const int32_t *seqlens, int32_t max_seqlen,
                                     float softmax_scale, int32_t causal, float *out, float *out_lse,
                                     nf_stream_t stream) {
    nf_status st = check_layer(kv);
    if (st != NF_OK) return st;
    if (kv->fmt != NF_KV_K8V4) return fail(NF_ERR_UNSUPPORTED, "prefill: kv->fmt %d (only NF_KV_K8V4)", kv->fmt);
    if (q_dtype != NF_BF16) return fail(NF_ERR_UNSUPPORTED, "prefill: q_dtype %d (only NF_BF16)", q_dtype);
    if (batch < 1 || n_q < 1 || num_q_heads < 1)
        return fail(NF_ERR_INVALID_ARG, "batch %d, n_q %d, num_q_heads %d must be >= 1", batch, n_q,
                    num_q_heads);
    if (batch > 65535 || kv->num_kv_heads > 65535)
        return fail(NF_ERR_UNSUPPORTED, "batch %d / num_kv_heads %d above 65535", batch, kv->num_kv_heads);
    if (num_q_heads % kv->num_kv_heads != 0)
        return fail(NF_ERR_INVALID_ARG, "num_q_heads %d not a multiple of num_kv_heads %d",
                    num_q_heads, kv->num_kv_heads);
    if (max_seqlen < n_q) return fail(NF_ERR_INVALID_ARG, "max_seqlen %d < n_q %d", max_seqlen, n_q);
    if ((long long)max_blocks * nf::kBlock < max_seqlen)
        return fail(NF_ERR_INVALID_ARG, "max_blocks %d cannot hold max_seqlen %d", max_blocks, max_seqlen);
    if (!q || !block_table || !seqlens || !out) return fail(NF_ERR_INVALID_ARG, "a device pointer is NULL");
    if (!std::isfinite(softmax_scale)) return fail(NF_ERR_INVALID_ARG, "softmax_scale is not finite");
    if ((reinterpret_cast<uintptr_t>(q) & 15) || (reinterpret_cast<uintptr_t>(out) & 15))
        return fail(NF_ERR_INVALID_ARG, "q / out must be 16-byte aligned");
    const long long rows = (long long)(num_q_heads / kv->num_kv_heads) * n_q;
    const long long row_tiles = (rows + nf::kTcRows - 1) / nf::kTcRows;
    if (rows > 0x7fffffffLL || row_tiles > 0x7fffffffLL)
        return fail(NF_ERR_UNSUPPORTED, "prefill: %lld query rows per kv-head", rows);

    nf::PrefillParams p{};
    p.k_codes = static_cast<const int8_t *>(kv->k_codes);
    p.k_scales = static_cast<const __half *>(kv->k_scales);
    p.v_codes = static_cast<const uint8_t *>(kv->v_codes);
    p.v_scales = static_cast<const __half *>(kv->v_scales);
    p.num_blocks = kv->num_blocks;
    p.num_kv_heads = kv->num_kv_heads;
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.batch = batch;
    p.n_q = n_q;
    p.num_q_heads = num_q_heads;
    p.group = num_q_heads / kv->num_kv_heads;
    p.rows = (int)rows;
    p.row_tiles = (int)row_tiles;
    p.block_table = block_table;
    p.max_blocks = max_blocks;
    p.seqlens = seqlens;
    p.max_seqlen = max_seqlen;
    p.scale_log2 = softmax_scale * 1.4426950408889634f;
    p.causal = causal != 0;
    p.out = out;
    p.out_lse = out_lse;

    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(nf::prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        nf::TcSmem::kBytes);
    });
    if (attr_err != cudaSuccess)
        return fail(NF_ERR_CUDA, "prefill kernel attribute: %s", cudaGetErrorString(attr_err));
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)row_tiles, (unsigned)kv->num_kv_heads, (unsigned)batch);
    cfg.blockDim = dim3(nf::kTcThreads);
    cfg.dynamicSmemBytes = nf::TcSmem::kBytes;
    cfg.stream = reinterpret_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, nf::prefill_tc_kernel, p);
    if (e != cudaSuccess) {
        (void)cudaGetLastError();  // a refused launch leaves no sticky state for the next call
        return fail(NF_ERR_CUDA, "prefill kernel launch: %s", cudaGetErrorString(e));
    }
    return after_launch("prefill kernel launch");
}
