"""B200 (sm_100a) decode attention over a K8/V4-quantised, segmented KV cache.

Thin Python binding of ``libnf.so`` (the C ABI declared in ``include/nf.h``).
Every function here only marshals torch tensors into pointers and sizes and
calls the C entry point of the same name; all computation happens in the CUDA
kernels of ``csrc/``.  torch provides device memory and the current stream.
There is no CPU fallback: if ``libnf.so`` is missing, loading fails loudly.
"""
from __future__ import annotations

import ctypes
import os
import re
import threading

import torch

__all__ = [
    "NF_OK", "NF_KV_K8V4", "NF_KV_BF16", "NF_KV_K8V8", "NF_KV_F8", "NF_KV_K4V4", "NF_F32", "NF_BF16", "NfError", "KVLayer",
    "nf_kv_append_quant", "nf_decode_attn_workspace_size", "nf_decode_attn", "nf_decode_attn_noalloc",
    "nf_attn_combine", "nf_attn_packed_slot_floats", "nf_attn_combine_packed", "nf_prefill_attn",
    "nf_get_device_error", "nf_status_string", "library_path", "load_library",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
_ROOT = os.path.dirname(_PKG)
HEADER = os.path.join(_ROOT, "include", "nf.h")
_LIB_PATH = os.path.join(_PKG, "libnf.so")

NF_OK = 0
NF_ERR_INVALID_ARG, NF_ERR_UNSUPPORTED, NF_ERR_WORKSPACE, NF_ERR_CUDA, NF_ERR_DEVICE_CHECK = 1, 2, 3, 4, 5
NF_DEVERR_NONE, NF_DEVERR_BLOCK_ID, NF_DEVERR_TABLE, NF_DEVERR_SEQLEN = 0, 1, 2, 3
NF_DEVERR_TIMEOUT, NF_DEVERR_INTERNAL, NF_DEVERR_RANGE = 4, 5, 6
NF_F32, NF_BF16, NF_F16 = 0, 1, 2
NF_KV_K8V4, NF_KV_BF16, NF_KV_K8V8, NF_KV_F8, NF_KV_K4V4 = 0, 1, 2, 3, 4
BLOCK = 256
HEAD_DIM = 128


class NfError(RuntimeError):
    def __init__(self, status: int, where: str, message: str):
        super().__init__(f"{where}: {message} (status {status})")
        self.status = status


class nf_kv_layer(ctypes.Structure):
    _fields_ = [
        ("fmt", ctypes.c_int32), ("num_blocks", ctypes.c_int32), ("block_size", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("v_group", ctypes.c_int32),
        ("k_codes", ctypes.c_void_p), ("k_scales", ctypes.c_void_p),
        ("v_codes", ctypes.c_void_p), ("v_scales", ctypes.c_void_p),
    ]


_lock = threading.Lock()
_lib = None


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load libnf.so (built by ``python -m long_context_quantized_b200.build``)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_PATH):
            raise ImportError(f"{_LIB_PATH} is missing: build it with "
                              "`python -m long_context_quantized_b200.build`")
        lib = ctypes.CDLL(_LIB_PATH)
        P, I, S = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
        lib.nf_kv_append_quant.argtypes = [P, P, P, I, I, I, P, I, P, P]
        lib.nf_kv_append_quant.restype = I
        lib.nf_decode_attn_workspace_size.argtypes = [I, I, I, I, I, I]
        lib.nf_decode_attn_workspace_size.restype = S
        lib.nf_decode_attn.argtypes = [P, P, I, I, I, I, P, I, P, I, ctypes.c_float, I, P, P, P, S, P]
        lib.nf_decode_attn.restype = I
        lib.nf_decode_attn_ex.argtypes = [P, P, I, I, I, I, P, I, P, I, ctypes.c_float, I, ctypes.c_uint32, P, P,
                                          P, S, P]
        lib.nf_decode_attn_ex.restype = I
        lib.nf_decode_attn_noalloc.argtypes = [P, P, I, I, I, I, P, I, P, I, ctypes.c_float, I, P, P, P]
        lib.nf_decode_attn_noalloc.restype = I
        lib.nf_prefill_attn.argtypes = [P, P, I, I, I, I, P, I, P, I, ctypes.c_float, I, P, P, P]
        lib.nf_prefill_attn.restype = I
        lib.nf_selftest_bounded_wait.argtypes = [ctypes.c_uint32, P]
        lib.nf_selftest_bounded_wait.restype = I
        lib.nf_attn_combine.argtypes = [P, P, I, I, I, P, P, P]
        lib.nf_attn_combine.restype = I
        lib.nf_attn_packed_slot_floats.argtypes = [I, I]
        lib.nf_attn_packed_slot_floats.restype = S
        lib.nf_attn_combine_packed.argtypes = [P, I, I, I, P, P, P]
        lib.nf_attn_combine_packed.restype = I
        lib.nf_get_device_error.argtypes = [ctypes.POINTER(ctypes.c_int32)]
        lib.nf_get_device_error.restype = I
        lib.nf_status_string.argtypes = [I]
        lib.nf_status_string.restype = ctypes.c_char_p
        lib.nf_last_error.argtypes = []
        lib.nf_last_error.restype = ctypes.c_char_p
        _lib = lib
        return lib


def declared_symbols(header: str = HEADER) -> list:
    """Names of the functions include/nf.h declares."""
    text = open(header).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(nf_[a-z_0-9]+)\s*\(", text)))


def _check(st: int, where: str):
    if st != NF_OK:
        lib = load_library()
        raise NfError(st, where, lib.nf_last_error().decode() or lib.nf_status_string(st).decode())


def _dptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.float32:
        return NF_F32
    if dt == torch.bfloat16:
        return NF_BF16
    raise NfError(NF_ERR_UNSUPPORTED, "dtype", f"{dt} (float32 or bfloat16)")


def _need(t, name, dtype=None, device=True):
    if t is None:
        return
    if not t.is_contiguous():
        raise NfError(NF_ERR_INVALID_ARG, name, "tensor must be contiguous")
    if device and not t.is_cuda:
        raise NfError(NF_ERR_INVALID_ARG, name, "tensor must be on a CUDA device")
    if dtype is not None and t.dtype != dtype:
        raise NfError(NF_ERR_INVALID_ARG, name, f"dtype {t.dtype}, expected {dtype}")


class KVLayer:
    """One layer's KV pool planes (device tensors owned by torch) and the
    ``nf_kv_layer`` view the C ABI takes.  Layout: see ``include/nf.h``."""

    def __init__(self, fmt: int, k_codes, k_scales, v_codes, v_scales):
        self.fmt = fmt
        self.k_codes, self.k_scales, self.v_codes, self.v_scales = k_codes, k_scales, v_codes, v_scales
        self.num_blocks, self.num_kv_heads = k_codes.shape[0], k_codes.shape[1]
        self.c = nf_kv_layer(fmt, self.num_blocks, BLOCK, self.num_kv_heads, HEAD_DIM, 32,
                             k_codes.data_ptr(), 0 if k_scales is None else k_scales.data_ptr(),
                             v_codes.data_ptr(), 0 if v_scales is None else v_scales.data_ptr())

    @classmethod
    def empty(cls, fmt: int, num_blocks: int, num_kv_heads: int, device="cuda", fill: int | None = None):
        kw = dict(device=device)
        if fmt == NF_KV_K8V4:
            k = torch.empty((num_blocks, num_kv_heads, BLOCK, HEAD_DIM), dtype=torch.int8, **kw)
            ks = torch.empty((num_blocks, num_kv_heads, BLOCK), dtype=torch.float16, **kw)
            v = torch.empty((num_blocks, num_kv_heads, BLOCK, HEAD_DIM // 2), dtype=torch.uint8, **kw)
            vs = torch.empty((num_blocks, num_kv_heads, BLOCK, HEAD_DIM // 32), dtype=torch.float16, **kw)
        elif fmt == NF_KV_K4V4:
            k = torch.empty((num_blocks, num_kv_heads, BLOCK, HEAD_DIM // 2), dtype=torch.uint8, **kw)
            ks = torch.empty((num_blocks, num_kv_heads, BLOCK, HEAD_DIM // 32), dtype=torch.uint8, **kw)
            v = torch.empty((num_blocks, num_kv_heads, BLOCK, HEAD_DIM // 2), dtype=torch.uint8, **kw)
            vs = torch.empty((num_blocks, num_kv_heads, BLOCK, HEAD_DIM // 32), dtype=torch.uint8, **kw)
        elif fmt in (NF_KV_K8V8, NF_KV_F8):
            code = torch.int8 if fmt == NF_KV_K8V8 else torch.uint8  # fp8: e4m3 bytes
            k = torch.empty((num_blocks, num_kv_heads, BLOCK, HEAD_DIM), dtype=code, **kw)
            ks = torch.empty((num_blocks, num_kv_heads, BLOCK), dtype=torch.float16, **kw)
            v = torch.empty((num_blocks, num_kv_heads, BLOCK, HEAD_DIM), dtype=code, **kw)
            vs = torch.empty((num_blocks, num_kv_heads, BLOCK), dtype=torch.float16, **kw)
        elif fmt == NF_KV_BF16:
            k = torch.empty((num_blocks, num_kv_heads, BLOCK, HEAD_DIM), dtype=torch.bfloat16, **kw)
            v = torch.empty((num_blocks, num_kv_heads, BLOCK, HEAD_DIM), dtype=torch.bfloat16, **kw)
            ks = vs = None
        else:
            raise NfError(NF_ERR_UNSUPPORTED, "KVLayer.empty", f"fmt {fmt}")
        if fill is not None:
            for t in (k, ks, v, vs):
                if t is not None:
                    t.view(torch.uint8).fill_(fill)
        return cls(fmt, k, ks, v, vs)

    def planes(self):
        return [t for t in (self.k_codes, self.k_scales, self.v_codes, self.v_scales) if t is not None]

    def bytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in self.planes())


def nf_kv_append_quant(kv: KVLayer, k_new, v_new, block_table, seqlens_before, stream=None):
    """Quantise k_new / v_new [batch][n_new][H_kv][128] (fp32 or bf16) into the
    pool at positions seqlens_before[b] + i (see nf.h)."""
    _need(k_new, "k_new")
    _need(v_new, "v_new", k_new.dtype)
    _need(block_table, "block_table", torch.int32)
    _need(seqlens_before, "seqlens_before", torch.int32)
    B, n_new = k_new.shape[0], k_new.shape[1]
    st = load_library().nf_kv_append_quant(
        ctypes.byref(kv.c), _dptr(k_new), _dptr(v_new), _dtype_code(k_new.dtype), B, n_new,
        _dptr(block_table), block_table.shape[1], _dptr(seqlens_before), _stream(stream))
    _check(st, "nf_kv_append_quant")


def nf_decode_attn_workspace_size(batch, n_q, num_q_heads, num_kv_heads, max_seqlen, num_sms=None):
    if num_sms is None:
        num_sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    return int(load_library().nf_decode_attn_workspace_size(batch, n_q, num_q_heads, num_kv_heads,
                                                            max_seqlen, num_sms))


NF_DECODE_EARLY_KV = 1


def nf_decode_attn(kv: KVLayer, q, block_table, seqlens, max_seqlen: int, softmax_scale: float,
                   causal: bool, out, out_lse=None, workspace=None, stream=None):
    """Decode attention; q [batch][n_q][H_q][128] (fp32 or bf16), out fp32 of
    the same shape, out_lse fp32 [batch][n_q][H_q] or None (see nf.h)."""
    nf_decode_attn_ex(kv, q, block_table, seqlens, max_seqlen, softmax_scale, causal, 0, out, out_lse,
                      workspace, stream, _name="nf_decode_attn")


def nf_decode_attn_ex(kv: KVLayer, q, block_table, seqlens, max_seqlen: int, softmax_scale: float,
                      causal: bool, flags: int, out, out_lse=None, workspace=None, stream=None,
                      _name="nf_decode_attn_ex"):
    """nf_decode_attn with flags (NF_DECODE_EARLY_KV: see nf.h for the caller's
    guarantee)."""
    _need(q, "q")
    _need(block_table, "block_table", torch.int32)
    _need(seqlens, "seqlens", torch.int32)
    _need(out, "out", torch.float32)
    _need(out_lse, "out_lse", torch.float32)
    _need(workspace, "workspace")
    B, n_q, H_q = q.shape[0], q.shape[1], q.shape[2]
    if workspace is None:
        raise NfError(NF_ERR_WORKSPACE, _name, "workspace tensor required "
                      "(size: nf_decode_attn_workspace_size)")
    ws_bytes = workspace.numel() * workspace.element_size()
    st = load_library().nf_decode_attn_ex(
        ctypes.byref(kv.c), _dptr(q), _dtype_code(q.dtype), B, n_q, H_q, _dptr(block_table),
        block_table.shape[1], _dptr(seqlens), int(max_seqlen), float(softmax_scale), int(bool(causal)),
        int(flags), _dptr(out), _dptr(out_lse), _dptr(workspace), ws_bytes, _stream(stream))
    _check(st, _name)


def nf_prefill_attn(kv: KVLayer, q, block_table, seqlens, max_seqlen: int, softmax_scale: float,
                    causal: bool, out, out_lse=None, stream=None):
    """Chunked-prefill attention (see nf.h): the n_q queries of each sequence
    at positions L - n_q .. L - 1 against its K8/V4 cache; q bf16
    [batch][n_q][H_q][128], out fp32 of the same shape."""
    _need(q, "q")
    _need(block_table, "block_table", torch.int32)
    _need(seqlens, "seqlens", torch.int32)
    _need(out, "out", torch.float32)
    _need(out_lse, "out_lse", torch.float32)
    B, n_q, H_q = q.shape[0], q.shape[1], q.shape[2]
    st = load_library().nf_prefill_attn(
        ctypes.byref(kv.c), _dptr(q), _dtype_code(q.dtype), B, n_q, H_q, _dptr(block_table),
        block_table.shape[1], _dptr(seqlens), int(max_seqlen), float(softmax_scale), int(bool(causal)),
        _dptr(out), _dptr(out_lse), _stream(stream))
    _check(st, "nf_prefill_attn")


NF_NOALLOC_SCRATCH_BYTES = 8 << 20


def nf_decode_attn_noalloc(kv: KVLayer, q, block_table, seqlens, max_seqlen: int, softmax_scale: float,
                           causal: bool, out, out_lse=None, stream=None):
    """nf_decode_attn for callers that cannot allocate device memory at call
    time: the scratch is a fixed array inside libnf's device image (see nf.h).
    Calls on one device share it, so do not overlap them on the GPU."""
    _need(q, "q")
    _need(block_table, "block_table", torch.int32)
    _need(seqlens, "seqlens", torch.int32)
    _need(out, "out", torch.float32)
    _need(out_lse, "out_lse", torch.float32)
    B, n_q, H_q = q.shape[0], q.shape[1], q.shape[2]
    st = load_library().nf_decode_attn_noalloc(
        ctypes.byref(kv.c), _dptr(q), _dtype_code(q.dtype), B, n_q, H_q, _dptr(block_table),
        block_table.shape[1], _dptr(seqlens), int(max_seqlen), float(softmax_scale), int(bool(causal)),
        _dptr(out), _dptr(out_lse), _stream(stream))
    _check(st, "nf_decode_attn_noalloc")


def nf_attn_combine(part_o, part_lse, out, out_lse=None, stream=None):
    """part_o [S][rows][d], part_lse [S][rows] (fp32) -> out [rows][d], out_lse [rows]."""
    _need(part_o, "part_o", torch.float32)
    _need(part_lse, "part_lse", torch.float32)
    _need(out, "out", torch.float32)
    _need(out_lse, "out_lse", torch.float32)
    S, rows, d = part_o.shape
    st = load_library().nf_attn_combine(_dptr(part_o), _dptr(part_lse), S, rows, d, _dptr(out),
                                        _dptr(out_lse), _stream(stream))
    _check(st, "nf_attn_combine")


def nf_attn_packed_slot_floats(rows: int, head_dim: int = HEAD_DIM) -> int:
    """Floats of one packed split slot: o [rows][head_dim] then lse [rows],
    rounded up to a multiple of 4 (see nf.h)."""
    return int(load_library().nf_attn_packed_slot_floats(int(rows), int(head_dim)))


def nf_attn_combine_packed(parts, rows: int, out, out_lse=None, stream=None):
    """parts fp32 [S][slot] (packed split slots) -> out [rows][d], out_lse [rows]."""
    _need(parts, "parts", torch.float32)
    _need(out, "out", torch.float32)
    _need(out_lse, "out_lse", torch.float32)
    S = parts.shape[0]
    d = out.shape[-1]
    if parts.numel() != S * nf_attn_packed_slot_floats(rows, d):
        raise NfError(NF_ERR_INVALID_ARG, "nf_attn_combine_packed", "parts is not [S][slot]")
    st = load_library().nf_attn_combine_packed(_dptr(parts), S, int(rows), d, _dptr(out), _dptr(out_lse),
                                               _stream(stream))
    _check(st, "nf_attn_combine_packed")


def nf_get_device_error() -> int:
    """Read and clear the device error code (synchronises the device)."""
    code = ctypes.c_int32(0)
    st = load_library().nf_get_device_error(ctypes.byref(code))
    if st not in (NF_OK, NF_ERR_DEVICE_CHECK):
        _check(st, "nf_get_device_error")
    return code.value


def nf_status_string(status: int) -> str:
    return load_library().nf_status_string(int(status)).decode()


def nf_selftest_bounded_wait(limit_us: int, stream=None):
    """Run the bounded-wait self-test (see nf.h); afterwards
    nf_get_device_error() returns NF_DEVERR_TIMEOUT."""
    _check(load_library().nf_selftest_bounded_wait(int(limit_us), _stream(stream)), "nf_selftest_bounded_wait")
