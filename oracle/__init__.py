"""CPU oracle for K8/V4 (and int8 / fp8 / bf16) KV-cache decode attention (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The product
path (``long_context_quantized_b200``) never imports it, and this package
imports nothing from the product path: the two share no code.

The arithmetic lives in ``nfref.c`` (plain C: fp32 quantiser, fp64 attention,
plain loops).  This module only compiles it with gcc and marshals numpy arrays
through ctypes.  Every function cites the passage it follows in ``nfref.c``.

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py``
against closed forms, invariants, numpy's independent IEEE conversions and
brute force on tiny inputs.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nfref.c")
_LIB_PATH = os.path.join(_HERE, "libnfref.so")
_lock = threading.Lock()
_lib = None

FMT_K8V4 = 0
FMT_BF16 = 1
FMT_K8V8 = 2
FMT_F8 = 3
FMT_K4V4 = 4   # the "RK4V4-E8" reading: 4-bit K and V, power-of-two scale per 32 channels
BLOCK = 256

CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
          "-fexcess-precision=standard", "-fopenmp", "-shared", "-fPIC"]


def build(force: bool = False) -> str:
    """Compile nfref.c into oracle/libnfref.so with gcc (no FMA contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            P = ctypes.c_void_p
            I = ctypes.c_int
            lib.nfref_f32_to_f16.argtypes = [ctypes.c_float]
            lib.nfref_f32_to_f16.restype = ctypes.c_uint16
            lib.nfref_f16_to_f32.argtypes = [ctypes.c_uint16]
            lib.nfref_f16_to_f32.restype = ctypes.c_float
            lib.nfref_f32_to_bf16.argtypes = [ctypes.c_float]
            lib.nfref_f32_to_bf16.restype = ctypes.c_uint16
            lib.nfref_bf16_to_f32.argtypes = [ctypes.c_uint16]
            lib.nfref_bf16_to_f32.restype = ctypes.c_float
            for fn in ("nfref_f32_to_f16_n", "nfref_f16_to_f32_n",
                       "nfref_f32_to_bf16_n", "nfref_bf16_to_f32_n"):
                getattr(lib, fn).argtypes = [P, P, ctypes.c_int64]
                getattr(lib, fn).restype = None
            lib.nfref_e4m3_encode_n.argtypes = [P, P, ctypes.c_int64]
            lib.nfref_e4m3_encode_n.restype = None
            lib.nfref_e4m3_decode_n.argtypes = [P, P, ctypes.c_int64]
            lib.nfref_e4m3_decode_n.restype = None
            lib.nfref_quant_k.argtypes = [P, I, P, P]
            lib.nfref_quant_k.restype = None
            lib.nfref_quant_f8.argtypes = [P, I, P, P]
            lib.nfref_quant_f8.restype = None
            lib.nfref_quant_v.argtypes = [P, I, I, P, P]
            lib.nfref_quant_v.restype = None
            lib.nfref_quant_e8.argtypes = [P, I, P, P]
            lib.nfref_quant_e8.restype = None
            lib.nfref_e8_exponent.argtypes = [ctypes.c_float]
            lib.nfref_e8_exponent.restype = I
            lib.nfref_append.argtypes = [I, I, I, I, P, P, P, P, P, P, I, I, P, I, P]
            lib.nfref_append.restype = I
            lib.nfref_attn_row.argtypes = [I, I, I, P, P, P, P, P, I, I, P, I, ctypes.c_double, P, P]
            lib.nfref_attn_row.restype = None
            lib.nfref_decode_attn.argtypes = [I, I, I, P, P, P, P, P, I, I, I, P, I, P,
                                              ctypes.c_float, I, P, ctypes.c_int64, P, P, I]
            lib.nfref_decode_attn.restype = I
            lib.nfref_combine.argtypes = [P, P, I, I, I, P, P]
            lib.nfref_combine.restype = None
            _lib = lib
    return _lib


def _ptr(a):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else ctypes.c_void_p(0)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------- conversions
def _convert(fn, x, in_dtype, out_dtype):
    lib = _load()
    x = np.ascontiguousarray(np.asarray(x, dtype=in_dtype).ravel())
    out = np.zeros(x.shape, out_dtype)
    getattr(lib, fn)(_ptr(x), _ptr(out), ctypes.c_int64(x.size))
    return out


def f32_to_f16_bits(x) -> np.ndarray:
    """fp32 -> fp16 bits, round half to even, saturating at +-65504."""
    return _convert("nfref_f32_to_f16_n", x, np.float32, np.uint16)


def f16_bits_to_f32(h) -> np.ndarray:
    return _convert("nfref_f16_to_f32_n", h, np.uint16, np.float32)


def f32_to_bf16_bits(x) -> np.ndarray:
    """fp32 -> bf16 bits, round half to even."""
    return _convert("nfref_f32_to_bf16_n", x, np.float32, np.uint16)


def bf16_bits_to_f32(h) -> np.ndarray:
    return _convert("nfref_bf16_to_f32_n", h, np.uint16, np.float32)


def f32_to_e4m3_bits(x) -> np.ndarray:
    """fp32 -> fp8 e4m3 bits, round half to even, saturating at +-448."""
    return _convert("nfref_e4m3_encode_n", x, np.float32, np.uint8)


def e4m3_bits_to_f64(b) -> np.ndarray:
    return _convert("nfref_e4m3_decode_n", b, np.uint8, np.float64)


# --------------------------------------------------------------- quantisation
def quant_k(x):
    """One key vector (fp32, d values) -> (fp16 scale bits, int8 codes[d])."""
    lib = _load()
    x = _c(x, np.float32)
    codes = np.zeros(x.shape[-1], np.int8)
    scale = np.zeros(1, np.uint16)
    lib.nfref_quant_k(_ptr(x), x.shape[-1], _ptr(scale), _ptr(codes))
    return scale[0], codes


def quant_v(x, group: int = 32):
    """One value vector (fp32, d values) -> (fp16 scale bits[d/group], packed uint8[d/2])."""
    lib = _load()
    x = _c(x, np.float32)
    d = x.shape[-1]
    scales = np.zeros(d // group, np.uint16)
    packed = np.zeros(d // 2, np.uint8)
    lib.nfref_quant_v(_ptr(x), d, group, _ptr(scales), _ptr(packed))
    return scales, packed


def quant_e8(x):
    """One key or value vector of the RK4V4-E8 cache (fp32, d values) ->
    (exponent bytes uint8[d/32], packed nibbles uint8[d/2])."""
    lib = _load()
    x = _c(x, np.float32)
    d = x.shape[-1]
    scales = np.zeros(d // 32, np.uint8)
    packed = np.zeros(d // 2, np.uint8)
    lib.nfref_quant_e8(_ptr(x), d, _ptr(scales), _ptr(packed))
    return scales, packed


def e8_exponent(s) -> int:
    """The scale exponent of a group whose fp32 absmax / 7 is s."""
    return int(_load().nfref_e8_exponent(float(np.float32(s))))


def quant_f8(x):
    """One key or value vector of the fp8 cache (fp32, d values) -> (fp16 scale
    bits, e4m3 codes uint8[d])."""
    lib = _load()
    x = _c(x, np.float32)
    codes = np.zeros(x.shape[-1], np.uint8)
    scale = np.zeros(1, np.uint16)
    lib.nfref_quant_f8(_ptr(x), x.shape[-1], _ptr(scale), _ptr(codes))
    return scale[0], codes


# ----------------------------------------------------------------------- pool
class Pool:
    """One layer's host-side pool (planes laid out as in nfref.c)."""

    def __init__(self, fmt: int, num_blocks: int, num_kv_heads: int, head_dim: int = 128,
                 poison: int | None = 0xA5):
        self.fmt, self.num_blocks, self.H, self.d = fmt, num_blocks, num_kv_heads, head_dim
        if fmt == FMT_K8V4:
            self.k = np.zeros((num_blocks, num_kv_heads, BLOCK, head_dim), np.int8)
            self.k_scale = np.zeros((num_blocks, num_kv_heads, BLOCK), np.uint16)
            self.v = np.zeros((num_blocks, num_kv_heads, BLOCK, head_dim // 2), np.uint8)
            self.v_scale = np.zeros((num_blocks, num_kv_heads, BLOCK, head_dim // 32), np.uint16)
        elif fmt == FMT_K4V4:
            self.k = np.zeros((num_blocks, num_kv_heads, BLOCK, head_dim // 2), np.uint8)
            self.k_scale = np.zeros((num_blocks, num_kv_heads, BLOCK, head_dim // 32), np.uint8)
            self.v = np.zeros((num_blocks, num_kv_heads, BLOCK, head_dim // 2), np.uint8)
            self.v_scale = np.zeros((num_blocks, num_kv_heads, BLOCK, head_dim // 32), np.uint8)
        elif fmt in (FMT_K8V8, FMT_F8):
            code = np.int8 if fmt == FMT_K8V8 else np.uint8
            self.k = np.zeros((num_blocks, num_kv_heads, BLOCK, head_dim), code)
            self.k_scale = np.zeros((num_blocks, num_kv_heads, BLOCK), np.uint16)
            self.v = np.zeros((num_blocks, num_kv_heads, BLOCK, head_dim), code)
            self.v_scale = np.zeros((num_blocks, num_kv_heads, BLOCK), np.uint16)
        else:
            self.k = np.zeros((num_blocks, num_kv_heads, BLOCK, head_dim), np.uint16)
            self.v = np.zeros((num_blocks, num_kv_heads, BLOCK, head_dim), np.uint16)
            self.k_scale = np.zeros(1, np.uint16)
            self.v_scale = np.zeros(1, np.uint16)
        if poison is not None:
            for a in (self.k, self.k_scale, self.v, self.v_scale):
                a.view(np.uint8)[...] = poison

    def planes(self):
        return self.k, self.k_scale, self.v, self.v_scale


def append(pool: Pool, k_new, v_new, block_table, seqlens_before) -> int:
    """Quantise k_new/v_new (fp32 values [B][n_new][H][d]) into the pool."""
    lib = _load()
    k_new = _c(k_new, np.float32)
    v_new = _c(v_new, np.float32)
    bt = _c(block_table, np.int32)
    sb = _c(seqlens_before, np.int32)
    B, n_new, H, d = k_new.shape
    assert H == pool.H and d == pool.d
    return lib.nfref_append(pool.fmt, pool.num_blocks, pool.H, pool.d,
                            _ptr(pool.k), _ptr(pool.k_scale), _ptr(pool.v), _ptr(pool.v_scale),
                            _ptr(k_new), _ptr(v_new), B, n_new, _ptr(bt), bt.shape[1], _ptr(sb))


def attn_row(pool: Pool, bt_row, k_begin: int, k_end: int, q, kvh: int, scale: float):
    """One query row over keys [k_begin, k_end): returns (o[d] fp64, lse fp64)."""
    lib = _load()
    bt_row = _c(bt_row, np.int32)
    q = _c(q, np.float64)
    o = np.zeros(pool.d, np.float64)
    lse = np.zeros(1, np.float64)
    lib.nfref_attn_row(pool.fmt, pool.H, pool.d, _ptr(pool.k), _ptr(pool.k_scale),
                       _ptr(pool.v), _ptr(pool.v_scale), _ptr(bt_row), k_begin, k_end,
                       _ptr(q), kvh, float(scale), _ptr(o), _ptr(lse))
    return o, lse[0]


def decode_attn(pool: Pool, q, block_table, seqlens, softmax_scale: float, causal: bool,
                rows=None, nthreads: int = 1):
    """Decode attention.  q: [B][n_q][H_q][d] (any float dtype, used exactly as
    fp64).  Returns (out [n_rows][d] fp64, lse [n_rows] fp64) for all rows
    (row id = (b * n_q + j) * H_q + h) or the listed ones."""
    lib = _load()
    q = _c(q, np.float64)
    B, n_q, H_q, d = q.shape
    bt = _c(block_table, np.int32)
    sl = _c(seqlens, np.int32)
    rows_a = None if rows is None else _c(rows, np.int64)
    n_rows = B * n_q * H_q if rows is None else len(rows_a)
    out = np.zeros((n_rows, d), np.float64)
    lse = np.zeros(n_rows, np.float64)
    st = lib.nfref_decode_attn(pool.fmt, pool.H, d, _ptr(pool.k), _ptr(pool.k_scale),
                               _ptr(pool.v), _ptr(pool.v_scale), _ptr(q), B, n_q, H_q,
                               _ptr(bt), bt.shape[1], _ptr(sl), np.float32(softmax_scale),
                               int(bool(causal)), _ptr(rows_a), n_rows, _ptr(out), _ptr(lse),
                               int(nthreads))
    if st != 0:
        raise ValueError("oracle decode_attn: a sequence is shorter than n_q")
    return out, lse


def combine(part_o, part_lse):
    """part_o [S][rows][d], part_lse [S][rows] -> (out [rows][d], lse [rows])."""
    lib = _load()
    po = _c(part_o, np.float64)
    pl = _c(part_lse, np.float64)
    S, rows, d = po.shape
    out = np.zeros((rows, d), np.float64)
    lse = np.zeros(rows, np.float64)
    lib.nfref_combine(_ptr(po), _ptr(pl), S, rows, d, _ptr(out), _ptr(lse))
    return out, lse
