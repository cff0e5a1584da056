"""CPU-side checks of the C ABI: libnf.so loads without a GPU, exports every
function include/nf.h declares, and rejects bad arguments on the host before
any launch.  No compute call is made here."""
import ctypes

import pytest

import long_context_quantized_b200 as nf


@pytest.fixture(scope="module")
def lib():
    from long_context_quantized_b200 import build
    build.build()
    return nf.load_library()


def test_header_declares_the_hot_path_calls():
    names = nf.declared_symbols()
    for required in ("nf_kv_append_quant", "nf_decode_attn", "nf_attn_combine",
                     "nf_decode_attn_workspace_size", "nf_get_device_error", "nf_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in nf.declared_symbols():
        assert hasattr(lib, name), f"libnf.so does not export {name}"


def test_status_strings(lib):
    assert nf.nf_status_string(0) == "ok"
    assert "workspace" in nf.nf_status_string(3)
    assert nf.nf_status_string(99) == "unknown status"


def test_workspace_size_host_only(lib):
    ws = nf.nf_decode_attn_workspace_size(1, 1, 32, 4, 32769, num_sms=148)
    assert ws > 0 and ws % 256 == 0
    assert nf.nf_decode_attn_workspace_size(2, 1, 32, 4, 90112, 148) > 0
    assert nf.nf_decode_attn_workspace_size(1, 4, 32, 4, 180228, 148) > 0
    # invalid shapes give 0
    assert nf.nf_decode_attn_workspace_size(1, 1, 30, 4, 1000, 148) == 0   # H_q % H_kv
    assert nf.nf_decode_attn_workspace_size(1, 0, 32, 4, 1000, 148) == 0   # n_q < 1
    assert nf.nf_decode_attn_workspace_size(1, 4, 32, 4, 3, 148) == 0      # max_seqlen < n_q
    assert nf.nf_decode_attn_workspace_size(0, 1, 32, 4, 1000, 148) == 0   # batch < 1


def _layer(fmt=nf.NF_KV_K8V4, head_dim=128, block=256, group=32, ptr=256):
    return nf.nf_kv_layer(fmt, 4, block, 2, head_dim, group, ptr, ptr, ptr, ptr)


def _decode(lib, kv, **over):
    args = dict(q=256, q_dtype=nf.NF_BF16, batch=1, n_q=1, H_q=4, bt=256, max_blocks=4, seqlens=256,
                max_seqlen=1000, scale=0.088, causal=0, out=256, lse=None, ws=256, ws_bytes=1 << 20)
    args.update(over)
    return lib.nf_decode_attn(None if kv is None else ctypes.byref(kv), args["q"], args["q_dtype"],
                              args["batch"], args["n_q"], args["H_q"], args["bt"], args["max_blocks"],
                              args["seqlens"], args["max_seqlen"], args["scale"], args["causal"],
                              args["out"], args["lse"], args["ws"], args["ws_bytes"], None)


def test_decode_rejects_bad_arguments_before_launch(lib):
    assert _decode(lib, None) == nf.NF_ERR_INVALID_ARG
    assert _decode(lib, _layer(head_dim=64)) == nf.NF_ERR_UNSUPPORTED
    assert _decode(lib, _layer(block=128)) == nf.NF_ERR_UNSUPPORTED
    assert _decode(lib, _layer(group=16)) == nf.NF_ERR_UNSUPPORTED
    assert _decode(lib, _layer(fmt=7)) == nf.NF_ERR_UNSUPPORTED
    assert _decode(lib, _layer(ptr=264)) == nf.NF_ERR_INVALID_ARG        # misaligned plane
    assert _decode(lib, _layer(), q_dtype=nf.NF_F16) == nf.NF_ERR_UNSUPPORTED
    assert _decode(lib, _layer(), H_q=3) == nf.NF_ERR_INVALID_ARG        # not a multiple of H_kv
    assert _decode(lib, _layer(), n_q=0) == nf.NF_ERR_INVALID_ARG
    assert _decode(lib, _layer(), max_seqlen=2000) == nf.NF_ERR_INVALID_ARG  # table too short
    assert _decode(lib, _layer(), q=None) == nf.NF_ERR_INVALID_ARG
    assert _decode(lib, _layer(), scale=float("inf")) == nf.NF_ERR_INVALID_ARG
    assert b"NULL" in lib.nf_last_error() or lib.nf_last_error()


def test_append_and_combine_host_paths(lib):
    kv = _layer()
    # nothing to append: OK without touching the device
    assert lib.nf_kv_append_quant(ctypes.byref(kv), None, None, nf.NF_BF16, 1, 0, None, 1, None, None) == 0
    assert lib.nf_kv_append_quant(ctypes.byref(kv), 256, 256, nf.NF_F16, 1, 1, 256, 1, 256, None) \
        == nf.NF_ERR_UNSUPPORTED
    assert lib.nf_kv_append_quant(ctypes.byref(kv), None, 256, nf.NF_BF16, 1, 1, 256, 1, 256, None) \
        == nf.NF_ERR_INVALID_ARG
    assert lib.nf_kv_append_quant(ctypes.byref(kv), 256, 256, nf.NF_BF16, -1, 1, 256, 1, 256, None) \
        == nf.NF_ERR_INVALID_ARG
    assert lib.nf_attn_combine(256, 256, 2, 0, 128, 256, None, None) == 0  # no rows
    assert lib.nf_attn_combine(256, 256, 0, 4, 128, 256, None, None) == nf.NF_ERR_INVALID_ARG
    assert lib.nf_attn_combine(256, 256, 2, 4, 130, 256, None, None) == nf.NF_ERR_UNSUPPORTED
    assert lib.nf_attn_combine(None, 256, 2, 4, 128, 256, None, None) == nf.NF_ERR_INVALID_ARG


def _prefill(lib, kv, **over):
    args = dict(q=256, q_dtype=nf.NF_BF16, batch=1, n_q=64, H_q=4, bt=256, max_blocks=4, seqlens=256,
                max_seqlen=1000, scale=0.088, causal=1, out=256, lse=None)
    args.update(over)
    return lib.nf_prefill_attn(None if kv is None else ctypes.byref(kv), args["q"], args["q_dtype"],
                               args["batch"], args["n_q"], args["H_q"], args["bt"], args["max_blocks"],
                               args["seqlens"], args["max_seqlen"], args["scale"], args["causal"],
                               args["out"], args["lse"], None)


def test_prefill_rejects_bad_arguments_before_launch(lib):
    assert _prefill(lib, None) == nf.NF_ERR_INVALID_ARG
    assert _prefill(lib, _layer(fmt=nf.NF_KV_K8V8)) == nf.NF_ERR_UNSUPPORTED   # K8/V4 only
    assert _prefill(lib, _layer(fmt=nf.NF_KV_BF16)) == nf.NF_ERR_UNSUPPORTED
    assert _prefill(lib, _layer(), q_dtype=nf.NF_F32) == nf.NF_ERR_UNSUPPORTED  # bf16 queries only
    assert _prefill(lib, _layer(), H_q=3) == nf.NF_ERR_INVALID_ARG
    assert _prefill(lib, _layer(), n_q=0) == nf.NF_ERR_INVALID_ARG
    assert _prefill(lib, _layer(), max_seqlen=32) == nf.NF_ERR_INVALID_ARG     # below n_q
    assert _prefill(lib, _layer(), max_seqlen=2000) == nf.NF_ERR_INVALID_ARG   # table too short
    assert _prefill(lib, _layer(), q=None) == nf.NF_ERR_INVALID_ARG
    assert _prefill(lib, _layer(), q=264) == nf.NF_ERR_INVALID_ARG            # not 16-byte aligned
    assert _prefill(lib, _layer(), scale=float("nan")) == nf.NF_ERR_INVALID_ARG
    assert _prefill(lib, _layer(), batch=70000) == nf.NF_ERR_UNSUPPORTED


def test_int8_fp8_and_k4v4_layers_need_their_scale_planes(lib):
    for fmt in (nf.NF_KV_K8V8, nf.NF_KV_F8, nf.NF_KV_K4V4):
        assert _decode(lib, nf.nf_kv_layer(fmt, 4, 256, 2, 128, 0, 256, 0, 256, 256)) == nf.NF_ERR_INVALID_ARG
        assert _decode(lib, nf.nf_kv_layer(fmt, 4, 256, 2, 128, 0, 256, 256, 256, 0)) == nf.NF_ERR_INVALID_ARG
        assert _decode(lib, nf.nf_kv_layer(fmt, 4, 256, 2, 128, 0, 256, 264, 256, 256)) == nf.NF_ERR_INVALID_ARG
        # v_group is not checked for these formats: the next refusal is the shape's
        assert _decode(lib, nf.nf_kv_layer(fmt, 4, 256, 2, 128, 7, 256, 256, 256, 256), H_q=3) \
            == nf.NF_ERR_INVALID_ARG
    assert _decode(lib, _layer(fmt=5)) == nf.NF_ERR_UNSUPPORTED
    assert _prefill(lib, _layer(fmt=nf.NF_KV_K4V4)) == nf.NF_ERR_UNSUPPORTED  # prefill: K8/V4 only
