"""bench.py's algorithmic byte and FLOP counts against closed forms (CPU)."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import workloads  # noqa: E402


def test_bytes_per_token_head_by_format():
    # K8/V4: 128 K codes + 1 fp16 K scale + 64 bytes of V nibbles + 4 fp16 V scales
    assert workloads.kv_bytes_per_token_head("k8v4") == 128 + 2 + 64 + 8 == 202
    # int8 and fp8: 128 + 2 bytes for each of K and V
    assert workloads.kv_bytes_per_token_head("k8v8") == workloads.kv_bytes_per_token_head("f8") == 260
    assert workloads.kv_bytes_per_token_head("bf16") == 512
    # RK4V4-E8: 64 bytes of nibbles and 4 exponent bytes for each of K and V
    assert workloads.kv_bytes_per_token_head("k4v4") == 2 * (64 + 4) == 136
    with pytest.raises(ValueError):
        workloads.kv_bytes_per_token_head("int4")


def _flops(w):
    pw = bench.PrefillWorkload.__new__(bench.PrefillWorkload)
    pw.w = w
    return pw.flops_per_launch()


def test_prefill_flops_closed_forms():
    # non-causal: every one of the n_q rows per head sees all L keys
    w = workloads.custom("f", cached=(1000,), n_new=24, n_q=24, num_q_heads=8, num_kv_heads=2, causal=False)
    assert _flops(w) == 4 * 128 * 8 * 24 * 1024
    # causal whole prompt (L = n_q): row j sees j + 1 keys, sum n (n + 1) / 2
    w = workloads.custom("f", cached=(0,), n_new=300, n_q=300, num_q_heads=4, num_kv_heads=1, causal=True)
    assert _flops(w) == 4 * 128 * 4 * (300 * 301 // 2)
    # the benchmark chunk: 1024 queries after 179200 cached keys
    w = workloads.get("prefill_chunk")
    keys = sum(179200 + j + 1 for j in range(1024))
    assert _flops(w) == 4 * 128 * 32 * keys == 3015075430400
