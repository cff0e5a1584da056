"""Seeded synthetic inputs for K8/V4 decode attention.

This module holds the workload shapes and the random-input recipes only: no
quantisation, no attention, nothing of the method's arithmetic.  Both the CUDA
path (tests, bench) and the CPU oracle (tests) take their inputs from here, so
the two sides see identical values.

The shapes echo the pages' operating points: single-request decode at 32K-256K
context (page "影片筆記：NInfer + 千问3.8 27b = 1.5倍速@256K上下文", section 一句話總結:
256K on one GPU; page "3090 单卡跑 Qwen3.8-27B：NInfer 上机实测", section 二 测评:
8K-178K inputs, two concurrent requests, 3 MTP draft tokens, a 184320-token
KV pool).  The pages measure on real prompts that are not available here; these
seeded tensors of the same shape stand in for them.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

BLOCK = 256
HEAD_DIM = 128


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int                 # seed offset
    cached: tuple              # tokens already in the cache per sequence
    n_new: int                 # tokens appended inside the timed step (0: none)
    n_q: int                   # query tokens per sequence
    num_q_heads: int
    num_kv_heads: int
    layers: int
    q_dtype: torch.dtype
    kv_in_dtype: torch.dtype   # dtype of the K/V fed to the quantiser
    pool_blocks: int
    causal: bool
    dist: str                  # input recipe, see layer_kv()
    table: str                 # "contiguous" | "shuffled" | "shared_perm"
    head_dim: int = HEAD_DIM

    @property
    def batch(self) -> int:
        return len(self.cached)

    @property
    def seqlens(self) -> tuple:
        """Keys per sequence after the step's append."""
        return tuple(c + self.n_new for c in self.cached)

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def max_blocks(self) -> int:
        return max(math.ceil(L / BLOCK) for L in self.seqlens)

    @property
    def softmax_scale(self) -> float:
        return float(np.float32(1.0 / math.sqrt(self.head_dim)))

    def kv_tokens_per_step(self) -> int:
        """Keys read per 16-layer step: each cached key once per layer."""
        return sum(self.seqlens) * self.layers


WORKLOADS = {
    # 1 sequence, 4096 keys, 16/2 heads, 1 layer, fp32 inputs, contiguous cache.
    "tiny": Workload("tiny", 1, (4096,), 0, 1, 16, 2, 1, torch.float32, torch.float32,
                     16, False, "normal", "contiguous"),
    # 32768 cached + 1 appended, 32/4 heads, 16 layers, 4 outlier K channels x8.
    "ctx32k_append": Workload("ctx32k_append", 2, (32768,), 1, 1, 32, 4, 16, torch.bfloat16,
                              torch.bfloat16, 129, False, "k_outlier_channels", "shuffled"),
    # Two ragged sequences 65536 + 90112 in a shared 184320-token pool.
    "ragged_c2": Workload("ragged_c2", 3, (65536, 90112), 0, 1, 32, 4, 16, torch.bfloat16,
                          torch.bfloat16, 720, False, "head_variance", "shared_perm"),
    # MTP verification: 180224 cached + 4 appended, 4 causal queries.
    "mtp_verify": Workload("mtp_verify", 4, (180224,), 4, 4, 32, 4, 16, torch.bfloat16,
                           torch.bfloat16, 720, True, "normal", "shuffled"),
    # 262144 keys, 40/8 heads (GQA 5), 2% attention-sink tokens with x6 norm.
    "longest": Workload("longest", 5, (262144,), 0, 1, 40, 8, 16, torch.bfloat16,
                        torch.bfloat16, 1024, False, "k_sinks", "shuffled"),
}

ORDER = ["tiny", "ctx32k_append", "ragged_c2", "mtp_verify", "longest"]

# Chunked prefill (the pages' --prefill-chunk 1024): the last 1024-token chunk
# of a 180224-token prompt, appended and then attended causally, 32/4 heads,
# 16 layers, in the MTP workload's 720-block pool.  A workload of the
# chunked-prefill attention call, not of the decode step.
PREFILL = {
    "prefill_chunk": Workload("prefill_chunk", 6, (179200,), 1024, 1024, 32, 4, 16, torch.bfloat16,
                              torch.bfloat16, 720, True, "normal", "shuffled"),
}
WORKLOADS.update(PREFILL)


def get(name: str) -> Workload:
    return WORKLOADS[name]


def custom(name="custom", cached=(300,), n_new=0, n_q=1, num_q_heads=8, num_kv_heads=1,
           layers=1, q_dtype=torch.float32, kv_in_dtype=torch.float32, pool_blocks=None,
           causal=False, dist="normal", table="shuffled", index=77) -> Workload:
    """A small workload for parity tests (ragged tails, odd GQA, ...)."""
    need = sum(math.ceil((c + n_new) / BLOCK) for c in cached)
    return Workload(name, index, tuple(cached), n_new, n_q, num_q_heads, num_kv_heads, layers,
                    q_dtype, kv_in_dtype, pool_blocks or need + 3, causal, dist, table)


def seed(w: Workload, layer: int, kind: int) -> int:
    return (1000 + w.index) * 100003 + layer * 97 + kind


def block_table(w: Workload) -> np.ndarray:
    """int32 [batch][max_blocks]; unused entries are -1."""
    rng = np.random.default_rng(seed(w, 0, 11))
    nb = [math.ceil(L / BLOCK) for L in w.seqlens]
    bt = np.full((w.batch, w.max_blocks), -1, np.int32)
    if w.table == "contiguous":
        ids = np.arange(w.pool_blocks)
    else:  # a seeded permutation of the pool, sequences take consecutive runs of it
        ids = rng.permutation(w.pool_blocks)
    assert sum(nb) <= w.pool_blocks, "pool too small"
    off = 0
    for b, n in enumerate(nb):
        bt[b, :n] = ids[off:off + n]
        off += n
    return bt


def _gen(device, s):
    g = torch.Generator(device=device)
    g.manual_seed(s)
    return g


def layer_kv(w: Workload, layer: int, b: int, device="cpu"):
    """K and V for every position of sequence b in one layer (cached keys first,
    then the step's appended keys): two tensors [L_b][H_kv][d] of kv_in_dtype."""
    L = w.seqlens[b]
    H, d = w.num_kv_heads, w.head_dim
    gk = _gen(device, seed(w, layer, 20 + 2 * b))
    gv = _gen(device, seed(w, layer, 21 + 2 * b))
    k = torch.randn((L, H, d), generator=gk, device=device, dtype=torch.float32)
    v = torch.randn((L, H, d), generator=gv, device=device, dtype=torch.float32)
    rng = np.random.default_rng(seed(w, layer, 5))
    if w.dist == "k_outlier_channels":      # 4 random K channels per kv-head scaled x8
        for h in range(H):
            ch = torch.as_tensor(rng.choice(d, 4, replace=False), device=device)
            k[:, h, ch] *= 8.0
    elif w.dist == "head_variance":         # per (layer, kv-head, K or V) variance ~ U[0.5, 2]
        var = rng.uniform(0.5, 2.0, size=(2, H))
        k *= torch.as_tensor(np.sqrt(var[0]), dtype=torch.float32, device=device)[None, :, None]
        v *= torch.as_tensor(np.sqrt(var[1]), dtype=torch.float32, device=device)[None, :, None]
    elif w.dist == "k_sinks":               # 2% of token positions (all heads) with x6 norm
        n_sink = max(1, int(round(0.02 * L)))
        idx = torch.as_tensor(rng.choice(L, n_sink, replace=False), device=device)
        k[idx] *= 6.0
    elif w.dist != "normal":
        raise ValueError(w.dist)
    return k.to(w.kv_in_dtype), v.to(w.kv_in_dtype)


def layer_q(w: Workload, layer: int, device="cpu"):
    """q [batch][n_q][H_q][d] of q_dtype, ~N(0, 1)."""
    g = _gen(device, seed(w, layer, 3))
    q = torch.randn((w.batch, w.n_q, w.num_q_heads, w.head_dim), generator=g, device=device,
                    dtype=torch.float32)
    return q.to(w.q_dtype)


def kv_bytes_per_token_head(fmt: str = "k8v4", d: int = HEAD_DIM) -> int:
    """Bytes one cached key/value pair occupies per kv-head: K8/V4 stores d int8
    K codes, one fp16 K scale, d/2 bytes of V nibbles and d/32 fp16 V scales;
    the int8 (fp8) cache d int8 (e4m3) codes and one fp16 scale for each of K
    and V; the RK4V4-E8 cache d/2 bytes of nibbles and d/32 exponent bytes for
    each of K and V."""
    if fmt == "k8v4":
        return d + 2 + d // 2 + 2 * (d // 32)
    if fmt in ("k8v8", "f8"):
        return 2 * (d + 2)
    if fmt == "k4v4":  # RK4V4-E8: d/2 bytes of nibbles and d/32 exponent bytes for each of K and V
        return 2 * (d // 2 + d // 32)
    if fmt == "bf16":
        return 4 * d  # bf16 K and V
    raise ValueError(f"unknown KV format {fmt!r}")
