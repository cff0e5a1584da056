"""Context-sharded decode attention across GPUs.

A request's KV cache is split by position across the ranks of a process group.
Each rank holds whole 256-token blocks of every sequence and computes decode
attention of the (replicated) queries against its own keys: a partial output
and log-sum-exp per query row.  One all-gather exchanges the partials, and
every rank merges them with the log-sum-exp combine (``nf_attn_combine``).
The pages run one request per GPU; this is the multi-GPU form of their
segment-at-a-time decode (page "標籤: vLLM", section 2: the KV cache is
managed in segments by context length), with the flash-decoding merge across
segments.

Causal MTP queries (query j at position L - n_q + j sees keys up to it) need
no special kernel: every shard boundary is placed at or before position
L - n_q, so all shards but the last hold only keys every query sees (decoded
without the mask) and the last shard, which ends at L and holds at least the
n_q newest keys, is decoded causally with its own length.
"""
from __future__ import annotations

import dataclasses
import math

import torch

import long_context_quantized_b200 as nf

BLOCK = 256


@dataclasses.dataclass(frozen=True)
class ShardSpec:
    """One rank's part of a batch: per sequence the range [first_block,
    first_block + n_blocks) of its block table and the keys in it."""
    rank: int
    world_size: int
    first_block: tuple   # per sequence
    n_blocks: tuple      # per sequence
    lengths: tuple       # keys of the sequence in this shard (0: none)
    causal: bool         # this shard holds the newest keys of every sequence

    @property
    def max_length(self) -> int:
        return max(self.lengths) if self.lengths else 0


def shard_plan(seqlens, n_q: int, world_size: int, causal: bool) -> list:
    """Split each sequence's blocks into world_size contiguous ranges.

    Rank r gets blocks [floor(nb r / W), floor(nb (r + 1) / W)) of a sequence
    of nb blocks, with every boundary moved back, if needed, to the last block
    edge at or before position L - n_q.  Every rank but the last then holds
    only keys below the first query's position, and the last rank holds at
    least the n_q newest keys.
    """
    if world_size < 1:
        raise ValueError("world_size must be >= 1")
    specs = []
    bounds = []  # per sequence: block-index boundaries b_0 = 0 <= ... <= b_W = nb
    for L in seqlens:
        if L < n_q:
            raise ValueError(f"sequence length {L} < n_q {n_q}")
        nb = math.ceil(L / BLOCK)
        cap = (L - n_q) // BLOCK  # boundaries at or before position L - n_q
        b = [0] + [min(nb * r // world_size, cap) for r in range(1, world_size)] + [nb]
        for r in range(1, world_size):
            b[r] = max(b[r], b[r - 1])
        bounds.append(b)
    for r in range(world_size):
        first = tuple(b[r] for b in bounds)
        count = tuple(b[r + 1] - b[r] for b in bounds)
        lengths = tuple(max(0, min(BLOCK * b[r + 1], L) - BLOCK * b[r]) for b, L in zip(bounds, seqlens))
        specs.append(ShardSpec(r, world_size, first, count, lengths, causal and r == world_size - 1))
    return specs


def local_block_table(spec: ShardSpec, block_table: torch.Tensor) -> torch.Tensor:
    """The shard's rows of the block table: row b = block_table[b, first:first + n]
    (padded with -1), in the same block-id space as the given table."""
    width = max(1, max(spec.n_blocks) if spec.n_blocks else 1)
    out = torch.full((block_table.shape[0], width), -1, dtype=torch.int32, device=block_table.device)
    for b, (f, n) in enumerate(zip(spec.first_block, spec.n_blocks)):
        if n:
            out[b, :n] = block_table[b, f:f + n]
    return out


def decode_partial(kv, q, spec: ShardSpec, local_bt: torch.Tensor, softmax_scale: float, workspace=None):
    """This shard's partial decode attention: (o [B][n_q][H_q][128], lse
    [B][n_q][H_q]) over its keys.  Sequences with no key here get o = 0 and
    lse = -inf (they add nothing to the merge) without a kernel call."""
    B, n_q, H_q, d = q.shape
    dev = q.device
    o = torch.zeros((B, n_q, H_q, d), dtype=torch.float32, device=dev)
    lse = torch.full((B, n_q, H_q), float("-inf"), dtype=torch.float32, device=dev)
    active = [b for b in range(B) if spec.lengths[b] > 0]
    if not active:
        return o, lse
    idx = torch.as_tensor(active, dtype=torch.long, device=dev)
    q_a = q.index_select(0, idx).contiguous()
    bt_a = local_bt.index_select(0, idx).contiguous()
    sl = torch.as_tensor([spec.lengths[b] for b in active], dtype=torch.int32, device=dev)
    msl = max(spec.lengths[b] for b in active)
    o_a = torch.empty((len(active), n_q, H_q, d), dtype=torch.float32, device=dev)
    lse_a = torch.empty((len(active), n_q, H_q), dtype=torch.float32, device=dev)
    if workspace is None:
        ws = nf.nf_decode_attn_workspace_size(len(active), n_q, H_q, kv.num_kv_heads, msl)
        workspace = torch.zeros(ws, dtype=torch.uint8, device=dev)
    nf.nf_decode_attn(kv, q_a, bt_a, sl, msl, softmax_scale, spec.causal, o_a, lse_a, workspace)
    o.index_copy_(0, idx, o_a)
    lse.index_copy_(0, idx, lse_a)
    return o, lse


def gather_partials(o: torch.Tensor, lse: torch.Tensor, group=None):
    """All-gather every rank's partial: ([W][rows][d], [W][rows]) in rank order."""
    import torch.distributed as dist
    W = dist.get_world_size(group)
    d = o.shape[-1]
    o2 = o.reshape(-1, d).contiguous()
    l2 = lse.reshape(-1).contiguous()
    # outputs concatenated along dim 0 (the form every backend accepts), viewed per rank
    part_o = torch.empty((W * o2.shape[0], d), dtype=o2.dtype, device=o2.device)
    part_l = torch.empty((W * l2.shape[0],), dtype=l2.dtype, device=l2.device)
    dist.all_gather_into_tensor(part_o, o2, group=group)
    dist.all_gather_into_tensor(part_l, l2, group=group)
    return part_o.view(W, -1, d), part_l.view(W, -1)


def sharded_decode_attn(kv, q, spec: ShardSpec, local_bt: torch.Tensor, softmax_scale: float, group=None,
                        workspace=None):
    """Decode attention of q against the keys of all ranks' shards: the local
    partial, one all-gather, and the merge.  Returns (out [B][n_q][H_q][128],
    lse [B][n_q][H_q]) on every rank."""
    o, lse = decode_partial(kv, q, spec, local_bt, softmax_scale, workspace)
    if spec.world_size == 1:
        return o, lse
    part_o, part_l = gather_partials(o, lse, group)
    out = torch.empty_like(part_o[0])
    out_lse = torch.empty_like(part_l[0])
    nf.nf_attn_combine(part_o, part_l, out, out_lse)
    return out.reshape(o.shape), out_lse.reshape(lse.shape)
