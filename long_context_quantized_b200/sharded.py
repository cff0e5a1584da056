"""Context-sharded decode attention across GPUs.

A request's KV cache is split by position across the ranks of a process group.
Each rank holds whole 256-token blocks of every sequence and computes decode
attention of the (replicated) queries against its own keys: a partial output
and log-sum-exp per query row, written into one packed slot (o rows, then the
lse values).  One all-gather exchanges the slots, and every rank merges them
with the log-sum-exp combine (``nf_attn_combine_packed``).
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


def shard_positions(spec: ShardSpec, b: int) -> range:
    """Global key positions of sequence b held by this shard."""
    start = BLOCK * spec.first_block[b]
    return range(start, start + spec.lengths[b])


def local_pool_table(spec: ShardSpec, device=None) -> torch.Tensor:
    """Block table of a rank that stores only its own shard: sequence b's
    n_blocks[b] blocks are local blocks off_b .. off_b + n_blocks[b] - 1 (off_b
    the blocks of the sequences before it), so a pool of sum(n_blocks) blocks
    holds the shard; local position p of sequence b (global position
    BLOCK * first_block[b] + p) is in local block off_b + p // BLOCK.  Rows are
    padded with -1."""
    width = max(1, max(spec.n_blocks) if spec.n_blocks else 1)
    out = torch.full((len(spec.n_blocks), width), -1, dtype=torch.int32)
    off = 0
    for b, n in enumerate(spec.n_blocks):
        if n:
            out[b, :n] = torch.arange(off, off + n, dtype=torch.int32)
        off += n
    return out.to(device) if device is not None else out


def local_block_table(spec: ShardSpec, block_table: torch.Tensor) -> torch.Tensor:
    """The shard's rows of the block table: row b = block_table[b, first:first + n]
    (padded with -1), in the same block-id space as the given table."""
    width = max(1, max(spec.n_blocks) if spec.n_blocks else 1)
    out = torch.full((block_table.shape[0], width), -1, dtype=torch.int32, device=block_table.device)
    for b, (f, n) in enumerate(zip(spec.first_block, spec.n_blocks)):
        if n:
            out[b, :n] = block_table[b, f:f + n]
    return out


def packed_views(slot: torch.Tensor, B: int, n_q: int, H_q: int, d: int = 128):
    """(o [B][n_q][H_q][d], lse [B][n_q][H_q]) views of one packed split slot
    (o rows first, then the lse values: the layout nf_attn_combine_packed
    reads)."""
    rows = B * n_q * H_q
    return slot[:rows * d].view(B, n_q, H_q, d), slot[rows * d:rows * (d + 1)].view(B, n_q, H_q)


def decode_partial_into(kv, q, spec: ShardSpec, local_bt: torch.Tensor, softmax_scale: float, slot: torch.Tensor,
                        workspace: torch.Tensor, seqlens: torch.Tensor = None):
    """This shard's partial decode attention written into its packed slot:
    o and lse over the shard's keys.  Sequences with no key here get o = 0
    and lse = -inf (they add nothing to the merge).  seqlens: the shard's
    lengths as a device int32 tensor (made from spec.lengths when None)."""
    B, n_q, H_q, d = q.shape
    o, lse = packed_views(slot, B, n_q, H_q, d)
    active = [b for b in range(B) if spec.lengths[b] > 0]
    if len(active) == B:
        sl = torch.as_tensor(spec.lengths, dtype=torch.int32, device=q.device) if seqlens is None else seqlens
        nf.nf_decode_attn(kv, q, local_bt, sl, spec.max_length, softmax_scale, spec.causal, o, lse, workspace)
        return
    o.zero_()
    lse.fill_(float("-inf"))
    if not active:
        return
    idx = torch.as_tensor(active, dtype=torch.long, device=q.device)
    q_a = q.index_select(0, idx).contiguous()
    bt_a = local_bt.index_select(0, idx).contiguous()
    sl = torch.as_tensor([spec.lengths[b] for b in active], dtype=torch.int32, device=q.device)
    o_a = torch.empty((len(active), n_q, H_q, d), dtype=torch.float32, device=q.device)
    lse_a = torch.empty((len(active), n_q, H_q), dtype=torch.float32, device=q.device)
    nf.nf_decode_attn(kv, q_a, bt_a, sl, spec.max_length, softmax_scale, spec.causal, o_a, lse_a, workspace)
    o.index_copy_(0, idx, o_a)
    lse.index_copy_(0, idx, lse_a)


def decode_partial(kv, q, spec: ShardSpec, local_bt: torch.Tensor, softmax_scale: float, workspace=None):
    """This shard's partial decode attention: (o [B][n_q][H_q][128], lse
    [B][n_q][H_q]) over its keys (views of a fresh packed slot)."""
    B, n_q, H_q, d = q.shape
    slot = torch.empty(nf.nf_attn_packed_slot_floats(B * n_q * H_q, d), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.zeros(nf.nf_decode_attn_workspace_size(B, n_q, H_q, kv.num_kv_heads,
                                                                 max(1, spec.max_length)),
                                dtype=torch.uint8, device=q.device)
    decode_partial_into(kv, q, spec, local_bt, softmax_scale, slot, workspace)
    return packed_views(slot, B, n_q, H_q, d)


def gather_packed(slot: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather every rank's packed slot in one collective: [W][slot] in
    rank order."""
    import torch.distributed as dist
    W = dist.get_world_size(group)
    out = torch.empty((W * slot.numel(),), dtype=slot.dtype, device=slot.device)
    dist.all_gather_into_tensor(out, slot.contiguous(), group=group)
    return out.view(W, -1)


class ShardedDecoder:
    """Context-sharded decode attention of one shard plan, with its buffers
    (the rank's packed slot, the gathered slots, the outputs and one decode
    workspace) allocated once and reused for every layer and step."""

    def __init__(self, spec: ShardSpec, batch: int, n_q: int, num_q_heads: int, num_kv_heads: int,
                 device, group=None):
        self.spec, self.group = spec, group
        self.B, self.n_q, self.H_q = batch, n_q, num_q_heads
        rows = batch * n_q * num_q_heads
        self.rows = rows
        slot = nf.nf_attn_packed_slot_floats(rows, 128)
        self.slot = torch.empty(slot, dtype=torch.float32, device=device)
        self.gathered = torch.empty((spec.world_size, slot), dtype=torch.float32, device=device)
        self.out = torch.empty((batch, n_q, num_q_heads, 128), dtype=torch.float32, device=device)
        self.out_lse = torch.empty((batch, n_q, num_q_heads), dtype=torch.float32, device=device)
        ws = nf.nf_decode_attn_workspace_size(batch, n_q, num_q_heads, num_kv_heads, max(n_q, spec.max_length))
        self.workspace = torch.zeros(ws, dtype=torch.uint8, device=device)
        self.seqlens = torch.as_tensor(spec.lengths, dtype=torch.int32, device=device)  # once, not per call

    def __call__(self, kv, q, local_bt: torch.Tensor, softmax_scale: float, out=None, out_lse=None):
        """One layer: the local partial, one all-gather of the packed slots, the
        merge into out / out_lse (fp32 [B][n_q][H_q][128] / [B][n_q][H_q];
        this object's buffers when None).  Returns (out, out_lse) on every
        rank.  With one rank the decode writes out directly."""
        out = self.out if out is None else out
        out_lse = self.out_lse if out_lse is None else out_lse
        if self.spec.world_size == 1:
            if all(n > 0 for n in self.spec.lengths):
                nf.nf_decode_attn(kv, q, local_bt, self.seqlens, self.spec.max_length, softmax_scale,
                                  self.spec.causal, out, out_lse, self.workspace)
                return out, out_lse
            decode_partial_into(kv, q, self.spec, local_bt, softmax_scale, self.slot, self.workspace, self.seqlens)
            o, lse = packed_views(self.slot, self.B, self.n_q, self.H_q)
            out.copy_(o)
            out_lse.copy_(lse)
            return out, out_lse
        decode_partial_into(kv, q, self.spec, local_bt, softmax_scale, self.slot, self.workspace, self.seqlens)
        import torch.distributed as dist
        dist.all_gather_into_tensor(self.gathered.view(-1), self.slot, group=self.group)
        nf.nf_attn_combine_packed(self.gathered, self.rows, out.view(self.rows, 128), out_lse.view(-1))
        return out, out_lse


def sharded_decode_attn(kv, q, spec: ShardSpec, local_bt: torch.Tensor, softmax_scale: float, group=None,
                        workspace=None):
    """Decode attention of q against the keys of all ranks' shards: the local
    partial, one all-gather of the packed partials, and the merge.  Returns
    (out [B][n_q][H_q][128], lse [B][n_q][H_q]) on every rank."""
    B, n_q, H_q, d = q.shape
    slot = torch.empty(nf.nf_attn_packed_slot_floats(B * n_q * H_q, d), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.zeros(nf.nf_decode_attn_workspace_size(B, n_q, H_q, kv.num_kv_heads,
                                                                 max(n_q, spec.max_length)),
                                dtype=torch.uint8, device=q.device)
    decode_partial_into(kv, q, spec, local_bt, softmax_scale, slot, workspace)
    if spec.world_size == 1:
        return packed_views(slot, B, n_q, H_q, d)
    parts = gather_packed(slot, group)
    out = torch.empty((B, n_q, H_q, d), dtype=torch.float32, device=q.device)
    out_lse = torch.empty((B, n_q, H_q), dtype=torch.float32, device=q.device)
    nf.nf_attn_combine_packed(parts, B * n_q * H_q, out.view(-1, d), out_lse.view(-1))
    return out, out_lse
