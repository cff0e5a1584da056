"""Run one seeded workload layer through the CUDA path and through the CPU
oracle, and compare.  Inputs come from ``workloads`` (generated on the GPU and
copied to the host for the oracle); nothing the oracle sees comes from the
CUDA kernels."""
from __future__ import annotations

import math
import os

import numpy as np
import torch

import long_context_quantized_b200 as nf
import oracle
import workloads

# Tolerance on attention outputs against the oracle's fp64 result (per layer
# tensor), and on the log-sum-exp.
ATOL = 2e-3
REL_L2 = 1e-3
LSE_ATOL = 2e-3
POISON = 0xA5


def gpu_layer(w, layer, fmt, q_override=None, max_seqlen=None, bt=None, seqlens=None, attn="decode"):
    """Fill one layer's pool on the GPU (bulk append of the cached keys, then
    the step's appended keys), run decode (or chunked-prefill) attention.
    Returns dict of tensors."""
    dev = "cuda"
    bt_np = workloads.block_table(w) if bt is None else bt
    if max_seqlen is not None and bt_np.shape[1] * 256 < max_seqlen:
        # the table must span the host bound; the extra columns are never read
        pad = np.full((bt_np.shape[0], math.ceil(max_seqlen / 256) - bt_np.shape[1]), -1, np.int32)
        bt_np = np.concatenate([bt_np, pad], axis=1)
    bt_t = torch.as_tensor(bt_np, dtype=torch.int32, device=dev)
    kv = nf.KVLayer.empty(fmt, w.pool_blocks, w.num_kv_heads, device=dev, fill=POISON)
    kvin = []
    for b in range(w.batch):
        k, v = workloads.layer_kv(w, layer, b, device=dev)
        kvin.append((k, v))
        c = w.cached[b]
        row = bt_t[b:b + 1]
        if c:
            nf.nf_kv_append_quant(kv, k[None, :c].contiguous(), v[None, :c].contiguous(), row,
                                  torch.zeros(1, dtype=torch.int32, device=dev))
        if w.n_new:
            nf.nf_kv_append_quant(kv, k[None, c:].contiguous(), v[None, c:].contiguous(), row,
                                  torch.full((1,), c, dtype=torch.int32, device=dev))
    q = workloads.layer_q(w, layer, device=dev) if q_override is None else q_override
    sl = torch.as_tensor(w.seqlens if seqlens is None else seqlens, dtype=torch.int32, device=dev)
    msl = max(w.seqlens) if max_seqlen is None else max_seqlen
    out = torch.empty((w.batch, w.n_q, w.num_q_heads, 128), dtype=torch.float32, device=dev)
    lse = torch.empty((w.batch, w.n_q, w.num_q_heads), dtype=torch.float32, device=dev)
    if attn == "prefill":
        nf.nf_prefill_attn(kv, q, bt_t, sl, msl, w.softmax_scale, w.causal, out, lse)
    else:
        ws = torch.zeros(nf.nf_decode_attn_workspace_size(w.batch, w.n_q, w.num_q_heads, w.num_kv_heads, msl),
                         dtype=torch.uint8, device=dev)
        nf.nf_decode_attn(kv, q, bt_t, sl, msl, w.softmax_scale, w.causal, out, lse, ws)
    torch.cuda.synchronize()
    return dict(kv=kv, q=q, out=out, lse=lse, bt=bt_np, kvin=kvin)


def oracle_pool(w, fmt, kvin, bt, heads=None):
    """The oracle's own pool from the same raw inputs (fp32 values), for all
    kv-heads or only the listed ones (as a pool with len(heads) heads)."""
    hs = list(range(w.num_kv_heads)) if heads is None else list(heads)
    pool = oracle.Pool(fmt, w.pool_blocks, len(hs), 128, poison=POISON)
    for b, (k, v) in enumerate(kvin):
        kk = k[:, hs].float().cpu().numpy()[None]
        vv = v[:, hs].float().cpu().numpy()[None]
        assert oracle.append(pool, kk, vv, bt[b:b + 1], np.zeros(1, np.int32)) == 0
    return pool, hs


def compare_pool(kv, pool, heads):
    """Bit-exact comparison of every byte of the planes (for the listed heads)."""
    gpu = [t[:, heads].contiguous().view(torch.uint8).cpu().numpy() for t in kv.planes()]
    ref = [a for a in pool.planes()] if kv.fmt != nf.NF_KV_BF16 else [pool.k, pool.v]
    for gp, rp in zip(gpu, ref):
        g8 = np.ascontiguousarray(gp).view(np.uint8).reshape(-1)
        r8 = np.ascontiguousarray(rp).view(np.uint8).reshape(-1)
        assert g8.shape == r8.shape
        bad = np.nonzero(g8 != r8)[0]
        assert bad.size == 0, f"{bad.size} bytes differ, first at {bad[:5]}"


def oracle_attention(w, pool, hs, q, bt, seqlens=None, nthreads=None):
    """Oracle attention for the q heads that map to the kv-heads in hs."""
    G = w.group
    qn = q.float().cpu().numpy().astype(np.float64)
    qsel = np.concatenate([qn[:, :, h * G:(h + 1) * G] for h in hs], axis=2)
    sl = np.array(w.seqlens if seqlens is None else seqlens, np.int32)
    out, lse = oracle.decode_attn(pool, qsel, bt, sl, w.softmax_scale, w.causal,
                                  nthreads=nthreads or os.cpu_count())
    return out.reshape(w.batch, w.n_q, len(hs) * G, 128), lse.reshape(w.batch, w.n_q, len(hs) * G)


def select_heads(t, w, hs):
    G = w.group
    return torch.cat([t[:, :, h * G:(h + 1) * G] for h in hs], dim=2)


def check_attention(got_o, got_lse, ref_o, ref_lse):
    go = got_o.cpu().numpy().astype(np.float64)
    gl = got_lse.cpu().numpy().astype(np.float64)
    err = np.abs(go - ref_o)
    rel = np.linalg.norm(go - ref_o) / max(np.linalg.norm(ref_o), 1e-300)
    assert np.all(np.isfinite(go)), "non-finite output"
    assert err.max() <= ATOL, f"max abs err {err.max():.3e} > {ATOL}"
    assert rel <= REL_L2, f"rel L2 err {rel:.3e} > {REL_L2}"
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(gl), fin)
    if fin.any():
        lerr = np.abs(gl[fin] - ref_lse[fin]).max()
        assert lerr <= LSE_ATOL, f"lse err {lerr:.3e}"
    return float(err.max()), float(rel)


def run_case(w, layer=0, fmt=nf.NF_KV_K8V4, heads=None, **kw):
    g = gpu_layer(w, layer, fmt, **kw)
    pool, hs = oracle_pool(w, fmt, g["kvin"], g["bt"], heads)
    compare_pool(g["kv"], pool, hs)
    ref_o, ref_l = oracle_attention(w, pool, hs, g["q"], g["bt"], kw.get("seqlens"))
    return check_attention(select_heads(g["out"], w, hs), select_heads(g["lse"], w, hs), ref_o, ref_l)


def blocks_for(lengths):
    return sum(math.ceil(L / 256) for L in lengths)
