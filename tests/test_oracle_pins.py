"""Pins for the CPU oracle: it is checked against things other than itself.

- IEEE conversions against numpy's / torch's own float16 and bfloat16 casts;
  the fp8 e4m3 conversions against torch's float8_e4m3fn type and a search
  over all 254 finite codes.
- The quantiser against a numpy re-derivation (numpy float32 division, float16
  cast, rint) and against hand-derived cases (tests/golden/).
- Attention against closed forms (q = 0 gives the mean of the visible values,
  one key gives that key's value, two keys give logistic weights), invariants
  (block permutation, split + combine, GQA head mapping, causal prefix) and a
  brute-force numpy computation on tiny inputs whose dequantisation is done by
  numpy from the raw pool bytes.
Each pin is chosen so that a plausible slip in the oracle (a dropped term, a
wrong sign or index, a transposed operand, an off-by-one in the causal limit,
a wrong nibble order or rounding mode) fails at least one of them.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "k8v4_rounding_cases.txt")
RNG = np.random.default_rng(1234)


# ------------------------------------------------------------ numpy helpers
def np_f16_sat(x32):
    """numpy's IEEE fp32->fp16 cast (round half to even) with saturation."""
    with np.errstate(over="ignore"):
        h = np.asarray(x32, np.float32).astype(np.float16)
    h = np.where(np.isinf(h), np.copysign(np.float16(65504), h), h).astype(np.float16)
    return h


def np_quant(x, qmax):
    """Independent numpy statement of the quantiser for one vector."""
    x = np.asarray(x, np.float32)
    a = np.max(np.abs(x)).astype(np.float32)
    s32 = np.float32(a) / np.float32(qmax)
    s16 = np_f16_sat(s32)
    sig = np.float32(s16)
    if sig == 0:
        return s16.view(np.uint16), np.zeros(x.shape, np.int64)
    c = np.rint(x / sig).astype(np.float64)
    return s16.view(np.uint16), np.clip(c, -qmax, qmax).astype(np.int64)


def torch_e4m3(codes):
    """fp64 values of e4m3 bytes through torch's own float8_e4m3fn type."""
    t = torch.from_numpy(np.ascontiguousarray(codes, np.uint8))
    return t.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def e4m3_table():
    """The finite e4m3 codes and their values (torch's decoding)."""
    codes = np.array([c for c in range(256) if c & 0x7F != 0x7F], np.uint8)
    return codes, torch_e4m3(codes)


def brute_e4m3(x):
    """Nearest finite e4m3 code of each fp32 value by search over all codes:
    ties go to the code with the even mantissa, magnitudes past 448 to +-448,
    a zero result keeps the sign of x."""
    codes, vals = e4m3_table()
    x = np.asarray(x, np.float32).astype(np.float64)
    out = np.empty(x.shape, np.uint8)
    for i, xv in enumerate(x.ravel()):
        d = np.abs(vals - np.clip(xv, -448.0, 448.0))
        best = np.flatnonzero(d == d.min())
        if best.size > 1:
            best = best[(codes[best] & 1) == 0]
        c = codes[best]
        if vals[best[0]] == 0.0:  # +0 and -0 tie: the sign of x decides
            c = np.array([0x80 if np.signbit(xv) else 0x00])
        assert c.size == 1
        out.ravel()[i] = c[0]
    return out


def np_unpack_v(packed):
    p = np.asarray(packed, np.uint8).astype(np.int64)
    lo, hi = p & 0xF, p >> 4
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), np.int64)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


def np_dequant_pool(pool):
    """fp64 K_hat, V_hat [nb][H][256][d] from the raw pool bytes, via numpy."""
    if pool.fmt == oracle.FMT_BF16:
        k = (pool.k.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        v = (pool.v.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        return k, v
    if pool.fmt == oracle.FMT_K4V4:
        k = np_unpack_v(pool.k).astype(np.float64) * np.repeat(np.ldexp(1.0, pool.k_scale.astype(np.int64) - 127), 32,
                                                                axis=-1)
        v = np_unpack_v(pool.v).astype(np.float64) * np.repeat(np.ldexp(1.0, pool.v_scale.astype(np.int64) - 127), 32,
                                                                axis=-1)
        return k, v
    ks = pool.k_scale.view(np.float16).astype(np.float64)
    vs = pool.v_scale.view(np.float16).astype(np.float64)
    k = pool.k.astype(np.float64) * ks[..., None]
    if pool.fmt == oracle.FMT_K8V8:
        return k, pool.v.astype(np.float64) * vs[..., None]
    if pool.fmt == oracle.FMT_F8:
        return (torch_e4m3(pool.k) * ks[..., None], torch_e4m3(pool.v) * vs[..., None])
    vc = np_unpack_v(pool.v).astype(np.float64)
    v = vc * np.repeat(vs, 32, axis=-1)
    return k, v


def make_pool(fmt, cached, H, d=128, nb_extra=3, seed=0, shuffle=True, k_scale_mul=1.0):
    """Fill a pool by the oracle's own append; returns pool, table, k, v (fp32)."""
    rng = np.random.default_rng(seed)
    nblk = [math.ceil(L / 256) for L in cached]
    nb = sum(nblk) + nb_extra
    ids = rng.permutation(nb) if shuffle else np.arange(nb)
    bt = np.full((len(cached), max(nblk)), -1, np.int32)
    off = 0
    for b, n in enumerate(nblk):
        bt[b, :n] = ids[off:off + n]
        off += n
    pool = oracle.Pool(fmt, nb, H, d)
    ks, vs = [], []
    for b, L in enumerate(cached):
        k = (rng.standard_normal((1, L, H, d)) * k_scale_mul).astype(np.float32)
        v = rng.standard_normal((1, L, H, d)).astype(np.float32)
        assert oracle.append(pool, k, v, bt[b:b + 1], np.array([0], np.int32)) == 0
        ks.append(k[0])
        vs.append(v[0])
    return pool, bt, ks, vs


def np_attention(pool, bt, seqlens, q, scale, causal):
    """Brute-force fp64 softmax attention with numpy, from numpy-dequantised pool."""
    kh, vh = np_dequant_pool(pool)
    B, n_q, Hq, d = q.shape
    G = Hq // pool.H
    out = np.zeros((B, n_q, Hq, d))
    lse = np.zeros((B, n_q, Hq))
    for b in range(B):
        L = seqlens[b]
        pos = np.arange(L)
        blk = bt[b, pos // 256]
        for h in range(Hq):
            K = kh[blk, h // G, pos % 256]
            V = vh[blk, h // G, pos % 256]
            for j in range(n_q):
                n = L - n_q + j + 1 if causal else L
                s = np.float64(np.float32(scale)) * (K[:n] @ q[b, j, h].astype(np.float64))
                m = s.max()
                w = np.exp(s - m)
                out[b, j, h] = (w @ V[:n]) / w.sum()
                lse[b, j, h] = m + np.log(w.sum())
    return out.reshape(-1, d), lse.reshape(-1)


# ------------------------------------------------------------- conversions
def test_f16_from_f32_matches_numpy():
    exps = RNG.integers(-30, 18, size=200000)
    x = (RNG.uniform(1, 2, size=exps.size) * np.exp2(exps)).astype(np.float32)
    x *= np.where(RNG.random(x.size) < 0.5, -1, 1).astype(np.float32)
    # exact ties between fp16 neighbours, subnormal ties, and overflow region
    ties = (np.arange(1, 2048, dtype=np.float64) + 0.5) * 2.0 ** -24
    big = np.array([65504, 65519.99, 65520, 65536, 1e6, -7e5, 2.0 ** -25, 3 * 2.0 ** -26])
    x = np.concatenate([x, ties.astype(np.float32), big.astype(np.float32), [0.0, -0.0]]).astype(np.float32)
    got = oracle.f32_to_f16_bits(x)
    want = np_f16_sat(x).view(np.uint16)
    assert np.array_equal(got, want)


def test_f16_to_f32_all_patterns():
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    want = h.view(np.float16).astype(np.float32)
    got = oracle.f16_bits_to_f32(h)
    fin = np.isfinite(want)
    assert np.array_equal(got[fin], want[fin])
    assert np.array_equal(np.isnan(got), np.isnan(want))


def test_bf16_conversions_match_torch():
    x = torch.randn(100000, dtype=torch.float32) * torch.exp2(torch.randint(-60, 60, (100000,)).float())
    x = torch.cat([x, torch.tensor([0.0, -0.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1e-40, -3e-39])])
    want = x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.f32_to_bf16_bits(x.numpy())
    assert np.array_equal(got, want)
    back = oracle.bf16_bits_to_f32(want)
    assert np.array_equal(back, torch.from_numpy(want.view(np.int16)).view(torch.bfloat16).float().numpy())


# ------------------------------------------------------------- quantiser
def _parse_val(tok):
    if "*2^" in tok:
        m, e = tok.split("*2^")
        return float(np.float32(int(m) * 2.0 ** int(e)))
    return float(tok)


def _golden_cases():
    cases = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            head, tail = line.split("|")
            parts = head.split()
            cases.append((parts[0], parts[1:], [t for t in tail.split()]))
    return cases


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c[0] + ":" + " ".join(c[1][:3]))
def test_quant_golden(case):
    kind, head, tail = case
    if kind == "PACK":
        codes = [int(t) for t in head]
        want = np.array([int(t, 16) for t in tail], np.uint8)
        # V group whose scale is 1/4 exactly: x = code * 0.25, absmax 1.75 -> codes back
        x = np.zeros(128, np.float32)
        x[:len(codes)] = np.array(codes, np.float32) * 0.25
        x[len(codes)] = 1.75 if max(abs(c) for c in codes) < 7 else 0.0
        _, packed = oracle.quant_v(x)
        assert np.array_equal(packed[:len(want)], want)
        return
    bits = int(head[0], 16)
    xs = np.array([_parse_val(t) for t in head[1:]], np.float32)
    want = np.array([int(t) for t in tail], np.int64)
    if kind == "K":
        x = np.zeros(128, np.float32)
        x[:len(xs)] = xs
        s, c = oracle.quant_k(x)
        assert int(s) == bits
        assert np.array_equal(c[:len(want)].astype(np.int64), want)
        assert np.all(c[len(want):] == 0)
    else:
        x = np.zeros(128, np.float32)
        x[:len(xs)] = xs
        s, packed = oracle.quant_v(x)
        assert int(s[0]) == bits
        codes = np_unpack_v(packed)
        assert np.array_equal(codes[:len(want)], want)


def _random_vectors(n, d=128):
    out = []
    for i in range(n):
        kind = i % 6
        if kind == 0:
            x = RNG.standard_normal(d)
        elif kind == 1:  # outlier channels
            x = RNG.standard_normal(d)
            x[RNG.choice(d, 4, replace=False)] *= 8
        elif kind == 2:  # tiny values: subnormal fp16 scales
            x = RNG.standard_normal(d) * 10.0 ** RNG.uniform(-9, -4)
        elif kind == 3:  # large values: near the fp16 scale limit
            x = RNG.standard_normal(d) * 10.0 ** RNG.uniform(3, 7)
        elif kind == 4:  # values on the quantisation grid (ties)
            x = (RNG.integers(-254, 255, d) / 2.0) * 2.0 ** RNG.integers(-8, 4)
        else:  # sparse
            x = RNG.standard_normal(d) * (RNG.random(d) < 0.1)
        out.append(x.astype(np.float32))
    return out


def test_quant_k_matches_numpy_rederivation():
    for x in _random_vectors(3000):
        s, c = oracle.quant_k(x)
        ws, wc = np_quant(x, 127)
        assert int(s) == int(ws)
        assert np.array_equal(c.astype(np.int64), wc)


def test_quant_v_matches_numpy_rederivation():
    for x in _random_vectors(3000):
        s, packed = oracle.quant_v(x)
        codes = np_unpack_v(packed)
        for g in range(4):
            ws, wc = np_quant(x[32 * g:32 * g + 32], 7)
            assert int(s[g]) == int(ws)
            assert np.array_equal(codes[32 * g:32 * g + 32], wc)


def test_quant_roundtrip_and_scale_bounds():
    for x in _random_vectors(1200):
        s, c = oracle.quant_k(x)
        sig = float(oracle.f16_bits_to_f32([s])[0])
        a = float(np.max(np.abs(x)))
        if sig == 0:
            assert np.all(c == 0)
            continue
        if a / 127 < 65504 and a / 127 >= 2.0 ** -14:  # normal fp16 range
            assert abs(sig - a / 127) <= 2.0 ** -11 * (a / 127) * (1 + 1e-6)
        err = np.abs(x.astype(np.float64) - c.astype(np.float64) * sig)
        unclamped = np.abs(x.astype(np.float64) / sig) <= 127.5
        assert np.all(err[unclamped] <= sig / 2 * (1 + 1e-6))
        assert np.all(err[~unclamped] <= np.abs(x[~unclamped]) - 127 * sig + 1e-12)
        assert c.min() >= -127 and c.max() <= 127


# ---------------------------------------------------------------- append
def test_append_places_tokens_through_block_table():
    H, d = 3, 128
    nb = 7
    bt = np.array([[5, 2, 6], [0, 4, -1]], np.int32)
    pool = oracle.Pool(oracle.FMT_K8V4, nb, H, d, poison=0x5A)
    before = [p.copy() for p in pool.planes()]
    sb = np.array([250, 37], np.int32)
    k = RNG.standard_normal((2, 10, H, d)).astype(np.float32)
    v = RNG.standard_normal((2, 10, H, d)).astype(np.float32)
    assert oracle.append(pool, k, v, bt, sb) == 0
    touched = np.zeros((nb, H, 256), bool)
    for b in range(2):
        for i in range(10):
            pos = sb[b] + i
            blk, slot = bt[b, pos // 256], pos % 256
            for h in range(H):
                ws, wc = np_quant(k[b, i, h], 127)
                assert pool.k_scale[blk, h, slot] == ws
                assert np.array_equal(pool.k[blk, h, slot].astype(np.int64), wc)
                codes = np_unpack_v(pool.v[blk, h, slot])
                for g in range(4):
                    vs, vc = np_quant(v[b, i, h, 32 * g:32 * g + 32], 7)
                    assert pool.v_scale[blk, h, slot, g] == vs
                    assert np.array_equal(codes[32 * g:32 * g + 32], vc)
                touched[blk, h, slot] = True
    # everything else keeps its poison bytes
    for now, old in zip(pool.planes(), before):
        assert np.array_equal(now[~touched], old[~touched])


def test_append_k8v8_quantises_v_by_the_k_rule():
    # int8 KV: V codes and scales equal the numpy statement of the quantiser
    # with the K limit (127), one scale per (token, kv-head), int8 codes
    rng = np.random.default_rng(23)
    H, d, L = 2, 128, 300
    pool = oracle.Pool(oracle.FMT_K8V8, 3, H, d, poison=0x5A)
    bt = np.array([[2, 0]], np.int32)
    k = rng.standard_normal((1, L, H, d)).astype(np.float32)
    v = (rng.standard_normal((1, L, H, d)) * rng.uniform(0.01, 40, (1, L, H, 1))).astype(np.float32)
    v[0, 7, 1] = 0.0                        # a zero vector: scale 0, codes 0
    assert oracle.append(pool, k, v, bt, np.array([0], np.int32)) == 0
    for p_ in range(L):
        blk, slot = bt[0, p_ // 256], p_ % 256
        for h in range(H):
            s16, codes = np_quant(v[0, p_, h], 127)
            assert pool.v_scale[blk, h, slot] == s16
            assert np.array_equal(pool.v[blk, h, slot].astype(np.int64), codes)
            s16k, ck = np_quant(k[0, p_, h], 127)
            assert pool.k_scale[blk, h, slot] == s16k
            assert np.array_equal(pool.k[blk, h, slot].astype(np.int64), ck)
    # untouched slots keep the poison
    assert np.all(pool.v[1].view(np.uint8) == 0x5A) and np.all(pool.v[0, :, 300 - 256:].view(np.uint8) == 0x5A)


def test_e4m3_decode_matches_torch_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    got = oracle.e4m3_bits_to_f64(codes)
    ref = torch_e4m3(codes)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    fin = ~np.isnan(ref)
    assert np.array_equal(got[fin], ref[fin])
    assert np.array_equal(np.signbit(got[fin]), np.signbit(ref[fin]))
    # the largest finite value and the smallest subnormal
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and got[0xFE] == -448.0


def test_e4m3_encode_is_the_nearest_code():
    codes, vals = e4m3_table()
    pos = np.unique(vals[vals > 0])
    mids = (pos[:-1] + pos[1:]) / 2                     # exact ties (representable in fp32)
    nudge = np.concatenate([np.nextafter(mids.astype(np.float32), np.float32(0)),
                            np.nextafter(mids.astype(np.float32), np.float32(1e9))])
    rnd = np.exp(RNG.uniform(np.log(1e-4), np.log(600.0), 4000)).astype(np.float32)
    x = np.concatenate([mids.astype(np.float32), nudge, rnd, pos.astype(np.float32),
                        np.float32([0.0, 1e-6, 2.0 ** -10, 448.0, 449.0, 463.9, 464.0, 500.0, 1e30])])
    x = np.concatenate([x, -x, np.float32([-0.0, -1e-7])])
    got = oracle.f32_to_e4m3_bits(x)
    ref = brute_e4m3(x)
    bad = np.flatnonzero(got != ref)
    assert bad.size == 0, f"{bad.size} mismatches, e.g. x={x[bad[:4]]} got={got[bad[:4]]} ref={ref[bad[:4]]}"


def test_e4m3_encode_matches_torch_cast_in_range():
    # torch's own fp32 -> float8_e4m3fn cast (round half to even) inside +-448
    x = np.concatenate([RNG.uniform(-448, 448, 20000), RNG.standard_normal(20000) * 0.01]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.f32_to_e4m3_bits(x), ref)


def test_quant_f8_matches_numpy_statement_and_error_bound():
    for trial in range(200):
        mag = 10.0 ** RNG.uniform(-6, 4)
        x = (RNG.standard_normal(128) * mag).astype(np.float32)
        if trial % 7 == 0:
            x[RNG.integers(128)] *= 50.0                    # an outlier channel
        if trial == 3:
            x[:] = 0.0
        s16, codes = oracle.quant_f8(x)
        a = np.max(np.abs(x)).astype(np.float32)
        ref_s = np_f16_sat(np.float32(a) / np.float32(448.0))
        assert s16 == ref_s.view(np.uint16)
        sig = np.float32(ref_s)
        if sig == 0:
            assert np.all(codes == 0)
            continue
        assert np.array_equal(codes, brute_e4m3(np.clip(x / sig, -448, 448)))
        # dequantised error of the values x / scale does not clamp: half a step
        # of 3 mantissa bits, or half the subnormal spacing 2^-9, times the
        # scale; clamped values (a scale rounded below absmax / 448, e.g. in the
        # fp16 subnormal range) err by their excess over 448 scales
        err = np.abs(torch_e4m3(codes) * np.float64(sig) - x.astype(np.float64))
        t = np.abs(x.astype(np.float64)) / np.float64(sig)
        unclamped = t <= 448.0
        bound = np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10 * np.float64(sig)) * (1 + 1e-6)
        assert np.all(err[unclamped] <= bound[unclamped])
        assert np.all(err[~unclamped] <= (t[~unclamped] - 448.0) * np.float64(sig) * (1 + 1e-6) + 1e-30)
        if 2.0 ** -14 <= a / 448:                           # a normal fp16 scale: nothing clamps
            assert unclamped.all() or np.max(t) < 448.0 * (1 + 2.0 ** -11)


def test_append_f8_quantises_k_and_v():
    rng = np.random.default_rng(29)
    H, d, L = 2, 128, 260
    pool = oracle.Pool(oracle.FMT_F8, 2, H, d, poison=0x5A)
    bt = np.array([[1, 0]], np.int32)
    k = (rng.standard_normal((1, L, H, d)) * rng.uniform(0.001, 30, (1, L, H, 1))).astype(np.float32)
    v = (rng.standard_normal((1, L, H, d)) * rng.uniform(0.001, 30, (1, L, H, 1))).astype(np.float32)
    v[0, 5, 0] = 0.0
    assert oracle.append(pool, k, v, bt, np.array([0], np.int32)) == 0
    for p_ in range(L):
        blk, slot = bt[0, p_ // 256], p_ % 256
        for h in range(H):
            for src, codes, scales in ((k, pool.k, pool.k_scale), (v, pool.v, pool.v_scale)):
                s16, c = oracle.quant_f8(src[0, p_, h])
                assert scales[blk, h, slot] == s16 and np.array_equal(codes[blk, h, slot], c)
    assert np.all(pool.v[0, :, L - 256:].view(np.uint8) == 0x5A)


def test_append_rejects_out_of_range():
    pool = oracle.Pool(oracle.FMT_K8V4, 2, 1, 128)
    k = np.zeros((1, 1, 1, 128), np.float32)
    assert oracle.append(pool, k, k, np.array([[0, 7]], np.int32), np.array([256], np.int32)) == -1
    assert oracle.append(pool, k, k, np.array([[0, 1]], np.int32), np.array([512], np.int32)) == -1


# ------------------------------------------------------------- attention
SCALE = float(np.float32(1 / math.sqrt(128)))


@pytest.mark.parametrize("fmt", [oracle.FMT_K8V4, oracle.FMT_BF16, oracle.FMT_K8V8, oracle.FMT_F8, oracle.FMT_K4V4])
def test_attention_zero_query_is_mean_of_visible_values(fmt):
    # q = 0 -> all scores 0 -> o = mean of visible v_hat, lse = log(#visible).
    # Causal with n_q = 4: query j sees L - 4 + j + 1 keys.
    cached = [517, 300]
    pool, bt, _, _ = make_pool(fmt, cached, H=2, seed=3)
    _, vh = np_dequant_pool(pool)
    q = np.zeros((2, 4, 4, 128))
    for causal in (False, True):
        out, lse = oracle.decode_attn(pool, q, bt, cached, SCALE, causal)
        out = out.reshape(2, 4, 4, 128)
        lse = lse.reshape(2, 4, 4)
        for b, L in enumerate(cached):
            pos = np.arange(L)
            for h in range(4):
                V = vh[bt[b, pos // 256], h // 2, pos % 256]
                for j in range(4):
                    n = L - 4 + j + 1 if causal else L
                    assert np.allclose(out[b, j, h], V[:n].mean(0), rtol=0, atol=1e-12)
                    assert lse[b, j, h] == pytest.approx(math.log(n), abs=1e-12)


def test_attention_single_key_and_two_key_closed_forms():
    pool, bt, _, _ = make_pool(oracle.FMT_K8V4, [2], H=1, seed=5)
    kh, vh = np_dequant_pool(pool)
    blk = bt[0, 0]
    k0, k1 = kh[blk, 0, 0], kh[blk, 0, 1]
    v0, v1 = vh[blk, 0, 0], vh[blk, 0, 1]
    q = RNG.standard_normal(128)
    # one key: o = v0 exactly, lse = s0
    o, lse = oracle.attn_row(pool, bt[0], 0, 1, q, 0, SCALE)
    assert np.array_equal(o, v0)
    assert lse == pytest.approx(SCALE * float(q @ k0), rel=1e-13, abs=1e-13)
    # two keys: weight of key 0 is the logistic function of s0 - s1
    o, lse = oracle.attn_row(pool, bt[0], 0, 2, q, 0, SCALE)
    s0, s1 = SCALE * float(q @ k0), SCALE * float(q @ k1)
    w0 = 1.0 / (1.0 + math.exp(s1 - s0))
    assert np.allclose(o, w0 * v0 + (1 - w0) * v1, rtol=1e-12, atol=1e-13)
    assert lse == pytest.approx(max(s0, s1) + math.log1p(math.exp(-abs(s0 - s1))), abs=1e-12)
    # key order within the range does not matter, and the two keys are not interchangeable
    o_rev, _ = oracle.attn_row(pool, bt[0], 1, 2, q, 0, SCALE)
    assert np.array_equal(o_rev, v1)


def test_attention_uniform_scores_return_mean_value():
    # every key identical -> every score identical -> o = mean(v_hat) for any q
    H, L = 1, 300
    pool = oracle.Pool(oracle.FMT_K8V4, 2, H, 128)
    kvec = RNG.standard_normal(128).astype(np.float32)
    k = np.broadcast_to(kvec, (1, L, H, 128)).copy()
    v = RNG.standard_normal((1, L, H, 128)).astype(np.float32)
    bt = np.array([[1, 0]], np.int32)
    oracle.append(pool, k, v, bt, np.array([0], np.int32))
    _, vh = np_dequant_pool(pool)
    pos = np.arange(L)
    V = vh[bt[0, pos // 256], 0, pos % 256]
    q = RNG.standard_normal((1, 1, 1, 128)) * 3
    out, _ = oracle.decode_attn(pool, q, bt, [L], SCALE, False)
    assert np.allclose(out[0], V.mean(0), rtol=0, atol=1e-12)


def test_attention_gqa_head_mapping():
    # kv-heads carry different values; q head h must read kv-head h // G
    pool, bt, _, _ = make_pool(oracle.FMT_K8V4, [40], H=3, seed=9)
    _, vh = np_dequant_pool(pool)
    q = np.zeros((1, 1, 6, 128))
    out, _ = oracle.decode_attn(pool, q, bt, [40], SCALE, False)
    for h in range(6):
        assert np.allclose(out[h], vh[bt[0, 0], h // 2, :40].mean(0), atol=1e-12)
        assert not np.allclose(out[h], vh[bt[0, 0], (h // 2 + 1) % 3, :40].mean(0), atol=1e-6)


def test_attention_block_permutation_invariance():
    cached = [700]
    pool, bt, _, _ = make_pool(oracle.FMT_K8V4, cached, H=2, seed=11, nb_extra=2)
    q = RNG.standard_normal((1, 1, 4, 128))
    out1, lse1 = oracle.decode_attn(pool, q, bt, cached, SCALE, False)
    perm = RNG.permutation(pool.num_blocks)
    pool2 = oracle.Pool(oracle.FMT_K8V4, pool.num_blocks, 2, 128)
    for a_new, a_old in zip(pool2.planes(), pool.planes()):
        a_new[perm] = a_old
    bt2 = np.where(bt >= 0, perm[np.maximum(bt, 0)], -1).astype(np.int32)
    out2, lse2 = oracle.decode_attn(pool2, q, bt2, cached, SCALE, False)
    assert np.array_equal(out1, out2) and np.array_equal(lse1, lse2)


def test_attention_split_and_combine_equals_whole():
    pool, bt, _, _ = make_pool(oracle.FMT_K8V4, [1000], H=1, seed=13)
    q = RNG.standard_normal(128) * 2
    whole, lse_w = oracle.attn_row(pool, bt[0], 0, 1000, q, 0, SCALE)
    cuts = [0, 1, 255, 256, 600, 1000]
    parts = [oracle.attn_row(pool, bt[0], a, b, q, 0, SCALE) for a, b in zip(cuts[:-1], cuts[1:])]
    po = np.stack([p[0] for p in parts])[:, None, :]
    pl = np.array([p[1] for p in parts])[:, None]
    o, lse = oracle.combine(po, pl)
    assert np.allclose(o[0], whole, rtol=1e-12, atol=1e-14)
    assert lse[0] == pytest.approx(lse_w, abs=1e-12)


@pytest.mark.parametrize("fmt", [oracle.FMT_K8V4, oracle.FMT_BF16, oracle.FMT_K8V8, oracle.FMT_F8, oracle.FMT_K4V4])
@pytest.mark.parametrize("causal", [False, True])
def test_attention_matches_numpy_brute_force(fmt, causal):
    cached = [300, 513]
    pool, bt, _, _ = make_pool(fmt, cached, H=2, seed=17, k_scale_mul=2.0)
    q = RNG.standard_normal((2, 3, 10, 128)).astype(np.float32)
    q[:, :, :, :4] *= 5
    out, lse = oracle.decode_attn(pool, q, bt, cached, SCALE, causal, nthreads=2)
    want, want_lse = np_attention(pool, bt, cached, q, SCALE, causal)
    assert np.allclose(out, want, rtol=1e-11, atol=1e-13)
    assert np.allclose(lse, want_lse, rtol=1e-12, atol=1e-12)
    # a subset of rows gives the same numbers as the full run
    rows = np.array([0, 7, 59], np.int64)
    o2, l2 = oracle.decode_attn(pool, q, bt, cached, SCALE, causal, rows=rows)
    assert np.array_equal(o2, out[rows]) and np.array_equal(l2, lse[rows])


@pytest.mark.parametrize("n_q", [160, 37])
def test_attention_prefill_chunk_matches_torch_sdpa(n_q):
    # a prefill chunk (many causal queries, the last n_q positions; n_q = L is
    # a whole prompt) against torch's own scaled_dot_product_attention in fp64
    # over the numpy-dequantised pool, the causal mask stated as positions
    L = 160
    pool, bt, _, _ = make_pool(oracle.FMT_K8V4, [L], H=2, seed=31)
    q = RNG.standard_normal((1, n_q, 4, 128)).astype(np.float32)
    out, lse = oracle.decode_attn(pool, q, bt, [L], SCALE, True, nthreads=2)
    kh, vh = np_dequant_pool(pool)
    pos = np.arange(L)
    K = torch.from_numpy(kh[bt[0, pos // 256], :, pos % 256].transpose(1, 0, 2).copy())   # [H_kv][L][d]
    V = torch.from_numpy(vh[bt[0, pos // 256], :, pos % 256].transpose(1, 0, 2).copy())
    K, V = K.repeat_interleave(2, dim=0), V.repeat_interleave(2, dim=0)                    # GQA 2
    Q = torch.from_numpy(q[0].astype(np.float64)).transpose(0, 1)                          # [H_q][n_q][d]
    qpos = torch.arange(L - n_q, L)[:, None]
    mask = torch.arange(L)[None, :] <= qpos                                                # True = attend
    ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=mask,
                                                           scale=float(np.float32(SCALE)))
    assert np.allclose(out.reshape(n_q, 4, 128), ref.transpose(0, 1).numpy(), rtol=1e-10, atol=1e-12)


def test_attention_softmax_scale_is_used():
    # doubling q and halving the scale leaves every score, hence o, unchanged;
    # a different scale changes o
    pool, bt, _, _ = make_pool(oracle.FMT_K8V4, [90], H=1, seed=19)
    q = RNG.standard_normal((1, 1, 1, 128))
    a, _ = oracle.decode_attn(pool, q, bt, [90], 0.25, False)
    b, _ = oracle.decode_attn(pool, 2 * q, bt, [90], 0.125, False)
    c, _ = oracle.decode_attn(pool, q, bt, [90], 0.5, False)
    assert np.allclose(a, b, rtol=1e-13, atol=1e-14)
    assert not np.allclose(a, c, atol=1e-6)


def test_attention_rejects_short_sequence():
    pool, bt, _, _ = make_pool(oracle.FMT_K8V4, [3], H=1, seed=2)
    with pytest.raises(ValueError):
        oracle.decode_attn(pool, np.zeros((1, 4, 1, 128)), bt, [3], SCALE, True)


# ---------------------------------------------------------------- combine
def test_combine_identity_and_skips_empty_splits():
    rows, d = 5, 128
    o = RNG.standard_normal((1, rows, d))
    lse = RNG.standard_normal((1, rows))
    out, l2 = oracle.combine(o, lse)
    assert np.array_equal(out, o[0]) and np.allclose(l2, lse[0], atol=1e-15)
    # adding a split with lse = -inf (and garbage o) changes nothing
    o2 = np.concatenate([o, np.full((1, rows, d), 1e30)])
    lse2 = np.concatenate([lse, np.full((1, rows), -np.inf)])
    out2, l3 = oracle.combine(o2, lse2)
    assert np.array_equal(out2, out) and np.array_equal(l3, l2)
    # every split empty -> o = 0, lse = -inf
    out3, l4 = oracle.combine(np.ones((2, 1, d)), np.full((2, 1), -np.inf))
    assert np.all(out3 == 0) and l4[0] == -np.inf


def test_combine_weights_two_splits():
    # two splits with lse a and b: weights exp(a)/(exp(a)+exp(b)) and the rest
    o = RNG.standard_normal((2, 1, 128))
    a, b = 0.3, -1.7
    out, lse = oracle.combine(o, np.array([[a], [b]]))
    wa = 1 / (1 + math.exp(b - a))
    assert np.allclose(out[0], wa * o[0, 0] + (1 - wa) * o[1, 0], rtol=1e-13)
    assert lse[0] == pytest.approx(math.log(math.exp(a) + math.exp(b)), abs=1e-14)


# ------------------------------------------------ RK4V4-E8 (format 4)
GOLDEN_E8 = os.path.join(os.path.dirname(__file__), "golden", "k4v4_e8_cases.txt")


def _e8_cases():
    cases = []
    with open(GOLDEN_E8) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            head, tail = line.split("|")
            parts = head.split()
            cases.append((parts[0], parts[1:], tail.split()))
    return cases


@pytest.mark.parametrize("case", _e8_cases(), ids=lambda c: c[0] + ":" + " ".join(c[1][:2]))
def test_quant_e8_golden(case):
    kind, head, tail = case
    x = np.zeros(128, np.float32)
    if kind == "PACK":
        xs = np.array([_parse_val(t) for t in head], np.float32)
        x[:len(xs)] = xs
        _, packed = oracle.quant_e8(x)
        want = np.array([int(t, 16) for t in tail], np.uint8)
        assert np.array_equal(packed[:len(want)], want)
        return
    xs = np.array([_parse_val(t) for t in head[1:]], np.float32)
    x[:len(xs)] = xs
    scales, packed = oracle.quant_e8(x)
    assert int(scales[0]) == int(head[0])
    codes = np_unpack_v(packed)
    want = np.array([int(t) for t in tail], np.int64)
    assert np.array_equal(codes[:len(want)], want)
    assert np.all(codes[len(want):32] == 0)


def np_quant_e8(x):
    """Independent statement of the format: the exponent by searching all
    powers of two 2^-126 .. 2^127 for the smallest one >= fp32(absmax / 7),
    the codes by numpy fp32 division and rint.  Returns (bytes[4], codes[128])."""
    x = np.asarray(x, np.float32)
    pows = 2.0 ** np.arange(-126, 128)
    bytes_, codes = [], []
    for g in range(4):
        xg = x[32 * g:32 * g + 32]
        s = np.float32(np.max(np.abs(xg))) / np.float32(7.0)
        e = int(np.arange(-126, 128)[np.argmax(pows >= float(s))]) if s > 0 else -126
        scale = np.float32(2.0 ** e)
        c = np.clip(np.rint(xg / scale), -7, 7).astype(np.int64)
        bytes_.append(e + 127)
        codes.append(c)
    return np.array(bytes_), np.concatenate(codes)


def _e8_vectors(n):
    out = list(_random_vectors(n))
    for i in range(n // 4):  # groups of very different magnitudes in one vector
        x = RNG.standard_normal(128)
        for g in range(4):
            x[32 * g:32 * g + 32] *= 10.0 ** RNG.uniform(-30, 30)
        out.append(x.astype(np.float32))
    for i in range(n // 8):  # subnormal groups: the exponent clamps at -126
        x = RNG.standard_normal(128) * 10.0 ** RNG.uniform(-44, -37)
        out.append(x.astype(np.float32))
    return out


def test_quant_e8_matches_numpy_statement():
    for x in _e8_vectors(2400):
        scales, packed = oracle.quant_e8(x)
        wb, wc = np_quant_e8(x)
        assert np.array_equal(scales.astype(np.int64), wb)
        assert np.array_equal(np_unpack_v(packed), wc)


def test_quant_e8_roundtrip_and_scale_bounds():
    for x in _e8_vectors(1200):
        scales, packed = oracle.quant_e8(x)
        codes = np_unpack_v(packed)
        for g in range(4):
            e = int(scales[g]) - 127
            xg = x[32 * g:32 * g + 32].astype(np.float64)
            s = float(np.float32(np.max(np.abs(x[32 * g:32 * g + 32]))) / np.float32(7.0))
            assert 2.0 ** e >= s                          # no code is clamped ...
            assert e == -126 or 2.0 ** (e - 1) < s        # ... and the scale is the smallest such
            err = np.abs(xg - codes[32 * g:32 * g + 32] * 2.0 ** e)
            assert np.all(err <= 2.0 ** (e - 1))           # half a step
            assert codes.min() >= -7 and codes.max() <= 7


def test_append_k4v4_places_both_planes_through_block_table():
    H, d = 2, 128
    rng = np.random.default_rng(41)
    pool = oracle.Pool(oracle.FMT_K4V4, 3, H, d, poison=0x5A)
    bt = np.array([[2, 0]], np.int32)
    k = rng.standard_normal((1, 300, H, d)).astype(np.float32)
    v = (rng.standard_normal((1, 300, H, d)) * 3).astype(np.float32)
    assert oracle.append(pool, k, v, bt, np.array([0], np.int32)) == 0
    for t in (0, 255, 256, 299):
        blk, slot = bt[0, t // 256], t % 256
        for h in range(H):
            ks, kp = oracle.quant_e8(k[0, t, h])
            vs, vp = oracle.quant_e8(v[0, t, h])
            assert np.array_equal(pool.k[blk, h, slot], kp) and np.array_equal(pool.k_scale[blk, h, slot], ks)
            assert np.array_equal(pool.v[blk, h, slot], vp) and np.array_equal(pool.v_scale[blk, h, slot], vs)
    # slots past the end keep their poison
    assert np.all(pool.k[0, :, 44:] == 0x5A) and np.all(pool.v_scale[0, :, 44:] == 0x5A)
    assert np.all(pool.k[1] == 0x5A)
