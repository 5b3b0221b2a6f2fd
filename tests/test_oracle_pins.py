"""Pins of the CPU oracle against things other than itself.

Each check is chosen so that a plausible slip inside the oracle (a dropped
term, a wrong sign or index, a transposed operand, an off-by-one at a block
boundary, a wrong rounding direction) fails at least one of them:

* number formats: exhaustive against numpy/torch decoders; the E4M3 encoder
  against a brute-force nearest search over all codes and against torch's
  cast;
* addressing: the slot of a position must point at the row a block-wise copy
  (torch/numpy indexing, no slot formula) put that position's data in;
* decode: fp64 torch scaled_dot_product_attention on the contiguous K/V the
  pool was filled from (the unpaged definition), permutation invariance,
  shared-prefix == private copies, closed forms (one token, equal keys, a
  dominant key, hand cases at block boundaries), partition-combine identity;
* reshape_and_cache: torch-view reads of the written rows, untouched rows keep
  a sentinel, FP8 codes equal torch's rounding of x/scale.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle.block_manager import BlockManager, OutOfBlocks
from paged_kv_cache_448_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def load_golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# --------------------------------------------------------------- helpers

def to_f64(codes, dt):
    """Independent decoder (numpy/torch) of raw codes to fp64."""
    codes = np.ascontiguousarray(codes)
    if dt == "f16":
        return codes.view(np.float16).astype(np.float64)
    if dt == "bf16":
        return torch.from_numpy(codes.view(np.int16)).view(torch.bfloat16).double().numpy()
    if dt == "e4m3":
        return torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    raise ValueError(dt)


def from_f32(x, dt):
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dt == "f16":
        with np.errstate(over="ignore"):
            return x.astype(np.float16).view(np.uint16)
    if dt == "bf16":
        return torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    raise ValueError(dt)


def random_e4m3_codes(rng, shape):
    c = rng.integers(0, 256, size=shape).astype(np.uint8)
    c[(c & 0x7F) == 0x7F] = 0x3C  # no NaN codes
    return c


def build_paged(rng, contig_k, contig_v, ctxs, bs, spare=5):
    """Scatter per-sequence contiguous K/V ([n, Hkv, D] raw codes) into a
    block pool with a random permutation, block by block (numpy indexing
    only). Returns (key_cache, value_cache, block_table)."""
    nblk = [-(-n // bs) for n in ctxs]
    NB = sum(nblk) + spare
    perm = rng.permutation(NB)
    Hkv, D = contig_k[0].shape[1:]
    dt = contig_k[0].dtype
    kc = np.zeros((NB, bs, Hkv, D), dt)
    vc = np.zeros((NB, bs, Hkv, D), dt)
    table = np.full((len(ctxs), max(1, max(nblk))), -1, np.int32)
    cur = 0
    for s, n in enumerate(ctxs):
        for j in range(nblk[s]):
            b = int(perm[cur]); cur += 1
            table[s, j] = b
            rows = slice(j * bs, min(n, (j + 1) * bs))
            cnt = rows.stop - rows.start
            kc[b, :cnt] = contig_k[s][rows]
            vc[b, :cnt] = contig_v[s][rows]
    return kc, vc, table


def sdpa_reference(q, Ks, Vs, scale, group):
    """fp64 torch SDPA per sequence on contiguous K/V (unpaged attention)."""
    outs = []
    for s in range(len(Ks)):
        qs = torch.from_numpy(q[s]).unsqueeze(1)                       # [H, 1, D]
        k = torch.from_numpy(Ks[s]).permute(1, 0, 2).repeat_interleave(group, 0)  # [H, n, D]
        v = torch.from_numpy(Vs[s]).permute(1, 0, 2).repeat_interleave(group, 0)
        if k.shape[1] == 0:
            outs.append(np.zeros_like(q[s]))
            continue
        o = torch.nn.functional.scaled_dot_product_attention(qs, k, v, scale=scale)
        outs.append(o.squeeze(1).numpy())
    return np.stack(outs)


# ---------------------------------------------------------- number formats

def test_f16_decoder_exhaustive():
    codes = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.decode_array(codes, "f16")
    ref = to_f64(codes, "f16")
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    m = ~np.isnan(ref)
    assert np.array_equal(ours[m], ref[m])
    assert np.array_equal(np.signbit(ours[m]), np.signbit(ref[m]))


def test_bf16_decoder_exhaustive():
    codes = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.decode_array(codes, "bf16")
    ref = to_f64(codes, "bf16")
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    m = ~np.isnan(ref)
    assert np.array_equal(ours[m], ref[m])
    assert np.array_equal(np.signbit(ours[m]), np.signbit(ref[m]))


def test_e4m3_decoder_exhaustive():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.decode_array(codes, "e4m3")
    ref = to_f64(codes, "e4m3")
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    assert np.isnan(ours[0x7F]) and np.isnan(ours[0xFF])
    m = ~np.isnan(ref)
    assert np.array_equal(ours[m], ref[m])
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9


def test_e4m3_encoder_roundtrip_all_codes():
    for c in range(256):
        if (c & 0x7F) == 0x7F:
            continue
        v = oracle.decode_e4m3(c)
        assert oracle.encode_e4m3(v) == c, hex(c)


def _e4m3_sweep(rng):
    mags = to_f64(np.arange(0x7F, dtype=np.uint8), "e4m3")        # codes 0..126 ascending
    mids = (mags[1:] + mags[:-1]) / 2
    mids32 = mids.astype(np.float32)
    assert np.array_equal(mids32.astype(np.float64), mids)        # midpoints exact in fp32
    pts = [np.linspace(-500, 500, 100001, dtype=np.float32), mids32, -mids32,
           np.nextafter(mids32, np.float32(np.inf)), np.nextafter(mids32, np.float32(0)),
           (2.0 ** rng.uniform(-14, 9.5, 50000)).astype(np.float32),
           np.array([0.0, -0.0, 448.0, 449.0, 464.0, 479.9, 480.0, 1e30, -1e30, 2.0 ** -10,
                     2.0 ** -11, 3 * 2.0 ** -11], np.float32)]
    return mags, np.concatenate(pts)


def test_e4m3_encoder_is_nearest_even_saturating():
    """Brute force: nearest of the 127 finite magnitudes, ties to the even
    code, |x| >= 448 saturates; sign from the sign bit."""
    rng = np.random.default_rng(5)
    mags, xs = _e4m3_sweep(rng)
    a = np.abs(xs.astype(np.float64))
    expect = np.empty(len(xs), np.int64)
    for i0 in range(0, len(xs), 20000):
        blk = a[i0:i0 + 20000]
        d = np.abs(blk[:, None] - mags[None, :])
        best = d.min(axis=1, keepdims=True)
        cand = d == best
        codes = np.arange(127)[None, :]
        # among equally near codes prefer the even one
        pick = np.where(cand & (codes % 2 == 0), codes, 10 ** 6).min(axis=1)
        pick = np.where(pick == 10 ** 6, np.where(cand, codes, 10 ** 6).min(axis=1), pick)
        expect[i0:i0 + 20000] = pick
    expect[a >= 448.0] = 0x7E
    expect |= np.where(np.signbit(xs), 0x80, 0)
    ours = np.array([oracle.encode_e4m3(float(x)) for x in xs])
    bad = np.nonzero(ours != expect)[0]
    assert len(bad) == 0, [(float(xs[i]), hex(ours[i]), hex(expect[i])) for i in bad[:5]]


def test_e4m3_encoder_matches_torch_cast_in_range():
    rng = np.random.default_rng(6)
    _, xs = _e4m3_sweep(rng)
    xs = xs[np.abs(xs) <= 464.0]          # torch does not saturate above that
    ref = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = np.array([oracle.encode_e4m3(float(x)) for x in xs], dtype=np.uint8)
    # torch maps -x that rounds to zero to 0x80 as well
    assert np.array_equal(ours, ref)


@pytest.mark.parametrize("dt", ["f16", "bf16"])
def test_16bit_encoders_match_library_rounding(dt):
    rng = np.random.default_rng(7)
    x = np.concatenate([rng.standard_normal(20000).astype(np.float32) * 1000,
                        (2.0 ** rng.uniform(-30, 17, 20000)).astype(np.float32),
                        np.array([65504, 65519, 65520, 7e4, 2 ** -24, 2 ** -25, 3 * 2 ** -26,
                                  1e-45], np.float32)])
    ours = np.array([oracle.encode_f16(float(v)) if dt == "f16" else oracle.encode_bf16(float(v))
                     for v in x], dtype=np.uint16)
    assert np.array_equal(ours, from_f32(x, dt))


def test_fp32_division_is_ieee_single():
    rng = np.random.default_rng(8)
    a = rng.standard_normal(5000).astype(np.float32)
    b = (rng.uniform(0.001, 0.02, 5000)).astype(np.float32)
    ours = np.array([oracle.div_f32(float(x), float(y)) for x, y in zip(a, b)], np.float32)
    assert np.array_equal(ours, a / b)


# -------------------------------------------------------------- addressing

def _marker_pool(table, bs, nb, n_pos):
    """Block-wise copy of a marker sequence (value = position) into a pool
    of nb blocks following `table` (numpy indexing, no slot arithmetic)."""
    pool = np.full((nb, bs), -7, np.int64)
    marks = np.arange(len(table) * bs, dtype=np.int64)
    for j, b in enumerate(table):
        pool[b] = marks[j * bs:(j + 1) * bs]
    return pool.reshape(-1)


def test_slot_translation_hand_example():
    g = load_golden("hand_cases.json")["slot_translation"]
    bs, table, pos = g["block_size"], g["block_table"], g["positions"]
    slots = oracle.slot_mapping(np.array([table], np.int32), np.array(pos, np.int32), bs,
                                seq_ids=np.zeros(len(pos), np.int32))
    rows = _marker_pool(table, bs, max(table) + 1, len(pos))
    assert [int(rows[s]) for s in slots] == pos


def test_slot_translation_random_tables():
    rng = np.random.default_rng(9)
    for bs in (16, 32):
        S, mb = 7, 9
        nb = S * mb + 3
        perm = rng.permutation(nb)[:S * mb].reshape(S, mb).astype(np.int32)
        seq = rng.integers(0, S, 300).astype(np.int32)
        pos = rng.integers(0, mb * bs, 300).astype(np.int32)
        pos[::17] = -1
        slots = oracle.slot_mapping(perm, pos, bs, seq_ids=seq)
        for i in range(300):
            if pos[i] < 0:
                assert slots[i] == -1
                continue
            rows = _marker_pool(perm[seq[i]], bs, nb, 0)
            assert rows[slots[i]] == pos[i]


def test_slot_translation_rejects_bad_tables():
    t = np.array([[3, -1]], np.int32)
    with pytest.raises(ValueError):
        oracle.slot_mapping(t, np.array([16], np.int32), 16)      # entry -1
    with pytest.raises(ValueError):
        oracle.slot_mapping(t, np.array([32], np.int32), 16)      # past the table


# ------------------------------------------------------- reshape_and_cache

@pytest.mark.parametrize("dt", ["f16", "bf16"])
def test_reshape_and_cache_copies_rows(dt):
    rng = np.random.default_rng(10)
    T, Hkv, D, bs, NB = 37, 3, 64, 16, 11
    key = from_f32(rng.standard_normal((T, Hkv, D)), dt)
    val = from_f32(rng.standard_normal((T, Hkv, D)), dt)
    slots = rng.permutation(NB * bs)[:T].astype(np.int32)
    slots[5] = -1
    kc = np.full((NB, bs, Hkv, D), 0xA5A5, np.uint16)
    vc = np.full((NB, bs, Hkv, D), 0x5A5A, np.uint16)
    oracle.reshape_and_cache(key, val, kc, vc, slots, block_size=bs, kv_dtype=dt, cache_dtype=dt)
    krows, vrows = kc.reshape(NB * bs, Hkv, D), vc.reshape(NB * bs, Hkv, D)
    written = np.zeros(NB * bs, bool)
    for n in range(T):
        if slots[n] < 0:
            continue
        written[slots[n]] = True
        assert np.array_equal(krows[slots[n]], key[n])
        assert np.array_equal(vrows[slots[n]], val[n])
    assert np.all(krows[~written] == 0xA5A5) and np.all(vrows[~written] == 0x5A5A)


def test_reshape_and_cache_fp8_matches_torch_rounding():
    rng = np.random.default_rng(11)
    T, Hkv, D, bs, NB = 20, 4, 128, 16, 6
    xk = rng.standard_normal((T, Hkv, D)).astype(np.float32) * 3
    xv = rng.standard_normal((T, Hkv, D)).astype(np.float32) * 3
    key, val = from_f32(xk, "bf16"), from_f32(xv, "bf16")
    ks = (np.abs(to_f64(key, "bf16")).max(axis=(0, 2)) / 448.0 * 0.9).astype(np.float32)
    vs = (np.abs(to_f64(val, "bf16")).max(axis=(0, 2)) / 448.0 * 1.1).astype(np.float32)
    slots = rng.permutation(NB * bs)[:T].astype(np.int32)
    kc = np.full((NB, bs, Hkv, D), 0x11, np.uint8)
    vc = np.full((NB, bs, Hkv, D), 0x22, np.uint8)
    oracle.reshape_and_cache(key, val, kc, vc, slots, block_size=bs, kv_dtype="bf16",
                             cache_dtype="e4m3", k_scale=ks, v_scale=vs)
    kx = torch.from_numpy(to_f64(key, "bf16").astype(np.float32))
    vx = torch.from_numpy(to_f64(val, "bf16").astype(np.float32))
    qk = kx / torch.from_numpy(ks).view(1, -1, 1)
    qv = vx / torch.from_numpy(vs).view(1, -1, 1)
    ek = qk.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ev = qv.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    # k scaled by 0.9: some |x/scale| exceed 448 -> saturate (torch gives NaN there)
    sat = np.abs(qk.numpy()) > 464
    ek = np.where(sat, np.where(qk.numpy() < 0, 0xFE, 0x7E), ek)
    assert sat.any()
    krows, vrows = kc.reshape(NB * bs, Hkv, D), vc.reshape(NB * bs, Hkv, D)
    for n in range(T):
        assert np.array_equal(krows[slots[n]], ek[n])
        assert np.array_equal(vrows[slots[n]], ev[n])


def test_reshape_and_cache_rejects_bad_slots():
    key = np.zeros((2, 1, 64), np.uint16)
    kc = np.zeros((2, 16, 1, 64), np.uint16)
    with pytest.raises(ValueError):
        oracle.reshape_and_cache(key, key, kc, kc.copy(), np.array([3, 3], np.int32),
                                 block_size=16, kv_dtype="f16", cache_dtype="f16")
    with pytest.raises(ValueError):
        oracle.reshape_and_cache(key, key, kc, kc.copy(), np.array([3, 32], np.int32),
                                 block_size=16, kv_dtype="f16", cache_dtype="f16")


# ------------------------------------------------------------------ decode

DECODE_CASES = [
    # (q/cache dtype, H, Hkv, D, bs, contexts)
    ("f16", "f16", 4, 4, 64, 16, [1, 17, 33, 100]),
    ("bf16", "bf16", 6, 2, 128, 32, [31, 32, 33, 64, 65, 5]),
    ("f16", "f16", 8, 1, 64, 16, [15, 16, 48, 0, 3]),
    ("bf16", "e4m3", 8, 2, 128, 16, [1, 50, 160]),
    ("f16", "e4m3", 4, 4, 64, 32, [40, 7]),
]


@pytest.mark.parametrize("qdt,cdt,H,Hkv,D,bs,ctxs", DECODE_CASES)
def test_decode_equals_unpaged_sdpa(qdt, cdt, H, Hkv, D, bs, ctxs):
    rng = np.random.default_rng(12 + H + D + bs)
    S = len(ctxs)
    q = from_f32(rng.standard_normal((S, H, D)), qdt)
    if cdt == "e4m3":
        Kc = [random_e4m3_codes(rng, (n, Hkv, D)) for n in ctxs]
        Vc = [random_e4m3_codes(rng, (n, Hkv, D)) for n in ctxs]
        ks = rng.uniform(0.001, 0.01, Hkv).astype(np.float32)
        vs = rng.uniform(0.001, 0.01, Hkv).astype(np.float32)
    else:
        Kc = [from_f32(rng.standard_normal((n, Hkv, D)), cdt) for n in ctxs]
        Vc = [from_f32(rng.standard_normal((n, Hkv, D)), cdt) for n in ctxs]
        ks = vs = None
    kc, vc, table = build_paged(rng, Kc, Vc, ctxs, bs)
    scale = 1.0 / math.sqrt(D)
    ours = oracle.decode(q, kc, vc, table, np.array(ctxs, np.int32), scale=np.float32(scale),
                         q_dtype=qdt, cache_dtype=cdt, k_scale=ks, v_scale=vs)
    Kf = [to_f64(k, cdt) * (1.0 if ks is None else ks.astype(np.float64)[None, :, None])
          for k in Kc]
    Vf = [to_f64(v, cdt) * (1.0 if vs is None else vs.astype(np.float64)[None, :, None])
          for v in Vc]
    ref = sdpa_reference(to_f64(q, qdt), Kf, Vf, float(np.float32(scale)), H // Hkv)
    np.testing.assert_allclose(ours, ref, rtol=1e-12, atol=1e-13)


PREFILL_CASES = [
    # (q/cache dtype, H, Hkv, D, bs, contexts, query lengths)
    ("f16", "f16", 4, 4, 64, 16, [17, 40, 5, 33], [17, 9, 1, 16]),
    ("bf16", "bf16", 8, 2, 128, 32, [64, 100, 70], [64, 3, 33]),
    ("bf16", "e4m3", 8, 1, 64, 16, [50, 20], [7, 20]),
]


def _prefill_inputs(qdt, cdt, H, Hkv, D, bs, ctxs, qlens, seed):
    rng = np.random.default_rng(seed)
    T = sum(qlens)
    q = from_f32(rng.standard_normal((T, H, D)), qdt)
    if cdt == "e4m3":
        Kc = [random_e4m3_codes(rng, (n, Hkv, D)) for n in ctxs]
        Vc = [random_e4m3_codes(rng, (n, Hkv, D)) for n in ctxs]
        ks = rng.uniform(0.001, 0.01, Hkv).astype(np.float32)
        vs = rng.uniform(0.001, 0.01, Hkv).astype(np.float32)
    else:
        Kc = [from_f32(rng.standard_normal((n, Hkv, D)), cdt) for n in ctxs]
        Vc = [from_f32(rng.standard_normal((n, Hkv, D)), cdt) for n in ctxs]
        ks = vs = None
    kc, vc, table = build_paged(rng, Kc, Vc, ctxs, bs)
    cu = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    return q, Kc, Vc, ks, vs, kc, vc, table, cu


@pytest.mark.parametrize("qdt,cdt,H,Hkv,D,bs,ctxs,qlens", PREFILL_CASES)
def test_chunked_prefill_equals_masked_sdpa(qdt, cdt, H, Hkv, D, bs, ctxs, qlens):
    """Against fp64 torch SDPA on the contiguous K/V with an explicit boolean
    mask (row i of sequence s sees keys 0 .. ctx - qlen + i); where the chunk
    is the whole context, against SDPA's own is_causal rule as well."""
    q, Kc, Vc, ks, vs, kc, vc, table, cu = _prefill_inputs(qdt, cdt, H, Hkv, D, bs, ctxs, qlens,
                                                          seed=H + D + bs)
    scale = float(np.float32(1.0 / math.sqrt(D)))
    ours = oracle.chunked_prefill(q, kc, vc, table, np.array(ctxs, np.int32), cu,
                                  scale=np.float32(scale), q_dtype=qdt, cache_dtype=cdt,
                                  k_scale=ks, v_scale=vs)
    G = H // Hkv
    qf = to_f64(q, qdt)
    for s, (n, ql) in enumerate(zip(ctxs, qlens)):
        K = to_f64(Kc[s], cdt) * (1.0 if ks is None else ks.astype(np.float64)[None, :, None])
        V = to_f64(Vc[s], cdt) * (1.0 if vs is None else vs.astype(np.float64)[None, :, None])
        k = torch.from_numpy(K).permute(1, 0, 2).repeat_interleave(G, 0)     # [H, n, D]
        v = torch.from_numpy(V).permute(1, 0, 2).repeat_interleave(G, 0)
        qs = torch.from_numpy(qf[cu[s]:cu[s + 1]]).permute(1, 0, 2)         # [H, ql, D]
        pos = torch.arange(n - ql, n)[:, None]
        mask = torch.arange(n)[None, :] <= pos                               # [ql, n]
        ref = torch.nn.functional.scaled_dot_product_attention(qs, k, v, attn_mask=mask,
                                                               scale=scale)
        np.testing.assert_allclose(ours[cu[s]:cu[s + 1]], ref.permute(1, 0, 2).numpy(),
                                   rtol=1e-12, atol=1e-13)
        if ql == n:
            causal = torch.nn.functional.scaled_dot_product_attention(qs, k, v, is_causal=True,
                                                                      scale=scale)
            np.testing.assert_allclose(ours[cu[s]:cu[s + 1]], causal.permute(1, 0, 2).numpy(),
                                       rtol=1e-12, atol=1e-13)


def test_chunked_prefill_with_one_token_per_sequence_is_decode():
    q, Kc, Vc, ks, vs, kc, vc, table, cu = _prefill_inputs("bf16", "bf16", 8, 2, 128, 16,
                                                          [1, 30, 77], [1, 1, 1], seed=4)
    ctx = np.array([1, 30, 77], np.int32)
    a = oracle.chunked_prefill(q, kc, vc, table, ctx, cu, scale=np.float32(0.1), q_dtype="bf16",
                               cache_dtype="bf16")
    b = oracle.decode(q, kc, vc, table, ctx, scale=np.float32(0.1), q_dtype="bf16",
                      cache_dtype="bf16")
    assert np.array_equal(a, b)


def test_chunked_prefill_first_row_of_a_full_chunk_returns_v0():
    q, Kc, Vc, ks, vs, kc, vc, table, cu = _prefill_inputs("f16", "f16", 4, 4, 64, 16,
                                                          [20], [20], seed=8)
    out = oracle.chunked_prefill(q, kc, vc, table, np.array([20], np.int32), cu,
                                 scale=np.float32(0.125), q_dtype="f16", cache_dtype="f16")
    assert np.array_equal(out[0], to_f64(Vc[0][0], "f16"))     # sees only token 0
    with pytest.raises(ValueError):                              # chunk longer than context
        oracle.chunked_prefill(q, kc, vc, table, np.array([19], np.int32), cu,
                               scale=np.float32(0.125), q_dtype="f16", cache_dtype="f16")


def _small_workload(cfg):
    sp = wl.spec(cfg, small=True)
    st = wl.structure(sp)
    return sp, st, wl.host_data(sp, st)


def _decode(sp, st, hd, table=None, kc=None, vc=None, **kw):
    return oracle.decode(hd.query, hd.key_cache if kc is None else kc,
                         hd.value_cache if vc is None else vc,
                         st.block_tables if table is None else table, sp.context_lens,
                         scale=sp.scale, q_dtype=sp.q_dtype, cache_dtype=sp.cache_dtype,
                         k_scale=hd.k_scale, v_scale=hd.v_scale, **kw)


@pytest.mark.parametrize("cfg", [1, 3, 5])
def test_decode_invariant_under_block_permutation(cfg):
    sp, st, hd = _small_workload(cfg)
    base = _decode(sp, st, hd)
    pi = np.random.default_rng(13).permutation(st.num_blocks)
    kc = np.empty_like(hd.key_cache); vc = np.empty_like(hd.value_cache)
    kc[pi] = hd.key_cache; vc[pi] = hd.value_cache
    table = np.where(st.block_tables >= 0, pi[np.maximum(st.block_tables, 0)], -1).astype(np.int32)
    assert np.array_equal(_decode(sp, st, hd, table=table, kc=kc, vc=vc), base)


def test_decode_shared_prefix_equals_private_copies():
    sp, st, hd = _small_workload(5)
    base = _decode(sp, st, hd)
    assert st.refcounts.max() == 4
    shared = np.nonzero(st.refcounts > 1)[0]
    # give every sequence its own copy of each shared block
    extra = []
    table = st.block_tables.copy()
    nb = st.num_blocks
    for s in range(sp.num_seqs):
        for j in range(table.shape[1]):
            b = table[s, j]
            if b >= 0 and b in shared:
                extra.append(b)
                table[s, j] = nb + len(extra) - 1
    kc = np.concatenate([hd.key_cache, hd.key_cache[extra]])
    vc = np.concatenate([hd.value_cache, hd.value_cache[extra]])
    priv = _decode(sp, st, hd, table=table, kc=kc, vc=vc)
    assert np.array_equal(priv, base)


def test_decode_single_token_returns_v0():
    sp, st, hd = _small_workload(1)           # context lengths {1, 17, 33, 100}
    out = _decode(sp, st, hd)
    b0 = st.block_tables[0, 0]
    v0 = to_f64(hd.value_cache[b0, 0], "f16")     # [Hkv, D]
    assert np.array_equal(out[0], v0)


def test_decode_equal_keys_gives_mean_of_values():
    rng = np.random.default_rng(14)
    n, D, bs = 45, 64, 16
    k_row = from_f32(rng.standard_normal((1, 1, D)), "f16")
    Kc = [np.repeat(k_row, n, axis=0)]
    Vc = [from_f32(rng.standard_normal((n, 1, D)), "f16")]
    kc, vc, table = build_paged(rng, Kc, Vc, [n], bs)
    q = from_f32(rng.standard_normal((1, 1, D)), "f16")
    out = oracle.decode(q, kc, vc, table, np.array([n], np.int32), scale=0.3, q_dtype="f16",
                        cache_dtype="f16")
    np.testing.assert_allclose(out[0, 0], to_f64(Vc[0], "f16")[:, 0].mean(axis=0), rtol=0,
                               atol=1e-13)


def test_decode_dominant_key_selects_its_value():
    rng = np.random.default_rng(15)
    n, D, bs = 40, 64, 16
    Kf = rng.standard_normal((n, 1, D)).astype(np.float32) * 0.05
    qf = rng.standard_normal((1, 1, D)).astype(np.float32)
    # scale * q.k_23 = 60 while every other |logit| is ~0.01: weight of the rest < 1e-24
    Kf[23, 0] = qf[0, 0] * (60.0 / (0.02 * float(qf[0, 0] @ qf[0, 0])))
    Kc = [from_f32(Kf, "f16")]
    Vc = [from_f32(rng.standard_normal((n, 1, D)), "f16")]
    kc, vc, table = build_paged(rng, Kc, Vc, [n], bs)
    out = oracle.decode(from_f32(qf, "f16"), kc, vc, table, np.array([n], np.int32), scale=0.02,
                        q_dtype="f16", cache_dtype="f16")
    np.testing.assert_allclose(out[0, 0], to_f64(Vc[0], "f16")[23, 0], rtol=0, atol=1e-12)


def test_decode_zero_context_gives_zeros():
    rng = np.random.default_rng(16)
    Kc = [from_f32(rng.standard_normal((n, 2, 64)), "f16") for n in (0, 5)]
    Vc = [from_f32(rng.standard_normal((n, 2, 64)), "f16") for n in (0, 5)]
    kc, vc, table = build_paged(rng, Kc, Vc, [0, 5], 16)
    q = from_f32(rng.standard_normal((2, 2, 64)), "f16")
    out = oracle.decode(q, kc, vc, table, np.array([0, 5], np.int32), scale=0.125, q_dtype="f16",
                        cache_dtype="f16")
    assert np.all(out[0] == 0.0) and np.all(np.isfinite(out[1]))


def test_decode_hand_two_token_case():
    g = load_golden("hand_cases.json")["two_token"]
    q = np.array(g["q"], np.float32).reshape(1, 1, 4)
    K = np.array(g["k"], np.float32).reshape(2, 1, 4)
    V = np.array(g["v"], np.float32).reshape(2, 1, 4)
    kc, vc, table = build_paged(np.random.default_rng(0), [from_f32(K, "f16")],
                                [from_f32(V, "f16")], [2], g["block_size"])
    out = oracle.decode(from_f32(q, "f16"), kc, vc, table, np.array([2], np.int32),
                        scale=g["scale"], q_dtype="f16", cache_dtype="f16")
    w1 = math.exp(0.5) / (1 + math.exp(0.5))
    expect = (1 - w1) * V[0, 0].astype(np.float64) + w1 * V[1, 0].astype(np.float64)
    np.testing.assert_allclose(out[0, 0], expect, rtol=1e-14, atol=1e-15)


@pytest.mark.parametrize("n", load_golden("hand_cases.json")["block_boundary"]["contexts"])
def test_decode_hand_block_boundary(n):
    g = load_golden("hand_cases.json")["block_boundary"]
    K = np.zeros((n, 1, 4), np.float32)
    K[n - 1, 0, 0] = 1.0
    V = np.stack([np.array([t, 1.0, -t, 0.25], np.float32) for t in range(n)]).reshape(n, 1, 4)
    q = np.array(g["q"], np.float32).reshape(1, 1, 4)
    kc, vc, table = build_paged(np.random.default_rng(n), [from_f32(K, "f16")],
                                [from_f32(V, "f16")], [n], g["block_size"])
    out = oracle.decode(from_f32(q, "f16"), kc, vc, table, np.array([n], np.int32),
                        scale=g["scale"], q_dtype="f16", cache_dtype="f16")
    e = math.e
    V64 = V[:, 0].astype(np.float64)
    expect = (V64[:n - 1].sum(axis=0) + e * V64[n - 1]) / (n - 1 + e)
    np.testing.assert_allclose(out[0, 0], expect, rtol=1e-14, atol=1e-14)


@pytest.mark.parametrize("cfg,P", [(2, 256), (3, 512), (4, 512), (5, 128)])
def test_partition_combine_is_an_identity(cfg, P):
    sp, st, hd = _small_workload(cfg)
    one = _decode(sp, st, hd)
    split = _decode(sp, st, hd, partition_tokens=P)
    np.testing.assert_allclose(split, one, rtol=1e-12, atol=1e-14)


def test_decode_ignores_slots_past_the_context():
    sp, st, hd = _small_workload(3)
    base = _decode(sp, st, hd)
    kc, vc = hd.key_cache.copy(), hd.value_cache.copy()
    bs = sp.block_size
    for s, n in enumerate(sp.context_lens):
        if n % bs:
            b = st.block_tables[s, n // bs]
            kc[b, n % bs:] = 0x7FC0        # bf16 NaN
            vc[b, n % bs:] = 0xFF80        # bf16 -inf
    assert np.array_equal(_decode(sp, st, hd, kc=kc, vc=vc), base)


# ---------------------------------------------------- allocator (oracle model)

def test_block_manager_fifo_and_oom_all_or_nothing():
    bm = BlockManager(6, initial_free_order=[4, 1, 5, 0, 3, 2])
    assert bm.allocate(2) == [4, 1]
    assert bm.allocate(3) == [5, 0, 3]
    with pytest.raises(OutOfBlocks):
        bm.allocate(2)
    assert bm.free_blocks == [2]
    bm.free([0, 4])
    assert bm.free_blocks == [2, 0, 4]
    assert bm.allocate(3) == [2, 0, 4]


def test_block_manager_refcounted_sharing():
    bm = BlockManager(4)
    ids = bm.allocate(2)
    for _ in range(3):
        bm.share(ids[0])                 # four sequences reference the prefix block
    bm.free([ids[0]] * 3)
    assert bm.num_free() == 2 and bm.refcount[ids[0]] == 1
    bm.free(ids)
    assert bm.num_free() == 4 and bm.free_blocks[-2:] == ids
    with pytest.raises(ValueError):
        bm.free([ids[1]])                # already free: nothing changes
    assert bm.num_free() == 4


def test_block_manager_copy_on_write():
    bm = BlockManager(5, initial_free_order=[3, 0, 4, 1, 2])
    a, b = bm.allocate(2)                  # 3, 0
    assert bm.copy_on_write(a) == (a, False)          # sole holder writes in place
    bm.share(b); bm.share(b)               # three holders
    new, copy = bm.copy_on_write(b)
    assert (new, copy) == (4, True)        # head of the free list
    assert bm.refcount[b] == 2 and bm.refcount[new] == 1 and bm.free_blocks == [1, 2]
    bm.allocate(2)
    with pytest.raises(OutOfBlocks):
        bm.copy_on_write(b)                # nothing changes on failure
    assert bm.refcount[b] == 2 and bm.free_blocks == []
    with pytest.raises(ValueError):
        BlockManager(2).copy_on_write(0)   # a free block has no holder


def test_copy_blocks_hand_example():
    src = np.arange(4 * 3, dtype=np.uint16).reshape(4, 3)
    dst = np.full((5, 3), 7, np.uint16)
    oracle.copy_blocks(src, dst, [(0, 2), (3, 0)])
    assert dst.tolist() == [[9, 10, 11], [7, 7, 7], [0, 1, 2], [7, 7, 7], [7, 7, 7]]
    with pytest.raises(AssertionError):
        oracle.copy_blocks(src, src, [(0, 1), (1, 2)])   # 1 is read and written
    with pytest.raises(AssertionError):
        oracle.copy_blocks(src, dst, [(0, 1), (2, 1)])   # two writers of block 1


def _manager_for(st, sp):
    """A BlockManager driven through the same allocations as the workload
    structure (prefix blocks once per group, then shared by every member)."""
    bm = BlockManager(st.num_blocks, initial_free_order=st.free_order)
    tables = []
    pblk = sp.prefix_tokens // sp.block_size
    per = sp.num_seqs // sp.shared_groups
    for g in range(sp.shared_groups):
        prefix = bm.allocate(pblk)
        for _ in range(per - 1):
            for b in prefix:
                bm.share(b)
        for j in range(per):
            s = g * per + j
            tables.append(prefix + bm.allocate(len(st.seq_block_ids[s]) - pblk))
    return bm, tables


def test_copy_on_write_gives_the_writer_a_private_block():
    """[P4]: a physical block may back the logical blocks of several
    sequences. After copy-on-write of one shared prefix block for one
    sequence and a write into the copy, every other sequence's output is
    unchanged bit for bit, and so is the writer's until the write."""
    sp, st, hd = _small_workload(5)
    bm, tables = _manager_for(st, sp)
    assert [t for t in tables] == [list(x) for x in st.seq_block_ids]
    assert bm.refcount == st.refcounts.tolist()
    base = _decode(sp, st, hd)
    s0, j = 5, 2                                   # second member of group 1, prefix block 2
    old = int(st.block_tables[s0, j])
    free_before = bm.num_free()
    new, must_copy = bm.copy_on_write(old)
    assert must_copy and bm.refcount[old] == 3 and bm.num_free() == free_before - 1
    kc, vc = hd.key_cache.copy(), hd.value_cache.copy()
    oracle.copy_blocks(kc, kc, [(old, new)])
    oracle.copy_blocks(vc, vc, [(old, new)])
    table = st.block_tables.copy()
    table[s0, j] = new
    assert np.array_equal(_decode(sp, st, hd, table=table, kc=kc, vc=vc), base)
    # overwrite token 3 of the copy (e4m3 codes) for s0 only
    kc[new, 3] = 0x38                              # 1.0 in every dimension
    vc[new, 3] = 0xB8                              # -1.0
    after = _decode(sp, st, hd, table=table, kc=kc, vc=vc)
    others = [s for s in range(sp.num_seqs) if s != s0]
    assert np.array_equal(after[others], base[others])
    assert not np.array_equal(after[s0], base[s0])


def test_swap_out_and_back_in_keeps_outputs():
    """[P3] §5: blocks migrate to host memory and back. A sequence whose
    blocks go to a host pool, whose device blocks are then overwritten, and
    which comes back into other device blocks (table rewritten) attends
    exactly as before."""
    sp, st, hd = _small_workload(3)
    base = _decode(sp, st, hd)
    s0 = int(np.argmax(sp.context_lens))
    ids = list(st.seq_block_ids[s0])
    others = {b for s, x in enumerate(st.seq_block_ids) if s != s0 for b in x}
    host_k = np.zeros((len(ids) + 2,) + hd.key_cache.shape[1:], hd.key_cache.dtype)
    host_v = np.zeros_like(host_k)
    kc, vc = hd.key_cache.copy(), hd.value_cache.copy()
    out_pairs = [(b, i + 2) for i, b in enumerate(ids)]
    oracle.copy_blocks(kc, host_k, out_pairs)
    oracle.copy_blocks(vc, host_v, out_pairs)
    kc[ids] = 0x7FC0; vc[ids] = 0x7FC0             # reused by someone else (NaN codes)
    targets = [b for b in np.random.default_rng(2).permutation(st.num_blocks).tolist()
               if b not in others][:len(ids)]
    in_pairs = [(i + 2, t) for i, t in enumerate(targets)]
    oracle.copy_blocks(host_k, kc, in_pairs)
    oracle.copy_blocks(host_v, vc, in_pairs)
    table = st.block_tables.copy()
    table[s0, :len(ids)] = targets
    assert np.array_equal(_decode(sp, st, hd, table=table, kc=kc, vc=vc), base)


def _fips_messages():
    for v in load_golden("sha256_fips180.json")["vectors"]:
        m = b"a" * 1000000 if v["message"] == "a*1000000" else v["message"].encode()
        yield m, bytes.fromhex(v["sha256"])


def test_block_hash_is_sha256_of_the_standard():
    """The oracle's block hash is SHA-256: with a zero parent and the tokens
    that spell a FIPS 180-2 example after the 32-byte parent, it must give
    the published digest of (32 zero bytes + message) -- checked through the
    published digests of the examples themselves and the chaining layout."""
    import hashlib
    from oracle.block_manager import block_hash
    for m, digest in _fips_messages():
        assert hashlib.sha256(m).digest() == digest
    # layout: parent bytes, then int32 little-endian tokens
    toks = [1, 256, -1]
    expect = hashlib.sha256(bytes(32) + bytes([1, 0, 0, 0, 0, 1, 0, 0, 255, 255, 255, 255]))
    assert block_hash(None, toks) == expect.digest()
    p = bytes(range(32))
    assert block_hash(p, [7]) == hashlib.sha256(p + bytes([7, 0, 0, 0])).digest()


def test_prompt_hashes_identify_whole_prefixes():
    from oracle.block_manager import prompt_block_hashes
    rng = np.random.default_rng(5)
    a = rng.integers(0, 32000, 16 * 6 + 5).tolist()
    b = list(a)
    b[16 * 3 + 2] += 1                     # differ inside block 3
    ha, hb = prompt_block_hashes(a, 16), prompt_block_hashes(b, 16)
    assert len(ha) == 6                    # the partial last block has no hash
    assert ha[:3] == hb[:3] and all(x != y for x, y in zip(ha[3:], hb[3:]))
    c = list(a)
    c[0] += 1                              # a change in block 0 changes every hash
    assert all(x != y for x, y in zip(ha, prompt_block_hashes(c, 16)))
    # same block content after a different prefix: different hash
    d = a[16:32] + a[16:32]
    hd = prompt_block_hashes(d, 16)
    assert hd[0] != hd[1]


def test_prefix_cache_policy_hand_trace():
    from oracle.block_manager import prompt_block_hashes
    bm = BlockManager(6, initial_free_order=[0, 1, 2, 3, 4, 5])
    sys_prompt = list(range(100, 132))                     # two full blocks of 16
    h1 = prompt_block_hashes(sys_prompt + [1] * 16, 16)    # request 1: 3 blocks
    ids1, hits = bm.acquire_prefix(h1)
    assert (ids1, hits) == ([0, 1, 2], 0)
    h2 = prompt_block_hashes(sys_prompt + [2] * 16, 16)    # request 2 shares 2 blocks
    ids2, hits = bm.acquire_prefix(h2)
    assert (ids2, hits) == ([0, 1, 3], 2) and bm.refcount[:4] == [2, 2, 1, 1]
    bm.free(ids1)
    bm.free(ids2)                                          # all free, hashes kept
    assert bm.free_blocks == [4, 5, 2, 0, 1, 3] and bm.lookup(h1[0]) == 0
    ids3, hits = bm.acquire_prefix(h2)                     # back out of the free list
    assert (ids3, hits) == ([0, 1, 3], 3) and bm.free_blocks == [4, 5, 2]
    assert bm.allocate(2) == [4, 5] and bm.lookup(h1[2]) == 2
    assert bm.allocate(1) == [2] and bm.lookup(h1[2]) == -1   # handed out: evicted
    with pytest.raises(OutOfBlocks):
        bm.acquire_prefix(h1)                              # needs one fresh block, none free
    assert bm.refcount == [1, 1, 1, 1, 1, 1]


def test_blocks_for_prompt_and_waste_bound():
    facts = load_golden("page_facts.json")
    bs = facts["block_size_tokens"]["value"]
    for n in [1, 15, 16, 17, 2048, 4095]:
        nblk = -(-n // bs)
        assert (nblk - 1) * bs < n <= nblk * bs     # only the last block is partial
        assert nblk * bs - n < bs


# ------------------------------------------------------------- workloads

def test_workload_structure_is_consistent():
    for cfg in (1, 2, 3, 4, 5):
        sp = wl.spec(cfg, small=cfg != 1)
        st = wl.structure(sp)
        used = [b for ids in st.seq_block_ids for b in ids]
        assert all(0 <= b < st.num_blocks for b in used)
        for s, ids in enumerate(st.seq_block_ids):
            assert len(ids) == -(-int(sp.context_lens[s]) // sp.block_size)
        if sp.shared_groups:
            assert st.refcounts.max() == 4
        else:
            assert len(set(used)) == len(used)
    sp1 = wl.spec(1)
    assert wl.structure(sp1).num_blocks == 64
