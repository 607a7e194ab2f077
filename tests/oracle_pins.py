"""Pins for the CPU oracle: checks against facts that do not come from the oracle itself.

Each ``check_*`` function takes an oracle library handle and raises
AssertionError when the oracle disagrees with a closed form, a library routine,
an invariant stated by the pages or a worked example. ``test_oracle_pins.py``
runs them on the oracle; ``test_oracle_mutants.py`` runs them on copies of the
oracle with one planted mistake each and requires that some check fails.
"""
from __future__ import annotations

import math
import os

import numpy as np
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ------------------------------------------------------------------ helpers

def page_sequences(Ks, Vs, block_size, num_blocks, rng, dtype=np.float32, fill=0.0):
    """Scatter per-sequence contiguous K/V ([L, Hkv, d] each) into a pool through a
    random permutation; return (k_cache, v_cache, block_tables, seq_lens)."""
    Hkv, d = Ks[0].shape[1], Ks[0].shape[2]
    nbs = [-(-K.shape[0] // block_size) for K in Ks]
    MB = max(1, max(nbs))
    assert sum(nbs) <= num_blocks
    perm = rng.permutation(num_blocks)
    kc = np.full((num_blocks, Hkv, block_size, d), fill, dtype=dtype)
    vc = np.full((num_blocks, Hkv, block_size, d), fill, dtype=dtype)
    bt = np.full((len(Ks), MB), -1, dtype=np.int32)
    nxt = 0
    for s, (K, V) in enumerate(zip(Ks, Vs)):
        L = K.shape[0]
        for j in range(nbs[s]):
            p = int(perm[nxt]); nxt += 1
            bt[s, j] = p
            t0, t1 = j * block_size, min(L, (j + 1) * block_size)
            kc[p, :, : t1 - t0, :] = np.transpose(K[t0:t1], (1, 0, 2))
            vc[p, :, : t1 - t0, :] = np.transpose(V[t0:t1], (1, 0, 2))
    return kc, vc, bt, np.array([K.shape[0] for K in Ks], dtype=np.int32)


def sdpa_fp64(q, K, V, scale):
    """torch's scaled_dot_product_attention in float64 with grouped KV heads.
    q [Hq, d], K/V [L, Hkv, d] -> [Hq, d]."""
    qt = torch.from_numpy(np.asarray(q, dtype=np.float64))[None, :, None, :]
    kt = torch.from_numpy(np.asarray(K, dtype=np.float64)).permute(1, 0, 2)[None]
    vt = torch.from_numpy(np.asarray(V, dtype=np.float64)).permute(1, 0, 2)[None]
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=float(scale), enable_gqa=True)
    return o[0, :, 0, :].numpy()


def _decode_f32(lib, q, kc, vc, bt, sl, Hq, Hkv, d, bs, scale):
    return oracle.paged_decode(q, "f32", kc, vc, "f32", bt, sl, Hq, Hkv, d, bs, kc.shape[0], scale, lib=lib)


def _random_case(rng, lengths, Hq=8, Hkv=2, d=16):
    Ks = [rng.standard_normal((L, Hkv, d)).astype(np.float32) for L in lengths]
    Vs = [rng.standard_normal((L, Hkv, d)).astype(np.float32) for L in lengths]
    q = rng.standard_normal((len(lengths), Hq, d)).astype(np.float32)
    return q, Ks, Vs


# ------------------------------------------------------------ E4M3 format

def e4m3_library_values():
    """All 256 E4M3 codes decoded by torch's float8_e4m3fn (an independent implementation)."""
    return torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def check_e4m3_decode_table(lib):
    ref = e4m3_library_values()
    got = np.array([oracle.e4m3_value(c, lib) for c in range(256)])
    nan_ref, nan_got = np.isnan(ref), np.isnan(got)
    assert np.array_equal(nan_ref, nan_got)
    assert np.array_equal(ref[~nan_ref], got[~nan_got])
    assert np.array_equal(np.signbit(ref[~nan_ref]), np.signbit(got[~nan_got]))


def check_e4m3_spot_values(lib):
    # OCP 8-bit floating point spec: bias 7, subnormal step 2^-9, max 448, S.1111.111 NaN
    expect = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x38: 1.0,
              0x3C: 1.5, 0x77: 240.0, 0x7E: 448.0, 0xFE: -448.0, 0xB8: -1.0}
    for c, v in expect.items():
        assert oracle.e4m3_value(c, lib) == v, hex(c)
    assert math.isnan(oracle.e4m3_value(0x7F, lib)) and math.isnan(oracle.e4m3_value(0xFF, lib))


def check_e4m3_encode_vs_library(lib, n=200_000, seed=7):
    rng = np.random.default_rng(seed)
    mag = np.exp2(rng.uniform(-12.0, np.log2(463.9), size=n)).astype(np.float32)
    x = np.where(rng.random(n) < 0.5, -mag, mag).astype(np.float32)
    x = np.concatenate([x, rng.standard_normal(n).astype(np.float32) * 100]).astype(np.float32)
    x = x[np.abs(x) < 464]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle.e4m3_encode(x, lib)
    bad = np.nonzero(ref != got)[0]
    assert bad.size == 0, f"{bad.size} mismatches, e.g. x={x[bad[:3]]} ref={ref[bad[:3]]} got={got[bad[:3]]}"


def check_e4m3_ties_to_even(lib):
    finite = [oracle.e4m3_value(c, lib) for c in range(127)]
    for c in range(126):
        lo, hi = finite[c], finite[c + 1]
        mid = np.float32((lo + hi) / 2)
        assert float(mid) == (lo + hi) / 2
        even = c if c % 2 == 0 else c + 1
        got = oracle.e4m3_encode([mid, np.nextafter(mid, np.float32(np.inf)), np.nextafter(mid, np.float32(0)),
                                  -mid], lib)
        assert got[0] == even, (c, got)
        assert got[1] == c + 1 and got[2] == c, (c, got)
        assert got[3] == (0x80 | even)


def check_e4m3_saturation_and_roundtrip(lib):
    big = np.array([448.0, 448.5, 463.99, 464.0, 1e6, np.inf], dtype=np.float32)
    assert np.all(oracle.e4m3_encode(big, lib) == 0x7E)
    assert np.all(oracle.e4m3_encode(-big, lib) == 0xFE)
    assert oracle.e4m3_encode([np.nan], lib)[0] & 0x7F == 0x7F
    vals = np.array([oracle.e4m3_value(c, lib) for c in range(256)])
    codes = [c for c in range(256) if not np.isnan(vals[c])]
    assert np.array_equal(oracle.e4m3_encode(vals[codes].astype(np.float32), lib), np.array(codes, dtype=np.uint8))


# ------------------------------------------------------------- attention

def check_length_one_is_v(lib):
    rng = np.random.default_rng(11)
    q, Ks, Vs = _random_case(rng, [1, 1, 1])
    kc, vc, bt, sl = page_sequences(Ks, Vs, 16, 8, rng)
    out = _decode_f32(lib, q, kc, vc, bt, sl, 8, 2, 16, 16, 0.25)
    for s in range(3):
        for g in range(8):
            assert np.array_equal(out[s, g], Vs[s][0, g // 4].astype(np.float64))


def check_length_two_closed_form(lib):
    # hand-written d = 4 case: out = V0 + sigmoid(x1 - x0) (V1 - V0), x_t = scale q.K_t
    q = np.array([[[1.0, -2.0, 0.5, 3.0]]], dtype=np.float32)
    K = np.array([[[0.5, 1.0, -1.0, 0.25]], [[-1.5, 0.0, 2.0, 1.0]]], dtype=np.float32)
    V = np.array([[[1.0, 2.0, 3.0, 4.0]], [[-4.0, 0.0, 8.0, 0.5]]], dtype=np.float32)
    kc, vc, bt, sl = page_sequences([K], [V], 4, 3, np.random.default_rng(0))
    scale = 0.5
    out = _decode_f32(lib, q, kc, vc, bt, sl, 1, 1, 4, 4, scale)
    x0 = scale * (0.5 - 2.0 - 0.5 + 0.75)       # = -0.625
    x1 = scale * (-1.5 + 0.0 + 1.0 + 3.0)        # = 1.25
    sig = 1.0 / (1.0 + math.exp(-(x1 - x0)))
    expect = np.array([1.0, 2.0, 3.0, 4.0]) + sig * (np.array([-4.0, 0.0, 8.0, 0.5]) - np.array([1.0, 2.0, 3.0, 4.0]))
    assert np.allclose(out[0, 0], expect, rtol=0, atol=1e-14), (out[0, 0], expect)


def check_equal_keys_give_mean(lib):
    rng = np.random.default_rng(12)
    L = 37
    k = rng.standard_normal((1, 2, 16)).astype(np.float32)
    K = np.repeat(k, L, axis=0)
    V = rng.standard_normal((L, 2, 16)).astype(np.float32)
    q = rng.standard_normal((1, 8, 16)).astype(np.float32)
    kc, vc, bt, sl = page_sequences([K], [V], 8, 16, rng)
    out = _decode_f32(lib, q, kc, vc, bt, sl, 8, 2, 16, 8, 0.3)
    mean = V.astype(np.float64).mean(axis=0)
    for g in range(8):
        assert np.allclose(out[0, g], mean[g // 4], rtol=0, atol=1e-13)


def check_large_scores_pick_argmax(lib):
    # one key aligned with q by a wide margin: softmax is one-hot, out = that V (needs max subtraction)
    rng = np.random.default_rng(13)
    L, d = 21, 16
    q = np.zeros((1, 1, d), np.float32); q[0, 0, 0] = 1.0
    K = rng.uniform(-1, 1, (L, 1, d)).astype(np.float32)
    K[:, 0, 0] = np.linspace(-100, 100, L).astype(np.float32)
    K[9, 0, 0] = 300.0
    V = rng.standard_normal((L, 1, d)).astype(np.float32)
    kc, vc, bt, sl = page_sequences([K], [V], 4, 8, rng)
    out = _decode_f32(lib, q, kc, vc, bt, sl, 1, 1, d, 4, 20.0)
    assert np.all(np.isfinite(out))
    assert np.array_equal(out[0, 0], V[9, 0].astype(np.float64))


def check_matches_library_sdpa(lib):
    rng = np.random.default_rng(14)
    lengths = [1, 15, 16, 17, 40, 64, 5]
    q, Ks, Vs = _random_case(rng, lengths, Hq=8, Hkv=2, d=16)
    kc, vc, bt, sl = page_sequences(Ks, Vs, 16, 40, rng)
    out = _decode_f32(lib, q, kc, vc, bt, sl, 8, 2, 16, 16, 0.25)
    for s in range(len(lengths)):
        ref = sdpa_fp64(q[s], Ks[s], Vs[s], 0.25)
        assert np.allclose(out[s], ref, rtol=0, atol=1e-12), (s, np.abs(out[s] - ref).max())


def check_gqa_grouping(lib):
    # KV head h holds V == h everywhere: query head g must return g // (Hq/Hkv)
    rng = np.random.default_rng(15)
    Hq, Hkv, d, L = 12, 3, 8, 9
    K = rng.standard_normal((L, Hkv, d)).astype(np.float32)
    V = np.broadcast_to(np.arange(Hkv, dtype=np.float32)[None, :, None], (L, Hkv, d)).copy()
    q = rng.standard_normal((1, Hq, d)).astype(np.float32)
    kc, vc, bt, sl = page_sequences([K], [V], 4, 6, rng)
    out = _decode_f32(lib, q, kc, vc, bt, sl, Hq, Hkv, d, 4, 0.5)
    for g in range(Hq):
        assert np.allclose(out[0, g], g // (Hq // Hkv), rtol=0, atol=1e-14), g


def check_permutation_invariance(lib):
    rng = np.random.default_rng(16)
    q, Ks, Vs = _random_case(rng, [33, 7, 64, 16], Hq=4, Hkv=2, d=16)
    kc, vc, bt, sl = page_sequences(Ks, Vs, 16, 24, rng)
    base = _decode_f32(lib, q, kc, vc, bt, sl, 4, 2, 16, 16, 0.2)
    perm = rng.permutation(kc.shape[0])           # new position of old block i is perm[i]
    kc2 = np.empty_like(kc); vc2 = np.empty_like(vc)
    kc2[perm] = kc; vc2[perm] = vc
    bt2 = np.where(bt >= 0, perm[np.maximum(bt, 0)], -1).astype(np.int32)
    again = _decode_f32(lib, q, kc2, vc2, bt2, sl, 4, 2, 16, 16, 0.2)
    assert np.array_equal(base, again)


def check_block_size_invariance(lib):
    rng = np.random.default_rng(17)
    q, Ks, Vs = _random_case(rng, [70, 3, 32, 95], Hq=4, Hkv=1, d=8)
    outs = []
    for bs in (8, 16, 32):
        kc, vc, bt, sl = page_sequences(Ks, Vs, bs, 64, np.random.default_rng(bs))
        outs.append(_decode_f32(lib, q, kc, vc, bt, sl, 4, 1, 8, bs, 0.35))
    assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[0], outs[2])


def load_worked_table():
    """The block table printed in the Aliyun article, section 4 (logical -> physical)."""
    mapping = {}
    with open(os.path.join(GOLDEN, "aliyun_s4_block_table.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                a, b = line.split()
                mapping[int(a)] = int(b)
    return mapping


def check_worked_block_table(lib):
    mapping = load_worked_table()
    nlog = len(mapping)
    bs, Hkv, d, Hq = 16, 2, 16, 8
    L = nlog * bs
    pool = max(mapping.values()) + 1
    rng = np.random.default_rng(18)
    K = rng.standard_normal((L, Hkv, d)).astype(np.float32)
    V = rng.standard_normal((L, Hkv, d)).astype(np.float32)
    q = rng.standard_normal((1, Hq, d)).astype(np.float32)
    kc = np.full((pool, Hkv, bs, d), np.nan, np.float32)   # blocks not in the table are poison
    vc = np.full((pool, Hkv, bs, d), np.nan, np.float32)
    bt = np.zeros((1, nlog), np.int32)
    for j, p in mapping.items():
        bt[0, j] = p
        kc[p] = np.transpose(K[j * bs:(j + 1) * bs], (1, 0, 2))
        vc[p] = np.transpose(V[j * bs:(j + 1) * bs], (1, 0, 2))
    out = _decode_f32(lib, q, kc, vc, bt, np.array([L], np.int32), Hq, Hkv, d, bs, 0.25)
    ref = sdpa_fp64(q[0], K, V, 0.25)
    assert np.all(np.isfinite(out))
    assert np.allclose(out[0], ref, rtol=0, atol=1e-12)


def check_zero_length(lib):
    rng = np.random.default_rng(19)
    q, Ks, Vs = _random_case(rng, [5], Hq=2, Hkv=1, d=8)
    kc, vc, bt, sl = page_sequences(Ks, Vs, 4, 4, rng)
    sl[0] = 0
    out = _decode_f32(lib, q, kc, vc, bt, sl, 2, 1, 8, 4, 1.0)
    assert np.array_equal(out, np.zeros_like(out))


# ----------------------------------------------------------------- append

def check_append_golden(lib):
    """Hand-built append: slot = block * block_size + offset, negative slots write nothing."""
    bs, Hkv, d, nb = 16, 2, 4, 3
    k = np.arange(3 * Hkv * d, dtype=np.float32).reshape(3, Hkv, d) + 1
    v = -k
    slots = np.array([5, -1, 17], dtype=np.int64)
    kc = oracle.empty_cache(nb, Hkv, bs, d, "f32"); vc = oracle.empty_cache(nb, Hkv, bs, d, "f32")
    oracle.reshape_and_cache(k, v, "f32", kc, vc, "f32", slots, Hkv, d, bs, nb, lib=lib)
    expect_k = np.zeros_like(kc)
    expect_k[0, :, 5, :] = k[0]
    expect_k[1, :, 1, :] = k[2]
    assert np.array_equal(kc, expect_k)
    assert np.array_equal(vc, -expect_k)


def check_append_fp8_vs_library(lib):
    rng = np.random.default_rng(20)
    T, Hkv, d, bs, nb = 40, 2, 32, 8, 8
    k = rng.standard_normal((T, Hkv, d)).astype(np.float32) * 3
    v = rng.standard_normal((T, Hkv, d)).astype(np.float32)
    ks = np.float32(np.abs(k).max() / np.float32(448)); vs = np.float32(np.abs(v).max() / np.float32(448))
    slots = rng.permutation(nb * bs)[:T].astype(np.int64)
    kc = oracle.empty_cache(nb, Hkv, bs, d, "e4m3"); vc = oracle.empty_cache(nb, Hkv, bs, d, "e4m3")
    oracle.reshape_and_cache(k, v, "f32", kc, vc, "e4m3", slots, Hkv, d, bs, nb, ks, vs, lib=lib)
    for t in range(T):
        b, o = divmod(int(slots[t]), bs)
        ek = torch.from_numpy((k[t] / ks).astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        ev = torch.from_numpy((v[t] / vs).astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(kc[b, :, o, :], ek) and np.array_equal(vc[b, :, o, :], ev)


def check_fp8_attention_dequant(lib):
    """Attention over an E4M3 cache equals attention over the library-decoded values times the scale."""
    rng = np.random.default_rng(21)
    nb, Hkv, bs, d, Hq = 6, 2, 8, 16, 4
    kc = rng.integers(0, 256, (nb, Hkv, bs, d), dtype=np.uint8)
    vc = rng.integers(0, 256, (nb, Hkv, bs, d), dtype=np.uint8)
    kc[(kc & 0x7F) == 0x7F] = 0x10; vc[(vc & 0x7F) == 0x7F] = 0x22     # no NaN codes
    ks, vs = np.float32(0.0125), np.float32(0.5)
    lut = e4m3_library_values()
    kf = (lut[kc] * float(ks)); vf = (lut[vc] * float(vs))
    q = rng.standard_normal((2, Hq, d)).astype(np.float32)
    bt = np.array([[3, 1, 4], [0, 5, -1]], np.int32)
    sl = np.array([20, 11], np.int32)
    got = oracle.paged_decode(q, "f32", kc, vc, "e4m3", bt, sl, Hq, Hkv, d, bs, nb, 0.25, ks, vs, lib=lib)
    for s in range(2):
        L = int(sl[s])
        K = np.concatenate([np.transpose(kf[bt[s, j]], (1, 0, 2)) for j in range(-(-L // bs))])[:L]
        V = np.concatenate([np.transpose(vf[bt[s, j]], (1, 0, 2)) for j in range(-(-L // bs))])[:L]
        ref = sdpa_fp64(q[s], K, V, 0.25)
        assert np.allclose(got[s], ref, rtol=0, atol=1e-12)


# ------------------------------------------------------------ E5M2 format

def e5m2_library_values():
    """All 256 E5M2 codes decoded by torch's float8_e5m2 (an independent implementation)."""
    return torch.arange(256, dtype=torch.uint8).view(torch.float8_e5m2).to(torch.float64).numpy()


def check_e5m2_decode_table(lib):
    ref = e5m2_library_values()
    got = np.array([oracle.e5m2_value(c, lib) for c in range(256)])
    nan_ref, nan_got = np.isnan(ref), np.isnan(got)
    assert np.array_equal(nan_ref, nan_got)
    assert np.array_equal(ref[~nan_ref], got[~nan_got])
    assert np.array_equal(np.signbit(ref[~nan_ref]), np.signbit(got[~nan_got]))


def check_e5m2_spot_values(lib):
    # OCP 8-bit floating point spec: bias 15, subnormal step 2^-16, max 57344, S.11111.00 inf
    expect = {0x00: 0.0, 0x01: 2.0 ** -16, 0x03: 3 * 2.0 ** -16, 0x04: 2.0 ** -14, 0x3C: 1.0,
              0x3E: 1.5, 0x7B: 57344.0, 0xFB: -57344.0, 0x7C: np.inf, 0xFC: -np.inf, 0xBC: -1.0}
    for c, v in expect.items():
        assert oracle.e5m2_value(c, lib) == v, hex(c)
    for c in (0x7D, 0x7E, 0x7F, 0xFD, 0xFE, 0xFF):
        assert math.isnan(oracle.e5m2_value(c, lib))


def check_e5m2_encode_vs_library(lib, n=200_000, seed=8):
    rng = np.random.default_rng(seed)
    mag = np.exp2(rng.uniform(-20.0, np.log2(57343.0), size=n)).astype(np.float32)
    x = np.where(rng.random(n) < 0.5, -mag, mag).astype(np.float32)
    x = np.concatenate([x, rng.standard_normal(n).astype(np.float32) * 100]).astype(np.float32)
    x = x[np.abs(x) < 57344]
    ref = torch.from_numpy(x).to(torch.float8_e5m2).view(torch.uint8).numpy()
    got = oracle.e5m2_encode(x, lib)
    bad = np.nonzero(ref != got)[0]
    assert bad.size == 0, f"{bad.size} mismatches, e.g. x={x[bad[:3]]} ref={ref[bad[:3]]} got={got[bad[:3]]}"


def check_e5m2_ties_saturation_roundtrip(lib):
    finite = [oracle.e5m2_value(c, lib) for c in range(124)]
    for c in range(123):
        lo, hi = finite[c], finite[c + 1]
        mid = np.float32((lo + hi) / 2)
        assert float(mid) == (lo + hi) / 2
        even = c if c % 2 == 0 else c + 1
        got = oracle.e5m2_encode([mid, np.nextafter(mid, np.float32(np.inf)), np.nextafter(mid, np.float32(0)),
                                  -mid], lib)
        assert got[0] == even and got[1] == c + 1 and got[2] == c and got[3] == (0x80 | even), (c, got)
    big = np.array([57344.0, 60000.0, 61440.0, 1e9, np.inf], dtype=np.float32)
    assert np.all(oracle.e5m2_encode(big, lib) == 0x7B) and np.all(oracle.e5m2_encode(-big, lib) == 0xFB)
    assert oracle.e5m2_encode([np.nan], lib)[0] == 0x7F
    codes = [c for c in range(256) if np.isfinite(oracle.e5m2_value(c, lib))]
    vals = np.array([oracle.e5m2_value(c, lib) for c in codes], dtype=np.float32)
    assert np.array_equal(oracle.e5m2_encode(vals, lib), np.array(codes, dtype=np.uint8))


def check_append_e5m2_vs_library(lib):
    rng = np.random.default_rng(22)
    T, Hkv, d, bs, nb = 40, 2, 32, 8, 8
    k = rng.standard_normal((T, Hkv, d)).astype(np.float32) * 3
    v = rng.standard_normal((T, Hkv, d)).astype(np.float32)
    ks = np.float32(np.abs(k).max() / np.float32(57344)); vs = np.float32(np.abs(v).max() / np.float32(57344))
    slots = rng.permutation(nb * bs)[:T].astype(np.int64)
    kc = oracle.empty_cache(nb, Hkv, bs, d, "e5m2"); vc = oracle.empty_cache(nb, Hkv, bs, d, "e5m2")
    oracle.reshape_and_cache(k, v, "f32", kc, vc, "e5m2", slots, Hkv, d, bs, nb, ks, vs, lib=lib)
    for t in range(T):
        b, o = divmod(int(slots[t]), bs)
        ek = torch.from_numpy((k[t] / ks).astype(np.float32)).to(torch.float8_e5m2).view(torch.uint8).numpy()
        ev = torch.from_numpy((v[t] / vs).astype(np.float32)).to(torch.float8_e5m2).view(torch.uint8).numpy()
        assert np.array_equal(kc[b, :, o, :], ek) and np.array_equal(vc[b, :, o, :], ev)


def check_e5m2_attention_dequant(lib):
    """Attention over an E5M2 cache equals attention over the library-decoded values times the scale."""
    rng = np.random.default_rng(23)
    nb, Hkv, bs, d, Hq = 6, 2, 8, 16, 4
    kc = rng.integers(0, 256, (nb, Hkv, bs, d), dtype=np.uint8)
    vc = rng.integers(0, 256, (nb, Hkv, bs, d), dtype=np.uint8)
    kc[(kc & 0x7C) == 0x7C] = 0x31; vc[(vc & 0x7C) == 0x7C] = 0x2A     # no inf / NaN codes
    ks, vs = np.float32(2.0 ** -12), np.float32(2.0 ** -14)
    lut = e5m2_library_values()
    kf = (lut[kc] * float(ks)); vf = (lut[vc] * float(vs))
    q = rng.standard_normal((2, Hq, d)).astype(np.float32)
    bt = np.array([[3, 1, 4], [0, 5, -1]], np.int32)
    sl = np.array([20, 11], np.int32)
    got = oracle.paged_decode(q, "f32", kc, vc, "e5m2", bt, sl, Hq, Hkv, d, bs, nb, 0.25, ks, vs, lib=lib)
    for s in range(2):
        L = int(sl[s])
        K = np.concatenate([np.transpose(kf[bt[s, j]], (1, 0, 2)) for j in range(-(-L // bs))])[:L]
        V = np.concatenate([np.transpose(vf[bt[s, j]], (1, 0, 2)) for j in range(-(-L // bs))])[:L]
        ref = sdpa_fp64(q[s], K, V, 0.25)
        assert np.allclose(got[s], ref, rtol=0, atol=1e-12)


# ------------------------------------------------------------- several queries per sequence

def check_multi_query_matches_causal_sdpa(lib):
    """q_len new tokens per sequence: torch SDPA (fp64) with an explicit causal mask over the
    contiguous K/V equals the paged oracle; query j sees tokens 0 .. L - q_len + j."""
    rng = np.random.default_rng(31)
    Hq, Hkv, d, bs, q_len = 8, 2, 16, 4, 3
    lengths = [3, 5, 9, 14]
    _, Ks, Vs = _random_case(rng, lengths, Hq, Hkv, d)
    q = rng.standard_normal((len(lengths), q_len, Hq, d))
    kc, vc, bt, sl = page_sequences(Ks, Vs, bs, sum(-(-L // bs) for L in lengths) + 3, rng)
    got = oracle.paged_decode(q.astype(np.float32), "f32", kc, vc, "f32", bt, sl, Hq, Hkv, d, bs, kc.shape[0], 0.3,
                              lib=lib, q_len=q_len)
    for s, L in enumerate(lengths):
        qt = torch.from_numpy(q[s].astype(np.float32).astype(np.float64)).permute(1, 0, 2)[None]   # [1, Hq, q_len, d]
        kt = torch.from_numpy(Ks[s].astype(np.float64)).permute(1, 0, 2)[None]
        vt = torch.from_numpy(Vs[s].astype(np.float64)).permute(1, 0, 2)[None]
        pos = torch.arange(L - q_len, L)[:, None]
        mask = torch.arange(L)[None, :] <= pos                                                  # [q_len, L]
        ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=0.3,
                                                                enable_gqa=True)[0].permute(1, 0, 2).numpy()
        assert np.allclose(got[s], ref, rtol=0, atol=1e-12), s


def check_multi_query_is_decode_at_each_position(lib):
    """Query j of a q_len chunk equals the single-query decode of a sequence cut at length
    L - q_len + 1 + j (bit for bit: the same definition, the same order)."""
    rng = np.random.default_rng(32)
    Hq, Hkv, d, bs, q_len = 4, 1, 8, 8, 4
    lengths = [4, 7, 20]
    _, Ks, Vs = _random_case(rng, lengths, Hq, Hkv, d)
    q = rng.standard_normal((len(lengths), q_len, Hq, d)).astype(np.float32)
    kc, vc, bt, sl = page_sequences(Ks, Vs, bs, sum(-(-L // bs) for L in lengths) + 3, rng)
    got = oracle.paged_decode(q, "f32", kc, vc, "f32", bt, sl, Hq, Hkv, d, bs, kc.shape[0], 0.5, lib=lib,
                              q_len=q_len)
    for j in range(q_len):
        cut = (sl - q_len + 1 + j).astype(np.int32)
        one = oracle.paged_decode(np.ascontiguousarray(q[:, j]), "f32", kc, vc, "f32", bt, cut, Hq, Hkv, d, bs,
                                  kc.shape[0], 0.5, lib=lib)
        assert np.array_equal(got[:, j], one), j


# ------------------------------------------------------------- per-KV-head FP8 scales

def check_head_scales_equal_per_head_runs(lib):
    """One scale per KV head: appending and attending with head scales (s0, s1) equals, head by
    head, the per-tensor oracle run with that head's scale (bit for bit); equal head scales
    equal the per-tensor run."""
    rng = np.random.default_rng(41)
    T, Hkv, d, bs, nb, Hq = 24, 2, 16, 8, 6, 4
    k = rng.standard_normal((T, Hkv, d)).astype(np.float32)
    v = rng.standard_normal((T, Hkv, d)).astype(np.float32)
    k[:, 1] *= 20; v[:, 1] *= 0.05                                  # heads of very different ranges
    khs = (np.abs(k).max(axis=(0, 2)) / 448).astype(np.float32)
    vhs = (np.abs(v).max(axis=(0, 2)) / 448).astype(np.float32)
    blocks = [int(b) for b in rng.permutation(nb)[: T // bs]]          # T is a multiple of bs
    slots = np.array([blocks[t // bs] * bs + t % bs for t in range(T)], np.int64)
    bt = np.array([blocks], np.int32); sl = np.array([T], np.int32)
    q = rng.standard_normal((1, Hq, d)).astype(np.float32)
    kc = oracle.empty_cache(nb, Hkv, bs, d, "e4m3"); vc = oracle.empty_cache(nb, Hkv, bs, d, "e4m3")
    oracle.reshape_and_cache(k, v, "f32", kc, vc, "e4m3", slots, Hkv, d, bs, nb, lib=lib,
                             k_head_scales=khs, v_head_scales=vhs)
    got = oracle.paged_decode(q, "f32", kc, vc, "e4m3", bt, sl, Hq, Hkv, d, bs, nb, 0.25, lib=lib,
                              k_head_scales=khs, v_head_scales=vhs)
    G = Hq // Hkv
    for h in range(Hkv):
        kc1 = oracle.empty_cache(nb, 1, bs, d, "e4m3"); vc1 = oracle.empty_cache(nb, 1, bs, d, "e4m3")
        oracle.reshape_and_cache(np.ascontiguousarray(k[:, h:h + 1]), np.ascontiguousarray(v[:, h:h + 1]), "f32",
                                 kc1, vc1, "e4m3", slots, 1, d, bs, nb, khs[h], vhs[h], lib=lib)
        assert np.array_equal(kc[:, h], kc1[:, 0]) and np.array_equal(vc[:, h], vc1[:, 0])
        one = oracle.paged_decode(np.ascontiguousarray(q[:, h * G:(h + 1) * G]), "f32", kc1, vc1, "e4m3", bt, sl,
                                  G, 1, d, bs, nb, 0.25, khs[h], vhs[h], lib=lib)
        assert np.array_equal(got[:, h * G:(h + 1) * G], one), h
    same = oracle.paged_decode(q, "f32", kc, vc, "e4m3", bt, sl, Hq, Hkv, d, bs, nb, 0.25, 0.5, 0.25, lib=lib)
    same_h = oracle.paged_decode(q, "f32", kc, vc, "e4m3", bt, sl, Hq, Hkv, d, bs, nb, 0.25, lib=lib,
                                 k_head_scales=[0.5, 0.5], v_head_scales=[0.25, 0.25])
    assert np.array_equal(same, same_h)


# ------------------------------------------------------------- INT8 caches

def check_int8_encode_vs_library(lib, n=200_000, seed=9):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal(n) * 60).astype(np.float32)
    x = np.concatenate([x, np.arange(-130, 131, 0.5, dtype=np.float32)])        # every tie, both clamps
    ref = np.clip(np.rint(x), -127, 127).astype(np.int8)                          # numpy rounds ties to even
    got = np.array([lib.orc_int8_encode(float(v)) for v in x], dtype=np.int8)
    assert np.array_equal(ref, got)
    assert lib.orc_int8_encode(float("nan")) == 0


def check_append_int8_vs_library(lib):
    rng = np.random.default_rng(24)
    T, Hkv, d, bs, nb = 40, 2, 32, 8, 8
    k = rng.standard_normal((T, Hkv, d)).astype(np.float32) * 3
    v = rng.standard_normal((T, Hkv, d)).astype(np.float32)
    ks = np.float32(np.abs(k).max() / np.float32(127)); vs = np.float32(np.abs(v).max() / np.float32(127))
    slots = rng.permutation(nb * bs)[:T].astype(np.int64)
    kc = oracle.empty_cache(nb, Hkv, bs, d, "int8"); vc = oracle.empty_cache(nb, Hkv, bs, d, "int8")
    oracle.reshape_and_cache(k, v, "f32", kc, vc, "int8", slots, Hkv, d, bs, nb, ks, vs, lib=lib)
    for t in range(T):
        b, o = divmod(int(slots[t]), bs)
        ek = np.clip(np.rint((k[t] / ks).astype(np.float32)), -127, 127).astype(np.int8)
        ev = np.clip(np.rint((v[t] / vs).astype(np.float32)), -127, 127).astype(np.int8)
        assert np.array_equal(kc[b, :, o, :], ek) and np.array_equal(vc[b, :, o, :], ev)


def check_int8_attention_dequant(lib):
    rng = np.random.default_rng(25)
    nb, Hkv, bs, d, Hq = 6, 2, 8, 16, 4
    kc = rng.integers(-127, 128, (nb, Hkv, bs, d), dtype=np.int8)
    vc = rng.integers(-127, 128, (nb, Hkv, bs, d), dtype=np.int8)
    ks, vs = np.float32(0.01), np.float32(0.003)
    kf = kc.astype(np.float64) * float(ks); vf = vc.astype(np.float64) * float(vs)
    q = rng.standard_normal((2, Hq, d)).astype(np.float32)
    bt = np.array([[3, 1, 4], [0, 5, -1]], np.int32)
    sl = np.array([20, 11], np.int32)
    got = oracle.paged_decode(q, "f32", kc, vc, "int8", bt, sl, Hq, Hkv, d, bs, nb, 0.25, ks, vs, lib=lib)
    for s in range(2):
        L = int(sl[s])
        K = np.concatenate([np.transpose(kf[bt[s, j]], (1, 0, 2)) for j in range(-(-L // bs))])[:L]
        V = np.concatenate([np.transpose(vf[bt[s, j]], (1, 0, 2)) for j in range(-(-L // bs))])[:L]
        assert np.allclose(got[s], sdpa_fp64(q[s], K, V, 0.25), rtol=0, atol=1e-12)


# ------------------------------------------------------------ log-sum-exp of the scores

def check_lse_matches_library_logsumexp(lib):
    """The row's log softmax denominator against torch.logsumexp of the scores (fp64 matmul
    on the contiguous K); equal keys give score + log L; a row that sees nothing gives -inf."""
    rng = np.random.default_rng(21)
    lengths = [1, 2, 15, 16, 17, 40, 0]
    q, Ks, Vs = _random_case(rng, lengths, Hq=8, Hkv=2, d=16)
    kc, vc, bt, sl = page_sequences(Ks, Vs, 16, 40, rng)
    _, lse = oracle.paged_decode(q, "f32", kc, vc, "f32", bt, sl, 8, 2, 16, 16, kc.shape[0], 0.25, lib=lib,
                                 return_lse=True)
    _, sub = oracle.paged_decode(q, "f32", kc, vc, "f32", bt, sl, 8, 2, 16, 16, kc.shape[0], 0.25, seqs=[4, 0],
                                 lib=lib, return_lse=True)
    assert np.array_equal(sub, lse[[4, 0]])          # rows follow `seqs`
    for s, L in enumerate(lengths):
        for g in range(8):
            if L == 0:
                assert lse[s, g] == -np.inf
                continue
            K = torch.from_numpy(Ks[s][:, g // 4, :].astype(np.float64))
            x = 0.25 * (K @ torch.from_numpy(q[s, g].astype(np.float64)))
            assert abs(lse[s, g] - float(torch.logsumexp(x, 0))) <= 1e-12, (s, g)
    L = 23
    K = np.repeat(rng.standard_normal((1, 1, 16)).astype(np.float32), L, axis=0)
    V = rng.standard_normal((L, 1, 16)).astype(np.float32)
    q1 = rng.standard_normal((1, 1, 16)).astype(np.float32)
    kc, vc, bt, sl = page_sequences([K], [V], 4, 8, rng)
    _, lse = oracle.paged_decode(q1, "f32", kc, vc, "f32", bt, sl, 1, 1, 16, 4, 8, 0.5, lib=lib, return_lse=True)
    score = 0.5 * float(np.dot(q1[0, 0].astype(np.float64), K[0, 0].astype(np.float64)))
    assert abs(lse[0, 0] - (score + math.log(L))) <= 1e-12
    # several new tokens: row (j, g) covers the tokens up to position L - q_len + j
    QL, lengths = 3, [5, 19]
    qm, Ks, Vs = _random_case(rng, lengths, Hq=4, Hkv=2, d=16)
    qm = rng.standard_normal((len(lengths), QL, 4, 16)).astype(np.float32)
    kc, vc, bt, sl = page_sequences(Ks, Vs, 8, 8, rng)
    _, lse = oracle.paged_decode(qm, "f32", kc, vc, "f32", bt, sl, 4, 2, 16, 8, 8, 0.25, lib=lib, q_len=QL,
                                 return_lse=True)
    for s, L in enumerate(lengths):
        for j in range(QL):
            for g in range(4):
                K = torch.from_numpy(Ks[s][: L - QL + 1 + j, g // 2, :].astype(np.float64))
                x = 0.25 * (K @ torch.from_numpy(qm[s, j, g].astype(np.float64)))
                assert abs(lse[s, j, g] - float(torch.logsumexp(x, 0))) <= 1e-12, (s, j, g)


def check_lse_splits_combine(lib):
    """A sequence cut after its first a blocks: attention over the first part (its table
    cut to a blocks) and over the rest (the table shifted by a blocks, length L - a*bs)
    combine, weighted by exp(lse), into the attention over the whole sequence. This is the
    decomposition a shared-prefix decode relies on (a shared head of the table plus each
    sequence's own tail)."""
    rng = np.random.default_rng(22)
    bs, Hq, Hkv, d = 8, 8, 2, 16
    lengths = [9, 16, 17, 40, 57]
    q, Ks, Vs = _random_case(rng, lengths, Hq=Hq, Hkv=Hkv, d=d)
    for kv in ("f32", "e4m3"):
        kc, vc, bt, sl = page_sequences(Ks, Vs, bs, 40, rng)
        ks = vs = 1.0
        if kv == "e4m3":
            ks, vs = 0.01, 0.02
            kc = oracle.e4m3_encode(kc / np.float32(ks), lib=lib).reshape(kc.shape)
            vc = oracle.e4m3_encode(vc / np.float32(vs), lib=lib).reshape(vc.shape)
        nb = kc.shape[0]
        full, lse = oracle.paged_decode(q, "f32", kc, vc, kv, bt, sl, Hq, Hkv, d, bs, nb, 0.25, ks, vs, lib=lib,
                                        return_lse=True)
        for s, L in enumerate(lengths):
            for a in range(1, -(-L // bs) + 1):
                head_t = np.full_like(bt[s:s + 1], -1)
                head_t[0, :a] = bt[s, :a]
                tail_t = np.full_like(bt[s:s + 1], -1)
                tail_t[0, :bt.shape[1] - a] = bt[s, a:]
                n1, n2 = min(L, a * bs), max(0, L - a * bs)
                o1, l1 = oracle.paged_decode(q[s:s + 1], "f32", kc, vc, kv, head_t, np.array([n1], np.int32), Hq,
                                             Hkv, d, bs, nb, 0.25, ks, vs, lib=lib, return_lse=True)
                o2, l2 = oracle.paged_decode(q[s:s + 1], "f32", kc, vc, kv, tail_t, np.array([n2], np.int32), Hq,
                                             Hkv, d, bs, nb, 0.25, ks, vs, lib=lib, return_lse=True)
                M = np.maximum(l1, l2)
                w1, w2 = np.exp(l1 - M), np.exp(l2 - M)
                comb = (w1[..., None] * o1 + w2[..., None] * o2) / (w1 + w2)[..., None]
                assert np.allclose(comb[0], full[s], rtol=0, atol=1e-12), (kv, s, a)
                assert np.allclose(M + np.log(w1 + w2), lse[s:s + 1], rtol=0, atol=1e-12), (kv, s, a)


ALL_CHECKS = [
    check_e4m3_decode_table, check_e4m3_spot_values, check_e4m3_encode_vs_library, check_e4m3_ties_to_even,
    check_e4m3_saturation_and_roundtrip, check_length_one_is_v, check_length_two_closed_form,
    check_equal_keys_give_mean, check_large_scores_pick_argmax, check_matches_library_sdpa, check_gqa_grouping,
    check_permutation_invariance, check_block_size_invariance, check_worked_block_table, check_zero_length,
    check_append_golden, check_append_fp8_vs_library, check_fp8_attention_dequant,
    check_e5m2_decode_table, check_e5m2_spot_values, check_e5m2_encode_vs_library,
    check_e5m2_ties_saturation_roundtrip, check_append_e5m2_vs_library, check_e5m2_attention_dequant,
    check_multi_query_matches_causal_sdpa, check_multi_query_is_decode_at_each_position,
    check_head_scales_equal_per_head_runs, check_int8_encode_vs_library, check_append_int8_vs_library,
    check_int8_attention_dequant, check_lse_matches_library_logsumexp, check_lse_splits_combine,
]
