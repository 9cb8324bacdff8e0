"""Pins of the CPU oracle against facts fixed by the definitions and by mathematics.

None of these re-types the oracle's code: each compares it with an independent
statement of the same fact (IEEE-754 neighbours from numpy's float16 table,
textbook softmax attention written here in numpy, brute-force subset search,
hand-derived bytes for inputs whose codes equal their values, invariants).
"""
from itertools import combinations

import numpy as np
import pytest

import synth
from oracle import oracle as orc
from tests.helpers import bf16_bits, bf16_value, bits_of, class_capacities

D, GROUP = 128, 32

# --------------------------------------------------------------------------
# fp32 -> fp16 directed rounding: largest fp16 <= x and smallest fp16 >= x
# --------------------------------------------------------------------------
_ALL16 = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
_VALS16 = _ALL16.view(np.float16).astype(np.float64)
_FIN = np.isfinite(_VALS16)
_SORTED = np.unique(_VALS16[_FIN])            # -65504 ... 65504 (one zero)


def _rd_ref(x):
    i = np.searchsorted(_SORTED, x, side="right") - 1
    return -np.inf if i < 0 else _SORTED[i]


def _ru_ref(x):
    i = np.searchsorted(_SORTED, x, side="left")
    return np.inf if i >= len(_SORTED) else _SORTED[i]


def _probe_values():
    rng = np.random.default_rng(1)
    vals = list(rng.standard_normal(3000).astype(np.float32))
    vals += list((rng.standard_normal(2000) * 1e-5).astype(np.float32))   # fp16 subnormal range
    vals += list((rng.standard_normal(500) * 3e4).astype(np.float32))
    vals += [65504.0, 65519.0, 65520.0, 70000.0, -65504.0, -65505.0, -70000.0,
             2.0 ** -24, 2.0 ** -25, -(2.0 ** -25), 2.0 ** -14, 1.0, -1.0, 1e-30, -1e-30]
    # midpoints and near-midpoints of adjacent fp16 values
    mids = (_SORTED[:-1] + _SORTED[1:]) / 2
    sel = rng.choice(len(mids), 2000, replace=False)
    vals += list(mids[sel].astype(np.float32))
    vals += list(np.nextafter(mids[sel].astype(np.float32), np.float32(np.inf)))
    return np.array(vals, dtype=np.float32)


def test_f16_directed_rounding_matches_ieee_neighbours():
    for x in _probe_values():
        xf = float(x)
        rd = orc.f16_value(orc.f16_rd(xf))
        ru = orc.f16_value(orc.f16_ru(xf))
        assert rd == _rd_ref(xf), (xf, rd, _rd_ref(xf))
        assert ru == _ru_ref(xf), (xf, ru, _ru_ref(xf))


def test_f16_rounding_is_identity_on_fp16_values():
    fin = _ALL16[_FIN & (_VALS16 != 0)]
    for h in fin[:: 7]:
        x = float(_VALS16[h])
        assert orc.f16_rd(x) == h and orc.f16_ru(x) == h


def test_f16_bits_decode_matches_numpy():
    for h in _ALL16[_FIN][::5]:
        assert orc.f16_value(int(h)) == _VALS16[h]


# --------------------------------------------------------------------------
# group quantisation
# --------------------------------------------------------------------------
@pytest.mark.parametrize("bits", [2, 4, 8])
def test_ramp_gives_every_code(bits):
    """Values zero + j*scale (exact) quantise to j: codes 0..2^b-1 all appear."""
    qmax = (1 << bits) - 1
    cases = [(0.0, 1.0), (-2.0, 0.5), (3.0, 0.25) if bits < 8 else (-64.0, 0.5)]
    for zero, scale in cases:
        levels = np.arange(qmax + 1)
        # 32 elements: cover 0 and qmax, spread the rest
        idx = np.round(np.linspace(0, qmax, GROUP)).astype(int)
        x = (zero + idx * scale).astype(np.float32)
        assert np.all(bf16_value(bf16_bits(x)) == x)
        s, z, codes = orc.quantize_group(x, bits)
        assert orc.f16_value(z) == zero and orc.f16_value(s) == scale
        assert np.array_equal(codes, idx)
        if bits == 2:
            x2 = (zero + np.resize(levels, GROUP) * scale).astype(np.float32)
            _, _, c2 = orc.quantize_group(x2, bits)
            assert np.array_equal(c2, np.resize(levels, GROUP))


def test_half_way_codes_round_to_even():
    """(x - zero)/scale = k + 1/2 exactly -> the even one of k, k+1."""
    # 2 bits, zero 0, scale 1 (max 3): 0.5 -> 0, 1.5 -> 2, 2.5 -> 2
    x = np.array([0, 3, 0.5, 1.5, 2.5] + [0] * 27, dtype=np.float32)
    _, _, c = orc.quantize_group(x, 2)
    assert list(c[:5]) == [0, 3, 0, 2, 2]
    # 4 bits, zero 0, scale 1 (max 15): k + 0.5 -> even
    x = np.array([0, 15] + [k + 0.5 for k in range(14)] + [0] * 16, dtype=np.float32)
    _, _, c = orc.quantize_group(x, 4)
    assert list(c[2:16]) == [k if k % 2 == 0 else k + 1 for k in range(14)]


def test_constant_group():
    x = np.full(GROUP, 1.5, dtype=np.float32)
    s, z, c = orc.quantize_group(x, 4)
    assert orc.f16_value(s) == 0.0 and orc.f16_value(z) == 1.5 and not c.any()


def test_zero_rounds_down_scale_rounds_up():
    """zero <= min and zero + qmax*scale >= max, so [zero, zero+qmax*scale] covers the group."""
    rng = np.random.default_rng(7)
    for bits in (2, 4, 8):
        qmax = (1 << bits) - 1
        for _ in range(300):
            x = bf16_value(bf16_bits(rng.standard_normal(GROUP) * rng.choice([1e-6, 1e-3, 1, 30])))
            s, z, _ = orc.quantize_group(x, bits)
            zs, ss = orc.f16_value(z), orc.f16_value(s)
            assert zs <= x.min() and zs + qmax * ss >= x.max()
            assert zs == _rd_ref(float(x.min()))


def _ulp32(a):
    return np.spacing(np.abs(a).astype(np.float32)).astype(np.float64)


def _check_error_bound(x, bits):
    s, z, codes = orc.quantize_group(x, bits)
    ss, zs = orc.f16_value(s), orc.f16_value(z)
    xhat = codes.astype(np.float64) * ss + zs
    err = np.abs(x.astype(np.float64) - xhat)
    if ss == 0:
        bound = np.spacing(np.float16(zs)) if zs != 0 else 2.0 ** -24
        assert np.all(err <= bound)
    else:
        bound = ss / 2 + 4 * _ulp32(np.maximum(np.abs(x), abs(zs)))
        assert np.all(err <= bound), (err.max(), ss)


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_error_bound_random_groups(bits):
    rng = np.random.default_rng(bits)
    for _ in range(500):
        x = bf16_value(bf16_bits(rng.standard_normal(GROUP) * rng.choice([1e-4, 1, 10, 300])))
        _check_error_bound(x, bits)


def test_error_bound_every_element_tiny_workload():
    """|x - x_hat| <= scale/2 (+ fp32 slack) on every K/V element of the 2k-token workload."""
    w = synth.WORKLOADS["tiny_b1_ctx2k"]
    for tid in (synth.TID_K, synth.TID_V):
        x = bf16_value(bits_of(synth.normal_bf16(0, 0, tid, w["B"], w["Hkv"], 0, w["ctx"], D)))
        groups = x.reshape(-1, GROUP)
        for bits in (2, 4, 8):
            for g in groups[:: 17]:
                _check_error_bound(g, bits)
    # outlier channels (x10) too
    k = synth.apply_k_outliers(synth.normal_bf16(0, 0, synth.TID_K, 1, 2, 0, 256, D), 0, 0)
    for g in bf16_value(bits_of(k)).reshape(-1, GROUP):
        for bits in (2, 4, 8):
            _check_error_bound(g, bits)


# --------------------------------------------------------------------------
# record packing.  Layout: K codes | V codes | K scales | K zeros | V scales | V zeros.
# A code block is four 32-element quarters; quarter q holds 16 pairs of dims,
#   K pair p: 32*(p//4) + 8q + 2*(p%4) + {0,1};   V pair p: 8p + 2q + {0,1},
# and a 32-bit word holds 16/b pairs, pair s of the word at elements s and s + 16/b.
# --------------------------------------------------------------------------
def test_pack_hand_built_q2():
    # K[d] = d % 4: zero 0.0, scale 1.0 (fp16 0x3C00), code = d % 4.  In a word (16 elements)
    # element e holds pair s = e % 8 (dims 2*(s%4) + e//8 above a multiple of 8 + 8q), so
    # code = 2*(e % 2) + e // 8: elements 0-7 -> 0,2,0,2,... (bytes 0x88, 0x88),
    # elements 8-15 -> 1,3,1,3,... (bytes 0xDD, 0xDD).
    k = bf16_bits(np.arange(D) % 4)
    # V[d] = -1 + 0.5 * ((d // 4) % 4): zero -1.0 (0xBC00), scale 0.5 (0x3800),
    # code = (d // 4) % 4.  V pair p of quarter q is dims 8p + 2q + {0,1}, so its code is
    # (2p + q // 2) % 4 = (2s + q // 2) % 4: quarters 0, 1 -> 0,2,0,2 (0x88);
    # quarters 2, 3 -> 1,3,1,3 (0xDD).
    v = bf16_bits(-1 + 0.5 * ((np.arange(D) // 4) % 4))
    rec = orc.pack_record(2, k, v)
    assert rec.size == 96
    assert list(rec[:32]) == [0x88, 0x88, 0xDD, 0xDD] * 8
    assert list(rec[32:64]) == [0x88] * 16 + [0xDD] * 16
    meta = rec[64:].view(np.uint16)
    assert list(meta) == [0x3C00] * 4 + [0x0000] * 4 + [0x3800] * 4 + [0xBC00] * 4


def test_pack_hand_built_q4_q8():
    # 4 bits, K[d] = V[d] = d % 16: zero 0, scale 1.  A word holds 8 nibbles = 4 pairs.
    # K: element e is dim 8q + 2*(e%4) + e//4 (mod 16): q even -> 0,2,4,6,1,3,5,7
    #    (bytes 20 64 31 75), q odd -> +8 (bytes A8 EC B9 FD); 4 equal words per quarter.
    # V: element e is dim 8*blk + 2q + e//4 with blk % 2 = e % 2: 8*(e%2) + 2q + e//4,
    #    q = 0..3 -> bytes (80 80 91 91), (A2 A2 B3 B3), (C4 C4 D5 D5), (E6 E6 F7 F7).
    k = bf16_bits(np.arange(D) % 16)
    rec = orc.pack_record(4, k, k)
    kq = {0: [0x20, 0x64, 0x31, 0x75], 1: [0xA8, 0xEC, 0xB9, 0xFD]}
    assert list(rec[:64]) == sum((kq[q % 2] * 4 for q in range(4)), [])
    vq = [[0x80, 0x80, 0x91, 0x91], [0xA2, 0xA2, 0xB3, 0xB3], [0xC4, 0xC4, 0xD5, 0xD5],
          [0xE6, 0xE6, 0xF7, 0xF7]]
    assert list(rec[64:128]) == sum((vq[q] * 4 for q in range(4)), [])
    assert list(rec[128:].view(np.uint16)[:8]) == [0x3C00] * 4 + [0] * 4
    # 8 bits: K[d] = 8 * (d % 32), except 255 where d % 32 == 31: zero 0, scale 1,
    # codes = values.  Element e of word w in quarter q is dim 8q + 4*(w%2) + [0,2,1,3][e]
    # (mod 32), so a word holds 8*[m, m+2, m+1, m+3] with m = 8q + 4*(w%2).
    g = np.array([8 * i for i in range(31)] + [255], dtype=np.float32)
    k = bf16_bits(np.tile(g, 4))
    rec = orc.pack_record(8, k, k)
    exp = []
    for q in range(4):
        for w in range(8):
            m = 8 * q + 4 * (w % 2)
            exp += [min(255, 8 * x) if x != 31 else 255 for x in (m, m + 2, m + 1, m + 3)]
    assert list(rec[:128]) == exp
    assert rec.size == 288


def test_pack_bf16_storage_order():
    """bf16 records store raw bits in the same order (b = 16: one pair per word)."""
    d = np.arange(D)
    rec = orc.pack_record(16, bf16_bits(d), bf16_bits(d - 64))
    u = bf16_value(rec.view(np.uint16)).astype(int)
    # K quarter q: for each group g the dims 32g + 8q .. 32g + 8q + 7 in order
    k_exp = [32 * g + 8 * q + j for q in range(4) for g in range(4) for j in range(8)]
    # V quarter q: for each 8-dim block the dims 8blk + 2q, 8blk + 2q + 1
    v_exp = [8 * b + 2 * q + j - 64 for q in range(4) for b in range(16) for j in range(2)]
    assert list(u[:D]) == k_exp and list(u[D:]) == v_exp


@pytest.mark.parametrize("bits", [2, 4, 8, 16])
def test_unpack_of_pack_matches_numpy_dequant(bits):
    """Dequantise with an independent numpy reading of the byte layout."""
    rng = np.random.default_rng(11)
    k = bf16_bits(rng.standard_normal(D) * 3)
    v = bf16_bits(rng.standard_normal(D))
    rec = orc.pack_record(bits, k, v)
    kh, vh = orc.unpack_record(bits, rec)
    ref_k, ref_v = _np_dequant(rec, bits)
    assert np.array_equal(kh, ref_k) and np.array_equal(vh, ref_v)
    if bits == 16:
        assert np.array_equal(kh, bf16_value(k)) and np.array_equal(vh, bf16_value(v))


def _np_dims(is_v, bits):
    """Head-dim index of every storage element of a code block (from the layout rule)."""
    dims = []
    ppw = 16 // bits
    for q in range(4):
        for w in range(bits):                       # 32 elements of b bits = b words
            for e in range(32 // bits):
                p, hi = w * ppw + e % ppw, e // ppw
                dims.append(8 * p + 2 * q + hi if is_v else 32 * (p // 4) + 8 * q + 2 * (p % 4) + hi)
    return np.array(dims)


def _np_dequant(rec, bits):
    if bits == 16:
        u = rec.view(np.uint16)
        out = []
        for w in range(2):
            x = np.zeros(D)
            x[_np_dims(w, 16)] = bf16_value(u[w * D:(w + 1) * D])
            out.append(x)
        return out[0], out[1]
    cb = D * bits // 8
    per = 8 // bits
    meta = rec[2 * cb:].view(np.uint16).view(np.float16).astype(np.float64)
    out = []
    for w in range(2):
        by = rec[w * cb:(w + 1) * cb]
        stored = np.array([(by[i // per] >> (bits * (i % per))) & ((1 << bits) - 1)
                           for i in range(D)], dtype=np.float64)
        codes = np.zeros(D)
        codes[_np_dims(w, bits)] = stored
        sc = np.repeat(meta[w * 8:w * 8 + 4], GROUP)
        zr = np.repeat(meta[w * 8 + 4:w * 8 + 8], GROUP)
        out.append(codes * sc + zr)
    return out[0], out[1]


def test_storage_order_is_a_permutation():
    for bits in (2, 4, 8, 16):
        for is_v in (0, 1):
            assert sorted(_np_dims(is_v, bits)) == list(range(D))


# --------------------------------------------------------------------------
# attention: special cases that reduce to textbook softmax attention
# --------------------------------------------------------------------------
def _textbook_attention(q, K, V, scale):
    """q [G, D], K/V [N, D] float64 -> out [G, D], p [G, N]."""
    s = (q @ K.T) * scale
    s = s - s.max(axis=1, keepdims=True)
    e = np.exp(s)
    p = e / e.sum(axis=1, keepdims=True)
    return p @ V, p


def _fill(cache, ctx, cls, seed=0, outliers=False):
    B, Hkv = cache.B, cache.Hkv
    k = synth.normal_bf16(seed, 0, synth.TID_K, B, Hkv, 0, ctx, D)
    v = synth.normal_bf16(seed, 0, synth.TID_V, B, Hkv, 0, ctx, D)
    if outliers:
        k = synth.apply_k_outliers(k, seed, 0)
    pos = synth.positions(B, 0, ctx)
    st = cache.append(bits_of(k), bits_of(v), cls[:, :ctx].numpy(), pos.numpy())
    assert st == orc.ORC_OK
    return k, v


def test_all_bf16_no_eviction_equals_exact_softmax_attention():
    B, Hkv, G, ctx = 2, 2, 4, 300
    cls = synth.class_ids(0, B, ctx, 0.4, 0.4)
    cache = orc.OracleCache(B, Hkv, G, cap=[ctx, 0, 0, 0], n_protect=ctx)
    k, v = _fill(cache, ctx, cls)
    q = synth.normal_bf16(0, 0, synth.TID_Q, B, Hkv * G, ctx, 1, D)[:, :, 0]
    scale = 1 / np.sqrt(D)
    out, p = cache.attend(bits_of(q), scale, s_dbg=3)
    qf = bf16_value(bits_of(q)).astype(np.float64)
    kf = bf16_value(bits_of(k)).astype(np.float64)
    vf = bf16_value(bits_of(v)).astype(np.float64)
    for b in range(B):
        for h in range(Hkv):
            ref, pref = _textbook_attention(qf[b, h * G:(h + 1) * G], kf[b, h], vf[b, h],
                                            float(np.float32(scale)))
            got = out[b, h * G:(h + 1) * G].astype(np.float64)
            assert np.all(np.abs(got - ref) <= np.spacing(np.abs(ref).astype(np.float32)) / 2 + 1e-12)
            if b * Hkv + h == 3:
                assert np.max(np.abs(p - pref)) <= 1e-12
    assert np.max(np.abs(p.sum(axis=1) - 1)) <= 1e-12


def test_quantized_attention_equals_softmax_over_dequantized_records():
    """Mixed-precision cache: attention equals textbook attention over the values
    dequantised (by an independent numpy reading) from the live records."""
    B, Hkv, G, ctx = 1, 2, 4, 700
    cls = synth.class_ids(5, B, ctx, 0.4, 0.4)
    caps = class_capacities(cls, 4)
    cache = orc.OracleCache(B, Hkv, G, cap=caps, n_protect=4)
    _fill(cache, ctx, cls, seed=5, outliers=True)
    q = synth.normal_bf16(5, 0, synth.TID_Q, B, Hkv * G, ctx, 1, D)[:, :, 0]
    out = cache.attend(bits_of(q), 0.0883883)
    qf = bf16_value(bits_of(q)).astype(np.float64)
    for h in range(Hkv):
        Ks, Vs = [], []
        for c in range(4):
            handles, _, _ = cache.live(h, c)
            for hd in handles:
                kd, vd = _np_dequant(cache.state[f"pool{c}"][h, hd], orc.BITS[c])
                Ks.append(kd)
                Vs.append(vd)
        ref, _ = _textbook_attention(qf[0, h * G:(h + 1) * G], np.array(Ks), np.array(Vs),
                                     float(np.float32(0.0883883)))
        got = out[0, h * G:(h + 1) * G].astype(np.float64)
        assert np.all(np.abs(got - ref) <= np.spacing(np.abs(ref).astype(np.float32)) / 2 + 1e-12)


def test_scores_gain_exactly_G_per_step_and_new_token_counts():
    B, Hkv, G, ctx = 1, 2, 4, 257
    cls = synth.class_ids(1, B, ctx, 0.4, 0.4)
    cache = orc.OracleCache(B, Hkv, G, cap=class_capacities(cls, 4), n_protect=4)
    _fill(cache, ctx, cls, seed=1)
    q = synth.normal_bf16(1, 0, synth.TID_Q, B, Hkv * G, ctx, 1, D)[:, :, 0]
    before = sum(cache.state[f"score{c}"].astype(np.float64).sum() for c in range(4))
    cache.attend(bits_of(q), 1 / np.sqrt(D))
    after = sum(cache.state[f"score{c}"].astype(np.float64).sum() for c in range(4))
    assert abs((after - before) - B * Hkv * G) < 1e-4
    for c in range(4):
        _, _, sc = cache.live(0, c)
        assert np.all(sc > 0)


def test_empty_stream_gives_zero_output():
    cache = orc.OracleCache(1, 1, 4, cap=[4, 4, 4, 4], n_protect=0)
    q = bf16_bits(np.ones((1, 4, D)))
    out = cache.attend(q, 0.1)
    assert not out.any()


# --------------------------------------------------------------------------
# append allocation and capacity
# --------------------------------------------------------------------------
def test_append_class_override_and_capacity():
    B, Hkv, T = 1, 1, 10
    cache = orc.OracleCache(B, Hkv, 4, cap=[3, 2, 8, 8], n_protect=3)
    k = synth.normal_bf16(0, 0, synth.TID_K, B, Hkv, 0, T, D)
    cls = np.array([[1, 1, 2, 1, 1, 1, 2, 3, 3, 2]], dtype=np.uint8)
    pos = np.arange(T, dtype=np.int32).reshape(1, T)
    st = cache.append(bits_of(k), bits_of(k), cls, pos)
    # positions 0..2 -> class 0; class 1 gets positions 3, 4 and position 5 overflows
    assert st == orc.ORC_ERR_CAPACITY
    assert list(cache.state["n"][0]) == [3, 2, 2, 2]
    assert list(cache.live(0, 0)[1]) == [0, 1, 2]
    assert list(cache.live(0, 1)[1]) == [3, 4]
    assert list(cache.live(0, 2)[1]) == [6, 9]
    assert list(cache.live(0, 3)[1]) == [7, 8]
    assert list(cache.state["hw"][0]) == [3, 2, 2, 2]


def test_append_invalid_class_is_dropped():
    cache = orc.OracleCache(1, 1, 4, cap=[4, 4, 4, 4], n_protect=0)
    k = synth.normal_bf16(0, 0, synth.TID_K, 1, 1, 0, 3, D)
    st = cache.append(bits_of(k), bits_of(k), np.array([[1, 7, 2]], np.uint8),
                      np.arange(3, dtype=np.int32).reshape(1, 3))
    assert st == orc.ORC_ERR_INVALID
    assert list(cache.state["n"][0]) == [0, 1, 1, 0]


# --------------------------------------------------------------------------
# eviction: top-k under the total order, against brute force
# --------------------------------------------------------------------------
def _order_key(score, pos, c, i):
    return (-float(score), pos, c, i)


def _brute_force_kept(entries, budget):
    """The unique size-budget subset whose every member precedes every non-member."""
    idx = range(len(entries))
    found = []
    for sub in combinations(idx, min(budget, len(entries))):
        S = set(sub)
        ok = all(_order_key(*entries[a]) < _order_key(*entries[b])
                 for a in S for b in idx if b not in S)
        if ok:
            found.append(S)
    assert len(found) == 1
    return found[0]


def _tiny_cache_with_scores(rng, n_tok, n_protect, tie_pool):
    caps = [n_tok] * 4
    cache = orc.OracleCache(1, 1, 1, cap=caps, n_protect=n_protect)
    k = synth.normal_bf16(int(rng.integers(1 << 20)), 0, synth.TID_K, 1, 1, 0, n_tok, D)
    cls = rng.integers(1, 4, size=(1, n_tok)).astype(np.uint8)
    pos = np.arange(n_tok, dtype=np.int32).reshape(1, n_tok)
    assert cache.append(bits_of(k), bits_of(k), cls, pos) == 0
    for c in range(4):
        n = cache.state["n"][0, c]
        cache.state[f"score{c}"][0, :n] = rng.choice(tie_pool, size=n).astype(np.float32)
    return cache


@pytest.mark.parametrize("trial", range(40))
def test_kept_set_equals_brute_force(trial):
    rng = np.random.default_rng(100 + trial)
    n_tok = int(rng.integers(3, 11))
    n_protect = int(rng.integers(0, 3))
    tie_pool = [0.0, 0.25, 0.5, 1.0, 1.0, 2.0] if trial % 2 else list(rng.random(20))
    cache = _tiny_cache_with_scores(rng, n_tok, n_protect, tie_pool)
    before = cache.copy_state()
    entries, keys = [], []
    for c in range(4):
        for i in range(before["n"][0, c]):
            if before[f"pos{c}"][0, i] >= n_protect:
                entries.append((before[f"score{c}"][0, i], before[f"pos{c}"][0, i], c, i))
                keys.append((c, i))
    budget = int(rng.integers(0, n_tok + 1))
    assert cache.evict(budget) == 0
    kept_pos = set()
    for c in range(4):
        kept_pos |= set(cache.live(0, c)[1].tolist())
    if budget >= len(entries):
        expect = set(range(len(entries)))
    else:
        expect = _brute_force_kept(entries, budget)
    exp_pos = {int(entries[j][1]) for j in expect} | set(range(min(n_protect, n_tok)))
    assert kept_pos == exp_pos
    _check_table_invariants(cache, before)


def _check_table_invariants(cache, before):
    S = cache.S
    for s in range(S):
        for c in range(4):
            cap = cache.cap[c]
            n, ft, hw = (cache.state[x][s, c] for x in ("n", "ft", "hw"))
            live = cache.state[f"handle{c}"][s, :n].tolist()
            free = cache.state[f"fs{c}"][s, :ft].tolist()
            assert sorted(live + free + list(range(hw, cap))) == list(range(cap))
            p = cache.state[f"pos{c}"][s, :n]
            assert np.all(np.diff(p) > 0)
            # scores carried over: every kept (pos -> score) pair existed before
            nb = before["n"][s, c]
            old = dict(zip(before[f"pos{c}"][s, :nb].tolist(),
                           zip(before[f"score{c}"][s, :nb].tolist(),
                               before[f"handle{c}"][s, :nb].tolist())))
            for pp, sc, hd in zip(p.tolist(), cache.state[f"score{c}"][s, :n].tolist(), live):
                assert old[pp] == (sc, hd)
            # evicted slots pushed in reverse table order (earliest evicted on top)
            ev = [old_h for old_p, (old_s, old_h) in old.items() if old_p not in set(p.tolist())]
            ftb = before["ft"][s, c]
            pushed = cache.state[f"fs{c}"][s, ftb:ft].tolist()
            assert pushed == ev[::-1]


def test_evict_noop_when_budget_covers_candidates():
    rng = np.random.default_rng(5)
    cache = _tiny_cache_with_scores(rng, 8, 2, [0.1, 0.2])
    before = cache.copy_state()
    assert cache.evict(6) == 0
    for key in before:
        assert np.array_equal(before[key], cache.state[key])


def test_all_scores_equal_keeps_lowest_positions():
    rng = np.random.default_rng(9)
    cache = _tiny_cache_with_scores(rng, 10, 1, [0.75])
    cache.evict(4)
    kept = sorted(sum((cache.live(0, c)[1].tolist() for c in range(4)), []))
    assert kept == [0, 1, 2, 3, 4]


def test_reuse_after_eviction_pops_earliest_evicted_slot():
    rng = np.random.default_rng(12)
    cache = _tiny_cache_with_scores(rng, 10, 0, [0.0])
    cache.evict(2)   # keeps positions 0, 1 (all scores equal)
    st = cache.copy_state()
    c = int(np.argmax([st["ft"][0, cc] for cc in range(4)]))
    top = st[f"fs{c}"][0, st["ft"][0, c] - 1]
    k = synth.normal_bf16(0, 0, synth.TID_K, 1, 1, 10, 1, D)
    assert cache.append(bits_of(k), bits_of(k), np.array([[c]], np.uint8),
                        np.array([[10]], np.int32)) == 0
    n = cache.state["n"][0, c]
    assert cache.state[f"handle{c}"][0, n - 1] == top
    assert cache.state[f"pos{c}"][0, n - 1] == 10 and cache.state[f"score{c}"][0, n - 1] == 0


def test_scores_accumulate_over_steps():
    """score_t after two steps = sum over both steps and all G heads of p_t (cumulative mass)."""
    B, Hkv, G, ctx = 1, 2, 4, 200
    cls = synth.class_ids(2, B, ctx, 0.4, 0.4)
    cache = orc.OracleCache(B, Hkv, G, cap=class_capacities(cls, 4), n_protect=4)
    _fill(cache, ctx, cls, seed=2)
    total = np.zeros(ctx)
    for step in range(2):
        q = synth.normal_bf16(2, 0, synth.TID_Q, B, Hkv * G, ctx + step, 1, D)[:, :, 0]
        _, p = cache.attend(bits_of(q), 1 / np.sqrt(D), s_dbg=1)
        total += p.sum(axis=0)
    got = np.concatenate([cache.live(1, c)[2] for c in range(4)]).astype(np.float64)
    assert np.max(np.abs(got - total) / total) < 2e-7


# --------------------------------------------------------------------------
# dense placement: same results as in-place reuse, records kept contiguous
# --------------------------------------------------------------------------
def test_dense_placement_matches_in_place_reuse():
    B, Hkv, G, ctx = 1, 2, 4, 900
    cls = synth.class_ids(4, B, ctx + 40, 0.4, 0.4)
    caps = class_capacities(cls, 4, extra=40)
    ct = orc.OracleCache(B, Hkv, G, cap=caps, n_protect=4)
    dn = orc.OracleCache(B, Hkv, G, cap=caps, n_protect=4, dense=True)
    k = synth.normal_bf16(4, 0, synth.TID_K, B, Hkv, 0, ctx + 40, D)
    v = synth.normal_bf16(4, 0, synth.TID_V, B, Hkv, 0, ctx + 40, D)
    pos = synth.positions(B, 0, ctx + 40).numpy()
    kb, vb, c = bits_of(k), bits_of(v), cls.numpy()
    for cache in (ct, dn):
        assert cache.append(kb[:, :, :ctx], vb[:, :, :ctx], c[:, :ctx], pos[:, :ctx]) == 0
    for step in range(3):
        q = bits_of(synth.normal_bf16(4, 0, synth.TID_Q, B, Hkv * G, ctx + step, 1, D)[:, :, 0])
        o1, o2 = ct.attend(q, 0.09), dn.attend(q, 0.09)
        assert np.array_equal(o1, o2)
        for cache in (ct, dn):
            t = ctx + step
            cache.append(kb[:, :, t:t + 1], vb[:, :, t:t + 1], c[:, t:t + 1], pos[:, t:t + 1])
        for cache in (ct, dn):
            cache.evict(150 - 30 * step)
        for s in range(ct.S):
            for cc in range(4):
                n = ct.state["n"][s, cc]
                assert dn.state["n"][s, cc] == n
                assert np.array_equal(ct.state[f"pos{cc}"][s, :n], dn.state[f"pos{cc}"][s, :n])
                assert np.array_equal(ct.state[f"score{cc}"][s, :n], dn.state[f"score{cc}"][s, :n])
                # dense: entry i lives in slot i, holding the record the in-place cache has
                assert np.array_equal(dn.state[f"handle{cc}"][s, :n], np.arange(n))
                assert dn.state["hw"][s, cc] == n and dn.state["ft"][s, cc] == 0
                hs = ct.state[f"handle{cc}"][s, :n]
                assert np.array_equal(dn.state[f"pool{cc}"][s, :n], ct.state[f"pool{cc}"][s, hs])


# --------------------------------------------------------------------------
# local window (DYNTS, section 2.3): the most recent tokens are kept
# --------------------------------------------------------------------------
@pytest.mark.parametrize("trial", range(20))
def test_local_window_kept_set_equals_brute_force(trial):
    rng = np.random.default_rng(500 + trial)
    n_tok = int(rng.integers(3, 11))
    n_protect = int(rng.integers(0, 3))
    tie_pool = [0.0, 0.25, 0.5, 1.0, 1.0] if trial % 2 else list(rng.random(20))
    cache = _tiny_cache_with_scores(rng, n_tok, n_protect, tie_pool)
    before = cache.copy_state()
    keep_from = int(rng.integers(0, n_tok + 2))
    entries = []
    for c in range(4):
        for i in range(before["n"][0, c]):
            p = before[f"pos{c}"][0, i]
            if n_protect <= p < keep_from:
                entries.append((before[f"score{c}"][0, i], p, c, i))
    budget = int(rng.integers(0, n_tok + 1))
    assert cache.evict_window(budget, keep_from) == 0
    kept_pos = set()
    for c in range(4):
        kept_pos |= set(cache.live(0, c)[1].tolist())
    expect = set(range(len(entries))) if budget >= len(entries) else _brute_force_kept(entries, budget)
    fixed = {p for p in range(n_tok) if p < n_protect or p >= keep_from}
    assert kept_pos == {int(entries[j][1]) for j in expect} | fixed
    _check_table_invariants(cache, before)


def test_local_window_past_every_position_is_plain_eviction():
    rng = np.random.default_rng(77)
    a = _tiny_cache_with_scores(rng, 10, 2, list(rng.random(10)))
    b = orc.OracleCache(1, 1, 1, cap=a.cap, n_protect=2)
    b.load_state(a.copy_state())
    assert a.evict_window(4, 1 << 30) == 0 and b.evict(4) == 0
    for key in a.state:
        assert np.array_equal(a.state[key], b.state[key]), key
