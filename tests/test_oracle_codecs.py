"""Pins of the oracle's floating-point class codecs (ThinKV page, Metodologia, TBQ:
FP8 or NVFP4 for Reasoning tokens, ternary for Transition tokens); CPU only.

FP8 E4M3 is pinned against torch's float8_e4m3fn conversions (a library routine:
every code's value, round-to-nearest-even on random and half-way inputs); E2M1
against the OCP table of its eight magnitudes and a brute-force nearest search;
the group quantisers against their error bounds, exact round trips and hand cases;
the FP-class records against an independent numpy/torch reading of their layout, and
attention over an FP-class cache against softmax attention over the decoded records."""
import numpy as np
import pytest
import torch

import synth
from oracle import oracle as orc
from tests.helpers import bits_of
from tests.test_record_layout import header_position

# OCP MX: the magnitudes of the E2M1 codes 0..7 (bit 3 is the sign)
E2M1_TABLE = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e4m3_decode_matches_torch_for_every_code():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    for c in range(256):
        got = orc.e4m3_decode(c)
        if np.isnan(ref[c]):
            assert np.isnan(got), c
        else:
            assert got == ref[c] and np.signbit(got) == np.signbit(ref[c]), c


def _torch_e4m3_code(x):
    return int(torch.tensor([x], dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8)[0])


def test_e4m3_encode_matches_torch_round_to_nearest_even():
    rng = np.random.default_rng(0)
    xs = np.concatenate([rng.uniform(-440, 440, 3000), rng.normal(0, 1, 3000),
                         rng.uniform(-2 ** -6, 2 ** -6, 1000), rng.normal(0, 1e-3, 500)]).astype(np.float32)
    # every half-way point between neighbouring finite codes (ties go to the even code)
    vals = sorted({orc.e4m3_decode(c) for c in range(0x7F)})
    mids = np.array([(a + b) / 2 for a, b in zip(vals, vals[1:])], np.float32)
    for x in np.concatenate([xs, mids, -mids]):
        assert orc.e4m3_encode(x) == _torch_e4m3_code(float(x)), x


def test_e4m3_saturates_and_rounds_up():
    assert orc.e4m3_encode(448.0) == 0x7E and orc.e4m3_encode(1e9) == 0x7E and orc.e4m3_encode(-500) == 0xFE
    assert np.isnan(orc.e4m3_decode(orc.e4m3_encode(float("nan"))))
    rng = np.random.default_rng(1)
    for y in np.concatenate([rng.uniform(1e-4, 440, 2000), [2 ** -9, 1.0, 448.0]]).astype(np.float32):
        c = orc.e4m3_round_up(y)
        v = orc.e4m3_decode(c)
        assert v >= y and (c == 0 or orc.e4m3_decode(c - 1) < y), y


def test_e2m1_table_and_brute_force_nearest():
    for c in range(16):
        mag = E2M1_TABLE[c & 7]
        assert orc.e2m1_decode(c) == (-mag if c & 8 else mag)
    rng = np.random.default_rng(2)
    mids = [(a + b) / 2 for a, b in zip(E2M1_TABLE, E2M1_TABLE[1:])]
    xs = np.concatenate([rng.uniform(-6.5, 6.5, 4000), mids, [-m for m in mids], [7.0, -100.0]])
    for x in xs.astype(np.float32):
        a = min(abs(float(x)), 6.0)
        best = min(range(8), key=lambda k: (abs(E2M1_TABLE[k] - a), k % 2))   # nearest, then even
        assert orc.e2m1_encode(x) & 7 == best, x
        assert (orc.e2m1_encode(x) >> 3) == (1 if np.signbit(x) else 0)


def _e4m3_half_gap(a):
    """Half the E4M3 spacing at magnitude a (the largest rounding error there)."""
    ex = -6 if a < 2 ** -6 else int(np.floor(np.log2(a)))
    return 2.0 ** (ex - 3) / 2


@pytest.mark.parametrize("scale", [1.0, 0.01, 37.0])
def test_fp8_group_error_bound_and_range(scale):
    rng = np.random.default_rng(3)
    for _ in range(200):
        x = (rng.normal(0, 1, 32) * scale).astype(np.float32)
        sh, codes = orc.quantize_group_fp8(x)
        s = orc.f16_value(sh)
        amax = float(np.max(np.abs(x)))
        assert s >= amax / 448 and s > 0
        for xi, c in zip(x, codes):
            r = np.float32(xi) / np.float32(s)
            assert abs(float(r)) <= 448
            xh = orc.e4m3_decode(int(c)) * s
            assert abs(xh - float(xi)) <= (_e4m3_half_gap(abs(float(r))) + 2 ** -20 * abs(float(r))) * s


def test_fp8_group_round_trip_of_representable_values():
    s_bits = orc.f16_rd(0.25)
    s = orc.f16_value(s_bits)
    codes = np.array([0x38, 0x39, 0x3F, 0x01, 0x7E, 0xB8, 0x00, 0x10] * 4, np.uint8)
    x = np.array([orc.e4m3_decode(int(c)) * s for c in codes], np.float32)
    sh, got = orc.quantize_group_fp8(x)
    assert orc.f16_value(sh) == s          # amax = 448 s, so the scale is s itself
    assert np.array_equal(got, codes)


def test_nvfp4_block_error_bound():
    rng = np.random.default_rng(4)
    for _ in range(300):
        x = (rng.normal(0, 1, 16) * rng.choice([0.01, 1.0, 30.0])).astype(np.float32)
        sc, codes = orc.quantize_block_nvfp4(x)
        s = orc.e4m3_decode(int(sc))
        amax = float(np.max(np.abs(x)))
        assert s >= amax / 6 and (sc == 0 or orc.e4m3_decode(int(sc) - 1) < np.float32(amax) / np.float32(6))
        for xi, c in zip(x, codes):
            r = abs(float(np.float32(xi) / np.float32(s)))
            assert r <= 6.0 + 1e-6
            gap = 0.5 if r <= 2 else (1.0 if r <= 4 else 2.0)
            xh = orc.e2m1_decode(int(c)) * s
            assert abs(xh - float(xi)) <= (gap / 2 + 1e-6) * s


def test_ternary_hand_cases():
    x = np.array([3.0, -3.0] + [0.25] * 30, np.float32)      # mean |x| = 0.421875, delta = 0.2953125
    sh, codes = orc.quantize_group_ternary(x)
    assert orc.f16_value(sh) == 3.0
    assert codes.tolist() == [1, 3] + [0] * 30
    x = np.full(32, -2.0, np.float32)                          # every element beyond delta = 1.4
    sh, codes = orc.quantize_group_ternary(x)
    assert orc.f16_value(sh) == 2.0 and codes.tolist() == [3] * 32
    sh, codes = orc.quantize_group_ternary(np.zeros(32, np.float32))
    assert orc.f16_value(sh) == 0.0 and codes.tolist() == [0] * 32


def test_ternary_scale_is_the_mean_magnitude_above_the_threshold():
    rng = np.random.default_rng(5)
    for _ in range(200):
        x = rng.normal(0, 1, 32).astype(np.float32)
        sh, codes = orc.quantize_group_ternary(x)
        delta = np.float32(0.7) * (np.float32(np.sum(np.abs(x), dtype=np.float32)) / np.float32(32))
        big = np.abs(x) > delta
        assert codes.tolist() == [1 if v > delta else (3 if v < -delta else 0) for v in x]
        assert abs(orc.f16_value(sh) - float(np.abs(x[big]).mean())) <= 2 ** -10 * float(np.abs(x[big]).mean()) + 1e-6


# --------------------------------------------------------------------------
# FP-class records in the cache (codec = 1: classes 1/2/3 = FP8 / NVFP4 / ternary)
# --------------------------------------------------------------------------
D = 128


def _codes_by_dim(block, bits, is_v):
    """Codes of a K or V block read at the positions the header's element order gives
    (the same order as the integer records of that width)."""
    out = np.zeros(D, np.int64)
    for dim in range(D):
        byte, bit = header_position(bits, is_v, dim)
        word = int.from_bytes(bytes(block[byte:byte + 4]), "little")
        out[dim] = (word >> bit) & ((1 << bits) - 1)
    return out


def _np_decode_record(fmt, rec):
    """Independent reading of the documented FP record layouts (numpy + torch)."""
    rec = np.asarray(rec, np.uint8)
    out = []
    for which in range(2):
        if fmt == orc.FMT_FP8:
            c = _codes_by_dim(rec[which * D:(which + 1) * D], 8, which == 1).astype(np.uint8)
            codes = torch.from_numpy(c).view(torch.float8_e4m3fn).double().numpy()
            sc = rec[2 * D:2 * D + 16].view(np.float16).astype(np.float64)[which * 4:(which + 1) * 4]
            out.append(codes * np.repeat(sc, 32))
        elif fmt == orc.FMT_NVFP4:
            nib = _codes_by_dim(rec[which * 64:(which + 1) * 64], 4, which == 1)
            mag = np.array(E2M1_TABLE)[nib & 7] * np.where(nib & 8, -1.0, 1.0)
            sc = torch.from_numpy(rec[D + which * 8:D + (which + 1) * 8].copy()).view(torch.float8_e4m3fn).double().numpy()
            out.append(mag * np.repeat(sc, 16))
        else:
            codes = _codes_by_dim(rec[which * 32:(which + 1) * 32], 2, which == 1)
            sc = rec[64:80].view(np.float16).astype(np.float64)[which * 4:(which + 1) * 4]
            out.append(np.select([codes == 1, codes == 3], [1.0, -1.0], 0.0) * np.repeat(sc, 32))
    return out


def test_fp_record_sizes():
    assert [orc.record_bytes_fmt(f) for f in (orc.FMT_FP8, orc.FMT_NVFP4, orc.FMT_TERNARY)] == [272, 144, 80]


@pytest.mark.parametrize("fmt", [108, 104, 102])
def test_fp_records_decode_as_documented(fmt):
    for t in range(20):
        k = synth.normal_bf16(t, 0, synth.TID_K, 1, 1, 0, 1, D)[0, 0, 0] * (1 + 5 * (t % 3))
        v = synth.normal_bf16(t, 0, synth.TID_V, 1, 1, 0, 1, D)[0, 0, 0]
        rec = orc.pack_record_fmt(fmt, bits_of(k), bits_of(v))
        kh, vh = orc.unpack_record_fmt(fmt, rec)
        nk, nv = _np_decode_record(fmt, rec)
        assert np.array_equal(kh, nk) and np.array_equal(vh, nv)
        # codes of each element are those of its own group / block quantiser
        x = k.float().numpy()
        if fmt == orc.FMT_FP8:
            sh, codes = orc.quantize_group_fp8(x[:32])
            assert np.array_equal(_codes_by_dim(rec[:D], 8, False)[:32], codes)
        elif fmt == orc.FMT_NVFP4:
            sc, codes = orc.quantize_block_nvfp4(x[:16])
            assert rec[D] == sc and np.array_equal(_codes_by_dim(rec[:64], 4, False)[:16], codes & 15)
        else:
            sh, codes = orc.quantize_group_ternary(x[:32])
            assert np.array_equal(_codes_by_dim(rec[:32], 2, False)[:32], codes)


def test_attention_over_fp_class_records_equals_softmax_over_the_decoded_records():
    B, Hkv, G, ctx = 1, 2, 4, 400
    cls = synth.class_ids(6, B, ctx, 0.4, 0.4)
    caps = [ctx] * 4
    cache = orc.OracleCache(B, Hkv, G, cap=caps, n_protect=4, codec=1)
    k = synth.normal_bf16(6, 0, synth.TID_K, B, Hkv, 0, ctx, D)
    v = synth.normal_bf16(6, 0, synth.TID_V, B, Hkv, 0, ctx, D)
    assert cache.append(bits_of(k), bits_of(v), cls.numpy(), synth.positions(B, 0, ctx).numpy()) == 0
    q = synth.normal_bf16(6, 0, synth.TID_Q, B, Hkv * G, ctx, 1, D)[:, :, 0]
    out = cache.attend(bits_of(q), 1 / np.sqrt(D))
    for s in range(Hkv):
        K, V = [], []
        for c in range(4):
            fmt = orc.class_format(orc.BITS[c], 1)
            for h in cache.live(s, c)[0]:
                rec = cache.state[f"pool{c}"][s, h]
                if fmt == 16:
                    kh, vh = orc.unpack_record_fmt(16, rec)
                else:
                    kh, vh = _np_decode_record(fmt, rec)
                K.append(kh)
                V.append(vh)
        K, V = np.array(K), np.array(V)
        qd = q[0, s * G:(s + 1) * G].double().numpy()
        sl = (qd @ K.T) / np.sqrt(D)
        p = np.exp(sl - sl.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        ref = p @ V
        assert np.max(np.abs(out[0, s * G:(s + 1) * G] - ref)) < 1e-6


def test_fp_class_cache_dense_matches_reuse_after_eviction():
    B, Hkv, G, ctx = 1, 1, 4, 300
    cls = synth.class_ids(7, B, ctx, 0.4, 0.4)
    k = synth.normal_bf16(7, 0, synth.TID_K, B, Hkv, 0, ctx, D)
    v = synth.normal_bf16(7, 0, synth.TID_V, B, Hkv, 0, ctx, D)
    q = synth.normal_bf16(7, 0, synth.TID_Q, B, Hkv * G, ctx, 1, D)[:, :, 0]
    caches = []
    for dense in (False, True):
        c = orc.OracleCache(B, Hkv, G, cap=[ctx] * 4, n_protect=4, dense=dense, codec=1)
        assert c.append(bits_of(k), bits_of(v), cls.numpy(), synth.positions(B, 0, ctx).numpy()) == 0
        c.attend(bits_of(q), 1 / np.sqrt(D))
        assert c.evict(60) == 0
        caches.append(c)
    ct, dn = caches
    for c in range(4):
        n = ct.state["n"][0, c]
        assert dn.state["n"][0, c] == n
        for i, h in enumerate(ct.state[f"handle{c}"][0, :n]):
            assert np.array_equal(dn.state[f"pool{c}"][0, i], ct.state[f"pool{c}"][0, h])
    out_ct = ct.attend(bits_of(q), 1 / np.sqrt(D))
    out_dn = dn.attend(bits_of(q), 1 / np.sqrt(D))
    assert np.array_equal(out_ct, out_dn)


# --------------------------------------------------------------------------
# attention sparsity of a step (ThinKV, Metodologia: thought types differ in the
# sparsity of their attention); measure 1 - H(p) / ln N
# --------------------------------------------------------------------------
def _bf16_cache_with_key_column(col0):
    """All-bf16 cache whose keys are zero except dimension 0 = col0 (exact in bf16)."""
    N = len(col0)
    cache = orc.OracleCache(1, 1, 1, cap=[N, 0, 0, 0], n_protect=N)
    k = torch.zeros((1, 1, N, D), dtype=torch.bfloat16)
    k[0, 0, :, 0] = torch.tensor(col0, dtype=torch.float32).to(torch.bfloat16)
    v = torch.zeros_like(k)
    assert cache.append(bits_of(k), bits_of(v), np.ones((1, N), np.uint8),
                        np.arange(N, dtype=np.int32).reshape(1, N)) == 0
    q = torch.zeros((1, 1, D), dtype=torch.bfloat16)
    q[0, 0, 0] = 1.0
    return cache, bits_of(q)


def test_sparsity_uniform_attention_is_zero():
    cache, q = _bf16_cache_with_key_column([2.0] * 50)
    assert abs(cache.attention_sparsity(q, 1.0)[0, 0]) < 1e-12


@pytest.mark.parametrize("m,N,a,b", [(1, 10, 3.0, 0.0), (5, 40, 1.0, -2.0), (30, 64, 0.5, 0.25)])
def test_sparsity_two_level_closed_form(m, N, a, b):
    cache, q = _bf16_cache_with_key_column([a] * m + [b] * (N - m))
    z = m * np.exp(a) + (N - m) * np.exp(b)
    ph, pl = np.exp(a) / z, np.exp(b) / z
    H = -(m * ph * np.log(ph) + (N - m) * pl * np.log(pl))
    assert abs(cache.attention_sparsity(q, 1.0)[0, 0] - (1 - H / np.log(N))) < 1e-12


def test_sparsity_one_dominant_token_and_degenerate_sizes():
    cache, q = _bf16_cache_with_key_column([40.0] + [0.0] * 99)
    assert cache.attention_sparsity(q, 1.0)[0, 0] > 0.99
    cache, q = _bf16_cache_with_key_column([1.0])
    assert cache.attention_sparsity(q, 1.0)[0, 0] == 0.0


def test_sparsity_classification_thresholds():
    assert [orc.classify_sparsity(s, 0.3, 0.6) for s in (0.0, 0.29, 0.3, 0.59, 0.6, 1.0)] == [2, 2, 1, 1, 3, 3]
