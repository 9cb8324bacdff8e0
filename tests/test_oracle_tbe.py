"""Pins of the oracle's segment-level eviction (ThinKV, Metodologia, TBE) and of its
annealing schedule.  CPU only.

The segment selection is pinned by (1) its reduction to the token-level eviction,
which is itself pinned against brute force over all subsets, when one segment holds
every candidate; (2) the defining property of a per-segment top-r, checked pairwise
on random caches; (3) the entries the reading always keeps.  The schedule is pinned by
the page's own 64 -> 32 -> 16 sequence and hand-derived rows (tests/golden)."""
from pathlib import Path

import numpy as np
import pytest

import synth
from oracle import oracle as orc
from tests.helpers import bits_of
from tests.test_oracle import _check_table_invariants, _order_key

D = 128
GOLDEN = Path(__file__).parent / "golden" / "tbe_schedule.txt"


def _golden_rows():
    rows = []
    for line in GOLDEN.read_text().splitlines():
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        lab, exp = line.split("|")
        rows.append(([int(x) for x in lab.split()], [int(x) for x in exp.split()]))
    return rows


@pytest.mark.parametrize("labels,expected", _golden_rows())
def test_schedule_golden_rows(labels, expected):
    assert orc.tbe_schedule(labels, 64, 16).tolist() == expected


def test_schedule_pages_sequence_for_any_r0():
    """One R segment followed by k transitions keeps r0, r0/2, r0/4, ... and reaches 0."""
    for r0 in (64, 100, 7):
        got = [int(orc.tbe_schedule([1] + [3] * k, r0, 5)[0]) for k in range(1, 12)]
        assert got == [r0 >> (k - 1) for k in range(1, 12)]
        assert got[-1] == 0


def test_schedule_rejects_bad_arguments():
    with pytest.raises(ValueError):
        orc.tbe_schedule([1, 4], 64, 16)
    with pytest.raises(ValueError):
        orc.tbe_schedule([1, 3], -1, 16)


def _cache(rng, n_tok, n_protect, cls, score_pool, dense=False, Hkv=1):
    cache = orc.OracleCache(1, Hkv, 1, cap=[n_tok] * 4, n_protect=n_protect, dense=dense)
    k = synth.normal_bf16(int(rng.integers(1 << 20)), 0, synth.TID_K, 1, Hkv, 0, n_tok, D)
    pos = np.arange(n_tok, dtype=np.int32).reshape(1, n_tok)
    assert cache.append(bits_of(k), bits_of(k), cls.reshape(1, n_tok), pos) == 0
    for s in range(Hkv):
        for c in range(4):
            n = cache.state["n"][s, c]
            cache.state[f"score{c}"][s, :n] = rng.choice(score_pool, size=n).astype(np.float32)
    return cache


@pytest.mark.parametrize("dense", [False, True])
@pytest.mark.parametrize("trial", range(12))
def test_one_segment_equals_token_level_eviction(trial, dense):
    """All candidates in one class and one segment with retention r: the segment
    eviction must leave exactly the state the token-level eviction to r leaves."""
    rng = np.random.default_rng(300 + trial)
    n_tok = int(rng.integers(5, 60))
    n_protect = int(rng.integers(0, 4))
    c = int(rng.integers(1, 4))
    cls = np.full(n_tok, c, np.uint8)
    pool = [0.0, 0.5, 0.5, 1.0] if trial % 2 else list(rng.random(30))
    a = _cache(rng, n_tok, n_protect, cls, pool, dense, Hkv=2)
    b = orc.OracleCache(1, 2, 1, cap=a.cap, n_protect=n_protect, dense=dense)
    b.load_state(a.copy_state())
    r = int(rng.integers(0, n_tok + 2))
    starts = np.array([[0]], np.int32)
    labels = np.array([[c]], np.uint8)
    keeps = np.array([[r]], np.int32)
    assert a.evict_segments(starts, labels, keeps, np.array([1], np.int32)) == 0
    assert b.evict(r) == 0
    for key in a.state:
        assert np.array_equal(a.state[key], b.state[key]), key


def _segments(rng, n_tok):
    """Random segmentation of [first, n_tok): starts, labels, retention per segment."""
    first = int(rng.integers(0, 3))
    starts, t = [], first
    while t < n_tok:
        starts.append(t)
        t += int(rng.integers(1, 9))
    ns = len(starts)
    labels = rng.integers(0, 4, size=ns).astype(np.uint8)
    keeps = rng.choice([-1, 0, 1, 2, 3, 5, 50], size=ns).astype(np.int32)
    return np.array(starts, np.int32), labels, keeps


def _seg_of(starts, p):
    j = -1
    for k, s0 in enumerate(starts):
        if s0 <= p:
            j = k
    return j


def _random_case(trial):
    rng = np.random.default_rng(700 + trial)
    n_tok = int(rng.integers(4, 70))
    n_protect = int(rng.integers(0, 5))
    starts, labels, keeps = _segments(rng, n_tok)
    # token classes follow their segment's label, except a few foreign ones
    cls = np.zeros(n_tok, np.uint8)
    for p in range(n_tok):
        j = _seg_of(starts, p)
        cls[p] = labels[j] if j >= 0 else rng.integers(0, 4)
        if rng.random() < 0.1:
            cls[p] = rng.integers(0, 4)
    pool = [0.0, 0.25, 0.25, 1.0] if trial % 3 == 0 else list(rng.random(40))
    return rng, n_tok, n_protect, starts, labels, keeps, cls, pool


@pytest.mark.parametrize("trial", range(25))
def test_each_segment_keeps_its_top_r(trial):
    rng, n_tok, n_protect, starts, labels, keeps, cls, pool = _random_case(trial)
    cache = _cache(rng, n_tok, n_protect, cls, pool)
    before = cache.copy_state()
    ns = len(starts)
    assert cache.evict_segments(starts.reshape(1, ns), labels.reshape(1, ns), keeps.reshape(1, ns),
                                np.array([ns], np.int32)) == 0
    kept = set()
    for c in range(4):
        kept |= set(cache.live(0, c)[1].tolist())
    # every entry before: (score, pos, class, index)
    groups = {}
    for c in range(4):
        for i in range(before["n"][0, c]):
            p = int(before[f"pos{c}"][0, i])
            sc = before[f"score{c}"][0, i]
            j = _seg_of(starts, p)
            ranked = p >= n_protect and j >= 0 and labels[j] == c and keeps[j] >= 0
            if not ranked:
                assert p in kept, "protected, unsegmented, foreign or keep-all entries stay"
                continue
            groups.setdefault(j, []).append((sc, p, c, i))
    for j, ent in groups.items():
        kin = [e for e in ent if e[1] in kept]
        kout = [e for e in ent if e[1] not in kept]
        assert len(kin) == min(len(ent), int(keeps[j]))
        for a in kin:                        # every kept entry precedes every evicted one
            for b in kout:
                assert _order_key(*a) < _order_key(*b)
    _check_table_invariants(cache, before)


@pytest.mark.parametrize("trial", range(10))
def test_dense_placement_matches_in_place_reuse(trial):
    """Same tables in both placements; dense records sit at slot = table index and
    equal the records the reuse placement keeps at their handles."""
    rng, n_tok, n_protect, starts, labels, keeps, cls, pool = _random_case(trial)
    ct = _cache(np.random.default_rng(trial), n_tok, n_protect, cls, pool)
    dn = orc.OracleCache(1, 1, 1, cap=ct.cap, n_protect=n_protect, dense=True)
    dn.load_state(ct.copy_state())   # no eviction yet: handle[i] == i, records identical
    ns = len(starts)
    args = (starts.reshape(1, ns), labels.reshape(1, ns), keeps.reshape(1, ns), np.array([ns], np.int32))
    assert ct.evict_segments(*args) == 0 and dn.evict_segments(*args) == 0
    for c in range(4):
        n = ct.state["n"][0, c]
        assert dn.state["n"][0, c] == n and dn.state["hw"][0, c] == n and dn.state["ft"][0, c] == 0
        assert np.array_equal(ct.state[f"pos{c}"][0, :n], dn.state[f"pos{c}"][0, :n])
        assert np.array_equal(ct.state[f"score{c}"][0, :n], dn.state[f"score{c}"][0, :n])
        assert dn.state[f"handle{c}"][0, :n].tolist() == list(range(n))
        for i, h in enumerate(ct.state[f"handle{c}"][0, :n]):
            assert np.array_equal(dn.state[f"pool{c}"][0, i], ct.state[f"pool{c}"][0, h])


def test_equal_scores_keep_the_earliest_positions_of_each_segment():
    rng = np.random.default_rng(5)
    n_tok = 40
    cls = np.full(n_tok, 2, np.uint8)
    cache = _cache(rng, n_tok, 0, cls, [0.5])
    starts = np.array([[0, 10, 25]], np.int32)
    labels = np.array([[2, 2, 2]], np.uint8)
    keeps = np.array([[3, -1, 0]], np.int32)
    assert cache.evict_segments(starts, labels, keeps, np.array([3], np.int32)) == 0
    assert cache.live(0, 2)[1].tolist() == [0, 1, 2] + list(range(10, 25))


def test_no_segments_is_a_no_op():
    rng = np.random.default_rng(6)
    cache = _cache(rng, 20, 2, rng.integers(0, 4, 20).astype(np.uint8), [0.1, 0.2])
    before = cache.copy_state()
    z = np.zeros((1, 4), np.int32)
    assert cache.evict_segments(z, z.astype(np.uint8), z - 1, np.array([0], np.int32)) == 0
    for key in before:
        assert np.array_equal(before[key], cache.state[key])


# --------------------------------------------------------------------------
# thought-aware budgets with pivotal tokens (TAM page, sections 2.B-2.C)
# --------------------------------------------------------------------------
def _cache_with_scores(n_tok, cls, scores, n_protect=0, dense=False):
    cache = orc.OracleCache(1, 1, 1, cap=[n_tok] * 4, n_protect=n_protect, dense=dense)
    k = synth.normal_bf16(3, 0, synth.TID_K, 1, 1, 0, n_tok, D)
    pos = np.arange(n_tok, dtype=np.int32).reshape(1, n_tok)
    assert cache.append(bits_of(k), bits_of(k), cls.reshape(1, n_tok), pos) == 0
    for c in range(4):
        n = cache.state["n"][0, c]
        p = cache.state[f"pos{c}"][0, :n]
        cache.state[f"score{c}"][0, :n] = scores[p]
    return cache


def test_tam_budgets_follow_sqrt_w_times_n():
    """Three R segments of 10, 20 and 30 tokens with constant scores 1, 4 and 9
    (sqrt w = 1, 2, 3): sum sqrt(w) n = 140, so a budget of 70 gives 5, 20 and 45,
    the last capped at its 30 tokens.  c = 10 puts delta (60) above every score."""
    n_tok = 60
    scores = np.array([1.0] * 10 + [4.0] * 20 + [9.0] * 30, np.float32)
    cache = _cache_with_scores(n_tok, np.full(n_tok, 1, np.uint8), scores)
    st = np.array([[0, 10, 30]], np.int32)
    assert cache.evict_tam(st, np.array([[1, 1, 1]], np.uint8), np.array([3], np.int32), 70, 10.0) == 0
    kept = cache.live(0, 1)[1].tolist()
    # equal scores inside a segment: the earliest positions stay
    assert kept == list(range(0, 5)) + list(range(10, 30)) + list(range(30, 60))


def test_tam_pivotal_tokens_are_kept_and_leave_the_rest_of_the_budget():
    """Mean score 1.0 and c = 3: the two tokens scoring 9 are pivotal and kept; the
    remaining budget 10 - 2 = 8 splits as for scores without them."""
    n_tok = 40
    scores = np.full(n_tok, 0.5, np.float32)
    scores[[7, 33]] = 9.0
    scores[20:] = 0.5 + np.arange(20, dtype=np.float32) / 1000.0
    scores[33] = 9.0
    cache = _cache_with_scores(n_tok, np.full(n_tok, 2, np.uint8), scores)
    mean = float(scores.astype(np.float64).mean())
    assert 3 * mean < 9.0 and np.sort(scores)[-3] < 3 * mean   # exactly two pivotal tokens
    st = np.array([[0, 20]], np.int32)
    assert cache.evict_tam(st, np.array([[2, 2]], np.uint8), np.array([2], np.int32), 10, 3.0) == 0
    kept = set(cache.live(0, 2)[1].tolist())
    assert {7, 33} <= kept
    # budgets by hand: w over each segment's candidates (pivotal included), T' = 8
    w0 = scores[:20].astype(np.float64).mean()
    w1 = scores[20:].astype(np.float64).mean()
    Dn = np.sqrt(w0) * 20 + np.sqrt(w1) * 20
    t0 = int(np.floor(8 * (np.sqrt(w0) * 20 / Dn) + 1e-9))
    t1 = int(np.floor(8 * (np.sqrt(w1) * 20 / Dn) + 1e-9))
    seg0 = sorted(p for p in kept if p < 20 and p != 7)
    seg1 = sorted(p for p in kept if p >= 20 and p != 33)
    assert seg0 == list(range(t0))                               # equal scores: earliest
    order1 = sorted(range(20, 40), key=lambda p: (-scores[p], p))
    assert seg1 == sorted([p for p in order1 if p != 33][:t1])


@pytest.mark.parametrize("dense", [False, True])
@pytest.mark.parametrize("trial", range(8))
def test_tam_one_segment_without_pivotal_equals_token_level_eviction(trial, dense):
    """One segment holding every candidate and no pivotal token (c huge): its budget
    is min(n, budget), i.e. the token-level eviction."""
    rng = np.random.default_rng(900 + trial)
    n_tok = int(rng.integers(5, 60))
    n_protect = int(rng.integers(0, 4))
    c = int(rng.integers(1, 4))
    a = _cache(rng, n_tok, n_protect, np.full(n_tok, c, np.uint8), list(rng.random(30) + 0.1), dense, Hkv=2)
    b = orc.OracleCache(1, 2, 1, cap=a.cap, n_protect=n_protect, dense=dense)
    b.load_state(a.copy_state())
    r = int(rng.integers(0, n_tok + 2))
    assert a.evict_tam(np.array([[0]], np.int32), np.array([[c]], np.uint8), np.array([1], np.int32),
                       r, 1e30) == 0
    assert b.evict(r) == 0
    for key in a.state:
        assert np.array_equal(a.state[key], b.state[key]), key


@pytest.mark.parametrize("trial", range(20))
def test_tam_keeps_pivotal_and_per_segment_top_t(trial):
    rng, n_tok, n_protect, starts, labels, keeps, cls, pool = _random_case(trial)
    cache = _cache(rng, n_tok, n_protect, cls, pool)
    before = cache.copy_state()
    ns = len(starts)
    budget, cc = int(rng.integers(0, n_tok)), float(rng.choice([0.5, 1.5, 3.0]))
    assert cache.evict_tam(starts.reshape(1, ns), labels.reshape(1, ns), np.array([ns], np.int32),
                           budget, cc) == 0
    kept = set()
    for c in range(4):
        kept |= set(cache.live(0, c)[1].tolist())
    groups, allc = {}, []
    for c in range(4):
        for i in range(before["n"][0, c]):
            p = int(before[f"pos{c}"][0, i])
            sc = before[f"score{c}"][0, i]
            j = _seg_of(starts, p)
            if p < n_protect or j < 0 or labels[j] != c:
                assert p in kept
                continue
            groups.setdefault(j, []).append((sc, p, c, i))
            allc.append(float(sc))
    if not allc:
        return
    delta = cc * (sum(np.float64(x) for x in allc) / len(allc))
    nonpiv_kept = 0
    for j, ent in groups.items():
        piv = [e for e in ent if np.float64(e[0]) >= delta]
        rest = [e for e in ent if np.float64(e[0]) < delta]
        assert all(e[1] in kept for e in piv)
        kin = [e for e in rest if e[1] in kept]
        kout = [e for e in rest if e[1] not in kept]
        nonpiv_kept += len(kin)
        for a in kin:
            for b in kout:
                assert _order_key(*a) < _order_key(*b)
    P = sum(1 for x in allc if np.float64(x) >= delta)
    assert nonpiv_kept <= max(0, budget - P)
    _check_table_invariants(cache, before)


# --------------------------------------------------------------------------
# exact score sums behind the TAM means (TAM page, sections 2.B-2.C)
# --------------------------------------------------------------------------
def _wide_f32(rng, n):
    """fp32 values spread over the whole exponent range, subnormals and zeros included."""
    e = rng.integers(-149, 128, n)
    m = rng.random(n) + 0.5
    v = np.ldexp(m, e).astype(np.float32)          # overflow to inf is dropped below
    v[rng.random(n) < 0.1] = 0.0
    v[rng.random(n) < 0.1] = np.float32(1e-45) * rng.integers(1, 1 << 23, 1).astype(np.float32)
    return v[np.isfinite(v)]


@pytest.mark.parametrize("trial", range(12))
def test_exact_sum_is_the_correctly_rounded_sum(trial):
    """math.fsum returns the exact sum of its (double) inputs rounded once; every fp32
    is a double, so the two must agree bit for bit, in any order of the terms."""
    import math
    rng = np.random.default_rng(4400 + trial)
    n = int(rng.integers(0, 3000))
    v = _wide_f32(rng, n) if trial % 2 else (rng.random(n) * 3).astype(np.float32)
    want = math.fsum(float(x) for x in v)
    assert orc.sum_f32_exact(v) == want
    assert orc.sum_f32_exact(v[rng.permutation(len(v))]) == want


def test_exact_sum_cancellation_free_cases():
    """Closed forms: 2^24 + 1 + 1 (a naive fp32 loop returns 2^24), 2^k tails far below
    the leading term, the largest and smallest fp32, and the rule for negative and
    non-finite terms (they count as 0)."""
    big = np.float32(2.0 ** 24)
    assert orc.sum_f32_exact(np.array([big, 1, 1], np.float32)) == 2.0 ** 24 + 2
    tiny = np.float32(2.0 ** -149)
    assert orc.sum_f32_exact(np.array([tiny] * 3, np.float32)) == 3 * 2.0 ** -149
    v = np.array([2.0 ** 100, 2.0 ** -100], np.float32)
    assert orc.sum_f32_exact(v) == 2.0 ** 100                      # 2^-200 relative: rounds away
    v = np.array([2.0 ** 20, 2.0 ** -33, 2.0 ** -33], np.float32)   # exactly 2^20 + 2^-32: one ulp up
    assert orc.sum_f32_exact(v) == 2.0 ** 20 + 2.0 ** -32
    fmax = float(np.finfo(np.float32).max)
    assert orc.sum_f32_exact(np.array([fmax] * 5, np.float32)) == 5 * fmax
    assert orc.sum_f32_exact(np.array([1.5, -7.0, np.inf, np.nan, 2.5], np.float32)) == 4.0
    assert orc.sum_f32_exact(np.zeros(0, np.float32)) == 0.0
    # 2^60 + 2^-60 + 2^-60: one rounding of the exact sum (ties to even are not reached)
    v = np.array([2.0 ** 60, 2.0 ** -60, 2.0 ** -60], np.float32)
    assert orc.sum_f32_exact(v) == 2.0 ** 60


def test_tam_delta_is_the_exact_mean():
    """Scores 2^24 then 2^24 ones: the exact mean is (2^24 + n) / (n + 1), which a
    running fp32 sum would lose; c = 1 then makes exactly the first token pivotal."""
    n_tok = 33
    scores = np.ones(n_tok, np.float32)
    scores[0] = np.float32(2.0 ** 24)
    cache = _cache_with_scores(n_tok, np.full(n_tok, 1, np.uint8), scores)
    st = np.array([[0]], np.int32)
    assert cache.evict_tam(st, np.array([[1]], np.uint8), np.array([1], np.int32), 4, 1.0) == 0
    kept = cache.live(0, 1)[1].tolist()
    # pivotal: position 0 (2^24 >= mean); T' = 3; t = min(32, floor(3 * 1 + 1e-9)) = 3
    assert kept == [0, 1, 2, 3]
