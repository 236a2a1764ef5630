"""Pins for the CPU oracle: every check compares it with something other than
itself -- a closed form, a textbook special case, an invariant, a library
routine on a special case, or brute force.  CPU only.

Source page: "The future-offset average in TriAttention can be precomputed".
"""
import cmath
import json
import math
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16(x):
    """Round a float array to bf16; return (uint16 bits, exact float64 values)."""
    t = torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)
    bits = t.view(torch.int16).numpy().view(np.uint16).copy()
    vals = t.to(torch.float64).numpy()
    return bits, vals


def rand_case(n, d, seed, spread=0.3):
    rng = np.random.default_rng(seed)
    c = rng.standard_normal(d)
    k = c + spread * rng.standard_normal((n, d))
    k[rng.random(n) < 0.05] *= 5.0
    bits, vals = bf16(k)
    q = rng.standard_normal(d).astype(np.float32)
    return bits, vals, q


def band_pairs(d, pairing):
    if pairing == 0:
        return [(f, f + d // 2) for f in range(d // 2)]
    return [(2 * f, 2 * f + 1) for f in range(d // 2)]


def textbook_omega(theta, d):
    # inverse frequencies as RoPE implementations write them: 1 / theta^(2i/d)
    return 1.0 / (theta ** (np.arange(0, d, 2, dtype=np.float64) / d))


def rope(x, pos, theta, pairing):
    """Textbook RoPE of vectors x [n][d] at position pos (rotate-half or interleaved)."""
    d = x.shape[-1]
    om = textbook_omega(theta, d)
    ang = pos * om
    c, s = np.cos(ang), np.sin(ang)
    y = np.empty_like(x)
    if pairing == 0:
        x1, x2 = x[..., : d // 2], x[..., d // 2:]
        y[..., : d // 2] = x1 * c - x2 * s
        y[..., d // 2:] = x2 * c + x1 * s
    else:
        x1, x2 = x[..., 0::2], x[..., 1::2]
        y[..., 0::2] = x1 * c - x2 * s
        y[..., 1::2] = x2 * c + x1 * s
    return y


ALL_FORMS = ("cosine", "literal", "folded", "polar", "realdot")


def all_scores(orc, bits, q, theta, D, delta0, pairing):
    out = {
        "cosine": orc.score_cosine(bits, q, theta, D, delta0, pairing),
        "literal": orc.score_literal(bits, q, theta, D, delta0, pairing),
        "folded": orc.score_folded(bits, q, theta, D, delta0, pairing),
        "polar": orc.score_polar(bits, q, theta, D, delta0, pairing),
    }
    w = orc.fold_w(q[None, :], theta, D, delta0, pairing)[0]
    out["realdot"] = orc.score_realdot(bits, w)
    return out


# ------------------------------------------------------------ page values

def test_page_parameters_fixture():
    g = json.load(open(os.path.join(GOLDEN, "page_parameters.json")))
    assert g["offset_schedule"]["value"] == [2 ** e for e in range(17)]
    import gen
    assert list(gen.WORKLOADS["tiny"].offsets) == [float(x) for x in g["offset_schedule"]["value"]]
    assert gen.WORKLOADS["tiny"].theta == g["rotary_base_theta"]["value"]
    assert gen.WORKLOADS["qwen3_full"].budget == g["kv_budget_default"]["value"]
    assert gen.WORKLOADS["llama3_long"].budget == g["kv_budget_chat"]["value"]


def test_frequencies_closed_values(orc):
    # theta = 10000, d = 128: omega_f = 10^(-f/16): 1, 0.1, 0.01, 0.001 at f = 0, 16, 32, 48
    om = orc.frequencies(10000.0, 128)
    assert om.shape == (64,)
    for f, v in ((0, 1.0), (16, 0.1), (32, 0.01), (48, 0.001)):
        assert om[f] == pytest.approx(v, rel=1e-15)
    # geometric with ratio theta^(-2/d)
    r = om[1:] / om[:-1]
    assert np.allclose(r, 10000.0 ** (-2.0 / 128), rtol=1e-14)
    np.testing.assert_allclose(om, textbook_omega(10000.0, 128), rtol=1e-14)


# ------------------------------------------------------------ W_f

@pytest.mark.parametrize("theta,M", [(5e5, 1024), (1e4, 7), (1e6, 100)])
def test_offset_weight_uniform_dirichlet(orc, theta, M):
    """D = {1..M}: the geometric series sum_{k=1}^M e^{ik w} in closed form."""
    D = [float(i) for i in range(1, M + 1)]
    W = orc.offset_weights(theta, 128, D)
    for f, w in enumerate(textbook_omega(theta, 128)):
        if abs(math.sin(w / 2)) < 1e-300:
            ref = 1.0
        else:
            ref = cmath.exp(1j * w * (M + 1) / 2) * math.sin(M * w / 2) / math.sin(w / 2) / M
        assert abs(W[f] - ref) < 1e-11, (f, W[f], ref)


@pytest.mark.parametrize("theta", [1e4, 1e6])
def test_offset_weight_geometric_by_squaring(orc, theta):
    """D = {2^0..2^16}: e^{i w 2^(k+1)} = (e^{i w 2^k})^2, so W is the mean of
    17 repeated squares of e^{i w} -- no trig of large arguments involved."""
    D = [float(2 ** e) for e in range(17)]
    W = orc.offset_weights(theta, 128, D)
    for f, w in enumerate(textbook_omega(theta, 128)):
        z = complex(math.cos(w), math.sin(w))
        acc = 0j
        for _ in range(17):
            acc += z
            z = z * z
            z /= abs(z)          # keep the unit length against drift
        assert abs(W[f] - acc / 17) < 1e-9, f


def test_offset_weight_singleton_and_bound(orc):
    rng = np.random.default_rng(3)
    d0 = 12345.0
    W = orc.offset_weights(1e4, 128, [d0])
    np.testing.assert_allclose(W, np.exp(1j * textbook_omega(1e4, 128) * d0), atol=1e-12)
    for _ in range(5):
        D = rng.uniform(0, 1e5, size=rng.integers(1, 40))
        W = orc.offset_weights(1e6, 128, D)
        assert np.all(np.abs(W) <= 1 + 1e-12)
    # a duplicated offset counts twice (D is a multiset)
    W2 = orc.offset_weights(1e4, 128, [1.0, 1.0, 8.0])
    om = textbook_omega(1e4, 128)
    np.testing.assert_allclose(W2, (2 * np.exp(1j * om) + np.exp(8j * om)) / 3, atol=1e-13)


# ------------------------------------------------------------ special cases

@pytest.mark.parametrize("pairing", [0, 1])
def test_zero_offset_is_plain_dot(orc, pairing):
    """D = {0}, delta0 = 0: every form reduces to the real dot product q . k."""
    bits, vals, q = rand_case(64, 128, seed=1)
    ref = vals @ q.astype(np.float64)
    for name, s in all_scores(orc, bits, q, 1e4, [0.0], 0.0, pairing).items():
        np.testing.assert_allclose(s, ref, rtol=1e-11, atol=1e-10, err_msg=name)


@pytest.mark.parametrize("pairing", [0, 1])
@pytest.mark.parametrize("theta,m,n,delta0", [(1e4, 70000, 4464, 0.0), (1e6, 300, 297, 0.0),
                                              (1e4, 9000, 100, 3.0)])
def test_single_offset_is_textbook_rope(orc, pairing, theta, m, n, delta0):
    """D = {delta}: the score is RoPE(q at m) . RoPE(k at n) with m - n = delta0 + delta.
    Pins the sign of the rotation, the conjugation and the band pairing."""
    bits, vals, q = rand_case(48, 128, seed=2)
    delta = float(m - n) - delta0
    qr = rope(q.astype(np.float64)[None, :], m, theta, pairing)[0]
    kr = rope(vals, n, theta, pairing)
    ref = kr @ qr
    scale = np.abs(vals) @ np.abs(q.astype(np.float64))
    for name, s in all_scores(orc, bits, q, theta, [delta], delta0, pairing).items():
        assert np.all(np.abs(s - ref) <= 1e-9 * scale), name
    # the opposite sign convention would fail
    qr_bad = rope(q.astype(np.float64)[None, :], n, theta, pairing)[0]
    kr_bad = rope(vals, m, theta, pairing)
    assert np.max(np.abs(kr_bad @ qr_bad - ref)) > 1e-3


@pytest.mark.parametrize("pairing", [0, 1])
@pytest.mark.parametrize("f", [0, 5, 31, 63])
def test_single_band_closed_form(orc, pairing, f):
    """A key with only band f non-zero, D = {1..M}:
    mean_k cos(w(delta0 + k) + phi) = sin(Mw/2)/(M sin(w/2)) * cos(w delta0 + phi + (M+1)w/2)
    (Lagrange's trigonometric identity), times |q_f| |k_f|."""
    d, M, theta, delta0 = 128, 50, 1e4, 7.0
    re, im = band_pairs(d, pairing)[f]
    kv = np.zeros((1, d))
    kv[0, re], kv[0, im] = 1.5, -0.75          # exact in bf16
    bits, vals = bf16(kv)
    rng = np.random.default_rng(f)
    q = rng.standard_normal(d).astype(np.float32)
    w = textbook_omega(theta, d)[f]
    qf = complex(float(q[re]), float(q[im]))
    kf = complex(1.5, -0.75)
    phi = cmath.phase(qf) - cmath.phase(kf)
    dir_ = math.sin(M * w / 2) / (M * math.sin(w / 2))
    ref = abs(qf) * abs(kf) * dir_ * math.cos(w * delta0 + phi + (M + 1) * w / 2)
    D = [float(i) for i in range(1, M + 1)]
    for name, s in all_scores(orc, bits, q, theta, D, delta0, pairing).items():
        assert s[0] == pytest.approx(ref, rel=1e-10, abs=1e-12), name


@pytest.mark.parametrize("pairing", [0, 1])
def test_cosine_equals_complex_band_by_band(orc, pairing):
    """Cosine form and complex form, one band at a time (single-band keys)."""
    d = 128
    rng = np.random.default_rng(11)
    q = rng.standard_normal(d).astype(np.float32)
    D = [float(2 ** e) for e in range(17)]
    rows = []
    for f, (re, im) in enumerate(band_pairs(d, pairing)):
        r = np.zeros(d)
        r[re], r[im] = rng.standard_normal(2)
        rows.append(r)
    bits, vals = bf16(np.array(rows))
    c = orc.score_cosine(bits, q, 1e4, D, 0.0, pairing)
    l = orc.score_literal(bits, q, 1e4, D, 0.0, pairing)
    scale = np.array([abs(complex(q[a], q[b])) * abs(complex(v[a], v[b]))
                      for v, (a, b) in zip(vals, band_pairs(d, pairing))])
    assert np.all(np.abs(c - l) <= 1e-12 * scale + 1e-300)


# ------------------------------------------------------------ fold identity

@pytest.mark.parametrize("pairing", [0, 1])
@pytest.mark.parametrize("theta,D,delta0", [
    (1e4, [float(2 ** e) for e in range(17)], 0.0),
    (1e6, [float(2 ** e) for e in range(17)], 123.0),
    (5e5, [float(i) for i in range(1, 1025)], 0.0),
    (1e4, [3.0, 3.0, 17.5, 1000.25], 2.5),
])
def test_folded_equals_literal(orc, pairing, theta, D, delta0):
    """Folded forms (complex, polar, real 2x2 map) equal the literal average."""
    bits, vals, q = rand_case(96, 128, seed=5)
    s = all_scores(orc, bits, q, theta, D, delta0, pairing)
    scale = np.abs(vals) @ np.abs(q.astype(np.float64))
    for name in ALL_FORMS:
        err = np.abs(s[name] - s["literal"]) / scale
        assert err.max() <= 1e-10, (name, err.max())


def test_fold_w_is_a_real_map_of_the_center(orc):
    """w is linear in the center and independent of the keys."""
    rng = np.random.default_rng(9)
    D = [float(2 ** e) for e in range(17)]
    a = rng.standard_normal(128).astype(np.float32)
    b = rng.standard_normal(128).astype(np.float32)
    wa = orc.fold_w(a[None], 1e6, D)[0]
    wb = orc.fold_w(b[None], 1e6, D)[0]
    wab = orc.fold_w((a + b)[None], 1e6, D)[0]
    np.testing.assert_allclose(wab, wa + wb, atol=1e-6)
    # batch of centers == one at a time
    wbatch = orc.fold_w(np.stack([a, b]), 1e6, D)
    np.testing.assert_array_equal(wbatch[0], wa)
    np.testing.assert_array_equal(wbatch[1], wb)


def test_ranks_unchanged_bruteforce(orc):
    """Tiny inputs, random schedules: the full order of the keys under the
    literal average equals the order under the folded score."""
    rng = np.random.default_rng(21)
    for trial in range(30):
        d = int(rng.choice([4, 8, 128]))
        n = int(rng.integers(2, 65))
        bits, vals, q = rand_case(n, d, seed=100 + trial)
        D = list(rng.choice([1.0, 2.0, 4.0, 16.0, 1000.0, 65536.0, 3.5], size=rng.integers(1, 8)))
        theta = float(rng.choice([1e4, 1e6, 5e5]))
        lit = orc.score_literal(bits, q, theta, D)
        w = orc.fold_w(q[None], theta, D)[0]
        fol = orc.score_realdot(bits, w)
        scale = np.abs(vals) @ np.abs(w)
        order_l = sorted(range(n), key=lambda i: (-lit[i], i))
        order_f = sorted(range(n), key=lambda i: (-fol[i], i))
        # positions may differ only inside groups of (near) ties
        for a, b in zip(order_l, order_f):
            if a != b:
                assert abs(lit[a] - lit[b]) <= 1e-12 * (scale[a] + scale[b])


def test_max_over_offsets_does_not_fold(orc):
    """The fold needs a linear aggregate: a max over offsets differs from
    the folded mean (so the max variant needs its own kernel)."""
    bits, vals, q = rand_case(64, 128, seed=4)
    D = [float(2 ** e) for e in range(17)]
    per = np.stack([orc.score_literal(bits, q, 1e4, [dl]) for dl in D])
    mx = per.max(axis=0)
    mean = per.mean(axis=0)
    fol = orc.score_folded(bits, q, 1e4, D)
    scale = np.abs(vals) @ np.abs(q.astype(np.float64))
    assert np.max(np.abs(mean - fol) / scale) < 1e-10
    assert np.max(np.abs(mx - fol) / scale) > 1e-2


# ------------------------------------------------------------ select

def lexsort_top(s, B):
    """Reference top-B by a library sort: keys (NaN flag, -score, index)."""
    s = np.asarray(s, dtype=np.float64)
    isn = np.isnan(s)
    key = np.where(isn, 0.0, -s) + 0.0      # -0 -> +0
    order = np.lexsort((np.arange(len(s)), key, isn))
    return np.sort(order[:min(B, len(s))])


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
def test_select_matches_library_sort(orc, dtype):
    rng = np.random.default_rng(7)
    for trial in range(40):
        n = int(rng.integers(0, 300))
        s = rng.standard_normal(n).astype(dtype)
        if n and trial % 3 == 0:                      # many exact ties
            s = rng.integers(-3, 4, size=n).astype(dtype)
        if n and trial % 5 == 0:
            s[rng.integers(0, n, size=3)] = np.nan
            s[rng.integers(0, n, size=3)] = -0.0
            s[rng.integers(0, n, size=2)] = np.inf
            s[rng.integers(0, n, size=2)] = -np.inf
        for B in (1, 5, n // 2 + 1, n, n + 7):
            if B < 1:
                continue
            got = orc.select(s, B)
            np.testing.assert_array_equal(got, lexsort_top(s, B))


def test_select_invariants(orc):
    rng = np.random.default_rng(8)
    s = rng.integers(0, 50, size=1000).astype(np.float32)
    B = 137
    kept = orc.select(s, B)
    assert len(kept) == B and np.all(np.diff(kept) > 0)
    ev = np.setdiff1d(np.arange(1000), kept)
    assert s[kept].min() >= s[ev].max()
    t = s[kept].min()
    # among keys equal to the threshold, the kept ones have the lowest indices
    eq = np.flatnonzero(s == t)
    kept_eq = np.intersect1d(eq, kept)
    assert np.array_equal(kept_eq, eq[: len(kept_eq)])
    # -0 and +0 tie; NaN is last
    z = np.array([0.0, -0.0, np.nan, 0.0], dtype=np.float32)
    np.testing.assert_array_equal(orc.select(z, 2), [0, 1])
    np.testing.assert_array_equal(orc.select(z, 3), [0, 1, 3])


# ------------------------------------------------------------ compaction

def test_gather_rows(orc):
    rng = np.random.default_rng(12)
    rows = rng.integers(0, 65536, size=(100, 128), dtype=np.uint16)
    kept = np.sort(rng.choice(100, size=30, replace=False)).astype(np.int32)
    np.testing.assert_array_equal(orc.gather_rows(rows, kept), rows[kept])


def test_holefill_invariants(orc):
    rng = np.random.default_rng(13)
    for trial in range(50):
        n = int(rng.integers(1, 200))
        B = int(rng.integers(1, 220))
        s = rng.standard_normal(n)
        kept = orc.select(s, B)
        rows = rng.integers(0, 65536, size=(n, 16), dtype=np.uint16)
        rows[:, 0] = np.arange(n)                     # tag rows by index
        out, moved = orc.holefill(rows, kept, B)
        m = min(n, B)
        if n <= B:
            assert moved == 0 and np.array_equal(out, rows)
            continue
        # the first min(B, n) rows are exactly the kept rows (as a set)
        assert sorted(out[:m, 0].tolist()) == kept.tolist()
        # survivors below B did not move; rows past B are untouched
        for i in kept[kept < B]:
            assert out[i, 0] == i
        assert np.array_equal(out[B:], rows[B:])
        # holes (ascending) take movers (ascending): the map is increasing
        holes = [p for p in range(B) if p not in set(kept.tolist())]
        assert moved == len(holes) == int(np.sum(kept >= B))
        src = [int(out[h, 0]) for h in holes]
        assert src == sorted(src) and all(x >= B for x in src)


# ------------------------------------------------------------ max over offsets

@pytest.mark.parametrize("pairing", [0, 1])
def test_max_over_offsets_is_max_of_textbook_rope(orc, pairing):
    """max_delta of RoPE(q at n + delta0 + delta) . RoPE(k at n), computed with
    textbook RoPE in numpy, for a geometric schedule."""
    bits, vals, q = rand_case(40, 128, seed=31)
    theta, n_pos, delta0 = 1e6, 777, 5.0
    D = [float(2 ** e) for e in range(17)]
    kr = rope(vals, n_pos, theta, pairing)
    per = np.stack([kr @ rope(q.astype(np.float64)[None, :], n_pos + delta0 + dl, theta, pairing)[0] for dl in D])
    ref = per.max(axis=0)
    got = orc.score_max_literal(bits, q, theta, D, delta0, pairing)
    scale = np.abs(vals) @ np.abs(q.astype(np.float64))
    assert np.all(np.abs(got - ref) <= 1e-9 * scale)


def test_max_over_offsets_special_cases(orc):
    bits, vals, q = rand_case(50, 128, seed=32)
    D = [1.0, 64.0, 4096.0]
    mx = orc.score_max_literal(bits, q, 1e4, D)
    # a single offset: the literal score itself
    np.testing.assert_allclose(orc.score_max_literal(bits, q, 1e4, [64.0]), orc.score_literal(bits, q, 1e4, [64.0]),
                               rtol=1e-12, atol=1e-12)
    # a repeated offset changes nothing; the max is at least the mean
    np.testing.assert_allclose(orc.score_max_literal(bits, q, 1e4, D + [64.0, 1.0]), mx, rtol=0, atol=0)
    assert np.all(mx >= orc.score_literal(bits, q, 1e4, D) - 1e-9)


# ------------------------------------------------------------ per-key distances

@pytest.mark.parametrize("pairing", [0, 1])
def test_per_key_distance_is_textbook_rope(orc, pairing):
    """D = {delta}: key i at position p_i, query at t: RoPE(q, t + delta) . RoPE(k_i, p_i)."""
    bits, vals, q = rand_case(30, 128, seed=41)
    rng = np.random.default_rng(41)
    pos = rng.integers(0, 100000, size=30)
    t, delta, theta = 131000, 64.0, 5e5
    qr = rope(q.astype(np.float64)[None, :], t + delta, theta, pairing)[0]
    ref = np.array([rope(vals[i:i + 1], int(pos[i]), theta, pairing)[0] @ qr for i in range(30)])
    got = orc.score_at_positions(bits, q, theta, [delta], pos, t, pairing)
    scale = np.abs(vals) @ np.abs(q.astype(np.float64))
    assert np.all(np.abs(got - ref) <= 1e-9 * scale)


def test_per_key_distance_constant_positions(orc):
    """Every key at the same position p: the single-distance average with delta0 = t - p."""
    bits, vals, q = rand_case(40, 128, seed=42)
    D = [float(2 ** e) for e in range(17)]
    got = orc.score_at_positions(bits, q, 1e6, D, np.full(40, 1000), 4321)
    ref = orc.score_literal(bits, q, 1e6, D, delta0=3321.0)
    np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-10)


def test_abs_dot_is_the_absolute_term_sum(orc):
    """The parity bar's scale sum_j |w_j k_j|: at least |sum_j w_j k_j|
    (triangle inequality) and equal to it when every term has one sign;
    blind to the signs of the key and of the weights; linear in |w|; and on a
    one-hot weight it is the one key element's magnitude."""
    bits, vals, _ = rand_case(257, 128, seed=41)
    rng = np.random.default_rng(42)
    w = rng.standard_normal(128)
    a = orc.abs_dot(bits, w)
    s = orc.score_realdot(bits, w)
    assert a.shape == (257,)
    assert np.all(a >= np.abs(s) * (1 - 1e-12))
    assert np.all(a > np.abs(s) * (1 + 1e-6))          # mixed signs: strictly larger here
    pos_bits = bits & np.uint16(0x7FFF)                 # |k| (bf16 sign bit cleared)
    np.testing.assert_allclose(orc.abs_dot(pos_bits, np.abs(w)), orc.score_realdot(pos_bits, np.abs(w)),
                               rtol=1e-13)
    np.testing.assert_array_equal(orc.abs_dot(bits ^ np.uint16(0x8000), -w), a)
    np.testing.assert_array_equal(orc.abs_dot(bits, 2.0 * w), 2.0 * a)
    for j in (0, 63, 64, 127):
        e = np.zeros(128)
        e[j] = -3.0
        np.testing.assert_array_equal(orc.abs_dot(bits, e), 3.0 * np.abs(vals[:, j]))


def test_threads_do_not_change_results(orc):
    """Keys are split across host threads; each key's sum runs in one thread
    in a fixed order, so any thread count gives the same bits."""
    bits, _, q = rand_case(203, 128, seed=61)          # 203 keys: uneven chunks for 7 threads
    D = [1.0, 3.0, 17.5, 1024.0]
    rng = np.random.default_rng(62)
    pos = np.sort(rng.choice(4 * 203, size=203, replace=False)).astype(np.int32)
    w = orc.fold_w(q[None, :], 1e4, D, 0.0, 0)[0]
    for pairing in (0, 1):
        calls = [
            lambda t: orc.score_cosine(bits, q, 1e4, D, 2.0, pairing, threads=t),
            lambda t: orc.score_literal(bits, q, 1e4, D, 2.0, pairing, threads=t),
            lambda t: orc.score_max_literal(bits, q, 1e4, D, 2.0, pairing, threads=t),
            lambda t: orc.score_folded(bits, q, 1e4, D, 2.0, pairing, threads=t),
            lambda t: orc.score_polar(bits, q, 1e4, D, 2.0, pairing, threads=t),
            lambda t: orc.score_at_positions(bits, q, 1e4, D, pos, 4 * 203, pairing, threads=t),
        ]
        for fn in calls:
            np.testing.assert_array_equal(fn(1), fn(7))
    np.testing.assert_array_equal(orc.score_realdot(bits, w, threads=1), orc.score_realdot(bits, w, threads=7))
    np.testing.assert_array_equal(orc.abs_dot(bits, w, threads=1), orc.abs_dot(bits, w, threads=7))
