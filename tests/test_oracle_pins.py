"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: hand-derived
fixtures (tests/golden), closed forms, invariants, or an independent library
routine (torch.cdist, torch scaled_dot_product_attention).  The last test
plants mistakes in copies of oracle functions and checks the pins catch them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import lvq_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ----------------------------------------------------------------------------- encode

def test_nearest_entry_hand_fixture():
    fx = _golden("nearest_tiny.json")
    C = np.array(fx["codebook"], dtype=np.float64)
    X = np.array([c["x"] for c in fx["cases"]], dtype=np.float64)
    idx, d1, d2 = O.nearest_entry(X, C)
    assert idx.tolist() == [c["idx"] for c in fx["cases"]]
    np.testing.assert_array_equal(d1, [c["d1"] for c in fx["cases"]])
    np.testing.assert_array_equal(d2, [c["d2"] for c in fx["cases"]])


def test_entries_reencode_to_own_index_and_duplicates_go_low():
    rng = np.random.default_rng(3)
    C = rng.standard_normal((256, 16)).astype(np.float32).astype(np.float64)
    idx, d1, _ = O.nearest_entry(C, C)
    assert (idx == np.arange(256)).all() and (d1 == 0).all()
    C2 = C.copy()
    C2[200] = C2[37]  # duplicate entry: both 37 and 200 are exact matches
    idx2, d1b, d2b = O.nearest_entry(C2[[200, 37]], C2)
    assert idx2.tolist() == [37, 37]
    assert O.near_tie(d1b, d2b).all()


def test_near_tie_fixture():
    """The near-tie rule that decides which GPU/oracle code mismatches are acceptable:
    relative to d1, inclusive at the bound, and only exact duplicates when d1 = 0."""
    fx = _golden("near_tie.json")
    d1 = np.array([c["d1"] for c in fx["cases"]])
    d2 = np.array([c["d2"] for c in fx["cases"]])
    assert O.NEAR_TIE_REL == fx["rel"]
    got = O.near_tie(d1, d2)
    assert got.tolist() == [c["tie"] for c in fx["cases"]], [c["why"] for c, g in zip(fx["cases"], got)
                                                             if g != c["tie"]]


def test_near_tie_from_nearest_entry_geometry():
    """Distances from nearest_entry feed near_tie: x exactly between two entries is a tie;
    moved off the midpoint by a hand-chosen amount it is or is not, as the relative gap says."""
    C = np.zeros((256, 2))
    C[:, 0] = 1000.0                     # every other entry far away
    C[3] = [0.0, 0.0]
    C[9] = [2.0, 0.0]
    for shift, tie in ((0.0, True), (2.0 ** -22, True), (2.0 ** -18, False)):
        x = np.array([[1.0 - shift, 0.0]])   # d1 = (1 - shift)^2, d2 = (1 + shift)^2
        idx, d1, d2 = O.nearest_entry(x, C)
        assert idx[0] == 3
        # gap 4 * shift over d1 ~ 1: 2^-20 = 9.5e-7 <= 1e-6 (tie), 2^-16 = 1.5e-5 (not)
        assert bool(O.near_tie(d1, d2)[0]) == tie


def test_tc1_encode_matches_cdist_argmin():
    """At Tc = 1 the joint vector is G channels of one step: textbook VQ."""
    rng = np.random.default_rng(5)
    T, N, H, d, G = 2, 300, 2, 32, 8
    x = rng.standard_normal((T, N, H, d))
    n_g = d // G
    cb = rng.standard_normal((T, H, n_g, 256, G))
    codes, _, _ = O.encode(x, cb, Tc=1, G=G)
    for t in range(T):
        for h in range(H):
            for g in range(n_g):
                xs = torch.from_numpy(x[t, :, h, g * G:(g + 1) * G])
                D = torch.cdist(xs, torch.from_numpy(cb[t, h, g])) ** 2
                ref = D.argmin(dim=1).numpy()
                assert (codes[t, :, h, g] == ref).all()


def test_encode_is_brute_force_over_all_entries():
    """Random tiny case: the chosen entry's distance is <= every entry's distance."""
    rng = np.random.default_rng(11)
    X = rng.standard_normal((50, 4))
    C = rng.standard_normal((256, 4))
    idx, d1, d2 = O.nearest_entry(X, C)
    for m in range(50):
        ds = [float(np.sum((X[m] - C[k]) ** 2)) for k in range(256)]
        assert idx[m] == int(np.argmin(ds))
        assert d1[m] == pytest.approx(min(ds), rel=1e-15)
        assert d2[m] == pytest.approx(sorted(ds)[1], rel=1e-15)


def test_joint_vector_order_fixture():
    fx = _golden("joint_vector_order.json")
    T, Tc, G, d = fx["T"], fx["Tc"], fx["G"], fx["d"]
    x = np.zeros((T, 1, 1, d))
    for t in range(T):
        for ch in range(d):
            x[t, 0, 0, ch] = 100 * t + ch
    X = O.joint_vectors(x, Tc, G)
    for case in fx["cases"]:
        assert X[case["block"], 0, 0, case["group"]].tolist() == case["vector"]
    # codebooks made of the vectors themselves: encode then dequant restores x per step
    c, n_g, n_blk = O.geometry(d, T, Tc, G)
    cb = np.zeros((n_blk, 1, n_g, 256, G))
    for b in range(n_blk):
        for g in range(n_g):
            cb[b, 0, g, 7] = X[b, 0, 0, g]
            cb[b, 0, g, 8:] = 1e6  # far away
    codes, d1, _ = O.encode(x, cb, Tc, G)
    assert (codes == 7).all() and (d1 == 0).all()
    for case in fx["dequant"]:
        got = O.dequant_step(codes, cb, case["step"], Tc, G)[0, 0]
        assert got.tolist() == case["expect"]


def test_bits_per_element_closed_form():
    # [summary, "how it differs"]: b/G bits per element; 8-bit codes
    assert O.bits_per_element(128, 4, 4, 16) == 0.5
    assert O.bits_per_element(128, 4, 4, 32) == 0.25
    assert O.bits_per_element(128, 4, 2, 16) == 0.5
    assert O.bits_per_element(64, 4, 4, 16) == 0.5
    assert O.bits_per_element(128, 4, 1, 16) == 0.5
    for (d, T, Tc, G) in [(128, 4, 4, 16), (128, 4, 2, 16), (128, 4, 4, 32), (64, 4, 4, 16)]:
        c, n_g, n_blk = O.geometry(d, T, Tc, G)
        assert n_blk * n_g * 8 / (T * d) == 8 / G
    with pytest.raises(ValueError):
        O.geometry(128, 4, 3, 16)
    with pytest.raises(ValueError):
        O.geometry(128, 6, 4, 16)


# ----------------------------------------------------------------------------- dequant

def test_step_slice_isolation_nan_poison():
    """A step-t read touches only columns [s*c, (s+1)*c) of each code's entry."""
    rng = np.random.default_rng(7)
    T, Tc, G, d, N = 4, 2, 16, 32, 40
    c, n_g, n_blk = O.geometry(d, T, Tc, G)
    cb = rng.standard_normal((n_blk, 1, n_g, 256, G))
    codes = rng.integers(0, 256, (n_blk, N, 1, n_g)).astype(np.uint8)
    for t in range(T):
        s = t % Tc
        poisoned = cb.copy()
        mask = np.ones(G, bool)
        mask[s * c:(s + 1) * c] = False
        poisoned[..., mask] = np.nan
        clean = O.dequant_step(codes, cb, t, Tc, G)
        got = O.dequant_step(codes, poisoned, t, Tc, G)
        assert np.isfinite(got).all()
        np.testing.assert_array_equal(got, clean)


# ----------------------------------------------------------------------------- RoPE

def test_rope_hand_values():
    # d = 4: theta_0 = 1, theta_1 = 10000^(-1/2) = 0.01
    y = O.rope(np.array([1.0, 0.0, 0.0, 0.0]), np.array(1.0))
    np.testing.assert_allclose(y, [math.cos(1), 0.0, math.sin(1), 0.0], rtol=0, atol=1e-15)
    y = O.rope(np.array([0.0, 1.0, 0.0, 0.0]), np.array(100.0))
    np.testing.assert_allclose(y, [0.0, math.cos(1), 0.0, math.sin(1)], rtol=0, atol=1e-14)
    y = O.rope(np.array([0.0, 0.0, 1.0, 0.0]), np.array(2.0))
    np.testing.assert_allclose(y, [-math.sin(2), 0.0, math.cos(2), 0.0], rtol=0, atol=1e-15)


def test_rope_identity_norm_and_relative_position():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((20, 128))
    np.testing.assert_array_equal(O.rope(x, np.zeros(20)), x)
    pos = rng.integers(0, 70000, 20).astype(np.float64)
    np.testing.assert_allclose(np.linalg.norm(O.rope(x, pos), axis=1), np.linalg.norm(x, axis=1),
                               rtol=1e-13)
    q = rng.standard_normal(128)
    for shift in (1.0, 17.0, 4096.0):
        s0 = O.rope(x, pos) @ O.rope(q[None], np.array([500.0]))[0]
        s1 = O.rope(x, pos + shift) @ O.rope(q[None], np.array([500.0 + shift]))[0]
        np.testing.assert_allclose(s1, s0, rtol=0, atol=1e-9 * (1 + np.abs(s0).max()))


def test_rope_matches_complex_rotation():
    """Pair (i, i+d/2) as the complex number x_i + j x_{i+d/2}, multiplied by e^{j pos theta_i}."""
    rng = np.random.default_rng(2)
    d = 64
    x = rng.standard_normal((5, d))
    pos = np.array([0.0, 3.0, 1000.0, 32767.0, 65535.0])
    z = (x[:, :d // 2] + 1j * x[:, d // 2:]) * np.exp(
        1j * pos[:, None] * 10000.0 ** (-np.arange(d // 2) * 2.0 / d))
    np.testing.assert_allclose(O.rope(x, pos), np.concatenate([z.real, z.imag], axis=1),
                               rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------- attention

def test_softmax_attention_closed_forms():
    rng = np.random.default_rng(4)
    n, d = 37, 64
    v = rng.standard_normal((n, d))
    q = rng.standard_normal(d)
    out, lse = O.softmax_attention(q, np.zeros((n, d)), v)   # zero keys: uniform weights
    np.testing.assert_allclose(out, v.mean(axis=0), rtol=1e-13, atol=1e-15)
    assert lse == pytest.approx(math.log(n), rel=1e-14)
    k = rng.standard_normal((1, d))
    out1, lse1 = O.softmax_attention(q, k, v[:1])              # one key: out = v, lse = s
    np.testing.assert_allclose(out1, v[0], rtol=1e-14)
    assert lse1 == pytest.approx(float(k[0] @ q) / math.sqrt(d), rel=1e-13)
    out0, lse0 = O.softmax_attention(q, np.zeros((0, d)), np.zeros((0, d)))
    assert lse0 == -math.inf and (out0 == 0).all()


def test_softmax_attention_matches_torch_sdpa():
    rng = np.random.default_rng(6)
    for n in (1, 5, 300):
        d = 128
        q, k, v = rng.standard_normal(d), rng.standard_normal((n, d)) * 3, rng.standard_normal((n, d))
        out, lse = O.softmax_attention(q, k, v)
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q)[None, None, None], torch.from_numpy(k)[None, None],
            torch.from_numpy(v)[None, None])[0, 0, 0].numpy()
        np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)
        s = torch.from_numpy(k) @ torch.from_numpy(q) / math.sqrt(d)
        assert lse == pytest.approx(float(torch.logsumexp(s, 0)), rel=1e-13)


def test_split_ranges_reading():
    assert O.split_ranges(492, 4) == [(0, 128), (128, 256), (256, 384), (384, 492)]
    assert O.split_ranges(100, 8) == [(0, 32), (32, 64), (64, 96), (96, 100)] + [(100, 100)] * 4
    assert O.split_ranges(0, 3) == [(0, 0)] * 3
    assert O.split_ranges(32636, 16)[-1] == (30720, 32636)
    rs = O.split_ranges(32636, 16)
    assert rs[0] == (0, 2048) and all(b - a == 2048 for a, b in rs[:-1])


def test_split_lse_merge_equals_unsplit():
    rng = np.random.default_rng(8)
    d = 64
    q = rng.standard_normal(d)
    k = rng.standard_normal((500, d)) * 2
    v = rng.standard_normal((500, d))
    out, lse = O.softmax_attention(q, k, v)
    for ns in (1, 2, 7, 16, 64):
        parts = [O.softmax_attention(q, k[a:b], v[a:b]) for a, b in O.split_ranges(500, ns)]
        m_out, m_lse = O.lse_merge(parts)
        np.testing.assert_allclose(m_out, out, rtol=0, atol=1e-12)
        assert abs(m_lse - lse) < 1e-12


def _tiny_cache(rng, d=32, T=4, Tc=2, G=8, S=3, L=70, R=11):
    c, n_g, n_blk = O.geometry(d, T, Tc, G)
    return dict(
        sink_k=rng.standard_normal((S, d)), sink_v=rng.standard_normal((S, d)),
        codes_k=rng.integers(0, 256, (n_blk, L, n_g)).astype(np.uint8),
        codes_v=rng.integers(0, 256, (n_blk, L, n_g)).astype(np.uint8),
        cb_k=rng.standard_normal((n_blk, n_g, 256, G)), cb_v=rng.standard_normal((n_blk, n_g, 256, G)),
        ring_k=rng.standard_normal((R, d)), ring_v=rng.standard_normal((R, d)))


def test_decode_attention_against_explicit_assembly_and_sdpa():
    """Dequantize by hand from the codebook entries, RoPE every key at its absolute position,
    and run torch SDPA: the oracle's decode must agree."""
    rng = np.random.default_rng(9)
    d, T, Tc, G = 32, 4, 2, 8
    cache = _tiny_cache(rng, d, T, Tc, G)
    q = rng.standard_normal(d)
    c = G // Tc
    S, L, R = 3, 70, 11
    for t in range(T):
        b, s = t // Tc, t % Tc
        kh = np.array([[cache["cb_k"][b, g, cache["codes_k"][b, n, g], s * c + e]
                        for g in range(d // c) for e in range(c)] for n in range(L)])
        vh = np.array([[cache["cb_v"][b, g, cache["codes_v"][b, n, g], s * c + e]
                        for g in range(d // c) for e in range(c)] for n in range(L)])
        keys = np.concatenate([cache["sink_k"], kh, cache["ring_k"]])
        vals = np.concatenate([cache["sink_v"], vh, cache["ring_v"]])
        pos = np.arange(S + L + R, dtype=np.float64)
        kr = O.rope(keys, pos)
        qr = O.rope(q[None], np.array([S + L + R - 1.0]))[0]
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(qr)[None, None, None], torch.from_numpy(kr)[None, None],
            torch.from_numpy(vals)[None, None])[0, 0, 0].numpy()
        out, lse, sl = O.decode_attention(q, t, Tc, G, n_splits=5, **cache)
        np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)
        merged = O.lse_merge([(np.zeros(d), x) for x in sl])[1]
        assert abs(merged - lse) < 1e-12


def test_identical_codes_with_zero_key_slice_give_uniform_attention():
    """All coded tokens share one entry whose step-t key share is zero, and the bf16 part is
    empty: every score is 0 after RoPE, so p = 1/L, lse = ln L and out is that entry's V share."""
    rng = np.random.default_rng(10)
    d, T, Tc, G, L = 32, 4, 4, 16, 123
    c, n_g, n_blk = O.geometry(d, T, Tc, G)
    cb_k = rng.standard_normal((n_blk, n_g, 256, G))
    cb_v = rng.standard_normal((n_blk, n_g, 256, G))
    t = 2
    cb_k[0, :, 42, t * c:(t + 1) * c] = 0.0
    codes = np.full((n_blk, L, n_g), 42, np.uint8)
    empty = np.zeros((0, d))
    out, lse, _ = O.decode_attention(rng.standard_normal(d), t, Tc, G, empty, empty, codes, codes,
                                     cb_k, cb_v, empty, empty)
    assert lse == pytest.approx(math.log(L), rel=1e-14)
    np.testing.assert_allclose(out, cb_v[0, :, 42, t * c:(t + 1) * c].reshape(-1), rtol=1e-14)


def test_page_encode_equals_prefill_encode():
    rng = np.random.default_rng(12)
    T, Tc, G, d, H = 4, 2, 16, 64, 2
    c, n_g, n_blk = O.geometry(d, T, Tc, G)
    x = rng.standard_normal((2, T, 40, H, d))
    cb = rng.standard_normal((2, n_blk, H, n_g, 256, G))
    full_k, _, _ = O.encode(x[0], cb[0], Tc, G)
    full_v, _, _ = O.encode(x[1], cb[1], Tc, G)
    pk, pv = O.page_encode(x[0, :, 16:], x[1, :, 16:], cb[0], cb[1], Tc, G)
    assert (pk == full_k[:, 16:24]).all() and (pv == full_v[:, 16:24]).all()


# ----------------------------------------------------------------------------- codebook construction

def test_kmeans_hand_fixture():
    fx = _golden("kmeans_tiny.json")
    C = np.array(fx["codebook"])
    X = np.array(fx["x"])
    codes, C_new, counts = O.kmeans_step(X, C)
    assert codes.tolist() == fx["codes"]
    np.testing.assert_array_equal(C_new, fx["new_codebook"])
    assert counts.tolist() == fx["counts"]


def test_kmeans_update_matches_sklearn_one_lloyd_iteration():
    """No empty entries here (scikit-learn relocates empty clusters, the oracle keeps them)."""
    from sklearn.cluster import KMeans
    rng = np.random.default_rng(11)
    K, G = 16, 4
    centers = rng.standard_normal((K, G)) * 6
    X = np.concatenate([centers[k] + rng.standard_normal((40, G)) for k in range(K)])
    C = centers + rng.standard_normal((K, G)) * 0.5
    codes, _, _ = O.nearest_entry(X, C)
    assert len(set(codes.tolist())) == K
    C_new, counts = O.kmeans_update(X, codes, C)
    km = KMeans(n_clusters=K, init=C, n_init=1, max_iter=1, algorithm="lloyd", tol=0.0).fit(X)
    np.testing.assert_allclose(C_new, km.cluster_centers_, rtol=0, atol=1e-12)
    assert counts.sum() == X.shape[0]


def test_kmeans_update_never_raises_the_objective():
    """Lloyd descent: the mean minimises each entry's sum of squares, and re-assigning to
    the nearest entry can only lower it further."""
    rng = np.random.default_rng(5)
    X = rng.standard_normal((3000, 8))
    C = X[rng.choice(3000, 64, replace=False)] + 0.1
    def sse(C_):
        _, d1, _ = O.nearest_entry(X, C_)
        return d1.sum()
    codes, _, _ = O.nearest_entry(X, C)
    C_new, counts = O.kmeans_update(X, codes, C)
    assert sse(C_new) <= sse(C)
    # the update is the minimiser: moving any used entry a little raises its members' sum
    k = int(np.argmax(counts))
    m = X[codes == k]
    base = ((m - C_new[k]) ** 2).sum()
    for dv in np.eye(8) * 1e-3:
        assert ((m - (C_new[k] + dv)) ** 2).sum() > base


def test_kmeans_empty_entry_keeps_its_value():
    C = np.array([[0.0, 0.0], [100.0, 100.0], [-3.0, 7.0]])
    X = np.array([[0.5, 0.0], [0.0, 0.5]])
    C_new, counts = O.kmeans_update(X, np.array([0, 0]), C)
    np.testing.assert_array_equal(C_new[1:], C[1:])
    assert counts.tolist() == [2, 0, 0]


def test_round_bf16_matches_torch_on_fp32_values_and_ties_go_even():
    rng = np.random.default_rng(2)
    x = (rng.standard_normal(50000) * np.exp(rng.standard_normal(50000) * 8)).astype(np.float32)
    ref = torch.tensor(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.round_bf16(x.astype(np.float64)), ref)
    # halfway cases from fp64 (not representable in fp32 rounding twice): ties to even
    assert O.round_bf16(np.array([1 + 2.0 ** -8]))[0] == 1.0
    assert O.round_bf16(np.array([1 + 3 * 2.0 ** -8]))[0] == 1 + 2.0 ** -6
    assert O.round_bf16(np.array([1 + 2.0 ** -8 + 2.0 ** -40]))[0] == 1 + 2.0 ** -7
    assert O.round_bf16(np.array([2.0 ** -134]))[0] == 0.0          # half the smallest subnormal
    assert O.round_bf16(np.array([2.0 ** 128]))[0] == np.inf


# ----------------------------------------------------------------------------- planted mistakes

def test_pins_catch_planted_mistakes(monkeypatch):
    """Each mutant of an oracle function must fail at least one pin above."""
    fx = _golden("joint_vector_order.json")

    def gather_transposed(x, Tc, G):  # element order e*Tc + s instead of s*c + e
        T, N, H, d = x.shape
        c, n_g, n_blk = O.geometry(d, T, Tc, G)
        X = np.empty((n_blk, N, H, n_g, G))
        for b in range(n_blk):
            for s in range(Tc):
                for g in range(n_g):
                    for e in range(c):
                        X[b, :, :, g, e * Tc + s] = x[b * Tc + s, :, :, g * c + e]
        return X

    monkeypatch.setattr(O, "joint_vectors", gather_transposed)
    with pytest.raises(AssertionError):
        test_joint_vector_order_fixture()
    monkeypatch.undo()

    def rope_wrong_sign(x, pos, base=10000.0):
        d = x.shape[-1]
        half = d // 2
        th = np.power(float(base), -2.0 * np.arange(half) / d)
        phi = np.asarray(pos, dtype=np.float64)[..., None] * th
        lo, hi = x[..., :half], x[..., half:]
        return np.concatenate([lo * np.cos(phi) + hi * np.sin(phi), hi * np.cos(phi) - lo * np.sin(phi)], -1)

    monkeypatch.setattr(O, "rope", rope_wrong_sign)
    with pytest.raises(AssertionError):
        test_rope_hand_values()
    with pytest.raises(AssertionError):
        test_rope_matches_complex_rotation()
    monkeypatch.undo()

    def nearest_highest_tie(X, C, chunk=4096):
        D = ((X[:, None, :] - C[None, :, :]) ** 2).sum(axis=2)
        k = (C.shape[0] - 1) - D[:, ::-1].argmin(axis=1)
        srt = np.sort(D, axis=1)
        return k, srt[:, 0], srt[:, 1]

    monkeypatch.setattr(O, "nearest_entry", nearest_highest_tie)
    with pytest.raises(AssertionError):
        test_nearest_entry_hand_fixture()
    monkeypatch.undo()

    def dequant_wrong_slice(codes, cb, t, Tc, G):  # reads step (t+1) % Tc's share
        return O.__dict__["_dq_orig"](codes, cb, (t // Tc) * Tc + (t + 1) % Tc, Tc, G)

    O._dq_orig = O.dequant_step
    monkeypatch.setattr(O, "dequant_step", dequant_wrong_slice)
    with pytest.raises(AssertionError):
        test_joint_vector_order_fixture()
    monkeypatch.undo()
    del O._dq_orig

    def update_sum_not_mean(X, codes, C):       # forgets to divide by the count
        C_new = np.array(C, dtype=np.float64, copy=True)
        counts = np.zeros(C.shape[0], dtype=np.int64)
        for k in range(C.shape[0]):
            m = X[codes == k]
            counts[k] = m.shape[0]
            if counts[k]:
                C_new[k] = m.sum(axis=0)
        return C_new, counts

    monkeypatch.setattr(O, "kmeans_update", update_sum_not_mean)
    with pytest.raises(AssertionError):
        test_kmeans_hand_fixture()
    with pytest.raises(AssertionError):
        test_kmeans_update_matches_sklearn_one_lloyd_iteration()
    monkeypatch.undo()

    def update_zeroes_empty(X, codes, C):      # empty entries collapse to the origin
        C_new = np.zeros_like(np.asarray(C, dtype=np.float64))
        counts = np.zeros(C.shape[0], dtype=np.int64)
        for k in range(C.shape[0]):
            m = X[codes == k]
            counts[k] = m.shape[0]
            if counts[k]:
                C_new[k] = m.mean(axis=0)
        return C_new, counts

    monkeypatch.setattr(O, "kmeans_update", update_zeroes_empty)
    with pytest.raises(AssertionError):
        test_kmeans_empty_entry_keeps_its_value()
    monkeypatch.undo()

    # near-tie rule: a looser bound, an absolute gap, a strict inequality, relative to d2
    for mutant in (lambda d1, d2: (d2 - d1) <= 1e-3 * d1,
                   lambda d1, d2: (d2 - d1) <= 1e-6,
                   lambda d1, d2: (d2 - d1) < 1e-6 * d1,
                   lambda d1, d2: (d2 - d1) <= 1e-6 * d2):
        monkeypatch.setattr(O, "near_tie", mutant)
        with pytest.raises(AssertionError):
            test_near_tie_fixture()
        monkeypatch.undo()

    def round_via_fp32(x):                      # double rounding fp64 -> fp32 -> bf16
        return torch.tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).to(torch.float64).numpy()

    monkeypatch.setattr(O, "round_bf16", round_via_fp32)
    with pytest.raises(AssertionError):
        test_round_bf16_matches_torch_on_fp32_values_and_ties_go_even()
    monkeypatch.undo()
