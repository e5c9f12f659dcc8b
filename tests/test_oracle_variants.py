"""Pins for the oracle's A2V norm producer and its ablation variants (mapping
exponent, guidance terms, density definitions, Top-k-only / Top-p-only).
Each test checks the oracle against a closed form, an invariant, a special
case that reduces to the method itself, or an independent formulation.
No GPU needed."""
import math

import numpy as np
import pytest

from oracle import prism_oracle as O


# ------------------------------------------------------------- A2V norm
def test_a2v_norm_closed_forms():
    C = 3072
    h = np.zeros((5, C))
    h[0] = 0.75                                  # constant row: |c| sqrt(C)
    h[1, 7], h[1, 2000] = 3.0, -4.0              # Pythagorean pair -> 5
    h[2, 11] = -2.5                              # one-hot -> |x|
    h[3, :9] = 2.0                               # nine 2s -> 6
    a = O.a2v_norm(h)
    np.testing.assert_allclose(a, [0.75 * math.sqrt(C), 5.0, 2.5, 6.0, 0.0], rtol=1e-15)


def test_a2v_norm_equals_math_hypot_and_is_homogeneous():
    """math.hypot over a row is an independent formulation of the L2 norm;
    scaling by 2^k scales the norm by exactly 2^k."""
    rng = np.random.default_rng(11)
    h = rng.normal(size=(40, 136)) * rng.uniform(0.01, 10, size=(40, 1))
    a = O.a2v_norm(h)
    want = np.array([math.hypot(*row) for row in h])
    np.testing.assert_allclose(a, want, rtol=1e-14)
    assert np.array_equal(O.a2v_norm(h * 8.0), a * 8.0)
    assert np.array_equal(O.a2v_norm(h[:, ::-1]), O.a2v_norm(h[:, ::-1]))  # deterministic
    np.testing.assert_allclose(O.a2v_norm(h[:, rng.permutation(136)]), a, rtol=1e-14)


def test_a2v_norm_feeds_the_plan_like_its_magnitudes():
    """h_hat = a * (unit vector) has norm a, so the plan built from the norms
    of h_hat equals the plan built from a itself."""
    rng = np.random.default_rng(12)
    T, H, W = 8, 16, 16
    N = T * H * W
    a = np.abs(rng.normal(size=N)) + np.exp(-((np.arange(N) % W) - 4.0) ** 2 / 4.0)
    u = rng.normal(size=(N, 64))
    u /= np.sqrt((u * u).sum(axis=1, keepdims=True))
    an = O.a2v_norm(a[:, None] * u)
    np.testing.assert_allclose(an, a, rtol=1e-13)
    V = rng.normal(size=(N, 2, 8))
    p1, p2 = O.plan(V, a, T, H, W), O.plan(V, an, T, H, W)
    for h1, h2 in zip(p1.heads, p2.heads):
        np.testing.assert_allclose(h1.g, h2.g, rtol=1e-12)
        assert np.array_equal(h1.shape, h2.shape)


# ------------------------------------------------------------- mapping exponent
def test_exponent_half_is_the_method():
    rng = np.random.default_rng(13)
    g = 2.0 ** rng.uniform(-8, 8, size=(200, 3))
    B = rng.choice([64, 128, 256], size=200)
    assert np.array_equal(O.lstar(g, B, 0.5), O.lstar(g, B))


@pytest.mark.parametrize("alpha", [0.25, 1.0, 2.0])
def test_exponent_stationarity(alpha):
    """l*_d = -alpha log2 g_d + c with sum_d l*_d = log2 B: g_d^(2 alpha)
    4^(l*_d) is the same on every axis (b*_d proportional to g_d^-alpha)."""
    rng = np.random.default_rng(14)
    g = 2.0 ** rng.uniform(-6, 6, size=(300, 3))
    B = rng.choice([64, 128, 256], size=300)
    ls = O.lstar(g, B, alpha)
    np.testing.assert_allclose(ls.sum(axis=1), np.log2(B), atol=1e-11)
    lhs = g ** (2 * alpha) * 4.0 ** ls
    np.testing.assert_allclose(lhs / lhs[:, :1], 1.0, rtol=1e-9)


def test_exponent_zero_and_flat_guidance_give_isotropic_shapes():
    """alpha = 0 (or g the same on every axis) puts l*_d = log2(B)/3 on each
    axis; the nearest candidates are then (4,4,4) for 64, a three-way tie
    won by (4,4,8) for 128, and a three-way tie won by (4,8,8) for 256."""
    rng = np.random.default_rng(15)
    g = 2.0 ** rng.uniform(-6, 6, size=(30, 3))
    for B, want in ((64, 3), (128, 8), (256, 13)):
        Bs = np.full(30, B)
        ls = O.lstar(g, Bs, 0.0)
        np.testing.assert_allclose(ls, np.log2(B) / 3.0, atol=1e-14)
        ids, _ = O.nearest_shape(ls, Bs)
        assert (ids == want).all()
        assert O.candidate_shapes()[want] == {64: (4, 4, 4), 128: (4, 4, 8), 256: (4, 8, 8)}[B]


def test_larger_exponent_sharpens_the_shape():
    """With most variation along T, a stronger mapping gives a shorter b_T."""
    g = np.array([[0.90, 0.05, 0.05]])
    B = np.array([128])
    ids = [O.nearest_shape(O.lstar(g, B, al), B)[0][0] for al in (0.1, 0.5, 2.0)]
    bT = [O.candidate_shapes()[i][0] for i in ids]
    assert bT[0] >= bT[1] >= bT[2] and bT[2] == 2 and bT[0] == 4


# ------------------------------------------------------------- guidance terms
def test_guidance_terms_and_their_sums():
    rng = np.random.default_rng(16)
    r = O.shares(rng.random((12, 3)))
    vhat = O.shares(rng.random((12, 3)))
    abar = rng.random(12)
    e = 1e-6
    full = O.variation_indicator(r, abar, vhat, e)
    no_v = O.variation_indicator(r, abar, vhat, e, video=False)
    no_a = O.variation_indicator(r, abar, vhat, e, audio=False)
    none = O.variation_indicator(r, abar, vhat, e, video=False, audio=False)
    np.testing.assert_allclose(no_v.sum(axis=1), abar + 3 * e, rtol=1e-13)
    np.testing.assert_allclose(no_a.sum(axis=1), 1.0 + 3 * e, rtol=1e-14)
    np.testing.assert_allclose(full - no_v, r, atol=1e-15)
    np.testing.assert_allclose(full - no_a, abar[:, None] * vhat, atol=1e-15)
    assert (none == e).all()


def test_plan_without_a2v_term_equals_first_layer_plan():
    rng = np.random.default_rng(17)
    T, H, W = 8, 16, 16
    V = rng.normal(size=(T * H * W, 2, 8)) * rng.uniform(0.3, 3, size=(T * H * W, 1, 1))
    a = np.abs(rng.normal(size=T * H * W))
    p1, p2 = O.plan(V, a, T, H, W, guidance=2), O.plan(V, None, T, H, W)
    for h1, h2 in zip(p1.heads, p2.heads):
        assert np.array_equal(h1.g, h2.g) and np.array_equal(h1.shape, h2.shape)
        assert np.array_equal(h1.perm, h2.perm)


def test_plan_without_any_guidance_is_isotropic():
    rng = np.random.default_rng(18)
    T, H, W = 8, 16, 16
    V = rng.normal(size=(T * H * W, 1, 8)) * rng.uniform(0.3, 3, size=(T * H * W, 1, 1))
    hp = O.plan(V, np.abs(rng.normal(size=T * H * W)), T, H, W, guidance=3).heads[0]
    iso = {64: 3, 128: 8, 256: 13}
    assert all(hp.shape[m] == iso[int(hp.B[m])] for m in range(len(hp.B)))
    assert (hp.g == 1e-6).all()


# ------------------------------------------------------------- density definitions
def test_density_definitions_on_a_separable_field():
    """V = A(t) + B(y) + C(x): the spatial term is var(B) + var(C) and the
    temporal term is the mean squared frame step of A.  One zone ramps in t
    only (spatial 0), the other is static in t (temporal 0)."""
    rng = np.random.default_rng(19)
    D = 4
    T, H, W = 8, 8, 16
    t, y, x = np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij")
    t, y, x = t.reshape(-1), y.reshape(-1), x.reshape(-1)
    By = rng.normal(size=(8, D))
    V = np.where((x < 8)[:, None], t[:, None] * np.ones(D), By[y])[:, None, :]   # zone 0: ramp; zone 1: static
    sp_t = O.plan(V, None, T, H, W, density=1).heads[0]
    tp_t = O.plan(V, None, T, H, W, density=2).heads[0]
    both = O.plan(V, None, T, H, W).heads[0]
    assert sp_t.rho.tolist() == [0.0, 1.0] and tp_t.rho.tolist() == [1.0, 0.0]
    pop = np.mean(np.mean((By - By.mean(axis=0)) ** 2, axis=0))
    raw = np.array([1.0, pop])                                  # temporal of the ramp; spatial of zone 1
    np.testing.assert_allclose(both.rho, raw / raw.max(), rtol=1e-12)
    assert sp_t.B.tolist() == [256, 64] and tp_t.B.tolist() == [64, 256]


def test_a2v_strength_density_is_shared_by_heads():
    rng = np.random.default_rng(20)
    T, H, W = 8, 16, 16
    N = T * H * W
    V = rng.normal(size=(N, 3, 8)) * rng.uniform(0.3, 3, size=(N, 3, 1))
    a = np.abs(rng.normal(size=N)) * 0.1
    a[(np.arange(N) % W) < 8] += 1.0                             # left zones carry the audio
    pl = O.plan(V, a, T, H, W, density=3)
    abar_raw, _ = O.zone_a2v_stats(a, T, H, W)
    for hp in pl.heads:
        np.testing.assert_allclose(hp.rho, abar_raw / abar_raw.max(), rtol=1e-14)
        assert np.array_equal(hp.B, pl.heads[0].B)
    with pytest.raises(ValueError):
        O.plan(V, None, T, H, W, density=3)


# ------------------------------------------------------------- sparsity variants
def test_topk_only_and_topp_only_rows():
    """top_p = 0 keeps exactly the k best blocks; k = 1 with p > 0 keeps the
    shortest prefix whose softmax mass reaches p (brute force by sorting)."""
    rng = np.random.default_rng(21)
    for _ in range(50):
        nb = int(rng.integers(3, 60))
        s = rng.normal(size=nb).astype(np.float32) * 3
        k = int(rng.integers(1, nb + 1))
        kept, _ = O.hybrid_select_row(s, k, 0.0)
        order = sorted(range(nb), key=lambda j: (-float(s[j]), j))
        assert sorted(kept) == sorted(order[:k])
        p = float(rng.uniform(0.05, 0.95))
        kept, _ = O.hybrid_select_row(s, 1, p)
        w = np.exp(s.astype(np.float64) - s.max())
        w /= w.sum()
        c, n = 0.0, 0
        while c < p:
            c += w[order[n]]
            n += 1
        assert sorted(kept) == sorted(order[:n])
        kept, _ = O.hybrid_select_row(s, 1, 1.0)                 # p = 1 keeps every block
        assert sorted(kept) == list(range(nb))


def test_value_projection_closed_forms():
    """project_v: the identity weight returns X; a permutation weight permutes
    X's channels; a loop over the definition on a tiny case; linearity in
    Wv."""
    rng = np.random.default_rng(31)
    X = rng.normal(size=(6, 8))
    np.testing.assert_array_equal(O.project_v(X, np.eye(8)), X)
    perm = rng.permutation(8)
    Wp = np.eye(8)[perm]                       # output channel o reads input channel perm[o]
    np.testing.assert_array_equal(O.project_v(X, Wp), X[:, perm])
    W = rng.normal(size=(4, 8))
    loop = np.array([[sum(X[n, c] * W[o, c] for c in range(8)) for o in range(4)] for n in range(6)])
    np.testing.assert_allclose(O.project_v(X, W), loop, rtol=1e-14, atol=1e-14)
    W2 = rng.normal(size=(4, 8))
    np.testing.assert_allclose(O.project_v(X, W + 2.0 * W2), O.project_v(X, W) + 2.0 * O.project_v(X, W2),
                               rtol=1e-12, atol=1e-12)


def test_plan_from_orthogonally_mixed_values_equals_plan_from_values():
    """The projection inputs the benchmark uses (synth.make_projection): a
    per-head orthogonal mix of the channels keeps the zone statistics, so the
    oracle's plan of X Wv^T equals its plan of V (up to float64 rounding in
    the statistics, far from any decision on this grid)."""
    import torch
    from dynamic_block_sparse_stats_b200.synth import WORKLOADS, make_inputs, make_projection
    w = WORKLOADS["small"]
    inp = make_inputs(w, "cpu")
    X, Wv = make_projection(inp["V"])
    Vp = O.project_v(X.float().numpy(), Wv.float().numpy()).reshape(w.N, w.heads, w.head_dim)
    a = inp["a"].numpy()
    ref = O.plan(inp["V"].float().numpy(), a, w.T, w.H, w.W)
    got = O.plan(Vp, a, w.T, w.H, w.W)
    for hr, hg in zip(ref.heads, got.heads):
        np.testing.assert_allclose(hg.rho, hr.rho, rtol=1e-2, atol=1e-3)
        assert (hg.shape == hr.shape).mean() > 0.97
