"""Pins for the CPU oracle: each test checks the oracle against something other
than itself (closed forms, hand-worked values, invariants, brute force, or an
independent formulation), so that a dropped term, a swapped axis or a wrong
sign in the oracle fails here.  No GPU needed."""
import math
import os

import numpy as np
import pytest
import torch

from oracle import prism_oracle as O


def _read_table(path):
    rows = []
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        rows.append(line)
    return rows


# ---------------------------------------------------------------- candidates
def test_candidate_pool_matches_hand_table(golden_dir):
    rows = _read_table(os.path.join(golden_dir, "candidate_shapes.txt"))
    table = [tuple(int(x) for x in r.split()) for r in rows]
    cands = O.candidate_shapes()
    assert len(cands) == 16
    for (i, bT, bH, bW, B), c in zip(table, cands):
        assert c == (bT, bH, bW) and bT * bH * bW == B
    assert sorted(set(e for c in cands for e in c)) == [2, 4, 8]
    counts = {B: sum(1 for c in cands if np.prod(c) == B) for B in (64, 128, 256)}
    assert counts == {64: 7, 128: 6, 256: 3}


# ---------------------------------------------------------------- zone stats
def _one_zone_field(f):
    """f(t, y, x, c) over a single 8x8x8 zone -> [512, D] in raster order."""
    t, y, x = np.meshgrid(np.arange(8), np.arange(8), np.arange(8), indexing="ij")
    return f(t.reshape(-1), y.reshape(-1), x.reshape(-1))


def test_rv_and_rho_separable_closed_form():
    """V = a(t) + b(y) + c(x) per channel.  Mean-pooling along the other two
    axes leaves each profile equal to its own term plus constants, so
    sigma^2_d = channel mean of the population variance of that term; the
    spatial term = var(b) + var(c); the temporal term = mean of squared
    consecutive differences of a."""
    rng = np.random.default_rng(0)
    D = 5
    A, Bp, Cp = rng.normal(size=(8, D)), rng.normal(size=(8, D)) * 2, rng.normal(size=(8, D)) * 0.5
    V = _one_zone_field(lambda t, y, x: A[t] + Bp[y] + Cp[x])
    sig2, spatial, temporal = O.zone_video_stats(V, 8, 8, 8)
    pop = lambda P: np.mean(np.mean((P - P.mean(axis=0)) ** 2, axis=0))
    np.testing.assert_allclose(sig2[0], [pop(A), pop(Bp), pop(Cp)], rtol=1e-12)
    np.testing.assert_allclose(spatial[0], pop(Bp) + pop(Cp), rtol=1e-12)
    want_t = np.mean(np.sum((A[1:] - A[:-1]) ** 2, axis=0) / 7.0)
    np.testing.assert_allclose(temporal[0], want_t, rtol=1e-12)
    r = O.shares(sig2)
    np.testing.assert_allclose(r[0], np.array([pop(A), pop(Bp), pop(Cp)]) / (pop(A) + pop(Bp) + pop(Cp)),
                               rtol=1e-12)


def test_frame_ramp_hand_values():
    """V_t = t on every channel: frame means 0..7, population variance 5.25
    along T, nothing along H or W; no spatial spread; every frame step is 1."""
    V = _one_zone_field(lambda t, y, x: np.repeat(t[:, None].astype(float), 3, axis=1))
    sig2, spatial, temporal = O.zone_video_stats(V, 8, 8, 8)
    np.testing.assert_allclose(sig2[0], [5.25, 0.0, 0.0], atol=1e-14)
    assert spatial[0] == 0.0
    np.testing.assert_allclose(temporal[0], 1.0, rtol=1e-14)
    np.testing.assert_allclose(O.shares(sig2)[0], [1.0, 0.0, 0.0])


def test_static_zone_has_exactly_zero_temporal_term():
    rng = np.random.default_rng(3)
    frame = rng.normal(size=(64, 7))
    V = np.tile(frame, (8, 1))                       # 8 identical frames
    sig2, spatial, temporal = O.zone_video_stats(V, 8, 8, 8)
    # frame differences are exactly zero; the profile variance along T is zero
    # up to the rounding of the mean of eight equal float64 values
    assert temporal[0] == 0.0 and sig2[0, 0] < 1e-30
    assert spatial[0] > 0 and sig2[0, 1] > 1e-3


def test_power_of_two_scaling_leaves_shares_and_density_identical():
    rng = np.random.default_rng(4)
    V = rng.normal(size=(16 * 8 * 16, 2, 6))
    a = np.abs(rng.normal(size=16 * 8 * 16))
    p1 = O.plan(V, a, 16, 8, 16)
    p2 = O.plan(V * 2.0, a * 4.0, 16, 8, 16)
    for h1, h2 in zip(p1.heads, p2.heads):
        assert np.array_equal(h1.g, h2.g) and np.array_equal(h1.rho, h2.rho)
        assert np.array_equal(h1.shape, h2.shape)


def test_h_w_transpose_swaps_axes():
    rng = np.random.default_rng(5)
    T, S = 8, 16
    V = rng.normal(size=(T, S, S, 1, 4)) * np.linspace(0.5, 2, S)[None, :, None, None, None]
    Vt = V.transpose(0, 2, 1, 3, 4)
    s1, sp1, tp1 = O.zone_video_stats(V.reshape(-1, 4), T, S, S)
    s2, sp2, tp2 = O.zone_video_stats(Vt.reshape(-1, 4), T, S, S)
    # zone (zh, zw) of V is zone (zw, zh) of the transpose
    idx = np.arange(4).reshape(2, 2).T.reshape(-1)
    np.testing.assert_allclose(s1[:, [0, 2, 1]], s2[idx], rtol=1e-12)
    np.testing.assert_allclose(sp1, sp2[idx], rtol=1e-12)
    np.testing.assert_allclose(tp1, tp2[idx], rtol=1e-12)


def test_a2v_stats_blob_and_normalisation():
    """A field that varies only along W: all of its directional variance is on
    W.  abar is the zone mean over the largest zone mean."""
    T, H, W = 8, 8, 16
    x = np.arange(W)
    a = np.broadcast_to((x % 8).astype(float), (T, H, W)).reshape(-1).copy()
    a[: T * H * W] += np.repeat([0.0, 1.0], 8)[np.arange(T * H * W) % W]  # zone 1 brighter
    abar_raw, sig2a = O.zone_a2v_stats(a, T, H, W)
    np.testing.assert_allclose(abar_raw, [3.5, 4.5])
    np.testing.assert_allclose(O.normalise_by_max(abar_raw), [3.5 / 4.5, 1.0])
    np.testing.assert_allclose(O.shares(sig2a), [[0, 0, 1], [0, 0, 1]], atol=1e-15)


def test_a2v_direction_shares_follow_the_axis_of_variation():
    """v_hat_{a,d}: a field that varies along one axis only puts its whole
    share on that axis; a sum f(t) + g(y) splits it in the closed-form ratio
    var f : var g (population variances of the 8-position profiles)."""
    T, H, W = 8, 8, 8
    t, y, x = np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij")
    for d, field in enumerate((t, y, x)):
        _, sig2a = O.zone_a2v_stats(field.astype(float).reshape(-1), T, H, W)
        want = np.zeros(3)
        want[d] = 1.0
        np.testing.assert_allclose(O.shares(sig2a)[0], want, atol=1e-15)
    f = np.array([0, 1, 0, 1, 0, 1, 0, 1], float)          # var 1/4
    g = np.array([0, 0, 0, 0, 2, 2, 2, 2], float)          # var 1
    a = (f[t] + g[y]).reshape(-1)
    _, sig2a = O.zone_a2v_stats(a, T, H, W)
    np.testing.assert_allclose(sig2a[0], [0.25, 1.0, 0.0], atol=1e-15)
    np.testing.assert_allclose(O.shares(sig2a)[0], [0.2, 0.8, 0.0], atol=1e-15)


def test_variation_indicator_terms_and_invariant():
    rng = np.random.default_rng(6)
    r = O.shares(rng.random((10, 3)))
    vhat = O.shares(rng.random((10, 3)))
    abar = rng.random(10)
    g = O.variation_indicator(r, abar, vhat, eps=1e-6)
    np.testing.assert_allclose(g.sum(axis=1), 1.0 + abar + 3e-6, rtol=1e-14)
    np.testing.assert_allclose(g, r + abar[:, None] * vhat + 1e-6)
    np.testing.assert_allclose(O.variation_indicator(r, eps=1e-6), r + 1e-6)


# ---------------------------------------------------------------- volumes
def test_volume_thresholds():
    rho = np.array([1.0, 0.5, 0.4999, 0.25, 0.2499, 0.0])
    B, m = O.volumes(rho, 0.5, 0.25)
    assert B.tolist() == [64, 64, 128, 128, 256, 256]
    np.testing.assert_allclose(m, [0.5, 0.0, 1e-4, 0.0, 1e-4, 0.25], atol=1e-12)


def test_constant_values_give_coarsest_isotropic_block():
    V = np.full((8 * 16 * 16, 1, 4), 0.75)
    pl = O.plan(V, None, 8, 16, 16)
    hp = pl.heads[0]
    assert (hp.rho == 0).all() and (hp.B == 256).all()
    np.testing.assert_allclose(hp.g, 1.0 / 3.0 + 1e-6)
    assert (hp.shape == 13).all()           # (4,8,8) wins the three-way tie


def test_max_density_zone_gets_finest_volume():
    rng = np.random.default_rng(7)
    V = rng.normal(size=(16 * 16 * 16, 3, 8)) * rng.uniform(0.2, 3, size=(16 * 16 * 16, 1, 1))
    pl = O.plan(V, None, 16, 16, 16)
    for hp in pl.heads:
        assert hp.B[np.argmax(hp.rho)] == 64 and hp.rho.max() == 1.0


# ---------------------------------------------------------------- shapes
def test_lstar_golden(golden_dir):
    for row in _read_table(os.path.join(golden_dir, "lstar_cases.txt")):
        gB, ls, sid, margin = [p.split() for p in row.split("|")]
        g = np.array([float(v) for v in gB[:3]])
        B = np.array([int(gB[3])])
        got = O.lstar(g[None], B)[0]
        np.testing.assert_allclose(got, [float(v) for v in ls], atol=1e-12)
        ids, m = O.nearest_shape(got[None], B)
        assert ids[0] == int(sid[0])
        np.testing.assert_allclose(m[0], float(margin[0]), atol=1e-9)


def test_lstar_is_the_lagrange_stationary_point():
    """At the optimum of sum g_d b_d^2 under prod b_d = B, g_d b_d^2 is equal
    across axes and sum l_d = log2 B."""
    rng = np.random.default_rng(8)
    g = 2.0 ** rng.uniform(-12, 12, size=(500, 3))
    B = rng.choice([64, 128, 256], size=500)
    ls = O.lstar(g, B)
    np.testing.assert_allclose(ls.sum(axis=1), np.log2(B), atol=1e-11)
    lhs = g * 4.0 ** ls
    np.testing.assert_allclose(lhs / lhs[:, :1], 1.0, rtol=1e-10)


def test_nearest_log2_shape_equals_bruteforce_minimum_of_J():
    """The shape loss J = sum_d g_d (b_d^2 - 1): its brute-force minimum over
    the candidates of volume B agrees with the nearest-log2 choice."""
    rng = np.random.default_rng(9)
    cands = O.candidate_shapes()
    g = 2.0 ** rng.uniform(-10, 10, size=(3000, 3))
    for B in (64, 128, 256):
        Bs = np.full(len(g), B)
        ids, margin = O.nearest_shape(O.lstar(g, Bs), Bs)
        for gi, sid, m in zip(g, ids, margin):
            J = [(sum(gi[d] * (c[d] ** 2 - 1) for d in range(3)), i)
                 for i, c in enumerate(cands) if c[0] * c[1] * c[2] == B]
            if m > 1e-9:
                assert min(J)[1] == sid


def test_candidate_proportional_guidance_selects_that_candidate():
    for sid, (bT, bH, bW) in enumerate(O.candidate_shapes()):
        g = np.array([4.0 ** -math.log2(bT), 4.0 ** -math.log2(bH), 4.0 ** -math.log2(bW)]) * 3.7
        B = np.array([bT * bH * bW])
        ids, m = O.nearest_shape(O.lstar(g[None], B), B)
        assert ids[0] == sid and m[0] > 0.5


# ---------------------------------------------------------------- tiny workload
def _tiny():
    from dynamic_block_sparse_stats_b200.synth import make_inputs
    inp = make_inputs("tiny", "cpu")
    return inp, inp["workload"]


def test_tiny_plan_expectations():
    """Noise zones have rho_raw near 1 (unit variance, small frame-mean
    differences); the zone with the amplitude-3 sinusoid along H has
    rho_raw near 5.5, so it is the only 64-volume zone, split finest
    along H; the others fall under tau_256: 3*2 + 8 = 14 blocks."""
    inp, w = _tiny()
    pl = O.plan(inp["V"].float().numpy(), inp["a"].numpy(), w.T, w.H, w.W)
    hp = pl.heads[0]
    assert hp.B.tolist() == [256, 64, 256, 256]
    assert O.candidate_shapes()[hp.shape[1]][1] == 2
    assert hp.blocks.shape[0] == 14
    assert np.argmax(hp.g[1]) == 1


# ---------------------------------------------------------------- permutation
def test_permutation_is_a_block_contiguous_bijection():
    rng = np.random.default_rng(10)
    T, H, W = 16, 16, 24
    sid = rng.integers(0, 16, size=(T // 8) * (H // 8) * (W // 8))
    blocks = O.head_blocks(T, H, W, sid)
    perm = O.permutation(T, H, W, blocks)
    assert np.array_equal(np.sort(perm), np.arange(T * H * W))
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size)
    assert np.array_equal(perm[inv], np.arange(perm.size))
    grid = np.arange(T * H * W).reshape(T, H, W)
    cands = O.candidate_shapes()
    off = 0
    for (t0, y0, x0, s, B, p0) in blocks:
        bT, bH, bW = cands[s]
        assert p0 == off and B == bT * bH * bW
        box = grid[t0:t0 + bT, y0:y0 + bH, x0:x0 + bW].reshape(-1)
        assert np.array_equal(perm[p0:p0 + B], box)
        off += B
    assert off == T * H * W


# ---------------------------------------------------------------- selection
def test_block_means_and_scores_on_exact_inputs():
    """Inputs on a coarse grid (multiples of 1/16, |x| < 4) make every fp32 sum
    exact, so the fp32 block means must equal the float64 box means and the
    scores the float64 dot products."""
    rng = np.random.default_rng(11)
    T, H, W = 8, 16, 16
    sid = np.array([0, 7, 13, 3])
    blocks = O.head_blocks(T, H, W, sid)
    hp = O.HeadPlan(None, sid, None, None, None, None, blocks, O.permutation(T, H, W, blocks))
    X = rng.integers(-63, 64, size=(T * H * W, 8)) / 16.0
    Y = rng.integers(-63, 64, size=(T * H * W, 8)) / 16.0
    xb = O.block_means_fp32(X, hp)
    grid = X.reshape(T, H, W, 8)
    cands = O.candidate_shapes()
    for b, (t0, y0, x0, s, B, p0) in enumerate(blocks):
        bT, bH, bW = cands[s]
        np.testing.assert_array_equal(xb[b], grid[t0:t0 + bT, y0:y0 + bH, x0:x0 + bW].mean(axis=(0, 1, 2)))
    yb = O.block_means_fp32(Y, hp)
    s = O.block_scores_fp32(xb, yb, 1.0)
    np.testing.assert_allclose(s, xb.astype(np.float64) @ yb.astype(np.float64).T, rtol=2e-6)
    # the attention scale multiplies the scores (a power of two scales exactly)
    s8 = O.block_scores_fp32(xb, yb, 0.125)
    np.testing.assert_array_equal(s8, s * np.float32(0.125))


def _brute_select(s, k, p):
    """Full sort, accumulate probabilities until the running sum reaches p."""
    nb = len(s)
    order = sorted(range(nb), key=lambda j: (-float(s[j]), j))
    m = max(float(v) for v in s)
    e = [math.exp(float(s[j]) - m) for j in order]
    Z = math.fsum(e)
    run, n_p = 0.0, nb
    for n in range(1, nb + 1):
        run += e[n - 1]
        if run >= p * Z:
            n_p = n
            break
    return sorted(order[:max(k, n_p)]), n_p


@pytest.mark.parametrize("seed", range(6))
def test_hybrid_select_matches_bruteforce_and_properties(seed):
    rng = np.random.default_rng(100 + seed)
    nb = int(rng.integers(5, 80))
    s = (rng.normal(size=nb) * rng.uniform(0.1, 6)).astype(np.float32)
    if seed == 0:
        s[3:9] = s[2]               # exact ties: broken by lower index
    k = int(rng.integers(1, nb + 1))
    p = float(np.float32(rng.uniform(0.05, 0.99)))
    ids, info = O.hybrid_select_row(s, k, p)
    want, n_p = _brute_select(s, k, p)
    if info["p_margin"] > 1e-12:
        assert ids.tolist() == want and info["n_p"] == n_p
    P = np.exp(s.astype(np.float64) - s.max())
    P /= P.sum()
    assert len(ids) >= k and P[ids].sum() >= p - 1e-12
    # the kept set is a prefix of the (score desc, index asc) order
    kept = set(ids.tolist())
    order = sorted(range(nb), key=lambda j: (-float(s[j]), j))
    assert set(order[:len(ids)]) == kept


def test_select_all_and_topk_only_limits():
    s = np.array([3.0, 1.0, 2.0, 2.0, -1.0], np.float32)
    ids, info = O.hybrid_select_row(s, 5, 0.5)
    assert ids.tolist() == [0, 1, 2, 3, 4]
    ids, info = O.hybrid_select_row(s, 2, 1e-9)      # Top-p takes 1 block, Top-k 2
    assert ids.tolist() == [0, 2] and info["n_p"] == 1
    ids, info = O.hybrid_select_row(s, 1, 0.0)
    assert ids.tolist() == [0]
    assert O.topk_count(100, 0.04, 0) == 4 and O.topk_count(100, 0.0, 7) == 7
    assert O.topk_count(10, 0.001, 0) == 1 and O.topk_count(10, 0.0, 50) == 10


def test_top_p_crossing_exactly_at_p_is_kept():
    """Reading: the Top-p prefix is the shortest whose mass is >= p.  Four
    equal scores give P = 1/4 each, exactly, so the mass reaches p = 1/2 at
    the second block and p = 3/4 at the third (a strict > would take one
    more)."""
    s = np.ones(4, np.float32)
    ids, info = O.hybrid_select_row(s, 1, 0.5)
    assert info["n_p"] == 2 and ids.tolist() == [0, 1]
    ids, info = O.hybrid_select_row(s, 1, 0.75)
    assert info["n_p"] == 3 and ids.tolist() == [0, 1, 2]


def test_top_p_one_keeps_blocks_whose_weight_underflows():
    """Every softmax weight is positive, so p = 1 is reached only with the
    last block, even when float64 rounds the tail weights to 0 (exp(-800))."""
    s = np.array([0.0, -800.0, -900.0, -800.0], np.float32)
    ids, info = O.hybrid_select_row(s, 1, 1.0)
    assert info["n_p"] == 4 and ids.tolist() == [0, 1, 2, 3]
    ids, info = O.hybrid_select_row(s, 1, 0.999)
    assert info["n_p"] == 1 and ids.tolist() == [0]


# ---------------------------------------------------------------- attention
def _dense_attention_loops(q, k, v, scale, mask=None):
    """Independent plain formulation: one query at a time, explicit masking."""
    out = np.zeros_like(q, dtype=np.float64)
    lse = np.zeros(q.shape[0])
    for i in range(q.shape[0]):
        s = (k @ q[i]) * scale
        if mask is not None:
            s = np.where(mask[i], s, -np.inf)
        m = s.max()
        w = np.exp(s - m)
        out[i] = (w[:, None] * v).sum(axis=0) / w.sum()
        lse[i] = m + math.log(w.sum())
    return out, lse


def _small_problem(seed=12, T=8, H=16, W=16, heads=1, D=16):
    rng = np.random.default_rng(seed)
    N = T * H * W
    Q = rng.normal(size=(N, heads, D)) * 0.8
    K = rng.normal(size=(N, heads, D)) * 0.8
    V = rng.normal(size=(N, heads, D))
    V[: N // 2] *= 3.0
    pl = O.plan(V, None, T, H, W)
    return Q, K, V, pl


def test_attention_select_all_equals_dense():
    Q, K, V, pl = _small_problem()
    nb = pl.heads[0].blocks.shape[0]
    sel = O.select(Q, K, pl, topk_abs=nb, top_p=0.5)
    scale = 0.25
    Os, Ls = O.attention_fwd(Q, K, V, pl, sel, scale)
    Od, Ld = _dense_attention_loops(Q[:, 0], K[:, 0], V[:, 0], scale)
    np.testing.assert_allclose(Os[:, 0], Od, atol=1e-12)
    np.testing.assert_allclose(Ls[0], Ld, atol=1e-12)


def test_attention_equals_masked_dense_and_rows_normalise():
    Q, K, V, pl = _small_problem(13)
    sel = O.select(Q, K, pl, topk_abs=2, top_p=0.3)
    hp = pl.heads[0]
    N = Q.shape[0]
    mask = np.zeros((N, N), dtype=bool)
    for (i, ids, _info) in sel[0]:
        qi = hp.perm[hp.blocks[i, 5]:hp.blocks[i, 5] + hp.blocks[i, 4]]
        for j in ids:
            kj = hp.perm[hp.blocks[j, 5]:hp.blocks[j, 5] + hp.blocks[j, 4]]
            mask[np.ix_(qi, kj)] = True
    scale = 0.25
    Os, Ls = O.attention_fwd(Q, K, V, pl, sel, scale)
    Od, Ld = _dense_attention_loops(Q[:, 0], K[:, 0], V[:, 0], scale, mask)
    np.testing.assert_allclose(Os[:, 0], Od, atol=1e-12)
    np.testing.assert_allclose(Ls[0], Ld, atol=1e-12)
    # softmax rows of the selected keys sum to one
    s = (Q[:, 0] @ K[:, 0].T) * scale
    rows = np.where(mask, np.exp(s - Ls[0][:, None]), 0.0).sum(axis=1)
    np.testing.assert_allclose(rows, 1.0, atol=1e-12)


def test_backward_matches_central_differences():
    Q, K, V, pl = _small_problem(14, D=8)
    sel = O.select(Q, K, pl, topk_abs=2, top_p=0.4)
    rng = np.random.default_rng(15)
    dO = rng.normal(size=Q.shape)
    scale = 0.35
    dQ, dK, dV = O.attention_bwd(Q, K, V, dO, pl, sel, scale)

    def f(Qx, Kx, Vx):
        Ox, _ = O.attention_fwd(Qx, Kx, Vx, pl, sel, scale)
        return float((Ox * dO).sum())

    eps = 1e-6
    for name, X, G in (("Q", Q, dQ), ("K", K, dK), ("V", V, dV)):
        for idx in [(3, 0, 1), (700, 0, 5), (1500, 0, 7), (2047, 0, 0)]:
            Xp, Xm = X.copy(), X.copy()
            Xp[idx] += eps
            Xm[idx] -= eps
            args_p = {"Q": Q, "K": K, "V": V}
            args_m = dict(args_p)
            args_p[name], args_m[name] = Xp, Xm
            num = (f(args_p["Q"], args_p["K"], args_p["V"]) - f(args_m["Q"], args_m["K"], args_m["V"])) / (2 * eps)
            assert abs(num - G[idx]) < 1e-6 * max(1.0, abs(num)), (name, idx, num, G[idx])


def test_backward_select_all_equals_torch_autograd():
    Q, K, V, pl = _small_problem(16, T=8, H=8, W=16, D=8)
    nb = pl.heads[0].blocks.shape[0]
    sel = O.select(Q, K, pl, topk_abs=nb, top_p=0.5)
    rng = np.random.default_rng(17)
    dO = rng.normal(size=Q.shape)
    scale = 0.3
    dQ, dK, dV = O.attention_bwd(Q, K, V, dO, pl, sel, scale)
    q, k, v = (torch.tensor(x[:, 0], dtype=torch.float64, requires_grad=True) for x in (Q, K, V))
    o = torch.softmax((q @ k.T) * scale, dim=1) @ v
    o.backward(torch.tensor(dO[:, 0]))
    np.testing.assert_allclose(dQ[:, 0], q.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dK[:, 0], k.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dV[:, 0], v.grad.numpy(), atol=1e-11)


def test_key_block_backward_matches_central_differences_and_the_full_backward():
    """attention_bwd_key_block (one key block's dK, dV from the rows that
    selected it) against float64 central differences of <O, dO> with respect
    to that block's keys and values, and against attention_bwd's rows of the
    same block, on every key block of a small grid."""
    Q, K, V, pl = _small_problem(18, D=8)
    sel = O.select(Q, K, pl, topk_abs=2, top_p=0.4)
    rng = np.random.default_rng(19)
    dO = rng.normal(size=Q.shape)
    scale = 0.35
    hp = pl.heads[0]
    _, gK, gV = O.attention_bwd(Q, K, V, dO, pl, sel, scale)
    rows = {i: ids for (i, ids, _info) in sel[0]}
    nb = hp.blocks.shape[0]
    for j in range(nb):
        users = [(i, ids) for i, ids in rows.items() if j in ids]
        kj, dK, dV = O.attention_bwd_key_block(Q[:, 0], K[:, 0], V[:, 0], dO[:, 0], hp, j, users, scale)
        np.testing.assert_allclose(dK, gK[kj, 0], atol=1e-12)
        np.testing.assert_allclose(dV, gV[kj, 0], atol=1e-12)

    def f(Kx, Vx):
        Ox, _ = O.attention_fwd(Q, Kx, Vx, pl, sel, scale)
        return float((Ox * dO).sum())

    j = max(range(nb), key=lambda b: sum(b in ids for ids in rows.values()))   # the most-used key block
    users = [(i, ids) for i, ids in rows.items() if j in ids]
    kj, dK, dV = O.attention_bwd_key_block(Q[:, 0], K[:, 0], V[:, 0], dO[:, 0], hp, j, users, scale)
    eps = 1e-6
    for t in (0, kj.size // 2, kj.size - 1):
        for c in (0, 5):
            for X, G in ((K, dK), (V, dV)):
                Xp, Xm = X.copy(), X.copy()
                Xp[kj[t], 0, c] += eps
                Xm[kj[t], 0, c] -= eps
                if X is K:
                    num = (f(Xp, V) - f(Xm, V)) / (2 * eps)
                else:
                    num = (f(K, Xp) - f(K, Xm)) / (2 * eps)
                assert abs(num - G[t, c]) < 1e-6 * max(1.0, abs(num)), (t, c, num, G[t, c])
