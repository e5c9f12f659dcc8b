"""CPU oracle for the Prism dynamic block-sparse video self-attention path.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may import this module.  The
product path (the CUDA library and its Python binding) never calls it, and it
shares no code, tables or helpers with that path.

It is a plain, slow, step-by-step restatement of what the pages describe,
in float64 unless a step's result decides an integer in the kernel's
precision (block means and block scores, see below).

Sources, cited by page title and section:
  [DIGEST]  "Prism：为原生 2K 视频音频联合生成设计的动态稀疏注意力"
            (nanless.github.io audio-paper digest).  Sections
            "每个宏区如何估计视觉变化与音频影响" (zone guidance signals),
            "信息密度如何决定块体积与具体边长" (density, volume, shape; the
            equations for g_d(m), rho_raw(m) and J(b_T,b_H,b_W)),
            "混合块选择如何为每个查询定稀疏度" (hybrid Top-k/Top-p),
            "模型如何训练与哪些参数更新" (gradients, 64-token units).
  [REVIEW]  "Prism: динамическое разреженное внимание для нативного обучения
            моделей совместной генерации видео и аудио в 2K" (xyznot.com).
            Method section 1 (sigma^2_{v,d}, r_{v,d}, g_d), section 2
            (B(m), tau_128, tau_256, closed form l*_d, nearest candidate in
            log2 space), section 3 (S_i = Top-k(P_i,k) U Top-p(P_i,p)).

Readings of points the pages leave open are marked READING where they are
applied; each states the choice and why.

Parity status: every function below is pinned by a ``-m "not gpu"`` test
(closed forms, invariants, brute force, independent dense formulations);
tests/mutation_check.py plants plausible mistakes in a copy of this module
and confirms that each one fails a test.  Agreement with the authors' own
implementation on the READING points is unpinned (no implementation is
available).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

ZONE = 8  # Z_T = Z_H = Z_W = 8  [DIGEST] Fig. 2 description; [REVIEW] Key ideas
VOLUMES = (64, 128, 256)  # [DIGEST] density section; [REVIEW] Method §2


# ---------------------------------------------------------------------------
# Candidate shape pool
# ---------------------------------------------------------------------------
def candidate_shapes():
    """The candidate pool: edges from {2,4,8} whose product is 64, 128 or 256
    ([DIGEST] density section: 16 combinations, edges only 2/4/8, product
    exactly 64/128/256).  Enumerating that rule gives exactly 16 shapes.

    Canonical id order (READING): volume ascending, then (b_T,b_H,b_W)
    lexicographic.  Ties in the nearest-shape choice go to the lowest id.
    """
    out = []
    for B in VOLUMES:
        for bT in (2, 4, 8):
            for bH in (2, 4, 8):
                for bW in (2, 4, 8):
                    if bT * bH * bW == B:
                        out.append((bT, bH, bW))
    return out


# ---------------------------------------------------------------------------
# Zone statistics
# ---------------------------------------------------------------------------
def _zones(x, T, H, W):
    """View x[T,H,W,...] as [ZT,8,ZH,8,ZW,8,...] -> [Z, 8(t), 8(y), 8(x), ...]
    with zones in raster order (zT, zH, zW), zW fastest."""
    ZT, ZH, ZW = T // ZONE, H // ZONE, W // ZONE
    rest = x.shape[3:]
    y = x.reshape((ZT, ZONE, ZH, ZONE, ZW, ZONE) + rest)
    perm = (0, 2, 4, 1, 3, 5) + tuple(range(6, 6 + len(rest)))
    return y.transpose(perm).reshape((ZT * ZH * ZW, ZONE, ZONE, ZONE) + rest)


def zone_video_stats(Vh, T, H, W):
    """Per-zone statistics of one head's values Vh [N, D] (float64).

    sigma2[z, d]: [REVIEW] Method §1, sigma^2_{v,d}(m) = (1/D) sum_c
        (1/Z_d) sum_i (Vbar^{(d)}_{m,i,c} - mu^{(d)}_{m,c})^2, where
        Vbar^{(d)}_{m,i} is V mean-pooled over the other two axes at position
        i along axis d and mu^{(d)} is the mean of that profile.
    spatial[z], temporal[z]: the two terms of rho_raw(m) ([DIGEST] density
        section, equation for rho_raw): the channel-mean of the intra-zone
        variance around each frame's mean, and the channel-mean of the
        squared difference of consecutive frame means averaged over the 7
        frame pairs.
    """
    D = Vh.shape[-1]
    v = _zones(Vh.reshape(T, H, W, D).astype(np.float64), T, H, W)   # [Z,8t,8y,8x,D]
    prof_T = v.mean(axis=(2, 3))        # [Z, 8, D]  frame means  mu_bar_{m,t,c}
    prof_H = v.mean(axis=(1, 3))        # [Z, 8, D]  row means
    prof_W = v.mean(axis=(1, 2))        # [Z, 8, D]  column means
    sig2 = np.empty((v.shape[0], 3))
    for d, prof in enumerate((prof_T, prof_H, prof_W)):
        mu = prof.mean(axis=1, keepdims=True)               # mu^{(d)}_{m,c}
        sig2[:, d] = ((prof - mu) ** 2).mean(axis=1).mean(axis=1)
    spatial = ((v - prof_T[:, :, None, None, :]) ** 2).mean(axis=(1, 2, 3)).mean(axis=1)
    diff = prof_T[:, 1:, :] - prof_T[:, :-1, :]             # t = 1..Z_T-1
    temporal = (diff ** 2).sum(axis=1).mean(axis=1) / (ZONE - 1)
    return sig2, spatial, temporal


def a2v_norm(hhat):
    """a = ||h_hat||_2 per video token from the bridge output h_hat [N, C]
    ([DIGEST] zone-guidance section: the vector length of each video
    position's audio-to-video attention output is its audio injection
    strength; [REVIEW] Method §1, a_{t,h,w} = ||h_hat_{t,h,w}||_2).
    float64 from the given (bf16-rounded) values."""
    h = np.asarray(hhat, dtype=np.float64)
    return np.sqrt((h * h).sum(axis=1))


def zone_a2v_stats(a, T, H, W):
    """Per-zone A2V-norm statistics from a [N] (float64), shared by all heads.

    [DIGEST] zone-guidance section: the per-position norm of the
    audio-to-video attention output is averaged over the zone and normalised
    by the global maximum to give the coupling strength; its directional
    variance shares along the axes give the audio direction term.
    [REVIEW] Method §1: abar(m) in [0,1], vhat_{a,d}(m) normalised.

    READING: abar(m) = zone mean / max over zones of the zone mean;
    vhat_{a,d} is the sigma^2 construction of r_{v,d} applied to the scalar
    field a (profiles along d, population variance), divided by its sum
    over d (1/3 each when that sum is 0).
    """
    z = _zones(a.reshape(T, H, W).astype(np.float64), T, H, W)       # [Z,8,8,8]
    abar_raw = z.mean(axis=(1, 2, 3))
    sig2 = np.empty((z.shape[0], 3))
    for d, ax in enumerate(((2, 3), (1, 3), (1, 2))):
        prof = z.mean(axis=ax)                               # [Z, 8]
        mu = prof.mean(axis=1, keepdims=True)
        sig2[:, d] = ((prof - mu) ** 2).mean(axis=1)
    return abar_raw, sig2


def shares(sig2):
    """Normalise per-axis variances to shares summing to 1 ([REVIEW] Method
    §1, r_{v,d} = sigma^2_d / sum_d' sigma^2_d').  READING: a zone whose
    three variances are all 0 gets 1/3 on every axis."""
    tot = sig2.sum(axis=-1, keepdims=True)
    out = np.full_like(sig2, 1.0 / 3.0)
    nz = tot[..., 0] > 0
    out[nz] = sig2[nz] / tot[nz]
    return out


def variation_indicator(r, abar=None, vhat=None, eps=1e-6, video=True, audio=True):
    """g_d(m) = r_{v,d}(m) + abar(m) * vhat_{a,d}(m) + eps  ([DIGEST]
    equation for g_d(m); [REVIEW] Method §1).  Layer 1 has no cached
    audio-to-video output, so only the video term is used ([DIGEST]
    zone-guidance section).  video=False / audio=False drop a term, as in
    the guidance ablation ([DIGEST] ablation section)."""
    g = r if video else np.zeros_like(r)
    if audio and abar is not None:
        g = g + abar[:, None] * vhat
    return g + eps


def normalise_by_max(x):
    """x / max(x) over zones ([DIGEST] density section: normalised by the
    global maximum to [0,1]).  READING: 0 everywhere when the maximum is 0."""
    m = x.max()
    if m <= 0:
        return np.zeros_like(x)
    return x / m


def volumes(rho, tau128=0.5, tau256=0.25):
    """B(m) from the normalised density ([DIGEST] density section: high
    density -> 64, low -> 256, middle -> 128, thresholds 0.5 and 0.25;
    [REVIEW] Method §2).  READING: rho >= tau_128 -> 64;
    tau_256 <= rho < tau_128 -> 128; rho < tau_256 -> 256.
    Returns (B, margin) with margin = distance to the nearer threshold."""
    B = np.where(rho >= tau128, 64, np.where(rho >= tau256, 128, 256))
    margin = np.minimum(np.abs(rho - tau128), np.abs(rho - tau256))
    return B, margin


def lstar(g, B, alpha=0.5):
    """Closed-form optimum of J = sum_d g_d (b_d^2 - 1) subject to
    prod_d b_d = B, in log2 space ([REVIEW] Method §2):
      l*_d = -1/2 log2 g_d + 1/3 (S + 1/2 sum_d' log2 g_d'),  S = log2 B.
    alpha generalises the exponent of b*_d proportional to g_d^(-alpha)
    (the mapping ablation of [DIGEST]; 1/2 is the Lagrange value).
    g: [..., 3], B: [...]."""
    lg = np.log2(g)
    S = np.log2(B.astype(np.float64))
    return -alpha * lg + (S[..., None] + alpha * lg.sum(axis=-1, keepdims=True)) / 3.0


def nearest_shape(ls, B):
    """Shape id minimising the Euclidean distance in log2 space between a
    candidate of volume B and l* ([REVIEW] Method §2; [DIGEST] density
    section: quantised to the nearest candidate after a log transform).
    Ties go to the lowest canonical id.  Returns (id, margin) where margin is
    the gap between the best and second-best squared distances."""
    cands = candidate_shapes()
    ids = np.empty(B.shape, dtype=np.int64)
    margin = np.empty(B.shape)
    for idx in np.ndindex(B.shape):
        best, second, best_id = math.inf, math.inf, -1
        for cid, (bT, bH, bW) in enumerate(cands):
            if bT * bH * bW != B[idx]:
                continue
            l = (math.log2(bT), math.log2(bH), math.log2(bW))
            dist = sum((l[d] - ls[idx][d]) ** 2 for d in range(3))
            if dist < best:
                second, best, best_id = best, dist, cid
            elif dist < second:
                second = dist
        ids[idx] = best_id
        margin[idx] = second - best
    return ids, margin


# ---------------------------------------------------------------------------
# Plan: volumes, shapes, blocks, permutation
# ---------------------------------------------------------------------------
@dataclass
class HeadPlan:
    B: np.ndarray            # [Z] volume per zone
    shape: np.ndarray        # [Z] candidate id per zone
    g: np.ndarray            # [Z,3]
    rho: np.ndarray          # [Z]
    vol_margin: np.ndarray   # [Z]
    shape_margin: np.ndarray  # [Z]
    blocks: np.ndarray       # [Nb, 6]: t0, y0, x0, shape id, B, p0
    perm: np.ndarray         # [N] natural token index of permuted position p


@dataclass
class Plan:
    T: int
    H: int
    W: int
    heads: list = field(default_factory=list)  # HeadPlan per head


def block_tokens(T, H, W, t0, y0, x0, shape_id):
    """Natural indices of one block's tokens in raster (t, y, x) order, x
    fastest (READING: the pages only require blocks to be contiguous after
    the permutation)."""
    bT, bH, bW = candidate_shapes()[shape_id]
    t = np.arange(t0, t0 + bT)[:, None, None]
    y = np.arange(y0, y0 + bH)[None, :, None]
    x = np.arange(x0, x0 + bW)[None, None, :]
    return ((t * H + y) * W + x).reshape(-1)


def head_blocks(T, H, W, shape_per_zone):
    """Blocks of one head: zones in raster order (zW fastest); inside a zone
    the blocks in raster order of the (8/b_T, 8/b_H, 8/b_W) block grid; each
    zone holds 512 tokens, so zone m starts at permuted position 512*m.
    One shape per zone, no token-level mixing ([DIGEST] density section)."""
    ZT, ZH, ZW = T // ZONE, H // ZONE, W // ZONE
    cands = candidate_shapes()
    rows = []
    m = 0
    for zt in range(ZT):
        for zh in range(ZH):
            for zw in range(ZW):
                sid = int(shape_per_zone[m])
                bT, bH, bW = cands[sid]
                B = bT * bH * bW
                p0 = m * ZONE ** 3
                for it in range(ZONE // bT):
                    for ih in range(ZONE // bH):
                        for iw in range(ZONE // bW):
                            rows.append((zt * ZONE + it * bT, zh * ZONE + ih * bH,
                                         zw * ZONE + iw * bW, sid, B, p0))
                            p0 += B
                m += 1
    return np.array(rows, dtype=np.int64)


def permutation(T, H, W, blocks):
    """perm[p] = natural index of the token at permuted position p; tokens
    of each block are contiguous, Q, K and V share it ([DIGEST] hybrid
    selection section: queries, keys and values share one partition)."""
    perm = np.empty(T * H * W, dtype=np.int64)
    for (t0, y0, x0, sid, B, p0) in blocks:
        perm[p0:p0 + B] = block_tokens(T, H, W, t0, y0, x0, sid)
    return perm


def project_v(X, Wv):
    """The layer's value features V = X Wv^T ([DIGEST] zone-guidance section
    and Figure 4: the zone statistics are taken from the value features that
    the video self-attention computes from the tokens).  X [N, C], Wv
    [heads*D, C] (linear-layer weight layout); float64, from the given
    (bf16-rounded) values.  Returns [N, heads*D]."""
    return np.asarray(X, dtype=np.float64) @ np.asarray(Wv, dtype=np.float64).T


def density_raw(spatial, temporal, abar_raw, mode=0):
    """rho_raw(m) ([DIGEST] density section: the intra-zone spatial variance
    plus the temporal frame-difference variance).  The density ablation of
    [DIGEST] swaps it for the spatial term alone (mode 1), the temporal term
    alone (2) or the zone's audio strength (3, the zone mean of a)."""
    if mode == 1:
        return spatial
    if mode == 2:
        return temporal
    if mode == 3:
        if abar_raw is None:
            raise ValueError("density mode 3 needs the A2V norms")
        return abar_raw
    return spatial + temporal


def plan(V, a, T, H, W, tau128=0.5, tau256=0.25, eps=1e-6, map_exponent=0.5, guidance=0, density=0):
    """Per-head plan ([DIGEST] overview: shapes and sparsity are computed per
    head and per layer).  V: [N, heads, D] (bf16 values, any float dtype;
    the guidance ablation of [DIGEST] also feeds K or Q here);
    a: [N] or None (first layer).  map_exponent, guidance (bit 0 drops the
    video term, bit 1 the A2V term) and density select the ablation
    variants; their defaults are the method."""
    V = np.asarray(V)
    heads = V.shape[1]
    abar = vhat = abar_raw = None
    if a is not None:
        abar_raw, sig2a = zone_a2v_stats(np.asarray(a, dtype=np.float64), T, H, W)
        abar = normalise_by_max(abar_raw)
        vhat = shares(sig2a)
    out = Plan(T, H, W)
    for h in range(heads):
        sig2, spatial, temporal = zone_video_stats(V[:, h, :], T, H, W)
        r = shares(sig2)
        g = variation_indicator(r, abar, vhat, eps, video=not (guidance & 1), audio=not (guidance & 2))
        rho = normalise_by_max(density_raw(spatial, temporal, abar_raw, density))
        B, vmargin = volumes(rho, tau128, tau256)
        sid, smargin = nearest_shape(lstar(g, B, map_exponent), B)
        blocks = head_blocks(T, H, W, sid)
        out.heads.append(HeadPlan(B, sid, g, rho, vmargin, smargin, blocks,
                                  permutation(T, H, W, blocks)))
    return out


# ---------------------------------------------------------------------------
# Selection
# ---------------------------------------------------------------------------
def block_means_fp32(Xh, hp: HeadPlan):
    """Block mean of one head's features Xh [N, D] over each block's tokens
    ([DIGEST] hybrid selection section: mean pooling gives each block's
    representative; [REVIEW] Method §3).

    Precision (READING, because the result decides the selected indices):
    fp32 running sum over the block's tokens in its raster order, then a
    multiplication by 1/B (exact, B is a power of two)."""
    X32 = np.asarray(Xh, dtype=np.float32)
    nb = hp.blocks.shape[0]
    out = np.empty((nb, X32.shape[1]), dtype=np.float32)
    by_B = {}
    for b, (t0, y0, x0, sid, B, p0) in enumerate(hp.blocks):
        by_B.setdefault(int(B), []).append(b)
    for B, bl in by_B.items():
        bl = np.array(bl)
        toks = hp.perm[hp.blocks[bl, 5][:, None] + np.arange(B)[None, :]]   # [nb_B, B]
        acc = np.zeros((bl.size, X32.shape[1]), dtype=np.float32)
        for r in range(B):          # left-to-right fp32 sum
            acc = acc + X32[toks[:, r]]
        out[bl] = acc * np.float32(1.0 / B)
    return out


def block_scores_fp32(Qbar, Kbar, scale):
    """s_ij = (Qbar_i . Kbar_j) * scale ([DIGEST] hybrid selection section:
    dot product of block representatives, then softmax).

    READINGS: the scale is the attention scale 1/sqrt(D); precision is fp32,
    the dot product accumulated left to right over channels with the product
    and the sum each rounded to fp32, then one fp32 multiply by the scale."""
    Qbar = np.asarray(Qbar, dtype=np.float32)
    Kbar = np.asarray(Kbar, dtype=np.float32)
    acc = np.zeros((Qbar.shape[0], Kbar.shape[0]), dtype=np.float32)
    for c in range(Qbar.shape[1]):
        acc = acc + np.multiply.outer(Qbar[:, c], Kbar[:, c])
    return acc * np.float32(scale)


def topk_count(nb, topk_frac, topk_abs):
    """k for Top-k.  READING: a positive absolute count wins; otherwise the
    kept fraction of key blocks, rounded up, at least 1, at most N_b."""
    if topk_abs > 0:
        return min(nb, int(topk_abs))
    return min(nb, max(1, int(math.ceil(float(np.float32(topk_frac)) * nb))))


def hybrid_select_row(s_row, k, p):
    """S_i = Top-k(P_i, k) U Top-p(P_i, p) for one query block
    ([REVIEW] Method §3; [DIGEST] hybrid selection section: Top-k gives a
    minimum cover, Top-p adds blocks from the most relevant down until the
    cumulative weight passes the threshold).

    P_i = softmax(s_i) computed in float64 from the fp32 scores.  Order:
    score descending, then index ascending.  READING: "passes" means >= and
    the crossing block is included.  Both sets are prefixes of one order, so
    the union is the prefix of length max(k, n_p).  With p >= 1 every block
    is kept: every P_ij is positive, so in exact arithmetic the cumulative
    probability reaches 1 only with the last block (float64 rounding of the
    running sum must not cut that tail short).

    Returns (sorted ids, info) with info = n, k, n_p and the decision
    margins: the score gap at the prefix boundary and the distance of the
    cumulative probability from p at the Top-p crossing."""
    s = np.asarray(s_row, dtype=np.float32)
    nb = s.size
    j = np.arange(nb)
    order = np.lexsort((j, -s))
    s64 = s[order].astype(np.float64)
    e = np.exp(s64 - s64[0])
    Z = e.sum()
    csum = np.cumsum(e)
    target = float(np.float32(p)) * Z
    if p <= 0:
        n_p = 0
    elif p >= 1:
        n_p = nb
    else:
        hit = np.nonzero(csum >= target)[0]
        n_p = int(hit[0]) + 1 if hit.size else nb
    n = max(k, n_p)
    gap = float(s64[n - 1] - s64[n]) if n < nb else math.inf
    pm = math.inf
    if 0 < n_p <= nb:
        pm = abs(csum[n_p - 1] / Z - p)
        if n_p >= 2:
            pm = min(pm, abs(csum[n_p - 2] / Z - p))
    return np.sort(order[:n]), dict(n=n, k=k, n_p=n_p, score_gap=gap, p_margin=pm)


def select(Q, K, pl: Plan, topk_frac=0.0, topk_abs=0, top_p=0.9, scale=None, heads=None,
           rows=None):
    """Per head: block means, block scores, hybrid selection for every query
    block (or only the query blocks listed in `rows`).  Returns, per head, a
    list of (query block, sorted key ids, info)."""
    Q = np.asarray(Q)
    K = np.asarray(K)
    D = Q.shape[-1]
    if scale is None:
        scale = float(np.float32(1.0 / math.sqrt(D)))
    res = []
    for h in (range(len(pl.heads)) if heads is None else heads):
        hp = pl.heads[h]
        qb = block_means_fp32(Q[:, h, :], hp)
        kb = block_means_fp32(K[:, h, :], hp)
        nb = qb.shape[0]
        k = topk_count(nb, topk_frac, topk_abs)
        want = list(range(nb)) if rows is None else [i for i in rows if i < nb]
        s_all = block_scores_fp32(qb[want], kb, scale) if want else np.zeros((0, nb), np.float32)
        out = []
        for r, i in enumerate(want):
            ids, info = hybrid_select_row(s_all[r], k, top_p)
            out.append((i, ids, info))
        res.append(out)
    return res


# ---------------------------------------------------------------------------
# Attention over the selected blocks
# ---------------------------------------------------------------------------
def attention_fwd_block(Qh, Kh, Vh, hp: HeadPlan, i, key_blocks, scale):
    """Exact attention of the queries of block i over the union of the tokens
    of the selected key blocks ([DIGEST] hybrid selection section: exact
    attention with the full query tokens and the selected key/value blocks,
    online softmax; the result goes back to the original order).
    Returns (natural query indices, O [B_i, D], LSE [B_i]) in float64."""
    t0, y0, x0, sid, B, p0 = hp.blocks[i]
    qi = hp.perm[p0:p0 + B]
    keys = np.concatenate([hp.perm[hp.blocks[j, 5]:hp.blocks[j, 5] + hp.blocks[j, 4]]
                           for j in key_blocks])
    q = Qh[qi].astype(np.float64)
    k = Kh[keys].astype(np.float64)
    v = Vh[keys].astype(np.float64)
    s = (q @ k.T) * scale
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=1, keepdims=True)
    o = (e @ v) / l
    lse = (m + np.log(l))[:, 0]
    return qi, o, lse


def attention_fwd(Q, K, V, pl: Plan, sel, scale, heads=None, rows=None):
    """O [N, heads, D] and LSE [heads, N] (float64, natural order).  Rows not
    computed (when `rows` restricts the query blocks) are NaN."""
    Q, K, V = (np.asarray(x) for x in (Q, K, V))
    N, nh, D = Q.shape
    O = np.full((N, nh, D), np.nan)
    LSE = np.full((nh, N), np.nan)
    for hi, h in enumerate(range(nh) if heads is None else heads):
        hp = pl.heads[h]
        for (i, ids, _info) in sel[hi]:
            if rows is not None and i not in rows:
                continue
            qi, o, lse = attention_fwd_block(Q[:, h], K[:, h], V[:, h], hp, i, ids, scale)
            O[qi, h] = o
            LSE[h, qi] = lse
    return O, LSE


def attention_bwd(Q, K, V, dO, pl: Plan, sel, scale, heads=None):
    """Gradients of the block-sparse attention ([DIGEST] training section:
    shape assignment and block selection are constants; gradients flow only
    through the sparse attention on the selected blocks).
    Textbook backward of softmax attention restricted to the selected keys:
      P = softmax(s), dV = P^T dO, dP = dO V^T, D_q = sum_k P dP,
      dS = P (dP - D_q), dQ = scale dS K, dK = scale dS^T Q.
    Returns dQ, dK, dV [N, heads, D] float64."""
    Q, K, V, dO = (np.asarray(x) for x in (Q, K, V, dO))
    N, nh, D = Q.shape
    dQ = np.zeros((N, nh, D))
    dK = np.zeros((N, nh, D))
    dV = np.zeros((N, nh, D))
    for hi, h in enumerate(range(nh) if heads is None else heads):
        hp = pl.heads[h]
        for (i, ids, _info) in sel[hi]:
            t0, y0, x0, sid, B, p0 = hp.blocks[i]
            qi = hp.perm[p0:p0 + B]
            keys = np.concatenate([hp.perm[hp.blocks[j, 5]:hp.blocks[j, 5] + hp.blocks[j, 4]]
                                   for j in ids])
            q = Q[qi, h].astype(np.float64)
            k = K[keys, h].astype(np.float64)
            v = V[keys, h].astype(np.float64)
            do = dO[qi, h].astype(np.float64)
            s = (q @ k.T) * scale
            P = np.exp(s - s.max(axis=1, keepdims=True))
            P /= P.sum(axis=1, keepdims=True)
            dv = P.T @ do
            dP = do @ v.T
            Dq = (P * dP).sum(axis=1, keepdims=True)
            dS = P * (dP - Dq)
            dQ[qi, h] += scale * (dS @ k)
            np.add.at(dK[:, h], keys, scale * (dS.T @ q))
            np.add.at(dV[:, h], keys, dv)
    return dQ, dK, dV


def attention_bwd_key_block(Qh, Kh, Vh, dOh, hp: HeadPlan, j, users, scale):
    """dK and dV of the tokens of one key block j, from the query blocks that
    selected it (the same textbook backward as attention_bwd, restricted to
    the outputs of block j; [DIGEST] training section).  Each user row needs
    its full softmax over its own selection (for P and for
    D_q = sum_k P_qk dP_qk = dO_q . O_q), but only block j's columns of dS
    and P enter the result:
      dV_j = sum_i P_{i,j}^T dO_i,   dK_j = scale * sum_i dS_{i,j}^T Q_i.
    users: (query block i, its selected key blocks) pairs, j among them.
    Returns (natural key indices of block j, dK_j [B_j, D], dV_j [B_j, D])
    in float64."""
    kj = hp.perm[hp.blocks[j, 5]:hp.blocks[j, 5] + hp.blocks[j, 4]]
    D = Qh.shape[1]
    dK = np.zeros((kj.size, D))
    dV = np.zeros((kj.size, D))
    for (i, ids) in users:
        qi = hp.perm[hp.blocks[i, 5]:hp.blocks[i, 5] + hp.blocks[i, 4]]
        keys = np.concatenate([hp.perm[hp.blocks[b, 5]:hp.blocks[b, 5] + hp.blocks[b, 4]] for b in ids])
        q = Qh[qi].astype(np.float64)
        do = dOh[qi].astype(np.float64)
        k = Kh[keys].astype(np.float64)
        v = Vh[keys].astype(np.float64)
        s = (q @ k.T) * scale
        P = np.exp(s - s.max(axis=1, keepdims=True))
        P /= P.sum(axis=1, keepdims=True)
        o = P @ v
        Dq = (do * o).sum(axis=1, keepdims=True)          # = sum_k P dP over the row
        at = int(np.searchsorted(np.asarray(ids), j))     # ids ascending: block j's columns in the row
        c0 = int(sum(hp.blocks[b, 4] for b in ids[:at]))
        Pj = P[:, c0:c0 + kj.size]
        dPj = do @ Vh[kj].astype(np.float64).T
        dSj = Pj * (dPj - Dq)
        dV += Pj.T @ do
        dK += scale * (dSj.T @ q)
    return kj, dK, dV


def csr_from_selection(sel, nb_cap):
    """Flatten a per-head selection into row_ptr [heads*nb_cap+1] and col, the
    layout the library returns (row = head*nb_cap + query block)."""
    counts = np.zeros(len(sel) * nb_cap, dtype=np.int64)
    cols = {}
    for h, rows in enumerate(sel):
        for (i, ids, _info) in rows:
            counts[h * nb_cap + i] = len(ids)
            cols[h * nb_cap + i] = ids
    row_ptr = np.zeros(counts.size + 1, dtype=np.int64)
    np.cumsum(counts, out=row_ptr[1:])
    col = np.zeros(int(row_ptr[-1]), dtype=np.int64)
    for r, ids in cols.items():
        col[row_ptr[r]:row_ptr[r + 1]] = ids
    return row_ptr, col
