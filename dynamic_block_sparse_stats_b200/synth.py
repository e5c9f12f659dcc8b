"""Seeded synthetic inputs for the Prism video self-attention path.

This module only draws inputs.  It contains none of the method's arithmetic
(no zone statistics, shapes, pooling, scores or attention), so both the CPU
oracle and the CUDA path may take their inputs from it.

The workloads imitate the shapes the Prism pages describe: latent grids of
720p, 1080p and native 2K video (about 870K tokens at 2K, "Prism" digest,
section on data and benchmarks), with a smooth repeated background and a few
compact, fast-changing "sounding" regions (the same digest, section on why
full attention and fixed sparsity fail at 2K), plus an audio-to-video
cross-attention norm map that is strong on some of those regions.

Layout of every returned tensor (natural raster token order
n = (t*H + y)*W + x):
  Q, K, V, dO : bf16 [N, heads, head_dim]
  a           : fp32 [N]   (norm of the audio-to-video attention output)

All random draws come from torch generators seeded with (seed, tensor id,
chunk id).  Bits are reproducible on one device type; CPU and CUDA draw
different bits, which is fine because both sides of every parity check are
fed the same tensors.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, asdict

import torch

ZONE = 8  # macro-zone edge; only used here to place static zones


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    H: int
    W: int
    heads: int
    head_dim: int
    topk_frac: float = 0.0
    topk_abs: int = 0
    top_p: float = 0.9
    kind: str = "regions"      # "tiny" or "regions"
    regions: int = 0           # moving high-variance regions in V
    radius: float = 0.0        # disc radius of those regions, in tokens
    a_regions: int = 0         # regions that also carry an A2V norm blob
    static_frac: float = 0.0   # share of untouched zones made exactly static
    zoom: bool = False         # one region's radius doubles over the clip
    s_q: float = 3.0           # query sharpness outside static zones
    s_q_static: float = 0.5    # query sharpness inside static zones
    backward: bool = False

    @property
    def N(self) -> int:
        return self.T * self.H * self.W

    def describe(self) -> dict:
        d = asdict(self)
        d["tokens"] = self.N
        return d


WORKLOADS = {
    # 8x16x16 grid, one head, D=64: four zones; one zone carries an
    # amplitude-3 sinusoid along H, one zone an A2V blob.
    "tiny": Workload("tiny", 8, 16, 16, 1, 64, topk_abs=2, top_p=0.9, kind="tiny"),
    # the same grid and fields at D=128 (the fused backward's head size)
    "tiny_d128": Workload("tiny_d128", 8, 16, 16, 1, 128, topk_abs=2, top_p=0.9, kind="tiny"),
    # Parity-test grids: small enough for the oracle, several tiles, and
    # a zone count that is not a multiple of any tile size.
    "small": Workload("small", 16, 24, 40, 2, 128, topk_frac=0.10, top_p=0.9,
                      regions=2, radius=4, a_regions=1, static_frac=0.3),
    "small_d64": Workload("small_d64", 8, 32, 24, 3, 64, topk_frac=0.15, top_p=0.9,
                          regions=2, radius=4, a_regions=1),
    "720p": Workload("720p", 24, 48, 80, 24, 128, topk_frac=0.08, top_p=0.9,
                     regions=3, radius=6, a_regions=2),
    # 720p grid with 8 heads: every tensor (189 MB) exceeds L2, a few GB in
    # total -- sized for kernel profiling
    "720p_h8": Workload("720p_h8", 24, 48, 80, 8, 128, topk_frac=0.08, top_p=0.9,
                        regions=3, radius=6, a_regions=2),
    "1080p": Workload("1080p", 32, 72, 120, 24, 128, topk_frac=0.06, top_p=0.9,
                      regions=6, radius=8, a_regions=3, static_frac=0.3),
    "2k": Workload("2k", 56, 96, 160, 24, 128, topk_frac=0.04, top_p=0.9,
                   regions=10, radius=10, a_regions=4, zoom=True),
    "2k_train": Workload("2k_train", 56, 96, 160, 24, 128, topk_frac=0.04, top_p=0.9,
                         regions=10, radius=10, a_regions=4, zoom=True, backward=True),
}

# tensor ids used as generator streams
_ID_VBG, _ID_VREG, _ID_F, _ID_N1, _ID_N2, _ID_ANOISE, _ID_DO, _ID_LAYOUT, _ID_HHAT, _ID_WV = range(1, 11)
_CHUNK = 256  # channels per generation chunk (fixed, so bits do not depend on memory)


def _gen(device, seed: int, tid: int, chunk: int = 0) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + tid * 10_007 + chunk) & 0x7FFFFFFFFFFFFFFF)
    return g


def _taps(sigma: float = 2.0, radius: int = 6) -> list[float]:
    w = [math.exp(-(k * k) / (2.0 * sigma * sigma)) for k in range(-radius, radius + 1)]
    s = sum(w)
    return [v / s for v in w]


def _blur_axis(x: torch.Tensor, dim: int, taps: list[float]) -> torch.Tensor:
    r = len(taps) // 2
    out = x * taps[r]
    n = x.shape[dim]
    for k in range(1, r + 1):
        if k >= n:
            break
        wk = taps[r + k]
        # out[i] += w * x[i-k]  and  out[i] += w * x[i+k]   (zero outside)
        out.narrow(dim, k, n - k).add_(x.narrow(dim, 0, n - k), alpha=wk)
        out.narrow(dim, 0, n - k).add_(x.narrow(dim, k, n - k), alpha=wk)
    return out


def _lowpass_noise(shape_thw, channels, device, seed, tid, std):
    """White N(0,1) noise [T,H,W,channels] blurred by a separable Gaussian
    (sigma 2 tokens per axis, zero padded), scaled so that the interior std
    equals `std`.  Generated in fixed channel chunks."""
    T, H, W = shape_thw
    taps = _taps()
    interior_std = sum(t * t for t in taps) ** 1.5   # std of blurred unit white noise
    out = torch.empty((T, H, W, channels), dtype=torch.float32, device=device)
    for c0 in range(0, channels, _CHUNK):
        c1 = min(channels, c0 + _CHUNK)
        z = torch.randn((T, H, W, c1 - c0), generator=_gen(device, seed, tid, c0 // _CHUNK),
                        device=device, dtype=torch.float32)
        for d in range(3):
            z = _blur_axis(z, d, taps)
        out[..., c0:c1] = z * (std / interior_std)
    return out


@dataclass
class Layout:
    centers: list = field(default_factory=list)   # per region: list of (y, x) per frame
    radii: list = field(default_factory=list)     # per region: list of radius per frame
    static_zones: list = field(default_factory=list)  # (zT, zH, zW)


def _region_layout(w: Workload, device, seed) -> Layout:
    g = _gen("cpu", seed, _ID_LAYOUT)
    lay = Layout()
    for r in range(w.regions):
        zoom = w.zoom and r == 0
        rad_t = [w.radius * (2.0 ** (t / w.T)) if zoom else w.radius for t in range(w.T)]
        rmax = max(rad_t)
        axis = int(torch.randint(0, 2, (1,), generator=g))       # 0: moves along H, 1: along W
        sign = 1 if int(torch.randint(0, 2, (1,), generator=g)) else -1
        L_move = w.H if axis == 0 else w.W
        L_other = w.W if axis == 0 else w.H
        travel = w.T - 1
        lo = rmax + (travel if sign < 0 else 0)
        hi = L_move - rmax - (travel if sign > 0 else 0)
        if hi < lo:  # grid too short for the full path: start centred
            lo = hi = L_move / 2.0
        u = float(torch.rand((1,), generator=g))
        v = float(torch.rand((1,), generator=g))
        start = lo + u * (hi - lo)
        other = rmax + v * max(0.0, L_other - 2 * rmax)
        cs = []
        for t in range(w.T):
            m = start + sign * t
            cs.append((m, other) if axis == 0 else (other, m))
        lay.centers.append(cs)
        lay.radii.append(rad_t)
    if w.static_frac > 0:
        ZT, ZH, ZW = w.T // ZONE, w.H // ZONE, w.W // ZONE
        free = []
        for zt in range(ZT):
            for zh in range(ZH):
                for zw in range(ZW):
                    touched = False
                    for cs, rs in zip(lay.centers, lay.radii):
                        for t in range(zt * ZONE, zt * ZONE + ZONE):
                            cy, cx = cs[t]
                            rr = rs[t]
                            # distance from the centre to the zone's box
                            dy = max(zh * ZONE - cy, 0.0, cy - (zh * ZONE + ZONE - 1))
                            dx = max(zw * ZONE - cx, 0.0, cx - (zw * ZONE + ZONE - 1))
                            if dy * dy + dx * dx <= rr * rr:
                                touched = True
                                break
                        if touched:
                            break
                    if not touched:
                        free.append((zt, zh, zw))
        want = min(len(free), int(round(w.static_frac * ZT * ZH * ZW)))
        order = torch.randperm(len(free), generator=g).tolist()
        lay.static_zones = sorted(free[i] for i in order[:want])
    return lay


def _disc_masks(w: Workload, lay: Layout, device):
    """[regions, T, H, W] boolean discs and [regions, T, H, W] Gaussian blobs."""
    ys = torch.arange(w.H, device=device, dtype=torch.float32).view(1, w.H, 1)
    xs = torch.arange(w.W, device=device, dtype=torch.float32).view(1, 1, w.W)
    discs, blobs = [], []
    for cs, rs in zip(lay.centers, lay.radii):
        cy = torch.tensor([c[0] for c in cs], device=device, dtype=torch.float32).view(w.T, 1, 1)
        cx = torch.tensor([c[1] for c in cs], device=device, dtype=torch.float32).view(w.T, 1, 1)
        rr = torch.tensor(rs, device=device, dtype=torch.float32).view(w.T, 1, 1)
        d2 = (ys - cy) ** 2 + (xs - cx) ** 2
        discs.append(d2 <= rr * rr)
        blobs.append(torch.exp(-d2 / (2.0 * rr * rr)))
    return discs, blobs


def make_inputs(w: Workload | str, device="cpu", seed: int = 0, with_grad: bool | None = None):
    """Draw Q, K, V, a (and dO) for workload `w` on `device`.

    Returns a dict with bf16 tensors Q, K, V (and dO), fp32 `a`, and
    `layout` (region paths and static zones) for reporting.
    """
    if isinstance(w, str):
        w = WORKLOADS[w]
    with_grad = w.backward if with_grad is None else with_grad
    device = torch.device(device)
    T, H, W, h, D = w.T, w.H, w.W, w.heads, w.head_dim
    N = T * H * W
    C = h * D
    out = {"workload": w}

    if w.kind == "tiny":
        q = torch.randn((N, h, D), generator=_gen(device, seed, _ID_N1), device=device)
        k = torch.randn((N, h, D), generator=_gen(device, seed, _ID_N2), device=device)
        v = torch.randn((N, h, D), generator=_gen(device, seed, _ID_VBG), device=device)
        v5 = v.view(T, H, W, h, D)
        # zone (zT=0, zH=0, zW=1): add 3*sin(2*pi*y_local/8) on every channel
        y = torch.arange(8, device=device, dtype=torch.float32)
        wave = 3.0 * torch.sin(2.0 * math.pi * y / 8.0)
        v5[0:8, 0:8, 8:16] += wave.view(1, 8, 1, 1, 1)
        an = torch.randn((N,), generator=_gen(device, seed, _ID_ANOISE), device=device).abs() * 0.1
        ys = torch.arange(H, device=device, dtype=torch.float32).view(H, 1)
        xs = torch.arange(W, device=device, dtype=torch.float32).view(1, W)
        # blob of peak 1, sigma 2 tokens, centred in zone (zT=0, zH=1, zW=0)
        blob = torch.exp(-((ys - 11.5) ** 2 + (xs - 3.5) ** 2) / (2.0 * 2.0 ** 2))
        a = an.view(T, H, W) + blob.view(1, H, W)
        out.update(Q=q.to(torch.bfloat16), K=k.to(torch.bfloat16), V=v.to(torch.bfloat16),
                   a=a.reshape(N).contiguous().float(), layout=Layout())
        if with_grad:
            out["dO"] = torch.randn((N, h, D), generator=_gen(device, seed, _ID_DO),
                                    device=device).to(torch.bfloat16)
        return out

    lay = _region_layout(w, device, seed)
    discs, blobs = _disc_masks(w, lay, device)

    # V: low-pass background (std 0.2) + white N(0, 1.5^2) inside moving discs
    V = _lowpass_noise((T, H, W), C, device, seed, _ID_VBG, 0.2)
    for zt, zh, zw in lay.static_zones:
        t0, y0, x0 = zt * ZONE, zh * ZONE, zw * ZONE
        V[t0 + 1:t0 + ZONE, y0:y0 + ZONE, x0:x0 + ZONE] = V[t0:t0 + 1, y0:y0 + ZONE, x0:x0 + ZONE]
    if discs:
        any_disc = torch.zeros((T, H, W), dtype=torch.bool, device=device)
        for dsk in discs:
            any_disc |= dsk
        idx = any_disc.reshape(-1).nonzero().squeeze(1)
        Vf = V.view(N, C)
        for c0 in range(0, C, _CHUNK):
            c1 = min(C, c0 + _CHUNK)
            z = torch.randn((idx.numel(), c1 - c0), generator=_gen(device, seed, _ID_VREG, c0 // _CHUNK),
                            device=device)
            Vf[idx, c0:c1] += 1.5 * z
    out["V"] = V.view(N, h, D).to(torch.bfloat16)
    del V

    # per-zone query sharpness
    sq = torch.full((T, H, W), w.s_q, device=device)
    for zt, zh, zw in lay.static_zones:
        sq[zt * ZONE:(zt + 1) * ZONE, zh * ZONE:(zh + 1) * ZONE, zw * ZONE:(zw + 1) * ZONE] = w.s_q_static
    sq = sq.reshape(N, 1)

    F = _lowpass_noise((T, H, W), C, device, seed, _ID_F, 1.0).view(N, C)
    Q = torch.empty((N, C), dtype=torch.bfloat16, device=device)
    K = torch.empty((N, C), dtype=torch.bfloat16, device=device)
    for c0 in range(0, C, _CHUNK):
        c1 = min(C, c0 + _CHUNK)
        n1 = torch.randn((N, c1 - c0), generator=_gen(device, seed, _ID_N1, c0 // _CHUNK), device=device)
        Q[:, c0:c1] = (sq * (F[:, c0:c1] + 0.5 * n1)).to(torch.bfloat16)
        del n1
        n2 = torch.randn((N, c1 - c0), generator=_gen(device, seed, _ID_N2, c0 // _CHUNK), device=device)
        K[:, c0:c1] = (F[:, c0:c1] + 0.5 * n2).to(torch.bfloat16)
        del n2
    del F
    out["Q"] = Q.view(N, h, D)
    out["K"] = K.view(N, h, D)

    sig_a = 0.05
    a = torch.randn((N,), generator=_gen(device, seed, _ID_ANOISE), device=device).abs() * sig_a
    a = a.view(T, H, W)
    for r in range(min(w.a_regions, len(blobs))):
        a = a + blobs[r]
    out["a"] = a.reshape(N).contiguous().float()
    out["layout"] = lay
    if with_grad:
        out["dO"] = torch.randn((N, h, D), generator=_gen(device, seed, _ID_DO),
                                device=device).to(torch.bfloat16)
    return out


def make_bridge_output(a: torch.Tensor, width: int, seed: int = 0) -> torch.Tensor:
    """A stand-in for a layer's audio-to-video bridge output h_hat, bf16
    [N, width] on a's device: row n is (a[n] / sqrt(width)) * z_n with z_n
    i.i.d. N(0, 1), so its length is a[n] up to chi-distribution spread
    (relative ~ 1/sqrt(2 width)).  The norms of its rows carry the A2V map
    of the workload; nothing here computes them."""
    N = a.numel()
    out = torch.empty((N, width), dtype=torch.bfloat16, device=a.device)
    scale = (a.float() / math.sqrt(width)).view(N, 1)
    for c0 in range(0, width, _CHUNK):
        c1 = min(width, c0 + _CHUNK)
        z = torch.randn((N, c1 - c0), generator=_gen(a.device, seed, _ID_HHAT, c0 // _CHUNK), device=a.device)
        out[:, c0:c1] = (scale * z).to(torch.bfloat16)
        del z
    return out


def make_projection(V: torch.Tensor, seed: int = 0):
    """Inputs of a value projection whose output has the workload's value
    structure: X = the workload's V viewed as token features [N, heads*D]
    (bf16), and Wv [heads*D, heads*D] (bf16) block-diagonal with one seeded
    random orthogonal D x D block per head (the Q factor of a Gaussian
    matrix).  An orthogonal mix of a head's channels keeps every sum of
    squares over its channels, so X Wv^T carries the workload's zone
    structure; the projection still multiplies the full dense matrix."""
    N, h, D = V.shape
    X = V.reshape(N, h * D).contiguous()
    W = torch.zeros((h * D, h * D), dtype=torch.float32)
    for k in range(h):
        g = torch.randn((D, D), generator=_gen("cpu", seed, _ID_WV, k), dtype=torch.float64)
        q, r = torch.linalg.qr(g)
        q = q * torch.sign(torch.diagonal(r)).view(1, D)
        W[k * D:(k + 1) * D, k * D:(k + 1) * D] = q.float()
    return X, W.to(torch.bfloat16).to(V.device)
