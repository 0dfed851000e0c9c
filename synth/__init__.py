"""Seeded synthetic inputs shaped like video-DiT self-attention.

This module only makes data.  It holds none of the attention or mask arithmetic:
both the fp64 oracle and the CUDA path receive the tensors built here as plain
inputs, so neither one's result can leak into the other's.

Token layout.  A latent video of T frames x Hl x Wl tokens is flattened the way
the NABLA paper describes its token reordering ("∇NABLA: Neighborhood Adaptive
Block-Level Attention", §3.1.1 and Figure 3): inside each frame the tokens of
one P x P spatial patch are contiguous, patches follow each other in row-major
patch order, and frames keep their time order.  Patches cut by the frame edge
keep only their valid tokens (row-major inside the patch).  The flat sequence is
then cut into 64-token blocks; the last block may be partial.

Block coordinates.  Each 64-token block is tagged with the tile coordinate
(t, y // P, x // P) of its first token.  These coordinates are an input of the
sliding-tile (STA) neighbourhood mask and of the locality term below.

Values.  For every token of block b (per sample and head):

    x = eps + m_b + l_b

* eps ~ N(0, 1), drawn independently for Q, K, V and the upstream gradient dO;
* m_b ~ N(0, sigma^2 I_D), one vector per block, shared by Q, K, V and dO of
  that block (this creates the block structure the mask builder detects);
* l_b (optional locality term) = sum of anchors a_c over the tile coordinates c
  with ||c - coord_b||_inf <= 2 (truncated at the grid edge), divided by the
  square root of the number of such c; anchors a_c ~ N(0, sigma^2 I_D), one per
  tile coordinate.  Neighbouring blocks therefore share part of their mean.

sigma defaults to 0.5: "N(0, 0.5)" in the workload description is read as
mean 0, standard deviation 0.5.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

BLOCK = 64


def num_blocks(S: int, block: int = BLOCK) -> int:
    return -(-S // block)


def fractal_token_coords(T: int, Hl: int, Wl: int, P: int = 8) -> np.ndarray:
    """(t, y, x) of every token of the flattened sequence, in sequence order."""
    out = []
    ny, nx = -(-Hl // P), -(-Wl // P)
    frame = []
    for py in range(ny):
        for px in range(nx):
            ys = np.arange(py * P, min(py * P + P, Hl))
            xs = np.arange(px * P, min(px * P + P, Wl))
            yy, xx = np.meshgrid(ys, xs, indexing="ij")
            frame.append(np.stack([yy.ravel(), xx.ravel()], 1))
    frame = np.concatenate(frame, 0)
    for t in range(T):
        out.append(np.concatenate([np.full((frame.shape[0], 1), t), frame], 1))
    return np.concatenate(out, 0).astype(np.int64)


def block_coords(T: int, Hl: int, Wl: int, P: int = 8, block: int = BLOCK) -> np.ndarray:
    """int32 [nb, 3] tile coordinate (t, y // P, x // P) of each block's first token."""
    tok = fractal_token_coords(T, Hl, Wl, P)
    first = tok[::block]
    return np.stack([first[:, 0], first[:, 1] // P, first[:, 2] // P], 1).astype(np.int32)


def _box_sum(x: torch.Tensor, dim: int, r: int) -> torch.Tensor:
    """Sum over a window of radius r along dim, truncated at both ends."""
    n = x.shape[dim]
    zero = torch.zeros_like(x.narrow(dim, 0, 1))
    cs = torch.cat([zero, torch.cumsum(x, dim)], dim)
    hi = torch.clamp(torch.arange(n) + r + 1, max=n)
    lo = torch.clamp(torch.arange(n) - r, min=0)
    return cs.index_select(dim, hi) - cs.index_select(dim, lo)


@dataclass
class Workload:
    """One synthetic workload: shapes, dtype, thresholds, STA window, seed."""
    name: str
    B: int
    H: int
    T: int
    Hl: int
    Wl: int
    D: int
    dtype: str                 # "bf16" or "fp32"
    thresholds: list
    seed: int
    locality: bool
    sta_window: tuple | None = None   # (wT, wH, wW) in tiles
    with_grad: bool = False
    sigma: float = 0.5
    P: int = 8

    @property
    def S(self) -> int:
        return self.T * self.Hl * self.Wl

    @property
    def nb(self) -> int:
        return num_blocks(self.S)

    def scaled(self, **kw) -> "Workload":
        d = dict(self.__dict__)
        d.update(kw)
        return Workload(**d)


# The workloads: a tiny fp32 case, 480p- and 720p-shaped forwards, a
# pretraining-shaped forward+backward, a threshold sweep at the 720p shape, and
# the configurations of Table 1 (§4.1): the 720p latent with every frame padded
# from 45 to 48 token rows, so that the 21 x 6 x 10 tiles of 8 x 8 tokens are
# exactly the 64-token blocks (80,640 tokens; the padding rows carry synthetic
# values like the rest); and the 720p sweep again with block means and locality
# anchors of standard deviation 0.6 instead of 0.5 (same seed, so the same noise
# with the block-structure terms scaled by 1.2): sparser masks, about 92 % and
# 82 % sparsity at thr 0.7 and 0.8, the range of Table 1's NABLA rows.
WORKLOADS = {
    1: Workload("tiny_fp32", 1, 2, 4, 32, 32, 64, "fp32", [0.9], 0, False),
    2: Workload("fwd_480p", 1, 40, 21, 30, 52, 128, "bf16", [0.7, 0.8, 0.9], 2, True),
    3: Workload("fwd_720p", 1, 40, 21, 45, 80, 128, "bf16", [0.8], 3, True, sta_window=(3, 3, 3)),
    4: Workload("train_512", 2, 16, 16, 32, 32, 128, "bf16", [0.8], 4, False, with_grad=True),
    5: Workload("sweep_720p", 1, 40, 21, 45, 80, 128, "bf16",
                [0.5, 0.7, 0.8, 0.9, 0.95, 1.0], 3, True),
    6: Workload("table1_720p_padded", 1, 40, 21, 48, 80, 128, "bf16", [0.7, 0.4, 0.5, 0.2], 6, True),
    7: Workload("sweep_720p_sigma06", 1, 40, 21, 45, 80, 128, "bf16",
                [0.5, 0.7, 0.8, 0.9, 0.95, 1.0], 3, True, sigma=0.6),
}

# Table 1 (§4.1): method name, NABLA threshold (None: no NABLA selection) and
# STA window in tokens (frames, rows, columns; None: no STA).  A window of w
# tokens spans w / 8 tiles of 8 x 8 tokens; the frame count is already in tiles.
TABLE1 = [
    ("Baseline", 1.0, None),
    ("STA(18,40,40)", None, (18, 40, 40)),
    ("NABLA(0.7)", 0.7, None),
    ("NABLA(0.5)+STA(11,40,40)", 0.5, (11, 40, 40)),
    ("STA(18,24,24)", None, (18, 24, 24)),
    ("NABLA(0.4)", 0.4, None),
    ("NABLA(0.2)+STA(11,24,24)", 0.2, (11, 24, 24)),
]


def sta_tiles(window_tokens: tuple, P: int = 8) -> tuple:
    """(frames, rows, columns) in tokens -> the window in tiles."""
    wt, wh, ww = window_tokens
    return (wt, wh // P, ww // P)


def make_inputs(w: Workload, heads: list | None = None) -> dict:
    """Build Q, K, V (and dO) as CPU torch tensors [B, H, S, D] in w.dtype.

    heads, if given, restricts generation to those head indices (same values as
    the full generation for those heads), which lets tests sample large
    workloads cheaply.
    """
    S, nb, D = w.S, w.nb, w.D
    g = torch.Generator().manual_seed(w.seed)
    coords = block_coords(w.T, w.Hl, w.Wl, w.P)
    tok_block = torch.arange(S) // BLOCK
    m = torch.randn(w.B, w.H, nb, D, generator=g) * w.sigma
    if w.locality:
        ny, nx = -(-w.Hl // w.P), -(-w.Wl // w.P)
        a = torch.randn(w.B, w.H, w.T, ny, nx, D, generator=g) * w.sigma
        ones = torch.ones(w.T, ny, nx)
        box, cnt = a, ones
        for dim in range(3):
            box = _box_sum(box, dim + 2, 2)
            cnt = _box_sum(cnt, dim, 2)
        c = torch.from_numpy(coords.astype(np.int64))
        loc = box[:, :, c[:, 0], c[:, 1], c[:, 2], :] / torch.sqrt(cnt[c[:, 0], c[:, 1], c[:, 2]])[None, None, :, None]
        m = m + loc
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    names = ["q", "k", "v"] + (["do"] if w.with_grad else [])
    hsel = list(range(w.H)) if heads is None else list(heads)
    out = {n: torch.empty(w.B, len(hsel), S, D, dtype=dt) for n in names}
    hpos = {h: i for i, h in enumerate(hsel)}
    for b in range(w.B):
        for h in hsel:
            # one generator per (sample, head) so that any subset of heads can
            # be regenerated alone with identical values
            gh = torch.Generator().manual_seed(w.seed * 1_000_003 + b * 10_007 + h)
            mean_tok = m[b, h][tok_block]
            for n in names:
                eps = torch.randn(S, D, generator=gh)
                out[n][b, hpos[h]] = (eps + mean_tok).to(dt)
    out["coords"] = torch.from_numpy(coords)
    out["S"], out["nb"], out["heads"] = S, nb, hsel
    return out


def make_random_qkv(B: int, H: int, S: int, D: int, dtype: str, seed: int,
                    sigma: float = 0.5, with_grad: bool = False) -> dict:
    """Flat variant for arbitrary S (ragged tails, edge cases): block means
    without the locality term, blocks taken in sequence order."""
    nb = num_blocks(S)
    g = torch.Generator().manual_seed(seed)
    m = torch.randn(B, H, nb, D, generator=g) * sigma
    mean_tok = m[:, :, torch.arange(S) // BLOCK, :]
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    names = ["q", "k", "v"] + (["do"] if with_grad else [])
    out = {n: (torch.randn(B, H, S, D, generator=g) + mean_tok).to(dt) for n in names}
    out["S"], out["nb"] = S, nb
    return out


def line_coords(nb: int, T: int = 1, ny: int = 1) -> torch.Tensor:
    """Simple block coordinates for flat inputs: blocks laid out on a
    T x ny x (nb / (T ny)) grid in sequence order."""
    nx = -(-nb // (T * ny))
    i = np.arange(nb)
    c = np.stack([i // (ny * nx), (i // nx) % ny, i % nx], 1).astype(np.int32)
    return torch.from_numpy(c)


def make_projection_inputs(B: int, S: int, C: int, H: int, D: int, seed: int,
                           sigma: float = 0.5, device: str = "cpu") -> dict:
    """Hidden states and weights for the Eq. 1 projection Q = X W_Q (and K, V).

    X [B, S, C] bf16: eps ~ N(0, 1) per token plus one mean vector per 64-token
    block ~ N(0, sigma^2 I_C), so the projected Q and K carry block structure
    for the mask builder to find.  Wt [3, H D, C] bf16: the transposed W_Q,
    W_K, W_V (one row per output feature), entries ~ N(0, 1 / C), which keeps
    the projected values at unit scale.  device="cuda" draws the same kind of
    values on the GPU (a different stream of random numbers) for sizes the
    host would take long to fill."""
    g = torch.Generator(device=device).manual_seed(seed)
    nb = num_blocks(S)
    m = torch.randn(B, nb, C, generator=g, device=device) * sigma
    tok_block = torch.arange(S, device=device) // BLOCK
    X = torch.empty(B, S, C, dtype=torch.bfloat16, device=device)
    for b in range(B):
        X[b] = (torch.randn(S, C, generator=g, device=device) + m[b][tok_block]).to(torch.bfloat16)
    Wt = (torch.randn(3, H * D, C, generator=g, device=device) / math.sqrt(C)).to(torch.bfloat16)
    return {"x": X, "wt": Wt, "S": S, "nb": nb}
