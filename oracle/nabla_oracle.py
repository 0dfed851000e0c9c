"""fp64 CPU oracle for the NABLA hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, links or runs
this module; only the tests, the package smoke check and the benchmark's CPU
baseline leg use it.  It shares no code with the CUDA library: it is a slow,
plain restatement of what the method computes, so that the kernels can be
compared against it element by element.

Sources (the paper "∇NABLA: Neighborhood Adaptive Block-Level Attention",
arXiv 2507.13546v1):

* Algorithm 1 "NABLA Sparse Mask Generation" (§3.1.2): block average pooling
  of Q and K, the reduced attention map softmax(Qa Ka^T / sqrt(D)), row-wise
  ascending sort, cumulative sum, binarisation cvals >= 1 - thr and the
  restoration of the original order.
* §3.1.3: the final mask is the union of the NABLA mask and the STA mask.
* §2.2, Eq. 4: masked attention softmax(QK^T / sqrt(D) + M) V with
  M in {-inf, 0}; §2.1, Eq. 2-3: dense attention.
* §2.2: the STA window is a fixed 3D window of tiles centred on the query tile.
* §3.1.1, Figure 3: fractal flattening of the token sequence (P x P patches
  made contiguous, temporal order kept) and its inverse.
* the pith.science review of v2 (Appendix C): the fixed-budget Top-k selection the CDF
  rule is compared with, and the per-block fidelity check of the pooling
  proxy (token-level attention mass inside the retained blocks).

Readings where the paper is silent (each with its reason):

* sort direction: ascending, so that cvals >= 1 - thr keeps the largest
  entries and thr = 1 keeps every block;
* ties in the sort: stable (lower block index first);
* 1 - thr is formed in fp64 from the float32 value of thr;
* a partial last block (S not a multiple of 64) is averaged over its valid
  tokens, and its missing key positions are excluded from attention;
* STA window: |dt| <= wT // 2, |dy| <= wH // 2, |dx| <= wW // 2 in tile units,
  truncated at the grid edge (no shifting of the window);
* the mask is a constant of the backward pass (no gradient through pooling);
* edge patches of a frame whose sides are not multiples of P keep their valid
  tokens, row-major.

Every function here is pinned by the CPU tests in tests/test_oracle_*.py
against values the paper fixes (Table 1 STA sparsities), closed forms,
library routines on special cases and brute force on tiny inputs.
"""
from __future__ import annotations

import numpy as np

BLOCK = 64


def num_blocks(S: int, N: int = BLOCK) -> int:
    return -(-S // N)


def as_f64(x) -> np.ndarray:
    """Exact fp64 copy of a numpy array or torch tensor (bf16 and fp32 values
    are exactly representable in fp64)."""
    if hasattr(x, "detach"):
        x = x.detach().float().cpu().numpy()
    return np.asarray(x, dtype=np.float64)


# ---------------------------------------------------------------- Algorithm 1

def block_pool(X: np.ndarray, N: int = BLOCK) -> np.ndarray:
    """Block averaging of Algorithm 1: view the S tokens as S/N blocks of N
    tokens and take the mean over each block.  X: [..., S, D] -> [..., nb, D].
    A partial last block is averaged over its valid tokens only."""
    S = X.shape[-2]
    nb = num_blocks(S, N)
    out = np.empty(X.shape[:-2] + (nb, X.shape[-1]), dtype=np.float64)
    for i in range(nb):
        lo, hi = i * N, min(i * N + N, S)
        out[..., i, :] = X[..., lo:hi, :].sum(axis=-2) / (hi - lo)
    return out


def reduced_scores(Qa: np.ndarray, Ka: np.ndarray) -> np.ndarray:
    """Logits of the reduced attention map of Algorithm 1: Qa Ka^T / sqrt(D),
    with D the head dimension.  [..., nb, D] x [..., nb, D] -> [..., nb, nb]."""
    D = Qa.shape[-1]
    return np.matmul(Qa, np.swapaxes(Ka, -1, -2)) / np.sqrt(D)


def row_softmax(L: np.ndarray) -> np.ndarray:
    """Softmax along the last dimension (max-subtracted)."""
    z = L - L.max(axis=-1, keepdims=True)
    e = np.exp(z)
    return e / e.sum(axis=-1, keepdims=True)


def cdf_binarize(A: np.ndarray, thr: float):
    """Binarisation via the CDF (Algorithm 1): sort every row ascending, take
    the cumulative sum, keep the sorted positions whose cumulative value is
    >= 1 - thr, and put the decisions back in the original column order.

    Returns (M, C): the boolean mask and, at each original position, the
    cumulative mass its sorted position reached (used for the tolerance band
    around the threshold)."""
    one_minus = 1.0 - float(np.float32(thr))
    order = np.argsort(A, axis=-1, kind="stable")
    vals = np.take_along_axis(A, order, axis=-1)
    cvals = np.cumsum(vals, axis=-1)
    keep_sorted = cvals >= one_minus
    M = np.zeros(A.shape, dtype=bool)
    C = np.zeros(A.shape, dtype=np.float64)
    np.put_along_axis(M, order, keep_sorted, axis=-1)
    np.put_along_axis(C, order, cvals, axis=-1)
    return M, C


def topk_binarize(A: np.ndarray, k: int) -> np.ndarray:
    """Fixed-budget comparator of the CDF rule (the Top-k selection the paper's
    Appendix C compares against, per the pith.science review): every row keeps its k
    largest entries.  Reading: k is clipped to [1, nb]; among equal values the
    order is that of the stable ascending sort used by cdf_binarize (the
    higher column index ranks higher), so exactly k entries are kept."""
    nb = A.shape[-1]
    k = min(max(int(k), 1), nb)
    order = np.argsort(A, axis=-1, kind="stable")
    keep_sorted = np.zeros(A.shape, dtype=bool)
    keep_sorted[..., nb - k:] = True
    M = np.zeros(A.shape, dtype=bool)
    np.put_along_axis(M, order, keep_sorted, axis=-1)
    return M


def topk_mask(Q, K, k: int, coords=None, window=None, N: int = BLOCK):
    """Top-k counterpart of nabla_mask: the same pooled scores and softmax
    (the order is that of the logits), k blocks per row, optional STA union."""
    Qa = block_pool(as_f64(Q), N)
    Ka = block_pool(as_f64(K), N)
    P = row_softmax(reduced_scores(Qa, Ka))
    M = topk_binarize(P, k)
    if window is not None:
        M = M | sta_mask(coords, window)[None, None]
    return M, P


def sta_mask(coords: np.ndarray, window) -> np.ndarray:
    """Sliding-tile mask on block tile coordinates (§2.2, §3.1.3): block j is
    visible from block i iff every tile-coordinate difference lies inside the
    window centred on i.  coords: int [nb, 3] (t, y, x); window (wT, wH, wW)."""
    c = np.asarray(coords, dtype=np.int64)
    r = np.array([w // 2 for w in window], dtype=np.int64)
    d = np.abs(c[:, None, :] - c[None, :, :])
    return np.all(d <= r[None, None, :], axis=-1)


def sta_grid_coords(T: int, Hy: int, Wx: int) -> np.ndarray:
    """All tile coordinates of a T x Hy x Wx tile grid, time-major."""
    t, y, x = np.meshgrid(np.arange(T), np.arange(Hy), np.arange(Wx), indexing="ij")
    return np.stack([t.ravel(), y.ravel(), x.ravel()], 1)


def nabla_mask(Q, K, thr: float, coords=None, window=None, N: int = BLOCK):
    """Full mask builder for Q, K [B, H, S, D]: returns (M, C, P) with
    M bool [B, H, nb, nb] = M_nabla OR M_STA (STA only if window is given),
    C the cumulative mass of each entry in its sorted row and P the reduced
    attention map."""
    Qa = block_pool(as_f64(Q), N)
    Ka = block_pool(as_f64(K), N)
    P = row_softmax(reduced_scores(Qa, Ka))
    M, C = cdf_binarize(P, thr)
    if window is not None:
        M = M | sta_mask(coords, window)[None, None]
    return M, C, P


def band_mask(C: np.ndarray, thr: float, band: float = 1e-5) -> np.ndarray:
    """Entries whose cumulative mass lies within `band` of 1 - thr; there the
    decision depends on rounding and a compared implementation may differ."""
    return np.abs(C - (1.0 - float(np.float32(thr)))) <= band


# --------------------------------------------------- mask -> index structures

def mask_to_bits(M: np.ndarray) -> np.ndarray:
    """Bool [..., nb, nb] -> uint32 [..., nb, ceil(nb/32)], bit (j % 32) of
    word j // 32 set iff block j is kept."""
    nb = M.shape[-1]
    W = -(-nb // 32)
    pad = np.zeros(M.shape[:-1] + (W * 32,), dtype=np.uint64)
    pad[..., :nb] = M
    pad = pad.reshape(M.shape[:-1] + (W, 32))
    w = (pad << np.arange(32, dtype=np.uint64)).sum(axis=-1)
    return w.astype(np.uint32)


def bits_to_mask(bits: np.ndarray, nb: int) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint64)[..., :, None] >> np.arange(32, dtype=np.uint64)
    return (b & 1).astype(bool).reshape(bits.shape[:-1] + (-1,))[..., :nb]


# ----------------------------------------------------------------- projection

def qkv_project(X, Wt, H: int, D: int):
    """Eq. 1 (§2.1): Q = X W_Q, K = X W_K, V = X W_V, for every sample.

    X [B, S, C] holds the tokens' hidden states.  The multi-head reading: W_Q
    is C x (H D), and head h of Q takes its columns h D .. h D + D - 1.  Wt
    [3, H D, C] holds the transposes W_Q^T, W_K^T, W_V^T (one row per output
    feature, n = h D + d), the way a linear layer stores its weight.
    Returns Q, K, V as fp64 [B, H, S, D]."""
    X, Wt = as_f64(X), as_f64(Wt)
    B, S, C = X.shape
    if Wt.shape != (3, H * D, C):
        raise ValueError(f"Wt must be [3, {H * D}, {C}], got {list(Wt.shape)}")
    out = []
    for m in range(3):
        Y = np.matmul(X, Wt[m].T)                              # [B, S, H D] = X W
        out.append(Y.reshape(B, S, H, D).transpose(0, 2, 1, 3))  # head h: columns h D + d
    return tuple(np.ascontiguousarray(y) for y in out)


# ------------------------------------------------------------------ attention

def _allowed_keys(M_row: np.ndarray, S: int, N: int = BLOCK) -> np.ndarray:
    """Token indices of the keys inside the kept blocks of one mask row."""
    blocks = np.nonzero(M_row)[0]
    if blocks.size == 0:
        return np.zeros(0, dtype=np.int64)
    return np.concatenate([np.arange(j * N, min(j * N + N, S)) for j in blocks])


def masked_attention(Q, K, V, M: np.ndarray, N: int = BLOCK):
    """Eq. 4 with a block mask: for every query token, softmax over the keys of
    the kept blocks of its block row (all other keys get -inf), then the
    weighted sum of values.  Q, K, V [B, H, S, D]; M bool [B, H, nb, nb].
    Returns (O [B, H, S, D], LSE [B, H, S]) in fp64, LSE = log sum exp of the
    scaled logits over the allowed keys."""
    Q, K, V = as_f64(Q), as_f64(K), as_f64(V)
    B, H, S, D = Q.shape
    nb = num_blocks(S, N)
    O = np.zeros_like(Q)
    LSE = np.full((B, H, S), -np.inf)
    for b in range(B):
        for h in range(H):
            for i in range(nb):
                rows = slice(i * N, min(i * N + N, S))
                keys = _allowed_keys(M[b, h, i], S, N)
                if keys.size == 0:
                    continue
                logit = Q[b, h, rows] @ K[b, h, keys].T / np.sqrt(D)
                mx = logit.max(axis=-1, keepdims=True)
                e = np.exp(logit - mx)
                s = e.sum(axis=-1, keepdims=True)
                O[b, h, rows] = (e / s) @ V[b, h, keys]
                LSE[b, h, rows] = (mx + np.log(s))[:, 0]
    return O, LSE


def masked_attention_rows(Q, K, V, M: np.ndarray, b: int, h: int, rows, N: int = BLOCK):
    """Same as masked_attention for a few query tokens of one (b, h); returns
    (O [len(rows), D], LSE [len(rows)])."""
    Qh, Kh, Vh = as_f64(Q[b, h]), as_f64(K[b, h]), as_f64(V[b, h])
    S, D = Qh.shape
    rows = np.asarray(rows)
    O = np.zeros((rows.size, D))
    LSE = np.full(rows.size, -np.inf)
    for n, s in enumerate(rows):
        keys = _allowed_keys(M[b, h, s // N], S, N)
        if keys.size == 0:
            continue
        logit = Kh[keys] @ Qh[s] / np.sqrt(D)
        mx = logit.max()
        e = np.exp(logit - mx)
        O[n] = e @ Vh[keys] / e.sum()
        LSE[n] = mx + np.log(e.sum())
    return O, LSE


def round_bf16(x: np.ndarray) -> np.ndarray:
    """x rounded to fp32, then to bfloat16 (the top 16 bits of the fp32
    pattern, rounding to nearest with ties to even), returned as fp64."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def masked_attention_bwd(Q, K, V, dO, M: np.ndarray, N: int = BLOCK, ds_bound: bool = False,
                         ds_format: str | None = None):
    """Gradients of masked_attention with the mask held constant: with
    P = softmax(Q K_sel^T / sqrt(D)) per query block,
      dV_sel += P^T dO,  dP = dO V_sel^T,  dS = P * (dP - rowsum(P * dP)),
      dQ = dS K_sel / sqrt(D),  dK_sel += dS^T Q / sqrt(D).
    rowsum(P * dP) equals rowsum(dO * O).
    Returns (dQ, dK, dV) fp64 [B, H, S, D].  ds_bound=True also returns
    (bQ, bK): every gradient entry's sum of term magnitudes through dS,
    bQ = |dS| |K_sel| / sqrt(D) and bK_sel += |dS|^T |Q| / sqrt(D), the scale
    of the error that rounding dS before these products can cause.
    ds_format="bf16" rounds dS to bfloat16 (nearest even) before the dQ and
    dK products, the operand a bf16 tensor-core backward multiplies; the
    default is the exact (textbook) gradient."""
    Q, K, V, dO = as_f64(Q), as_f64(K), as_f64(V), as_f64(dO)
    B, H, S, D = Q.shape
    nb = num_blocks(S, N)
    dQ, dK, dV = np.zeros_like(Q), np.zeros_like(K), np.zeros_like(V)
    bQ, bK = np.zeros_like(Q), np.zeros_like(K)
    scale = 1.0 / np.sqrt(D)
    for b in range(B):
        for h in range(H):
            for i in range(nb):
                rows = slice(i * N, min(i * N + N, S))
                keys = _allowed_keys(M[b, h, i], S, N)
                if keys.size == 0:
                    continue
                logit = Q[b, h, rows] @ K[b, h, keys].T * scale
                e = np.exp(logit - logit.max(axis=-1, keepdims=True))
                P = e / e.sum(axis=-1, keepdims=True)
                g = dO[b, h, rows]
                dV[b, h, keys] += P.T @ g
                dP = g @ V[b, h, keys].T
                delta = (P * dP).sum(axis=-1, keepdims=True)
                dS = P * (dP - delta)
                dSm = round_bf16(dS) if ds_format == "bf16" else dS
                dQ[b, h, rows] = dSm @ K[b, h, keys] * scale
                dK[b, h, keys] += dSm.T @ Q[b, h, rows] * scale
                if ds_bound:
                    bQ[b, h, rows] = np.abs(dS) @ np.abs(K[b, h, keys]) * scale
                    bK[b, h, keys] += np.abs(dS).T @ np.abs(Q[b, h, rows]) * scale
    if ds_bound:
        return dQ, dK, dV, bQ, bK
    return dQ, dK, dV


# ------------------------------------------------- block fidelity of a mask

def block_mass(Q, K, N: int = BLOCK) -> np.ndarray:
    """True token-level attention mass per block: with the dense attention
    distribution p_s = softmax(q_s K^T / sqrt(D)) of every query token s over
    all S keys (§2.1, Eq. 2-3), A[i, j] is the mean over the valid query
    tokens s of block i of the mass p_s puts on the keys of block j.  Every row
    of A sums to 1.  This is the per-block fidelity quantity the pith.science review
    asks for ("what fraction of token-level attention mass falls inside the
    retained blocks").  Q, K [B, H, S, D] -> A [B, H, nb, nb]."""
    Q, K = as_f64(Q), as_f64(K)
    B, H, S, D = Q.shape
    nb = num_blocks(S, N)
    A = np.zeros((B, H, nb, nb))
    for b in range(B):
        for h in range(H):
            L = Q[b, h] @ K[b, h].T / np.sqrt(D)
            P = np.exp(L - L.max(-1, keepdims=True))
            P /= P.sum(-1, keepdims=True)
            for i in range(nb):
                rows = P[i * N:min(i * N + N, S)]
                for j in range(nb):
                    A[b, h, i, j] = rows[:, j * N:min(j * N + N, S)].sum(-1).mean()
    return A


def block_mass_rows(Q, K, b: int, h: int, blocks, N: int = BLOCK) -> np.ndarray:
    """Rows `blocks` of block_mass for one (b, h): the same definition on the
    query tokens of the listed blocks only (for full-size spot checks).
    Returns [len(blocks), nb]."""
    q, k = as_f64(Q[b, h]), as_f64(K[b, h])
    S, D = k.shape
    nb = num_blocks(S, N)
    out = np.zeros((len(blocks), nb))
    for r, i in enumerate(blocks):
        L = q[i * N:min(i * N + N, S)] @ k.T / np.sqrt(D)
        P = np.exp(L - L.max(-1, keepdims=True))
        P /= P.sum(-1, keepdims=True)
        for j in range(nb):
            out[r, j] = P[:, j * N:min(j * N + N, S)].sum(-1).mean()
    return out


def mask_recall(A: np.ndarray, M: np.ndarray) -> np.ndarray:
    """Kept token-level mass of each query block under block mask M:
    R[..., i] = sum_j M[..., i, j] A[..., i, j] (1 when the mask keeps all the
    attention mass of the block's queries)."""
    return (A * M).sum(-1)


# ------------------------------------------------- §3.1.1 token reordering

def fractal_order(T: int, Hl: int, Wl: int, P: int = 8) -> np.ndarray:
    """Fractal flattening of §3.1.1 (Figure 3) as a gather index: entry f is
    the raster index t * Hl * Wl + y * Wl + x of the token that lands at
    position f of the reordered sequence.  Frames keep their temporal order;
    inside a frame the P x P patches follow in row-major patch order, each
    patch's tokens contiguous and row-major inside the patch.  Edge patches of
    a frame whose height or width is not a multiple of P hold only their
    valid tokens, still row-major (the reading used throughout)."""
    order = []
    for t in range(T):
        for py in range(0, Hl, P):
            for px in range(0, Wl, P):
                for y in range(py, min(py + P, Hl)):
                    for x in range(px, min(px + P, Wl)):
                        order.append((t * Hl + y) * Wl + x)
    return np.asarray(order, dtype=np.int64)


def block_tile_coords(T: int, Hl: int, Wl: int, P: int = 8, S: int | None = None, N: int = BLOCK) -> np.ndarray:
    """STA tile coordinate of every N-token block of the reordered sequence
    (§3.1.1 token order; the window of §2.2 is centred on the query tile): the
    (t, y // P, x // P) of the block's first token, read off the gather index
    of fractal_order.  S (default T * Hl * Wl) sets the number of blocks,
    ceil(S / N); every block must start at a latent token.  int64 [nb, 3]."""
    order = fractal_order(T, Hl, Wl, P)
    S = len(order) if S is None else S
    nb = num_blocks(S, N)
    out = np.empty((nb, 3), dtype=np.int64)
    for i in range(nb):
        r = int(order[i * N])            # raster index t * Hl * Wl + y * Wl + x
        t, rem = divmod(r, Hl * Wl)
        y, x = divmod(rem, Wl)
        out[i] = (t, y // P, x // P)
    return out


def fractal_reorder(X, T: int, Hl: int, Wl: int, P: int = 8, inverse: bool = False) -> np.ndarray:
    """Applies the reordering to X [B, S, ...] (S = T * Hl * Wl): the network
    input goes from raster to fractal order; inverse=True is the output-stage
    inverse, fractal back to raster order (§3.1.1)."""
    X = np.asarray(X)
    perm = fractal_order(T, Hl, Wl, P)
    if not inverse:
        return X[:, perm]
    out = np.empty_like(X)
    out[:, perm] = X
    return out


# ------------------------------------------------------------ error metrics

def max_abs(x, ref) -> float:
    x, ref = as_f64(x), as_f64(ref)
    return float(np.max(np.abs(x - ref))) if ref.size else 0.0


def mean_rel(x, ref) -> float:
    """mean |x - ref| / mean |ref| (a ratio of means, robust near zero)."""
    x, ref = as_f64(x), as_f64(ref)
    den = float(np.mean(np.abs(ref)))
    return float(np.mean(np.abs(x - ref))) / den if den > 0 else float(np.mean(np.abs(x)))
