"""GPU parity of the Eq. 1 projection with the block pooling fused into it
("∇NABLA: Neighborhood Adaptive Block-Level Attention", §2.1 Eq. 1 and the
pooling of Algorithm 1, §3.1.2), through the C ABI.

Bars.
* Q, K, V against the fp64 oracle (qkv_project): each element within one
  bf16 ulp of the exact value (2^-8 relative: the kernel rounds its fp32
  accumulation to bf16 once) plus 2^-16 * sum_c |x_c w_c| for the fp32
  accumulation, far below the O(1) error of a wrong index or operand.
* The fused pooling: the mask built from the means the projection leaves in
  the workspace (nabla_build_mask_pooled) equals, bit for bit, the mask that
  nabla_build_mask builds from the stored Q and K, and the oracle's mask of
  those Q and K outside the 1e-5 band."""
import numpy as np
import pytest
import torch

import block_sparse_attention_nabla_b200 as nabla
import synth
from oracle import nabla_oracle as orc
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


def _bound(x, wt, rows=None):
    """sum_c |x_c w_c| of every projected value, per weight: three
    [B, S', H D] fp64 arrays (rows: the token indices to take, else all)."""
    X = np.abs(orc.as_f64(x))
    if rows is not None:
        X = X[:, rows]
    Wt = np.abs(orc.as_f64(wt))
    return [np.matmul(X, Wt[m].T) for m in range(3)]


def _same_mask(a, b, transpose):
    """Two masks equal: bitmask, counts and work list exactly, and every list
    up to its count (entries past the count are not defined)."""
    for name in ("bits", "cnt", "work") + (("cnt_t",) if transpose else ()):
        assert torch.equal(getattr(a, name), getattr(b, name)), name
    for lst, cnt in (("idx", "cnt"),) + ((("idx_t", "cnt_t"),) if transpose else ()):
        n = getattr(a, cnt)
        valid = torch.arange(n.shape[-1], device=n.device) < n[..., None]
        assert torch.equal(getattr(a, lst)[valid], getattr(b, lst)[valid]), lst


def _check_projection(outs, x, wt, H, D, rows=None):
    X = orc.as_f64(x)
    if rows is not None:
        X = X[:, rows]
    ref = orc.qkv_project(X, wt, H, D)
    mags = _bound(x, wt, rows)
    B, S = X.shape[:2]
    for m, name in enumerate("qkv"):
        got = orc.as_f64(outs[m] if rows is None else outs[m][:, :, rows])
        tol = 2.0 ** -8 * np.abs(ref[m]) + 2.0 ** -16 * mags[m].reshape(B, S, H, D).transpose(0, 2, 1, 3)
        err = np.abs(got - ref[m])
        worst = float((err / tol).max())
        assert worst <= 1.0, f"{name}: max error / tolerance = {worst:.3f}"


@pytest.mark.parametrize("B,H,S,D,C", [
    (1, 2, 200, 128, 192),     # ragged token tile and block, 3 K slices
    (2, 3, 130, 64, 72),       # two samples, odd H (a partial feature tile), C not a multiple of 64
    (1, 2, 1000, 128, 256),
    (1, 1, 64, 128, 8),        # the smallest C
    (1, 4, 4096, 64, 320),
])
def test_projection_matches_the_oracle(B, H, S, D, C):
    d = synth.make_projection_inputs(B, S, C, H, D, seed=100 + S + C)
    x, wt = d["x"].cuda(), d["wt"].cuda()
    q, k, v, ws = nabla.qkv_project(x, wt, H, D)
    torch.cuda.synchronize()
    assert nabla.workspace_status(ws) == 0
    _check_projection([q.cpu(), k.cpu(), v.cpu()], d["x"], d["wt"], H, D)


@pytest.mark.parametrize("sta", [False, True])
@pytest.mark.parametrize("B,H,S,D,C,thr", [(1, 2, 4096, 128, 256, 0.8), (2, 3, 1000, 128, 192, 0.9),
                                           (1, 2, 130, 128, 64, 0.5), (1, 5, 3000, 64, 320, 0.7)])
def test_pooled_build_equals_the_build_from_q_and_k(B, H, S, D, C, thr, sta):
    d = synth.make_projection_inputs(B, S, C, H, D, seed=7 + S)
    x, wt = d["x"].cuda(), d["wt"].cuda()
    q, k, v, ws = nabla.qkv_project(x, wt, H, D)
    nb = d["nb"]
    coords = synth.line_coords(nb, T=2, ny=2).cuda() if sta else None
    win = (3, 3, 3) if sta else None
    pooled = nabla.build_mask_pooled(q.shape, thr, ws, sta_coords=coords, sta_window=win)
    torch.cuda.synchronize()
    assert nabla.workspace_status(ws) == 0
    direct = nabla.build_mask(q, k, thr, sta_coords=coords, sta_window=win)
    torch.cuda.synchronize()
    _same_mask(pooled, direct, transpose=True)
    M, Cm, stam = gu.oracle_mask(q.cpu(), k.cpu(), thr, coords.cpu().numpy() if sta else None, win)
    bad, band, diff = gu.compare_mask(pooled, M, Cm, thr, stam)
    assert bad == 0, (bad, band, diff)
    gu.check_lists(pooled, nb)


def test_projection_full_720p_shape():
    # B=1, H=40, S=75,600, D=128, C=5120 (the hidden size of 40 heads of 128):
    # Q, K, V on 48 sampled tokens of every head, and the pooled mask against
    # the mask built from the stored Q and K on the full shape
    B, H, S, D, C = 1, 40, 75600, 128, 5120
    d = synth.make_projection_inputs(B, S, C, H, D, seed=3, device="cuda")
    x, wt = d["x"], d["wt"]
    q, k, v, ws = nabla.qkv_project(x, wt, H, D)
    torch.cuda.synchronize()
    assert nabla.workspace_status(ws) == 0
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([rng.choice(S, 44, replace=False), [0, 127, 128, S - 1]]))
    ridx = torch.from_numpy(rows).cuda()
    _check_projection([q[:, :, ridx].cpu(), k[:, :, ridx].cpu(), v[:, :, ridx].cpu()],
                      x[:, ridx].cpu(), wt.cpu(), H, D)
    pooled = nabla.build_mask_pooled(q.shape, 0.8, ws, transpose=False)
    torch.cuda.synchronize()
    assert nabla.workspace_status(ws) == 0
    direct = nabla.build_mask(q, k, 0.8, transpose=False)
    torch.cuda.synchronize()
    _same_mask(pooled, direct, transpose=False)
    # two heads against the oracle
    nb = d["nb"]
    for h in (0, 39):
        M, Cm, _ = gu.oracle_mask(q[:, h:h + 1].cpu(), k[:, h:h + 1].cpu(), 0.8)
        G = orc.bits_to_mask(gu.gpu_bits(pooled), nb)[:, h:h + 1]
        exempt = orc.band_mask(Cm, 0.8, gu.BAND)
        assert int(((G != M) & ~exempt).sum()) == 0, h


def test_projection_with_tiny_wait_limit_stops_cleanly():
    """With a 1 ns limit the projection's first wait that is not already
    satisfied runs out: the kernel stops, lets its own copies and MMAs land,
    frees TMEM and reports NABLA_ERR_TIMEOUT (0 if every wait happened to be
    satisfied at once).  The next call with the default limit is correct, and
    so is the mask built from its means."""
    B, H, S, D, C = 1, 4, 2000, 128, 512
    d = synth.make_projection_inputs(B, S, C, H, D, seed=41)
    x, wt = d["x"].cuda(), d["wt"].cuda()
    q, k, v, ws = nabla.qkv_project(x, wt, H, D)
    torch.cuda.synchronize()
    try:
        nabla.set_wait_limit_ns(1)
        nabla.qkv_project(x, wt, H, D, q, k, v, ws)
        torch.cuda.synchronize()
        assert nabla.workspace_status(ws) in (0, 4)
    finally:
        nabla.set_wait_limit_ns(0)
    nabla.qkv_project(x, wt, H, D, q, k, v, ws)
    pooled = nabla.build_mask_pooled(q.shape, 0.8, ws)
    torch.cuda.synchronize()
    assert nabla.workspace_status(ws) == 0
    _check_projection([q.cpu(), k.cpu(), v.cpu()], d["x"], d["wt"], H, D)
    _same_mask(pooled, nabla.build_mask(q, k, 0.8), transpose=True)
