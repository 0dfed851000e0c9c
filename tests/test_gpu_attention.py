"""GPU parity of block-sparse attention (Eq. 4 of "∇NABLA: Neighborhood
Adaptive Block-Level Attention", §2.2, over the kept tiles of the NABLA mask)
against the fp64 oracle, computed under the oracle's own mask.

Bar: max-abs 2e-2 and mean-rel 5e-3 for bf16 outputs, 1e-4 (both metrics)
for fp32.  bf16 gradients dQ, dK, dV: elementwise |x - ref| <= 2e-2 + 2^-8 |ref|
and mean-rel 5e-3 (see gpu_util.GRAD_REL for why the absolute bar scales)."""
import numpy as np
import pytest
import torch

import block_sparse_attention_nabla_b200 as nabla
import synth
from oracle import nabla_oracle as orc
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


def _fwd_parity(x, M, kind):
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    mask = gu.mask_on_gpu(M, tuple(q.shape), q.dtype)
    ws = nabla.workspace(q)
    o, lse = nabla.attn_fwd(q, k, v, mask, ws=ws)
    torch.cuda.synchronize()
    assert nabla.workspace_status(ws) == 0
    O, LSE = orc.masked_attention(x["q"], x["k"], x["v"], M)
    gu.assert_close(o, O, kind, "O")
    rows = np.isfinite(LSE)
    assert np.abs(lse.cpu().numpy()[rows] - LSE[rows]).max() < (1e-3 if kind == "bf16" else 1e-5)
    return o, lse, mask


def test_fwd_tiny_fp32_workload():
    w = synth.WORKLOADS[1]
    x = synth.make_inputs(w)
    M, C, _ = gu.oracle_mask(x["q"], x["k"], w.thresholds[0])
    _fwd_parity(x, M, "fp32")


@pytest.mark.parametrize("S,D", [(1000, 128), (414, 128), (1000, 64), (130, 64), (64, 128), (37, 128)])
@pytest.mark.parametrize("thr", [0.5, 0.9, 1.0])
def test_fwd_small_bf16(S, D, thr):
    x = synth.make_random_qkv(2, 2, S, D, "bf16", seed=3 * S + D)
    M, C, _ = gu.oracle_mask(x["q"], x["k"], thr)
    _fwd_parity(x, M, "bf16")


@pytest.mark.parametrize("S,D", [(1000, 128), (130, 64), (37, 128)])
def test_fwd_small_fp32(S, D):
    # the fp32 inputs run on the CUDA cores: ragged tails at both head sizes
    x = synth.make_random_qkv(2, 2, S, D, "fp32", seed=5 * S + D)
    M, C, _ = gu.oracle_mask(x["q"], x["k"], 0.7)
    _fwd_parity(x, M, "fp32")


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_fwd_edge_masks(dtype):
    # empty rows, a full row, only the ragged tail block, a random pattern
    S, nb = 64 * 9 + 7, 10
    x = synth.make_random_qkv(1, 2, S, 128, dtype, seed=11)
    rng = np.random.default_rng(4)
    M = rng.random((1, 2, nb, nb)) < 0.3
    M[0, 0, 3] = False
    M[0, 0, 4] = False            # both rows of pair 2 empty
    M[0, 1, 5] = True
    M[0, 1, 9] = False
    M[0, 1, 9, 9] = True
    M[0, 1, 0] = False
    M[0, 1, 0, 9] = True          # row 0 only sees the tail block
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    mask = gu.mask_on_gpu(M, tuple(q.shape), q.dtype)
    o, lse = nabla.attn_fwd(q, k, v, mask)
    torch.cuda.synchronize()
    O, LSE = orc.masked_attention(x["q"], x["k"], x["v"], M)
    gu.assert_close(o, O, dtype, "O")
    empty = np.zeros((1, 2, S), dtype=bool)
    empty[0, 0, 3 * 64:5 * 64] = True
    assert (o.float().cpu().numpy()[empty] == 0).all()
    assert np.isneginf(lse.cpu().numpy()[empty]).all()


@pytest.mark.parametrize("wid,heads", [(2, list(range(40))), (3, list(range(40))), (7, list(range(40)))])
def test_fwd_full_size_sampled_rows(wid, heads):
    """Full-size forward (the benchmark's launch configuration) under the
    oracle's mask, checked on sampled rows of every head of the 480p and 720p
    shapes."""
    w = synth.WORKLOADS[wid]
    x = synth.make_inputs(w)
    thr = w.thresholds[0]
    M, C, _ = gu.oracle_mask(x["q"], x["k"], thr)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    mask = gu.mask_on_gpu(M, tuple(q.shape), q.dtype)
    ws = nabla.workspace(q)
    o, lse = nabla.attn_fwd(q, k, v, mask, ws=ws)
    torch.cuda.synchronize()
    assert nabla.workspace_status(ws) == 0
    rng = np.random.default_rng(wid)
    S = w.S
    rows = np.unique(np.concatenate([[0, 1, 63, 64, 127, 128, S - 1, S - 2, S - 17],
                                     rng.integers(0, S, size=40)]))
    for h in heads:
        Or, Lr = orc.masked_attention_rows(x["q"], x["k"], x["v"], M, 0, h, rows)
        gu.assert_close(o[0, h, rows], Or, "bf16", f"head {h}")
        assert np.abs(lse[0, h, rows].cpu().numpy() - Lr).max() < 1e-3
    assert torch.isfinite(o.float()).all()


def test_fwd_uses_gpu_built_mask_end_to_end():
    w = synth.WORKLOADS[2].scaled(H=4)
    x = synth.make_inputs(w)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    mask = nabla.build_mask(q, k, 0.8)
    o, lse = nabla.attn_fwd(q, k, v, mask)
    torch.cuda.synchronize()
    G = orc.bits_to_mask(gu.gpu_bits(mask), w.nb)
    rows = np.arange(0, w.S, 997)
    for h in range(4):
        Or, _ = orc.masked_attention_rows(x["q"], x["k"], x["v"], G, 0, h, rows)
        gu.assert_close(o[0, h, rows], Or, "bf16", f"head {h}")


# ---------------------------------------------------------------- backward

def _bwd_parity(x, M, kind, heads=None, residual=False):
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    mask = gu.mask_on_gpu(M, tuple(q.shape), q.dtype)
    o_res = torch.empty_like(q) if residual else None
    o, lse = nabla.attn_fwd(q, k, v, mask, o_res=o_res)
    ws = nabla.workspace(q, want_bwd=True)
    dq, dk, dv = nabla.attn_bwd(q, k, v, o, do, lse, mask, ws=ws, o_res=o_res)
    torch.cuda.synchronize()
    assert nabla.workspace_status(ws) == 0
    for (b, h) in ([(b, h) for b in range(q.shape[0]) for h in range(q.shape[1])] if heads is None else heads):
        sl = (slice(b, b + 1), slice(h, h + 1))
        dQ, dK, dV = orc.masked_attention_bwd(x["q"][sl], x["k"][sl], x["v"][sl], x["do"][sl], M[sl])
        gu.assert_close(dq[sl], dQ, kind, f"dQ b{b} h{h}", grad=True)
        gu.assert_close(dk[sl], dK, kind, f"dK b{b} h{h}", grad=True)
        gu.assert_close(dv[sl], dV, kind, f"dV b{b} h{h}", grad=True)


def test_bwd_tiny_fp32():
    w = synth.WORKLOADS[1].scaled(with_grad=True)
    x = synth.make_inputs(w)
    M, C, _ = gu.oracle_mask(x["q"], x["k"], w.thresholds[0])
    _bwd_parity(x, M, "fp32")


@pytest.mark.parametrize("residual", [False, True])
@pytest.mark.parametrize("S,D", [(1000, 128), (414, 64), (130, 128)])
def test_bwd_small_bf16(S, D, residual):
    x = synth.make_random_qkv(1, 2, S, D, "bf16", seed=S, with_grad=True)
    M, C, _ = gu.oracle_mask(x["q"], x["k"], 0.8)
    _bwd_parity(x, M, "bf16", residual=residual)


@pytest.mark.parametrize("S,D", [(1000, 128), (130, 64)])
def test_bwd_small_fp32(S, D):
    x = synth.make_random_qkv(1, 2, S, D, "fp32", seed=7 * S + D, with_grad=True)
    M, C, _ = gu.oracle_mask(x["q"], x["k"], 0.8)
    _bwd_parity(x, M, "fp32")


@pytest.mark.parametrize("residual,heads", [
    (False, [(0, 0), (1, 15)]),
    # the training configuration (residual mode): eight heads over both samples
    (True, [(b, h) for b in (0, 1) for h in (0, 5, 10, 15)]),
])
def test_bwd_pretraining_workload(residual, heads):
    w = synth.WORKLOADS[4]
    x = synth.make_inputs(w)
    M, C, _ = gu.oracle_mask(x["q"], x["k"], w.thresholds[0])
    _bwd_parity(x, M, "bf16", heads=heads, residual=residual)


@pytest.mark.parametrize("B,H,S,seed", [(1, 2, 1000, 21), (2, 3, 2000, 22), (1, 1, 64, 23)])
def test_bwd_external_mask_empty_rows_columns_and_odd_lists(B, H, S, seed):
    """A mask given as bits (not built here): some query blocks keep nothing,
    some key blocks are kept by no query block, list lengths are odd and even,
    so the stacked pairs of both backward kernels end ragged."""
    x = synth.make_random_qkv(B, H, S, 128, "bf16", seed=seed, with_grad=True)
    nb = -(-S // 64)
    rng = np.random.default_rng(seed)
    M = rng.random((B, H, nb, nb)) < 0.45
    if nb > 3:
        M[:, :, 1, :] = False           # a query block that attends to nothing
        M[:, :, :, 2] = False           # a key block nobody attends to
        M[:, :, 3, :] = False
        M[:, :, 3, nb - 1] = True       # one kept block: a lone (odd) step, ragged tail keys
    _bwd_parity(x, M, "bf16", residual=True)


@pytest.mark.parametrize("S,D", [(1000, 128), (414, 64)])
def test_forward_residual_carries_o_beyond_bf16(S, D):
    """Residual mode of the forward: o alone still meets the bf16 output bar,
    and o + o_res matches the fp64 oracle's O to about 2^-13 relative (P V with
    P in two bf16 terms; the residual of O rounded to bf16), where bf16 alone
    is 2^-9.  Rows of a block that keeps nothing get o = o_res = 0."""
    x = synth.make_random_qkv(1, 2, S, D, "bf16", seed=3 * S + D)
    M, C, _ = gu.oracle_mask(x["q"], x["k"], 0.8)
    M[0, 1, 2, :] = False                               # an empty query block
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    mask = gu.mask_on_gpu(M, tuple(q.shape), q.dtype)
    ws = nabla.workspace(q)
    o_res = torch.full_like(q, 7.0)
    o, lse = nabla.attn_fwd(q, k, v, mask, ws=ws, o_res=o_res)
    torch.cuda.synchronize()
    assert nabla.workspace_status(ws) == 0
    O, L = orc.masked_attention(x["q"], x["k"], x["v"], M)
    gu.assert_close(o, O, "bf16", "o in residual mode")
    full = orc.as_f64(o) + orc.as_f64(o_res)
    err = np.abs(full - O)
    assert (err <= 2e-5 + 2.0 ** -13 * np.abs(O)).all(), float((err - 2.0 ** -13 * np.abs(O)).max())
    assert orc.mean_rel(full, O) < 2e-5
    assert (orc.as_f64(o_res)[0, 1, 128:192] == 0).all()
    assert np.abs(lse.cpu().numpy()[np.isfinite(L)] - L[np.isfinite(L)]).max() < 1e-3
    # the plain forward's o agrees with the residual mode's o to a bf16 ulp
    o2, _ = nabla.attn_fwd(q, k, v, mask, ws=ws)
    torch.cuda.synchronize()
    assert np.abs(orc.as_f64(o2) - orc.as_f64(o)).max() <= 2.0 ** -7 * max(1.0, float(np.abs(O).max()))


# ------------------------------------------------------ bounded waits

def test_bounded_wait_runs_out_and_reports_timeout():
    """A wait on a barrier that nothing arrives on runs out after its limit;
    the kernel records NABLA_ERR_TIMEOUT and the context stays usable."""
    x = synth.make_random_qkv(1, 2, 1000, 128, "bf16", seed=5)
    M, C, _ = gu.oracle_mask(x["q"], x["k"], 0.8)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    ws = nabla.workspace(q)
    assert nabla.selftest_wait_timeout(ws, 2_000_000) == 4
    mask = gu.mask_on_gpu(M, tuple(q.shape), q.dtype)
    o, lse = nabla.attn_fwd(q, k, v, mask, ws=ws)
    torch.cuda.synchronize()
    assert nabla.workspace_status(ws) == 0
    O, _ = orc.masked_attention(x["q"], x["k"], x["v"], M)
    gu.assert_close(o, O, "bf16", "O after a timed-out wait")


def test_forward_with_tiny_wait_limit_stops_cleanly():
    """With a 1 ns limit the forward kernel's first wait that is not already
    satisfied runs out: the kernel stops, drains its own copies and MMAs,
    frees TMEM and reports NABLA_ERR_TIMEOUT (0 if every wait happened to be
    satisfied at once).  The next call with the default limit is correct."""
    x = synth.make_random_qkv(1, 4, 4096, 128, "bf16", seed=5)
    M, C, _ = gu.oracle_mask(x["q"], x["k"], 1.0)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    mask = gu.mask_on_gpu(M, tuple(q.shape), q.dtype)
    ws = nabla.workspace(q)
    try:
        nabla.set_wait_limit_ns(1)
        nabla.attn_fwd(q, k, v, mask, ws=ws)
        torch.cuda.synchronize()
        assert nabla.workspace_status(ws) in (0, 4)
    finally:
        nabla.set_wait_limit_ns(0)
    o, lse = nabla.attn_fwd(q, k, v, mask, ws=ws)
    torch.cuda.synchronize()
    assert nabla.workspace_status(ws) == 0
    O, _ = orc.masked_attention(x["q"][:, :1], x["k"][:, :1], x["v"][:, :1], M[:, :1])
    gu.assert_close(o[:, :1], O, "bf16", "O after timeout")


def test_forward_with_long_runs_of_empty_units():
    """External mask whose query-block pairs are empty in long runs, with many
    more units (16 heads x 32 pairs = 512) than CTAs (two per SM), so each CTA
    draws several units and meets empty units back to back, and after units
    with tiles.  Rows of an empty block get O = 0 and LSE = -inf; the rest
    match the oracle (Eq. 4 of §2.2), and no bounded wait runs out."""
    B, H, S = 1, 16, 4096
    x = synth.make_random_qkv(B, H, S, 128, "bf16", seed=41)
    nb = S // 64
    rng = np.random.default_rng(41)
    M = rng.random((B, H, nb, nb)) < 0.3
    for h in range(H):
        # runs of empty pairs: pairs [a, a + len) of this head keep nothing
        a = int(rng.integers(0, 20))
        M[0, h, 2 * a:2 * (a + 6 + h % 3)] = False
        if h % 2:
            M[0, h, 0:2] = False                       # the head's first pair
        if h % 4 == 1:
            M[0, h, nb - 6:] = False                   # its last three pairs
        M[0, h, 2 * (a + 10), :] = False               # one empty block inside a non-empty pair
    M[0, 3] = False                                    # one head with no tile at all
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    mask = gu.mask_on_gpu(M, tuple(q.shape), q.dtype)
    ws = nabla.workspace(q)
    o, lse = nabla.attn_fwd(q, k, v, mask, ws=ws)
    torch.cuda.synchronize()
    assert nabla.workspace_status(ws) == 0
    O, L = orc.masked_attention(x["q"], x["k"], x["v"], M)
    gu.assert_close(o, O, "bf16", "long runs of empty units")
    empty = ~M.any(-1)                                 # [B, H, nb] query blocks that keep nothing
    rows = np.repeat(empty, 64, axis=-1)[..., :S]
    assert rows.sum() > 0
    assert (o.float().cpu().numpy()[rows] == 0).all()
    assert np.isneginf(lse.cpu().numpy()[rows]).all()
    lg = lse.cpu().numpy()[~rows]
    assert np.abs(lg - L[~rows]).max() < 1e-3
