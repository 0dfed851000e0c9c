"""GPU edge cases through the C ABI, against the fp64 oracle: logits far
outside the usual range (softmax rows that are one-hot in fp32, most
exponentials underflowing), and STA windows wider than the tile grid.  Masks
follow Algorithm 1 and the STA union of "∇NABLA: Neighborhood Adaptive
Block-Level Attention" (§3.1.2-3.1.3); attention is Eq. 4 (§2.2)."""
import numpy as np
import pytest
import torch

import block_sparse_attention_nabla_b200 as nabla
import synth
from oracle import nabla_oracle as orc
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("scale", [8.0, 30.0])
def test_extreme_logits_mask_and_forward(scale):
    x = synth.make_random_qkv(1, 2, 1000, 128, "bf16", seed=int(scale))
    for n in ("q", "k"):
        x[n] = (x[n].float() * scale).to(torch.bfloat16)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    thr = 0.8
    ws = nabla.workspace(q)
    mask = nabla.build_mask(q, k, thr, ws=ws)
    o, lse = nabla.attn_fwd(q, k, v, mask, ws=ws)
    torch.cuda.synchronize()
    assert nabla.workspace_status(ws) == 0
    M, C, _ = gu.oracle_mask(x["q"], x["k"], thr)
    bad, band, diff = gu.compare_mask(mask, M, C, thr)
    assert bad == 0, (bad, band, diff)
    gu.check_lists(mask, x["nb"])
    G = orc.bits_to_mask(gu.gpu_bits(mask), x["nb"])
    O, L = orc.masked_attention(x["q"], x["k"], x["v"], G)
    gu.assert_close(o, O, "bf16", f"scale {scale}")
    assert torch.isfinite(o.float()).all()
    # the LSE comes from fp32 logits of magnitude up to ~1e3 here: allow 1e-4
    # of that magnitude on top of the usual 1e-3
    assert np.abs(lse.cpu().numpy() - L).max() < 1e-4 * max(1.0, float(np.abs(L).max())) + 1e-3


def test_sta_window_wider_than_the_grid_keeps_everything():
    w = synth.WORKLOADS[6]
    coords = nabla.sta_block_coords(w.T, w.Hl, w.Wl, w.P)
    mask = nabla.build_sta_mask((1, 1, w.S, w.D), coords.cuda(), (99, 999, 999))
    torch.cuda.synchronize()
    G = orc.bits_to_mask(gu.gpu_bits(mask), w.nb)
    assert G.all()
    assert (orc.sta_mask(gu.oracle_coords(w), (99, 999, 999)) == G[0, 0]).all()
    gu.check_lists(mask, w.nb)


@pytest.mark.parametrize("scale", [2.0, 8.0])
def test_extreme_logits_backward(scale):
    """Steep softmax rows (Q and K scaled by 2 and 8): dS = P (dP - Delta)
    cancels for the dominant key, so Delta = rowsum(dO * O) must come from an
    O accurate well beyond bf16.  The forward's residual mode supplies it (P
    enters P V as two bf16 terms and O's rounding residual is written), and the
    backward takes Delta from o + o_res.  Gradients are held to the usual
    gradient bar; at scale 8 the elementwise bar also allows what the bf16
    rounding of the dS operand of the dQ and dK products can cause, 2^-8 times
    the entry's sum of term magnitudes through dS (|dS| |K| / sqrt(D) for dQ,
    |dS|^T |Q| / sqrt(D) for dK): with keys of magnitude ~25 that exceeds the
    flat 2e-2 for any kernel that multiplies dS in bf16 on the tensor cores."""
    x = synth.make_random_qkv(1, 2, 1000, 128, "bf16", seed=31, with_grad=True)
    for n in ("q", "k"):
        x[n] = (x[n].float() * scale).to(torch.bfloat16)
    M, C, _ = gu.oracle_mask(x["q"], x["k"], 0.8)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    mask = gu.mask_on_gpu(M, tuple(q.shape), q.dtype)
    o_res = torch.empty_like(q)
    o, lse = nabla.attn_fwd(q, k, v, mask, o_res=o_res)
    ws = nabla.workspace(q, want_bwd=True)
    dq, dk, dv = nabla.attn_bwd(q, k, v, o, do, lse, mask, ws=ws, o_res=o_res)
    torch.cuda.synchronize()
    assert nabla.workspace_status(ws) == 0
    dQ, dK, dV, bQ, bK = orc.masked_attention_bwd(x["q"], x["k"], x["v"], x["do"], M, ds_bound=True)
    if scale <= 2.0:
        for got, r, name in zip((dq, dk, dv), (dQ, dK, dV), ("dQ", "dK", "dV")):
            gu.assert_close(got, r, "bf16", f"{name} scale {scale}", grad=True)
    else:
        for got, r, bnd, name in zip((dq, dk, dv), (dQ, dK, dV), (bQ, bK, 0.0), ("dQ", "dK", "dV")):
            g = orc.as_f64(got)
            assert np.isfinite(g).all(), name
            excess = np.abs(g - r) - gu.GRAD_REL * np.abs(r) - gu.GRAD_REL * bnd
            assert excess.max() <= gu.TOL["bf16"]["max_abs"], (name, float(excess.max()))
            assert orc.mean_rel(g, r) <= gu.TOL["bf16"]["mean_rel"], (name, orc.mean_rel(g, r))


def test_extreme_logits_block_mass():
    x = synth.make_random_qkv(1, 1, 1000, 128, "bf16", seed=32)
    for n in ("q", "k"):
        x[n] = (x[n].float() * 8.0).to(torch.bfloat16)
    A = nabla.block_mass(x["q"].cuda(), x["k"].cuda())
    torch.cuda.synchronize()
    ref = orc.block_mass(x["q"], x["k"])
    got = A.cpu().numpy()
    assert np.isfinite(got).all()
    assert np.abs(got - ref).max() < 1e-3
    assert np.abs(got.sum(-1) - 1.0).max() < 1e-3
