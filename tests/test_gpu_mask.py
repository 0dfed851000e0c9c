"""GPU parity of the mask builder (Algorithm 1 of "∇NABLA: Neighborhood
Adaptive Block-Level Attention", §3.1.2, with the STA union of §3.1.3)
against the fp64 oracle, through the C ABI.

Bar: the bitmask matches the oracle bit for bit except entries whose oracle
cumulative mass lies within 1e-5 of 1 - thr; cnt/idx, the transposed lists and
the work list follow exactly from the bitmask."""
import numpy as np
import pytest
import torch

import block_sparse_attention_nabla_b200 as nabla
import synth
from oracle import nabla_oracle as orc
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


def _run(w, heads=None, thr=None, sta=False):
    x = synth.make_inputs(w, heads=heads)
    thr = w.thresholds[0] if thr is None else thr
    q, k = x["q"].cuda(), x["k"].cuda()
    coords = gu.lib_coords(w) if sta else None
    mask = nabla.build_mask(q, k, thr, sta_coords=coords, sta_window=w.sta_window if sta else None)
    torch.cuda.synchronize()
    M, C, stam = gu.oracle_mask(x["q"], x["k"], thr, gu.oracle_coords(w) if sta else None,
                                w.sta_window if sta else None)
    return x, mask, M, C, stam


def test_mask_tiny_fp32_workload():
    w = synth.WORKLOADS[1]
    x, mask, M, C, _ = _run(w)
    bad, band, diff = gu.compare_mask(mask, M, C, w.thresholds[0])
    assert bad == 0, (bad, band, diff)
    gu.check_lists(mask, w.nb)


@pytest.mark.parametrize("S", [1000, 414, 64, 1, 130])
@pytest.mark.parametrize("D", [128, 64])
@pytest.mark.parametrize("thr", [0.3, 0.8, 1.0])
def test_mask_small_ragged_bf16(S, D, thr):
    x = synth.make_random_qkv(2, 3, S, D, "bf16", seed=S + D)
    q, k = x["q"].cuda(), x["k"].cuda()
    mask = nabla.build_mask(q, k, thr)
    torch.cuda.synchronize()
    M, C, _ = gu.oracle_mask(x["q"], x["k"], thr)
    bad, band, diff = gu.compare_mask(mask, M, C, thr)
    assert bad == 0, (bad, band, diff)
    gu.check_lists(mask, x["nb"])
    if thr == 1.0:
        assert orc.bits_to_mask(gu.gpu_bits(mask), x["nb"]).all()


@pytest.mark.parametrize("thr", [0.7, 0.8, 0.9])
def test_mask_480p_full_size(thr):
    w = synth.WORKLOADS[2]
    x, mask, M, C, _ = _run(w, thr=thr)
    bad, band, diff = gu.compare_mask(mask, M, C, thr)
    assert bad == 0, (bad, band, diff)
    gu.check_lists(mask, w.nb, check_transpose=(thr == 0.8))


@pytest.mark.parametrize("sta", [False, True])
def test_mask_720p_full_size(sta):
    w = synth.WORKLOADS[3]
    x, mask, M, C, stam = _run(w, sta=sta)
    bad, band, diff = gu.compare_mask(mask, M, C, w.thresholds[0], stam)
    assert bad == 0, (bad, band, diff)
    if sta:
        G = orc.bits_to_mask(gu.gpu_bits(mask), w.nb)
        assert (G >= stam[None, None]).all()     # every STA tile kept
    else:
        gu.check_lists(mask, w.nb, check_transpose=False)


@pytest.mark.parametrize("thr", [0.5, 0.8, 0.95])
def test_mask_720p_sigma06_sparse_masks(thr):
    # block means of std 0.6: 1.6 % of tiles kept at thr 0.5, 18 % at 0.8
    w = synth.WORKLOADS[7]
    x, mask, M, C, _ = _run(w, heads=list(range(0, 40, 5)), thr=thr)
    bad, band, diff = gu.compare_mask(mask, M, C, thr)
    assert bad == 0, (bad, band, diff)
    gu.check_lists(mask, w.nb, check_transpose=(thr == 0.5))


def test_mask_sta_only_window_matches_oracle():
    # thr tiny: the NABLA part keeps only each row's top block, STA adds its window.
    w = synth.WORKLOADS[3].scaled(H=2)
    x, mask, M, C, stam = _run(w, thr=1e-6, sta=True)
    bad, band, diff = gu.compare_mask(mask, M, C, 1e-6, stam)
    assert bad == 0
    gu.check_lists(mask, w.nb)


def test_mask_from_bits_edge_rows():
    S, nb = 64 * 9 + 7, 10
    rng = np.random.default_rng(0)
    M = rng.random((1, 2, nb, nb)) < 0.4
    M[0, 0, 3] = False            # empty row
    M[0, 1, 5] = True             # full row
    M[0, 1, 9] = False
    M[0, 1, 9, 9] = True          # only the ragged tail block
    mask = gu.mask_on_gpu(M, (1, 2, S, 128), torch.bfloat16)
    torch.cuda.synchronize()
    assert (orc.bits_to_mask(gu.gpu_bits(mask), nb) == M).all()
    gu.check_lists(mask, nb)


# ------------------------------------------------ fixed-budget comparator

def _topk_check(mask, M, X, nb, topk, sta=False):
    G = orc.bits_to_mask(gu.gpu_bits(mask), nb)
    bad = int(((G != M) & ~X).sum())
    assert bad == 0, (bad, int(X.sum()))
    if not sta:
        # exactly min(topk, nb) per row wherever no near-tie sits at the cut
        rows = ~X.any(-1)
        assert (G.sum(-1)[rows] == min(topk, nb)).all()
    gu.check_lists(mask, nb)


@pytest.mark.parametrize("S", [1000, 414, 64, 1, 130])
@pytest.mark.parametrize("D", [128, 64])
@pytest.mark.parametrize("topk", [1, 3, 8, 40])
def test_topk_small_ragged_bf16(S, D, topk):
    x = synth.make_random_qkv(2, 3, S, D, "bf16", seed=S + D + 7)
    q, k = x["q"].cuda(), x["k"].cuda()
    mask = nabla.build_mask_topk(q, k, topk)
    torch.cuda.synchronize()
    M, X = gu.oracle_topk(x["q"], x["k"], topk)
    _topk_check(mask, M, X, x["nb"], topk)


@pytest.mark.parametrize("sta", [False, True])
def test_topk_720p_two_heads_at_the_cdf_budget(sta):
    """720p frames, two heads, k = the mean kept count of the CDF rule at thr 0.8
    on the same heads (the equal-budget comparison of the pages)."""
    w = synth.WORKLOADS[3].scaled(H=2)
    x = synth.make_inputs(w)
    q, k = x["q"].cuda(), x["k"].cuda()
    cdf = nabla.build_mask(q, k, 0.8)
    topk = int(round(cdf.cnt.float().mean().item()))
    coords = gu.lib_coords(w) if sta else None
    mask = nabla.build_mask_topk(q, k, topk, sta_coords=coords, sta_window=w.sta_window if sta else None)
    torch.cuda.synchronize()
    M, X = gu.oracle_topk(x["q"], x["k"], topk, gu.oracle_coords(w) if sta else None,
                          w.sta_window if sta else None)
    _topk_check(mask, M, X, w.nb, topk, sta)
