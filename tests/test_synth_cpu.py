"""The seeded input generator's block structure (host only).

The second 720p sweep draws its inputs with block means and locality anchors
of standard deviation 0.6 instead of 0.5 and the same seed, so it must see the
same per-token noise with the block terms scaled by 1.2: the difference of the
two draws is constant over every 64-token block, and removing five times that
difference from the 0.5 draw leaves standard normal noise."""
import numpy as np

import synth


def _small(wid):
    # a few frames of the same generator in fp32 (no bf16 rounding)
    return synth.WORKLOADS[wid].scaled(H=2, T=2, Hl=16, Wl=24, dtype="fp32")


def test_sigma06_sweep_is_the_sigma05_sweep_with_scaled_block_terms():
    w5, w7 = _small(5), _small(7)
    assert (w5.seed, w5.sigma) == (w7.seed, 0.5) and w7.sigma == 0.6
    x5, x7 = synth.make_inputs(w5), synth.make_inputs(w7)
    S = w5.S
    assert S % synth.BLOCK == 0
    for n in ("q", "k", "v"):
        d = (x7[n] - x5[n]).double().reshape(w5.B, w5.H, S // synth.BLOCK, synth.BLOCK, w5.D)
        # one value per (block, dimension): the extra 0.1 / 0.5 of the block term
        assert (d - d[:, :, :, :1]).abs().max().item() < 1e-5
        assert d.abs().max().item() > 0.05
        eps = (x5[n].double() - 5.0 * (x7[n] - x5[n]).double()).numpy()
        assert abs(eps.mean()) < 0.02
        assert abs(eps.std() - 1.0) < 0.02


def test_sigma06_workload_shape_matches_the_720p_sweep():
    w5, w7 = synth.WORKLOADS[5], synth.WORKLOADS[7]
    assert (w7.B, w7.H, w7.S, w7.D, w7.dtype, w7.locality) == (w5.B, w5.H, w5.S, w5.D, w5.dtype, w5.locality)
    assert w7.thresholds == w5.thresholds == [0.5, 0.7, 0.8, 0.9, 0.95, 1.0]
    assert np.array_equal(synth.block_coords(w7.T, w7.Hl, w7.Wl, w7.P),
                          synth.block_coords(w5.T, w5.Hl, w5.Wl, w5.P))
