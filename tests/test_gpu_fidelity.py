"""GPU parity of the per-block fidelity kernels (the check the pith.science review of
"∇NABLA: Neighborhood Adaptive Block-Level Attention" asks of Algorithm 1's
pooling proxy) against the fp64 oracle: the true token-level block mass of
dense attention and the kept mass (recall) of a block mask.

Tolerance: the kernel forms the logits with bf16 operands exactly and fp32
accumulation, then sums fp32 exponentials; a block mass is a mean of sums of
at most 64 x 64 probabilities, so its error is a few fp32 ulps of the row
sums: bar 1e-4 absolute on every entry (masses lie in [0, 1])."""
import numpy as np
import pytest
import torch

import block_sparse_attention_nabla_b200 as nabla
import synth
from oracle import nabla_oracle as orc
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu
TOL = 1e-4


@pytest.mark.parametrize("B,H,S,D", [(1, 2, 1000, 128), (2, 1, 130, 64), (1, 1, 64, 128), (1, 2, 1, 64),
                                     (1, 1, 4096, 64)])
def test_block_mass_matches_oracle(B, H, S, D):
    x = synth.make_random_qkv(B, H, S, D, "bf16", seed=S + 31 * D)
    q, k = x["q"].cuda(), x["k"].cuda()
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    A = nabla.block_mass(q, k, ws=ws)
    torch.cuda.synchronize()
    assert nabla.workspace_status(ws) == 0
    ref = orc.block_mass(x["q"], x["k"])
    got = A.cpu().numpy()
    assert np.abs(got - ref).max() <= TOL
    assert np.abs(got.sum(-1) - 1).max() <= TOL


@pytest.mark.parametrize("thr", [0.5, 0.8, 1.0])
def test_recall_of_gpu_mask_matches_oracle(thr):
    x = synth.make_random_qkv(1, 2, 2000, 128, "bf16", seed=77)
    q, k = x["q"].cuda(), x["k"].cuda()
    mask = nabla.build_mask(q, k, thr)
    A = nabla.block_mass(q, k)
    R = nabla.mask_recall(A, mask, tuple(q.shape))
    torch.cuda.synchronize()
    G = orc.bits_to_mask(gu.gpu_bits(mask), x["nb"])
    ref = orc.mask_recall(orc.block_mass(x["q"], x["k"]), G)
    assert np.abs(R.cpu().numpy() - ref).max() <= TOL
    if thr == 1.0:
        assert np.abs(R.cpu().numpy() - 1).max() <= TOL


def test_block_mass_720p_sampled_rows():
    """720p frames (S = 75,600, nb = 1182), two heads: every row sums to 1 and
    sampled query blocks (first, last, ragged tail, random) match the oracle."""
    w = synth.WORKLOADS[3].scaled(H=2)
    x = synth.make_inputs(w)
    q, k = x["q"].cuda(), x["k"].cuda()
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    A = nabla.block_mass(q, k, ws=ws)
    torch.cuda.synchronize()
    assert nabla.workspace_status(ws) == 0
    got = A.cpu().numpy()
    assert np.abs(got.sum(-1) - 1).max() <= 1e-3
    assert (got >= 0).all()
    blocks = [0, 1, 590, 591, w.nb - 2, w.nb - 1] + list(np.random.default_rng(9).integers(0, w.nb, 4))
    for h in range(2):
        ref = orc.block_mass_rows(x["q"], x["k"], 0, h, blocks)
        assert np.abs(got[0, h, blocks] - ref).max() <= TOL
