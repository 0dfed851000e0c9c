"""GPU parity of the fractal token reordering (§3.1.1, Figure 3 of "∇NABLA:
Neighborhood Adaptive Block-Level Attention") against the oracle: a pure row
permutation, so the comparison is bit-exact."""
import numpy as np
import pytest
import torch

import block_sparse_attention_nabla_b200 as nabla
from oracle import nabla_oracle as orc

pytestmark = pytest.mark.gpu


def _rows(B, S, C, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randint(-32768, 32767, (B, S, C), dtype=torch.int16, generator=g)


@pytest.mark.parametrize("B,T,H,W,P,C", [
    (1, 1, 16, 16, 8, 8),        # Figure 3's latent, 16-byte rows
    (2, 3, 3, 5, 2, 8),          # partial patches on both edges
    (1, 2, 30, 52, 8, 64),       # 480p frames (52 = 6 * 8 + 4)
    (1, 3, 45, 80, 8, 24),       # 720p frames, 48-byte rows (3 chunks per row)
    (2, 1, 7, 9, 4, 264),        # 528-byte rows (33 chunks)
    (1, 1, 5, 1, 4, 1024),       # a single column
])
def test_reorder_and_inverse_bit_exact(B, T, H, W, P, C):
    x = _rows(B, T * H * W, C, seed=B * 1000 + H * W + C)
    xd = x.cuda()
    y = nabla.fractal_reorder(xd, T, H, W, P)
    back = nabla.fractal_reorder(y, T, H, W, P, inverse=True)
    torch.cuda.synchronize()
    ref = orc.fractal_reorder(x.numpy(), T, H, W, P)
    assert np.array_equal(y.cpu().numpy(), ref)
    assert np.array_equal(back.cpu().numpy(), x.numpy())
    ref_inv = orc.fractal_reorder(x.numpy(), T, H, W, P, inverse=True)
    assert np.array_equal(nabla.fractal_reorder(xd, T, H, W, P, inverse=True).cpu().numpy(), ref_inv)


def test_reorder_full_size_720p_bf16_activations():
    """The benchmark's configuration: B=1, 21 x 45 x 80 latent tokens, C = 5120
    bf16 channels per token (rows of 10 KB), forward and inverse."""
    T, H, W, P, C = 21, 45, 80, 8, 5120
    x = _rows(1, T * H * W, C, seed=7)
    xd = x.cuda()
    y = nabla.fractal_reorder(xd.view(torch.bfloat16), T, H, W, P)
    torch.cuda.synchronize()
    perm = orc.fractal_order(T, H, W, P)
    yh = y.view(torch.int16).cpu().numpy()
    assert np.array_equal(yh, x.numpy()[:, perm])
    back = nabla.fractal_reorder(y, T, H, W, P, inverse=True)
    assert torch.equal(back.view(torch.int16).cpu(), x)
