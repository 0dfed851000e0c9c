"""GPU parity at long sequences, through the C ABI: the selection's 64-word
register path (1,281 to 2,048 blocks per row), its shared-memory path (more
than 2,048 blocks: the row stays in the logits buffer and the cut-off is
found by binary search), the work list's shared-memory sort (more than 1,024
query-block pairs), and the largest problem the library accepts (8,192
blocks, S = 524,288 tokens), where the forward is checked on sampled rows.
Masks follow Algorithm 1 of "∇NABLA: Neighborhood Adaptive Block-Level
Attention" (§3.1.2); attention is Eq. 4 (§2.2)."""
import numpy as np
import pytest
import torch

import block_sparse_attention_nabla_b200 as nabla
import synth
from oracle import nabla_oracle as orc
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("nblocks,tail", [(1500, 64), (2101, 17)])
def test_mask_and_lists_long_rows(nblocks, tail):
    S = (nblocks - 1) * 64 + tail
    x = synth.make_random_qkv(1, 1, S, 128, "bf16", seed=nblocks)
    q, k = x["q"].cuda(), x["k"].cuda()
    thr = 0.8
    mask = nabla.build_mask(q, k, thr)
    torch.cuda.synchronize()
    M, C, _ = gu.oracle_mask(x["q"], x["k"], thr)
    bad, band, diff = gu.compare_mask(mask, M, C, thr)
    assert bad == 0, (bad, band, diff)
    gu.check_lists(mask, x["nb"])


def test_largest_supported_problem_mask_and_forward():
    S = 8192 * 64
    x = synth.make_random_qkv(1, 1, S, 128, "bf16", seed=8192)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    thr = 0.5
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
    rng = np.random.default_rng(8192)
    rows = np.unique(np.concatenate([[0, 63, 64, S - 64, S - 1], rng.integers(0, S, size=20)]))
    Or, Lr = orc.masked_attention_rows(x["q"], x["k"], x["v"], G, 0, 0, rows)
    gu.assert_close(o[0, 0, rows], Or, "bf16", "largest problem")
    assert np.abs(lse[0, 0, rows].cpu().numpy() - Lr).max() < 1e-3


@pytest.mark.parametrize("nblocks,topk", [(1500, 700), (2101, 1000)])
def test_topk_long_rows(nblocks, topk):
    """The fixed-budget comparator on long rows: the k-th largest entry's
    bucket is ranked by fp64 logits as in the CDF rule."""
    from tests.test_gpu_mask import _topk_check
    S = nblocks * 64 - 5
    x = synth.make_random_qkv(1, 1, S, 128, "bf16", seed=nblocks + topk)
    q, k = x["q"].cuda(), x["k"].cuda()
    mask = nabla.build_mask_topk(q, k, topk)
    torch.cuda.synchronize()
    M, X = gu.oracle_topk(x["q"], x["k"], topk)
    _topk_check(mask, M, X, x["nb"], topk)


def test_backward_long_rows_sparse_mask():
    """Backward with more than 2,048 blocks (long column and row lists), under a
    sparse external mask that keeps the fp64 oracle affordable: each query
    block keeps its own block and six random others."""
    S = 2101 * 64 - 47
    nb = -(-S // 64)
    x = synth.make_random_qkv(1, 1, S, 128, "bf16", seed=2101, with_grad=True)
    rng = np.random.default_rng(2101)
    M = np.zeros((1, 1, nb, nb), dtype=bool)
    for i in range(nb):
        M[0, 0, i, rng.choice(nb, size=6, replace=False)] = True
        M[0, 0, i, i] = True
    M[0, 0, :, nb - 1] |= rng.random(nb) < 0.01      # some rows reach the ragged last block
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    mask = gu.mask_on_gpu(M, tuple(q.shape), q.dtype)
    o, lse = nabla.attn_fwd(q, k, v, mask)
    ws = nabla.workspace(q, want_bwd=True)
    dq, dk, dv = nabla.attn_bwd(q, k, v, o, do, lse, mask, ws=ws)
    torch.cuda.synchronize()
    assert nabla.workspace_status(ws) == 0
    gu.check_lists(mask, nb)
    O, _ = orc.masked_attention(x["q"], x["k"], x["v"], M)
    gu.assert_close(o, O, "bf16", "forward")
    dQ, dK, dV = orc.masked_attention_bwd(x["q"], x["k"], x["v"], x["do"], M)
    gu.assert_close(dq, dQ, "bf16", "dQ", grad=True)
    gu.assert_close(dk, dK, "bf16", "dK", grad=True)
    gu.assert_close(dv, dV, "bf16", "dV", grad=True)


@pytest.mark.parametrize("nblocks", [2101, 8192])
def test_block_mass_long_rows(nblocks):
    """The block-fidelity pass on long rows (its per-row partial sums take
    16 nb bytes of shared memory: one CTA per SM at the largest size)."""
    S = nblocks * 64 - (5 if nblocks < 8192 else 0)
    x = synth.make_random_qkv(1, 1, S, 128, "bf16", seed=nblocks + 7)
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    A = nabla.block_mass(x["q"].cuda(), x["k"].cuda(), ws=ws)
    torch.cuda.synchronize()
    assert nabla.workspace_status(ws) == 0
    nb = x["nb"]
    blocks = [0, 1, nb - 1] + list(np.random.default_rng(nblocks).integers(0, nb, 3))
    got = A[0, 0, blocks].cpu().numpy()
    assert np.abs(got.sum(-1) - 1).max() <= 1e-3
    ref = orc.block_mass_rows(x["q"], x["k"], 0, 0, blocks)
    assert np.abs(got - ref).max() <= 1e-4
