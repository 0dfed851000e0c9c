"""The mask builder entry point that allocates nothing.

Callers that cannot allocate device memory while they build a mask (a
serving process that reserved all memory up front, code that must not risk
the synchronisation an allocation can cause) call nabla_build_mask_noalloc,
whose scratch is a static array inside the library.  These tests check,
through the C ABI, that it gives exactly the mask of nabla_build_mask on two
calls in a row with different inputs, and that shapes too large for the
static scratch are refused with a clear message.

The file is named so that pytest collects it last."""
import ctypes

import pytest
import torch

import block_sparse_attention_nabla_b200 as nabla
import synth

pytestmark = pytest.mark.gpu


def _same_mask(a: nabla.Mask, b: nabla.Mask) -> None:
    assert torch.equal(a.bits, b.bits)
    assert torch.equal(a.cnt, b.cnt)
    assert torch.equal(a.work, b.work)
    n = a.cnt.cpu()
    ia, ib = a.idx.cpu(), b.idx.cpu()
    ta, tb, nt = a.idx_t.cpu(), b.idx_t.cpu(), a.cnt_t.cpu()
    assert torch.equal(a.cnt_t, b.cnt_t)
    B, H, nb = n.shape
    for bb in range(B):
        for h in range(H):
            for i in range(nb):
                c = int(n[bb, h, i])
                assert torch.equal(ia[bb, h, i, :c], ib[bb, h, i, :c])
                c = int(nt[bb, h, i])
                assert torch.equal(ta[bb, h, i, :c], tb[bb, h, i, :c])


def test_noalloc_mask_equals_workspace_mask_on_two_calls():
    w = synth.WORKLOADS[3].scaled(H=2)                 # 720p frames, 2 heads, STA on
    inputs = [synth.make_inputs(w), synth.make_inputs(w.scaled(seed=77))]
    coords = nabla.sta_block_coords(w.T, w.Hl, w.Wl, w.P).cuda()
    for x, thr in zip(inputs, (0.8, 0.5)):
        q, k = x["q"].cuda(), x["k"].cuda()
        ref = nabla.build_mask(q, k, thr, sta_coords=coords, sta_window=w.sta_window)
        got = nabla.build_mask_noalloc(q, k, thr, sta_coords=coords, sta_window=w.sta_window)
        torch.cuda.synchronize()
        _same_mask(got, ref)


def test_noalloc_mask_fp32_and_ragged_tail():
    x = synth.make_random_qkv(2, 3, 1000, 64, "fp32", seed=3)
    q, k = x["q"].cuda(), x["k"].cuda()
    for thr in (0.9, 0.3):
        ref = nabla.build_mask(q, k, thr)
        got = nabla.build_mask_noalloc(q, k, thr)
        torch.cuda.synchronize()
        _same_mask(got, ref)


def test_noalloc_rejects_shapes_beyond_the_static_scratch():
    sh = nabla._Shape(1, 40, 75600, 128, 64, 0)           # needs about 97 MB of scratch
    m = nabla._Mask(1 << 20, 1 << 20, 1 << 20, None, None, 1 << 20)
    st = nabla.lib().nabla_build_mask_noalloc(ctypes.byref(sh), 1 << 20, 1 << 20, ctypes.c_float(0.8),
                                              None, ctypes.byref(m), None)
    assert st == 2
    msg = nabla.lib().nabla_last_error().decode()
    assert "static scratch" in msg and str(32 << 20) in msg


def test_noalloc_status_reads_back_a_timeout_and_recovers():
    """The score GEMM's bounded waits report into the static scratch's status
    word, which nabla_build_mask_noalloc_status reads back: 0 after a normal
    call; with a 1 ns wait limit the first wait that is not already satisfied
    runs out and the word reads 4 (0 if every wait happened to be satisfied at
    once); the next call with the default limit is correct again."""
    x = synth.make_random_qkv(1, 4, 4096, 128, "bf16", seed=9)
    q, k = x["q"].cuda(), x["k"].cuda()
    ref = nabla.build_mask(q, k, 0.7)
    nabla.build_mask_noalloc(q, k, 0.7)
    assert nabla.build_mask_noalloc_status() == 0
    try:
        nabla.set_wait_limit_ns(1)
        nabla.build_mask_noalloc(q, k, 0.7)
        assert nabla.build_mask_noalloc_status() in (0, 4)
    finally:
        nabla.set_wait_limit_ns(0)
    got = nabla.build_mask_noalloc(q, k, 0.7)
    assert nabla.build_mask_noalloc_status() == 0
    _same_mask(got, ref)
