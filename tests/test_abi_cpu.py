"""CPU checks of the C ABI: the library loads, exports every function that
include/nabla.h declares, and its host-side logic (workspace sizing, argument
validation) behaves as documented.  Every call here fails validation before
any CUDA call is made, so no GPU is needed."""
import ctypes
import os
import re

import pytest

import block_sparse_attention_nabla_b200 as nabla

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nabla.h")

OK, INVALID, UNSUPPORTED, CUDA, TIMEOUT, WORKSPACE = range(6)
FAKE = 1 << 20          # a non-null, 256-byte aligned address never dereferenced here


def declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"NABLA_API\s+[\w\s\*]+?\b(nabla_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(nabla.LIB_PATH):
        from block_sparse_attention_nabla_b200 import build
        build.build()
    return nabla.lib()


def shape(B=1, H=2, S=1000, D=128, block=64, dtype=0):
    return nabla._Shape(B, H, S, D, block, dtype)


def mask_struct(**kw):
    m = dict(bits=FAKE, cnt=FAKE, idx=FAKE, cnt_t=None, idx_t=None, work=FAKE)
    m.update(kw)
    return nabla._Mask(m["bits"], m["cnt"], m["idx"], m["cnt_t"], m["idx_t"], m["work"])


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) == 20
    assert sorted(nabla.SYMBOLS) == names
    for n in names:
        assert hasattr(L, n), n


def test_abi_version(L):
    assert L.nabla_abi_version() == 3


def test_workspace_size_formula(L):
    def align(x):
        return (x + 255) // 256 * 256
    for (B, H, S, D) in [(1, 2, 4096, 64), (1, 40, 75600, 128), (2, 16, 16384, 128), (1, 1, 1, 64)]:
        nb = -(-S // 64)
        pooled = align(B * H * nb * D * 8)
        ldl = (nb + 3) // 4 * 4
        counters = align(B * H * 2 * 4)      # per-(b, h) hand-off counters of the builder's kernels
        fwd = 256 + counters + 2 * pooled + 4 * align(B * H * nb * D * 4) + align(B * H * nb * ldl * 4)
        assert L.nabla_workspace_size(ctypes.byref(shape(B, H, S, D)), 0) == fwd
        # backward: Delta [B, H, S] and the block-padded LSE2 / Delta [B, H, nb * 64]
        bwd = align(B * H * S * 4) + 2 * align(B * H * nb * 64 * 4)
        assert L.nabla_workspace_size(ctypes.byref(shape(B, H, S, D)), 1) == fwd + bwd


def test_workspace_size_rejects_bad_shapes(L):
    assert L.nabla_workspace_size(None, 0) == 0
    assert L.nabla_workspace_size(ctypes.byref(shape(D=96)), 0) == 0
    assert L.nabla_workspace_size(ctypes.byref(shape(block=32)), 0) == 0
    assert L.nabla_workspace_size(ctypes.byref(shape(S=0)), 0) == 0
    assert L.nabla_workspace_size(ctypes.byref(shape(S=64 * 8192 + 1)), 0) == 0


def _build(L, sh=None, q=FAKE, k=FAKE, thr=0.5, sta=None, m=None, ws=FAKE, ws_bytes=1 << 40):
    sh = sh or shape()
    m = m or mask_struct()
    return L.nabla_build_mask(ctypes.byref(sh), q, k, ctypes.c_float(thr),
                              ctypes.byref(sta) if sta is not None else None, ctypes.byref(m), ws,
                              ws_bytes, None)


def test_build_mask_argument_errors(L):
    assert _build(L, thr=0.0) == INVALID
    assert b"thr" in L.nabla_last_error()
    assert _build(L, thr=1.5) == INVALID
    assert _build(L, thr=float("nan")) == INVALID
    assert _build(L, q=None) == INVALID
    assert b"q is NULL" in L.nabla_last_error()
    assert _build(L, k=FAKE + 8) == INVALID            # not 16-byte aligned
    assert b"aligned" in L.nabla_last_error()
    assert _build(L, sh=shape(D=96)) == UNSUPPORTED
    assert _build(L, sh=shape(block=128)) == UNSUPPORTED
    assert _build(L, sh=shape(dtype=7)) == INVALID
    assert _build(L, sh=shape(S=-5)) == INVALID
    assert _build(L, m=mask_struct(work=None)) == INVALID
    assert _build(L, m=mask_struct(cnt_t=FAKE)) == INVALID     # cnt_t without idx_t
    assert _build(L, sta=nabla._Sta(FAKE, 3, 0, 3)) == INVALID
    assert b"STA" in L.nabla_last_error()
    assert _build(L, ws=None) == WORKSPACE
    assert _build(L, ws_bytes=100) == WORKSPACE
    assert b"needed" in L.nabla_last_error()
    assert _build(L, ws=FAKE + 16) == WORKSPACE         # workspace must be 256-byte aligned


def test_projection_argument_errors(L):
    def proj(sh=None, C=256, x=FAKE, wt=FAKE, q=FAKE, k=FAKE, v=FAKE, ws=FAKE, ws_bytes=1 << 40):
        return L.nabla_qkv_project(ctypes.byref(sh or shape()), C, x, wt, q, k, v, ws, ws_bytes, None)
    assert proj(C=0) == INVALID
    assert proj(C=100) == INVALID                        # not a multiple of 8
    assert b"multiple of 8" in L.nabla_last_error()
    assert proj(C=(1 << 20) + 8) == UNSUPPORTED
    assert proj(sh=shape(dtype=1)) == UNSUPPORTED        # the projection runs on the tensor cores: bf16
    assert b"bf16" in L.nabla_last_error()
    assert proj(sh=shape(D=96)) == UNSUPPORTED
    assert proj(x=None) == INVALID
    assert b"x is NULL" in L.nabla_last_error()
    assert proj(wt=FAKE + 8) == INVALID
    assert proj(v=None) == INVALID
    assert proj(ws=None) == WORKSPACE
    assert proj(ws_bytes=1000) == WORKSPACE
    big = 1 << 36                                        # far apart: no overlap
    assert proj(k=FAKE + 16, q=FAKE, v=FAKE + big, x=FAKE + 2 * big, wt=FAKE + 3 * big,
                ws=FAKE + 4 * big) == INVALID            # q and k overlap
    assert b"overlaps" in L.nabla_last_error()
    assert proj(q=FAKE + big, k=FAKE + 2 * big, v=FAKE + 3 * big, x=FAKE + 3 * big + 256,
                wt=FAKE + 5 * big, ws=FAKE + 6 * big) == INVALID   # v over x


def test_pooled_build_argument_errors(L):
    def build(sh=None, thr=0.5, sta=None, m=None, ws=FAKE, ws_bytes=1 << 40):
        return L.nabla_build_mask_pooled(ctypes.byref(sh or shape()), ctypes.c_float(thr),
                                         ctypes.byref(sta) if sta is not None else None,
                                         ctypes.byref(m or mask_struct()), ws, ws_bytes, None)
    assert build(thr=0.0) == INVALID
    assert build(thr=1.5) == INVALID
    assert build(m=mask_struct(bits=None)) == INVALID
    assert build(sta=nabla._Sta(FAKE, 0, 3, 3)) == INVALID
    assert build(sh=shape(D=96)) == UNSUPPORTED
    assert build(ws=None) == WORKSPACE
    assert build(ws_bytes=100) == WORKSPACE


def test_attention_argument_errors(L):
    sh, m = shape(), mask_struct()
    fwd = lambda **kw: L.nabla_attn_fwd(ctypes.byref(kw.get("sh", sh)), kw.get("q", FAKE), FAKE, FAKE,
                                        ctypes.byref(kw.get("m", m)), kw.get("o", FAKE), kw.get("o_res", None),
                                        kw.get("lse", FAKE), kw.get("ws", FAKE), kw.get("wsb", 1 << 40), None)
    assert fwd(o=None) == INVALID
    assert fwd(o_res=FAKE + 8) == INVALID                # misaligned residual
    assert fwd(o_res=FAKE, sh=shape(dtype=1)) == INVALID  # fp32 has no residual
    assert b"o_res" in L.nabla_last_error()
    assert fwd(lse=FAKE + 2) == INVALID
    assert fwd(sh=shape(D=32)) == UNSUPPORTED
    assert fwd(wsb=10) == WORKSPACE
    bwd = lambda **kw: L.nabla_attn_bwd(ctypes.byref(kw.get("sh", sh)), FAKE, FAKE, FAKE, FAKE,
                                        kw.get("o_res", None), FAKE, FAKE,
                                        ctypes.byref(kw.get("m", m)), FAKE, FAKE, kw.get("dv", FAKE),
                                        FAKE, kw.get("wsb", 1 << 40), None)
    assert bwd() == INVALID                              # forward-only mask: no transposed lists
    assert b"cnt_t" in L.nabla_last_error()
    full = mask_struct(cnt_t=FAKE, idx_t=FAKE)
    assert bwd(m=full, dv=None) == INVALID
    assert bwd(m=full, o_res=FAKE + 4) == INVALID
    assert bwd(m=full, o_res=FAKE, sh=shape(dtype=1)) == INVALID
    assert bwd(m=full, wsb=1000) == WORKSPACE
    # the tensor-core dK / dV walks the bitmask columns: bits are required
    assert bwd(m=mask_struct(cnt_t=FAKE, idx_t=FAKE, bits=None)) == INVALID
    assert b"bits" in L.nabla_last_error()


def test_mask_from_bits_and_status_argument_errors(L):
    sh = shape()
    assert L.nabla_mask_from_bits(ctypes.byref(sh), None, ctypes.byref(mask_struct()), FAKE, 1 << 40, None) == INVALID
    assert L.nabla_mask_from_bits(ctypes.byref(sh), FAKE, ctypes.byref(mask_struct(idx=None)), FAKE, 1 << 40, None) == INVALID
    assert L.nabla_workspace_status(None, None, None) == INVALID
    assert L.nabla_selftest_wait_timeout(None, 1000, None) == WORKSPACE
    assert L.nabla_selftest_wait_timeout(FAKE, 0, None) == INVALID
    assert L.nabla_selftest_wait_timeout(FAKE, 10**11, None) == INVALID


def test_last_error_is_per_call(L):
    assert _build(L, thr=0.0) == INVALID
    assert L.nabla_last_error() != b""
    assert L.nabla_workspace_size(ctypes.byref(shape()), 0) > 0   # does not touch the message
    assert _build(L, q=None) == INVALID
    assert b"thr" not in L.nabla_last_error()


def test_fractal_reorder_argument_errors(L):
    ok = dict(x=FAKE, y=FAKE + (1 << 30), B=1, T=2, H=3, W=5, P=2, row_bytes=32, inverse=0)

    def call(**kw):
        a = dict(ok, **kw)
        return L.nabla_fractal_reorder(a["x"], a["y"], a["B"], a["T"], a["H"], a["W"], a["P"], a["row_bytes"],
                                       a["inverse"], None)
    assert call(x=None) == INVALID
    assert call(y=FAKE + 8) == INVALID                 # misaligned
    assert call(y=FAKE + 64) == INVALID                # overlaps x
    assert call(P=0) == INVALID
    assert call(H=0) == INVALID
    assert call(row_bytes=24) == INVALID
    assert call(inverse=2) == INVALID
    assert b"inverse" in L.nabla_last_error()


def test_build_mask_topk_argument_errors(L):
    sh = shape()
    ms = mask_struct()
    assert L.nabla_build_mask_topk(ctypes.byref(sh), FAKE, FAKE, 0, None, ctypes.byref(ms), FAKE, 1 << 40, None) == INVALID
    assert b"topk" in L.nabla_last_error()
    assert L.nabla_build_mask_topk(ctypes.byref(sh), None, FAKE, 4, None, ctypes.byref(ms), FAKE, 1 << 40, None) == INVALID
    assert L.nabla_build_mask_topk(ctypes.byref(sh), FAKE, FAKE, 4, None, ctypes.byref(ms), None, 0, None) == WORKSPACE


def test_block_mass_and_recall_argument_errors(L):
    sh = shape()
    assert L.nabla_block_mass(ctypes.byref(sh), FAKE, FAKE, FAKE, None, 0, None) == WORKSPACE
    assert L.nabla_block_mass(ctypes.byref(sh), FAKE, None, FAKE, FAKE, 256, None) == INVALID
    sh32 = shape(dtype=1)
    assert L.nabla_block_mass(ctypes.byref(sh32), FAKE, FAKE, FAKE, FAKE, 256, None) == UNSUPPORTED
    assert L.nabla_mask_recall(ctypes.byref(sh), FAKE, None, FAKE, None) == INVALID
    assert L.nabla_mask_recall(ctypes.byref(sh), FAKE + 2, FAKE, FAKE, None) == INVALID


def test_build_sta_mask_argument_errors(L):
    sh = shape()
    ms = mask_struct()
    sta = nabla._Sta(FAKE, 3, 3, 3)
    assert L.nabla_build_sta_mask(ctypes.byref(sh), None, ctypes.byref(ms), None) == INVALID
    assert b"sta" in L.nabla_last_error()
    assert L.nabla_build_sta_mask(ctypes.byref(sh), ctypes.byref(nabla._Sta(None, 3, 3, 3)), ctypes.byref(ms),
                                  None) == INVALID
    assert L.nabla_build_sta_mask(ctypes.byref(sh), ctypes.byref(nabla._Sta(FAKE + 2, 3, 3, 3)), ctypes.byref(ms),
                                  None) == INVALID
    assert L.nabla_build_sta_mask(ctypes.byref(sh), ctypes.byref(nabla._Sta(FAKE, 3, 0, 3)), ctypes.byref(ms),
                                  None) == INVALID
    assert b"window" in L.nabla_last_error()
    assert L.nabla_build_sta_mask(ctypes.byref(sh), ctypes.byref(sta), ctypes.byref(mask_struct(bits=None)),
                                  None) == INVALID
    assert L.nabla_build_sta_mask(ctypes.byref(shape(block=32)), ctypes.byref(sta), ctypes.byref(ms), None) == UNSUPPORTED


def test_binding_refuses_sta_coordinates_of_the_wrong_shape():
    import torch
    nb = nabla.num_blocks(1000)
    with pytest.raises(nabla.NablaError, match=r"\[nb, 3\]"):
        nabla._sta_struct(torch.zeros(nb - 1, 3, dtype=torch.int32), (3, 3, 3), 1000)
    with pytest.raises(nabla.NablaError, match=r"\[nb, 3\]"):
        nabla._sta_struct(torch.zeros(nb, 2, dtype=torch.int32), (3, 3, 3), 1000)
    with pytest.raises(nabla.NablaError, match="sta_window"):
        nabla._sta_struct(torch.zeros(nb, 3, dtype=torch.int32), None, 1000)
    with pytest.raises(nabla.NablaError, match="CUDA"):     # right shape, but a host tensor
        nabla._sta_struct(torch.zeros(nb, 3, dtype=torch.int32), (3, 3, 3), 1000)
    assert nabla._sta_struct(None, None, 1000) is None


def test_binding_refuses_masks_and_outputs_of_another_shape():
    import torch
    m = nabla.Mask.empty(1, 2, 1000, "cpu", transpose=False)
    m.check(1, 2, 1000, "cpu")                                  # its own shape
    with pytest.raises(nabla.NablaError, match="mask.cnt"):
        m.check(1, 2, 2000, "cpu")                              # built for fewer blocks
    with pytest.raises(nabla.NablaError, match="mask.cnt_t is required"):
        m.check(1, 2, 1000, "cpu", need_transpose=True)         # the backward needs the transposed lists
    m.work = m.work[:-1]
    with pytest.raises(nabla.NablaError, match="mask.work"):
        m.check(1, 2, 1000, "cpu")
    with pytest.raises(nabla.NablaError, match="lse"):
        nabla._check_f32(torch.zeros(1, 2, 999), (1, 2, 1000), "cpu", "lse")
    with pytest.raises(nabla.NablaError, match="lse"):
        nabla._check_f32(torch.zeros(1, 2, 1000, dtype=torch.float64), (1, 2, 1000), "cpu", "lse")
    nabla._check_f32(torch.zeros(1, 2, 1000), (1, 2, 1000), "cpu", "lse")


# ------------------------------------------------ STA block coordinates (host)

def _lib_coords(L, T, H, W, P, S):
    import numpy as np
    nb = -(-S // 64)
    out = (ctypes.c_int32 * (3 * nb))()
    st = L.nabla_sta_block_coords(T, H, W, P, S, ctypes.cast(out, ctypes.c_void_p))
    return st, np.frombuffer(out, dtype=np.int32).reshape(nb, 3)


@pytest.mark.parametrize("T,H,W,P,S", [
    (21, 30, 52, 8, 32760),       # 480p latent
    (21, 45, 80, 8, 75600),       # 720p latent
    (21, 48, 80, 8, 80640),       # 720p with frames padded to 48 rows (Table 1 layout)
    (4, 32, 32, 8, 4096),         # tiny case
    (16, 32, 32, 8, 16384),       # pretraining shape
    (3, 12, 20, 8, 768),          # 720 tokens padded to 12 blocks
    (2, 7, 9, 4, 126),            # patches of 4, ragged on both sides
])
def test_sta_block_coords_matches_the_oracle(L, T, H, W, P, S):
    from oracle import nabla_oracle as orc
    st, got = _lib_coords(L, T, H, W, P, S)
    assert st == OK, L.nabla_last_error()
    assert (got == orc.block_tile_coords(T, H, W, P, S)).all()


def test_sta_block_coords_binding_and_errors(L):
    from oracle import nabla_oracle as orc
    c = nabla.sta_block_coords(21, 45, 80)
    assert c.dtype.is_floating_point is False and tuple(c.shape) == (1182, 3) and not c.is_cuda
    assert (c.numpy() == orc.block_tile_coords(21, 45, 80, 8)).all()
    buf = (ctypes.c_int32 * 30)()
    assert L.nabla_sta_block_coords(1, 12, 12, 8, 144, None) == INVALID
    assert L.nabla_sta_block_coords(0, 12, 12, 8, 144, ctypes.cast(buf, ctypes.c_void_p)) == INVALID
    assert L.nabla_sta_block_coords(1, 12, 12, 0, 144, ctypes.cast(buf, ctypes.c_void_p)) == INVALID
    # block 3 of S = 193 would start at token 192, past the 144 latent tokens
    assert L.nabla_sta_block_coords(1, 12, 12, 8, 193, ctypes.cast(buf, ctypes.c_void_p)) == INVALID
    assert b"past" in L.nabla_last_error()
    assert L.nabla_sta_block_coords(1, 12, 12, 8, 192, ctypes.cast(buf, ctypes.c_void_p)) == OK
    with pytest.raises(nabla.NablaError, match="S must be"):
        nabla.sta_block_coords(1, 12, 12, 8, 0)


def test_noalloc_entry_points_refuse_bad_arguments_like_the_workspace_builder(L):
    ms = mask_struct()
    for thr, q, sh, word in ((0.0, FAKE, shape(), b"thr"), (0.5, None, shape(), b"q is NULL"),
                             (0.5, FAKE, shape(D=96), b"head dimension"),
                             (0.5, FAKE, shape(S=64 * 8192 + 1), b"blocks")):
        a = L.nabla_build_mask_noalloc(ctypes.byref(sh), q, FAKE, ctypes.c_float(thr), None, ctypes.byref(ms), None)
        msg_a = L.nabla_last_error()
        b = _build(L, sh=sh, q=q, thr=thr)
        assert a == b and a != OK and word in msg_a and msg_a == L.nabla_last_error()
    assert L.nabla_build_mask_noalloc_status(None, None) == INVALID
