"""NABLA adaptive block-sparse attention for B200 (sm_100a).

Python binding of libnabla.so (include/nabla.h).  This module only marshals
arguments: it checks tensor shapes and dtypes, allocates outputs with torch
and passes raw device pointers and the current CUDA stream to the C ABI.  Every
step of the computation runs in the library's CUDA kernels; if the library is
missing or fails to load, every call raises NablaError.

    mask = build_mask(q, k, thr=0.8)            # Algorithm 1 (+ optional STA)
    o, lse = attn_fwd(q, k, v, mask)            # Eq. 4 over the kept tiles
    dq, dk, dv = attn_bwd(q, k, v, o, do, lse, mask)
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

__all__ = ["NablaError", "Mask", "build_mask", "mask_from_bits", "attn_fwd", "attn_bwd",
           "workspace", "workspace_size", "workspace_status", "set_wait_limit_ns", "lib",
           "selftest_wait_timeout", "build_mask_noalloc", "build_mask_noalloc_status", "fractal_reorder",
           "build_mask_topk", "block_mass", "mask_recall", "sta_block_coords", "qkv_project",
           "build_mask_pooled",
           "BLOCK", "BF16", "FP32"]

BLOCK = 64
BF16, FP32 = 0, 1
_DTYPES = {torch.bfloat16: BF16, torch.float32: FP32}
LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libnabla.so")

# Exported symbols, in the order include/nabla.h declares them.
SYMBOLS = ["nabla_workspace_size", "nabla_build_mask", "nabla_build_mask_topk", "nabla_build_mask_noalloc",
           "nabla_build_mask_noalloc_status", "nabla_qkv_project", "nabla_build_mask_pooled",
           "nabla_build_sta_mask", "nabla_sta_block_coords",
           "nabla_mask_from_bits", "nabla_attn_fwd",
           "nabla_attn_bwd", "nabla_block_mass", "nabla_mask_recall", "nabla_fractal_reorder", "nabla_selftest_wait_timeout", "nabla_workspace_status",
           "nabla_set_wait_limit_ns",
           "nabla_last_error", "nabla_abi_version"]


class NablaError(RuntimeError):
    pass


class _Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("S", ctypes.c_int32),
                ("D", ctypes.c_int32), ("block", ctypes.c_int32), ("dtype", ctypes.c_int32)]


class _Sta(ctypes.Structure):
    _fields_ = [("block_coords", ctypes.c_void_p), ("wT", ctypes.c_int32),
                ("wH", ctypes.c_int32), ("wW", ctypes.c_int32)]


class _Mask(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_void_p), ("cnt", ctypes.c_void_p), ("idx", ctypes.c_void_p),
                ("cnt_t", ctypes.c_void_p), ("idx_t", ctypes.c_void_p), ("work", ctypes.c_void_p)]


_lib = None


def lib() -> ctypes.CDLL:
    """Loads libnabla.so (once) and declares the C signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise NablaError(f"{LIB_PATH} is missing; build it with "
                         "`python -m block_sparse_attention_nabla_b200.build`")
    try:
        L = ctypes.CDLL(LIB_PATH)
    except OSError as e:
        raise NablaError(f"cannot load {LIB_PATH}: {e}") from e
    P, I32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    SH, ST, MK = ctypes.POINTER(_Shape), ctypes.POINTER(_Sta), ctypes.POINTER(_Mask)
    L.nabla_workspace_size.argtypes, L.nabla_workspace_size.restype = [SH, I32], SZ
    L.nabla_build_mask.argtypes = [SH, P, P, ctypes.c_float, ST, MK, P, SZ, P]
    L.nabla_build_mask_topk.argtypes = [SH, P, P, I32, ST, MK, P, SZ, P]
    L.nabla_mask_from_bits.argtypes = [SH, P, MK, P, SZ, P]
    L.nabla_build_sta_mask.argtypes = [SH, ST, MK, P]
    L.nabla_build_mask_noalloc.argtypes = [SH, P, P, ctypes.c_float, ST, MK, P]
    L.nabla_build_mask_noalloc_status.argtypes = [ctypes.POINTER(I32), P]
    L.nabla_sta_block_coords.argtypes = [I32, I32, I32, I32, I32, P]
    L.nabla_qkv_project.argtypes = [SH, I32, P, P, P, P, P, P, SZ, P]
    L.nabla_build_mask_pooled.argtypes = [SH, ctypes.c_float, ST, MK, P, SZ, P]
    L.nabla_attn_fwd.argtypes = [SH, P, P, P, MK, P, P, P, P, SZ, P]
    L.nabla_attn_bwd.argtypes = [SH, P, P, P, P, P, P, P, MK, P, P, P, P, SZ, P]
    L.nabla_fractal_reorder.argtypes = [P, P, I32, I32, I32, I32, I32, SZ, I32, P]
    L.nabla_block_mass.argtypes = [SH, P, P, P, P, SZ, P]
    L.nabla_mask_recall.argtypes = [SH, P, P, P, P]
    L.nabla_workspace_status.argtypes = [P, ctypes.POINTER(I32), P]
    L.nabla_selftest_wait_timeout.argtypes = [P, ctypes.c_uint64, P]
    L.nabla_set_wait_limit_ns.argtypes, L.nabla_set_wait_limit_ns.restype = [ctypes.c_uint64], None
    L.nabla_last_error.argtypes, L.nabla_last_error.restype = [], ctypes.c_char_p
    L.nabla_abi_version.argtypes, L.nabla_abi_version.restype = [], I32
    for name in ("nabla_build_mask", "nabla_build_mask_topk", "nabla_build_mask_noalloc", "nabla_mask_from_bits",
                 "nabla_build_mask_noalloc_status", "nabla_qkv_project", "nabla_build_mask_pooled",
                 "nabla_build_sta_mask", "nabla_sta_block_coords",
                 "nabla_attn_fwd", "nabla_attn_bwd", "nabla_fractal_reorder", "nabla_block_mass",
                 "nabla_mask_recall",
                 "nabla_workspace_status", "nabla_selftest_wait_timeout"):
        getattr(L, name).restype = I32
    _lib = L
    return L


def _check(status: int, what: str) -> None:
    if status != 0:
        msg = lib().nabla_last_error().decode(errors="replace")
        raise NablaError(f"{what} failed with status {status}: {msg}")


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _shape_of(q: torch.Tensor) -> _Shape:
    if q.dim() != 4:
        raise NablaError(f"expected [B, H, S, D], got shape {tuple(q.shape)}")
    if q.dtype not in _DTYPES:
        raise NablaError(f"dtype must be bfloat16 or float32, got {q.dtype}")
    if not q.is_cuda:
        raise NablaError("tensors must be CUDA tensors")
    B, H, S, D = q.shape
    return _Shape(B, H, S, D, BLOCK, _DTYPES[q.dtype])


def _same(ref: torch.Tensor, *ts: torch.Tensor) -> None:
    for t in ts:
        if t.shape != ref.shape or t.dtype != ref.dtype or t.device != ref.device:
            raise NablaError(f"tensor {tuple(t.shape)} {t.dtype} does not match {tuple(ref.shape)} {ref.dtype}")
        if not t.is_contiguous():
            raise NablaError("tensors must be contiguous")


def _check_f32(t: torch.Tensor, shape: tuple, device, name: str) -> None:
    if tuple(t.shape) != tuple(shape) or t.dtype != torch.float32 or t.device != torch.device(device) \
            or not t.is_contiguous():
        raise NablaError(f"{name} must be a contiguous float32 tensor {list(shape)} on {device} "
                         f"(got {list(t.shape)} {t.dtype} {t.device})")


def num_blocks(S: int) -> int:
    return -(-S // BLOCK)


@dataclass
class Mask:
    """Device-side mask of one problem (layout in include/nabla.h)."""
    bits: torch.Tensor           # uint32 words as int32 [B, H, nb, W]
    cnt: torch.Tensor            # int32 [B, H, nb]
    idx: torch.Tensor            # int32 [B, H, nb, nb]
    work: torch.Tensor           # int32 [B * H * npairs, 2]
    cnt_t: torch.Tensor | None = None
    idx_t: torch.Tensor | None = None

    def check(self, B: int, H: int, S: int, device, need_bits: bool = True, need_transpose: bool = False) -> None:
        """Refuses tensors that do not have this problem's shapes: the kernels
        index them by the shape alone."""
        nb = num_blocks(S)
        W, npairs = -(-nb // 32), -(-nb // 2)
        want = {"cnt": (B, H, nb), "idx": (B, H, nb, nb), "work": (B * H * npairs, 2)}
        if need_bits:
            want["bits"] = (B, H, nb, W)
        if need_transpose or self.cnt_t is not None or self.idx_t is not None:
            want["cnt_t"], want["idx_t"] = (B, H, nb), (B, H, nb, nb)
        for name, shape in want.items():
            t = getattr(self, name)
            if t is None:
                raise NablaError(f"mask.{name} is required")
            if (tuple(t.shape) != shape or t.dtype != torch.int32 or t.device != torch.device(device)
                    or not t.is_contiguous()):
                raise NablaError(f"mask.{name} must be a contiguous int32 tensor {list(shape)} on {device} "
                                 f"(got {list(t.shape)} {t.dtype} {t.device})")

    def as_struct(self) -> _Mask:
        return _Mask(_ptr(self.bits), _ptr(self.cnt), _ptr(self.idx), _ptr(self.cnt_t),
                     _ptr(self.idx_t), _ptr(self.work))

    @staticmethod
    def empty(B: int, H: int, S: int, device, transpose: bool = True) -> "Mask":
        nb = num_blocks(S)
        W, npairs = -(-nb // 32), -(-nb // 2)
        i32 = dict(dtype=torch.int32, device=device)
        return Mask(bits=torch.empty(B, H, nb, W, **i32), cnt=torch.empty(B, H, nb, **i32),
                    idx=torch.empty(B, H, nb, nb, **i32), work=torch.empty(B * H * npairs, 2, **i32),
                    cnt_t=torch.empty(B, H, nb, **i32) if transpose else None,
                    idx_t=torch.empty(B, H, nb, nb, **i32) if transpose else None)

    def dense(self) -> torch.Tensor:
        """bool [B, H, nb, nb] view of the bitmask (host-side convenience)."""
        nb = self.cnt.shape[-1]
        b = self.bits.to(torch.int64) & 0xFFFFFFFF
        shifts = torch.arange(32, device=b.device)
        m = ((b[..., None] >> shifts) & 1).bool()
        return m.flatten(-2)[..., :nb]


def workspace_size(q_shape, dtype=torch.bfloat16, want_bwd: bool = False) -> int:
    B, H, S, D = q_shape
    sh = _Shape(B, H, S, D, BLOCK, _DTYPES[dtype])
    n = lib().nabla_workspace_size(ctypes.byref(sh), int(want_bwd))
    if n == 0:
        raise NablaError(f"invalid shape {tuple(q_shape)}")
    return n


def workspace(q: torch.Tensor, want_bwd: bool = False) -> torch.Tensor:
    n = workspace_size(tuple(q.shape), q.dtype, want_bwd)
    return torch.empty(n, dtype=torch.uint8, device=q.device)


def _sta_struct(sta_coords: torch.Tensor | None, sta_window, S: int):
    """The C struct for an STA window, or None.  The kernels read nb x 3 int32
    coordinates, so anything else is refused here rather than read past."""
    if sta_coords is None:
        return None
    if sta_window is None:
        raise NablaError("sta_window is required with sta_coords")
    nb = num_blocks(S)
    if tuple(sta_coords.shape) != (nb, 3):
        raise NablaError(f"sta_coords must have shape [nb, 3] = [{nb}, 3] (got {list(sta_coords.shape)})")
    if len(sta_window) != 3:
        raise NablaError("sta_window must be (wT, wH, wW) in tiles")
    if sta_coords.dtype != torch.int32 or not sta_coords.is_cuda or not sta_coords.is_contiguous():
        raise NablaError("sta_coords must be a contiguous int32 CUDA tensor [nb, 3]")
    return _Sta(sta_coords.data_ptr(), *[int(w) for w in sta_window])


def build_mask(q: torch.Tensor, k: torch.Tensor, thr: float, sta_coords: torch.Tensor | None = None,
               sta_window: tuple | None = None, out: Mask | None = None, ws: torch.Tensor | None = None,
               transpose: bool = True) -> Mask:
    """NABLA mask (Algorithm 1, plus the STA union when sta_coords/sta_window are given)."""
    sh = _shape_of(q)
    _same(q, k)
    out = out or Mask.empty(sh.B, sh.H, sh.S, q.device, transpose)
    out.check(sh.B, sh.H, sh.S, q.device)
    ws = ws if ws is not None else workspace(q)
    sta = _sta_struct(sta_coords, sta_window, sh.S)
    ms = out.as_struct()
    _check(lib().nabla_build_mask(ctypes.byref(sh), q.data_ptr(), k.data_ptr(), ctypes.c_float(thr),
                                  ctypes.byref(sta) if sta is not None else None, ctypes.byref(ms),
                                  ws.data_ptr(), ws.numel(), _stream()), "nabla_build_mask")
    return out


def build_mask_topk(q: torch.Tensor, k: torch.Tensor, topk: int, sta_coords: torch.Tensor | None = None,
                    sta_window: tuple | None = None, out: Mask | None = None, ws: torch.Tensor | None = None,
                    transpose: bool = True) -> Mask:
    """Fixed-budget comparator of build_mask: every row keeps its topk largest
    reduced-map entries (plus the STA union when given)."""
    sh = _shape_of(q)
    _same(q, k)
    out = out or Mask.empty(sh.B, sh.H, sh.S, q.device, transpose)
    out.check(sh.B, sh.H, sh.S, q.device)
    ws = workspace(q) if ws is None else ws
    sta = _sta_struct(sta_coords, sta_window, sh.S)
    ms = out.as_struct()
    _check(lib().nabla_build_mask_topk(ctypes.byref(sh), q.data_ptr(), k.data_ptr(), int(topk),
                                       ctypes.byref(sta) if sta is not None else None, ctypes.byref(ms),
                                       ws.data_ptr(), ws.numel(), _stream()), "nabla_build_mask_topk")
    return out


def build_mask_noalloc(q: torch.Tensor, k: torch.Tensor, thr: float,
                       sta_coords: torch.Tensor | None = None, sta_window: tuple | None = None,
                       out: Mask | None = None, transpose: bool = True) -> Mask:
    """Same mask as build_mask without a workspace: the library's static
    scratch is used instead, so no device memory is allocated for scratch
    (pass `out` to allocate nothing at all).  Calls must not overlap on the
    GPU; shapes whose scratch exceeds 32 MiB are rejected."""
    sh = _shape_of(q)
    _same(q, k)
    out = out or Mask.empty(sh.B, sh.H, sh.S, q.device, transpose)
    out.check(sh.B, sh.H, sh.S, q.device)
    sta = _sta_struct(sta_coords, sta_window, sh.S)
    ms = out.as_struct()
    _check(lib().nabla_build_mask_noalloc(ctypes.byref(sh), q.data_ptr(), k.data_ptr(),
                                          ctypes.c_float(thr),
                                          ctypes.byref(sta) if sta is not None else None,
                                          ctypes.byref(ms), _stream()), "nabla_build_mask_noalloc")
    return out


def build_mask_noalloc_status() -> int:
    """Status word of build_mask_noalloc's static scratch on the current device
    (0 = ok, 4 = a bounded wait of the last call ran out); synchronises the
    current stream."""
    out = ctypes.c_int32(-1)
    _check(lib().nabla_build_mask_noalloc_status(ctypes.byref(out), _stream()),
           "nabla_build_mask_noalloc_status")
    return out.value


def qkv_project(x: torch.Tensor, wt: torch.Tensor, H: int, D: int, q: torch.Tensor | None = None,
                k: torch.Tensor | None = None, v: torch.Tensor | None = None,
                ws: torch.Tensor | None = None):
    """Eq. 1: Q = X W_Q, K = X W_K, V = X W_V from hidden states x [B, S, C]
    and the transposed weights wt [3, H * D, C] (bf16 CUDA tensors), with the
    block means of Q and K written into the workspace on the way.  Returns
    (q, k, v, ws); build_mask_pooled(q.shape, thr, ws) then builds the mask
    from those means without reading q and k."""
    if x.dim() != 3 or wt.dim() != 3:
        raise NablaError("x must be [B, S, C] and wt [3, H * D, C]")
    B, S, C = x.shape
    if tuple(wt.shape) != (3, H * D, C):
        raise NablaError(f"wt must be [3, {H * D}, {C}], got {list(wt.shape)}")
    for t, name in ((x, "x"), (wt, "wt")):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise NablaError(f"{name} must be a contiguous bf16 CUDA tensor")
    outs = []
    for t in (q, k, v):
        t = torch.empty(B, H, S, D, dtype=torch.bfloat16, device=x.device) if t is None else t
        if tuple(t.shape) != (B, H, S, D) or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise NablaError(f"q, k, v must be contiguous bf16 [{B}, {H}, {S}, {D}]")
        outs.append(t)
    sh = _shape_of(outs[0])
    ws = workspace(outs[0]) if ws is None else ws
    _check(lib().nabla_qkv_project(ctypes.byref(sh), int(C), x.data_ptr(), wt.data_ptr(), outs[0].data_ptr(),
                                   outs[1].data_ptr(), outs[2].data_ptr(), ws.data_ptr(), ws.numel(), _stream()),
           "nabla_qkv_project")
    return outs[0], outs[1], outs[2], ws


def build_mask_pooled(q_shape, thr: float, ws: torch.Tensor, sta_coords: torch.Tensor | None = None,
                      sta_window: tuple | None = None, out: Mask | None = None, transpose: bool = True,
                      dtype=torch.bfloat16) -> Mask:
    """build_mask from the block means qkv_project left in ws (no read of Q, K)."""
    B, H, S, D = (int(x) for x in q_shape)
    if dtype not in _DTYPES:
        raise NablaError("dtype must be bfloat16 or float32")
    sh = _Shape(B, H, S, D, BLOCK, _DTYPES[dtype])
    out = out or Mask.empty(B, H, S, ws.device, transpose)
    out.check(B, H, S, ws.device)
    sta = _sta_struct(sta_coords, sta_window, S)
    ms = out.as_struct()
    _check(lib().nabla_build_mask_pooled(ctypes.byref(sh), ctypes.c_float(thr),
                                         ctypes.byref(sta) if sta is not None else None, ctypes.byref(ms),
                                         ws.data_ptr(), ws.numel(), _stream()), "nabla_build_mask_pooled")
    return out


def sta_block_coords(T: int, H: int, W: int, P: int = 8, S: int | None = None) -> torch.Tensor:
    """STA tile coordinates (t, y // P, x // P) of the first token of every
    64-token block of a T x H x W latent in the token order of §3.1.1, as a CPU
    int32 tensor [ceil(S / 64), 3] (S defaults to T * H * W).  Move it to the
    device for the sta_coords argument of build_mask / build_sta_mask."""
    S = T * H * W if S is None else int(S)
    if S < 1:
        raise NablaError(f"S must be >= 1 (got {S})")
    out = torch.empty(num_blocks(S), 3, dtype=torch.int32)
    _check(lib().nabla_sta_block_coords(int(T), int(H), int(W), int(P), S, out.data_ptr()),
           "nabla_sta_block_coords")
    return out


def build_sta_mask(q_shape, sta_coords: torch.Tensor, sta_window: tuple, dtype=torch.bfloat16,
                   out: Mask | None = None, transpose: bool = True) -> Mask:
    """Sliding-tile (STA) mask alone, the same for every (b, h): query block i
    keeps key block j iff j lies in the window (in tiles) centred on i."""
    B, H, S, D = q_shape
    sh = _Shape(B, H, S, D, BLOCK, _DTYPES[dtype])
    if sta_coords is None:
        raise NablaError("sta_coords is required")
    sta = _sta_struct(sta_coords, sta_window, S)
    out = out or Mask.empty(B, H, S, sta_coords.device, transpose)
    out.check(B, H, S, sta_coords.device)
    ms = out.as_struct()
    _check(lib().nabla_build_sta_mask(ctypes.byref(sh), ctypes.byref(sta), ctypes.byref(ms), _stream()),
           "nabla_build_sta_mask")
    return out


def mask_from_bits(bits: torch.Tensor, q_shape, dtype=torch.bfloat16, out: Mask | None = None,
                   ws: torch.Tensor | None = None, transpose: bool = True) -> Mask:
    """Index lists and work list for an externally supplied bitmask [B, H, nb, W]."""
    B, H, S, D = q_shape
    sh = _Shape(B, H, S, D, BLOCK, _DTYPES[dtype])
    bits = bits.to(torch.int32).contiguous()
    out = out or Mask.empty(B, H, S, bits.device, transpose)
    out.bits = bits
    out.check(B, H, S, bits.device)
    if ws is None:
        ws = torch.empty(workspace_size(q_shape, dtype), dtype=torch.uint8, device=bits.device)
    ms = out.as_struct()
    _check(lib().nabla_mask_from_bits(ctypes.byref(sh), bits.data_ptr(), ctypes.byref(ms),
                                      ws.data_ptr(), ws.numel(), _stream()), "nabla_mask_from_bits")
    return out


def block_mass(q: torch.Tensor, k: torch.Tensor, out: torch.Tensor | None = None,
               ws: torch.Tensor | None = None) -> torch.Tensor:
    """True token-level attention mass of every 64 x 64 block of dense attention,
    float [B, H, nb, nb] (rows sum to 1)."""
    sh = _shape_of(q)
    _same(q, k)
    nb = num_blocks(sh.S)
    out = torch.empty(sh.B, sh.H, nb, nb, dtype=torch.float32, device=q.device) if out is None else out
    _check_f32(out, (sh.B, sh.H, nb, nb), q.device, "out")
    ws = torch.zeros(256, dtype=torch.uint8, device=q.device) if ws is None else ws
    _check(lib().nabla_block_mass(ctypes.byref(sh), q.data_ptr(), k.data_ptr(), out.data_ptr(), ws.data_ptr(),
                                  ws.numel(), _stream()), "nabla_block_mass")
    return out


def mask_recall(mass: torch.Tensor, mask: Mask, q_shape, dtype=torch.bfloat16) -> torch.Tensor:
    """Kept token-level mass of every query block under `mask`, float [B, H, nb]."""
    B, H, S, D = q_shape
    sh = _Shape(B, H, S, D, BLOCK, _DTYPES[dtype])
    nb = num_blocks(S)
    _check_f32(mass, (B, H, nb, nb), mass.device, "mass")
    if mask.bits is None or tuple(mask.bits.shape) != (B, H, nb, -(-nb // 32)) or mask.bits.dtype != torch.int32 \
            or mask.bits.device != mass.device or not mask.bits.is_contiguous():
        raise NablaError(f"mask.bits must be a contiguous int32 tensor [{B}, {H}, {nb}, {-(-nb // 32)}] "
                         f"on {mass.device}")
    rec = torch.empty(mass.shape[:-1], dtype=torch.float32, device=mass.device)
    _check(lib().nabla_mask_recall(ctypes.byref(sh), mass.data_ptr(), mask.bits.data_ptr(), rec.data_ptr(),
                                   _stream()), "nabla_mask_recall")
    return rec


def fractal_reorder(x: torch.Tensor, T: int, H: int, W: int, P: int = 8, inverse: bool = False,
                    out: torch.Tensor | None = None) -> torch.Tensor:
    """Fractal token reordering of §3.1.1 on x [B, T*H*W, ...] (raster -> fractal
    order; inverse=True: fractal -> raster).  Rows are moved as bytes."""
    if not x.is_cuda or not x.is_contiguous():
        raise NablaError("x must be a contiguous CUDA tensor")
    B, S = x.shape[0], x.shape[1]
    if S != T * H * W:
        raise NablaError(f"x has {S} tokens, T * H * W = {T * H * W}")
    out = torch.empty_like(x) if out is None else out
    _same(x, out)
    row_bytes = x[0, 0].numel() * x.element_size()
    _check(lib().nabla_fractal_reorder(x.data_ptr(), out.data_ptr(), B, T, H, W, P, row_bytes,
                                       1 if inverse else 0, _stream()), "nabla_fractal_reorder")
    return out


def attn_fwd(q, k, v, mask: Mask, o=None, lse=None, ws=None, o_res=None):
    """Block-sparse attention forward; returns (o, lse).  Pass o_res (a bf16
    tensor shaped like q) to also get the rounding residual of o, for training:
    attn_bwd then takes rowsum(dO * O) from o + o_res."""
    sh = _shape_of(q)
    _same(q, k, v)
    o = o if o is not None else torch.empty_like(q)
    lse = lse if lse is not None else torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    _same(q, o)
    if o_res is not None:
        _same(q, o_res)
    _check_f32(lse, tuple(q.shape[:3]), q.device, "lse")
    mask.check(sh.B, sh.H, sh.S, q.device)
    ws = ws if ws is not None else workspace(q)
    ms = mask.as_struct()
    _check(lib().nabla_attn_fwd(ctypes.byref(sh), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                ctypes.byref(ms), o.data_ptr(), _ptr(o_res), lse.data_ptr(), ws.data_ptr(),
                                ws.numel(), _stream()), "nabla_attn_fwd")
    return o, lse


def attn_bwd(q, k, v, o, do, lse, mask: Mask, ws=None, dq=None, dk=None, dv=None, o_res=None):
    """Backward of attn_fwd under the same mask; returns (dq, dk, dv).  o_res:
    the forward's residual of o, if it wrote one."""
    sh = _shape_of(q)
    _same(q, k, v, o, do)
    if o_res is not None:
        _same(q, o_res)
    dq = dq if dq is not None else torch.empty_like(q)
    dk = dk if dk is not None else torch.empty_like(k)
    dv = dv if dv is not None else torch.empty_like(v)
    _same(q, dq, dk, dv)
    _check_f32(lse, tuple(q.shape[:3]), q.device, "lse")
    mask.check(sh.B, sh.H, sh.S, q.device, need_transpose=True)
    ws = ws if ws is not None else workspace(q, want_bwd=True)
    ms = mask.as_struct()
    _check(lib().nabla_attn_bwd(ctypes.byref(sh), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                o.data_ptr(), _ptr(o_res), do.data_ptr(), lse.data_ptr(), ctypes.byref(ms),
                                dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ws.data_ptr(),
                                ws.numel(), _stream()), "nabla_attn_bwd")
    return dq, dk, dv


def workspace_status(ws: torch.Tensor) -> int:
    """Device status word of a workspace (0 = ok, 4 = a bounded wait ran out)."""
    out = ctypes.c_int32(-1)
    _check(lib().nabla_workspace_status(ws.data_ptr(), ctypes.byref(out), _stream()),
           "nabla_workspace_status")
    return out.value


def selftest_wait_timeout(ws: torch.Tensor, limit_ns: int) -> int:
    """Runs the bounded-wait self-test kernel and returns the status word it
    leaves (4 = NABLA_ERR_TIMEOUT is the expected outcome)."""
    _check(lib().nabla_selftest_wait_timeout(ws.data_ptr(), int(limit_ns), _stream()),
           "nabla_selftest_wait_timeout")
    return workspace_status(ws)


def set_wait_limit_ns(ns: int) -> None:
    lib().nabla_set_wait_limit_ns(int(ns))
