"""Plants plausible mistakes in the oracle (CPU only) and checks that the pins
in test_oracle_pins.py catch every one of them: a wrong sort direction, a
strict comparison, an exclusive cumulative sum, thr for 1 - thr, a missing
order restoration, a tail block divided by 64, transposed or unscaled scores,
softmax over the wrong axis, a wrong STA half-width, a transposed block mask,
a dropped term in the backward pass, a fractal order with tokens or
patches taken column-major or edge patches moved to the end of the frame, and
an Eq. 1 projection with heads and dimensions swapped, one weight for Q, K and
V, or the stored weight read untransposed."""
import numpy as np
import pytest

from oracle import nabla_oracle as orc
from tests import test_oracle_pins as pins

_ORIG_ATTN = orc.masked_attention


def _all_pins():
    checks = []
    for case in pins._read_golden("cdf_select_cases.txt"):
        checks.append(lambda c=case: pins.test_cdf_hand_cases(c))
    for case in pins._read_golden("sta_table1.txt"):
        checks.append(lambda c=case: pins.test_sta_reproduces_table1_sparsity(c))
    for case in pins._read_golden("topk_select_cases.txt"):
        checks.append(lambda c=case: pins.test_topk_hand_cases(c))
    for case in pins._read_golden("fractal_order_cases.txt"):
        checks.append(lambda c=case: pins.test_fractal_order_hand_cases(c))
    for args in [(3, 30, 52, 8), (2, 45, 80, 8), (1, 7, 9, 4), (4, 8, 8, 8)]:
        checks.append(lambda a=args: pins.test_fractal_order_is_a_framewise_bijection_with_contiguous_patches(*a))
    for case in pins._read_golden("block_coords_cases.txt"):
        checks.append(lambda c=case: pins.test_block_tile_coords_hand_cases(c))
    for args in [(21, 6, 10), (4, 4, 4), (16, 4, 4)]:
        checks.append(lambda a=args: pins.test_block_tile_coords_full_patch_grids_are_the_tile_grid(*a))
    for args in [(21, 30, 52), (21, 45, 80), (3, 12, 20)]:
        checks.append(lambda a=args: pins.test_block_tile_coords_invariants(*a))
    for name in dir(pins):
        fn = getattr(pins, name)
        if name.startswith("test_") and callable(fn) and name not in (
                "test_cdf_hand_cases", "test_sta_reproduces_table1_sparsity", "test_fractal_order_hand_cases",
                "test_topk_hand_cases",
                "test_fractal_order_is_a_framewise_bijection_with_contiguous_patches",
                "test_block_tile_coords_hand_cases", "test_block_tile_coords_full_patch_grids_are_the_tile_grid",
                "test_block_tile_coords_invariants"):
            checks.append(fn)
    return checks


def _some_pin_fails():
    for check in _all_pins():
        try:
            check()
        except (AssertionError, ValueError, IndexError):
            return True
    return False


def _cdf_variant(descending=False, strict=False, exclusive=False, use_thr=False, no_reorder=False):
    def f(A, thr):
        lim = float(np.float32(thr)) if use_thr else 1.0 - float(np.float32(thr))
        order = np.argsort(-A if descending else A, axis=-1, kind="stable")
        vals = np.take_along_axis(A, order, axis=-1)
        c = np.cumsum(vals, axis=-1)
        if exclusive:
            c = c - vals
        keep = c > lim if strict else c >= lim
        M = np.zeros(A.shape, dtype=bool)
        C = np.zeros(A.shape)
        if no_reorder:
            M[...] = keep
            C[...] = c
        else:
            np.put_along_axis(M, order, keep, axis=-1)
            np.put_along_axis(C, order, c, axis=-1)
        return M, C
    return f


def _pool_div64(X, N=64):
    S = X.shape[-2]
    nb = orc.num_blocks(S, N)
    return np.stack([X[..., i * N:min(i * N + N, S), :].sum(-2) / N for i in range(nb)], -2)


def _sta_full_width(coords, window):
    c = np.asarray(coords, dtype=np.int64)
    d = np.abs(c[:, None, :] - c[None, :, :])
    return np.all(d <= np.array(window)[None, None, :], axis=-1)


def _attn_unscaled(Q, K, V, M, N=64):
    D = np.asarray(orc.as_f64(Q)).shape[-1]
    return _ORIG_ATTN(orc.as_f64(Q) * np.sqrt(D), K, V, M, N)


def _attn_transposed_mask(Q, K, V, M, N=64):
    return _ORIG_ATTN(Q, K, V, np.swapaxes(M, -1, -2), N)


def _bwd_no_rowsum(Q, K, V, dO, M, N=64, ds_bound=False, ds_format=None):
    Q, K, V, dO = (orc.as_f64(x) for x in (Q, K, V, dO))
    B, H, S, D = Q.shape
    dQ, dK, dV = np.zeros_like(Q), np.zeros_like(K), np.zeros_like(V)
    bQ, bK = np.zeros_like(Q), np.zeros_like(K)
    for b in range(B):
        for h in range(H):
            for i in range(orc.num_blocks(S, N)):
                rows = slice(i * N, min(i * N + N, S))
                keys = orc._allowed_keys(M[b, h, i], S, N)
                lg = Q[b, h, rows] @ K[b, h, keys].T / np.sqrt(D)
                e = np.exp(lg - lg.max(-1, keepdims=True))
                P = e / e.sum(-1, keepdims=True)
                dV[b, h, keys] += P.T @ dO[b, h, rows]
                dS = P * (dO[b, h, rows] @ V[b, h, keys].T)
                dSm = orc.round_bf16(dS) if ds_format == "bf16" else dS
                dQ[b, h, rows] = dSm @ K[b, h, keys] / np.sqrt(D)
                dK[b, h, keys] += dSm.T @ Q[b, h, rows] / np.sqrt(D)
                bQ[b, h, rows] = np.abs(dS) @ np.abs(K[b, h, keys]) / np.sqrt(D)
                bK[b, h, keys] += np.abs(dS).T @ np.abs(Q[b, h, rows]) / np.sqrt(D)
    return (dQ, dK, dV, bQ, bK) if ds_bound else (dQ, dK, dV)


def _fractal_variant(col_major_tokens=False, col_major_patches=False, edges_last=False):
    def f(T, Hl, Wl, P=8):
        order = []
        for t in range(T):
            frame, tail = [], []
            patches = [(py, px) for py in range(0, Hl, P) for px in range(0, Wl, P)]
            if col_major_patches:
                patches = [(py, px) for px in range(0, Wl, P) for py in range(0, Hl, P)]
            for py, px in patches:
                toks = [(y, x) for y in range(py, min(py + P, Hl)) for x in range(px, min(px + P, Wl))]
                if col_major_tokens:
                    toks = [(y, x) for x in range(px, min(px + P, Wl)) for y in range(py, min(py + P, Hl))]
                full = py + P <= Hl and px + P <= Wl
                (frame if full or not edges_last else tail).extend(toks)
            order += [(t * Hl + y) * Wl + x for y, x in frame + tail]
        return np.asarray(order, dtype=np.int64)
    return f


def _topk_variant(ties_low_first=False, smallest=False, one_more=False):
    def f(A, k):
        nb = A.shape[-1]
        k = min(max(int(k), 1), nb) + (1 if one_more else 0)
        k = min(k, nb)
        order = np.argsort(-A, axis=-1, kind="stable") if ties_low_first else np.argsort(A, axis=-1, kind="stable")[..., ::-1]
        if smallest:
            order = np.argsort(A, axis=-1, kind="stable")
        M = np.zeros(A.shape, dtype=bool)
        np.put_along_axis(M, order[..., :k], True, axis=-1)
        return M
    return f


_ORIG_MASS = orc.block_mass


def _mass_rows_summed(Q, K, N=64):
    A = _ORIG_MASS(Q, K, N)
    S = np.asarray(orc.as_f64(Q)).shape[-2]
    n = np.array([min(N, S - i * N) for i in range(A.shape[-1])], dtype=float)
    return A * n[:, None]


def _mass_transposed(Q, K, N=64):
    return np.swapaxes(_ORIG_MASS(Q, K, N), -1, -2)


def _mass_unscaled(Q, K, N=64):
    D = np.asarray(orc.as_f64(Q)).shape[-1]
    return _ORIG_MASS(orc.as_f64(Q) * np.sqrt(D), K, N)


def _coords_variant(last_token=False, xy_swapped=False):
    def f(T, Hl, Wl, P=8, S=None, N=64):
        order = orc.fractal_order(T, Hl, Wl, P)
        S = len(order) if S is None else S
        nb = -(-S // N)
        out = np.empty((nb, 3), dtype=np.int64)
        for i in range(nb):
            r = int(order[min(i * N + N - 1, len(order) - 1)] if last_token else order[i * N])
            t, rem = divmod(r, Hl * Wl)
            y, x = divmod(rem, Wl)
            out[i] = (t, x // P, y // P) if xy_swapped else (t, y // P, x // P)
        return out
    return f


def _project_variant(heads_inner=False, one_weight=False, untransposed=False):
    def f(X, Wt, H, D):
        X, Wt = orc.as_f64(X), orc.as_f64(Wt)
        B, S, C = X.shape
        out = []
        for m in range(3):
            w = Wt[0] if one_weight else Wt[m]
            w = w.reshape(C, H * D) if untransposed else w.T
            Y = np.matmul(X, w)
            if heads_inner:
                out.append(Y.reshape(B, S, D, H).transpose(0, 3, 1, 2))
            else:
                out.append(Y.reshape(B, S, H, D).transpose(0, 2, 1, 3))
        return tuple(out)
    return f


MUTANTS = {
    "projection_heads_inner": ("qkv_project", _project_variant(heads_inner=True)),
    "projection_one_weight_for_qkv": ("qkv_project", _project_variant(one_weight=True)),
    "projection_weight_not_transposed": ("qkv_project", _project_variant(untransposed=True)),
    "descending_sort": ("cdf_binarize", _cdf_variant(descending=True)),
    "strict_compare": ("cdf_binarize", _cdf_variant(strict=True)),
    "exclusive_cumsum": ("cdf_binarize", _cdf_variant(exclusive=True)),
    "thr_not_one_minus_thr": ("cdf_binarize", _cdf_variant(use_thr=True)),
    "no_order_restoration": ("cdf_binarize", _cdf_variant(no_reorder=True)),
    "tail_divided_by_64": ("block_pool", _pool_div64),
    "scores_transposed": ("reduced_scores",
                          lambda Qa, Ka: np.matmul(Ka, np.swapaxes(Qa, -1, -2)) / np.sqrt(Qa.shape[-1])),
    "scores_scaled_by_D": ("reduced_scores",
                           lambda Qa, Ka: np.matmul(Qa, np.swapaxes(Ka, -1, -2)) / Qa.shape[-1]),
    "softmax_wrong_axis": ("row_softmax",
                           lambda L: np.exp(L - L.max(-2, keepdims=True)) / np.exp(L - L.max(-2, keepdims=True)).sum(-2, keepdims=True)),
    "sta_full_width": ("sta_mask", _sta_full_width),
    "attention_unscaled": ("masked_attention", _attn_unscaled),
    "attention_mask_transposed": ("masked_attention", _attn_transposed_mask),
    "backward_no_rowsum": ("masked_attention_bwd", _bwd_no_rowsum),
    "topk_ties_lower_index_first": ("topk_binarize", _topk_variant(ties_low_first=True)),
    "topk_keeps_smallest": ("topk_binarize", _topk_variant(smallest=True)),
    "topk_keeps_one_more": ("topk_binarize", _topk_variant(one_more=True)),
    "block_mass_rows_summed": ("block_mass", _mass_rows_summed),
    "block_mass_transposed": ("block_mass", _mass_transposed),
    "block_mass_unscaled": ("block_mass", _mass_unscaled),
    "fractal_tokens_column_major": ("fractal_order", _fractal_variant(col_major_tokens=True)),
    "fractal_patches_column_major": ("fractal_order", _fractal_variant(col_major_patches=True)),
    "fractal_edge_patches_last": ("fractal_order", _fractal_variant(edges_last=True)),
    "block_coords_of_last_token": ("block_tile_coords", _coords_variant(last_token=True)),
    "block_coords_x_and_y_swapped": ("block_tile_coords", _coords_variant(xy_swapped=True)),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(orc, attr, fn)
    assert _some_pin_fails(), f"no pin caught the planted mistake {name}"


def test_unmutated_oracle_passes_every_pin():
    assert not _some_pin_fails()
