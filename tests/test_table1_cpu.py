"""Host-side checks of the Table 1 configurations ("∇NABLA: Neighborhood
Adaptive Block-Level Attention", §4.1, Table 1) without a GPU: the padded Wan
720p layout puts every 64-token block on exactly one 8 x 8 tile of the
21 x 6 x 10 grid, and the STA rows of the configuration list map to the tile
windows whose oracle sparsity is the one Table 1 prints."""
import numpy as np
import pytest

import synth
from oracle import nabla_oracle as orc
from tests.test_oracle_pins import _read_golden


def test_padded_layout_blocks_are_the_tile_grid():
    w = synth.WORKLOADS[6]
    assert (w.S, w.nb) == (80_640, 1260)
    c = synth.block_coords(w.T, w.Hl, w.Wl, w.P)
    assert (c == orc.sta_grid_coords(21, 6, 10)).all()
    # every token of block b sits on tile b: the first and last token agree
    tok = synth.fractal_token_coords(w.T, w.Hl, w.Wl, w.P)
    last = tok[63::64]
    assert (np.stack([last[:, 0], last[:, 1] // 8, last[:, 2] // 8], 1) == c).all()


def test_table1_sta_rows_map_to_the_printed_sparsities():
    printed = {tuple(int(x) for x in case[1]): float(case[2][0]) for case in _read_golden("sta_table1.txt")}
    coords = orc.sta_grid_coords(21, 6, 10)
    seen = 0
    for name, thr, win in synth.TABLE1:
        if thr is None:
            tiles = synth.sta_tiles(win)
            M = orc.sta_mask(coords, tiles)
            assert round(100.0 * (1.0 - M.mean()), 2) == printed[tiles], name
            seen += 1
    assert seen == 2


@pytest.mark.parametrize("name,thr,win", [c for c in synth.TABLE1 if c[2] is not None])
def test_table1_windows_are_whole_tiles(name, thr, win):
    wt, wh, ww = win
    assert wh % 8 == 0 and ww % 8 == 0
    assert synth.sta_tiles(win) == (wt, wh // 8, ww // 8)
