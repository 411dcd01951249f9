"""Device-side checks of caller-provided keep maps in the gather and the
nearest-kept broadcast ([PaperDaily] section 二: each dropped position takes
the update of its nearest kept position in the same frame).

Each test plants one bad entry in a map that is otherwise the one
fsdit_build_keep_map writes.  The kernels check every entry before they use
it, so no planted entry is ever followed (an index outside the grid is
compared, never dereferenced): the rows the bad entry would have produced are
left unwritten, every other row matches the oracle, and
fsdit_device_error() reports FSDIT_E_SHAPE.  A valid map leaves the word
clear.
"""

import numpy as np
import pytest
import torch

import oracle as O
from few_step_dit_b200 import api, build, lib as L

pytestmark = pytest.mark.gpu
DEV = "cuda"
E_SHAPE = -2
SENTINEL = 12345.0


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    L.load()
    torch.cuda.synchronize()
    api.device_error()          # start from a clear word
    yield
    torch.cuda.synchronize()


def _status():
    return L.load().fsdit_device_error(None)


def _gather(x, pos, keep_idx, n_grid):
    n_rows, hidden = x.shape
    n_keep = keep_idx.numel()
    n_out = n_keep + n_rows - n_grid
    xc = torch.full((n_out, hidden), SENTINEL, dtype=torch.float32, device=DEV)
    posc = torch.full((n_out, 3), -7, dtype=torch.int32, device=DEV)
    L.call("fsdit_gather_rows", L.ptr(x), L.ptr(pos), L.ptr(xc), L.ptr(posc), L.ptr(keep_idx), n_keep, n_grid,
           n_rows, hidden, None)
    return xc, posc


def _broadcast(x, yc, keep_idx, near_idx, grid):
    out = torch.full_like(x, SENTINEL)
    L.call("fsdit_broadcast_residual", L.ptr(x), L.ptr(yc), L.ptr(out), L.ptr(keep_idx), L.ptr(near_idx),
           keep_idx.numel(), *grid, x.shape[0], x.shape[1], None)
    return out


def _case(grid=(2, 9, 10), n_other=5, hidden=256, seed=0):
    T, H, W = grid
    V = T * H * W
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(V + n_other, hidden, generator=g)
    keep_idx, near_idx = O.keep_map(T, H, W)
    yc = torch.randn(len(keep_idx) + n_other, hidden, generator=g)
    return x, yc, keep_idx, near_idx, V


def _expect_broadcast(x, yc, keep_idx, near_idx, V):
    return O.broadcast_residual(x.numpy(), yc.numpy(), keep_idx, near_idx, V)


def test_valid_maps_leave_the_error_word_clear():
    x, yc, keep_idx, near_idx, V = _case()
    pos = torch.randint(0, 9, (x.shape[0], 3), dtype=torch.int32)
    k, n = torch.tensor(keep_idx).to(DEV), torch.tensor(near_idx).to(DEV)
    _gather(x.to(DEV), pos.to(DEV), k, V)
    _broadcast(x.to(DEV), yc.to(DEV), k, n, (2, 9, 10))
    assert _status() == 0


@pytest.mark.parametrize("bad", [10 ** 6, -3, 180])      # 180 = first row past the 2x9x10 grid
def test_gather_skips_an_out_of_grid_keep_entry(bad):
    x, _, keep_idx, _, V = _case()
    pos = torch.randint(0, 9, (x.shape[0], 3), dtype=torch.int32)
    ki = keep_idx.copy()
    ki[7] = bad
    xc, posc = _gather(x.to(DEV), pos.to(DEV), torch.tensor(ki).to(DEV), V)
    assert _status() == E_SHAPE
    assert "keep_idx" in L.last_error()
    xc, posc = xc.cpu().numpy(), posc.cpu().numpy()
    good = np.arange(xc.shape[0]) != 7
    np.testing.assert_array_equal(xc[good], O.gather_rows(x.numpy(), keep_idx, V)[good])
    np.testing.assert_array_equal(posc[good], O.gather_rows(pos.numpy(), keep_idx, V)[good])
    assert (xc[7] == SENTINEL).all() and (posc[7] == -7).all()     # unwritten, nothing read for it
    assert _status() == 0                                            # the word was cleared


def _broadcast_with(keep_idx, near_idx, x, yc, V, grid=(2, 9, 10)):
    out = _broadcast(x.to(DEV), yc.to(DEV), torch.tensor(keep_idx).to(DEV), torch.tensor(near_idx).to(DEV), grid)
    return out.cpu().numpy(), _status()


def test_broadcast_reports_a_near_entry_that_is_not_adjacent_and_writes_every_other_row():
    # dropped row p = (t 0, h 1, w 3) points at a kept token of another
    # column: in range, but no block owns p then; out of place, p stays
    # unwritten and the error is reported
    x, yc, keep_idx, near_idx, V = _case()
    p = 1 * 10 + 3
    ni = near_idx.copy()
    ni[p] = near_idx[p] + 2
    got, st = _broadcast_with(keep_idx, ni, x, yc, V)
    assert st == E_SHAPE
    ref = _expect_broadcast(x, yc, keep_idx, near_idx, V)
    rows = np.arange(x.shape[0]) != p
    np.testing.assert_allclose(got[rows], ref[rows], rtol=0, atol=1e-5)
    assert (got[p] == SENTINEL).all()


@pytest.mark.parametrize("where,value", [("keep", 10 ** 6), ("keep", -1), ("near", -5), ("near", 10 ** 6),
                                         ("near_frame", None), ("dup", None)])
def test_broadcast_reports_bad_entries_without_following_them(where, value):
    x, yc, keep_idx, near_idx, V = _case(seed=1)
    ki, ni = keep_idx.copy(), near_idx.copy()
    if where == "keep":
        ki[4] = value
    elif where == "near":
        ni[33] = value
    elif where == "near_frame":
        ni[5] = len(keep_idx) - 1          # a kept token of the other frame
    else:
        ki[2] = ki[3]                      # two kept tokens on one row
    got, st = _broadcast_with(ki, ni, x, yc, V)
    assert st == E_SHAPE, where
    # the rows no bad entry touches are still exact
    ref = _expect_broadcast(x, yc, keep_idx, near_idx, V)
    assert np.isfinite(got).all()
    touched = np.zeros(x.shape[0], bool)
    grid_rows = touched[:V]                # a view: marks go through to `touched`
    if where == "keep":
        grid_rows[near_idx == 4] = True
    elif where == "near":
        grid_rows[33] = True
    elif where == "near_frame":
        grid_rows[5] = True
    else:
        grid_rows[near_idx == 2] = True
    np.testing.assert_allclose(got[~touched], ref[~touched], rtol=0, atol=1e-5)


def test_compressed_block_with_a_bad_map_reports_it():
    # the same check through dit_block_forward's per-block form
    from few_step_dit_b200 import synthetic as S
    w = S.WORKLOADS["tiny_block_f32"]
    g = torch.Generator().manual_seed(S.SEED_WEIGHTS)
    bw = api.BlockWeights({k: v.to(DEV) for k, v in S.make_block_weights(w, g).items()})
    tags = S.pack_tokens(w)
    seq = api.Sequence.from_workload(w, tags, DEV)
    x = torch.randn(w.n_tokens, w.hidden, generator=torch.Generator().manual_seed(3)).to(DEV)
    dims = api.dims_of(w)
    api.block_forward(dims, bw, seq, x)
    assert _status() == 0
    seq.keep_idx[0] = w.n_video + 1000
    api.block_forward(dims, bw, seq, x)
    assert _status() == E_SHAPE
