"""Host logic of the long-video ABI against the oracle, on CPU: history
plans, row counts, chunk row tags and argument validation (everything here
returns before any device work)."""

import ctypes as C

import numpy as np
import pytest

from oracle import long_video as LV
from few_step_dit_b200 import api, lib as L


@pytest.fixture(scope="module")
def lib():
    return L.load()


def _plan(lib, n_before):
    out = (L.HistoryEntry * L.HISTORY_MAX_ENTRIES)()
    n = lib.fsdit_history_plan(n_before, out, L.HISTORY_MAX_ENTRIES)
    return out, n


@pytest.mark.parametrize("n_before", list(range(0, 40)) + [123, 4096])
def test_plan_matches_oracle_selection(lib, n_before):
    out, n = _plan(lib, n_before)
    assert [(out[i].frame, out[i].stride) for i in range(n)] == LV.history_select(n_before)
    for H, W in ((34, 60), (9, 10), (5, 7)):
        assert lib.fsdit_history_rows(out, n, H, W) == LV.history_token_count(n_before, H, W)


def test_plan_rejects_bad_arguments(lib):
    out = (L.HistoryEntry * 4)()
    assert lib.fsdit_history_plan(-1, out, 4) == -1
    assert lib.fsdit_history_plan(30, out, 4) == -1  # needs 11 entries
    assert lib.fsdit_history_plan(3, out, 4) == 3


@pytest.mark.parametrize("grid,base,has_b,n_hist,n_text,n_audio",
                         [((6, 34, 60), 25, True, 4140, 256, 64), ((6, 34, 60), 0, False, 0, 256, 64),
                          ((3, 4, 6), 7, True, 37, 16, 8), ((2, 1, 1), 1, True, 1, 0, 3)])
def test_chunk_tags_match_oracle(grid, base, has_b, n_hist, n_text, n_audio):
    got = api.chunk_tags(grid, base, has_b, n_hist, n_text, n_audio)
    ref = LV.chunk_tags(grid, base, np.zeros((n_hist, 3), np.int32), n_text, n_audio, has_b)
    for k in ("modality", "time_id", "out_mask", "pos"):
        np.testing.assert_array_equal(got[k], ref[k], err_msg=k)


def test_store_validation_before_any_device_work(lib):
    s = L.HistoryStore()
    fake = C.c_void_p(1 << 20)  # never dereferenced: every check below fails first or is host-only
    assert lib.fsdit_history_init(C.byref(s), fake, 11, 34, 60, 24) == -2   # capacity < 12
    assert lib.fsdit_history_init(C.byref(s), C.c_void_p((1 << 20) + 4), 12, 34, 60, 24) == -3
    assert lib.fsdit_history_init(C.byref(s), None, 12, 34, 60, 24) == -1
    assert lib.fsdit_history_init(C.byref(s), fake, 12, 34, 60, 24) == 0
    assert lib.fsdit_history_bytes(12, 34, 60, 24) == 12 * 34 * 60 * 24 * 4
    plan = (L.HistoryEntry * 1)()
    plan[0].frame, plan[0].stride = 0, 1
    # nothing pushed yet: frame 0 is not resident
    assert lib.fsdit_history_gather(C.byref(s), plan, 1, fake, 24, fake, None) == -2
    s.n_frames = 30
    plan[0].frame = 5          # overwritten by frame 16 (11 ring slots)
    assert lib.fsdit_history_gather(C.byref(s), plan, 1, fake, 24, fake, None) == -2
    plan[0].frame, plan[0].stride = 20, 3   # resident but stride 3 is not a history stride
    assert lib.fsdit_history_gather(C.byref(s), plan, 1, fake, 24, fake, None) == -2
    assert lib.fsdit_history_gather(C.byref(s), plan, 12, fake, 24, fake, None) == -2
    plan[0].stride = 4
    assert lib.fsdit_history_gather(C.byref(s), plan, 1, fake, 23, fake, None) == -2   # ld_lat < C
    assert lib.fsdit_history_copy_frame(C.byref(s), 5, fake, None) == -2
    assert lib.fsdit_history_push(C.byref(s), None, 1, None) == -1
