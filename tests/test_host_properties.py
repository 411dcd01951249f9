"""Property-based checks (hypothesis) of the library's host-side entry points
against the oracle, on CPU: kept-token counts, decoder frame counts, history
plans and their row counts, and the row tags of a long-video chunk, over
randomly drawn grids and video lengths rather than a fixed list."""

import numpy as np
import pytest
from hypothesis import given, settings, strategies as st

import oracle as O
from oracle import decoder as OD
from oracle import long_video as LV
from few_step_dit_b200 import api, build, lib as L

SETTINGS = settings(max_examples=100, deadline=None)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    L.load()


@SETTINGS
@given(T=st.integers(0, 12), H=st.integers(1, 70), W=st.integers(1, 90))
def test_keep_count_is_the_oracle_map_size(T, H, W):
    keep_idx, near_idx = O.keep_map(T, H, W)
    assert L.load().fsdit_keep_count(T, H, W) == len(keep_idx)
    assert len(near_idx) == T * H * W


@SETTINGS
@given(T=st.integers(1, 64), pt=st.integers(1, 8))
def test_decoder_frame_count_is_the_oracle_count(T, pt):
    assert L.load().fsdit_decoder_frames(T, pt) == OD.decoder_frames(T, pt)
    # and it equals the frames the oracle's unpatchify produces
    y = np.zeros((T, 1 * pt * 1 * 1))
    assert OD.unpatchify(y, T, 1, 1, 1, pt, 1).shape[0] == OD.decoder_frames(T, pt)


@SETTINGS
@given(n_before=st.integers(0, 200000), H=st.integers(1, 70), W=st.integers(1, 90))
def test_history_plan_and_rows_match_the_oracle(n_before, H, W):
    out = (L.HistoryEntry * L.HISTORY_MAX_ENTRIES)()
    n = L.load().fsdit_history_plan(n_before, out, L.HISTORY_MAX_ENTRIES)
    assert [(out[i].frame, out[i].stride) for i in range(n)] == LV.history_select(n_before)
    assert L.load().fsdit_history_rows(out, n, H, W) == LV.history_token_count(n_before, H, W)


@SETTINGS
@given(T=st.integers(1, 6), H=st.integers(1, 9), W=st.integers(1, 11), base=st.integers(0, 500),
       has_b=st.booleans(), n_hist=st.integers(0, 40), n_text=st.integers(0, 20), n_audio=st.integers(0, 20))
def test_chunk_tags_match_the_oracle(T, H, W, base, has_b, n_hist, n_text, n_audio):
    if has_b and T < 2:
        # a chunk with a boundary frame has at least one new frame
        with pytest.raises(L.FsditError, match="FSDIT_E_SHAPE"):
            api.chunk_tags((T, H, W), base, has_b, n_hist, n_text, n_audio)
        return
    got = api.chunk_tags((T, H, W), base, has_b, n_hist, n_text, n_audio)
    ref = LV.chunk_tags((T, H, W), base, np.zeros((n_hist, 3), np.int32), n_text, n_audio, has_b)
    for k in ("modality", "time_id", "out_mask", "pos"):
        np.testing.assert_array_equal(got[k], ref[k], err_msg=k)
