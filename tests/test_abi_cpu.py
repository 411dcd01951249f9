"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/fsdit.h declares, and rejects bad arguments on the
host before any launch (no compute call is made here)."""

import ctypes as C

import pytest

from few_step_dit_b200 import api, build, lib as L


@pytest.fixture(scope="module")
def fs():
    build.build()
    return L.load()


def test_library_exports_every_declared_symbol(fs):
    names = L.header_symbols()
    assert len(names) >= 15
    for n in names:
        assert hasattr(fs, n), n
    assert set(names) == set(L._SIGS), "binding signatures out of sync with the header"


def test_keep_count_closed_form(fs):
    assert fs.fsdit_keep_count(6, 34, 60) == 3348
    assert fs.fsdit_keep_count(2, 9, 10) == 60
    assert fs.fsdit_keep_count(1, 1, 1) == 1
    assert fs.fsdit_keep_count(0, 9, 10) == 0


def _dims(**kw):
    d = api.make_dims(5376, 42, 14336, L.BF16)
    for k, v in kw.items():
        setattr(d, k, v)
    return d


def test_workspace_size_rejects_bad_dims(fs):
    assert fs.fsdit_block_workspace_size(C.byref(_dims()), 12560, 3348) > 0
    assert fs.fsdit_block_workspace_size(C.byref(_dims(head_dim=64)), 100, 0) == 0
    assert fs.fsdit_block_workspace_size(C.byref(_dims(dtype=7)), 100, 0) == 0
    assert fs.fsdit_block_workspace_size(C.byref(_dims(ffn=100)), 100, 0) == 0


def test_block_workspace_grows_with_rows(fs):
    d = _dims()
    a = fs.fsdit_block_workspace_size(C.byref(d), 3668, 0)
    b = fs.fsdit_block_workspace_size(C.byref(d), 12560, 0)
    assert b > a > 0
    # bf16 GEMM operands + fp32 compressed residual
    H, F = 5376, 14336
    assert b >= 12560 * (H + 3 * H + F) * 2


def test_entry_points_reject_null_and_bad_shapes_without_launching(fs):
    d = _dims()
    s = None
    assert fs.fsdit_linear(C.byref(d), None, None, None, None, None, None, 8, 64, 64, 0, s) == -1
    fake = C.c_void_p(0x10000)            # never dereferenced: validation fails first
    odd = C.c_void_p(0x10004)
    assert fs.fsdit_linear(C.byref(d), odd, fake, fake, fake, None, None, 8, 64, 64, 0, s) == -3
    assert fs.fsdit_linear(C.byref(d), fake, fake, fake, fake, None, None, 8, 60, 64, 0, s) == -2
    assert fs.fsdit_linear(C.byref(d), fake, fake, fake, fake, None, None, 8, 64, 60, 0, s) == -2
    assert fs.fsdit_linear(C.byref(d), fake, fake, fake, fake, None, None, 8, 64, 64, 9, s) == -2
    # RoPE epilogue needs N == 3*hidden and a position array
    assert fs.fsdit_linear(C.byref(d), fake, fake, fake, fake, None, None, 8, 64, 64, 2, s) == -1
    assert fs.fsdit_build_keep_map(0, 9, 10, fake, fake, s) == -2
    assert fs.fsdit_gather_rows(fake, None, fake, None, fake, 0, 10, 10, 64, s) == -2
    assert fs.fsdit_broadcast_residual(fake, fake, fake, fake, fake, 5, 1, 3, 3, 10, 64, s) == -2  # 4 kept
    assert fs.fsdit_broadcast_residual(fake, fake, fake, fake, fake, 4, 1, 3, 3, 8, 64, s) == -2   # rows < grid
    assert fs.fsdit_rmsnorm_cast(fake, fake, fake, 4, 100, 1e-6, 1, s) == -2
    assert fs.fsdit_rmsnorm_cast(fake, fake, fake, 4, 64, 1e-6, 3, s) == -4
    tc = (C.c_float * 4)(0, 0.2, 0.5, 0)
    assert fs.flow_euler_step(fake, fake, None, None, 4, 24, tc, tc, s) == -1
    assert fs.flow_euler_step(fake, fake, fake, fake, 4, 0, tc, tc, s) == -2
    msg = L.last_error()
    assert "row_width" in msg


def test_block_forward_rejects_inconsistent_tokens(fs):
    d = _dims()
    fake = C.c_void_p(0x10000)
    w = L.BlockWeights(*([0x10000] * 10))
    tok = L.Tokens()
    tok.n_tokens, tok.n_vrows, tok.n_text, tok.n_audio = 100, 80, 10, 5   # 95 != 100
    tok.pos_thw = 0x10000
    assert fs.dit_block_forward(C.byref(d), C.byref(w), C.byref(tok), fake, fake, fake, 1 << 30, None) == -2
    tok.n_audio = 10
    tok.grid_t, tok.grid_h, tok.grid_w = 1, 9, 10                           # 90 > 80 video rows
    assert fs.dit_block_forward(C.byref(d), C.byref(w), C.byref(tok), fake, fake, fake, 1 << 30, None) == -2
    tok.grid_t, tok.grid_h, tok.grid_w = 1, 8, 10
    tok.keep_idx, tok.near_idx, tok.n_keep = 0x10000, 0x10000, 7            # should be 30
    assert fs.dit_block_forward(C.byref(d), C.byref(w), C.byref(tok), fake, fake, fake, 1 << 30, None) == -2
    tok.n_keep = 30
    # workspace too small
    assert fs.dit_block_forward(C.byref(d), C.byref(w), C.byref(tok), fake, fake, fake, 16, None) == -6


def _dec_io(**kw):
    io = L.DecoderIO(*([0x10000] * 5), 24, 3, 4, 16)
    for k, v in kw.items():
        setattr(io, k, v)
    return io


def test_decoder_frame_count_closed_form(fs):
    assert fs.fsdit_decoder_frames(6, 4) == 21
    assert fs.fsdit_decoder_frames(1, 4) == 1
    assert fs.fsdit_decoder_frames(5, 4) == 17
    assert fs.fsdit_decoder_frames(0, 4) == 0


def test_decoder_workspace_size_and_bad_io(fs):
    d = api.make_dims(2048, 16, 8192, L.BF16)
    n = fs.fsdit_decoder_workspace_size(C.byref(d), C.byref(_dec_io()), 6, 34, 60)
    # fp32 residual + bf16 GEMM operands (x_n, qkv, FFN) for 12,240 cells
    assert n >= 12240 * (2048 * 4 + (2048 + 3 * 2048 + 8192) * 2)
    assert fs.fsdit_decoder_workspace_size(C.byref(d), C.byref(_dec_io(patch_s=6)), 6, 34, 60) == 0
    assert fs.fsdit_decoder_workspace_size(C.byref(d), C.byref(_dec_io(c_lat=0)), 6, 34, 60) == 0
    assert fs.fsdit_decoder_workspace_size(C.byref(d), C.byref(_dec_io(c_lat=65)), 6, 34, 60) == 0
    assert fs.fsdit_decoder_workspace_size(C.byref(d), C.byref(_dec_io()), 0, 34, 60) == 0
    assert fs.fsdit_decoder_workspace_size(C.byref(d), C.byref(_dec_io(w_out=None)), 6, 34, 60) == 0


def test_decoder_forward_rejects_bad_arguments_without_launching(fs):
    d = api.make_dims(2048, 16, 8192, L.BF16)
    fake, odd = C.c_void_p(0x10000), C.c_void_p(0x10004)
    w = (L.BlockWeights * 1)(L.BlockWeights(*([0x10000] * 10)))
    big = 1 << 40
    f = fs.fsdit_decoder_forward
    rgb = L.PIXELS_RGB8
    assert f(C.byref(d), 1, w, C.byref(_dec_io()), 6, 34, 60, None, fake, 0, fake, big, None) == -1
    assert f(C.byref(d), 1, None, C.byref(_dec_io()), 6, 34, 60, fake, fake, 0, fake, big, None) == -1
    assert f(C.byref(d), 1, w, C.byref(_dec_io(patch_s=2)), 6, 34, 60, fake, fake, 0, fake, big, None) == -2
    assert f(C.byref(d), 1, w, C.byref(_dec_io()), 6, 0, 60, fake, fake, 0, fake, big, None) == -2
    assert f(C.byref(d), 1, w, C.byref(_dec_io()), 6, 34, 60, fake, odd, rgb, fake, big, None) == -3
    assert f(C.byref(d), 1, w, C.byref(_dec_io()), 6, 34, 60, fake, fake, 2, fake, big, None) == -4
    assert "pixel_format" in L.last_error()
    assert f(C.byref(d), 1, w, C.byref(_dec_io()), 6, 34, 60, fake, fake, rgb, fake, 1024, None) == -6
    assert "workspace" in L.last_error()


def test_linear_ws_rejects_bad_scratch_without_launching(fs):
    d = _dims()
    fake, odd = C.c_void_p(0x10000), C.c_void_p(0x10004)
    need = fs.fsdit_gemm_scratch_size()
    assert need >= 128 * 256 * 1024                          # 128 parts of 256 KB + counters
    f = fs.fsdit_linear_ws
    assert f(C.byref(d), fake, fake, fake, fake, None, None, 8, 64, 64, 0, fake, need - 1, None) == -6
    assert "scratch" in L.last_error()
    assert f(C.byref(d), fake, fake, fake, fake, None, None, 8, 64, 64, 0, odd, need, None) == -3
    assert f(C.byref(d), fake, fake, fake, fake, None, None, 8, 60, 64, 0, fake, need, None) == -2
    d8 = api.make_dims(5376, 42, 14336, L.BF16, proj_fp8=True)
    g = fs.fsdit_linear_fp8_ws
    assert g(C.byref(d8), fake, fake, fake, fake, fake, fake, None, None, 8, 64, 64, 0, fake, need - 1, None) == -6


NOALLOC_LIMITS = [  # (hidden, heads, ffn, dtype, largest uncompressed rows, largest compressed rows)
    (5376, 56, 14336, L.BF16, 387, 310), (5376, 56, 14336, L.F32, 194, 172),
    (2048, 16, 8192, L.BF16, 1008, 808), (2048, 16, 8192, L.F32, 508, 451),
    (256, 2, 512, L.BF16, 9362, 7262), (256, 2, 512, L.F32, 5041, 4362),
]


@pytest.mark.parametrize("hidden,heads,ffn,dtype,max_full,max_comp", NOALLOC_LIMITS)
def test_noalloc_limits_in_the_header_are_the_32_mib_boundaries(fs, hidden, heads, ffn, dtype, max_full, max_comp):
    # the limits include/fsdit.h lists for dit_block_forward_noalloc: the
    # largest row counts whose workspace fits the 32 MiB static array; one row
    # more is refused on the host (FSDIT_E_WORKSPACE) before any CUDA call.
    # At the limit the host checks pass and the call goes on to look up the
    # device (no GPU here, so it stops there with another status).
    d = api.make_dims(hidden, heads, ffn, dtype)
    lim = 32 << 20
    assert fs.fsdit_block_workspace_size(C.byref(d), max_full, 0) <= lim
    assert fs.fsdit_block_workspace_size(C.byref(d), max_full + 1, 0) > lim
    assert fs.fsdit_block_workspace_size(C.byref(d), max_comp, 1) <= lim
    assert fs.fsdit_block_workspace_size(C.byref(d), max_comp + 1, 1) > lim
    fake = C.c_void_p(0x10000)
    w = L.BlockWeights(*([0x10000] * 10))
    for compress, limit in ((False, max_full), (True, max_comp)):
        for extra in (0, 1):
            tok = L.Tokens()
            T, H, W = 2, 9, 10                       # 180 grid rows, 60 kept
            kept = 60 if compress else 180
            n = limit + extra + (180 - kept)         # rows such that the block's own row count is limit + extra
            tok.n_tokens, tok.n_vrows, tok.n_text, tok.n_audio = n, 180, n - 180, 0
            tok.grid_t, tok.grid_h, tok.grid_w = T, H, W
            tok.pos_thw = 0x10000
            if compress:
                tok.keep_idx, tok.n_keep, tok.near_idx = 0x10000, 60, 0x10000
            st = fs.dit_block_forward_noalloc(C.byref(d), C.byref(w), C.byref(tok), fake, fake, None)
            if extra:
                assert st == -6, (compress, L.last_error())
            else:
                assert st != -6, (compress, L.last_error())
