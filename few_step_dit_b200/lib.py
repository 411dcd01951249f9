"""ctypes binding of libfsdit.so (argument marshalling only).

Every compute step runs inside the CUDA library; this module turns torch
tensors into device pointers and ctypes structs, checks the status codes and
raises on failure.  There is no Python or CPU fallback: if the library is
missing, loading raises.
"""

from __future__ import annotations

import ctypes as C
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB_PATH = os.path.join(HERE, "libfsdit.so")
HEADER_PATH = os.path.join(ROOT, "include", "fsdit.h")

F32, BF16 = 0, 1
EPI_BIAS, EPI_BIAS_F32, EPI_QKV_ROPE, EPI_GELU, EPI_RESIDUAL = 0, 1, 2, 3, 4
STATUS = {0: "FSDIT_OK", -1: "FSDIT_E_NULL", -2: "FSDIT_E_SHAPE", -3: "FSDIT_E_ALIGN",
          -4: "FSDIT_E_DTYPE", -5: "FSDIT_E_CUDA", -6: "FSDIT_E_WORKSPACE", -7: "FSDIT_E_TIMEOUT"}


class FsditError(RuntimeError):
    def __init__(self, fn, status, msg):
        super().__init__(f"{fn} -> {STATUS.get(status, status)}: {msg}")
        self.status = status


class Dims(C.Structure):
    _fields_ = [("hidden", C.c_int), ("heads", C.c_int), ("head_dim", C.c_int), ("ffn", C.c_int),
                ("rope_split", C.c_int * 3), ("rms_eps", C.c_float), ("rope_theta", C.c_float),
                ("dtype", C.c_int), ("proj_fp8", C.c_int)]


BLOCK_FIELDS = ("w_qkv", "b_qkv", "w_o", "b_o", "w_1", "b_1", "w_2", "b_2", "g_attn", "g_ffn")
BLOCK_SCALE_FIELDS = ("s_qkv", "s_o", "s_1", "s_2")  # per-output-channel scales of E4M3 projections
IO_FIELDS = ("w_vin", "b_vin", "w_tin", "b_tin", "w_ain", "b_ain", "mod_emb", "w_t1", "b_t1",
             "w_t2", "b_t2", "g_out", "w_vout", "b_vout", "w_aout", "b_aout")


class BlockWeights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in BLOCK_FIELDS + BLOCK_SCALE_FIELDS]


class IOWeights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in IO_FIELDS] + [
        ("c_video", C.c_int), ("c_text", C.c_int), ("c_audio", C.c_int), ("t_freq", C.c_int)]


class Tokens(C.Structure):
    _fields_ = [("n_tokens", C.c_int), ("n_vrows", C.c_int), ("n_text", C.c_int),
                ("n_audio", C.c_int), ("grid_t", C.c_int), ("grid_h", C.c_int),
                ("grid_w", C.c_int), ("pos_thw", C.c_void_p), ("modality", C.c_void_p),
                ("time_id", C.c_void_p), ("out_mask", C.c_void_p), ("keep_idx", C.c_void_p),
                ("n_keep", C.c_int), ("near_idx", C.c_void_p)]


class HistoryEntry(C.Structure):
    _fields_ = [("frame", C.c_int), ("stride", C.c_int)]


class HistoryStore(C.Structure):
    _fields_ = [("frames", C.c_void_p), ("capacity", C.c_int), ("H", C.c_int), ("W", C.c_int),
                ("C", C.c_int), ("n_frames", C.c_int)]


HISTORY_MAX_ENTRIES = 11
HISTORY_MIN_SLOTS = 12

DECODER_IO_FIELDS = ("w_in", "b_in", "g_out", "w_out", "b_out")
PIXELS_F32, PIXELS_RGB8 = 0, 1


class DecoderIO(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in DECODER_IO_FIELDS] + [
        ("c_lat", C.c_int), ("c_pix", C.c_int), ("patch_t", C.c_int), ("patch_s", C.c_int)]


class ProfEntry(C.Structure):
    _fields_ = [("name", C.c_char * 32), ("scopes", C.c_int), ("launches", C.c_int),
                ("ms", C.c_double), ("flops", C.c_double), ("bytes", C.c_double)]


_P = C.c_void_p
_I = C.c_int
_F = C.c_float
_SIGS = {
    "fsdit_last_error": (C.c_char_p, []),
    "fsdit_version": (C.c_char_p, []),
    "fsdit_device_error": (_I, [_P]),
    "fsdit_keep_count": (_I, [_I, _I, _I]),
    "fsdit_profile_start": (_I, [_I]),
    "fsdit_profile_stop": (_I, [C.POINTER(ProfEntry), _I]),
    "fsdit_block_workspace_size": (C.c_size_t, [C.POINTER(Dims), _I, _I]),
    "fsdit_stack_workspace_size": (C.c_size_t, [C.POINTER(Dims), C.POINTER(IOWeights),
                                                C.POINTER(Tokens), _I]),
    "fsdit_build_keep_map": (_I, [_I, _I, _I, _P, _P, _P]),
    "fsdit_gather_rows": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _P]),
    "fsdit_broadcast_residual": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P]),
    "fsdit_rmsnorm_cast": (_I, [_P, _P, _P, _I, _I, _F, _I, _P]),
    "fsdit_linear": (_I, [C.POINTER(Dims), _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P]),
    "fsdit_attention": (_I, [C.POINTER(Dims), _P, _P, _I, _P]),
    "fsdit_set_attention_pair_min_rows": (_I, [_I]),
    "fsdit_attention_pair_min_rows": (_I, []),
    "fsdit_set_norm_after_gemm": (_I, [_I]),
    "fsdit_norm_after_gemm": (_I, []),
    "dit_block_forward": (_I, [C.POINTER(Dims), C.POINTER(BlockWeights), C.POINTER(Tokens), _P, _P,
                               _P, C.c_size_t, _P]),
    "dit_block_forward_noalloc": (_I, [C.POINTER(Dims), C.POINTER(BlockWeights), C.POINTER(Tokens),
                                       _P, _P, _P]),
    "dit_stack_forward": (_I, [C.POINTER(Dims), _I, C.POINTER(BlockWeights), C.POINTER(C.c_uint8),
                               C.POINTER(IOWeights), C.POINTER(Tokens), C.POINTER(_F), _I, _P, _P,
                               _P, _P, _P, _P, C.c_size_t, _P]),
    "flow_euler_step": (_I, [_P, _P, _P, _P, _I, _I, C.POINTER(_F), C.POINTER(_F), _P]),
    "dit_flow_sample": (_I, [C.POINTER(Dims), _I, C.POINTER(BlockWeights), C.POINTER(C.c_uint8),
                             C.POINTER(IOWeights), C.POINTER(Tokens), _I, C.POINTER(_F),
                             C.POINTER(_F), _P, _P, _P, _P, C.c_size_t, _P]),
    "fsdit_quantize_rows": (_I, [_P, _I, _I, _I, _P, _P, _P]),
    "fsdit_rmsnorm_quant": (_I, [_P, _P, _I, _I, _F, _P, _P, _P]),
    "fsdit_linear_fp8": (_I, [C.POINTER(Dims), _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P]),
    "fsdit_history_bytes": (C.c_size_t, [_I, _I, _I, _I]),
    "fsdit_history_init": (_I, [C.POINTER(HistoryStore), _P, _I, _I, _I, _I]),
    "fsdit_history_push": (_I, [C.POINTER(HistoryStore), _P, _I, _P]),
    "fsdit_history_plan": (_I, [_I, C.POINTER(HistoryEntry), _I]),
    "fsdit_history_rows": (_I, [C.POINTER(HistoryEntry), _I, _I, _I]),
    "fsdit_history_gather": (_I, [C.POINTER(HistoryStore), C.POINTER(HistoryEntry), _I, _P, _I, _P, _P]),
    "fsdit_history_copy_frame": (_I, [C.POINTER(HistoryStore), _I, _P, _P]),
    "fsdit_chunk_tags": (_I, [_I, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P]),
    "fsdit_check_bounded_wait": (_I, [_P, _P]),
    "fsdit_gemm_scratch_size": (C.c_size_t, []),
    "fsdit_linear_ws": (_I, [C.POINTER(Dims), _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, C.c_size_t, _P]),
    "fsdit_linear_fp8_ws": (_I, [C.POINTER(Dims), _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, C.c_size_t,
                                 _P]),
    "fsdit_decoder_frames": (_I, [_I, _I]),
    "fsdit_decoder_workspace_size": (C.c_size_t, [C.POINTER(Dims), C.POINTER(DecoderIO), _I, _I, _I]),
    "fsdit_decoder_forward": (_I, [C.POINTER(Dims), _I, C.POINTER(BlockWeights), C.POINTER(DecoderIO), _I, _I,
                                   _I, _P, _P, _I, _P, C.c_size_t, _P]),
}

_lib = None


def header_symbols(path=HEADER_PATH):
    """Names of every entry point include/fsdit.h declares."""
    text = open(path).read()
    return re.findall(r"FSDIT_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)


def load(path=LIB_PATH):
    """Load libfsdit.so (built by few_step_dit_b200.build); raise if absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libfsdit.so not found at {path}; build it with "
                           "`python -m few_step_dit_b200.build` (no fallback exists)")
    lib = C.CDLL(path)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def last_error():
    return load().fsdit_last_error().decode(errors="replace")


def check(fn_name, status):
    if status != 0:
        raise FsditError(fn_name, status, last_error())


def call(fn_name, *args):
    lib = load()
    check(fn_name, getattr(lib, fn_name)(*args))


def ptr(t):
    """Device (or host) address of a tensor, or None."""
    if t is None:
        return None
    return C.c_void_p(t.data_ptr())


def profile_start(max_launches=100000):
    call("fsdit_profile_start", max_launches)


def profile_stop():
    """Per-class launch statistics recorded since profile_start()."""
    lib = load()
    buf = (ProfEntry * 32)()
    n = lib.fsdit_profile_stop(buf, 32)
    if n < 0:
        check("fsdit_profile_stop", n)
    return {buf[i].name.decode(): dict(scopes=buf[i].scopes, launches=buf[i].launches, ms=buf[i].ms,
                                       flops=buf[i].flops, bytes=buf[i].bytes) for i in range(n)}
