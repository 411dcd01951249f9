"""The C ABI from a plain C program (tests/c_consumer.c), compiled with gcc
against include/fsdit.h and linked with libfsdit.so and the CUDA runtime: no
Python or torch between the caller and the library.

CPU: the header compiles as pedantic C89/C99 and C++17; the host-only entry
points give the oracle's keep counts, decoder frame counts and history plans,
and reject bad arguments with the documented status codes.
GPU: one fp32 DiT block (compressed and keep-all) run from C matches the
oracle at rel-L2 <= 1e-5, the bound of every fp32 block test.
"""

import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle as O
from oracle import decoder as OD
from oracle import long_video as LV
from few_step_dit_b200 import build, lib as L
from few_step_dit_b200 import synthetic as S

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")
PKG = os.path.join(ROOT, "few_step_dit_b200")
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")
SRC = os.path.join(ROOT, "tests", "c_consumer.c")

needs_gcc = pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not found")


def _run(cmd, **kw):
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, **kw)
    assert r.returncode == 0, f"{' '.join(cmd)}\n{r.stdout}\n{r.stderr}"
    return r.stdout


@pytest.fixture(scope="module")
def consumer(tmp_path_factory):
    build.build()
    L.load()
    exe = str(tmp_path_factory.mktemp("c_consumer") / "c_consumer")
    _run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-O1", "-I", INCLUDE, "-I",
          os.path.join(CUDA, "include"), SRC, "-o", exe, "-L", PKG, "-lfsdit", "-L", os.path.join(CUDA, "lib64"),
          "-lcudart", f"-Wl,-rpath,{PKG}", f"-Wl,-rpath,{os.path.join(CUDA, 'lib64')}"])
    return exe


@needs_gcc
@pytest.mark.parametrize("cmd", [["gcc", "-std=c89"], ["gcc", "-std=c99"], ["g++", "-std=c++17", "-x", "c++"]])
def test_header_compiles_as_plain_c_and_cpp(tmp_path, cmd):
    src = tmp_path / "h.c"
    src.write_text('#include "fsdit.h"\nint main(void) { return fsdit_keep_count(1, 1, 1) == 1 ? 0 : 1; }\n')
    _run(cmd + ["-pedantic", "-Wall", "-Wextra", "-Werror", "-fsyntax-only", "-I", INCLUDE, str(src)])


@pytest.fixture(scope="module")
def host_lines(consumer):
    out = _run([consumer, "host"])
    lines = {}
    for ln in out.splitlines():
        key, _, rest = ln.partition(" ")
        lines.setdefault(key, []).append(rest.split())
    return lines


@needs_gcc
def test_host_entry_points_match_the_oracle(host_lines):
    assert host_lines["version"][0][0] == "fsdit"
    for T, H, W, n in (map(int, r) for r in host_lines["keep"]):
        keep_idx, _ = O.keep_map(T, H, W)
        assert n == len(keep_idx), (T, H, W)
    for T, pt, n in (map(int, r) for r in host_lines["frames"]):
        assert n == OD.decoder_frames(T, pt)
    assert len(host_lines["plan"]) == 32
    for r in host_lines["plan"]:
        nb, n = int(r[0]), int(r[1])
        pairs = [(int(r[2 + 2 * k]), int(r[3 + 2 * k])) for k in range(n)]
        assert pairs == LV.history_select(nb), nb
        assert r[2 + 2 * n] == "rows" and int(r[3 + 2 * n]) == LV.history_token_count(nb, 34, 60)
    assert int(host_lines["plan_small"][0][0]) == -1
    assert int(host_lines["history_bytes"][0][0]) == 12 * 34 * 60 * 24 * 4
    a, b = map(int, host_lines["block_ws"][0])
    assert b > a > 0
    assert int(host_lines["block_ws_bad"][0][0]) == 0


@needs_gcc
def test_host_argument_checks_return_documented_codes(host_lines):
    st = {r[0]: (int(r[1]), int(r[2])) for r in host_lines["status"]}
    assert st["keep_map_null"] == (-1, 1)          # FSDIT_E_NULL, with a message
    assert st["history_init_null"] == (-1, 1)
    assert st["history_init_small"] == (-2, 1)     # FSDIT_E_SHAPE: capacity < 12
    assert st["euler_null"] == (-1, 1)


def _write_block_inputs(d, w, layer, x, tags):
    for k in L.BLOCK_FIELDS:
        np.ascontiguousarray(layer[k].float().numpy(), np.float32).tofile(os.path.join(d, f"{k}.bin"))
    np.ascontiguousarray(x.float().numpy(), np.float32).tofile(os.path.join(d, "x.bin"))
    np.ascontiguousarray(tags["pos"], np.int32).tofile(os.path.join(d, "pos.bin"))
    for k in ("modality", "time_id", "out_mask"):
        np.ascontiguousarray(tags[k], np.uint8).tofile(os.path.join(d, f"{k}.bin"))


@needs_gcc
@pytest.mark.gpu
@pytest.mark.parametrize("compress", [1, 0])
def test_block_from_c_matches_oracle(consumer, tmp_path, compress):
    w = S.WORKLOADS["tiny_block_f32"]
    layers, _ = S.make_weights(w, n_layers=1)
    x = S.make_inputs(w)["x"].float()
    tags = S.pack_tokens(w)
    _write_block_inputs(str(tmp_path), w, layers[0], x, tags)
    T, H, Wd = w.grid
    out = _run([consumer, "block", str(tmp_path), str(w.hidden), str(w.heads), str(w.ffn), str(T), str(H),
                str(Wd), str(w.n_text), str(w.n_audio), str(compress)])
    assert "block ok" in out
    got = np.fromfile(tmp_path / "out.bin", np.float32).reshape(w.n_tokens, w.hidden).astype(np.float64)
    wn = S.to_numpy64(layers[0])
    xn = x.double().numpy()
    if compress:
        k, n = O.keep_map(*w.grid)
        ref = O.dit_block_compressed(xn, wn, tags["pos"], w.heads, w.head_dim, k, n, w.n_video)
    else:
        ref = O.dit_block(xn, wn, tags["pos"], w.heads, w.head_dim)
    assert O.rel_l2(got, ref) < 1e-5
    assert O.rel_l2(got - xn, ref - xn) < 1e-5
