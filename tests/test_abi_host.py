"""C-ABI checks that need no GPU: the library loads, exports every declared
symbol, the ctypes layout matches the C structs, and host-side validation
returns the documented status before anything is launched."""
import ctypes
import os
import re
import subprocess

import pytest

import kv_cache_compression_fkv_b200 as fkv
from kv_cache_compression_fkv_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fkv.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\*?(fkv_\w+)\s*\(", src, flags=re.M)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert len(names) >= 14
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r" T (fkv_\w+)", out))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    assert set(names) == set(_lib.SIGNATURES)


def test_struct_layout_matches_header(tmp_path, lib):
    prog = tmp_path / "layout.c"
    prog.write_text(
        '#include <stdio.h>\n#include <stddef.h>\n#include "fkv.h"\n'
        "int main(void){printf(\"%zu %zu %zu %zu %zu\\n\", sizeof(fkv_params_t),"
        " offsetof(fkv_params_t, scale), offsetof(fkv_params_t, granularity),"
        " sizeof(fkv_step_io_t), offsetof(fkv_step_io_t, out)); return 0;}\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(prog), "-o", str(exe)], check=True)
    got = list(map(int, subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()))
    P, S = _lib.Params, _lib.StepIO
    assert got == [ctypes.sizeof(P), P.scale.offset, P.granularity.offset, ctypes.sizeof(S), S.out.offset]


def test_fp8_cache_layout_matches_header(tmp_path, lib):
    fields = _lib.FP8_CACHE_FIELDS
    prog = tmp_path / "layout8.c"
    body = " ".join(f'printf("%zu ", offsetof(fkv_fp8_cache_t, {f}));' for f in fields)
    prog.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "fkv.h"\n'
                    "int main(void){" + body + ' printf("%zu\\n", sizeof(fkv_fp8_cache_t)); return 0;}\n')
    exe = tmp_path / "layout8"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(prog), "-o", str(exe)], check=True)
    got = list(map(int, subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()))
    C = _lib.Fp8Cache
    assert got == [getattr(C, f).offset for f in fields] + [ctypes.sizeof(C)]


def _fp8_params(**kw):
    base = dict(L=1, H=2, D=128, T=128, F=4, Fc=1, dtype="bf16", comp_rows=4 * 128, score_stride=1)
    base.update(kw)
    return fkv.make_params(**base)


def test_fp8_entry_points_validate_before_launch(lib):
    p = _fp8_params()
    c = _lib.Fp8Cache()
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: validation fails first
    bp = ctypes.byref(p)
    # null cache struct / null members
    assert lib.fkv_compact_gather_fp8(bp, fake, fake, fake, fake, None, fake, None) == _lib.FKV_ERR_INVALID_ARG
    assert lib.fkv_compact_gather_fp8(bp, fake, fake, fake, fake, ctypes.byref(c), fake, None) == _lib.FKV_ERR_INVALID_ARG
    assert lib.fkv_quantize_chunk_fp8(bp, fake, fake, fake, ctypes.byref(c), fake, None) == _lib.FKV_ERR_INVALID_ARG
    assert lib.fkv_attend_compressed_fp8(bp, ctypes.byref(c), fake, fake, fake, None) == _lib.FKV_ERR_INVALID_ARG
    # unsupported configurations
    for bad in (_fp8_params(dtype="fp32", D=64), _fp8_params(granularity="token", n_score_q=4, sink_tokens=128,
                                                              recent_tokens=128)):
        assert lib.fkv_quantize_chunk_fp8(ctypes.byref(bad), fake, fake, fake, ctypes.byref(c), fake,
                                          None) == _lib.FKV_ERR_UNSUPPORTED
    small_t = _fp8_params(T=64, comp_rows=4 * 64)
    assert lib.fkv_attend_compressed_fp8(ctypes.byref(small_t), ctypes.byref(c), fake, fake, fake,
                                         None) == _lib.FKV_ERR_UNSUPPORTED
    # misaligned code buffer
    for f in _lib.FP8_CACHE_FIELDS:
        setattr(c, f, 1 << 20)
    c.k_comp = (1 << 20) + 8
    assert lib.fkv_compact_gather_fp8(bp, fake, fake, fake, fake, ctypes.byref(c), fake, None) == _lib.FKV_ERR_INVALID_ARG


def test_status_strings_and_version(lib):
    assert lib.fkv_abi_version() == 6
    for code in range(8):
        assert lib.fkv_status_string(code).decode().startswith("FKV_")
    assert lib.fkv_status_string(99) == b"FKV_ERR_UNKNOWN"


def _p(**kw):
    base = dict(L=1, H=4, D=128, T=32, F=6, Fc=1, dtype="bf16", score_stride=1)
    base.update(kw)
    return fkv.make_params(**base)


def test_param_validation(lib):
    chk = lambda p: lib.fkv_check_params(ctypes.byref(p))
    assert chk(_p()) == _lib.FKV_OK
    assert chk(_p(D=64)) == _lib.FKV_ERR_UNSUPPORTED          # bf16 path is head_dim 128
    assert chk(_p(D=64, dtype="fp32")) == _lib.FKV_OK
    assert chk(_p(D=66, dtype="fp32")) == _lib.FKV_ERR_UNSUPPORTED
    assert chk(_p(T=0)) == _lib.FKV_ERR_SHAPE
    assert chk(_p(Fc=0)) == _lib.FKV_ERR_SHAPE
    assert chk(_p(F=0)) == _lib.FKV_OK                          # empty history is allowed
    assert chk(_p(score_stride=0)) == _lib.FKV_ERR_SHAPE
    assert chk(_p(F=2000)) == _lib.FKV_ERR_SHAPE
    p = _p()
    p.dtype = 7
    assert chk(p) == _lib.FKV_ERR_INVALID_ARG
    for bad in (float("nan"), 0.0, -0.125, float("inf")):
        p = _p()
        p.scale = bad
        assert chk(p) == _lib.FKV_ERR_INVALID_ARG
    tok = _p(granularity="token", sink_tokens=40, recent_tokens=40, n_score_q=8)
    assert chk(tok) == _lib.FKV_OK
    tok.sink_tokens = 180
    assert chk(tok) == _lib.FKV_ERR_SHAPE                       # S + R > N
    assert lib.fkv_check_params(None) == _lib.FKV_ERR_INVALID_ARG
    p = _p()
    p.flags = 4                                                  # unknown flag bit
    assert chk(p) == _lib.FKV_ERR_INVALID_ARG
    assert chk(_p(score_with_chunk=True)) == _lib.FKV_OK
    assert chk(_p(granularity="token", sink_tokens=40, recent_tokens=40, n_score_q=8,
                  score_with_chunk=True)) == _lib.FKV_ERR_UNSUPPORTED


def test_derived_sizes(lib):
    s = fkv.sizes(_p())
    assert s["nseg"] == 6 and s["max_kept"] == 6 and s["max_comp_rows"] == 192
    # status block + (max, sum) per 128-key block of each frame and scoring
    # row (T = 32: one block per frame, no chunk entries), then per-row merges
    assert s["ws_bytes"] == 256 + 4 * 6 * 32 * 8 + 4 * 32 * 8
    # T = 300 (3 blocks per frame) with the chunk's 3 blocks in the normaliser
    a256 = lambda n: (n + 255) // 256 * 256  # noqa: E731  (each region 256-byte aligned)
    c = fkv.sizes(_p(T=300, score_with_chunk=True))
    assert c["ws_bytes"] == 256 + a256(4 * (6 * 3 + 3) * 300 * 8) + a256(4 * 300 * 8)
    # fp32 (CUDA-core) scoring: one entry per frame + one chunk slot
    f = fkv.sizes(_p(dtype="fp32", D=64))
    assert f["ws_bytes"] == 256 + 4 * (6 + 1) * 32 * 8 + 4 * 32 * 8
    t = fkv.sizes(_p(granularity="token", sink_tokens=40, recent_tokens=40, n_score_q=8))
    assert t["nseg"] == 192 - 80 and t["max_kept"] == 192 and t["max_comp_rows"] == 192


def test_null_and_misaligned_pointers_fail_before_launch(lib):
    p = _p()
    fake = 1 << 20  # never dereferenced: validation fails first
    assert lib.fkv_score_segments(ctypes.byref(p), fake, None, None, None, fake, fake, fake, None) == _lib.FKV_ERR_INVALID_ARG
    assert lib.fkv_score_segments(ctypes.byref(p), fake + 8, None, fake, None, fake, fake, fake, None) == _lib.FKV_ERR_INVALID_ARG
    assert lib.fkv_score_segments(ctypes.byref(p), fake, None, fake, None, fake, fake, fake + 16, None) == _lib.FKV_ERR_WORKSPACE
    pc = _p(score_with_chunk=True)                                # needs k_cur
    assert lib.fkv_score_segments(ctypes.byref(pc), fake, None, fake, None, fake, fake, fake, None) == _lib.FKV_ERR_INVALID_ARG
    assert lib.fkv_select_topk(ctypes.byref(p), fake, None, fake, fake, fake, fake, fake, None) == _lib.FKV_ERR_INVALID_ARG
    assert lib.fkv_compact_gather(ctypes.byref(p), fake, fake, fake, fake, fake, None, fake, None) == _lib.FKV_ERR_INVALID_ARG
    assert lib.fkv_attend_compressed(ctypes.byref(p), fake, fake, fake, fake, fake, fake, fake, None, None) == _lib.FKV_ERR_WORKSPACE
    io = _lib.StepIO()
    assert lib.fkv_step(ctypes.byref(p), ctypes.byref(io), fake, None) == _lib.FKV_ERR_INVALID_ARG
    assert lib.fkv_step(ctypes.byref(p), None, fake, None) == _lib.FKV_ERR_INVALID_ARG
    bad = _p(T=0)
    assert lib.fkv_step(ctypes.byref(bad), ctypes.byref(io), fake, None) == _lib.FKV_ERR_SHAPE
    assert lib.fkv_workspace_init(fake + 8, 512, None) == _lib.FKV_ERR_WORKSPACE
    assert lib.fkv_read_status(None, None, None, None) == _lib.FKV_ERR_WORKSPACE


def test_heuristic_selector_validates_before_launch(lib):
    p = _fp8_params()
    fake = ctypes.c_void_p(1 << 20)
    bp = ctypes.byref(p)
    assert lib.fkv_select_heuristic(bp, 7, 1, fake, fake, fake, fake, fake, None) == _lib.FKV_ERR_INVALID_ARG
    # random needs seg_score; uniform does not (but needs the kept arrays)
    assert lib.fkv_select_heuristic(bp, _lib.FKV_POLICY_RANDOM, 1, fake, None, fake, fake, fake,
                                    None) == _lib.FKV_ERR_INVALID_ARG
    assert lib.fkv_select_heuristic(bp, _lib.FKV_POLICY_UNIFORM, 1, fake, None, None, fake, fake,
                                    None) == _lib.FKV_ERR_INVALID_ARG
    tm = _fp8_params(static_token_mask=True)
    assert lib.fkv_select_heuristic(ctypes.byref(tm), _lib.FKV_POLICY_UNIFORM, 1, fake, None, fake,
                                    fake, fake, None) == _lib.FKV_ERR_UNSUPPORTED


def test_step_fp8_validates_before_launch(lib):
    p = _fp8_params()
    io = _lib.StepIO()
    c = _lib.Fp8Cache()
    fake = ctypes.c_void_p(1 << 20)
    assert lib.fkv_step_fp8(ctypes.byref(p), None, ctypes.byref(c), fake, None) == _lib.FKV_ERR_INVALID_ARG
    for f in _lib.STEP_IO_FIELDS:
        setattr(io, f, 1 << 20)
    # the e4m3 operands are checked before anything is launched
    assert lib.fkv_step_fp8(ctypes.byref(p), ctypes.byref(io), ctypes.byref(c), fake, None) == _lib.FKV_ERR_INVALID_ARG
    assert lib.fkv_step_fp8(ctypes.byref(p), ctypes.byref(io), None, fake, None) == _lib.FKV_ERR_INVALID_ARG
    small_t = _fp8_params(T=64, comp_rows=4 * 64)
    assert lib.fkv_step_fp8(ctypes.byref(small_t), ctypes.byref(io), ctypes.byref(c), fake, None) == _lib.FKV_ERR_UNSUPPORTED
