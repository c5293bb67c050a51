"""The C-ABI library loads, exports every entry point include/xlpk.h declares, and
rejects bad arguments on the host before touching a GPU.  CPU only."""
import ctypes as C
import os
import re

import pytest

from persistent_decode_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "xlpk.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(xlpk_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from persistent_decode_b200.build import build
    build()
    return _abi.load()


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert "xlpk_create" in names and "xlpk_decode" in names and "xlpk_decode_unfused" in names
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) <= set(_abi.SIGNATURES), set(names) - set(_abi.SIGNATURES)


def test_status_strings(lib):
    assert lib.xlpk_status_string(0) == b"XLPK_OK"
    assert lib.xlpk_status_string(-5) == b"XLPK_ERR_KV_FULL"
    assert lib.xlpk_status_string(-6) == b"XLPK_ERR_TIMEOUT"
    assert lib.xlpk_status_string(123) == b"XLPK_ERR_UNKNOWN"


def _tiny_cfg(**kw):
    c = _abi.xlpk_config(n_layers=2, hidden=256, n_q_heads=4, n_kv_heads=2, head_dim=64, ffn=1024,
                         vocab=4096, batch=1, max_seq=160, rope_theta=1e4, rms_eps=1e-5)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def test_host_side_argument_checks(lib):
    h = C.c_void_p()
    w = _abi.xlpk_weights()
    kv = _abi.xlpk_kv()
    assert lib.xlpk_create(None, C.byref(w), C.byref(kv), C.byref(h)) == _abi.XLPK_ERR_INVALID_ARG
    # bad shapes are rejected before any CUDA call
    for bad in (dict(n_layers=0), dict(n_q_heads=3), dict(batch=0), dict(max_seq=0), dict(vocab=1),
                dict(weight_dtype=7), dict(rope_theta=0.0), dict(kv_dtype=2),
                # e4m3 cache: scales must be powers of two in [2^-24, 2^24]
                dict(kv_dtype=1, k_scale=0.3, v_scale=0.25), dict(kv_dtype=1, k_scale=0.0, v_scale=1.0),
                dict(kv_dtype=1, k_scale=1.0, v_scale=2.0 ** -30), dict(kv_dtype=1, k_scale=-0.5, v_scale=0.5),
                dict(kv_dtype=1, k_scale=float("inf"), v_scale=0.5)):
        c = _tiny_cfg(**bad)
        assert lib.xlpk_create(C.byref(c), C.byref(w), C.byref(kv), C.byref(h)) == _abi.XLPK_ERR_INVALID_ARG, bad
    # FP8: K dims must be multiples of 256 (a row pair of 2K + K/16 bytes stays 16-byte aligned)
    for unsup in (dict(head_dim=96), dict(batch=3), dict(n_q_heads=16, n_kv_heads=2),
                  dict(weight_dtype=1, hidden=384)):
        c = _tiny_cfg(**unsup)
        assert lib.xlpk_create(C.byref(c), C.byref(w), C.byref(kv), C.byref(h)) == _abi.XLPK_ERR_UNSUPPORTED, unsup
    # a valid shape with missing weight pointers
    c = _tiny_cfg()
    assert lib.xlpk_create(C.byref(c), C.byref(w), C.byref(kv), C.byref(h)) == _abi.XLPK_ERR_INVALID_ARG
    # calls on a NULL handle
    assert lib.xlpk_decode(None, 1, None, None, None) == _abi.XLPK_ERR_INVALID_ARG
    assert lib.xlpk_decode_unfused(None, 1, None, None, None) == _abi.XLPK_ERR_INVALID_ARG
    assert lib.xlpk_get_status(None) == _abi.XLPK_ERR_INVALID_ARG
    assert lib.xlpk_destroy(None) == _abi.XLPK_ERR_INVALID_ARG
    info = _abi.xlpk_info()
    assert lib.xlpk_get_info(None, C.byref(info)) == _abi.XLPK_ERR_INVALID_ARG
    # the tensor-core tile: shapes and pointers are checked before any CUDA call
    p = C.c_void_p(1 << 20)
    for n, k in ((127, 64), (128, 0), (128, 96), (128, 8192)):
        assert lib.xlpk_tc_gemm_tile(p, n, k, p, p, None) == _abi.XLPK_ERR_INVALID_ARG, (n, k)
    assert lib.xlpk_tc_gemm_tile(None, 128, 64, p, p, None) == _abi.XLPK_ERR_INVALID_ARG
    assert lib.xlpk_tc_gemm_tile(C.c_void_p((1 << 20) + 8), 128, 64, p, p, None) == _abi.XLPK_ERR_INVALID_ARG


def test_struct_layout_matches_header(tmp_path):
    # every field of every struct at the offset a C compiler gives it from
    # include/xlpk.h (gcc on this host), against the ctypes mirror
    import subprocess
    structs = [_abi.xlpk_config, _abi.xlpk_linear, _abi.xlpk_layer_weights, _abi.xlpk_weights, _abi.xlpk_kv,
               _abi.xlpk_decode_io, _abi.xlpk_info]
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "xlpk.h"', 'int main(void) {']
    for st in structs:
        n = st.__name__
        lines.append(f'  printf("{n} size %zu\\n", sizeof({n}));')
        for f, _ in st._fields_:
            lines.append(f'  printf("{n} {f} %zu\\n", offsetof({n}, {f}));')
    lines += ['  return 0;', '}']
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
    got = {}
    for line in out:
        if line:
            parts = line.split()
            got[(parts[0], parts[1])] = int(parts[2])
    for st in structs:
        n = st.__name__
        assert got[(n, "size")] == C.sizeof(st), n
        for f, _ in st._fields_:
            assert got[(n, f)] == getattr(st, f).offset, (n, f)

def test_debug_logits_rejects_a_null_handle(lib):
    assert lib.xlpk_debug_logits(None, None, None) == _abi.XLPK_ERR_INVALID_ARG
